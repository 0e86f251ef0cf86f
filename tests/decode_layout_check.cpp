// Host check of the batch-1 decode kernel's static geometry: for every CTA of
// a grid, every bulk copy is 16-byte aligned, inside its source array and its
// shared-memory area; copies that are in flight together do not overlap; and
// every weight row and scale row the kernel reads sits where the copy put the
// matching source bytes.  Prints "ok" or the first failure.
//
//   decode_layout_check H I Is E k G
#include <cuda_fp16.h>

#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "../quantized_moe_bit_b200/csrc/decode_fused.cu"

using namespace moe;

static int fails = 0;
#define REQUIRE(cond, ...)                                  \
  do {                                                      \
    if (!(cond)) {                                          \
      if (fails++ < 10) {                                   \
        std::printf("FAIL %s:%d: ", __FILE__, __LINE__);    \
        std::printf(__VA_ARGS__);                           \
        std::printf("\n");                                  \
      }                                                     \
    }                                                       \
  } while (0)

struct Range { uint64_t a, b; const char* what; };

static void no_overlap(const std::vector<Range>& rs, int c, const char* set) {
  for (size_t i = 0; i < rs.size(); ++i)
    for (size_t j = i + 1; j < rs.size(); ++j)
      REQUIRE(rs[i].b <= rs[j].a || rs[j].b <= rs[i].a, "cta %d %s: %s [%llu,%llu) overlaps %s [%llu,%llu)", c, set,
              rs[i].what, (unsigned long long)rs[i].a, (unsigned long long)rs[i].b, rs[j].what,
              (unsigned long long)rs[j].a, (unsigned long long)rs[j].b);
}

int main(int argc, char** argv) {
  if (argc != 7) {
    std::printf("usage: %s H I Is E k G\n", argv[0]);
    return 2;
  }
  const int H = std::atoi(argv[1]), I = std::atoi(argv[2]), Is = std::atoi(argv[3]), E = std::atoi(argv[4]),
            k = std::atoi(argv[5]), G = std::atoi(argv[6]);
  if (!df_fits(H, I, Is, E, k, G)) {
    std::printf("does not fit\n");
    return 3;
  }
  // blob offsets (gate, up, down: q, s, b)
  size_t off[9];
  {
    const size_t q = static_cast<size_t>(I) * H / 2, s = static_cast<size_t>(I) * (H / 64) * 2;
    size_t o = 0;
    for (int m = 0; m < 3; ++m) {
      off[3 * m] = o; o += q;
      off[3 * m + 1] = o; o += s;
      off[3 * m + 2] = o; o += s;
    }
  }
  const uint64_t blob = off[8] + static_cast<uint64_t>(H) * (I / 64) * 2;
  // byte sizes of every copy source
  auto src_size = [&](int src) -> uint64_t {
    if (src < 8) return blob;
    if (src < DF_SRC_ROUTER) {
      const int m = (src - DF_SRC_SHARED) / 3, arr = (src - DF_SRC_SHARED) % 3;
      const uint64_t rows = m < 2 ? Is : H, K = m < 2 ? H : Is;
      return arr == 0 ? rows * K / 2 : rows * (K / 64) * 2;
    }
    const int arr = src - DF_SRC_ROUTER;
    return arr == 0 ? static_cast<uint64_t>(E) * H : static_cast<uint64_t>(E) * (H / 64) * 2;
  };
  DfGeom g0;
  g0.init(H, I, Is, E, k, G, 0);
  REQUIRE(g0.total <= static_cast<uint32_t>(DF_SMEM_LIMIT), "total %u", g0.total);
  REQUIRE(g0.f_xsum() + (H / 64) * 8 <= g0.M && g0.f_ssum() + (Is / 64) * 8 <= g0.M, "fragment area");
  REQUIRE(g0.m_bars() + DF_NBARS * 8 <= g0.total && g0.m_bars() % 8 == 0, "misc area");
  long pairs = 0, spairs = 0, rows = 0;

  for (int c = 0; c < G; ++c) {
    DfGeom g;
    g.init(H, I, Is, E, k, G, c);
    REQUIRE(g.U == g0.U && g.D == g0.D && g.RR == g0.RR && g.F == g0.F && g.M == g0.M && g.total == g0.total,
            "cta %d layout differs", c);
    pairs += g.np; spairs += g.nsp; rows += g.nrow;
    REQUIRE(g.np <= DF_MAX_RG_PAIRS && g.nsp <= DF_MAX_SG_PAIRS && g.nrow <= DF_MAX_ROWS, "cta %d counts", c);
    REQUIRE(g.ntR <= DF_BAR_D, "cta %d tiles", c);
    REQUIRE(g.n0 + g.n1 == g.np && g.n1 <= I, "cta %d runs", c);
    // every copy: alignment, inside its source, inside its area
    auto check_copy = [&](const DfCopy& C, uint32_t lo, uint32_t hi, const char* name) {
      REQUIRE(C.bytes > 0 && C.bytes % 16 == 0 && C.dst % 16 == 0 && C.src_off % 16 == 0,
              "cta %d %s: alignment dst %u bytes %u src %llu", c, name, C.dst, C.bytes,
              (unsigned long long)C.src_off);
      REQUIRE(C.src_off + C.bytes <= src_size(C.src), "cta %d %s: source overrun (src %d)", c, name, C.src);
      REQUIRE(C.dst >= lo && C.dst + C.bytes <= hi, "cta %d %s: [%u,+%u) outside [%u,%u)", c, name, C.dst, C.bytes,
              lo, hi);
      REQUIRE(C.bar >= 0 && C.bar < DF_NBARS, "cta %d %s: barrier", c, name);
    };
    std::vector<Range> rg, d, sd, sg, rr;
    for (int e = 0; e < df_rg_count(g); ++e) {
      const DfCopy C = df_rg_copy(g, off, e);
      check_copy(C, g.U, g.D, "rg");
      REQUIRE(C.src >= 0 && C.src < 8 && C.src < k, "cta %d rg slot %d", c, C.src);
      REQUIRE(C.bar < g.ntR, "cta %d rg barrier %d", c, C.bar);
      rg.push_back({C.dst, C.dst + C.bytes, "rg"});
    }
    for (int e = 0; e < df_d_count(g); ++e) {
      const DfCopy C = df_d_copy(g, off, e);
      check_copy(C, g.D, g.RR, "d");
      REQUIRE(C.src < k && C.bar == DF_BAR_D, "cta %d d", c);
      d.push_back({C.dst, C.dst + C.bytes, "d"});
    }
    for (int e = 0; e < df_sd_count(g); ++e) {
      const DfCopy C = df_sd_copy(g, e);
      check_copy(C, g.U, g.D, "sd");
      REQUIRE(C.bar == DF_BAR_SD, "cta %d sd", c);
      sd.push_back({C.dst, C.dst + C.bytes, "sd"});
    }
    for (int e = 0; e < df_sg_count(g); ++e) {
      const DfCopy C = df_sg_copy(g, e);
      check_copy(C, g.U, g.D, "sg");
      REQUIRE(C.bar == DF_BAR_SG, "cta %d sg", c);
      sg.push_back({C.dst, C.dst + C.bytes, "sg"});
    }
    for (int e = 0; e < df_rr_count(g); ++e) {
      const DfCopy C = df_rr_copy(g, e);
      check_copy(C, g.RR, g.F, "rr");
      REQUIRE(C.bar == DF_BAR_RR, "cta %d rr", c);
      rr.push_back({C.dst, C.dst + C.bytes, "rr"});
    }
    // copies live together: phase B (routed rows, down rows, the next router
    // row); from the end of phase B (shared down, the next layer's shared
    // gate/up, down rows, the next router row)
    std::vector<Range> s1 = rg, s2 = sd;
    s1.insert(s1.end(), d.begin(), d.end()); s1.insert(s1.end(), rr.begin(), rr.end());
    s2.insert(s2.end(), sg.begin(), sg.end()); s2.insert(s2.end(), d.begin(), d.end());
    s2.insert(s2.end(), rr.begin(), rr.end());
    no_overlap(s1, c, "phase B");
    no_overlap(s2, c, "phase C");

    // reads: the smem byte the kernel reads must hold the source byte it wants
    auto lands = [&](const std::vector<DfCopy>& cs, uint32_t smem, uint32_t n, int src, uint64_t want,
                     const char* what) {
      bool ok = false;
      for (const DfCopy& C : cs) {
        if (C.src != src || smem < C.dst || smem + n > C.dst + C.bytes) continue;
        ok = (smem - C.dst) == (want - C.src_off);
        if (ok) break;
      }
      REQUIRE(ok, "cta %d %s: smem %u (+%u) does not hold source %d byte %llu", c, what, smem, n, src,
              (unsigned long long)want);
    };
    std::vector<DfCopy> crg, cd, csd, csg, crr;
    for (int e = 0; e < df_rg_count(g); ++e) crg.push_back(df_rg_copy(g, off, e));
    for (int e = 0; e < df_d_count(g); ++e) cd.push_back(df_d_copy(g, off, e));
    for (int e = 0; e < df_sd_count(g); ++e) csd.push_back(df_sd_copy(g, e));
    for (int e = 0; e < df_sg_count(g); ++e) csg.push_back(df_sg_copy(g, e));
    for (int e = 0; e < df_rr_count(g); ++e) crr.push_back(df_rr_copy(g, e));
    const int arr[4] = {1, 2, 4, 5};
    for (int i = 0; i < g.np; ++i) {
      const int p = g.r0 + i, slot = p / I, row = p % I;
      for (int m = 0; m < 2; ++m)
        lands(crg, g.rg_row(i, m), H / 2, slot, off[3 * m] + static_cast<uint64_t>(row) * (H / 2), "rg row");
      for (int a = 0; a < 4; ++a)
        lands(crg, g.rg_scale(off, i, a), g.sbh, slot, off[arr[a]] + static_cast<uint64_t>(row) * g.sbh, "rg scale");
      REQUIRE((g.rg_row(i, 0) + 8) % 8 == 0 && g.rg_scale(off, i, 0) % 2 == 0, "cta %d rg read alignment", c);
    }
    for (int j = 0; j < k; ++j)
      for (int r = 0; r < g.nrow; ++r) {
        const uint64_t row = g.o0 + r;
        lands(cd, g.d_row(j, r), I / 2, j, off[6] + row * (I / 2), "d row");
        for (int a = 0; a < 2; ++a) lands(cd, g.d_scale(off, j, r, a), g.sbi, j, off[7 + a] + row * g.sbi, "d scale");
        REQUIRE(g.d_row(j, r) % 8 == 0, "cta %d d read alignment", c);
      }
    for (int r = 0; r < g.nrow; ++r) {
      const uint64_t row = g.o0 + r;
      lands(csd, g.sd_row(r), Is / 2, DF_SRC_SHARED + 6, row * (Is / 2), "sd row");
      for (int a = 0; a < 2; ++a) lands(csd, g.sd_scale(r, a), g.sbs, DF_SRC_SHARED + 7 + a, row * g.sbs, "sd scale");
    }
    for (int i = 0; i < g.nsp; ++i) {
      const uint64_t row = g.s0 + i;
      for (int m = 0; m < 2; ++m) {
        lands(csg, g.sg_row(i, m), H / 2, DF_SRC_SHARED + 3 * m, row * (H / 2), "sg row");
        for (int a = 0; a < 2; ++a)
          lands(csg, g.sg_scale(i, 2 * m + a), g.sbh, DF_SRC_SHARED + 3 * m + 1 + a, row * g.sbh, "sg scale");
      }
    }
    if (c < E) {
      lands(crr, g.RR, H, DF_SRC_ROUTER, static_cast<uint64_t>(c) * H, "rr row");
      for (int a = 0; a < 2; ++a)
        lands(crr, g.rr_scale(a), g.sbh, DF_SRC_ROUTER + 1 + a, static_cast<uint64_t>(c) * g.sbh, "rr scale");
    }
    // the copy table holds every list; list starts agree with the counts
    {
      int n = 0;
      for (int i = 0; i < 5; ++i) {
        REQUIRE(df_list_start(g, i) == n, "cta %d list start", c);
        for (int e = 0; e < df_list_count(g, i); ++e)
          REQUIRE(df_list_copy(g, off, i, e).src_off < (1ull << 32), "cta %d source offset", c);
        n += df_list_count(g, i);
      }
      REQUIRE(n <= DF_MAX_COPIES, "cta %d: %d copies", c, n);
      // every barrier is fed by one list only, which arrives on it with the
      // byte total (the mbarrier transaction count is below 2^20)
      const int lo[5] = {0, DF_BAR_D, DF_BAR_SD, DF_BAR_SG, DF_BAR_RR};
      const int hi[5] = {g.ntR, DF_BAR_D + 1, DF_BAR_SD + 1, DF_BAR_SG + 1, DF_BAR_RR + 1};
      uint64_t tx[DF_NBARS] = {};
      for (int i = 0; i < 5; ++i)
        for (int e = 0; e < df_list_count(g, i); ++e) {
          const DfCopy C = df_list_copy(g, off, i, e);
          REQUIRE(C.bar >= lo[i] && C.bar < hi[i], "cta %d list %d barrier %d", c, i, C.bar);
          tx[C.bar] += C.bytes;
        }
      for (int b = 0; b < DF_NBARS; ++b) REQUIRE(tx[b] < (1u << 20), "cta %d barrier %d: %llu bytes", c, b,
                                                 (unsigned long long)tx[b]);
      REQUIRE(g.m_tx() % 16 == 0 && g.m_btab() % 16 == 0, "cta %d tx table", c);
      REQUIRE(g.m_ctab() + DF_MAX_COPIES * 16u <= g.m_part() && g.m_ctab() % 16 == 0, "cta %d copy table", c);
    }
    // partial-sum slots
    REQUIRE(g.ntS <= g.sg_tiles_max() && g.ntR <= g.rg_tiles_max() && g.ntD <= g.d_tiles_max() &&
            g.ntSD <= g.sd_tiles_max(), "cta %d tiles beyond the slots", c);
    REQUIRE(g.slot_sg(DF_WARPS - 2, g.sg_tiles_max() - 1) < g.part_slots() &&
            g.slot_rg(DF_WARPS - 1, g.rg_tiles_max() - 1) < g.part_slots() &&
            g.slot_d(g.dp() - 1, g.d_tiles_max() - 1) < g.slot_sd(0, 0) &&
            g.slot_sd(DF_WARPS - 1, g.sd_tiles_max() - 1) < g.part_slots(), "cta %d partial-sum slots", c);
    REQUIRE(g.m_part() + g.part_slots() * 64u <= g.total, "cta %d part area", c);
  }
  REQUIRE(pairs == static_cast<long>(k) * I && spairs == Is && rows == H, "coverage %ld %ld %ld", pairs, spairs, rows);
  if (fails) {
    std::printf("%d failures\n", fails);
    return 1;
  }
  std::printf("ok smem=%u\n", g0.total);
  return 0;
}
