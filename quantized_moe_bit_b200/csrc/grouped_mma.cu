// Dequant-fused grouped GEMM of the routed experts for buckets of a few rows
// (prefill chunks, batched decode), on mma.sync fed from registers.
//
// At these bucket sizes (most experts of a 128-row chunk get 3..32 rows) the
// contraction is far from dense: the weights are read once and each weight
// serves a handful of rows, so the kernel is built like the batch-1 decode
// kernel rather than like a tiled GEMM.  A persistent CTA per SM walks the
// items (active expert, 64 weight rows); each item's weights and scale rows
// are bulk-copied into one of two shared-memory slots while the other slot is
// computed.  mma.sync m16n8k16 takes 16 weight rows as A (fp16 1024 + q from
// one LOP3 per pair, as in the decode kernel) and 8 bucket rows as the 8
// columns of B (the paired activation of each row: (v0,v4), (v1/16,v5/16),
// ...); per group of 64 inputs the fp32 epilogue adds S (dot - 1024 sum v') +
// B sum v for each (weight row, bucket row).  The 12 warps split an item as 4
// row tiles x 3 group parts; partial sums meet in shared memory and are added
// in a fixed order (results do not depend on timing).
//   mode 0: gate/up rows of 32 intermediate indices (a tile: 8 gate rows on
//           top of the 8 up rows of the same indices) -> act = gelu(g) * u
//   mode 1: 64 down rows -> y rows of the bucket's pairs
// Every wait is bounded; a wait that runs out sets the device check word.

namespace moe {

constexpr int GM_THREADS = 384;
constexpr int GM_WARPS = 12;
constexpr int GM_ROWS = 64;            // weight rows per item (4 tiles of 16)
constexpr int GM_GPARTS = 3;           // group parts per row tile (4 x 3 = 12 warps)
constexpr int GM_NMAX = 32;            // bucket rows handled here (4 n-tiles of 8)
constexpr int GM_CHUNK = 4;            // groups whose activation fragments are loaded together
constexpr int GM_SMEM_LIMIT = 232448;

struct GmItem {
  int e, pos0, cnt, tile;
};

struct GmArgs {
  int mode;                            // 0 gate/up + GeGLU, 1 down
  const uint4* P;                      // paired activation rows [rows][K/8]: mode 0 x (token rows), mode 1 act (bucket order)
  const float2* S;                     // their group sums [rows][K/64]: (1024 * sum of paired halves, sum of values)
  int T, H, I, E, k;
  const void* const* blob_ptrs;        // device [E] blob pointers (matrices at off[]), or null: mq/ms/mb
  const uint8_t* mq[3];
  const uint16_t* ms[3];
  const uint16_t* mb[3];
  size_t off[9];
  const int32_t* offsets;
  const int32_t* pairs;
  const int32_t* active;
  const int32_t* n_active;
  int lo, hi;                          // buckets with lo < rows <= hi
  __half* act_out;                     // mode 0: [T*k, I] fp16, bucket order
  float* y_out;                        // mode 1: [T*k, H] fp32, rows = pair ids
  unsigned* queue;                     // work counter (zero before the launch)
};

// Geometry of an item slot (same on host and device).
struct GmGeom {
  int K, NG, rowbytes, rstride, nrows, nwin, winrows, sb, tiles_per_expert;
  uint32_t win0, slot;                 // window area offset, slot bytes
  DF_HD void init(int mode, int H, int I) {
    K = mode == 0 ? H : I;
    NG = K / 64;
    rowbytes = K / 2;
    // rows a whole number of 64-byte lines apart would put the 8 rows of an
    // mma tile on the same banks: pad them by 16 bytes (one copy per row)
    rstride = (rowbytes % 64 == 0) ? rowbytes + 16 : rowbytes;
    nrows = GM_ROWS;
    nwin = mode == 0 ? 4 : 2;          // gate.s gate.b up.s up.b | down.s down.b
    winrows = mode == 0 ? GM_ROWS / 2 : GM_ROWS;
    sb = NG * 2;
    tiles_per_expert = mode == 0 ? I / (GM_ROWS / 2) : H / GM_ROWS;
    win0 = df_a16(static_cast<uint64_t>(nrows) * rstride);
    slot = (win0 + static_cast<uint32_t>(nwin) * df_a16(static_cast<uint64_t>(winrows) * sb) + 127u) & ~127u;
  }
  DF_HD uint32_t win(int w) const { return win0 + static_cast<uint32_t>(w) * df_a16(static_cast<uint64_t>(winrows) * sb); }
  DF_HD bool padded() const { return rstride != rowbytes; }
  DF_HD int copies() const { return (padded() ? nrows : (nwin == 4 ? 2 : 1)) + nwin; }
};

inline size_t grouped_mma_smem(int H, int I) {
  GmGeom a, b;
  a.init(0, H, I);
  b.init(1, H, I);
  const uint32_t slot = a.slot > b.slot ? a.slot : b.slot;
  return 2u * slot + static_cast<size_t>(GM_WARPS) * 16 * 8 * 4 + 2 * 8 + 2 * sizeof(GmItem) +
         (2 * GM_NMAX + 1) * 4 + 128;
}
// Shapes the kernel serves.
inline bool grouped_mma_ok(int H, int I) {
  if (H % 64 || I % 64 || I % (GM_ROWS / 2) || H % GM_ROWS) return false;
  return grouped_mma_smem(H, I) <= GM_SMEM_LIMIT;
}

#ifdef __CUDACC__
// Paired activation rows for the mma B operand: word u of row r (8 values)
// -> P[r][u], and per 64-value group (1024 * sum of the stored halves, sum of
// the values) -> S[r][u/8].  src is bf16 (src_bf16) or fp16, [rows, K].
__global__ void k_pair_rows(const uint16_t* __restrict__ src, int src_bf16, int rows, int K, uint4* __restrict__ P,
                            float2* __restrict__ S) {
  const long nw = static_cast<long>(rows) * (K / 8);           // K/8 is a multiple of 8: groups never straddle warps
  for (long base = static_cast<long>(blockIdx.x) * blockDim.x; base < nw; base += static_cast<long>(gridDim.x) * blockDim.x) {
    const long u = base + threadIdx.x;
    float off = 0.f, sum = 0.f;
    uint4 p = make_uint4(0u, 0u, 0u, 0u);
    if (u < nw) {
      const uint4 raw = *reinterpret_cast<const uint4*>(src + 8 * u);
      const uint32_t rw[4] = {raw.x, raw.y, raw.z, raw.w};
      float v[8];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        if (src_bf16) {
          v[2 * t] = __uint_as_float(rw[t] << 16);
          v[2 * t + 1] = __uint_as_float(rw[t] & 0xFFFF0000u);
        } else {
          const float2 f = unpack_half2(rw[t]);
          v[2 * t] = f.x;
          v[2 * t + 1] = f.y;
        }
      }
      p = df_pair8(v, off, sum);
    }
    off = oct_sum(off);
    sum = oct_sum(sum);
    if (u < nw) {
      P[u] = p;
      if ((threadIdx.x & 7) == 0) S[u / 8] = make_float2(1024.f * off, sum);
    }
  }
}

__global__ void __launch_bounds__(GM_THREADS, 1) k_group_mma(const __grid_constant__ GmArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  GmGeom g;
  g.init(a.mode, a.H, a.I);
  GmGeom g0, g1;
  g0.init(0, a.H, a.I);
  g1.init(1, a.H, a.I);
  const uint32_t slot_bytes = g0.slot > g1.slot ? g0.slot : g1.slot;
  float* part = reinterpret_cast<float*>(smem + 2 * slot_bytes);             // [12 warps][16 rows][8 cols]
  uint64_t* bars = reinterpret_cast<uint64_t*>(part + GM_WARPS * 16 * 8);    // [2]
  GmItem* items = reinterpret_cast<GmItem*>(bars + 2);                      // [2]: the item in each slot
  int* rowtab = reinterpret_cast<int*>(items + 2);                            // [2][GM_NMAX]
  int* n_mine = rowtab + 2 * GM_NMAX;
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = smem_addr(bars);
  const uint16_t* S16 = reinterpret_cast<const uint16_t*>(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
  const int rt = warp / GM_GPARTS, gp = warp % GM_GPARTS;
  const int gs0 = gp * g.NG / GM_GPARTS, gs1 = (gp + 1) * g.NG / GM_GPARTS;

  if (threadIdx.x == 0) {
    df_mbar_init(bar0, 1);
    df_mbar_init(bar0 + 8, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  const int n_cand = *a.n_active * g.tiles_per_expert;
  // warp 0: claim the next (active expert, tile) whose bucket is ours from the
  // shared work counter; -1 when the list is exhausted
  auto claim = [&](GmItem& it) -> bool {
    for (;;) {
      unsigned j = 0;
      if (lane == 0) j = atomicAdd(a.queue, 1u);
      j = __shfl_sync(0xffffffffu, j, 0);
      if (static_cast<int>(j) >= n_cand) return false;
      const int ai = static_cast<int>(j) / g.tiles_per_expert;
      it.tile = static_cast<int>(j) - ai * g.tiles_per_expert;
      it.e = a.active[ai];
      if (it.e < 0 || it.e >= a.E) { if (lane == 0) flag_check(CHECK_EXPERT_ID); continue; }
      it.pos0 = a.offsets[it.e];
      it.cnt = a.offsets[it.e + 1] - it.pos0;
      if (it.cnt > a.lo && it.cnt <= a.hi) return true;
    }
  };
  __syncthreads();

  // warp 0: copies of item q into slot s (completing on bars[s]) and its
  // bucket rows into rowtab[s]
  auto issue = [&](const GmItem& it, int s) {
    for (int n = lane; n < it.cnt; n += 32) {
      const int pr = a.pairs[it.pos0 + n];
      int v;
      if (a.mode == 0) {
        v = pr / a.k;
        if (pr < 0 || v >= a.T) { flag_check(CHECK_PAIR_ID); v = -1; }
      } else {
        v = pr;
        if (pr < 0 || pr >= a.T * a.k) { flag_check(CHECK_PAIR_ID); v = -1; }
      }
      rowtab[s * GM_NMAX + n] = v;
    }
    const uint8_t* blob = a.blob_ptrs ? static_cast<const uint8_t*>(a.blob_ptrs[it.e]) : nullptr;
    auto mq = [&](int m) { return blob ? blob + a.off[3 * m] : a.mq[m]; };
    auto msb = [&](int m, int sb_) {
      return blob ? blob + a.off[3 * m + 1 + sb_]
                  : reinterpret_cast<const uint8_t*>(sb_ ? a.mb[m] : a.ms[m]);
    };
    const uint32_t bar = bar0 + 8u * s, dst = sbase + static_cast<uint32_t>(s) * slot_bytes;
    const int nc = g.copies(), tile = it.tile;
    const int nrowcopies = nc - g.nwin;
    for (int c = lane; c < nc; c += 32) {
      const uint8_t* src;
      uint32_t d, bytes;
      if (c < nrowcopies) {
        if (g.padded()) {                  // one row
          const int r = c;
          int m, row;
          if (a.mode == 0) { m = r < GM_ROWS / 2 ? 0 : 1; row = tile * (GM_ROWS / 2) + (r % (GM_ROWS / 2)); }
          else { m = 2; row = tile * GM_ROWS + r; }
          src = mq(m) + static_cast<size_t>(row) * g.rowbytes;
          d = static_cast<uint32_t>(r) * g.rstride;
          bytes = g.rowbytes;
        } else {                           // a block of contiguous rows
          int m, row, n;
          if (a.mode == 0) { m = c; row = tile * (GM_ROWS / 2); n = GM_ROWS / 2; }
          else { m = 2; row = tile * GM_ROWS; n = GM_ROWS; }
          src = mq(m) + static_cast<size_t>(row) * g.rowbytes;
          d = static_cast<uint32_t>(a.mode == 0 ? c * (GM_ROWS / 2) : 0) * g.rstride;
          bytes = static_cast<uint32_t>(n) * g.rowbytes;
        }
      } else {                             // scale / bias window (rows start on 16 bytes: no skew)
        const int w = c - nrowcopies;
        int m, sbi, row;
        if (a.mode == 0) { m = w / 2; sbi = w % 2; row = tile * (GM_ROWS / 2); }
        else { m = 2; sbi = w; row = tile * GM_ROWS; }
        src = msb(m, sbi) + static_cast<size_t>(row) * g.sb;
        d = g.win(w);
        bytes = static_cast<uint32_t>(g.winrows) * g.sb;
      }
      df_bulk_tx(bar, dst + d, src, bytes);
    }
    __syncwarp();
    if (lane == 0) df_mbar_arrive(bar);
    __syncwarp();
  };

  // items[s]: the item in slot s (written by warp 0 before its copies are issued)
  if (warp == 0) {
    GmItem it{};
    const bool ok = claim(it);
    if (lane == 0) { items[0] = it; *n_mine = ok ? 1 : 0; }
    __syncwarp();
    if (ok) issue(it, 0);
  }
  __syncthreads();
  unsigned uses0 = 0u, uses1 = 0u;
  for (int q = 0; *n_mine > q; ++q) {
    const int s = q & 1;
    const GmItem it = items[s];
    if (warp == 0) {                     // the next item into the other slot
      GmItem nx{};
      const bool ok = claim(nx);
      if (lane == 0) { items[s ^ 1] = nx; if (ok) *n_mine = q + 2; }
      __syncwarp();
      if (ok) issue(nx, s ^ 1);
    }
    const int pos0 = it.pos0, cnt = it.cnt, tile = it.tile;
    df_mbar_wait(bar0 + 8u * s, (s ? uses1 : uses0) & 1u);
    if (s) ++uses1; else ++uses0;
    const int* rows = rowtab + s * GM_NMAX;
    const unsigned char* base = smem + static_cast<size_t>(s) * slot_bytes;
    const uint32_t sbase_off = static_cast<uint32_t>(s) * slot_bytes;
    // this lane's two weight rows of tile rt and their scale rows
    int ra, rb, wa_s, wa_b, wb_s, wb_b, wra, wrb;
    if (a.mode == 0) {
      ra = 8 * rt + gq; rb = GM_ROWS / 2 + 8 * rt + gq;
      wa_s = 0; wa_b = 1; wb_s = 2; wb_b = 3; wra = 8 * rt + gq; wrb = 8 * rt + gq;
    } else {
      ra = 16 * rt + gq; rb = 16 * rt + 8 + gq;
      wa_s = 0; wa_b = 1; wb_s = 0; wb_b = 1; wra = ra; wrb = rb;
    }
    const uint8_t* qa = base + static_cast<size_t>(ra) * g.rstride + 8 * tq;
    const uint8_t* qb = base + static_cast<size_t>(rb) * g.rstride + 8 * tq;
    const uint16_t* sa = S16 + (sbase_off + g.win(wa_s) + static_cast<uint32_t>(wra) * g.sb) / 2;
    const uint16_t* ba = S16 + (sbase_off + g.win(wa_b) + static_cast<uint32_t>(wra) * g.sb) / 2;
    const uint16_t* sbp = S16 + (sbase_off + g.win(wb_s) + static_cast<uint32_t>(wrb) * g.sb) / 2;
    const uint16_t* bbp = S16 + (sbase_off + g.win(wb_b) + static_cast<uint32_t>(wrb) * g.sb) / 2;
    const int ntiles = (cnt + 7) / 8;
    for (int nt = 0; nt < ntiles; ++nt) {
      // B column gq: bucket row 8 nt + gq; accumulator columns 2tq, 2tq + 1
      auto act_row = [&](int n) -> int {          // activation row of bucket row n, or -1
        if (n >= cnt) return -1;
        return a.mode == 0 ? rows[n] : pos0 + n;
      };
      const int rB = act_row(8 * nt + gq), rC0 = act_row(8 * nt + 2 * tq), rC1 = act_row(8 * nt + 2 * tq + 1);
      // activation fragments of one chunk of groups, loaded a chunk ahead
      auto load_chunk = [&](int c0, uint4 (&fb)[GM_CHUNK][2], float2 (&s0)[GM_CHUNK], float2 (&s1)[GM_CHUNK]) {
#pragma unroll
        for (int j = 0; j < GM_CHUNK; ++j) {
          const int gr = c0 + j;
          fb[j][0] = fb[j][1] = make_uint4(0u, 0u, 0u, 0u);
          s0[j] = s1[j] = make_float2(0.f, 0.f);
          if (gr < gs1) {
            if (rB >= 0) {
              const uint4* pr = a.P + static_cast<size_t>(rB) * (g.K / 8) + 8 * gr + 2 * tq;
              fb[j][0] = __ldcg(pr);
              fb[j][1] = __ldcg(pr + 1);
            }
            if (rC0 >= 0) s0[j] = __ldcg(a.S + static_cast<size_t>(rC0) * g.NG + gr);
            if (rC1 >= 0) s1[j] = __ldcg(a.S + static_cast<size_t>(rC1) * g.NG + gr);
          }
        }
      };
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      uint4 fbA[GM_CHUNK][2], fbB[GM_CHUNK][2];
      float2 s0A[GM_CHUNK], s1A[GM_CHUNK], s0B[GM_CHUNK], s1B[GM_CHUNK];
      load_chunk(gs0, fbA, s0A, s1A);
      for (int c0 = gs0; c0 < gs1; c0 += GM_CHUNK) {
        if (c0 + GM_CHUNK < gs1) load_chunk(c0 + GM_CHUNK, fbB, s0B, s1B);
#pragma unroll
        for (int j = 0; j < GM_CHUNK; ++j) {
          const int gr = c0 + j;
          if (gr < gs1) {
            const uint2 wa = *reinterpret_cast<const uint2*>(qa + 32 * gr);
            const uint2 wb = *reinterpret_cast<const uint2*>(qb + 32 * gr);
            float d[4];
            mma_group(d, wa, wb, fbA[j][0], fbA[j][1]);
            const float Sa = bf16_to_f32(sa[gr]), Ba = bf16_to_f32(ba[gr]);
            const float Sb = bf16_to_f32(sbp[gr]), Bb = bf16_to_f32(bbp[gr]);
            acc[0] += Sa * (d[0] - s0A[j].x) + Ba * s0A[j].y;
            acc[1] += Sa * (d[1] - s1A[j].x) + Ba * s1A[j].y;
            acc[2] += Sb * (d[2] - s0A[j].x) + Bb * s0A[j].y;
            acc[3] += Sb * (d[3] - s1A[j].x) + Bb * s1A[j].y;
          }
        }
#pragma unroll
        for (int j = 0; j < GM_CHUNK; ++j) {
          fbA[j][0] = fbB[j][0]; fbA[j][1] = fbB[j][1]; s0A[j] = s0B[j]; s1A[j] = s1B[j];
        }
      }
      float* pw = part + warp * 128;
      pw[gq * 8 + 2 * tq] = acc[0];
      pw[gq * 8 + 2 * tq + 1] = acc[1];
      pw[(gq + 8) * 8 + 2 * tq] = acc[2];
      pw[(gq + 8) * 8 + 2 * tq + 1] = acc[3];
      __syncthreads();
      if (a.mode == 0) {
        // thread: tile r4, intermediate m (0..7), column n
        for (int qq = threadIdx.x; qq < 4 * 8 * 8; qq += GM_THREADS) {
          const int r4 = qq >> 6, m = (qq >> 3) & 7, n = qq & 7;
          if (8 * nt + n >= cnt) continue;
          float gs = 0.f, us = 0.f;
#pragma unroll
          for (int p = 0; p < GM_GPARTS; ++p) {
            gs += part[(r4 * GM_GPARTS + p) * 128 + m * 8 + n];
            us += part[(r4 * GM_GPARTS + p) * 128 + (m + 8) * 8 + n];
          }
          const int i = tile * (GM_ROWS / 2) + 8 * r4 + m;
          a.act_out[static_cast<size_t>(pos0 + 8 * nt + n) * a.I + i] = __float2half_rn(gelu_tanh(gs) * us);
        }
      } else {
        for (int qq = threadIdx.x; qq < 4 * 16 * 8; qq += GM_THREADS) {
          const int r4 = qq >> 7, m = (qq >> 3) & 15, n = qq & 7;
          if (8 * nt + n >= cnt) continue;
          float ys = 0.f;
#pragma unroll
          for (int p = 0; p < GM_GPARTS; ++p) ys += part[(r4 * GM_GPARTS + p) * 128 + m * 8 + n];
          const int dst = rows[8 * nt + n];
          if (dst >= 0) a.y_out[static_cast<size_t>(dst) * a.H + tile * GM_ROWS + 16 * r4 + m] = ys;
        }
      }
      __syncthreads();                   // partial sums read out
    }
    __syncthreads();                     // slot s and its rows read out before they are refilled; n_mine settled
  }
}
#endif  // __CUDACC__

}  // namespace moe
