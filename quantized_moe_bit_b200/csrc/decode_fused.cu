// Batch-1 decode of a stack of routed-MoE layers in one persistent kernel.
//
// One cooperative launch runs every layer of the step, one CTA per SM (G
// CTAs of 12 warps).  CTA c owns, in every layer: router row c (c < E), the
// shared-expert gate/up pairs [c*Is/G, ...), the routed gate/up pairs
// [c*k*I/G, ...) of the flattened (slot, row) list, and the output rows
// [c*H/G, ...) with their k routed down rows and their shared down row.
//
// Dot products run on the tensor cores as exact integer mma.sync m16n8k32
// (u8 x s8 -> s32) straight from registers.  A warp takes a tile of 16
// weight rows; per quantisation group (64 inputs) each lane loads two 32-bit
// words of each of its two rows; one mask gives the four low nibbles of a
// word as u8 bytes, a shift and the mask the four high nibbles.  The
// activation of every group is 16-bit fixed point (step = max |v| / 32639,
// split into a high and a low int8 digit), laid out to match, so four mmas
// give the group's exact integer dot d = 256 (q . high) + (q . low) and the
// fp32 epilogue adds S step d + B sum v per row and group.  Gate/up tiles
// give all 8 mma columns the same x (rotated by group so that rows 1,408 B
// apart read distinct banks); down tiles give column j the activation of
// slot j, so one tile mixes rows of all k routed experts.
//
// Per layer:
//   A  rms norm of h (every CTA, same result) -> x and its fragments; router
//      logit c (warp 11) and the shared gate/up pairs from shared memory
//      staged the layer before -> logits, activations (global)
//   grid barrier
//   B  top-k by rank over the logits (every CTA); every routed byte of the
//      CTA -- gate/up rows (padded so fragment loads hit distinct banks), its
//      output rows of the k down matrices, their scale/bias windows -- goes
//      out at once as 1-D bulk copies, one mbarrier per 16-row tile; warps
//      compute each tile as it lands; then the shared down rows are fetched
//      into the freed area
//   grid barrier
//   C  fragments of all routed and shared activations; down tiles; y = sum_j
//      g_j y_j + ysh; h += y; the next layer's shared gate/up rows are fetched
//   grid barrier
// Grid barriers: named barrier, one atomic per CTA on a counter that grows
// by G per barrier, named barrier.  Every wait is bounded (about two
// seconds); a wait that runs out sets the device check word and the thread
// runs on to the end.
//
// The geometry (work split, shared-memory layout, copy lists) is plain C++
// shared by the host, which sizes shared memory from it and checks it.

namespace moe {

constexpr int DF_THREADS = 384;
constexpr int DF_WARPS = DF_THREADS / 32;
constexpr int DF_MAX_LAYERS = 48;
constexpr int DF_MAX_H = 3072;            // one 8-element word of h per thread in the norm
constexpr int DF_MAX_E = 256;
constexpr int DF_MAX_RG_PAIRS = 48;       // routed gate/up pairs per CTA (6 tiles)
constexpr int DF_MAX_SG_PAIRS = 24;       // shared gate/up pairs per CTA (3 tiles)
constexpr int DF_MAX_ROWS = 32;           // output rows per CTA (<= DF_MAX_E: staged in the logit area)
static_assert(DF_MAX_ROWS <= DF_MAX_E, "the combine stages h rows in the logit area");
constexpr int DF_MAX_COPIES = 64;         // entries of a CTA's copy table (all five lists)
constexpr int DF_STRIP = 4;               // quantisation groups a warp holds at once (its strip)
constexpr int DF_MAX_TILES = 18;          // routed + shared down tiles per CTA
constexpr int DF_SMEM_LIMIT = 232448;     // opt-in shared memory per block
constexpr int DF_MAX_ACT = 8 * DF_THREADS * 3;   // k*I + Is fp16 activations (3 words of 8 per thread)
constexpr int DF_ACT_ROUNDS = 3;
// mbarriers: routed gate/up tiles 0..5, then
constexpr int DF_BAR_D = 6, DF_BAR_SD = 7, DF_BAR_SG = 8, DF_BAR_RR = 9, DF_NBARS = 10;
constexpr int DF_TX_BYTES = (DF_NBARS * 4 + 15) & ~15;   // one u32 per barrier, 16-byte rounded
// copy sources besides routed slots 0..7: shared matrix m array a (q, s, b) at
// DF_SRC_SHARED + 3m + a, router arrays (q, s, b) at DF_SRC_ROUTER + a
constexpr int DF_SRC_SHARED = 8, DF_SRC_ROUTER = 17;

struct DfLayer {
  const uint32_t* rq; const uint16_t* rs; const uint16_t* rb;   // router [E, H], 8-bit
  const float* bias;                                            // [E] or null
  const void* const* blobs;                                     // device [E] blob pointers
  const uint32_t* sq[3]; const uint16_t* ss[3]; const uint16_t* sb[3];  // shared gate, up, down
};

struct DfArgs {
  float* h;                         // [H] residual, in place
  int H, I, Is, E, k, L;
  size_t off[9];                    // blob offsets
  __half* act;                      // workspace: k*I + Is fp16
  // router logits, each word tagged with the layer that wrote it ((l + 1)
  // << 32 | fp32 bits; zeroed by the kernel at start-up): the top-k polls
  // them instead of waiting at a grid barrier
  unsigned long long* logits;       // workspace: [E]
  unsigned* counter;                // workspace: grid barrier counter; word 32: abort flag (zeroed before launch)
  uint16_t* x_trace; uint16_t* y_trace; int32_t* idx_trace; float* gates_trace;
  unsigned long long* stamps;       // optional phase timestamps [L][G][16] (ns), or null
  DfLayer layer[DF_MAX_LAYERS];
};

// ------------------------------------------------------------------ geometry
#ifndef __CUDACC__
#define DF_HD
#else
#define DF_HD __host__ __device__
#endif

DF_HD constexpr uint32_t df_a16(uint64_t x) { return static_cast<uint32_t>((x + 15) & ~uint64_t(15)); }
// room for a 16-byte-aligned window over n rows of `per` bytes at any start
DF_HD constexpr uint32_t df_wres(int n, uint32_t per) { return df_a16(static_cast<uint64_t>(n) * per) + 32u; }

struct DfGeom {
  int H, I, Is, E, k, G, c;
  int s0, nsp, r0, np, o0, nrow;    // shared pairs, routed flat pairs, output rows
  int j0, n0, n1;                   // routed runs: first slot, pairs in it, pairs in the next slot
  int ntS, ntR, ntD, ntSD;          // 16-row tiles per phase
  uint32_t rowb;                    // gate/up row bytes (H/2)
  uint32_t sbh, sbi, sbs;           // scale row bytes for K = H, I, Is
  int npmax, nspmax, nrowmax;
  uint32_t U, D, RR, F, M, total;   // areas: union (RG | SD + SG), routed down, router row, fragments, misc
  uint32_t SGB;                     // shared gate/up inside the union area, after the shared down rows
  uint32_t dslot;                   // bytes per routed down slot

  DF_HD void init(int H_, int I_, int Is_, int E_, int k_, int G_, int c_) {
    H = H_; I = I_; Is = Is_; E = E_; k = k_; G = G_; c = c_;
    const long kI = static_cast<long>(k) * I;
    s0 = static_cast<int>(static_cast<long>(c) * Is / G);
    nsp = static_cast<int>(static_cast<long>(c + 1) * Is / G) - s0;
    r0 = static_cast<int>(c * kI / G);
    np = static_cast<int>((c + 1) * kI / G) - r0;
    o0 = static_cast<int>(static_cast<long>(c) * H / G);
    nrow = static_cast<int>(static_cast<long>(c + 1) * H / G) - o0;
    j0 = np > 0 ? r0 / I : 0;
    n0 = np > 0 ? ((j0 + 1) * I - r0 < np ? (j0 + 1) * I - r0 : np) : 0;
    n1 = np - n0;
    ntS = (nsp + 7) / 8;
    ntR = (np + 7) / 8;
    ntD = (k * nrow + 15) / 16;
    ntSD = (nrow + 15) / 16;
    rowb = static_cast<uint32_t>(H / 2);
    sbh = static_cast<uint32_t>(H / 64) * 2;
    sbi = static_cast<uint32_t>(I / 64) * 2;
    sbs = static_cast<uint32_t>(Is / 64) * 2;
    npmax = static_cast<int>((kI + G - 1) / G);
    nspmax = (Is + G - 1) / G;
    nrowmax = (H + G - 1) / G;
    // union area: the largest of the three layouts any CTA can have
    // two runs of n0 + n1 = np pairs: wres(n0) + wres(n1) <= a16(np * sbh) + 80
    const uint32_t rg = 2u * npmax * rowb + 4u * (df_a16(static_cast<uint64_t>(npmax) * sbh) + 80u);
    // shared down at the start, the next layer's shared gate/up after it
    const uint32_t sd = df_a16(static_cast<uint64_t>(nrowmax) * (Is / 2)) + 2u * df_wres(nrowmax, sbs);
    const uint32_t sg = 2u * nspmax * rowb + 4u * df_wres(nspmax, sbh);
    U = 0;
    SGB = (sd + 127u) & ~127u;
    const uint32_t u = rg > SGB + sg ? rg : SGB + sg;
    dslot = df_a16(static_cast<uint64_t>(nrowmax) * (I / 2)) + 2u * df_wres(nrowmax, sbi);
    D = (U + u + 127u) & ~127u;
    RR = D + 8u * dslot;
    const uint32_t rr = static_cast<uint32_t>(H) + 2u * df_wres(1, sbh);
    F = (RR + rr + 127u) & ~127u;
    M = (F + frag_bytes() + 127u) & ~127u;
    total = M + misc_bytes();
  }
  DF_HD uint32_t frag_bytes() const {
    const uint32_t xf = static_cast<uint32_t>(H) * 4 + static_cast<uint32_t>(H / 8) * 16 + static_cast<uint32_t>(H / 64) * 8;
    const uint32_t af = 8u * astride() + static_cast<uint32_t>(Is / 8) * 16 + 8u * (I / 64) * 8 +
                        static_cast<uint32_t>(Is / 64) * 8;
    return xf > af ? xf : af;
  }
  // Work split of the dots.  Gate/up: warp w holds groups [w*NGH/nw, ...)
  // of every tile (nw = 11 in phase A, where warp 11 computes the router
  // logit, and 12 in phase B).  Down: the routed tiles are split dp ways by
  // groups and 12/dp ways by tiles; the shared tiles 12 ways by groups.
  DF_HD int sg_tiles_max() const { return (nspmax + 7) / 8; }
  DF_HD int rg_tiles_max() const { return (npmax + 7) / 8; }
  DF_HD int d_tiles_max() const { return (k * nrowmax + 15) / 16; }
  DF_HD int sd_tiles_max() const { return (nrowmax + 15) / 16; }
  DF_HD int dp() const { return (I / 64 + DF_STRIP - 1) / DF_STRIP; }
  // partial-sum slots (16 floats each) of every phase
  DF_HD int slot_sg(int w, int t) const { return w * sg_tiles_max() + t; }
  DF_HD int slot_rg(int w, int t) const { return w * rg_tiles_max() + t; }
  DF_HD int slot_d(int gp, int t) const { return gp * d_tiles_max() + t; }
  DF_HD int slot_sd(int w, int t) const { return dp() * d_tiles_max() + w * sd_tiles_max() + t; }
  DF_HD int part_slots() const {
    const int a = (DF_WARPS - 1) * sg_tiles_max(), b = DF_WARPS * rg_tiles_max();
    const int c = dp() * d_tiles_max() + DF_WARPS * sd_tiles_max();
    const int m = a > b ? a : b;
    return m > c ? m : c;
  }
  DF_HD uint32_t misc_bytes() const {
    // logits, sel / selv / selg, red, bars, blob table, copy table, pair table, part
    return DF_MAX_E * 4 + 8 * 4 * 3 + 16 * 4 + DF_NBARS * 8 + DF_TX_BYTES + DF_MAX_E * 8 + DF_MAX_COPIES * 16 +
           (DF_MAX_RG_PAIRS + DF_MAX_SG_PAIRS) * 16 + static_cast<uint32_t>(part_slots()) * 64;
  }
  // misc sub-offsets
  DF_HD uint32_t m_lg() const { return M; }
  DF_HD uint32_t m_sel() const { return M + DF_MAX_E * 4; }
  DF_HD uint32_t m_selv() const { return m_sel() + 32; }
  DF_HD uint32_t m_selg() const { return m_sel() + 64; }
  DF_HD uint32_t m_red() const { return m_sel() + 96; }
  DF_HD uint32_t m_bars() const { return m_red() + 64; }
  DF_HD uint32_t m_tx() const { return m_bars() + DF_NBARS * 8; }       // bytes each barrier's copies bring
  DF_HD uint32_t m_btab() const { return m_tx() + DF_TX_BYTES; }         // this layer's E blob pointers
  DF_HD uint32_t m_ctab() const { return m_btab() + DF_MAX_E * 8; }      // the CTA's copy lists
  DF_HD uint32_t m_ptab() const { return m_ctab() + DF_MAX_COPIES * 16; }   // scale rows of every pair
  DF_HD uint32_t m_part() const { return m_ptab() + (DF_MAX_RG_PAIRS + DF_MAX_SG_PAIRS) * 16; }
  // fragment sub-offsets (phases A, B: x; phase C: activations)
  DF_HD uint32_t f_xs() const { return F; }
  DF_HD uint32_t f_xf() const { return F + static_cast<uint32_t>(H) * 4; }
  DF_HD uint32_t f_xsum() const { return f_xf() + static_cast<uint32_t>(H / 8) * 16; }
  DF_HD uint32_t astride() const { return static_cast<uint32_t>(I / 8 + 1) * 16; }   // padded: slots on other banks
  DF_HD uint32_t f_af() const { return F; }
  DF_HD uint32_t f_sf() const { return F + 8u * astride(); }
  DF_HD uint32_t f_asum() const { return f_sf() + static_cast<uint32_t>(Is / 8) * 16; }
  DF_HD uint32_t f_ssum() const { return f_asum() + 8u * (I / 64) * 8; }

  // ---- routed gate/up: pair i (0..np-1), m = 0 gate / 1 up
  // gate rows of the CTA's pairs one after the other, then the up rows
  DF_HD uint32_t rg_row(int i, int m) const { return U + (m * static_cast<uint32_t>(np) + i) * rowb; }
  DF_HD uint32_t rg_win0() const { return U + 2u * np * rowb; }
  // window of run `run` (0: slot j0, 1: slot j0+1), array a (0 gate.s, 1 gate.b, 2 up.s, 3 up.b)
  DF_HD uint32_t rg_win(int run, int a) const {
    return rg_win0() + (run ? 4u * df_wres(n0, sbh) : 0u) + a * df_wres(run ? n1 : n0, sbh);
  }
  DF_HD int rg_row0(int run) const { return run ? 0 : r0 - j0 * I; }   // first expert row of the run
  // byte offset from the (16-byte aligned) blob start of the run's first scale row
  DF_HD uint64_t rg_src(const size_t* off, int run, int a) const {
    const int arr = a < 2 ? 1 + a : 2 + a;   // gate.s, gate.b, up.s, up.b
    return off[arr] + static_cast<uint64_t>(rg_row0(run)) * sbh;
  }
  // shared-memory offset of the scale row (a = 0..3) of pair i
  DF_HD uint32_t rg_scale(const size_t* off, int i, int a) const {
    const int run = i < n0 ? 0 : 1;
    const int rin = run ? i - n0 : i;
    return rg_win(run, a) + static_cast<uint32_t>(rg_src(off, run, a) & 15) + rin * sbh;
  }
  // ---- routed down: slot j, row r (0..nrow-1)
  DF_HD uint32_t d_row(int j, int r) const { return D + j * dslot + r * static_cast<uint32_t>(I / 2); }
  DF_HD uint32_t d_win(int j, int a) const {   // a = 0 down.s, 1 down.b
    return D + j * dslot + df_a16(static_cast<uint64_t>(nrowmax) * (I / 2)) + a * df_wres(nrowmax, sbi);
  }
  DF_HD uint64_t d_src(const size_t* off, int a) const { return off[7 + a] + static_cast<uint64_t>(o0) * sbi; }
  DF_HD uint32_t d_scale(const size_t* off, int j, int r, int a) const {
    return d_win(j, a) + static_cast<uint32_t>(d_src(off, a) & 15) + r * sbi;
  }
  // ---- shared gate/up: pair i (0..nsp-1); windows gate.s, gate.b, up.s, up.b
  DF_HD uint32_t sg_row(int i, int m) const { return SGB + (m * static_cast<uint32_t>(nsp) + i) * rowb; }
  DF_HD uint32_t sg_win(int a) const { return SGB + 2u * nsp * rowb + a * df_wres(nsp, sbh); }
  DF_HD uint64_t sg_src() const { return static_cast<uint64_t>(s0) * sbh; }
  DF_HD uint32_t sg_scale(int i, int a) const { return sg_win(a) + static_cast<uint32_t>(sg_src() & 15) + i * sbh; }
  // ---- shared down: row r
  DF_HD uint32_t sd_row(int r) const { return U + r * static_cast<uint32_t>(Is / 2); }
  DF_HD uint32_t sd_win(int a) const {
    return U + df_a16(static_cast<uint64_t>(nrowmax) * (Is / 2)) + a * df_wres(nrowmax, sbs);
  }
  DF_HD uint64_t sd_src() const { return static_cast<uint64_t>(o0) * sbs; }
  DF_HD uint32_t sd_scale(int r, int a) const { return sd_win(a) + static_cast<uint32_t>(sd_src() & 15) + r * sbs; }
  // ---- router row c
  DF_HD uint32_t rr_win(int a) const { return RR + static_cast<uint32_t>(H) + a * df_wres(1, sbh); }
  DF_HD uint64_t rr_src() const { return static_cast<uint64_t>(c) * sbh; }
  DF_HD uint32_t rr_scale(int a) const { return rr_win(a) + static_cast<uint32_t>(rr_src() & 15); }
};

// One 1-D bulk copy: `bytes` from source `src` (a routed slot, or a shared /
// router array) at byte offset `src_off` to shared-memory offset `dst`,
// completing on mbarrier `bar`.
struct DfCopy {
  uint32_t dst, bytes;
  uint64_t src_off;
  int src, bar;
};

DF_HD inline DfCopy df_window(uint32_t dst, uint64_t first, int n, uint32_t per, int src, int bar) {
  DfCopy C;
  const uint64_t a = first & ~uint64_t(15), e = (first + static_cast<uint64_t>(n) * per + 15) & ~uint64_t(15);
  C.dst = dst; C.src_off = a; C.bytes = static_cast<uint32_t>(e - a); C.src = src; C.bar = bar;
  return C;
}
DF_HD inline DfCopy df_plain(uint32_t dst, uint64_t src_off, uint32_t bytes, int src, int bar) {
  DfCopy C;
  C.dst = dst; C.src_off = src_off; C.bytes = bytes; C.src = src; C.bar = bar;
  return C;
}

// routed gate/up: first the 4 scale/bias windows per run (bar 0, so that every
// tile can start as soon as its rows land), then per tile (8 pairs) and run
// the gate rows and the up rows of its pairs as two copies (bar = tile)
DF_HD inline int df_rg_pieces(const DfGeom& g) {
  int n = 0;
  for (int t = 0; t < g.ntR; ++t) {
    const int a = 8 * t, b = 8 * t + 8 < g.np ? 8 * t + 8 : g.np;
    n += (a < g.n0 && g.n0 < b) ? 2 : 1;
  }
  return n;
}
DF_HD inline int df_rg_count(const DfGeom& g) { return 2 * df_rg_pieces(g) + 4 * (g.n0 > 0) + 4 * (g.n1 > 0); }
DF_HD inline DfCopy df_rg_copy(const DfGeom& g, const size_t* off, int e) {
  const int nwin = 4 * (g.n0 > 0) + 4 * (g.n1 > 0);
  if (e < nwin) {
    const int run = e / 4, a = e % 4;
    return df_window(g.rg_win(run, a), g.rg_src(off, run, a), run ? g.n1 : g.n0, g.sbh, g.j0 + run, 0);
  }
  e -= nwin;
  {
    const int piece = e >> 1, m = e & 1;
    int t = 0, a = 0, b = 0, seen = 0;
    for (t = 0; t < g.ntR; ++t) {          // find the piece: tiles in order, a split tile gives two
      a = 8 * t;
      b = 8 * t + 8 < g.np ? 8 * t + 8 : g.np;
      if (a < g.n0 && g.n0 < b) {
        if (seen == piece) { b = g.n0; break; }
        if (seen + 1 == piece) { a = g.n0; break; }
        seen += 2;
      } else {
        if (seen == piece) break;
        seen += 1;
      }
    }
    const int run = a < g.n0 ? 0 : 1;
    const int row = g.rg_row0(run) + (run ? a - g.n0 : a);
    return df_plain(g.rg_row(a, m), off[3 * m] + static_cast<uint64_t>(row) * g.rowb, static_cast<uint32_t>(b - a) * g.rowb,
                    g.j0 + run, t);
  }
}
// routed down: per slot the nrow rows, then the two windows
DF_HD inline int df_d_count(const DfGeom& g) { return g.nrow > 0 ? 3 * g.k : 0; }
DF_HD inline DfCopy df_d_copy(const DfGeom& g, const size_t* off, int e) {
  const int j = e / 3, part = e % 3;
  if (part == 0)
    return df_plain(g.d_row(j, 0), off[6] + static_cast<uint64_t>(g.o0) * (g.I / 2),
                    static_cast<uint32_t>(g.nrow) * (g.I / 2), j, DF_BAR_D);
  return df_window(g.d_win(j, part - 1), g.d_src(off, part - 1), g.nrow, g.sbi, j, DF_BAR_D);
}
// shared down (matrix 2): rows, S window, B window
DF_HD inline int df_sd_count(const DfGeom& g) { return g.nrow > 0 ? 3 : 0; }
DF_HD inline DfCopy df_sd_copy(const DfGeom& g, int e) {
  if (e == 0)
    return df_plain(g.sd_row(0), static_cast<uint64_t>(g.o0) * (g.Is / 2), static_cast<uint32_t>(g.nrow) * (g.Is / 2),
                    DF_SRC_SHARED + 6, DF_BAR_SD);
  return df_window(g.sd_win(e - 1), g.sd_src(), g.nrow, g.sbs, DF_SRC_SHARED + 6 + e, DF_BAR_SD);
}
// shared gate/up (matrices 0, 1): the gate rows, the up rows, then gate.s, gate.b, up.s, up.b
DF_HD inline int df_sg_count(const DfGeom& g) { return g.nsp > 0 ? 6 : 0; }
DF_HD inline DfCopy df_sg_copy(const DfGeom& g, int e) {
  if (e < 2)
    return df_plain(g.sg_row(0, e), static_cast<uint64_t>(g.s0) * g.rowb, static_cast<uint32_t>(g.nsp) * g.rowb,
                    DF_SRC_SHARED + 3 * e, DF_BAR_SG);
  e -= 2;
  const int m = e / 2, a = e % 2;
  return df_window(g.sg_win(e), g.sg_src(), g.nsp, g.sbh, DF_SRC_SHARED + 3 * m + 1 + a, DF_BAR_SG);
}
// router row c: the row, S window, B window
DF_HD inline int df_rr_count(const DfGeom& g) { return g.c < g.E ? 3 : 0; }
DF_HD inline DfCopy df_rr_copy(const DfGeom& g, int e) {
  if (e == 0)
    return df_plain(g.RR, static_cast<uint64_t>(g.c) * g.H, static_cast<uint32_t>(g.H), DF_SRC_ROUTER, DF_BAR_RR);
  return df_window(g.rr_win(e - 1), g.rr_src(), 1, g.sbh, DF_SRC_ROUTER + e, DF_BAR_RR);
}

// The five copy lists of a CTA in one table: routed gate/up, routed down,
// shared down, shared gate/up, router row (list i starts at df_list_start(g, i)).
DF_HD inline int df_list_count(const DfGeom& g, int list) {
  return list == 0 ? df_rg_count(g) : list == 1 ? df_d_count(g) : list == 2 ? df_sd_count(g)
       : list == 3 ? df_sg_count(g) : df_rr_count(g);
}
DF_HD inline int df_list_start(const DfGeom& g, int list) {
  int n = 0;
  for (int i = 0; i < list; ++i) n += df_list_count(g, i);
  return n;
}
DF_HD inline DfCopy df_list_copy(const DfGeom& g, const size_t* off, int list, int e) {
  return list == 0 ? df_rg_copy(g, off, e) : list == 1 ? df_d_copy(g, off, e) : list == 2 ? df_sd_copy(g, e)
       : list == 3 ? df_sg_copy(g, e) : df_rr_copy(g, e);
}
// table entry: 16 bytes
struct DfCopyS {
  uint32_t dst, bytes, src_off;
  uint16_t src, bar;
};

// Shared-memory bytes of the kernel for these dims and grid (the layout is
// the same for every CTA).
inline size_t decode_fused_smem(int H, int I, int Is, int E, int k, int G) {
  DfGeom g;
  g.init(H, I, Is, E, k, G, 0);
  return g.total;
}

// Whether every CTA's work fits the kernel's fixed limits.
inline bool df_fits(int H, int I, int Is, int E, int k, int G) {
  if (G <= 0 || H % 64 || I % 64 || Is % 64 || H > DF_MAX_H || E > DF_MAX_E || E > G || k > 8) return false;
  if (k * I + Is > DF_MAX_ACT) return false;
  DfGeom g;
  g.init(H, I, Is, E, k, G, 0);
  if (g.npmax > DF_MAX_RG_PAIRS || g.npmax > I || g.nspmax > DF_MAX_SG_PAIRS || g.nrowmax > DF_MAX_ROWS) return false;
  const int tiles_d = (k * g.nrowmax + 15) / 16, tiles_sd = (g.nrowmax + 15) / 16;
  if (tiles_d + tiles_sd > DF_MAX_TILES) return false;
  // every CTA's copy lists fit the table; source offsets fit 32 bits
  if (static_cast<uint64_t>(I) * H * 2 > 0xFFFFFFFFull) return false;
  for (int c = 0; c < G; ++c) {
    DfGeom gc;
    gc.init(H, I, Is, E, k, G, c);
    int n = 0;
    for (int i = 0; i < 5; ++i) n += df_list_count(gc, i);
    if (n > DF_MAX_COPIES) return false;
  }
  // strips: gate/up K over 11 warps, routed down over dp (dividing 12) group
  // parts, shared down over 12 warps; no strip longer than DF_STRIP
  if ((H / 64 + DF_WARPS - 2) / (DF_WARPS - 1) > DF_STRIP) return false;
  if (DF_WARPS % g.dp() != 0 || (Is / 64 + DF_WARPS - 1) / DF_WARPS > DF_STRIP) return false;
  return g.total <= static_cast<uint32_t>(DF_SMEM_LIMIT);
}

#ifdef __CUDACC__
// ------------------------------------------------------------------ PTX bits
__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_gpu(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// tagged words: the 64-bit word carries its value and its layer tag and no
// other data travels with it, so relaxed stores and relaxed polls suffice
// (one single-copy-atomic word; a reader that sees the tag has the value)
__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint64_t df_clock() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void df_mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void df_mbar_arrive(uint32_t bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar) : "memory");
}
// the single arrival of a phase, announcing the bytes its copies will bring
__device__ __forceinline__ void df_mbar_arrive_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(bar),
               "r"(bytes)
               : "memory");
}
// bounded wait on a phase parity
__device__ __forceinline__ bool df_mbar_wait(uint32_t bar, uint32_t parity) {
  uint64_t t0 = 0;
  for (uint32_t i = 0;; ++i) {
    uint32_t ok;
    // the thread sleeps until the phase completes or about 1 us passes
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(1000u)
        : "memory");
    if (ok) return true;
    if ((i & 15u) == 0) {
      const uint64_t now = df_clock();
      if (t0 == 0) t0 = now;
      else if (now - t0 > 2000000000ull) break;
    }
  }
  flag_check(CHECK_WAIT);
  return false;
}
// One 1-D bulk copy completing `bytes` of transaction count on mbarrier
// `bar`; the count was announced beforehand by df_mbar_arrive_tx.
__device__ __forceinline__ void df_bulk(uint32_t bar, uint32_t dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}
// The same, announcing its own bytes first (for barriers whose arrival
// comes after the copies, by df_mbar_arrive).
__device__ __forceinline__ void df_bulk_tx(uint32_t bar, uint32_t dst, const void* src, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
  df_bulk(bar, dst, src, bytes);
}
__device__ __forceinline__ uint4 ldcg_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

// phase timestamps (when requested): layer l, CTA c, point p; df_stamp by
// thread 0, df_stamp_here by the calling thread
__device__ __forceinline__ void df_stamp_here(const DfArgs& a, int l, int p) {
  if (a.stamps != nullptr) a.stamps[(static_cast<size_t>(l) * gridDim.x + blockIdx.x) * 16 + p] = df_clock();
}
__device__ __forceinline__ void df_stamp(const DfArgs& a, int l, int p) {
  if (threadIdx.x == 0) df_stamp_here(a, l, p);
}

// ------------------------------------------------------------ tensor-core dot
// m16n8k32 integer mma: A u8 (4-bit codes), B s8 (one activation digit),
// s32 accumulators.
__device__ __forceinline__ void imma16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// One group (64 inputs) of tile rows g (words wa) and g+8 (words wb) in
// integer form.  Lane (g, t) holds words 2t, 2t+1 of the group (inputs
// 16t .. 16t+15); the low nibbles of a word (inputs 2i of its eight) are the
// u8 operands of k-slots 4t+i, its high nibbles (inputs 2i+1) those of
// k-slots 16+4t+i -- one mask (and one shift) per four codes.  fh, fl: the
// high and low int8 digits of the matching activations in this lane's
// column, as {word 2t even inputs, word 2t odd inputs, word 2t+1 even, odd}.
// d = 256 (codes . high digits) + (codes . low digits), exact in s32.
__device__ __forceinline__ void mma_group_q(int (&d)[4], uint2 wa, uint2 wb, uint4 fh, uint4 fl) {
  constexpr uint32_t M = 0x0F0F0F0Fu;
  int e[4] = {0, 0, 0, 0};
  d[0] = d[1] = d[2] = d[3] = 0;
  const uint32_t lax = wa.x & M, hax = (wa.x >> 4) & M, lbx = wb.x & M, hbx = (wb.x >> 4) & M;
  const uint32_t lay = wa.y & M, hay = (wa.y >> 4) & M, lby = wb.y & M, hby = (wb.y >> 4) & M;
  imma16832(d, lax, lbx, hax, hbx, fh.x, fh.y);
  imma16832(e, lax, lbx, hax, hbx, fl.x, fl.y);
  imma16832(d, lay, lby, hay, hby, fh.z, fh.w);
  imma16832(e, lay, lby, hay, hby, fl.z, fl.w);
#pragma unroll
  for (int i = 0; i < 4; ++i) d[i] = d[i] * 256 + e[i];
}

// How the 8 mma columns are used.  BCAST: every column carries the same
// vector (the result of row g is in accumulator 0/2 of every lane of quad g).
// SLOT: column j carries slot j's activation (row g's result in column
// slot(g)).  DIAG: quad g works on group g0 + (s + g) mod ng at step s and
// column g carries that group of the vector, so the row's result is column
// g -- rows one whole number of 128-byte lines apart then read distinct banks.
enum : int { DF_BCAST = 0, DF_SLOT = 1, DF_DIAG = 2 };

// This warp's strip of ng <= DF_STRIP groups (from g0) of one 16-row tile,
// for the lane's two rows: acc += S (step * idot) + B sum per group, idot
// the integer dot of the codes with the activation's fixed-point values.
// qa/qb: the rows' bytes at this lane's offset 8t; sa/ba, sb/bb: their bf16
// scale and bias rows; fb/xs: the lane's activation digits of the strip and
// the groups' (step, sum of values), in step order, held in registers for
// every tile; suma/sumb: per-row group (step, sum) (SLOT);
// ca/cb: the accumulator of the pair that holds the row's column (SLOT,
// DIAG); rs: the lane's rotation (DIAG).
template <int MODE>
__device__ __forceinline__ void df_strip(const uint8_t* qa, const uint8_t* qb, const uint16_t* sa, const uint16_t* ba,
                                         const uint16_t* sb, const uint16_t* bb, const uint4 (&fb)[DF_STRIP][2],
                                         const float2 (&xs)[DF_STRIP], const float2* suma, const float2* sumb,
                                         int ca, int cb, int g0, int ng, int rs, float& acc_a, float& acc_b) {
#pragma unroll
  for (int j = 0; j < DF_STRIP; ++j) {
    if (j < ng) {
      int gr = g0 + j;
      if (MODE == DF_DIAG) {
        int q = rs + j;
        if (q >= ng) q -= ng;
        gr = g0 + q;
      }
      const uint2 wa = *reinterpret_cast<const uint2*>(qa + 32 * gr);
      const uint2 wb = *reinterpret_cast<const uint2*>(qb + 32 * gr);
      int d[4];
      mma_group_q(d, wa, wb, fb[j][0], fb[j][1]);
      const float2 xa = MODE == DF_SLOT ? suma[gr] : xs[j], xb = MODE == DF_SLOT ? sumb[gr] : xs[j];
      const float va = __int2float_rn(MODE == DF_BCAST ? d[0] : (ca ? d[1] : d[0]));
      const float vb = __int2float_rn(MODE == DF_BCAST ? d[2] : (cb ? d[3] : d[2]));
      acc_a += bf16_to_f32(sa[gr]) * (xa.x * va) + bf16_to_f32(ba[gr]) * xa.y;
      acc_b += bf16_to_f32(sb[gr]) * (xb.x * vb) + bf16_to_f32(bb[gr]) * xb.y;
    }
  }
}
// DIAG strip with the lane's rotated group indices precomputed (gr[j] =
// g0 + (rs + j) mod ng); FULL: the strip holds DF_STRIP groups (no guards).
template <bool FULL>
__device__ __forceinline__ void df_strip_diag(const uint8_t* qa, const uint8_t* qb, const uint16_t* sa,
                                              const uint16_t* ba, const uint16_t* sb, const uint16_t* bb,
                                              const uint4 (&fb)[DF_STRIP][2], const float2 (&xs)[DF_STRIP],
                                              const int (&gr)[DF_STRIP], int odd, int ng, float& acc_a,
                                              float& acc_b) {
#pragma unroll
  for (int j = 0; j < DF_STRIP; ++j) {
    if (FULL || j < ng) {
      const uint2 wa = *reinterpret_cast<const uint2*>(qa + 32 * gr[j]);
      const uint2 wb = *reinterpret_cast<const uint2*>(qb + 32 * gr[j]);
      int d[4];
      mma_group_q(d, wa, wb, fb[j][0], fb[j][1]);
      const float va = __int2float_rn(odd ? d[1] : d[0]);
      const float vb = __int2float_rn(odd ? d[3] : d[2]);
      acc_a += bf16_to_f32(sa[gr[j]]) * (xs[j].x * va) + bf16_to_f32(ba[gr[j]]) * xs[j].y;
      acc_b += bf16_to_f32(sb[gr[j]]) * (xs[j].x * vb) + bf16_to_f32(bb[gr[j]]) * xs[j].y;
    }
  }
}
// The lane's rotated group indices of a DIAG strip.
__device__ __forceinline__ void df_strip_groups(int g0, int ng, int rs, int (&gr)[DF_STRIP]) {
#pragma unroll
  for (int j = 0; j < DF_STRIP; ++j) {
    int q = rs + j;
    if (ng > 0) q %= ng;
    gr[j] = g0 + q;
  }
}

// Load the strip's activation digits (vector f: per group, per lane t the
// high digits at entry 2t and the low digits at 2t+1) and, when given, the
// groups' (step, sum) into registers, rotated by rs (DIAG).
__device__ __forceinline__ void df_load_strip(const uint4* f, const float2* sums, int g0, int ng, int rs, int tq,
                                              uint4 (&fb)[DF_STRIP][2], float2 (&xs)[DF_STRIP]) {
#pragma unroll
  for (int j = 0; j < DF_STRIP; ++j) {
    if (j < ng) {
      int q = rs + j;
      if (q >= ng) q -= ng;
      fb[j][0] = f[8 * (g0 + q) + 2 * tq];
      fb[j][1] = f[8 * (g0 + q) + 2 * tq + 1];
      xs[j] = sums ? sums[g0 + q] : make_float2(0.f, 0.f);
    } else {
      fb[j][0] = fb[j][1] = make_uint4(0u, 0u, 0u, 0u);
      xs[j] = make_float2(0.f, 0.f);
    }
  }
}

// Pair 8 consecutive values into the mma activation word and return its
// (sum of the stored halves, sum of the values).
__device__ __forceinline__ uint4 df_pair8(const float v[8], float& off, float& sum) {
  uint32_t p[4];
  pair_word4(v, p);
  const float2 f0 = unpack_half2(p[0]), f1 = unpack_half2(p[1]), f2 = unpack_half2(p[2]), f3 = unpack_half2(p[3]);
  off = (f0.x + f0.y) + (f1.x + f1.y) + (f2.x + f2.y) + (f3.x + f3.y);
  sum = (f0.x + f0.y + f2.x + f2.y) + 16.f * (f1.x + f1.y + f3.x + f3.y);
  return make_uint4(p[0], p[1], p[2], p[3]);
}
// sum over the 8 lanes of an aligned lane octet
__device__ __forceinline__ float oct_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  v += __shfl_xor_sync(0xffffffffu, v, 4);
  return v;
}
__device__ __forceinline__ float oct_max(float v) {
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
  return v;
}
// largest fixed-point magnitude: 127 * 256 + 127, so both digits are int8
constexpr float DF_QMAX = 32639.f;
// Fixed-point form of one group of 64 activations, 8 per lane of an aligned
// octet (all 32 lanes call it): v ~ step * (256 hi + lo) with step = max|v| /
// DF_QMAX and hi, lo int8 (round to nearest).  Returns the lane's high and
// low digits as {inputs 0,2,4,6; inputs 1,3,5,7} words and the group's
// (step, sum of the values).
__device__ __forceinline__ void df_quant8(const float v[8], uint2& hi, uint2& lo, float2& ss) {
  float m = 0.f, s = 0.f;
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    m = fmaxf(m, fabsf(v[t]));
    s += v[t];
  }
  m = oct_max(m);
  s = oct_sum(s);
  const float inv = m > 0.f ? DF_QMAX / m : 0.f;
  uint32_t h[2] = {0u, 0u}, l[2] = {0u, 0u};
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    const int q = __float2int_rn(v[t] * inv);
    const int dl = ((q + 128) & 255) - 128;
    const int dh = (q - dl) >> 8;
    h[t & 1] |= static_cast<uint32_t>(dh & 255) << (8 * (t >> 1));
    l[t & 1] |= static_cast<uint32_t>(dl & 255) << (8 * (t >> 1));
  }
  hi = make_uint2(h[0], h[1]);
  lo = make_uint2(l[0], l[1]);
  ss = make_float2(m / DF_QMAX, s);
}
// Store word u's digits (8 consecutive inputs) into the digit vector f:
// group u / 8, lane t = (u % 8) / 2, word 2t + (u & 1) of the group.
__device__ __forceinline__ void df_store_digits(uint4* f, int u, uint2 hi, uint2 lo) {
  uint2* f2 = reinterpret_cast<uint2*>(f);
  f2[2 * (u & ~1) + (u & 1)] = hi;
  f2[2 * (u & ~1) + 2 + (u & 1)] = lo;
}

// --------------------------------------------------------------- the kernel
__global__ void __launch_bounds__(DF_THREADS, 1) k_decode_b1(const __grid_constant__ DfArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int H = a.H, I = a.I, Is = a.Is, E = a.E, k = a.k;
  const int G = gridDim.x, c = blockIdx.x;
  const int kI = k * I;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;        // mma fragment row and thread in the row's quad
  DfGeom g;
  g.init(H, I, Is, E, k, G, c);
  const int NGH = H / 64, NGI = I / 64, NGS = Is / 64;

  float* lg = reinterpret_cast<float*>(smem + g.m_lg());
  int* sel = reinterpret_cast<int*>(smem + g.m_sel());
  float* selv = reinterpret_cast<float*>(smem + g.m_selv());
  float* selg = reinterpret_cast<float*>(smem + g.m_selg());
  float* red = reinterpret_cast<float*>(smem + g.m_red());
  float* part = reinterpret_cast<float*>(smem + g.m_part());
  const void** btab = reinterpret_cast<const void**>(smem + g.m_btab());
  DfCopyS* ctab = reinterpret_cast<DfCopyS*>(smem + g.m_ctab());
  uint32_t* txb = reinterpret_cast<uint32_t*>(smem + g.m_tx());
  // per pair: shared-memory offsets of its gate.s, gate.b, up.s, up.b rows
  // (routed pairs at 0.., shared pairs at DF_MAX_RG_PAIRS..)
  uint4* ptab = reinterpret_cast<uint4*>(smem + g.m_ptab());
  int lst[6];                                     // copy-list starts
  lst[0] = 0;
#pragma unroll
  for (int i = 0; i < 5; ++i) lst[i + 1] = lst[i] + df_list_count(g, i);
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + g.m_bars();
  float* xs = reinterpret_cast<float*>(smem + g.f_xs());
  uint4* xf = reinterpret_cast<uint4*>(smem + g.f_xf());
  float2* xsum = reinterpret_cast<float2*>(smem + g.f_xsum());
  uint4* af = reinterpret_cast<uint4*>(smem + g.f_af());
  uint4* sf = reinterpret_cast<uint4*>(smem + g.f_sf());
  float2* asum = reinterpret_cast<float2*>(smem + g.f_asum());
  float2* ssum = reinterpret_cast<float2*>(smem + g.f_ssum());
  const int astride4 = static_cast<int>(g.astride() / 16);     // uint4 per slot of paired activation
  const uint16_t* S16 = reinterpret_cast<const uint16_t*>(smem);

  unsigned* abort_word = a.counter + 32;          // own 128-byte line
  unsigned bar_target = 0;
  auto BAR = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  // The CTA barrier orders every thread's writes before thread 0's release
  // add, and thread 0's acquire poll before every thread's reads after the
  // second CTA barrier; release and acquire are cumulative, so no separate
  // fences (the data crossing CTAs is read through L2).
  auto grid_sync = [&]() {
    __syncthreads();
    if (threadIdx.x == 0) {
      bar_target += static_cast<unsigned>(G);
      red_release_gpu(a.counter, 1u);
      const uint64_t t0 = df_clock();
      while (ld_acquire_gpu(a.counter) < bar_target) {
        __nanosleep(32);
        if (df_clock() - t0 > 2000000000ull) { flag_check(CHECK_WAIT); break; }
      }
    }
    __syncthreads();
  };
  // warp-wide: one arrive on each barrier in [b0, b1) with the bytes its
  // copies bring, then copy list `list` of layer W (routed slots through the
  // selection and the staged blob table)
  auto issue_list = [&](const DfLayer& W, int list, int b0, int b1) {
    if (lane < b1 - b0) df_mbar_arrive_tx(BAR(b0 + lane), txb[b0 + lane]);
    __syncwarp();
#pragma unroll 1
    for (int e = lst[list] + lane; e < lst[list + 1]; e += 32) {
      const DfCopyS C = ctab[e];
      const uint8_t* b;
      if (C.src < 8) {
        int x = sel[C.src];
        if (x < 0 || x >= E) { flag_check(CHECK_EXPERT_ID); x = 0; }
        b = static_cast<const uint8_t*>(btab[x]);
      } else if (C.src < DF_SRC_ROUTER) {
        const int m = (C.src - DF_SRC_SHARED) / 3, arr = (C.src - DF_SRC_SHARED) % 3;
        b = arr == 0 ? reinterpret_cast<const uint8_t*>(W.sq[m])
                     : reinterpret_cast<const uint8_t*>(arr == 1 ? W.ss[m] : W.sb[m]);
      } else {
        const int arr = C.src - DF_SRC_ROUTER;
        b = arr == 0 ? reinterpret_cast<const uint8_t*>(W.rq)
                     : reinterpret_cast<const uint8_t*>(arr == 1 ? W.rs : W.rb);
      }
      df_bulk(BAR(C.bar), sbase + C.dst, b + C.src_off, C.bytes);
    }
    __syncwarp();
  };
  auto issue_sg = [&](const DfLayer& W) { issue_list(W, 3, DF_BAR_SG, DF_BAR_SG + 1); };
  auto issue_rr = [&](const DfLayer& W) { issue_list(W, 4, DF_BAR_RR, DF_BAR_RR + 1); };

  // --------------------------------------------------------------- set-up
  if (threadIdx.x == 0) {
    for (int i = 0; i < DF_NBARS; ++i) df_mbar_init(BAR(i), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int i = threadIdx.x; i < g.np; i += DF_THREADS)
    ptab[i] = make_uint4(g.rg_scale(a.off, i, 0), g.rg_scale(a.off, i, 1), g.rg_scale(a.off, i, 2),
                         g.rg_scale(a.off, i, 3));
  for (int i = threadIdx.x; i < g.nsp; i += DF_THREADS)
    ptab[DF_MAX_RG_PAIRS + i] = make_uint4(g.sg_scale(i, 0), g.sg_scale(i, 1), g.sg_scale(i, 2), g.sg_scale(i, 3));
  // the CTA's copy lists (static: only routed sources change with the selection)
  for (int e = threadIdx.x; e < lst[5]; e += DF_THREADS) {
    int list = 0;
    while (e >= lst[list + 1]) ++list;
    const DfCopy C = df_list_copy(g, a.off, list, e - lst[list]);
    ctab[e] = DfCopyS{C.dst, C.bytes, static_cast<uint32_t>(C.src_off), static_cast<uint16_t>(C.src),
                      static_cast<uint16_t>(C.bar)};
  }
  __syncthreads();
  if (threadIdx.x < DF_NBARS) {          // static too: the byte counts do not depend on the selection
    uint32_t t = 0;
    for (int e = 0; e < lst[5]; ++e) t += ctab[e].bar == threadIdx.x ? ctab[e].bytes : 0u;
    txb[threadIdx.x] = t;
  }
  // every blob pointer is checked (non-null, 16-byte aligned) before any copy
  // reads one; a bad one stops every CTA at the same point
  {
    const long n = static_cast<long>(a.L) * E;
    for (long i = static_cast<long>(c) * DF_THREADS + threadIdx.x; i < n; i += static_cast<long>(G) * DF_THREADS) {
      const uintptr_t p = reinterpret_cast<uintptr_t>(a.layer[i / E].blobs[i % E]);
      if (p == 0 || (p & 15)) { flag_check(CHECK_EXPERT_ID); atomicOr(abort_word, 1u); }
    }
  }
  for (int e = c * DF_THREADS + threadIdx.x; e < E; e += G * DF_THREADS) a.logits[e] = 0ull;   // untagged
  grid_sync();
  if (__ldcg(abort_word) != 0u) return;
  if (warp == 0) {
    issue_sg(a.layer[0]);
    issue_rr(a.layer[0]);
  }
  // blob table and router bias of layer 0 (later layers: staged in phase C)
  for (int e = threadIdx.x; e < E; e += DF_THREADS) btab[e] = a.layer[0].blobs[e];
  float bias_c = (c < E && a.layer[0].bias) ? a.layer[0].bias[c] : 0.f;   // used by the router warp
  __syncthreads();

  for (int l = 0; l < a.L; ++l) {
    const DfLayer& W = a.layer[l];
    const uint32_t par = l & 1;
    df_stamp(a, l, 0);
    // ------------------------------------------------------ A0: rms norm
    {
      const int u = threadIdx.x;            // word u of h: elements 8u .. 8u+7
      float v[8];
      float ss = 0.f;
      if (u < H / 8) {
        const uint4 p0 = ldcg_v4(a.h + 8 * u), p1 = ldcg_v4(a.h + 8 * u + 4);
        v[0] = __uint_as_float(p0.x); v[1] = __uint_as_float(p0.y); v[2] = __uint_as_float(p0.z);
        v[3] = __uint_as_float(p0.w); v[4] = __uint_as_float(p1.x); v[5] = __uint_as_float(p1.y);
        v[6] = __uint_as_float(p1.z); v[7] = __uint_as_float(p1.w);
#pragma unroll
        for (int t = 0; t < 8; ++t) ss = fmaf(v[t], v[t], ss);
      } else {
#pragma unroll
        for (int t = 0; t < 8; ++t) v[t] = 0.f;
      }
      ss = warp_sum(ss);
      if (lane == 0) red[warp] = ss;
      if (threadIdx.x < 8) sel[threadIdx.x] = -1;
      __syncthreads();
      float tot = 0.f;
#pragma unroll
      for (int w = 0; w < DF_WARPS; ++w) tot += red[w];
      const float rr = sqrtf(tot / static_cast<float>(H) + 1e-6f);
      if (u < H / 8) {
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const uint16_t b = f32_to_bf16(__fdiv_rn(v[t], rr));
          v[t] = bf16_to_f32(b);
          xs[8 * u + t] = v[t];
          if (c == 0 && a.x_trace) a.x_trace[static_cast<size_t>(l) * H + 8 * u + t] = b;
        }
      }
      uint2 dh, dl;
      float2 gs;
      df_quant8(v, dh, dl, gs);
      if (u < H / 8) {
        df_store_digits(xf, u, dh, dl);
        if ((lane & 7) == 0) xsum[u >> 3] = gs;
      }
      __syncthreads();
    }
    df_stamp(a, l, 1);

    // --------------------------- router logit c, shared gate/up pairs
    // (the logit goes out as soon as it is computed; the shared pairs are
    // computed while the other CTAs' logits arrive)
    if (warp == DF_WARPS - 1) {
      if (c < E) {
        df_mbar_wait(BAR(DF_BAR_RR), par);
        const uint8_t* qrow = smem + g.RR;
        const uint16_t* S = S16 + g.rr_scale(0) / 2;
        const uint16_t* B = S16 + g.rr_scale(1) / 2;
        float acc = 0.f;
        for (int cc = lane; cc < H / 16; cc += 32) {
          const uint4 q4 = *reinterpret_cast<const uint4*>(qrow + 16 * cc);
          const float sc = bf16_to_f32(S[cc >> 2]), bi = bf16_to_f32(B[cc >> 2]);
          const float* xv = xs + 16 * cc;
          const uint32_t w[4] = {q4.x, q4.y, q4.z, q4.w};
          float a0 = 0.f, a1 = 0.f, sm = 0.f;
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const uint32_t p[2] = {pack_half2(xv[4 * m], xv[4 * m + 2]), pack_half2(xv[4 * m + 1], xv[4 * m + 3])};
            dot_word8(w[m], p, a0, a1);
            const float2 f0 = unpack_half2(p[0]), f1 = unpack_half2(p[1]);
            sm += (f0.x + f0.y) + (f1.x + f1.y);
          }
          acc += sc * ((a0 + a1) - 1024.f * sm) + bi * sm;
        }
        acc = warp_sum(acc);
        if (lane == 0)
          st_relaxed_u64(a.logits + c, (static_cast<unsigned long long>(l + 1) << 32) | __float_as_uint(acc + bias_c));
      }
    } else {
      // warp w < 11: groups [w*NGH/11, (w+1)*NGH/11) of every shared gate/up tile
      const int s0g = warp * NGH / (DF_WARPS - 1), ng = (warp + 1) * NGH / (DF_WARPS - 1) - s0g;
      const int rs = ng > 0 ? gq % ng : 0;
      uint4 fb[DF_STRIP][2];
      float2 xs2[DF_STRIP];
      df_load_strip(xf, xsum, s0g, ng, rs, tq, fb, xs2);
      int grs[DF_STRIP];
      df_strip_groups(s0g, ng, rs, grs);
      if (g.ntS > 0) df_mbar_wait(BAR(DF_BAR_SG), par);
      for (int tile = 0; tile < g.ntS; ++tile) {
        int i = 8 * tile + gq;
        if (i >= g.nsp) i = 8 * tile;
        float acc_a = 0.f, acc_b = 0.f;
        const uint4 sc = ptab[DF_MAX_RG_PAIRS + i];
        df_strip_diag<false>(smem + g.sg_row(i, 0) + 8 * tq, smem + g.sg_row(i, 1) + 8 * tq, S16 + sc.x / 2,
                               S16 + sc.y / 2, S16 + sc.z / 2, S16 + sc.w / 2, fb, xs2, grs, gq & 1, ng, acc_a, acc_b);
        if (tq == (gq >> 1)) {
          part[g.slot_sg(warp, tile) * 16 + gq] = acc_a;
          part[g.slot_sg(warp, tile) * 16 + 8 + gq] = acc_b;
        }
      }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < g.nsp; i += DF_THREADS) {
      const int tile = i / 8, r = i % 8;
      float gs = 0.f, us = 0.f;
      for (int w = 0; w < DF_WARPS - 1; ++w) {
        gs += part[g.slot_sg(w, tile) * 16 + r];
        us += part[g.slot_sg(w, tile) * 16 + 8 + r];
      }
      a.act[kI + g.s0 + i] = __float2half_rn(gelu_tanh(gs) * us);
    }
    df_stamp(a, l, 2);
    // ------------------------------------------------ top-k, routed bytes
    // every logit of layer l (tag l + 1).  Logits of layer l + 1 are written
    // only after the next grid barrier, when every CTA has read these.
    for (int e = threadIdx.x; e < E; e += DF_THREADS) {
      unsigned long long v = ld_relaxed_u64(a.logits + e);
      uint64_t t0 = 0;
      while (static_cast<uint32_t>(v >> 32) != static_cast<uint32_t>(l + 1)) {
        if (t0 == 0) t0 = df_clock();
        else if (df_clock() - t0 > 2000000000ull) { flag_check(CHECK_WAIT); break; }
        __nanosleep(20);
        v = ld_relaxed_u64(a.logits + e);
      }
      lg[e] = __uint_as_float(static_cast<uint32_t>(v));
    }
    __syncthreads();
    df_stamp(a, l, 3);
    for (int e = threadIdx.x; e < E; e += DF_THREADS) {
      const float v = lg[e];
      int rank = 0;
      const float4* l4 = reinterpret_cast<const float4*>(lg);
      for (int f = 0; f < E / 4; ++f) {      // E is a multiple of 8
        const float4 w = l4[f];
        rank += (w.x > v || (w.x == v && 4 * f + 0 < e)) ? 1 : 0;
        rank += (w.y > v || (w.y == v && 4 * f + 1 < e)) ? 1 : 0;
        rank += (w.z > v || (w.z == v && 4 * f + 2 < e)) ? 1 : 0;
        rank += (w.w > v || (w.w == v && 4 * f + 3 < e)) ? 1 : 0;
      }
      if (rank < k) { sel[rank] = e; selv[rank] = v; }
    }
    __syncthreads();
    df_stamp(a, l, 4);
    if (warp == 0) {
      if (lane < k) {
        float den = 0.f;
        for (int j = 0; j < k; ++j) den += expf(selv[j] - selv[0]);
        const float gj = expf(selv[lane] - selv[0]) / den;
        selg[lane] = gj;
        if (c == 0 && a.idx_trace) a.idx_trace[static_cast<size_t>(l) * k + lane] = sel[lane];
        if (c == 0 && a.gates_trace) a.gates_trace[static_cast<size_t>(l) * k + lane] = gj;
      }
    } else if (warp == DF_WARPS - 1) {  // routed gate/up rows and windows, down rows, the next router row
      issue_list(W, 0, 0, g.ntR);
      if (lane == 0) df_stamp_here(a, l, 14);
      issue_list(W, 1, DF_BAR_D, DF_BAR_D + 1);
      if (l + 1 < a.L) issue_rr(a.layer[l + 1]);
    }
    df_stamp(a, l, 5);

    // ------------------------------------------------------ routed gate/up
    {
      // warp w < 11: groups [w*NGH/11, (w+1)*NGH/11) of every routed tile, tile by tile as they land
      const int s0g = warp * NGH / (DF_WARPS - 1);
      const int ng = warp < DF_WARPS - 1 ? (warp + 1) * NGH / (DF_WARPS - 1) - s0g : 0;   // warp 11 issues copies
      const int rs = ng > 0 ? gq % ng : 0;
      uint4 fb[DF_STRIP][2];
      float2 xs2[DF_STRIP];
      df_load_strip(xf, xsum, s0g, ng, rs, tq, fb, xs2);
      int grs[DF_STRIP];
      df_strip_groups(s0g, ng, rs, grs);
      for (int tile = 0; warp < DF_WARPS - 1 && tile < g.ntR; ++tile) {
        df_mbar_wait(BAR(tile), par);
        if (tile != 0) df_mbar_wait(BAR(0), par);      // the scale windows complete on tile 0's barrier
        if (tile == g.ntR - 1 && threadIdx.x == 0) df_stamp_here(a, l, 15);
        int i = 8 * tile + gq;
        if (i >= g.np) i = 8 * tile;
        float acc_a = 0.f, acc_b = 0.f;
        const uint4 sc = ptab[i];
        df_strip_diag<false>(smem + g.rg_row(i, 0) + 8 * tq, smem + g.rg_row(i, 1) + 8 * tq, S16 + sc.x / 2,
                               S16 + sc.y / 2, S16 + sc.z / 2, S16 + sc.w / 2, fb, xs2, grs, gq & 1, ng, acc_a, acc_b);
        if (tq == (gq >> 1)) {
          part[g.slot_rg(warp, tile) * 16 + gq] = acc_a;
          part[g.slot_rg(warp, tile) * 16 + 8 + gq] = acc_b;
        }
      }
    }
    df_stamp(a, l, 6);
    __syncthreads();                     // the union area is read out
    if (warp == 0) {                     // shared down rows into it
      issue_list(W, 2, DF_BAR_SD, DF_BAR_SD + 1);
    } else if (warp == 1) {              // and the next layer's shared gate/up rows after them
      if (l + 1 < a.L) issue_sg(a.layer[l + 1]);
    }
    for (int i = threadIdx.x - 64; i >= 0 && i < g.np; i += DF_THREADS - 64) {
      const int tile = i / 8, r = i % 8;
      float gs = 0.f, us = 0.f;
      for (int w = 0; w < DF_WARPS - 1; ++w) {
        gs += part[g.slot_rg(w, tile) * 16 + r];
        us += part[g.slot_rg(w, tile) * 16 + 8 + r];
      }
      a.act[g.r0 + i] = __float2half_rn(gelu_tanh(gs) * us);
    }
    df_stamp(a, l, 7);
    grid_sync();
    df_stamp(a, l, 8);

    // ------------------------------------------------------------- phase C
    // the next layer's blob table and router bias (this layer's copies are all issued)
    if (l + 1 < a.L) {
      for (int e = threadIdx.x; e < E; e += DF_THREADS) btab[e] = a.layer[l + 1].blobs[e];
      if (warp == DF_WARPS - 1) bias_c = (c < E && a.layer[l + 1].bias) ? a.layer[l + 1].bias[c] : 0.f;
    }
    // this CTA's rows of h (only it writes them), read early for the combine
    float hpre = 0.f;
    if (threadIdx.x < g.nrow)      // issued here (volatile: not moved to its use in the combine)
      asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(hpre) : "l"(a.h + g.o0 + threadIdx.x));
    // fixed-point digits of the k routed slots' activations and of the shared
    // expert's: all loads first (DF_ACT_ROUNDS words per thread), then digits
    {
      const int nw = kI / 8 + Is / 8;
      uint4 raws[DF_ACT_ROUNDS];
#pragma unroll
      for (int r = 0; r < DF_ACT_ROUNDS; ++r) {
        const int u = r * DF_THREADS + threadIdx.x;
        raws[r] = u < nw ? ldcg_v4(a.act + 8 * u) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll 1                             // rolled: one copy of the digit code
      for (int r = 0; r < DF_ACT_ROUNDS; ++r) {
        const int u = r * DF_THREADS + threadIdx.x;
        const uint4 raw = raws[r];             // zero beyond nw
        const uint32_t rw[4] = {raw.x, raw.y, raw.z, raw.w};
        float v[8];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float2 f = unpack_half2(rw[t]);
          v[2 * t] = f.x;
          v[2 * t + 1] = f.y;
        }
        uint2 dh, dl;
        float2 ss;
        df_quant8(v, dh, dl, ss);              // an octet is one group (I, Is: multiples of 64)
        if (u < nw) {
          if (u < kI / 8) {
            const int j = u / (I / 8), w = u % (I / 8);
            df_store_digits(af + j * astride4, w, dh, dl);
            if ((lane & 7) == 0) asum[j * NGI + w / 8] = ss;
          } else {
            const int w = u - kI / 8;
            df_store_digits(sf, w, dh, dl);
            if ((lane & 7) == 0) ssum[w / 8] = ss;
          }
        }
      }
    }
    __syncthreads();
    df_stamp(a, l, 9);
    // down tiles: routed rows rho = j * nrow + r (a tile mixes slots; column j
    // carries slot j's activation), split dp ways by groups and 12/dp ways by
    // tiles; then the shared rows, split 12 ways by groups
    {
      const int colslot = gq < k ? gq : 0;
      {
        const int dp = g.dp(), tp = DF_WARPS / dp, gp = warp % dp, tw = warp / dp;
        const int s0g = gp * NGI / dp, ng = (gp + 1) * NGI / dp - s0g;
        const int t0 = tw * g.ntD / tp, t1 = (tw + 1) * g.ntD / tp;
        uint4 fb[DF_STRIP][2];
        float2 xs2[DF_STRIP];
        df_load_strip(af + colslot * astride4, nullptr, s0g, ng, 0, tq, fb, xs2);
        if (t1 > t0) df_mbar_wait(BAR(DF_BAR_D), par);
        const int kn = k * g.nrow;
        // rows 16 t0 + gq and 16 t0 + 8 + gq as (slot, row), advanced 16 per tile
        int ja = (16 * t0 + gq) / g.nrow, ia = (16 * t0 + gq) % g.nrow;
        int jb = (16 * t0 + 8 + gq) / g.nrow, ib = (16 * t0 + 8 + gq) % g.nrow;
        for (int tile = t0; tile < t1; ++tile) {
          const bool va = 16 * tile + gq < kn, vb = 16 * tile + 8 + gq < kn;
          const int xa = va ? ja : 0, ya = va ? ia : 0, xb = vb ? jb : 0, yb = vb ? ib : 0;
          float acc_a = 0.f, acc_b = 0.f;
          df_strip<DF_SLOT>(smem + g.d_row(xa, ya) + 8 * tq, smem + g.d_row(xb, yb) + 8 * tq,
                            S16 + g.d_scale(a.off, xa, ya, 0) / 2, S16 + g.d_scale(a.off, xa, ya, 1) / 2,
                            S16 + g.d_scale(a.off, xb, yb, 0) / 2, S16 + g.d_scale(a.off, xb, yb, 1) / 2, fb, xs2,
                            asum + xa * NGI, asum + xb * NGI, xa & 1, xb & 1, s0g, ng, 0, acc_a, acc_b);
          if (va && tq == (xa >> 1)) part[g.slot_d(gp, tile) * 16 + gq] = acc_a;
          if (vb && tq == (xb >> 1)) part[g.slot_d(gp, tile) * 16 + 8 + gq] = acc_b;
          ia += 16; while (ia >= g.nrow) { ia -= g.nrow; ++ja; }
          ib += 16; while (ib >= g.nrow) { ib -= g.nrow; ++jb; }
        }
      }
      {
        const int s0g = warp * NGS / DF_WARPS, ng = (warp + 1) * NGS / DF_WARPS - s0g;
        uint4 fb[DF_STRIP][2];
        float2 xs2[DF_STRIP];
        df_load_strip(sf, ssum, s0g, ng, 0, tq, fb, xs2);
        if (g.ntSD > 0) df_mbar_wait(BAR(DF_BAR_SD), par);
        for (int tile = 0; tile < g.ntSD; ++tile) {
          int ra = 16 * tile + gq, rb = 16 * tile + 8 + gq;
          if (ra >= g.nrow) ra = 0;
          if (rb >= g.nrow) rb = 0;
          float acc_a = 0.f, acc_b = 0.f;
          df_strip<DF_BCAST>(smem + g.sd_row(ra) + 8 * tq, smem + g.sd_row(rb) + 8 * tq, S16 + g.sd_scale(ra, 0) / 2,
                             S16 + g.sd_scale(ra, 1) / 2, S16 + g.sd_scale(rb, 0) / 2, S16 + g.sd_scale(rb, 1) / 2, fb,
                             xs2, nullptr, nullptr, 0, 0, s0g, ng, 0, acc_a, acc_b);
          if (tq == 0) {
            part[g.slot_sd(warp, tile) * 16 + gq] = acc_a;
            part[g.slot_sd(warp, tile) * 16 + 8 + gq] = acc_b;
          }
        }
      }
    }
    if (threadIdx.x < g.nrow) lg[threadIdx.x] = hpre;   // the logits are read (nrow <= DF_MAX_E)
    __syncthreads();
    df_stamp(a, l, 10);
    {
      // warp w combines rows w, w + 12, ...: the row's k * dp routed partials
      // (times their gates) and its DF_WARPS shared partials over the lanes,
      // then one warp sum
      const int dp = g.dp(), nr = k * dp, nq = nr + DF_WARPS, dtm = g.d_tiles_max(), stm = g.sd_tiles_max();
      for (int r = warp; r < g.nrow; r += DF_WARPS) {
        float y = 0.f;
#pragma unroll 1
        for (int q = lane; q < nq; q += 32) {
          int slot, row;
          float gate = 1.f;
          if (q < nr) {                    // slot_d(p, tile) = p * dtm + tile
            const int j = q / dp, rho = j * g.nrow + r;
            slot = (q - j * dp) * dtm + (rho >> 4);
            row = rho & 15;
            gate = selg[j];
          } else {                         // slot_sd(w, tile) = dp * dtm + w * stm + tile
            slot = dp * dtm + (q - nr) * stm + (r >> 4);
            row = r & 15;
          }
          y = fmaf(gate, part[slot * 16 + row], y);
        }
        y = warp_sum(y);
        if (lane == 0) {
          const int o = g.o0 + r;
          a.h[o] = lg[r] + y;
          if (a.y_trace) a.y_trace[static_cast<size_t>(l) * H + o] = f32_to_bf16(y);
        }
      }
    }
    df_stamp(a, l, 11);
    df_stamp(a, l, 12);
    if (l + 1 < a.L) grid_sync();
    df_stamp(a, l, 13);
  }
}
#endif  // __CUDACC__

}  // namespace moe
