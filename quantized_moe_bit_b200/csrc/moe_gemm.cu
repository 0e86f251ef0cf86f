// Persistent dequant-fused grouped GEMM of the MoE experts on the
// 5th-generation tensor cores (tcgen05 + TMEM), for steps of several rows
// (prefill chunks, batched decode, streamed chunks).
//
// One launch computes one projection for every (expert, row chunk) of a
// layer: the routed experts of the step's buckets and, when asked, the
// always-on shared expert (one expert whose bucket is every row).
//   phase 0 (gate/up): act[row][i] = fp16( gelu_tanh(W_g x_row)[i] * (W_u x_row)[i] )
//   phase 1 (down):    y[dest(row)][o] = (W_d act_row)[o]   (fp32)
// Swap-AB: 128 weight rows are the MMA's M side and up to 128 bucket rows
// its N side, so one pass over an expert's weights serves every row routed
// to it.  A work item is (expert chunk, m-tile): phase 0 m-tile mt holds gate
// rows 64mt.. and up rows 64mt.. interleaved (A row 2i gate, 2i+1 up, so the
// GeGLU pairs neighbouring TMEM lanes); phase 1 m-tile mt holds down rows
// 128mt...  K runs in atoms of 64 (one quantisation group and one
// 128-byte-swizzled fp16 atom).  Items are dealt to the persistent CTAs
// round-robin (item c, c + G, ...), shared-expert items first.
//
// Warp roles of a CTA (one per SM):
//   warps 0-3   epilogue: TMEM -> registers -> GeGLU / fp32 rows to global
//   warp 4      raw producer: per item its scale/bias rows (4 or 2 bulk
//               copies into a double buffer), then its packed 4-bit codes,
//               256 K-values of 128 rows (one stage) per ring slot as 2-D TMA tiles (a
//               routed expert's tensor maps are a template whose address
//               the warp patches per item into a small ring in global memory)
//   warp 5      B producer: per stage the bucket rows' fp16 activations as
//               one 2-D TMA tile per atom (128-byte swizzle)
//   warps 6-9   MMA issuers: 4 x tcgen05.mma (M=128, N, K=16) per atom, A
//               from TMEM, B from shared memory, into one of two TMEM
//               accumulator sets (the epilogue of an item overlaps the next
//               item's MMAs); the 4 MMAs of an atom go to up to 4 issuers
//               and accumulator chains, since a single thread issues about
//               one tcgen05.mma per 100 cycles whatever N is
//   warps 10-25 dequant (two groups of 8): w = S q + B in half2 arithmetic (q exact, w rounded
//               once to fp16) from a raw slot straight into an A atom of a
//               ring in TMEM (tcgen05.st): the fp16 operand, 4x the bytes of
//               the codes, never passes through shared memory, whose
//               bandwidth it would otherwise exhaust
// Every mbarrier wait is bounded; a wait that runs out sets the device check
// word and a CTA-wide abort flag, after which every role stops issuing work,
// the copies in flight are waited for (bounded) and TMEM is freed.
#include <cuda.h>   // CUtensorMap (the type only; tensor maps are encoded on the host)

#include "tc_utils.cuh"

namespace moe {

constexpr int GM_BM = 128;                   // weight rows per item (MMA M)
constexpr int GM_BK = 64;                    // K per atom (one quantisation group)
// The pipeline moves in stages of GM_APS atoms (K = 256): one raw slot of
// codes, one A stage in TMEM, one B stage of activation tiles.  Every
// barrier wait and release covers a whole stage: a single thread pays a few
// hundred cycles per tcgen05 instruction or mbarrier round trip, which per
// atom would cost more than the atom's data takes to arrive.
constexpr int GM_APS = 4;                    // atoms per stage
constexpr int GM_RAW_SLOT = GM_BM * 128;     // 128 rows x 128 B of codes (256 K values), 128-byte swizzle
constexpr int GM_RS = 3;                     // raw slots
constexpr int GM_ST = 2;                     // A stages (TMEM) and B stages (shared memory)
constexpr int GM_NMAX = 128;                 // bucket rows per chunk (MMA N; TMEM columns per accumulator)
constexpr int GM_ACOLS = GM_BK / 2;          // TMEM columns of one A atom (two fp16 per 32-bit column)
constexpr int GM_TMEM_COLS = 512;            // 2 accumulators of GM_NMAX columns, then the A stages
static_assert(2 * GM_NMAX + GM_ST * GM_APS * GM_ACOLS <= GM_TMEM_COLS, "TMEM budget");
// accumulator chains of an item with Np (padded) rows: as many (up to 4) as
// fit side by side in one accumulator of GM_NMAX columns
__device__ __forceinline__ int gm_chains(int Np) { return Np <= GM_NMAX / 4 ? 4 : Np <= GM_NMAX / 2 ? 2 : 1; }
constexpr int GM_BSLOT = GM_NMAX * 128;      // one atom's activation tile: up to GM_NMAX rows x 128 B
constexpr int GM_BSTAGE = GM_APS * GM_BSLOT;
constexpr int GM_MAX_G = 48;                 // quantisation groups per weight row (K <= 3072)
constexpr int GM_SC_BUF = 4 * (64 * GM_MAX_G * 2 + 16) + 64;   // scale/bias rows of one item (24,704 B)
static_assert(GM_SC_BUF % 128 == 0, "scale buffers keep the maps after them 128-byte aligned");
constexpr int GM_MAX_CHUNKS = 512;
constexpr int GM_PREP_W = (GM_MAX_G * 64 / 8 + 255) / 256;   // 16-byte words of a row per prep thread
constexpr int GM_MAX_CTAS = 160;             // grid cap (one CTA per SM)
// Per-CTA tensor-map sets (gate and up, or down) in global memory.  An
// item's set is patched after the wait that frees its first raw slot, which
// proves that every copy issued GM_RS slots before has landed; each item
// issues at least one slot, so a ring of more than GM_RS + 1 sets is never
// patched under a copy still in flight.
constexpr int GM_MAP_RING = 6;
static_assert(GM_MAP_RING > GM_RS + 1, "tensor-map ring vs raw ring");
// MMA issue: one thread issues about one tcgen05.mma per 100 cycles whatever
// N is, so small-N items are issue-bound; GM_MMA_WARPS warps issue in
// parallel, each into its own accumulator chain of the item (up to 4 chains
// of 128 / chains TMEM columns; the epilogue adds them).
// Dequant: 2 groups of 8 warps; in every stage group g takes the atoms g,
// g + 2 (an atom's dequant is a latency-bound chain of about 400 cycles, so
// two run at once).  In a group two warps share each TMEM sub-partition
// (warp w writes TMEM lanes 32 (w % 4) ..), each taking half of every atom
// row (4 code words).  Both groups take part in every stage's barriers.
// Epilogue: 8 warps, two per TMEM sub-partition (warps 0-3 and the four
// consecutive warps from GM_EPI_WARP1; warp w reads TMEM lanes 32 (w % 4) ..),
// each pair taking the item's 16-column blocks alternately.
constexpr int GM_RAW_WARP = 4, GM_B_WARP = 5, GM_MMA_WARP = 6, GM_MMA_WARPS = 4;
constexpr int GM_DQ_WARP0 = GM_MMA_WARP + GM_MMA_WARPS, GM_DQ_GROUPS = 2, GM_DQ_WARPS = 8 * GM_DQ_GROUPS;
constexpr int GM_EPI_WARP1 = GM_DQ_WARP0 + GM_DQ_WARPS, GM_EPI_WARPS = 8;
constexpr int GM_THREADS = (GM_EPI_WARP1 + 4) * 32;
// barriers: raw full/empty [RS], a full [ST], stage empty [ST], b full [ST], sc full/empty [2],
// acc full/empty [2], final
constexpr int GM_NBARS = 2 * GM_RS + 3 * GM_ST + 4 + 4 + 1;
constexpr size_t GM_SMEM = 1024 + static_cast<size_t>(GM_ST) * GM_BSTAGE +
                           static_cast<size_t>(GM_RS) * GM_RAW_SLOT + 2 * GM_SC_BUF + 256 + GM_NBARS * 8 + 64;
static_assert(GM_SC_BUF % 128 == 0 && GM_RAW_SLOT % 1024 == 0, "copy destinations: swizzle atoms 1024-byte, maps 128-byte aligned");
static_assert(GM_SMEM <= 232448, "shared memory of the grouped GEMM");

// Box heights of the activation tensor maps (rows of the TMA tile): 16, 32, .. GM_NMAX.
constexpr int GM_NBOX = GM_NMAX == 128 ? 4 : GM_NMAX == 64 ? 3 : GM_NMAX == 32 ? 2 : 1;
static_assert((16 << (GM_NBOX - 1)) == GM_NMAX, "GM_NMAX is 16, 32, 64 or 128");
static_assert(GM_BSLOT % 1024 == 0, "activation tiles are 1024-byte aligned swizzle atoms");
__host__ __device__ constexpr int gm_box_rows(int i) { return 16 << i; }

// A chunk: up to GM_NMAX consecutive rows of one expert's bucket.
//   w0 = expert id (routed) | segment << 31 (0 shared, 1 routed)
//   w1 = first row in the B / activation array | rows << 24
struct GmPlan {
  int n_chunks[2];        // shared, routed
  int pad[2];
  uint2 chunk[GM_MAX_CHUNKS];
};

struct GemmArgs {
  CUtensorMap tmB[2][GM_NBOX];   // activation tiles: [segment][box height 16, 32, 64, 128]
  // weight-code tiles (uint8 [rows, K/2 bytes], boxes of 128 bytes x 64 rows
  // (phase 0) or 128 rows (phase 1), 128-byte swizzle): the routed
  // matrices' template (its address is replaced per item on the device) and
  // the shared expert's matrices (phase 0: gate, up; phase 1: down in [0])
  CUtensorMap tmR;
  CUtensorMap tmS[2];
  CUtensorMap* map_ring;         // device [GM_MAX_CTAS][GM_MAP_RING][2] patched routed maps
  int phase;                     // 0 gate/up + GeGLU, 1 down
  int H;
  // routed segment
  int I, E, k;
  const void* const* blob_ptrs;  // device [E]
  const int32_t* pairs;          // device [P] (pair value t*k + j in bucket order)
  int P;                         // rows of the routed B / activation arrays (T * k)
  size_t off[9];
  __half* act_r;                 // phase 0 output [P, I] (bucket order); phase 1 input (in tmB[1])
  float* y_r;                    // phase 1 output [P, H], row = pair value
  // shared segment
  int Is, Ts;
  const uint8_t* sq[3];
  const uint16_t* ss[3];
  const uint16_t* sb[3];
  __half* act_s;                 // phase 0 output [Ts, Is]
  float* y_s;                    // phase 1 output [Ts, H]
  const GmPlan* plan;            // device, written by k_gm_prep
};

// byte offset of (row r, 16-byte chunk c) inside one 128-row x 128 B swizzled atom
__device__ __forceinline__ uint32_t gm_sw128(int r, int c) {
  return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ __half2 gm_h2(uint32_t v) { return *reinterpret_cast<__half2*>(&v); }
__device__ __forceinline__ uint32_t gm_u32(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }

// K order inside every block of 8 K values, for both MMA operands: stored
// position p holds element kperm(p) = {0, 4, 1, 5, 2, 6, 3, 7}[p] of the block,
// i.e. element e sits at position 2 (e % 4) + e / 4.  The nibble masks below
// produce the weights in exactly this order (q0 q4 | q1 q5 | q2 q6 | q3 q7),
// so the activations are written in it too (gather and GeGLU epilogue) and
// the sum over K is unchanged.
__host__ __device__ __forceinline__ int gm_kpos(int e) { return ((e & 7) & 3) * 2 + ((e & 7) >> 2) + (e & ~7); }

// 8 nibbles of one word -> 8 fp16 weights S*q + B in the permuted K order.
// Each nibble becomes the fp16 1024 + q (or 1024 + 16 q) by OR-ing it into
// the exponent pattern 0x6400, minus 1024 (exact); then one fma rounds S*q + B.
__device__ __forceinline__ uint4 gm_dequant_word(uint32_t w, __half2 s2, __half2 b2) {
  const __half2 k1024 = __floats2half2_rn(1024.f, 1024.f);
  const __half2 k16 = __floats2half2_rn(0.0625f, 0.0625f);
  const __half2 k64 = __floats2half2_rn(-64.f, -64.f);
  const uint32_t w8 = w >> 8;
  const __half2 q04 = __hsub2(gm_h2((w & 0x000F000Fu) | 0x64006400u), k1024);    // q0, q4
  const __half2 q15 = __hfma2(gm_h2((w & 0x00F000F0u) | 0x64006400u), k16, k64);  // q1, q5
  const __half2 q26 = __hsub2(gm_h2((w8 & 0x000F000Fu) | 0x64006400u), k1024);   // q2, q6
  const __half2 q37 = __hfma2(gm_h2((w8 & 0x00F000F0u) | 0x64006400u), k16, k64); // q3, q7
  uint4 o;
  o.x = gm_u32(__hfma2(q04, s2, b2));
  o.y = gm_u32(__hfma2(q15, s2, b2));
  o.z = gm_u32(__hfma2(q26, s2, b2));
  o.w = gm_u32(__hfma2(q37, s2, b2));
  return o;
}

__device__ __forceinline__ uint4 gm_lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ uint2 gm_lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t gm_lds_u16(uint32_t a) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ void gm_sts128(uint32_t a, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

// ------------------------------------------------------------------ prep
// Block 0 writes the chunk list: shared chunks first, then the routed
// buckets cut into chunks of at most GM_NMAX rows, largest chunks first (a
// counting sort by size; the order within a size is free), so that the
// grid's serpentine walk over the items balances the CTAs;
// every block gathers the layer input into bucket order as fp16
// (xs[pos] = x[pairs[pos] / k]) and, when xh is given, writes x as fp16;
// both in the permuted K order of gm_kpos.
__global__ void __launch_bounds__(256) k_gm_prep(const uint16_t* __restrict__ x, int T, int H, int k,
                                                 const int32_t* __restrict__ offsets,
                                                 const int32_t* __restrict__ pairs,
                                                 const int32_t* __restrict__ active,
                                                 const int32_t* __restrict__ n_active, int E, int routed,
                                                 int shared_rows, __half* __restrict__ xs, __half* __restrict__ xh,
                                                 GmPlan* __restrict__ plan) {
  if (blockIdx.x == 0) {
    __shared__ int s_cnt[GM_NMAX + 1];     // routed chunks per size, then the next slot of each size
    const int nsh = (shared_rows + GM_NMAX - 1) / GM_NMAX;
    for (int c = threadIdx.x; c < nsh; c += blockDim.x) {
      const int n0 = c * GM_NMAX, n = min(GM_NMAX, shared_rows - n0);
      plan->chunk[c] = make_uint2(0u, static_cast<uint32_t>(n0) | (static_cast<uint32_t>(n) << 24));
    }
    for (int i = threadIdx.x; i <= GM_NMAX; i += blockDim.x) s_cnt[i] = 0;
    int na = routed ? *n_active : 0;
    if (na < 0 || na > E) { if (threadIdx.x == 0) flag_check(CHECK_EXPERT_ID); na = 0; }
    auto bucket = [&](int a, int& e, int& pos0, int& cnt) {
      e = active[a];
      pos0 = 0;
      cnt = 0;
      if (e < 0 || e >= E) { flag_check(CHECK_EXPERT_ID); e = 0; }
      else { pos0 = offsets[e]; cnt = offsets[e + 1] - pos0; }
      if (cnt < 0) cnt = 0;
    };
    __syncthreads();
    for (int a = threadIdx.x; a < na; a += blockDim.x) {      // chunks per size
      int e, pos0, cnt;
      bucket(a, e, pos0, cnt);
      if (cnt / GM_NMAX) atomicAdd(&s_cnt[GM_NMAX], cnt / GM_NMAX);
      if (cnt % GM_NMAX) atomicAdd(&s_cnt[cnt % GM_NMAX], 1);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // first slot of every size, the largest chunks first (a warp scan over
      // sizes GM_NMAX .. 1, 32 at a time)
      const int lane = threadIdx.x;
      int base = nsh;
      for (int n0 = GM_NMAX; n0 >= 1; n0 -= 32) {
        const int n = n0 - lane;
        const int v = n >= 1 ? s_cnt[n] : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += t;
        }
        if (n >= 1) s_cnt[n] = base + incl - v;
        base += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) {
        int nr = base - nsh;
        if (base > GM_MAX_CHUNKS) { flag_check(CHECK_PAIR_ID); nr = GM_MAX_CHUNKS - nsh; }
        plan->n_chunks[0] = nsh;
        plan->n_chunks[1] = nr;
      }
    }
    __syncthreads();
    for (int a = threadIdx.x; a < na; a += blockDim.x) {      // every chunk into the next slot of its size
      int e, pos0, cnt;
      bucket(a, e, pos0, cnt);
      for (int n0 = 0; n0 < cnt; n0 += GM_NMAX) {
        const int n = min(GM_NMAX, cnt - n0);
        const int slot = atomicAdd(&s_cnt[n], 1);
        if (slot < GM_MAX_CHUNKS)
          plan->chunk[slot] = make_uint2(static_cast<uint32_t>(e) | 0x80000000u,
                                         static_cast<uint32_t>(pos0 + n0) | (static_cast<uint32_t>(n) << 24));
      }
    }
  }
  // gather, a row per block and step (the row's source looked up once): 8
  // values (16 bytes) per thread, all of a thread's loads of the row first
  const int w8 = H / 8;
  // routed rows: the bucketed pairs only; pair slots past offsets[E] belong
  // to no chunk (a caller may size T for more rows than it bucketed)
  int P = routed ? offsets[E] : 0;
  if (P < 0 || P > T * k) P = routed ? T * k : 0;
  const int nrow = P + (xh ? T : 0);
  for (int row = blockIdx.x; row < nrow; row += gridDim.x) {
    int t;
    __half* dst;
    if (row < P) {
      const int p = pairs[row];
      t = p / k;
      if (p < 0 || t >= T) { if (threadIdx.x == 0) flag_check(CHECK_PAIR_ID); t = -1; }
      dst = xs + static_cast<size_t>(row) * H;
    } else {
      t = row - P;
      dst = xh + static_cast<size_t>(t) * H;
    }
    uint4 u[GM_PREP_W];
#pragma unroll
    for (int j = 0; j < GM_PREP_W; ++j) {
      const int w = threadIdx.x + j * 256;
      u[j] = (t >= 0 && w < w8) ? *reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * H + 8 * w)
                                : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int j = 0; j < GM_PREP_W; ++j) {
      const int w = threadIdx.x + j * 256;
      if (w < w8) {
        // elements e0..e7 of the block in the permuted K order e0 e4 | e1 e5 | e2 e6 | e3 e7
        const uint4 v = u[j];
        const float e0 = __uint_as_float(v.x << 16), e1 = __uint_as_float(v.x & 0xFFFF0000u);
        const float e2 = __uint_as_float(v.y << 16), e3 = __uint_as_float(v.y & 0xFFFF0000u);
        const float e4 = __uint_as_float(v.z << 16), e5 = __uint_as_float(v.z & 0xFFFF0000u);
        const float e6 = __uint_as_float(v.w << 16), e7 = __uint_as_float(v.w & 0xFFFF0000u);
        uint4 o;
        o.x = pack_half2(e0, e4);
        o.y = pack_half2(e1, e5);
        o.z = pack_half2(e2, e6);
        o.w = pack_half2(e3, e7);
        *reinterpret_cast<uint4*>(dst + 8 * w) = o;
      }
    }
  }
}

// ------------------------------------------------------------------ items
struct GmItem {
  int seg;        // 0 shared, 1 routed
  int e;          // expert (routed)
  int row0;       // first row of the chunk in the segment's B / activation array
  int N;          // rows of the chunk
  int mt;         // m-tile
  int K, nkb;     // contraction length and its atoms
};

__device__ __forceinline__ GmItem gm_item(const GemmArgs& a, int n_sh, int item) {
  const int mts = a.phase == 0 ? a.Is / 64 : a.H / GM_BM;
  const int mtr = a.phase == 0 ? a.I / 64 : a.H / GM_BM;
  int c, mt;
  if (item < n_sh * mts) { c = item / mts; mt = item - c * mts; }
  else { const int j = item - n_sh * mts; c = n_sh + j / mtr; mt = j - (j / mtr) * mtr; }
  const uint2 ch = a.plan->chunk[c];
  GmItem it;
  it.seg = static_cast<int>(ch.x >> 31);
  it.e = static_cast<int>(ch.x & 0x7FFFFFFFu);
  it.row0 = static_cast<int>(ch.y & 0xFFFFFFu);
  it.N = static_cast<int>(ch.y >> 24);
  it.mt = mt;
  it.K = a.phase == 0 ? a.H : (it.seg ? a.I : a.Is);
  it.nkb = it.K / GM_BK;
  return it;
}

// The items of a launch go out in rounds of G (the grid): round r gives item
// r G + c to CTA c in even rounds and to CTA G - 1 - c in odd ones.  With the
// chunks sorted by size (cost) this serpentine evens out the CTAs' totals;
// every role of a CTA walks the same sequence.
__device__ __forceinline__ int gm_item_at(int r, int G) {
  return r * G + ((r & 1) ? G - 1 - static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.x));
}

// Matrix m (0 gate, 1 up, 2 down) of the item's expert: codes, scales, biases.
__device__ __forceinline__ const uint8_t* gm_q(const GemmArgs& a, const GmItem& it, int m) {
  if (it.seg == 0) return a.sq[m];
  return static_cast<const uint8_t*>(a.blob_ptrs[it.e]) + a.off[3 * m];
}
__device__ __forceinline__ const uint16_t* gm_s(const GemmArgs& a, const GmItem& it, int m, int which) {
  if (it.seg == 0) return which ? a.sb[m] : a.ss[m];
  return reinterpret_cast<const uint16_t*>(static_cast<const uint8_t*>(a.blob_ptrs[it.e]) + a.off[3 * m + 1 + which]);
}

// A routed item's blob must be a non-null 16-byte aligned address (the bulk
// copies need it); a bad one is flagged and stops the CTA.
__device__ __forceinline__ bool gm_blob_ok(const GemmArgs& a, const GmItem& it) {
  if (it.seg == 0) return true;
  const uintptr_t p = reinterpret_cast<uintptr_t>(a.blob_ptrs[it.e]);
  return p != 0 && (p & 15) == 0;
}

// Scale-buffer layout of an item: regions of `rows` rows x G groups (bf16),
// each padded by 16 bytes so that rows of different regions fall on
// different banks.  Phase 0: gate.s, gate.b, up.s, up.b (64 rows each);
// phase 1: down.s, down.b (128 rows each).
__device__ __forceinline__ uint32_t gm_region_bytes(int phase, int G) {
  return static_cast<uint32_t>((phase == 0 ? 64 : 128) * G * 2 + 16);
}

// One try_wait that lets the hardware suspend the thread until the phase
// completes or about `ns` nanoseconds pass: waiting warps then do not take
// issue slots from the dequant warps that share their sub-partition.
__device__ __forceinline__ bool gm_try(uint32_t bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}

// Bounded mbarrier wait (about two seconds) that also gives up when another
// role of the CTA has aborted (abort flag in shared memory).
__device__ __forceinline__ bool gm_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  if (gm_try(bar, parity, 0u)) return true;
  const uint64_t t0 = tc::globaltimer_ns();
  for (;;) {
    if (gm_try(bar, parity, 20000u)) return true;
    if (*abort_flag) return false;
    if (tc::globaltimer_ns() - t0 > 2000000000ull) break;
  }
  flag_check(CHECK_WAIT);
  *abort_flag = 1;
  return false;
}

// Bounded wait that ignores the abort flag (used on the way out, for copies
// already in flight and the last MMAs).
__device__ __forceinline__ void gm_wait_drain(uint32_t bar, uint32_t parity) {
  if (gm_try(bar, parity, 0u)) return;
  const uint64_t t0 = tc::globaltimer_ns();
  for (;;) {
    if (gm_try(bar, parity, 20000u)) return;
    if (tc::globaltimer_ns() - t0 > 2000000000ull) { flag_check(CHECK_WAIT); return; }
  }
}

// ------------------------------------------------------------------ kernel
__global__ void __launch_bounds__(GM_THREADS, 1) k_moe_gemm(const __grid_constant__ GemmArgs a) {
  extern __shared__ __align__(1024) unsigned char gm_smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(gm_smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sB = smem;                                      // [ST][GM_APS][GM_BSLOT], 1024-aligned
  unsigned char* sRaw = sB + GM_ST * GM_BSTAGE;                  // [RS][128 rows x 128 B], swizzled
  unsigned char* sSC = sRaw + GM_RS * GM_RAW_SLOT;               // [2][GM_SC_BUF]
  unsigned char* sMap = sSC + 2 * GM_SC_BUF;                     // [2][128 B] tensor maps being patched
  uint64_t* bars = reinterpret_cast<uint64_t*>(sMap + 256);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + GM_NBARS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + GM_NBARS) + 4;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar0 = tc::smem_u32(bars);
  auto raw_full = [&](int s) { return bar0 + 8u * s; };
  auto raw_empty = [&](int s) { return bar0 + 8u * (GM_RS + s); };
  auto a_full = [&](int s) { return bar0 + 8u * (2 * GM_RS + s); };
  auto st_empty = [&](int s) { return bar0 + 8u * (2 * GM_RS + GM_ST + s); };   // A and B stage s free
  auto b_full = [&](int s) { return bar0 + 8u * (2 * GM_RS + 2 * GM_ST + s); };
  const uint32_t barx = bar0 + 8u * (2 * GM_RS + 3 * GM_ST);
  auto sc_full = [&](int s) { return barx + 8u * s; };
  auto sc_empty = [&](int s) { return barx + 8u * (2 + s); };
  auto acc_full = [&](int s) { return barx + 8u * (4 + s); };
  auto acc_empty = [&](int s) { return barx + 8u * (6 + s); };
  const uint32_t final_bar = barx + 8u * 8;

  if (threadIdx.x == 0) {
    for (int s = 0; s < GM_RS; ++s) { tc::mbar_init(raw_full(s), 1); tc::mbar_init(raw_empty(s), GM_DQ_WARPS); }
    // a stage: every dequant warp arrives once when its atoms are in TMEM;
    // every MMA issuer commits once when its MMAs of the stage are done
    for (int s = 0; s < GM_ST; ++s) {
      tc::mbar_init(a_full(s), GM_DQ_WARPS);
      tc::mbar_init(st_empty(s), GM_MMA_WARPS);
      tc::mbar_init(b_full(s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(sc_full(s), 1);
      tc::mbar_init(sc_empty(s), GM_DQ_WARPS);
      tc::mbar_init(acc_full(s), GM_MMA_WARPS);
      tc::mbar_init(acc_empty(s), GM_EPI_WARPS);
    }
    tc::mbar_init(final_bar, GM_MMA_WARPS);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), GM_TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int n_sh = a.plan->n_chunks[0], n_r = a.plan->n_chunks[1];
  const int mts = a.phase == 0 ? a.Is / 64 : a.H / GM_BM;
  const int mtr = a.phase == 0 ? a.I / 64 : a.H / GM_BM;
  const int n_items = n_sh * mts + n_r * mtr;
  const int G = gridDim.x;

  if (warp == GM_RAW_WARP) {
    // ------------------------------------------------------------ raw codes
    uint32_t rs = 0, sc_issued = 0;
    int il = 0;
    bool ok = true;
    for (int rd = 0, item = gm_item_at(0, G); item < n_items && ok; item = gm_item_at(++rd, G), ++il) {
      const GmItem it = gm_item(a, n_sh, item);
      if (!gm_blob_ok(a, it)) {
        if (lane == 0) { flag_check(CHECK_EXPERT_ID); *abort_flag = 1; }
        break;
      }
      // the item's scale and bias rows into its half of the double buffer
      // (free once the dequant of item il - 2 is done)
      {
        const int sb = il & 1;
        if (il >= 2 && !(ok = gm_wait(sc_empty(sb), ((il >> 1) - 1) & 1, abort_flag))) break;
        const int Gq = it.nkb;
        const uint32_t reg = gm_region_bytes(a.phase, Gq);
        const uint32_t dst = tc::smem_u32(sSC + sb * GM_SC_BUF);
        if (a.phase == 0) {
          const uint32_t nb = static_cast<uint32_t>(64 * Gq * 2);
          if (lane == 0) tc::mbar_arrive_tx(sc_full(sb), 4 * nb);
          __syncwarp();
          if (lane < 4) {
            const int m = lane >> 1, which = lane & 1;     // gate.s, gate.b, up.s, up.b
            const uint16_t* src = gm_s(a, it, m, which) + static_cast<size_t>(64 * it.mt) * Gq;
            tc::bulk_g2s(dst + lane * reg, src, nb, sc_full(sb));
          }
        } else {
          const uint32_t nb = static_cast<uint32_t>(GM_BM * Gq * 2);
          if (lane == 0) tc::mbar_arrive_tx(sc_full(sb), 2 * nb);
          __syncwarp();
          if (lane < 2) {
            const uint16_t* src = gm_s(a, it, 2, lane) + static_cast<size_t>(GM_BM * it.mt) * Gq;
            tc::bulk_g2s(dst + lane * reg, src, nb, sc_full(sb));
          }
        }
        ++sc_issued;
      }
      const int nraw = (it.nkb + GM_APS - 1) / GM_APS;
      const CUtensorMap* map0 = &a.tmS[0];
      const CUtensorMap* map1 = &a.tmS[1];
      for (int j = 0; j < nraw; ++j, ++rs) {
        const int slot = rs % GM_RS;
        if (rs >= GM_RS && !(ok = gm_wait(raw_empty(slot), ((rs / GM_RS) - 1) & 1, abort_flag))) break;
        if (j == 0 && it.seg == 1) {
          // a routed expert's code maps: the template with the expert's
          // matrix address, patched into this CTA's ring (the shared
          // expert's maps come with the launch)
          const int nm = a.phase == 0 ? 2 : 1;
          CUtensorMap* ring = a.map_ring + (static_cast<size_t>(blockIdx.x) * GM_MAP_RING + (il % GM_MAP_RING)) * 2;
          if (lane < 8 * nm)       // stage the template: 16 bytes per lane
            *reinterpret_cast<uint4*>(sMap + (lane >> 3) * 128 + (lane & 7) * 16) =
                reinterpret_cast<const uint4*>(&a.tmR)[lane & 7];
          __syncwarp();
          if (lane == 0)
            for (int m = 0; m < nm; ++m)
              tc::tmap_replace_addr(tc::smem_u32(sMap + m * 128), gm_q(a, it, a.phase == 0 ? m : 2));
          __syncwarp();
          for (int m = 0; m < nm; ++m) tc::tmap_publish(ring + m, tc::smem_u32(sMap + m * 128));
          if (lane == 0)
            for (int m = 0; m < nm; ++m) tc::tmap_acquire(ring + m);
          map0 = ring;
          map1 = ring + 1;
        }
        if (lane == 0) {
          // the full box always lands (bytes beyond a row's end read as zero)
          tc::mbar_arrive_tx(raw_full(slot), GM_RAW_SLOT);
          const uint32_t dst = tc::smem_u32(sRaw + slot * GM_RAW_SLOT);
          if (a.phase == 0) {          // gate rows 64mt.. -> tile rows 0..63, up rows -> 64..127
            tc::tma_load_2d(dst, map0, 128 * j, 64 * it.mt, raw_full(slot));
            tc::tma_load_2d(dst + 64 * 128, map1, 128 * j, 64 * it.mt, raw_full(slot));
          } else {
            tc::tma_load_2d(dst, map0, 128 * j, GM_BM * it.mt, raw_full(slot));
          }
        }
        __syncwarp();
      }
    }
    // copies in flight land before the CTA ends (the last slots issued)
    for (uint32_t q = rs > GM_RS ? rs - GM_RS : 0; q < rs; ++q) gm_wait_drain(raw_full(q % GM_RS), (q / GM_RS) & 1);
    for (uint32_t q = sc_issued > 2 ? sc_issued - 2 : 0; q < sc_issued; ++q) gm_wait_drain(sc_full(q & 1), (q >> 1) & 1);
  } else if (warp == GM_B_WARP) {
    // ---------------------------------------------------- activation tiles
    uint32_t ss = 0;                                       // stages issued
    bool ok = true;
    for (int rd = 0, item = gm_item_at(0, G); item < n_items && ok; item = gm_item_at(++rd, G)) {
      const GmItem it = gm_item(a, n_sh, item);
      const int Np = (it.N + 15) & ~15;
      int bi = 0;
      while (bi < GM_NBOX - 1 && gm_box_rows(bi) < Np) ++bi;
      const uint32_t bbytes = static_cast<uint32_t>(gm_box_rows(bi)) * 128u;
      const CUtensorMap* tm = &a.tmB[it.seg][bi];
      const int nst = (it.nkb + GM_APS - 1) / GM_APS;
      for (int jst = 0; jst < nst; ++jst, ++ss) {
        const int slot = ss % GM_ST;
        if (ss >= GM_ST && !(ok = gm_wait(st_empty(slot), ((ss / GM_ST) - 1) & 1, abort_flag))) break;
        const int na = min(GM_APS, it.nkb - GM_APS * jst);
        if (lane == 0) {
          tc::mbar_arrive_tx(b_full(slot), na * bbytes);
          for (int aa = 0; aa < na; ++aa)
            tc::tma_load_2d(tc::smem_u32(sB + slot * GM_BSTAGE + aa * GM_BSLOT), tm, (GM_APS * jst + aa) * GM_BK,
                            it.row0, b_full(slot));
        }
        __syncwarp();
      }
    }
    for (uint32_t q = ss > GM_ST ? ss - GM_ST : 0; q < ss; ++q) gm_wait_drain(b_full(q % GM_ST), (q / GM_ST) & 1);
  } else if (warp >= GM_MMA_WARP && warp < GM_MMA_WARP + GM_MMA_WARPS) {
    // ---------------------------------------------------------- MMA issuers
    // issuer j < C (C chains for the item) issues MMAs kk = j, j + C, .. of
    // every atom into chain j (TMEM columns acc * GM_NMAX + j * GM_NMAX / C).
    // Every issuer, active or not, waits for every stage and item and
    // commits once per stage (st_empty) and once per item (acc_full): the
    // barriers count GM_MMA_WARPS arrivals, and no issuer runs ahead of the
    // rings (a parity wait is only unambiguous within one phase).
    const int j = warp - GM_MMA_WARP;
    uint32_t ss = 0;
    int il = 0;
    bool ok = true;
    for (int rd = 0, item = gm_item_at(0, G); item < n_items && ok; item = gm_item_at(++rd, G), ++il) {
      const GmItem it = gm_item(a, n_sh, item);
      const int Np = (it.N + 15) & ~15;
      const int C = gm_chains(Np);
      const int acc = il & 1;
      if (il >= 2 && !(ok = gm_wait(acc_empty(acc), ((il >> 1) - 1) & 1, abort_flag))) break;
      tc::tc_fence_after();
      const uint32_t idesc = tc::idesc_f16_f32(GM_BM, Np);
      const uint32_t dcol = tmem + static_cast<uint32_t>(acc * GM_NMAX + (j % C) * (GM_NMAX / C));
      const int nst = (it.nkb + GM_APS - 1) / GM_APS;
      for (int jst = 0; jst < nst; ++jst, ++ss) {
        const int slot = ss % GM_ST;
        if (!(ok = gm_wait(a_full(slot), (ss / GM_ST) & 1, abort_flag))) break;
        if (!(ok = gm_wait(b_full(slot), (ss / GM_ST) & 1, abort_flag))) break;
        tc::tc_fence_after();
        if (lane == 0) {
          if (j < C) {
            const int na = min(GM_APS, it.nkb - GM_APS * jst);
            const uint32_t aT = tmem + static_cast<uint32_t>(2 * GM_NMAX + slot * GM_APS * GM_ACOLS);
            const uint32_t bBase = tc::smem_u32(sB + slot * GM_BSTAGE);
            for (int aa = 0; aa < na; ++aa)
              for (int kk = j; kk < GM_BK / 16; kk += C)   // K = 16: 8 TMEM columns of A, 32 bytes of each B row
                tc::umma_f16_ta(dcol, aT + aa * GM_ACOLS + kk * 8, tc::sdesc_k_sw128(bBase + aa * GM_BSLOT + kk * 32),
                                idesc, (jst > 0 || aa > 0 || kk > j) ? 1u : 0u);
          }
          tc::umma_commit(st_empty(slot));
        }
        __syncwarp();
      }
      if (ok && lane == 0) tc::umma_commit(acc_full(acc));
      __syncwarp();
    }
    // every MMA issued has completed before TMEM is freed
    if (lane == 0) tc::umma_commit(final_bar);
    __syncwarp();
    gm_wait_drain(final_bar, 0);
  } else if (warp >= GM_DQ_WARP0 && warp < GM_DQ_WARP0 + GM_DQ_WARPS) {
    // -------------------------------------------------------------- dequant
    const int dw = warp - GM_DQ_WARP0;
    const int grp = dw >> 3;                             // dequant group: atoms grp, grp + 2 of every stage
    const int r = 32 * (warp & 3) + lane;                // A row = this thread's TMEM lane
    const int h = (dw >> 2) & 1;                         // half h of the row's 8 code words
    // code-tile row of A row r: phase 0 gate row i at tile row i, up row i at 64 + i
    const int R = a.phase == 0 ? (r & 1) * 64 + (r >> 1) : r;
    const uint32_t sRaw_u = tc::smem_u32(sRaw);
    const uint32_t tA = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16) + static_cast<uint32_t>(2 * GM_NMAX + 16 * h);
    uint32_t ss = 0;                                     // stages (= raw slots) consumed
    int il = 0;
    bool ok = true;
    for (int rd = 0, item = gm_item_at(0, G); item < n_items && ok; item = gm_item_at(++rd, G), ++il) {
      const GmItem it = gm_item(a, n_sh, item);
      const int sb = il & 1;
      if (!(ok = gm_wait(sc_full(sb), (il >> 1) & 1, abort_flag))) break;
      const int Gq = it.nkb;
      const uint32_t reg = gm_region_bytes(a.phase, Gq);
      const uint32_t scb = tc::smem_u32(sSC + sb * GM_SC_BUF);
      uint32_t sS_u, sB_u;                                 // this row's scale and bias rows (bf16 per group)
      if (a.phase == 0) {
        const int m = r & 1, i = r >> 1;
        sS_u = scb + (2 * m) * reg + 2 * i * Gq;
        sB_u = scb + (2 * m + 1) * reg + 2 * i * Gq;
      } else {
        sS_u = scb + 2 * r * Gq;
        sB_u = scb + reg + 2 * r * Gq;
      }
      const int nst = (it.nkb + GM_APS - 1) / GM_APS;
      for (int jst = 0; jst < nst; ++jst, ++ss) {
        const int rslot = ss % GM_RS, slot = ss % GM_ST;
        if (!(ok = gm_wait(raw_full(rslot), (ss / GM_RS) & 1, abort_flag))) break;
        if (ss >= GM_ST && !(ok = gm_wait(st_empty(slot), ((ss / GM_ST) - 1) & 1, abort_flag))) break;
        const int na = min(GM_APS, it.nkb - GM_APS * jst);
        const uint32_t raw = sRaw_u + rslot * GM_RAW_SLOT;
        for (int aa = grp; aa < na; aa += GM_DQ_GROUPS) {
          const int kb = GM_APS * jst + aa;
          // this thread's 4 code words of the atom row (16 bytes at 32 aa + 16 h)
          const uint4 v = gm_lds128(raw + gm_sw128(R, 2 * aa + h));
          const float sf = bf16_to_f32(static_cast<uint16_t>(gm_lds_u16(sS_u + 2 * kb)));
          const float bf = bf16_to_f32(static_cast<uint16_t>(gm_lds_u16(sB_u + 2 * kb)));
          const __half2 s2 = __floats2half2_rn(sf, sf), b2 = __floats2half2_rn(bf, bf);
          uint32_t wv[16];
          const uint32_t qw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 o = gm_dequant_word(qw[q], s2, b2);
            wv[4 * q + 0] = o.x; wv[4 * q + 1] = o.y; wv[4 * q + 2] = o.z; wv[4 * q + 3] = o.w;
          }
          // 32 K values = 16 TMEM columns of this lane in the atom's A slot
          tc::tmem_st16(tA + static_cast<uint32_t>((slot * GM_APS + aa) * GM_ACOLS), wv);
        }
        tc::tmem_wait_st();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          tc::mbar_arrive(a_full(slot));
          tc::mbar_arrive(raw_empty(rslot));
        }
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(sc_empty(sb));
    }
  } else if (warp < 4 || warp >= GM_EPI_WARP1) {
    // ------------------------------------------------------------- epilogue
    const int wq = warp & 3;                        // TMEM sub-partition (lanes 32 wq ..)
    const int half = warp >= GM_EPI_WARP1 ? 1 : 0;  // which 16-column blocks: 2 b + half
    int il = 0;
    bool ok = true;
    for (int rd = 0, item = gm_item_at(0, G); item < n_items && ok; item = gm_item_at(++rd, G), ++il) {
      const GmItem it = gm_item(a, n_sh, item);
      const int acc = il & 1;
      ok = __all_sync(0xffffffffu, gm_wait(acc_full(acc), (il >> 1) & 1, abort_flag));
      if (!ok) break;
      tc::tc_fence_after();
      const int Np = (it.N + 15) & ~15;
      const int row = 32 * wq + lane;               // TMEM lane = A row
      const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * wq) << 16) + static_cast<uint32_t>(acc * GM_NMAX);
      const int C = gm_chains(Np);
      for (int nc = 16 * half; nc < Np; nc += 32) {
        float v[16];
        tc::tmem_ld16(taddr + nc, v);
        for (int c = 1; c < C; ++c) {        // add the item's other accumulator chains
          float w2[16];
          tc::tmem_ld16(taddr + static_cast<uint32_t>(c * (GM_NMAX / C)) + nc, w2);
#pragma unroll
          for (int q = 0; q < 16; ++q) v[q] += w2[q];
        }
        if (a.phase == 0) {
          const int Iw = it.seg ? a.I : a.Is;
          __half* out = it.seg ? a.act_r : a.act_s;
          const int i = 64 * it.mt + (row >> 1);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float u = __shfl_xor_sync(0xffffffffu, v[j], 1);
            const int n = nc + j;
            if ((lane & 1) == 0 && n < it.N)
              out[static_cast<size_t>(it.row0 + n) * Iw + gm_kpos(i)] = __float2half_rn(gelu_tanh(v[j]) * u);
          }
        } else {
          const int o = GM_BM * it.mt + row;
          // destination rows of the 16 columns: the pair value (routed) or the row (shared)
          int dst = -1;
          if (lane < 16 && nc + lane < it.N) {
            if (it.seg) {
              dst = a.pairs[it.row0 + nc + lane];
              if (dst < 0 || dst >= a.P) { flag_check(CHECK_PAIR_ID); dst = -1; }
            } else {
              dst = it.row0 + nc + lane;
            }
          }
          float* out = it.seg ? a.y_r : a.y_s;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int d = __shfl_sync(0xffffffffu, dst, j);
            if (d >= 0) out[static_cast<size_t>(d) * a.H + o] = v[j];
          }
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(acc_empty(acc));
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 0) tc::tmem_dealloc(tmem, GM_TMEM_COLS);
}

}  // namespace moe
