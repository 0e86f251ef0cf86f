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
//               256 K-values of 128 rows per ring slot as 2-D TMA tiles (a
//               routed expert's tensor maps are a template whose address
//               the warp patches per item into a small ring in global memory)
//   warp 5      B producer: per atom the bucket rows' fp16 activations as
//               one 2-D TMA tile (128-byte swizzle)
//   warp 6      MMA issuer: 4 x tcgen05.mma (M=128, N, K=16) per atom into
//               one of two TMEM accumulators (the epilogue of an item
//               overlaps the next item's MMAs)
//   warps 7-14  dequant: w = S q + B in half2 arithmetic (q exact, w rounded
//               once to fp16) from a raw slot into an A atom of the ring
// Every mbarrier wait is bounded; a wait that runs out sets the device check
// word and a CTA-wide abort flag, after which every role stops issuing work,
// the copies in flight are waited for (bounded) and TMEM is freed.
#include <cuda.h>   // CUtensorMap (the type only; tensor maps are encoded on the host)

#include "tc_utils.cuh"

namespace moe {

constexpr int GM_BM = 128;                   // weight rows per item (MMA M)
constexpr int GM_BK = 64;                    // K per atom
constexpr int GM_APR = 4;                    // atoms per raw slot
constexpr int GM_RAW_SLOT = GM_BM * 128;     // 128 rows x 128 B of codes (256 K values), 128-byte swizzle
constexpr int GM_RS = 4;                     // raw slots
constexpr int GM_AS = 3;                     // dequantised A atoms
constexpr int GM_BS = 3;                     // activation (B) tiles
constexpr int GM_NMAX = 128;                 // bucket rows per chunk (MMA N; TMEM columns per accumulator)
constexpr int GM_ATOM = 128 * 128;           // 16 KB: 128 rows x 128 B
constexpr int GM_MAX_G = 48;                 // quantisation groups per weight row (K <= 3072)
constexpr int GM_SC_BUF = 4 * (64 * GM_MAX_G * 2 + 16) + 64;   // scale/bias rows of one item (24,704 B)
static_assert(GM_SC_BUF % 128 == 0, "scale buffers keep the maps after them 128-byte aligned");
constexpr int GM_MAX_CHUNKS = 512;
constexpr int GM_MAX_CTAS = 160;             // grid cap (one CTA per SM)
// Per-CTA tensor-map sets (gate and up, or down) in global memory.  An
// item's set is patched after the wait that frees its first raw slot, which
// proves that every copy issued GM_RS slots before has landed; each item
// issues at least one slot, so a ring of more than GM_RS + 1 sets is never
// patched under a copy still in flight.
constexpr int GM_MAP_RING = 6;
static_assert(GM_MAP_RING > GM_RS + 1, "tensor-map ring vs raw ring");
constexpr int GM_EPI_WARPS = 4, GM_RAW_WARP = 4, GM_B_WARP = 5, GM_MMA_WARP = 6, GM_DQ_WARP0 = 7, GM_DQ_WARPS = 8;
constexpr int GM_THREADS = (GM_DQ_WARP0 + GM_DQ_WARPS) * 32;
// barriers: raw full/empty [RS], a full/empty [AS], b full/empty [BS], sc full/empty [2], acc full/empty [2], final
constexpr int GM_NBARS = 2 * GM_RS + 2 * GM_AS + 2 * GM_BS + 4 + 4 + 1;
constexpr size_t GM_SMEM = 1024 + static_cast<size_t>(GM_AS) * GM_ATOM + static_cast<size_t>(GM_BS) * GM_ATOM +
                           static_cast<size_t>(GM_RS) * GM_RAW_SLOT + 2 * GM_SC_BUF + 256 + GM_NBARS * 8 + 64;
static_assert(GM_SC_BUF % 128 == 0 && GM_RAW_SLOT % 1024 == 0, "copy destinations: swizzle atoms 1024-byte, maps 128-byte aligned");
static_assert(GM_SMEM <= 232448, "shared memory of the grouped GEMM");

// Box heights of the activation tensor maps (rows of the TMA tile).
constexpr int GM_NBOX = 4;
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

// 8 nibbles of one word -> 8 fp16 weights S*q + B in element order.  Each
// nibble becomes the fp16 1024 + q (or 1024 + 16 q) by OR-ing it into the
// exponent pattern 0x6400, minus 1024 (exact); then one fma rounds S*q + B.
__device__ __forceinline__ uint4 gm_dequant_word(uint32_t w, __half2 s2, __half2 b2) {
  const __half2 k1024 = __floats2half2_rn(1024.f, 1024.f);
  const __half2 k16 = __floats2half2_rn(0.0625f, 0.0625f);
  const __half2 k64 = __floats2half2_rn(-64.f, -64.f);
  const uint32_t w8 = w >> 8;
  const __half2 q04 = __hsub2(gm_h2((w & 0x000F000Fu) | 0x64006400u), k1024);    // q0, q4
  const __half2 q15 = __hfma2(gm_h2((w & 0x00F000F0u) | 0x64006400u), k16, k64);  // q1, q5
  const __half2 q26 = __hsub2(gm_h2((w8 & 0x000F000Fu) | 0x64006400u), k1024);   // q2, q6
  const __half2 q37 = __hfma2(gm_h2((w8 & 0x00F000F0u) | 0x64006400u), k16, k64); // q3, q7
  const uint32_t a = gm_u32(__hfma2(q04, s2, b2)), b = gm_u32(__hfma2(q15, s2, b2));
  const uint32_t c = gm_u32(__hfma2(q26, s2, b2)), d = gm_u32(__hfma2(q37, s2, b2));
  uint4 o;
  o.x = __byte_perm(a, b, 0x5410);   // w0 w1
  o.y = __byte_perm(c, d, 0x5410);   // w2 w3
  o.z = __byte_perm(a, b, 0x7632);   // w4 w5
  o.w = __byte_perm(c, d, 0x7632);   // w6 w7
  return o;
}

// ------------------------------------------------------------------ prep
// Block 0 writes the chunk list (shared chunks first, then the routed
// buckets in active order, each cut into chunks of at most GM_NMAX rows);
// every block gathers the layer input into bucket order as fp16
// (xs[pos] = x[pairs[pos] / k]) and, when xh is given, writes x as fp16.
__global__ void __launch_bounds__(256) k_gm_prep(const uint16_t* __restrict__ x, int T, int H, int k,
                                                 const int32_t* __restrict__ offsets,
                                                 const int32_t* __restrict__ pairs,
                                                 const int32_t* __restrict__ active,
                                                 const int32_t* __restrict__ n_active, int E, int routed,
                                                 int shared_rows, __half* __restrict__ xs, __half* __restrict__ xh,
                                                 GmPlan* __restrict__ plan) {
  if (blockIdx.x == 0) {
    const int nsh = (shared_rows + GM_NMAX - 1) / GM_NMAX;
    for (int c = threadIdx.x; c < nsh; c += blockDim.x) {
      const int n0 = c * GM_NMAX, n = min(GM_NMAX, shared_rows - n0);
      plan->chunk[c] = make_uint2(0u, static_cast<uint32_t>(n0) | (static_cast<uint32_t>(n) << 24));
    }
    int na = routed ? *n_active : 0;
    if (na < 0 || na > E) { if (threadIdx.x == 0) flag_check(CHECK_EXPERT_ID); na = 0; }
    // one warp: 32 experts per round, chunk counts scanned across the warp
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      int base = nsh;
      for (int a0 = 0; a0 < na; a0 += 32) {
        const int a = a0 + lane;
        int e = 0, pos0 = 0, cnt = 0;
        if (a < na) {
          e = active[a];
          if (e < 0 || e >= E) { flag_check(CHECK_EXPERT_ID); e = 0; }
          else { pos0 = offsets[e]; cnt = offsets[e + 1] - pos0; }
          if (cnt < 0) cnt = 0;
        }
        const int nch = (cnt + GM_NMAX - 1) / GM_NMAX;
        int incl = nch;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        const int total = __shfl_sync(0xffffffffu, incl, 31);
        for (int c = 0; c < nch; ++c) {
          const int slot = base + incl - nch + c;
          if (slot < GM_MAX_CHUNKS) {
            const int n0 = c * GM_NMAX, n = min(GM_NMAX, cnt - n0);
            plan->chunk[slot] = make_uint2(static_cast<uint32_t>(e) | 0x80000000u,
                                           static_cast<uint32_t>(pos0 + n0) | (static_cast<uint32_t>(n) << 24));
          }
        }
        base += total;
      }
      if (lane == 0) {
        int nr = base - nsh;
        if (base > GM_MAX_CHUNKS) { flag_check(CHECK_PAIR_ID); nr = GM_MAX_CHUNKS - nsh; }
        plan->n_chunks[0] = nsh;
        plan->n_chunks[1] = nr;
      }
    }
  }
  // gather: 8 values (16 bytes) per thread and step
  const int w8 = H / 8;
  const long P = routed ? static_cast<long>(T) * k : 0;
  const long nxs = P * w8, nxh = xh ? static_cast<long>(T) * w8 : 0;
  for (long i = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; i < nxs + nxh;
       i += static_cast<long>(gridDim.x) * blockDim.x) {
    long row, w;
    int t;
    __half* dst;
    if (i < nxs) {
      row = i / w8; w = i - row * w8;
      const int p = pairs[row];
      t = p / k;
      if (p < 0 || t >= T) { flag_check(CHECK_PAIR_ID); t = -1; }
      dst = xs + row * H + 8 * w;
    } else {
      const long j = i - nxs;
      row = j / w8; w = j - row * w8;
      t = static_cast<int>(row);
      dst = xh + row * H + 8 * w;
    }
    uint4 o = make_uint4(0u, 0u, 0u, 0u);
    if (t >= 0) {
      const uint4 u = *reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * H + 8 * w);
      o.x = pack_half2(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u));
      o.y = pack_half2(__uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u));
      o.z = pack_half2(__uint_as_float(u.z << 16), __uint_as_float(u.z & 0xFFFF0000u));
      o.w = pack_half2(__uint_as_float(u.w << 16), __uint_as_float(u.w & 0xFFFF0000u));
    }
    *reinterpret_cast<uint4*>(dst) = o;
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

// Bounded mbarrier wait that also gives up when another role of the CTA
// has aborted (abort flag in shared memory).
__device__ __forceinline__ bool gm_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  uint64_t t0 = 0;
  for (uint32_t i = 0;; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    if (ok) return true;
    if ((i & 63u) == 0) {
      if (*abort_flag) return false;
      const uint64_t now = tc::globaltimer_ns();
      if (t0 == 0) t0 = now;
      else if (now - t0 > 2000000000ull) break;
    }
  }
  flag_check(CHECK_WAIT);
  *abort_flag = 1;
  return false;
}

// Bounded wait that ignores the abort flag (used on the way out, for copies
// already in flight and the last MMAs).
__device__ __forceinline__ void gm_wait_drain(uint32_t bar, uint32_t parity) {
  uint64_t t0 = 0;
  for (uint32_t i = 0;; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    if (ok) return;
    if ((i & 63u) == 0) {
      const uint64_t now = tc::globaltimer_ns();
      if (t0 == 0) t0 = now;
      else if (now - t0 > 2000000000ull) { flag_check(CHECK_WAIT); return; }
    }
  }
}

// ------------------------------------------------------------------ kernel
__global__ void __launch_bounds__(GM_THREADS, 1) k_moe_gemm(const __grid_constant__ GemmArgs a) {
  extern __shared__ __align__(1024) unsigned char gm_smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(gm_smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sA = smem;                                      // [AS][16 KB], 1024-aligned
  unsigned char* sB = sA + GM_AS * GM_ATOM;                      // [BS][16 KB], 1024-aligned
  unsigned char* sRaw = sB + GM_BS * GM_ATOM;                    // [RS][128 rows x 128 B], swizzled
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
  auto a_empty = [&](int s) { return bar0 + 8u * (2 * GM_RS + GM_AS + s); };
  auto b_full = [&](int s) { return bar0 + 8u * (2 * GM_RS + 2 * GM_AS + s); };
  auto b_empty = [&](int s) { return bar0 + 8u * (2 * GM_RS + 2 * GM_AS + GM_BS + s); };
  const uint32_t barx = bar0 + 8u * (2 * GM_RS + 2 * GM_AS + 2 * GM_BS);
  auto sc_full = [&](int s) { return barx + 8u * s; };
  auto sc_empty = [&](int s) { return barx + 8u * (2 + s); };
  auto acc_full = [&](int s) { return barx + 8u * (4 + s); };
  auto acc_empty = [&](int s) { return barx + 8u * (6 + s); };
  const uint32_t final_bar = barx + 8u * 8;

  if (threadIdx.x == 0) {
    for (int s = 0; s < GM_RS; ++s) { tc::mbar_init(raw_full(s), 1); tc::mbar_init(raw_empty(s), GM_DQ_WARPS); }
    for (int s = 0; s < GM_AS; ++s) { tc::mbar_init(a_full(s), GM_DQ_WARPS); tc::mbar_init(a_empty(s), 1); }
    for (int s = 0; s < GM_BS; ++s) { tc::mbar_init(b_full(s), 1); tc::mbar_init(b_empty(s), 1); }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(sc_full(s), 1);
      tc::mbar_init(sc_empty(s), GM_DQ_WARPS);
      tc::mbar_init(acc_full(s), 1);
      tc::mbar_init(acc_empty(s), GM_EPI_WARPS);
    }
    tc::mbar_init(final_bar, 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), 2 * GM_NMAX);
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
    for (int item = blockIdx.x; item < n_items && ok; item += G, ++il) {
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
      const int nraw = (it.nkb + GM_APR - 1) / GM_APR;
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
    uint32_t bs = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < n_items && ok; item += G) {
      const GmItem it = gm_item(a, n_sh, item);
      const int Np = (it.N + 15) & ~15;
      int bi = 0;
      while (bi < GM_NBOX - 1 && gm_box_rows(bi) < Np) ++bi;
      const uint32_t bbytes = static_cast<uint32_t>(gm_box_rows(bi)) * 128u;
      const CUtensorMap* tm = &a.tmB[it.seg][bi];
      for (int kb = 0; kb < it.nkb; ++kb, ++bs) {
        const int slot = bs % GM_BS;
        if (bs >= GM_BS && !(ok = gm_wait(b_empty(slot), ((bs / GM_BS) - 1) & 1, abort_flag))) break;
        if (lane == 0) {
          tc::mbar_arrive_tx(b_full(slot), bbytes);
          tc::tma_load_2d(tc::smem_u32(sB + slot * GM_ATOM), tm, kb * GM_BK, it.row0, b_full(slot));
        }
        __syncwarp();
      }
    }
    for (uint32_t q = bs > GM_BS ? bs - GM_BS : 0; q < bs; ++q) gm_wait_drain(b_full(q % GM_BS), (q / GM_BS) & 1);
  } else if (warp == GM_MMA_WARP) {
    // ----------------------------------------------------------- MMA issuer
    uint32_t as = 0;
    int il = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < n_items && ok; item += G, ++il) {
      const GmItem it = gm_item(a, n_sh, item);
      const int acc = il & 1;
      if (il >= 2 && !(ok = gm_wait(acc_empty(acc), ((il >> 1) - 1) & 1, abort_flag))) break;
      tc::tc_fence_after();
      const int Np = (it.N + 15) & ~15;
      const uint32_t idesc = tc::idesc_f16_f32(GM_BM, Np);
      const uint32_t dcol = tmem + static_cast<uint32_t>(acc * GM_NMAX);
      for (int kb = 0; kb < it.nkb; ++kb, ++as) {
        const int sa = as % GM_AS, sbb = as % GM_BS;
        if (!(ok = gm_wait(a_full(sa), (as / GM_AS) & 1, abort_flag))) break;
        if (!(ok = gm_wait(b_full(sbb), (as / GM_BS) & 1, abort_flag))) break;
        tc::tc_fence_after();
        if (lane == 0) {
          const uint32_t aBase = tc::smem_u32(sA + sa * GM_ATOM);
          const uint32_t bBase = tc::smem_u32(sB + sbb * GM_ATOM);
#pragma unroll
          for (int kk = 0; kk < GM_BK / 16; ++kk)
            tc::umma_f16(dcol, tc::sdesc_k_sw128(aBase + kk * 32), tc::sdesc_k_sw128(bBase + kk * 32), idesc,
                         (kb > 0 || kk > 0) ? 1u : 0u);
          tc::umma_commit(a_empty(sa));
          tc::umma_commit(b_empty(sbb));
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
  } else if (warp >= GM_DQ_WARP0) {
    // -------------------------------------------------------------- dequant
    const int t = threadIdx.x - GM_DQ_WARP0 * 32;      // 0..255
    const int r = t >> 1, h = t & 1;                     // A row, half of the atom's 64 K values
    // code-tile row of A row r: phase 0 gate row i at tile row i, up row i at 64 + i
    const int R = a.phase == 0 ? (r & 1) * 64 + (r >> 1) : r;
    uint32_t rs = 0, as = 0;
    int il = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < n_items && ok; item += G, ++il) {
      const GmItem it = gm_item(a, n_sh, item);
      const int sb = il & 1;
      if (!(ok = gm_wait(sc_full(sb), (il >> 1) & 1, abort_flag))) break;
      const int Gq = it.nkb;
      const uint32_t reg = gm_region_bytes(a.phase, Gq);
      const unsigned char* scb = sSC + sb * GM_SC_BUF;
      const uint16_t *sS, *sBv;
      if (a.phase == 0) {
        const int m = r & 1, i = r >> 1;
        sS = reinterpret_cast<const uint16_t*>(scb + (2 * m) * reg) + i * Gq;
        sBv = reinterpret_cast<const uint16_t*>(scb + (2 * m + 1) * reg) + i * Gq;
      } else {
        sS = reinterpret_cast<const uint16_t*>(scb) + r * Gq;
        sBv = reinterpret_cast<const uint16_t*>(scb + reg) + r * Gq;
      }
      for (int kb = 0; kb < it.nkb; ++kb, ++as) {
        const int aa = kb % GM_APR;
        if (aa == 0 && !(ok = gm_wait(raw_full(rs % GM_RS), (rs / GM_RS) & 1, abort_flag))) break;
        const int sa = as % GM_AS;
        if (as >= GM_AS && !(ok = gm_wait(a_empty(sa), ((as / GM_AS) - 1) & 1, abort_flag))) break;
        const uint4 qq = *reinterpret_cast<const uint4*>(sRaw + (rs % GM_RS) * GM_RAW_SLOT +
                                                         gm_sw128(R, 2 * aa + h));
        const float sf = bf16_to_f32(sS[kb]), bf = bf16_to_f32(sBv[kb]);
        const __half2 s2 = __floats2half2_rn(sf, sf), b2 = __floats2half2_rn(bf, bf);
        unsigned char* atom = sA + sa * GM_ATOM;
        *reinterpret_cast<uint4*>(atom + gm_sw128(r, 4 * h + 0)) = gm_dequant_word(qq.x, s2, b2);
        *reinterpret_cast<uint4*>(atom + gm_sw128(r, 4 * h + 1)) = gm_dequant_word(qq.y, s2, b2);
        *reinterpret_cast<uint4*>(atom + gm_sw128(r, 4 * h + 2)) = gm_dequant_word(qq.z, s2, b2);
        *reinterpret_cast<uint4*>(atom + gm_sw128(r, 4 * h + 3)) = gm_dequant_word(qq.w, s2, b2);
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(a_full(sa));
        if (aa == GM_APR - 1 || kb == it.nkb - 1) {
          if (lane == 0) tc::mbar_arrive(raw_empty(rs % GM_RS));
          ++rs;
        }
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(sc_empty(sb));
    }
  } else if (warp < GM_EPI_WARPS) {
    // ------------------------------------------------------------- epilogue
    int il = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < n_items && ok; item += G, ++il) {
      const GmItem it = gm_item(a, n_sh, item);
      const int acc = il & 1;
      ok = __all_sync(0xffffffffu, gm_wait(acc_full(acc), (il >> 1) & 1, abort_flag));
      if (!ok) break;
      tc::tc_fence_after();
      const int Np = (it.N + 15) & ~15;
      const int row = 32 * warp + lane;             // TMEM lane = A row
      const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * warp) << 16) + static_cast<uint32_t>(acc * GM_NMAX);
      for (int nc = 0; nc < Np; nc += 16) {
        float v[16];
        tc::tmem_ld16(taddr + nc, v);
        if (a.phase == 0) {
          const int Iw = it.seg ? a.I : a.Is;
          __half* out = it.seg ? a.act_r : a.act_s;
          const int i = 64 * it.mt + (row >> 1);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float u = __shfl_xor_sync(0xffffffffu, v[j], 1);
            const int n = nc + j;
            if ((lane & 1) == 0 && n < it.N)
              out[static_cast<size_t>(it.row0 + n) * Iw + i] = __float2half_rn(gelu_tanh(v[j]) * u);
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
  if (warp == 0) tc::tmem_dealloc(tmem, 2 * GM_NMAX);
}

}  // namespace moe
