// Batch-1 decode of a stack of routed-MoE layers in one persistent kernel.
//
// One launch runs every layer of the step.  The grid is a set of 8-CTA
// clusters, one CTA per SM, launched cooperatively (all CTAs resident).  Each
// CTA has one loader warp and DF_CW compute warps.
//
// Work of one layer, split statically over the G CTAs (CTA c, cluster rank r):
//   R   router rows [r*E/8, (r+1)*E/8)
//   SG  shared-expert gate/up row pairs [c*Is/G, (c+1)*Is/G)
//   RG  routed gate/up (slot, row) pairs [c*k*I/G, (c+1)*k*I/G) of the k*I list
//   D   output rows [c*H/G, (c+1)*H/G): per routed slot its down rows, then
//       the shared expert's down rows (DS)
// Each part is cut into jobs that fit one ring slot.  The loader warp walks
// the job list in order and copies each job's bytes (weight rows and the
// 16-byte-aligned windows of their scales and biases) into the next slot of a
// shared-memory ring with 1-D bulk copies (cp.async.bulk) that complete on
// the slot's mbarrier; it waits only for a free slot and, before the routed
// jobs of a layer, for that layer's routing.  The compute warps take the jobs
// round-robin (job q -> warp q % DF_CW) and read only shared memory:
//   rms norm of h (every CTA, same order, same result)
//   R jobs -> logits, broadcast to the 8 CTAs of the cluster with remote
//     shared-memory stores and remote mbarrier arrivals; every CTA selects
//     the top k itself, so routing needs no grid-wide step, and hands it to
//     its loader
//   SG, RG jobs -> fp16 activations act = gelu_tanh(gate) * up (global)
//   grid barrier (compute warps: named barrier, cluster mbarriers, one
//     atomic per cluster)
//   all activations staged in shared memory; D, DS jobs -> per-row dots;
//     y = sum_j g_j y_j + ysh in a fixed order; h += y
//   grid barrier
// HBM is kept busy with bulk L2 prefetches: when a layer's routing is known
// the loader prefetches all of its routed rows; when it starts a layer it
// prefetches the next layer's routing-independent rows and slices of the
// experts with the largest router bias (the likeliest choices).
// Every wait is bounded (about two seconds); a wait that runs out sets the
// device check word and the thread runs on to the end.
#include <cooperative_groups.h>

namespace moe {

constexpr int DF_CW = 15;                       // compute warps
constexpr int DF_THREADS = (DF_CW + 1) * 32;    // + loader warp (warp DF_CW)
constexpr int DF_CLUSTER = 8;
constexpr int DF_MAX_LAYERS = 48;
constexpr int DF_MAX_H = 3072;
constexpr int DF_CPL = 3;                       // uint4 chunks per lane of a gate/up row (H <= 3072)
constexpr int DF_MAX_ACT = 8192;                // k*I + Is
constexpr int DF_MAX_ROWS = 32;                 // output rows per CTA
constexpr int DF_NS = 16;                       // ring slots
constexpr int DF_SLOT_Q = 8192;                 // weight bytes per slot
constexpr int DF_SLOT_S = 1024;                 // scale/bias window bytes per slot
constexpr int DF_SLOT = DF_SLOT_Q + DF_SLOT_S;
constexpr int DF_MAX_E = 256;
constexpr int DF_MAX_JOBS = 80;                 // jobs per layer per CTA

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
  unsigned* counter;                // workspace: grid barrier counter (zeroed before launch)
  uint16_t* x_trace; uint16_t* y_trace; int32_t* idx_trace; float* gates_trace;
  int spec;                         // experts speculatively prefetched per layer
  int prefetch;                     // bit 0: routed rows into L2 once routed; bit 1: independent rows
  int rg_rows, d_rows, ds_rows;     // row pairs per SG/RG job, rows per D / DS job
  unsigned long long* stamps;       // optional phase timestamps [L][G][8] (ns), or null
  DfLayer layer[DF_MAX_LAYERS];
};

// ------------------------------------------------------------------ PTX bits
__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_gpu(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
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
__device__ __forceinline__ void df_mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(bar),
               "r"(bytes)
               : "memory");
}
// arrive on the mbarrier at the same shared-memory offset in CTA `rank` of the cluster
__device__ __forceinline__ void df_mbar_arrive_remote(uint32_t bar, uint32_t rank) {
  asm volatile(
      "{\n\t.reg .b32 ra;\n\tmapa.shared::cluster.u32 ra, %0, %1;\n\t"
      "mbarrier.arrive.release.cluster.shared::cluster.b64 _, [ra];\n\t}" ::"r"(bar),
      "r"(rank)
      : "memory");
}
__device__ __forceinline__ void df_st_remote_f32(uint32_t addr, uint32_t rank, float v) {
  asm volatile(
      "{\n\t.reg .b32 ra;\n\tmapa.shared::cluster.u32 ra, %0, %1;\n\tst.shared::cluster.f32 [ra], %2;\n\t}" ::"r"(
          addr),
      "r"(rank), "f"(v)
      : "memory");
}
// bounded wait on a phase parity; `cluster` acquires at cluster scope
__device__ __forceinline__ bool df_mbar_wait(uint32_t bar, uint32_t parity, bool cluster = false) {
  uint64_t t0 = 0;
  for (uint32_t i = 0;; ++i) {
    uint32_t ok;
    if (cluster)
      asm volatile(
          "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
          "selp.u32 %0, 1, 0, p;\n\t}"
          : "=r"(ok)
          : "r"(bar), "r"(parity)
          : "memory");
    else
      asm volatile(
          "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
          "selp.u32 %0, 1, 0, p;\n\t}"
          : "=r"(ok)
          : "r"(bar), "r"(parity)
          : "memory");
    if (ok) return true;
    if ((i & 255u) == 0) {
      const uint64_t now = df_clock();
      if (t0 == 0) t0 = now;
      else if (now - t0 > 2000000000ull) break;
    }
  }
  flag_check(CHECK_WAIT);
  return false;
}
__device__ __forceinline__ void df_bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}
// L2 prefetch of the 16-byte-aligned window around [p, p + bytes).  Arrays
// handed to this kernel are 16-byte aligned with sizes that are multiples of
// 16, so the window stays inside them.
__device__ __forceinline__ void prefetch_l2(const void* p, size_t bytes) {
  if (bytes == 0) return;
  uintptr_t a = reinterpret_cast<uintptr_t>(p) & ~uintptr_t(15);
  const uintptr_t e = (reinterpret_cast<uintptr_t>(p) + bytes + 15) & ~uintptr_t(15);
  while (a < e) {
    const uint32_t n = static_cast<uint32_t>((e - a) < 65536 ? (e - a) : 65536);
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a), "r"(n) : "memory");
    a += n;
  }
}
__device__ __forceinline__ void prefetch_slice(const void* base, size_t total, int c, int G) {
  const size_t b0 = total * c / G, b1 = total * (c + 1) / G;
  prefetch_l2(static_cast<const uint8_t*>(base) + b0, b1 - b0);
}
__device__ __forceinline__ uint4 ldcg_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}
__device__ __forceinline__ void df_named_sync() {   // the compute warps of this CTA
  asm volatile("bar.sync 1, %0;" ::"n"(DF_CW * 32) : "memory");
}

// phase timestamps (when requested): layer l, CTA c, phase p
__device__ __forceinline__ void df_stamp(const DfArgs& a, int l, int p) {
  if (a.stamps != nullptr && threadIdx.x == 0)
    a.stamps[(static_cast<size_t>(l) * gridDim.x + blockIdx.x) * 8 + p] = df_clock();
}

// ---------------------------------------------------------------- job list
enum : int { JOB_R = 0, JOB_SG = 1, JOB_RG = 2, JOB_D = 3, JOB_DS = 4 };

struct DfJob {
  int kind;
  int slot;      // routed slot (RG, D)
  int r0, n;     // first row (or row pair) and count
};

struct DfShape {
  int H, I, Is, E, k, G, c, rank;
  int epc, s0, s1, r0, r1, o0, o1;
  int rgn, dn, dsn;
  int nR, nSG, nRG, nD, nDS;
};

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

__device__ inline int df_rg_jobs(const DfShape& s) {
  if (s.r1 <= s.r0) return 0;
  int n = 0;
  for (int j = s.r0 / s.I; j <= (s.r1 - 1) / s.I; ++j) {
    const int a = max(s.r0, j * s.I), b = min(s.r1, (j + 1) * s.I);
    n += ceil_div(b - a, s.rgn);
  }
  return n;
}

__device__ inline DfJob df_job(const DfShape& s, int q) {
  DfJob J{};
  if (q < s.nR) {
    J.kind = JOB_R; J.r0 = s.rank * s.epc + q * 2; J.n = min(2, s.epc - q * 2);
    return J;
  }
  q -= s.nR;
  if (q < s.nSG) {
    J.kind = JOB_SG; J.r0 = s.s0 + q * s.rgn; J.n = min(s.rgn, s.s1 - J.r0);
    return J;
  }
  q -= s.nSG;
  if (q < s.nRG) {
    for (int j = s.r0 / s.I; j <= (s.r1 - 1) / s.I; ++j) {
      const int a = max(s.r0, j * s.I), b = min(s.r1, (j + 1) * s.I);
      const int nj = ceil_div(b - a, s.rgn);
      if (q < nj) {
        J.kind = JOB_RG; J.slot = j; J.r0 = a - j * s.I + q * s.rgn; J.n = min(s.rgn, b - a - q * s.rgn);
        return J;
      }
      q -= nj;
    }
  }
  q -= s.nRG;
  if (q < s.nD) {
    const int per = ceil_div(s.o1 - s.o0, s.dn);
    J.kind = JOB_D; J.slot = q / per; J.r0 = s.o0 + (q % per) * s.dn; J.n = min(s.dn, s.o1 - J.r0);
    return J;
  }
  q -= s.nD;
  J.kind = JOB_DS; J.r0 = s.o0 + q * s.dsn; J.n = min(s.dsn, s.o1 - J.r0);
  return J;
}

// 16-byte-aligned window covering rows [r0, r0+n) of a bf16 array with `per`
// values per row; skew = offset of row r0 inside the window.
__device__ __forceinline__ void sb_window(const uint16_t* base, int per, int r0, int n, const uint8_t*& src,
                                          uint32_t& bytes, uint32_t& skew) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(base) + static_cast<size_t>(r0) * per * 2;
  const uintptr_t e = a + static_cast<size_t>(n) * per * 2;
  const uintptr_t a16 = a & ~uintptr_t(15), e16 = (e + 15) & ~uintptr_t(15);
  src = reinterpret_cast<const uint8_t*>(a16);
  bytes = static_cast<uint32_t>(e16 - a16);
  skew = static_cast<uint32_t>(a - a16);
}

// The copies of one job: weight runs at the start of the slot (run i at
// i * qbytes), then the scale/bias windows in the slot's scale area; sk[i]
// is the offset of window i's first row inside that area.
struct DfJobCopies {
  const uint8_t* src[6];
  uint32_t dst[6];
  uint32_t len[6];
  int n;
  uint32_t qbytes;
  uint32_t sk[4];
  uint32_t bytes;
  int kind, slot, r0, rows;       // the job itself
};

__device__ inline DfJobCopies df_job_copies(const DfShape& s, const DfJob& J, const DfArgs& a, const DfLayer& W,
                                            const int* sel) {
  DfJobCopies C{};
  const int H = s.H, I = s.I, Is = s.Is;
  const uint8_t* q[2] = {nullptr, nullptr};
  const uint16_t* sc[4] = {nullptr, nullptr, nullptr, nullptr};
  int per = 0, nq = 0, ns = 0;
  if (J.kind == JOB_R) {
    q[0] = reinterpret_cast<const uint8_t*>(W.rq) + static_cast<size_t>(J.r0) * H;
    C.qbytes = static_cast<uint32_t>(J.n) * H; nq = 1;
    sc[0] = W.rs; sc[1] = W.rb; ns = 2; per = H / 64;
  } else if (J.kind == JOB_SG || J.kind == JOB_RG) {
    const uint8_t *gq, *uq;
    const uint16_t *gs, *gb, *us, *ub;
    if (J.kind == JOB_SG) {
      gq = reinterpret_cast<const uint8_t*>(W.sq[0]); uq = reinterpret_cast<const uint8_t*>(W.sq[1]);
      gs = W.ss[0]; gb = W.sb[0]; us = W.ss[1]; ub = W.sb[1];
    } else {
      const uint8_t* blob = static_cast<const uint8_t*>(W.blobs[sel[J.slot]]);
      gq = blob + a.off[0]; uq = blob + a.off[3];
      gs = reinterpret_cast<const uint16_t*>(blob + a.off[1]); gb = reinterpret_cast<const uint16_t*>(blob + a.off[2]);
      us = reinterpret_cast<const uint16_t*>(blob + a.off[4]); ub = reinterpret_cast<const uint16_t*>(blob + a.off[5]);
    }
    q[0] = gq + static_cast<size_t>(J.r0) * (H / 2);
    q[1] = uq + static_cast<size_t>(J.r0) * (H / 2);
    C.qbytes = static_cast<uint32_t>(J.n) * (H / 2); nq = 2;
    sc[0] = gs; sc[1] = gb; sc[2] = us; sc[3] = ub; ns = 4; per = H / 64;
  } else if (J.kind == JOB_D) {
    const uint8_t* blob = static_cast<const uint8_t*>(W.blobs[sel[J.slot]]);
    q[0] = blob + a.off[6] + static_cast<size_t>(J.r0) * (I / 2);
    C.qbytes = static_cast<uint32_t>(J.n) * (I / 2); nq = 1;
    sc[0] = reinterpret_cast<const uint16_t*>(blob + a.off[7]);
    sc[1] = reinterpret_cast<const uint16_t*>(blob + a.off[8]);
    ns = 2; per = I / 64;
  } else {
    q[0] = reinterpret_cast<const uint8_t*>(W.sq[2]) + static_cast<size_t>(J.r0) * (Is / 2);
    C.qbytes = static_cast<uint32_t>(J.n) * (Is / 2); nq = 1;
    sc[0] = W.ss[2]; sc[1] = W.sb[2]; ns = 2; per = Is / 64;
  }
  uint32_t total = 0;
  for (int i = 0; i < nq; ++i) {
    C.src[C.n] = q[i]; C.dst[C.n] = static_cast<uint32_t>(i) * C.qbytes; C.len[C.n] = C.qbytes; ++C.n;
    total += C.qbytes;
  }
  uint32_t so = 0;
  for (int i = 0; i < ns; ++i) {
    const uint8_t* src; uint32_t bytes, skew;
    sb_window(sc[i], per, J.r0, J.n, src, bytes, skew);
    C.src[C.n] = src; C.dst[C.n] = DF_SLOT_Q + so; C.len[C.n] = bytes; ++C.n;
    C.sk[i] = so + skew;
    so += bytes;
    total += bytes;
  }
  C.bytes = total;
  C.kind = J.kind; C.slot = J.slot; C.r0 = J.r0; C.rows = J.n;
  return C;
}

// --------------------------------------------------------------- the kernel
__global__ void __cluster_dims__(DF_CLUSTER, 1, 1) __launch_bounds__(DF_THREADS, 1)
k_decode_b1(const __grid_constant__ DfArgs a) {
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  extern __shared__ __align__(128) unsigned char smem[];
  DfShape s;
  s.H = a.H; s.I = a.I; s.Is = a.Is; s.E = a.E; s.k = a.k;
  s.G = gridDim.x; s.c = blockIdx.x; s.rank = static_cast<int>(cl.block_rank());
  s.epc = s.E / DF_CLUSTER;
  const int kI = s.k * s.I, nact = kI + s.Is;
  s.s0 = (int)((long)s.c * s.Is / s.G); s.s1 = (int)((long)(s.c + 1) * s.Is / s.G);
  s.r0 = (int)((long)s.c * kI / s.G); s.r1 = (int)((long)(s.c + 1) * kI / s.G);
  s.o0 = (int)((long)s.c * s.H / s.G); s.o1 = (int)((long)(s.c + 1) * s.H / s.G);
  s.rgn = a.rg_rows; s.dn = a.d_rows; s.dsn = a.ds_rows;
  s.nR = ceil_div(s.epc, 2);
  s.nSG = ceil_div(s.s1 - s.s0, s.rgn);
  s.nRG = df_rg_jobs(s);
  s.nD = s.k * ceil_div(s.o1 - s.o0, s.dn);
  s.nDS = ceil_div(s.o1 - s.o0, s.dsn);
  const int njobs = s.nR + s.nSG + s.nRG + s.nD + s.nDS;
  const int nhead = s.nR + s.nSG;            // jobs that do not depend on the routing
  const int H = s.H, I = s.I, Is = s.Is, E = s.E, k = s.k;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nch = H / 32, nch16 = H / 16;

  // shared memory
  unsigned char* ring = smem;                                          // [NS][DF_SLOT]
  DfJobCopies* tab = reinterpret_cast<DfJobCopies*>(ring + DF_NS * DF_SLOT);   // [2][MAX_JOBS]
  float* xs = reinterpret_cast<float*>(tab + 2 * DF_MAX_JOBS);         // [H] layer input (bf16 values)
  uint4* xP4 = reinterpret_cast<uint4*>(xs + DF_MAX_H);                // [4][nch] nibble-paired x
  float2* xS4 = reinterpret_cast<float2*>(xP4 + DF_MAX_H / 8);         // [nch] (off, sum)
  uint2* xP8 = reinterpret_cast<uint2*>(xS4 + DF_MAX_H / 32);          // [4][nch16] byte-paired x
  float* xS8 = reinterpret_cast<float*>(xP8 + DF_MAX_H / 4);           // [nch16] sum
  uint4* actP = reinterpret_cast<uint4*>(xS8 + DF_MAX_H / 16);         // [nact/8] paired activations
  float2* actS = reinterpret_cast<float2*>(actP + DF_MAX_ACT / 8);     // [nact/8] (off, sum) per word
  float* part = reinterpret_cast<float*>(actS + DF_MAX_ACT / 8);       // [MAX_ROWS][9]
  float* lg_all = part + DF_MAX_ROWS * 9;                              // [E]
  float* red = lg_all + DF_MAX_E;                                      // [32]
  int* sel = reinterpret_cast<int*>(red + 32);                         // [2][8]
  float* selg = reinterpret_cast<float*>(sel + 16);                    // [8]
  uint64_t* bars = reinterpret_cast<uint64_t*>(selg + 8);
  const uint32_t bar0 = smem_addr(bars);
  auto full_bar = [&](int i) { return bar0 + 8u * i; };
  auto empty_bar = [&](int i) { return bar0 + 8u * (DF_NS + i); };
  const uint32_t route_bar = bar0 + 8u * (2 * DF_NS);
  const uint32_t lg_bar = route_bar + 8u;
  const uint32_t clA_bar = route_bar + 16u;     // in rank 0: all CTAs of the cluster arrived
  const uint32_t clR_bar = route_bar + 24u;     // every CTA: released

  if (threadIdx.x == 0) {
    for (int i = 0; i < DF_NS; ++i) {
      df_mbar_init(full_bar(i), 1);
      df_mbar_init(empty_bar(i), 1);
    }
    df_mbar_init(route_bar, 1);
    df_mbar_init(lg_bar, DF_CLUSTER * s.epc);
    df_mbar_init(clA_bar, DF_CLUSTER);
    df_mbar_init(clR_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  cl.sync();        // every CTA's barriers initialised before any remote arrival

  if (warp == DF_CW) {
    // ================================================================ loader
    uint32_t g = 0;   // job sequence over the launch
    auto issue = [&](const DfJobCopies& C) {
      const int slot = g % DF_NS;
      if (g >= DF_NS) df_mbar_wait(empty_bar(slot), ((g / DF_NS) + 1) & 1);
      if (lane == 0) df_mbar_expect_tx(full_bar(slot), C.bytes);
      __syncwarp();
      if (lane < C.n)
        df_bulk_g2s(smem_addr(ring + slot * DF_SLOT + C.dst[lane]), C.src[lane], C.len[lane], full_bar(slot));
      __syncwarp();
      ++g;
    };
    for (int l = 0; l < a.L; ++l) {
      const DfLayer& W = a.layer[l];
      DfJobCopies* T = tab + (l & 1) * DF_MAX_JOBS;
      const int* sl = sel + 8 * (l & 1);
      // descriptors of the routing-independent jobs, one job per lane
      for (int q = lane; q < njobs; q += 32) {
        const DfJob J = df_job(s, q);
        if (J.kind == JOB_R || J.kind == JOB_SG || J.kind == JOB_DS) T[q] = df_job_copies(s, J, a, W, sl);
      }
      __syncwarp();
      if (lane == 0 && (a.prefetch & 2)) {
        // routing-independent rows of this layer (layer 0) and of the next one into L2
        for (int ll = (l == 0 ? 0 : l + 1); ll <= l + 1 && ll < a.L; ++ll) {
          const DfLayer& V = a.layer[ll];
          prefetch_l2(reinterpret_cast<const uint8_t*>(V.rq) + static_cast<size_t>(s.rank * s.epc) * H,
                      static_cast<size_t>(s.epc) * H);
          for (int m = 0; m < 2; ++m)
            prefetch_l2(reinterpret_cast<const uint8_t*>(V.sq[m]) + static_cast<size_t>(s.s0) * (H / 2),
                        static_cast<size_t>(s.s1 - s.s0) * (H / 2));
          prefetch_l2(reinterpret_cast<const uint8_t*>(V.sq[2]) + static_cast<size_t>(s.o0) * (Is / 2),
                      static_cast<size_t>(s.o1 - s.o0) * (Is / 2));
        }
      }
      if (l + 1 < a.L && a.spec > 0 && a.layer[l + 1].bias != nullptr) {
        // the experts of the next layer with the largest bias: slice c of G of each blob
        const DfLayer& V = a.layer[l + 1];
        unsigned taken = 0;
        int my_id = -1;
        for (int r = 0; r < a.spec && r < 8; ++r) {
          float v = -INFINITY;
          int id = 0x7fffffff;
          for (int t = 0, e = lane; e < E; ++t, e += 32) {
            if (taken & (1u << t)) continue;
            const float b = V.bias[e];
            if (b > v || (b == v && e < id)) { v = b; id = e; }
          }
          for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, v, o);
            const int oi = __shfl_xor_sync(0xffffffffu, id, o);
            if (ov > v || (ov == v && oi < id)) { v = ov; id = oi; }
          }
          if ((id & 31) == lane) taken |= 1u << (id >> 5);
          if (lane == r) my_id = id;
        }
        if (my_id >= 0 && my_id < E) {
          const size_t bb = a.off[8] + static_cast<size_t>(H) * (I / 64) * 2;
          prefetch_slice(V.blobs[my_id], bb, s.c, s.G);
        }
      }
      for (int q = 0; q < nhead; ++q) issue(T[q]);
      // the routed jobs need this layer's routing
      df_mbar_wait(route_bar, l & 1);
      for (int q = nhead + lane; q < njobs; q += 32) {
        const DfJob J = df_job(s, q);
        if (J.kind == JOB_RG || J.kind == JOB_D) {
          T[q] = df_job_copies(s, J, a, W, sl);
          if (a.prefetch & 1)
            for (int i = 0; i < T[q].n; ++i) prefetch_l2(T[q].src[i], T[q].len[i]);   // all routed rows into L2
        }
      }
      __syncwarp();
      for (int q = nhead; q < njobs; ++q) issue(T[q]);
    }
    return;
  }

  // ================================================================== compute
  uint32_t g = 0;            // job sequence (same numbering as the loader)
  unsigned bar_target = 0;
  unsigned gen = 0;          // grid barriers passed
  // grid barrier among the compute warps of all CTAs: named barrier, one
  // atomic per CTA on a counter that grows by G per barrier, named barrier
  auto grid_sync = [&]() {
    df_named_sync();
    if (threadIdx.x == 0) {
      __threadfence();
      bar_target += static_cast<unsigned>(s.G);
      red_release_gpu(a.counter, 1u);
      const uint64_t t0 = df_clock();
      while (ld_acquire_gpu(a.counter) < bar_target) {
        if (df_clock() - t0 > 2000000000ull) { flag_check(CHECK_WAIT); break; }
      }
      __threadfence();
    }
    ++gen;
    df_named_sync();
  };
  auto slot_of = [&](int q) { return static_cast<int>((g + q) % DF_NS); };
  unsigned long long waited = 0;
  auto wait_full = [&](int q) {
    const uint32_t gg = g + q;
    const unsigned long long t0 = (a.stamps && warp == 0 && lane == 0) ? df_clock() : 0ull;
    df_mbar_wait(full_bar(gg % DF_NS), (gg / DF_NS) & 1);
    if (t0) waited += df_clock() - t0;
  };
  auto release = [&](int q) {
    __syncwarp();
    if (lane == 0) df_mbar_arrive(empty_bar(slot_of(q)));
  };

  for (int l = 0; l < a.L; ++l) {
    const DfLayer& W = a.layer[l];
    const DfJobCopies* T = tab + (l & 1) * DF_MAX_JOBS;
    int* sl_sel = sel + 8 * (l & 1);
    df_stamp(a, l, 0);
    // ------------------------------------------------------ A0: rms norm
    float ss = 0.f;
    for (int i = threadIdx.x * 4; i < H; i += DF_CW * 32 * 4) {
      const uint4 u = ldcg_v4(a.h + i);
      const float v0 = __uint_as_float(u.x), v1 = __uint_as_float(u.y), v2 = __uint_as_float(u.z),
                  v3 = __uint_as_float(u.w);
      xs[i] = v0; xs[i + 1] = v1; xs[i + 2] = v2; xs[i + 3] = v3;
      ss = fmaf(v0, v0, ss); ss = fmaf(v1, v1, ss); ss = fmaf(v2, v2, ss); ss = fmaf(v3, v3, ss);
    }
    ss = warp_sum(ss);
    if (lane == 0) red[warp] = ss;
    df_named_sync();
    if (warp == 0) {
      float v = lane < DF_CW ? red[lane] : 0.f;
      v = warp_sum(v);
      if (lane == 0) red[DF_CW] = v;
    }
    df_named_sync();
    const float rr = sqrtf(red[DF_CW] / static_cast<float>(H) + 1e-6f);
    for (int i = threadIdx.x; i < H; i += DF_CW * 32) {
      const uint16_t b = f32_to_bf16(__fdiv_rn(xs[i], rr));
      xs[i] = bf16_to_f32(b);
      if (s.c == 0 && a.x_trace) a.x_trace[static_cast<size_t>(l) * H + i] = b;
    }
    df_named_sync();
    // paired copies of x: nibble-paired per 8-element word (4-bit rows) and
    // byte-paired per 4-element word (8-bit router), stored word-major
    for (int w = threadIdx.x; w < H / 8; w += DF_CW * 32) {
      float v[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) v[t] = xs[8 * w + t];
      uint32_t p[4];
      pair_word4(v, p);
      xP4[(w & 3) * nch + (w >> 2)] = make_uint4(p[0], p[1], p[2], p[3]);
    }
    for (int w = threadIdx.x; w < H / 4; w += DF_CW * 32) {
      const float* v = xs + 4 * w;
      xP8[(w & 3) * nch16 + (w >> 2)] = make_uint2(pack_half2(v[0], v[2]), pack_half2(v[1], v[3]));
    }
    df_named_sync();
    for (int cc = threadIdx.x; cc < nch; cc += DF_CW * 32) {
      float off = 0.f, sum = 0.f;
      for (int m = 0; m < 4; ++m) {
        const uint4 u = xP4[m * nch + cc];
        const float2 f0 = unpack_half2(u.x), f1 = unpack_half2(u.y), f2 = unpack_half2(u.z), f3 = unpack_half2(u.w);
        off += (f0.x + f0.y) + (f1.x + f1.y) + (f2.x + f2.y) + (f3.x + f3.y);
        sum += (f0.x + f0.y + f2.x + f2.y) + 16.f * (f1.x + f1.y + f3.x + f3.y);
      }
      xS4[cc] = make_float2(1024.f * off, sum);
    }
    for (int cc = threadIdx.x; cc < nch16; cc += DF_CW * 32) {
      float sum = 0.f;
      for (int m = 0; m < 4; ++m) {
        const uint2 u = xP8[m * nch16 + cc];
        const float2 f0 = unpack_half2(u.x), f1 = unpack_half2(u.y);
        sum += (f0.x + f0.y) + (f1.x + f1.y);
      }
      xS8[cc] = sum;
    }
    df_named_sync();

    // ------------------------------------------------------------- R jobs
    for (int q = warp; q < s.nR; q += DF_CW) {
      const DfJob J = df_job(s, q);      // (the descriptor is read only after the data landed)
      float bias_r[2] = {0.f, 0.f};
      for (int r = 0; r < J.n; ++r) bias_r[r] = W.bias ? W.bias[J.r0 + r] : 0.f;
      wait_full(q);
      const DfJobCopies& C = T[q];
      const unsigned char* slp = ring + slot_of(q) * DF_SLOT;
      for (int r = 0; r < C.rows; ++r) {
        const int e = C.r0 + r;
        const uint8_t* qrow = slp + static_cast<size_t>(r) * H;
        const uint16_t* S = reinterpret_cast<const uint16_t*>(slp + DF_SLOT_Q + C.sk[0]) + r * (H / 64);
        const uint16_t* B = reinterpret_cast<const uint16_t*>(slp + DF_SLOT_Q + C.sk[1]) + r * (H / 64);
        float acc = 0.f;
        for (int cc = lane; cc < nch16; cc += 32) {
          const uint4 q4 = *reinterpret_cast<const uint4*>(qrow + 16 * cc);
          const uint32_t w[4] = {q4.x, q4.y, q4.z, q4.w};
          float a0 = 0.f, a1 = 0.f;
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const uint2 pp = xP8[m * nch16 + cc];
            const uint32_t p[2] = {pp.x, pp.y};
            dot_word8(w[m], p, a0, a1);
          }
          const float sm = xS8[cc];
          acc += bf16_to_f32(S[cc >> 2]) * ((a0 + a1) - 1024.f * sm) + bf16_to_f32(B[cc >> 2]) * sm;
        }
        acc = warp_sum(acc) + (r == 0 ? bias_r[0] : bias_r[1]);
        if (lane < DF_CLUSTER) {          // broadcast the logit to every CTA of the cluster
          df_st_remote_f32(smem_addr(lg_all + e), lane, acc);
          df_mbar_arrive_remote(lg_bar, lane);
        }
      }
      release(q);
    }
    df_stamp(a, l, 1);

    // ----------------------------------------- register x for gate/up rows
    uint32_t xp[DF_CPL][16];
    float2 xst[DF_CPL];
#pragma unroll
    for (int j = 0; j < DF_CPL; ++j) {
      const int cc = lane + 32 * j;
      if (cc < nch) {
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const uint4 u = xP4[m * nch + cc];
          xp[j][4 * m + 0] = u.x; xp[j][4 * m + 1] = u.y; xp[j][4 * m + 2] = u.z; xp[j][4 * m + 3] = u.w;
        }
        xst[j] = xS4[cc];
      } else {
#pragma unroll
        for (int t = 0; t < 16; ++t) xp[j][t] = 0u;
        xst[j] = make_float2(0.f, 0.f);
      }
    }

    // -------------------------------------------------- routing (cluster)
    df_mbar_wait(lg_bar, l & 1, true);
    if (warp == 0) {
      unsigned taken = 0u;
      float sv[8];
      int si[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        sv[j] = 0.f;
        si[j] = 0;
        if (j < k) {
          float bv = -INFINITY;
          int bi = 0x7fffffff;
          for (int t = 0, e = lane; e < E; ++t, e += 32) {
            if (taken & (1u << t)) continue;
            const float v = lg_all[e];
            if (v > bv || (v == bv && e < bi)) { bv = v; bi = e; }
          }
          for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
          }
          if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
          sv[j] = bv;
          si[j] = bi;
        }
      }
      if (lane == 0) {
        float z[8], den = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          z[j] = j < k ? expf(sv[j] - sv[0]) : 0.f;
          den += z[j];
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (j < k) {
            sl_sel[j] = si[j];
            selg[j] = z[j] / den;
            if (s.c == 0 && a.idx_trace) a.idx_trace[static_cast<size_t>(l) * k + j] = si[j];
            if (s.c == 0 && a.gates_trace) a.gates_trace[static_cast<size_t>(l) * k + j] = z[j] / den;
          }
        }
        df_mbar_arrive(route_bar);      // hand the routing to the loader
      }
    }
    df_named_sync();                    // sl_sel visible to every compute warp
    df_stamp(a, l, 2);

    // ---------------------------------------------------- SG and RG jobs
    for (int q = s.nR + warp; q < s.nR + s.nSG + s.nRG; q += DF_CW) {
      wait_full(q);                     // (also orders the loader's descriptor writes)
      const DfJobCopies& C = T[q];
      const unsigned char* slp = ring + slot_of(q) * DF_SLOT;
      for (int r = 0; r < C.rows; ++r) {
        const uint8_t* gqr = slp + static_cast<size_t>(r) * (H / 2);
        const uint8_t* uqr = slp + C.qbytes + static_cast<size_t>(r) * (H / 2);
        const uint16_t* Sg = reinterpret_cast<const uint16_t*>(slp + DF_SLOT_Q + C.sk[0]) + r * (H / 64);
        const uint16_t* Bg = reinterpret_cast<const uint16_t*>(slp + DF_SLOT_Q + C.sk[1]) + r * (H / 64);
        const uint16_t* Su = reinterpret_cast<const uint16_t*>(slp + DF_SLOT_Q + C.sk[2]) + r * (H / 64);
        const uint16_t* Bu = reinterpret_cast<const uint16_t*>(slp + DF_SLOT_Q + C.sk[3]) + r * (H / 64);
        float ga = 0.f, ua = 0.f;
#pragma unroll
        for (int j = 0; j < DF_CPL; ++j) {
          const int cc = lane + 32 * j;
          if (cc < nch) {
            const uint4 q4g = *reinterpret_cast<const uint4*>(gqr + 16 * cc);
            const uint4 q4u = *reinterpret_cast<const uint4*>(uqr + 16 * cc);
            const float dg = dot_chunk4(q4g, xp[j]);
            const float du = dot_chunk4(q4u, xp[j]);
            ga += bf16_to_f32(Sg[cc >> 1]) * (dg - xst[j].x) + bf16_to_f32(Bg[cc >> 1]) * xst[j].y;
            ua += bf16_to_f32(Su[cc >> 1]) * (du - xst[j].x) + bf16_to_f32(Bu[cc >> 1]) * xst[j].y;
          }
        }
        ga = warp_sum(ga);
        ua = warp_sum(ua);
        if (lane == 0) {
          const int dst = C.kind == JOB_SG ? kI + C.r0 + r : C.slot * I + C.r0 + r;
          a.act[dst] = __float2half_rn(gelu_tanh(ga) * ua);
        }
      }
      release(q);
    }

    df_stamp(a, l, 3);
    if (a.stamps && threadIdx.x == 0)
      a.stamps[(static_cast<size_t>(l) * gridDim.x + blockIdx.x) * 8 + 7] = waited;
    waited = 0;
    grid_sync();
    df_stamp(a, l, 4);

    // ------------------------------------------------------------- phase C
    for (int w = threadIdx.x; w < nact / 8; w += DF_CW * 32) {
      const uint4 u = ldcg_v4(a.act + 8 * w);
      float v[8];
      const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float2 f = unpack_half2(uw[t]);
        v[2 * t] = f.x;
        v[2 * t + 1] = f.y;
      }
      uint32_t p[4];
      pair_word4(v, p);
      actP[w] = make_uint4(p[0], p[1], p[2], p[3]);
      float off = 0.f;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float2 f = unpack_half2(p[t]);
        off += f.x + f.y;
      }
      const float2 f0 = unpack_half2(p[0]), f1 = unpack_half2(p[1]), f2 = unpack_half2(p[2]), f3 = unpack_half2(p[3]);
      actS[w] = make_float2(1024.f * off, (f0.x + f0.y + f2.x + f2.y) + 16.f * (f1.x + f1.y + f3.x + f3.y));
    }
    df_named_sync();
    for (int q = nhead + s.nRG + warp; q < njobs; q += DF_CW) {
      wait_full(q);
      const DfJobCopies& C = T[q];
      const unsigned char* slp = ring + slot_of(q) * DF_SLOT;
      const int K = C.kind == JOB_D ? I : Is;
      const int wbase = C.kind == JOB_D ? C.slot * (I / 8) : kI / 8;
      const int unit = C.kind == JOB_D ? C.slot : k;
      const int nw = K / 8;
      for (int r = 0; r < C.rows; ++r) {
        const uint8_t* qrow = slp + static_cast<size_t>(r) * (K / 2);
        const uint16_t* S = reinterpret_cast<const uint16_t*>(slp + DF_SLOT_Q + C.sk[0]) + r * (K / 64);
        const uint16_t* B = reinterpret_cast<const uint16_t*>(slp + DF_SLOT_Q + C.sk[1]) + r * (K / 64);
        float acc = 0.f;
        for (int w = lane; w < nw; w += 32) {
          const uint32_t qw = *reinterpret_cast<const uint32_t*>(qrow + 4 * w);
          const uint4 pp = actP[wbase + w];
          const uint32_t p[4] = {pp.x, pp.y, pp.z, pp.w};
          float a0 = 0.f, a1 = 0.f;
          dot_word4(qw, p, a0, a1);
          const float2 st = actS[wbase + w];
          acc += bf16_to_f32(S[w >> 3]) * ((a0 + a1) - st.x) + bf16_to_f32(B[w >> 3]) * st.y;
        }
        acc = warp_sum(acc);
        if (lane == 0) part[(C.r0 + r - s.o0) * 9 + unit] = acc;
      }
      release(q);
    }
    df_named_sync();
    for (int ro = threadIdx.x; ro < s.o1 - s.o0; ro += DF_CW * 32) {
      float y = 0.f;
      for (int j = 0; j < k; ++j) y = fmaf(selg[j], part[ro * 9 + j], y);
      y += part[ro * 9 + k];
      const int o = s.o0 + ro;
      a.h[o] = __ldcg(a.h + o) + y;
      if (a.y_trace) a.y_trace[static_cast<size_t>(l) * H + o] = f32_to_bf16(y);
    }
    g += njobs;
    df_stamp(a, l, 5);
    if (l + 1 < a.L) grid_sync();
    df_stamp(a, l, 6);
  }
}

size_t decode_fused_smem() {
  return static_cast<size_t>(DF_NS) * DF_SLOT + 2 * DF_MAX_JOBS * sizeof(DfJobCopies) + DF_MAX_H * 4 +
         DF_MAX_H / 8 * 16 + DF_MAX_H / 32 * 8 + DF_MAX_H / 4 * 8 + DF_MAX_H / 16 * 4 +
         static_cast<size_t>(DF_MAX_ACT / 8) * (16 + 8) + DF_MAX_ROWS * 9 * 4 + DF_MAX_E * 4 + 32 * 4 + 16 * 4 +
         8 * 4 + (2 * DF_NS + 8) * 8 + 128;
}

// Rows per job so that one job fits a ring slot (0 if even one row does not).
inline int df_rows_fit(int runs, int qbytes_per_row, int windows, int sbytes_per_row) {
  int n = 0;
  while (true) {
    const int m = n + 1;
    if (runs * m * qbytes_per_row > DF_SLOT_Q) break;
    if (windows * (m * sbytes_per_row + 32) > DF_SLOT_S) break;
    n = m;
    if (n >= 64) break;
  }
  return n;
}

}  // namespace moe
