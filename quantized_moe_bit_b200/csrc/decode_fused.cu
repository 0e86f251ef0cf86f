// Batch-1 decode of a stack of routed-MoE layers in one persistent kernel.
//
// One cooperative launch runs every layer of the step, one CTA per SM (G
// CTAs).  Work of a layer, split statically over the CTAs (CTA c):
//   router row c (for c < E), shared-expert gate/up row pairs [c*Is/G, ...),
//   routed gate/up (slot, row) pairs [c*k*I/G, ...) of the k*I list, and
//   output rows [c*H/G, ...) (their k routed down rows and shared down row).
// Per layer:
//   A  rms norm of h (every CTA, same order, same result); router logit c and
//      the shared gate/up rows from L2 (prefetched a layer ahead) with plain
//      loads -> logits, fp16 activations (global)
//   grid barrier
//   B  every CTA selects the top k from the logits, then issues every byte of
//      its routed work at once -- gate/up row pairs and its output rows of the
//      k down matrices, with their scale/bias windows -- as 1-D bulk copies
//      (cp.async.bulk) into shared memory, one mbarrier per chunk, so a
//      layer's 26.8 MB of routed weights is in flight together; warps compute
//      each chunk as it lands -> fp16 activations
//   grid barrier
//   C  the shared expert's down rows (from L2) are bulk-copied into the freed
//      gate/up area; all activations are staged in shared memory; per output
//      row: k routed down dots and the shared down dot, combined in a fixed
//      order, y = sum_j g_j y_j + ysh; h += y.  The next layer's
//      routing-independent rows (and slices of the experts with the largest
//      router bias) are prefetched into L2 here.
//   grid barrier
// Grid barriers: named barrier, one atomic per CTA on a counter that grows
// by G per barrier, named barrier.  Every wait is bounded (about two
// seconds); a wait that runs out sets the device check word and the thread
// runs on to the end.
#include <cooperative_groups.h>

namespace moe {

constexpr int DF_THREADS = 384;
constexpr int DF_WARPS = DF_THREADS / 32;
constexpr int DF_MAX_LAYERS = 48;
constexpr int DF_MAX_H = 3072;
constexpr int DF_CPL = 3;                       // uint4 chunks per lane of a gate/up row (H <= 3072)
constexpr int DF_MAX_ACT = 8192;                // k*I + Is
constexpr int DF_MAX_ROWS = 32;                 // output rows per CTA
constexpr int DF_MAX_E = 256;
constexpr int DF_RGC = 10;                      // row pairs per routed gate/up chunk
constexpr int DF_MAX_CHUNKS = 32;               // routed chunks per CTA and layer (one per lane)
constexpr int DF_RS = 193536;                   // shared-memory staging for a CTA's routed bytes

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
  float* logits;                    // workspace: [E]
  unsigned* counter;                // workspace: grid barrier counter (zeroed before launch)
  uint16_t* x_trace; uint16_t* y_trace; int32_t* idx_trace; float* gates_trace;
  int spec;                         // experts speculatively prefetched per layer
  int prefetch;                     // bit 1: routing-independent rows of the next layer into L2
  unsigned long long* stamps;       // optional phase timestamps [L][G][16] (ns), or null
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

// phase timestamps (when requested): layer l, CTA c, phase p
__device__ __forceinline__ void df_stamp(const DfArgs& a, int l, int p) {
  if (a.stamps != nullptr && threadIdx.x == 0)
    a.stamps[(static_cast<size_t>(l) * gridDim.x + blockIdx.x) * 16 + p] = df_clock();
}


__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

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

enum : int { CH_RG = 0, CH_D = 1, CH_DS = 2, CH_SG = 3, CH_R = 4 };

// One chunk of staged bytes: weight runs (run i at i * qbytes from the chunk
// start), then scale/bias windows; sk[i] = offset of window i's first row
// from the chunk start.
struct DfChunk {
  const uint8_t* src[6];
  uint32_t dst[6];
  uint32_t len[6];
  int n;
  uint32_t qbytes, bytes, off;      // off: chunk start inside the staging area
  uint32_t sk[4];
  int kind, slot, r0, rows;
};

__device__ inline DfChunk df_chunk(int kind, int slot, int r0, int rows, int H, int I, int Is, const DfArgs& a,
                                   const DfLayer& W, const int* sel) {
  DfChunk C{};
  C.kind = kind; C.slot = slot; C.r0 = r0; C.rows = rows;
  const uint8_t* q[2] = {nullptr, nullptr};
  const uint16_t* sc[4] = {nullptr, nullptr, nullptr, nullptr};
  int per = 0, nq = 0, ns = 0;
  if (kind == CH_RG) {
    const uint8_t* blob = static_cast<const uint8_t*>(W.blobs[sel[slot]]);
    q[0] = blob + a.off[0] + static_cast<size_t>(r0) * (H / 2);
    q[1] = blob + a.off[3] + static_cast<size_t>(r0) * (H / 2);
    C.qbytes = static_cast<uint32_t>(rows) * (H / 2); nq = 2;
    sc[0] = reinterpret_cast<const uint16_t*>(blob + a.off[1]); sc[1] = reinterpret_cast<const uint16_t*>(blob + a.off[2]);
    sc[2] = reinterpret_cast<const uint16_t*>(blob + a.off[4]); sc[3] = reinterpret_cast<const uint16_t*>(blob + a.off[5]);
    ns = 4; per = H / 64;
  } else if (kind == CH_D) {
    const uint8_t* blob = static_cast<const uint8_t*>(W.blobs[sel[slot]]);
    q[0] = blob + a.off[6] + static_cast<size_t>(r0) * (I / 2);
    C.qbytes = static_cast<uint32_t>(rows) * (I / 2); nq = 1;
    sc[0] = reinterpret_cast<const uint16_t*>(blob + a.off[7]); sc[1] = reinterpret_cast<const uint16_t*>(blob + a.off[8]);
    ns = 2; per = I / 64;
  } else if (kind == CH_DS) {
    q[0] = reinterpret_cast<const uint8_t*>(W.sq[2]) + static_cast<size_t>(r0) * (Is / 2);
    C.qbytes = static_cast<uint32_t>(rows) * (Is / 2); nq = 1;
    sc[0] = W.ss[2]; sc[1] = W.sb[2]; ns = 2; per = Is / 64;
  } else if (kind == CH_SG) {
    q[0] = reinterpret_cast<const uint8_t*>(W.sq[0]) + static_cast<size_t>(r0) * (H / 2);
    q[1] = reinterpret_cast<const uint8_t*>(W.sq[1]) + static_cast<size_t>(r0) * (H / 2);
    C.qbytes = static_cast<uint32_t>(rows) * (H / 2); nq = 2;
    sc[0] = W.ss[0]; sc[1] = W.sb[0]; sc[2] = W.ss[1]; sc[3] = W.sb[1]; ns = 4; per = H / 64;
  } else {   // CH_R: router rows (8-bit, H bytes each)
    q[0] = reinterpret_cast<const uint8_t*>(W.rq) + static_cast<size_t>(r0) * H;
    C.qbytes = static_cast<uint32_t>(rows) * H; nq = 1;
    sc[0] = W.rs; sc[1] = W.rb; ns = 2; per = H / 64;
  }
  uint32_t o = 0;
  for (int i = 0; i < nq; ++i) {
    C.src[C.n] = q[i]; C.dst[C.n] = o; C.len[C.n] = C.qbytes; ++C.n;
    o += C.qbytes;
  }
  for (int i = 0; i < ns; ++i) {
    const uint8_t* src; uint32_t bytes, skew;
    sb_window(sc[i], per, r0, rows, src, bytes, skew);
    C.src[C.n] = src; C.dst[C.n] = o; C.len[C.n] = bytes; ++C.n;
    C.sk[i] = o + skew;
    o += bytes;
  }
  C.bytes = o;
  return C;
}

// Number of routed gate/up chunks of the flattened pair range [r0, r1).
__device__ inline int df_rg_chunks(int r0, int r1, int I) {
  if (r1 <= r0) return 0;
  int n = 0;
  for (int j = r0 / I; j <= (r1 - 1) / I; ++j) n += ceil_div(min(r1, (j + 1) * I) - max(r0, j * I), DF_RGC);
  return n;
}
// Chunk t of them: slot, first row, rows.
__device__ inline void df_rg_chunk_at(int r0, int r1, int I, int t, int& slot, int& row, int& rows) {
  for (int j = r0 / I; j <= (r1 - 1) / I; ++j) {
    const int a = max(r0, j * I), b = min(r1, (j + 1) * I);
    const int nj = ceil_div(b - a, DF_RGC);
    if (t < nj) { slot = j; row = a - j * I + t * DF_RGC; rows = min(DF_RGC, b - a - t * DF_RGC); return; }
    t -= nj;
  }
  slot = 0; row = 0; rows = 0;
}

// One gate/up row pair (rows of K = H nibbles each) against the register x:
// returns (gate . x, up . x) in every lane.  Weight rows and scale rows may be
// in shared or global memory.
__device__ __forceinline__ float2 df_pair(const uint8_t* gq, const uint8_t* uq, const uint16_t* gs,
                                          const uint16_t* gb, const uint16_t* us, const uint16_t* ub, int nch,
                                          const uint32_t (&xp)[DF_CPL][16], const float2 (&xst)[DF_CPL],
                                          bool global) {
  const int lane = threadIdx.x & 31;
  uint4 qg[DF_CPL], qu[DF_CPL];
  float sg[DF_CPL], bg[DF_CPL], su[DF_CPL], bu[DF_CPL];
#pragma unroll
  for (int j = 0; j < DF_CPL; ++j) {
    const int cc = lane + 32 * j;
    if (cc < nch) {
      if (global) {
        qg[j] = ldg_nc_v4(gq + 16 * cc); qu[j] = ldg_nc_v4(uq + 16 * cc);
        sg[j] = bf16_to_f32(ldg_u16(gs + (cc >> 1))); bg[j] = bf16_to_f32(ldg_u16(gb + (cc >> 1)));
        su[j] = bf16_to_f32(ldg_u16(us + (cc >> 1))); bu[j] = bf16_to_f32(ldg_u16(ub + (cc >> 1)));
      } else {
        qg[j] = *reinterpret_cast<const uint4*>(gq + 16 * cc); qu[j] = *reinterpret_cast<const uint4*>(uq + 16 * cc);
        sg[j] = bf16_to_f32(gs[cc >> 1]); bg[j] = bf16_to_f32(gb[cc >> 1]);
        su[j] = bf16_to_f32(us[cc >> 1]); bu[j] = bf16_to_f32(ub[cc >> 1]);
      }
    }
  }
  float ga = 0.f, ua = 0.f;
#pragma unroll
  for (int j = 0; j < DF_CPL; ++j) {
    const int cc = lane + 32 * j;
    if (cc < nch) {
      ga += sg[j] * (dot_chunk4(qg[j], xp[j]) - xst[j].x) + bg[j] * xst[j].y;
      ua += su[j] * (dot_chunk4(qu[j], xp[j]) - xst[j].x) + bu[j] * xst[j].y;
    }
  }
  return make_float2(warp_sum(ga), warp_sum(ua));
}

// --------------------------------------------------------------- the kernel
__global__ void __launch_bounds__(DF_THREADS, 1) k_decode_b1(const __grid_constant__ DfArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int H = a.H, I = a.I, Is = a.Is, E = a.E, k = a.k;
  const int G = gridDim.x, c = blockIdx.x;
  const int kI = k * I, nact = kI + Is;
  const int s0 = (int)((long)c * Is / G), s1 = (int)((long)(c + 1) * Is / G);
  const int r0 = (int)((long)c * kI / G), r1 = (int)((long)(c + 1) * kI / G);
  const int o0 = (int)((long)c * H / G), o1 = (int)((long)(c + 1) * H / G);
  const int nrow = o1 - o0;
  const int nrg = df_rg_chunks(r0, r1, I);
  const int nchunk = nrg + k;                  // routed chunks: gate/up pieces, then one down chunk per slot
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nch = H / 32;

  // shared memory
  unsigned char* rs = smem;                                            // [DF_RS] routed staging
  unsigned char* ax = rs + DF_RS;                                      // union: x (phase A) / activations (C)
  float* xs = reinterpret_cast<float*>(ax);                            // [H]
  uint4* actP = reinterpret_cast<uint4*>(ax);                          // [nact/8]
  float2* actS = reinterpret_cast<float2*>(actP + DF_MAX_ACT / 8);     // [nact/8]
  uint4* xP4 = reinterpret_cast<uint4*>(ax + (DF_MAX_ACT / 8) * 24);   // [4][nch]
  float2* xS4 = reinterpret_cast<float2*>(xP4 + DF_MAX_H / 8);         // [nch]
  float* part = reinterpret_cast<float*>(xS4 + DF_MAX_H / 32);         // [MAX_ROWS][9]
  float* red = part + DF_MAX_ROWS * 9;                                 // [32]
  int* sel = reinterpret_cast<int*>(red + 32);                         // [8]
  float* selg = reinterpret_cast<float*>(sel + 8);                     // [8]
  DfChunk* tab = reinterpret_cast<DfChunk*>(selg + 8);                 // [DF_MAX_CHUNKS + 3]
  uint64_t* bars = reinterpret_cast<uint64_t*>(tab + DF_MAX_CHUNKS + 3);   // [DF_MAX_CHUNKS + 3]
  const int IDX_DS = DF_MAX_CHUNKS, IDX_SG = DF_MAX_CHUNKS + 1, IDX_R = DF_MAX_CHUNKS + 2;
  const uint32_t bar0 = smem_addr(bars);

  if (threadIdx.x == 0) {
    for (int i = 0; i < DF_MAX_CHUNKS + 3; ++i) df_mbar_init(bar0 + 8u * i, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  unsigned bar_target = 0;
  auto grid_sync = [&]() {
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      bar_target += static_cast<unsigned>(G);
      red_release_gpu(a.counter, 1u);
      const uint64_t t0 = df_clock();
      while (ld_acquire_gpu(a.counter) < bar_target) {
        if (df_clock() - t0 > 2000000000ull) { flag_check(CHECK_WAIT); break; }
      }
      __threadfence();
    }
    __syncthreads();
  };
  // routing-independent rows of layer l (and likely experts) into L2
  auto prefetch_layer = [&](int l) {
    const DfLayer& V = a.layer[l];
    if (threadIdx.x == 0 && (a.prefetch & 2)) {
      for (int e = c; e < E; e += G) {
        prefetch_l2(reinterpret_cast<const uint8_t*>(V.rq) + static_cast<size_t>(e) * H, H);
        prefetch_l2(V.rs + static_cast<size_t>(e) * (H / 64), (H / 64) * 2);
        prefetch_l2(V.rb + static_cast<size_t>(e) * (H / 64), (H / 64) * 2);
      }
      for (int m = 0; m < 2; ++m) {
        prefetch_l2(reinterpret_cast<const uint8_t*>(V.sq[m]) + static_cast<size_t>(s0) * (H / 2),
                    static_cast<size_t>(s1 - s0) * (H / 2));
        prefetch_l2(V.ss[m] + static_cast<size_t>(s0) * (H / 64), static_cast<size_t>(s1 - s0) * (H / 64) * 2);
        prefetch_l2(V.sb[m] + static_cast<size_t>(s0) * (H / 64), static_cast<size_t>(s1 - s0) * (H / 64) * 2);
      }
      prefetch_l2(reinterpret_cast<const uint8_t*>(V.sq[2]) + static_cast<size_t>(o0) * (Is / 2),
                  static_cast<size_t>(nrow) * (Is / 2));
      prefetch_l2(V.ss[2] + static_cast<size_t>(o0) * (Is / 64), static_cast<size_t>(nrow) * (Is / 64) * 2);
      prefetch_l2(V.sb[2] + static_cast<size_t>(o0) * (Is / 64), static_cast<size_t>(nrow) * (Is / 64) * 2);
    }
    if (warp == 1 && a.spec > 0 && V.bias != nullptr) {
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
        prefetch_slice(V.blobs[my_id], bb, c, G);
      }
    }
  };
  // warp 0: chunk `idx` at `off` in the staging area, completing on its mbarrier
  auto issue_chunk = [&](int idx, const DfChunk& C0, uint32_t off) {
    if (lane == 0) {
      tab[idx] = C0;
      tab[idx].off = off;
      df_mbar_expect_tx(bar0 + 8u * idx, C0.bytes);
    }
    __syncwarp();
    const DfChunk& T = tab[idx];
    if (lane < T.n) df_bulk_g2s(smem_addr(rs + T.off + T.dst[lane]), T.src[lane], T.len[lane], bar0 + 8u * idx);
    __syncwarp();
  };
  // routing-independent rows of layer l's phase A: shared gate/up rows, router row c
  auto issue_phase_a = [&](int l) {
    const DfLayer& V = a.layer[l];
    DfChunk sg = df_chunk(CH_SG, 0, s0, s1 - s0, H, I, Is, a, V, sel);
    issue_chunk(IDX_SG, sg, 0u);
    if (c < E) {
      DfChunk rc = df_chunk(CH_R, 0, c, 1, H, I, Is, a, V, sel);
      issue_chunk(IDX_R, rc, (sg.bytes + 127u) & ~127u);
    }
  };
  prefetch_layer(0);
  if (warp == 0) issue_phase_a(0);

  for (int l = 0; l < a.L; ++l) {
    const DfLayer& W = a.layer[l];
    const uint32_t par = l & 1;
    df_stamp(a, l, 0);
    // ------------------------------------------------------ A0: rms norm
    float ss = 0.f;
    for (int i = threadIdx.x * 4; i < H; i += DF_THREADS * 4) {
      const uint4 u = ldcg_v4(a.h + i);
      const float v0 = __uint_as_float(u.x), v1 = __uint_as_float(u.y), v2 = __uint_as_float(u.z),
                  v3 = __uint_as_float(u.w);
      xs[i] = v0; xs[i + 1] = v1; xs[i + 2] = v2; xs[i + 3] = v3;
      ss = fmaf(v0, v0, ss); ss = fmaf(v1, v1, ss); ss = fmaf(v2, v2, ss); ss = fmaf(v3, v3, ss);
    }
    ss = warp_sum(ss);
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    if (warp == 0) {
      float v = lane < DF_WARPS ? red[lane] : 0.f;
      v = warp_sum(v);
      if (lane == 0) red[DF_WARPS] = v;
    }
    __syncthreads();
    const float rr = sqrtf(red[DF_WARPS] / static_cast<float>(H) + 1e-6f);
    for (int i = threadIdx.x; i < H; i += DF_THREADS) {
      const uint16_t b = f32_to_bf16(__fdiv_rn(xs[i], rr));
      xs[i] = bf16_to_f32(b);
      if (c == 0 && a.x_trace) a.x_trace[static_cast<size_t>(l) * H + i] = b;
    }
    __syncthreads();
    for (int w = threadIdx.x; w < H / 8; w += DF_THREADS) {
      float v[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) v[t] = xs[8 * w + t];
      uint32_t p[4];
      pair_word4(v, p);
      xP4[(w & 3) * nch + (w >> 2)] = make_uint4(p[0], p[1], p[2], p[3]);
    }
    __syncthreads();
    for (int cc = threadIdx.x; cc < nch; cc += DF_THREADS) {
      float off = 0.f, sum = 0.f;
      for (int m = 0; m < 4; ++m) {
        const uint4 u = xP4[m * nch + cc];
        const float2 f0 = unpack_half2(u.x), f1 = unpack_half2(u.y), f2 = unpack_half2(u.z), f3 = unpack_half2(u.w);
        off += (f0.x + f0.y) + (f1.x + f1.y) + (f2.x + f2.y) + (f3.x + f3.y);
        sum += (f0.x + f0.y + f2.x + f2.y) + 16.f * (f1.x + f1.y + f3.x + f3.y);
      }
      xS4[cc] = make_float2(1024.f * off, sum);
    }
    __syncthreads();
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

    df_stamp(a, l, 1);
    // --------------------------------- router logit and shared gate/up rows
    if (warp == DF_WARPS - 1) {
      if (c < E) {
        const DfChunk& C = tab[IDX_R];
        df_mbar_wait(bar0 + 8u * IDX_R, par);
        const uint8_t* qrow = rs + C.off;
        const uint16_t* S = reinterpret_cast<const uint16_t*>(rs + C.off + C.sk[0]);
        const uint16_t* B = reinterpret_cast<const uint16_t*>(rs + C.off + C.sk[1]);
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
        if (lane == 0) a.logits[c] = acc + (W.bias ? W.bias[c] : 0.f);
      }
    } else if (s1 > s0) {
      const DfChunk& C = tab[IDX_SG];
      df_mbar_wait(bar0 + 8u * IDX_SG, par);
      const unsigned char* base = rs + C.off;
      for (int r = warp; r < s1 - s0; r += DF_WARPS - 1) {
        const float2 gu = df_pair(base + r * (H / 2), base + C.qbytes + r * (H / 2),
                                  reinterpret_cast<const uint16_t*>(base + C.sk[0]) + r * (H / 64),
                                  reinterpret_cast<const uint16_t*>(base + C.sk[1]) + r * (H / 64),
                                  reinterpret_cast<const uint16_t*>(base + C.sk[2]) + r * (H / 64),
                                  reinterpret_cast<const uint16_t*>(base + C.sk[3]) + r * (H / 64), nch, xp, xst, false);
        if (lane == 0) a.act[kI + s0 + r] = __float2half_rn(gelu_tanh(gu.x) * gu.y);
      }
    }
    df_stamp(a, l, 2);
    grid_sync();
    df_stamp(a, l, 3);

    // ------------------------------------------------ top-k, issue routed bytes
    if (warp == 0) {
      unsigned taken = 0u;
      float sv[8];
      int si[8];
      float lv[DF_MAX_E / 32];            // this lane's logits, read once
#pragma unroll
      for (int t = 0; t < DF_MAX_E / 32; ++t) lv[t] = (lane + 32 * t < E) ? __ldcg(a.logits + lane + 32 * t) : 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        sv[j] = 0.f;
        si[j] = 0;
        if (j < k) {
          float bv = -INFINITY;
          int bi = 0x7fffffff;
#pragma unroll
          for (int t = 0; t < DF_MAX_E / 32; ++t) {
            const int e = lane + 32 * t;
            if (e >= E || (taken & (1u << t))) continue;
            const float v = lv[t];
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
      float z[8], den = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        z[j] = j < k ? expf(sv[j] - sv[0]) : 0.f;
        den += z[j];
      }
      if (lane < k) {
        float zl = 0.f;
        int il = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) if (j == lane) { zl = z[j]; il = si[j]; }
        sel[lane] = il;
        selg[lane] = zl / den;
        if (c == 0 && a.idx_trace) a.idx_trace[static_cast<size_t>(l) * k + lane] = il;
        if (c == 0 && a.gates_trace) a.gates_trace[static_cast<size_t>(l) * k + lane] = zl / den;
      }
      __syncwarp();
      if (lane == 0) df_stamp(a, l, 4);
      // chunk `lane`: its bytes, its place in the staging area (exclusive scan)
      DfChunk C{};
      if (lane < nchunk) {
        if (lane < nrg) {
          int slot, row, rows;
          df_rg_chunk_at(r0, r1, I, lane, slot, row, rows);
          C = df_chunk(CH_RG, slot, row, rows, H, I, Is, a, W, sel);
        } else {
          C = df_chunk(CH_D, lane - nrg, o0, nrow, H, I, Is, a, W, sel);
        }
      }
      uint32_t sz = lane < nchunk ? C.bytes : 0u, incl = sz;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      if (lane < nchunk) {
        C.off = incl - sz;
        tab[lane] = C;
        const uint32_t bar = bar0 + 8u * lane;
        df_mbar_expect_tx(bar, C.bytes);
        for (int i = 0; i < C.n; ++i) df_bulk_g2s(smem_addr(rs + C.off + C.dst[i]), C.src[i], C.len[i], bar);
      }
    }
    __syncthreads();
    df_stamp(a, l, 5);

    // ------------------------------------------------------ routed gate/up
    {
      const int npairs = r1 - r0;
      for (int p = warp; p < npairs; p += DF_WARPS) {
        const int t = p / DF_RGC;                // chunks hold DF_RGC pairs except at slot ends
        // find the chunk holding flat pair r0 + p (chunks are in flat order)
        int ch = 0, first = 0;
        for (int q = 0; q < nrg; ++q) {
          const DfChunk& Cq = tab[q];
          const int f = Cq.slot * I + Cq.r0 - r0;
          if (p >= f && p < f + Cq.rows) { ch = q; first = f; break; }
        }
        (void)t;
        const DfChunk& C = tab[ch];
        df_mbar_wait(bar0 + 8u * ch, par);
        const int r = p - first;
        const unsigned char* base = rs + C.off;
        const float2 gu = df_pair(base + r * (H / 2), base + C.qbytes + r * (H / 2),
                                  reinterpret_cast<const uint16_t*>(base + C.sk[0]) + r * (H / 64),
                                  reinterpret_cast<const uint16_t*>(base + C.sk[1]) + r * (H / 64),
                                  reinterpret_cast<const uint16_t*>(base + C.sk[2]) + r * (H / 64),
                                  reinterpret_cast<const uint16_t*>(base + C.sk[3]) + r * (H / 64), nch, xp, xst, false);
        if (lane == 0) a.act[C.slot * I + C.r0 + r] = __float2half_rn(gelu_tanh(gu.x) * gu.y);
      }
    }
    df_stamp(a, l, 6);
    // shared down rows of phase C into the gate/up part of the staging area
    // (free now) when it is large enough, else after the down chunks
    const int dsc = IDX_DS;
    __syncthreads();
    if (warp == 0) {
      const DfChunk C = df_chunk(CH_DS, 0, o0, nrow, H, I, Is, a, W, sel);
      const uint32_t rg_bytes = tab[nrg].off;
      const uint32_t used = tab[nchunk - 1].off + tab[nchunk - 1].bytes;
      issue_chunk(dsc, C, C.bytes <= rg_bytes ? 0u : ((used + 127u) & ~127u));
    }
    df_stamp(a, l, 7);
    grid_sync();
    df_stamp(a, l, 8);

    // ------------------------------------------------------------- phase C
    if (l + 1 < a.L) prefetch_layer(l + 1);
    df_stamp(a, l, 9);
    for (int w = threadIdx.x; w < nact / 8; w += DF_THREADS) {
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
    __syncthreads();
    df_stamp(a, l, 10);
    // units (piece u, block of DF_RB rows): u < k routed slot u (K = I),
    // u == k the shared expert (K = Is); the activation word is loaded once
    // and applied to the block's rows (independent accumulators)
    constexpr int DF_RB = 4;
    const int nblk = (nrow + DF_RB - 1) / DF_RB;
    for (int un = warp; un < nblk * (k + 1); un += DF_WARPS) {
      const int u = un % (k + 1), rb = un / (k + 1);
      const int ch = u < k ? nrg + u : dsc;
      const DfChunk& C = tab[ch];
      df_mbar_wait(bar0 + 8u * ch, par);
      const int K = u < k ? I : Is;
      const int wbase = u < k ? u * (I / 8) : kI / 8;
      const int rbeg = rb * DF_RB, nr = min(DF_RB, nrow - rbeg);
      const unsigned char* base = rs + C.off;
      const uint8_t* q0 = base + static_cast<size_t>(rbeg) * (K / 2);
      const uint16_t* S0 = reinterpret_cast<const uint16_t*>(base + C.sk[0]) + rbeg * (K / 64);
      const uint16_t* B0 = reinterpret_cast<const uint16_t*>(base + C.sk[1]) + rbeg * (K / 64);
      float acc[DF_RB];
#pragma unroll
      for (int t = 0; t < DF_RB; ++t) acc[t] = 0.f;
      for (int w = lane; w < K / 8; w += 32) {
        const uint4 pp = actP[wbase + w];
        const uint32_t p[4] = {pp.x, pp.y, pp.z, pp.w};
        const float2 st = actS[wbase + w];
#pragma unroll
        for (int t = 0; t < DF_RB; ++t) {
          if (t < nr) {
            const uint32_t qw = *reinterpret_cast<const uint32_t*>(q0 + t * (K / 2) + 4 * w);
            float a0 = 0.f, a1 = 0.f;
            dot_word4(qw, p, a0, a1);
            acc[t] += bf16_to_f32(S0[t * (K / 64) + (w >> 3)]) * ((a0 + a1) - st.x) +
                      bf16_to_f32(B0[t * (K / 64) + (w >> 3)]) * st.y;
          }
        }
      }
#pragma unroll
      for (int t = 0; t < DF_RB; ++t) {
        const float v = warp_sum(acc[t]);
        if (lane == 0 && t < nr) part[(rbeg + t) * 9 + u] = v;
      }
    }
    __syncthreads();
    df_stamp(a, l, 11);
    for (int r = threadIdx.x; r < nrow; r += DF_THREADS) {
      float y = 0.f;
      for (int j = 0; j < k; ++j) y = fmaf(selg[j], part[r * 9 + j], y);
      y += part[r * 9 + k];
      const int o = o0 + r;
      a.h[o] = __ldcg(a.h + o) + y;
      if (a.y_trace) a.y_trace[static_cast<size_t>(l) * H + o] = f32_to_bf16(y);
    }
    df_stamp(a, l, 12);
    if (l + 1 < a.L) {
      __syncthreads();                     // staging area read out
      if (warp == 0) issue_phase_a(l + 1);
    }
    df_stamp(a, l, 13);
    if (l + 1 < a.L) grid_sync();
    df_stamp(a, l, 14);
  }
}

size_t decode_fused_smem() {
  return static_cast<size_t>(DF_RS) + static_cast<size_t>(DF_MAX_ACT / 8) * 24 + DF_MAX_H / 8 * 16 +
         DF_MAX_H / 32 * 8 + DF_MAX_ROWS * 9 * 4 + 32 * 4 + 8 * 4 + 8 * 4 +
         (DF_MAX_CHUNKS + 3) * sizeof(DfChunk) + (DF_MAX_CHUNKS + 3) * 8 + 128;
}

// Staging bytes a CTA needs for its routed chunks (worst case over CTAs), or
// -1 if more chunks than DF_MAX_CHUNKS.
inline long df_staging_need(int H, int I, int Is, int k, int G) {
  const int pairs = (k * I + G - 1) / G, rows = (H + G - 1) / G;
  const int nrg = (pairs + DF_RGC - 1) / DF_RGC + 1;
  if (nrg + k > DF_MAX_CHUNKS) return -1;
  const long rg = static_cast<long>(pairs) * H + static_cast<long>(nrg) * 4 * (DF_RGC * 2 * (H / 64) + 32);
  const long d = static_cast<long>(k) * (rows * (I / 2) + 2 * (rows * 2 * (I / 64) + 32));
  const long ds = static_cast<long>(rows) * (Is / 2) + 2 * (rows * 2 * (Is / 64) + 32);
  return rg + d + (ds > rg ? ds + 128 : 0);
}

}  // namespace moe
