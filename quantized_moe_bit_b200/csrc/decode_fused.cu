// Batch-1 decode of a stack of routed-MoE layers in one persistent kernel.
//
// One launch runs every layer of the step.  The grid is a set of 8-CTA
// clusters, one CTA per SM, launched cooperatively (all CTAs resident).  Per
// layer:
//   phase A  every CTA computes the RMS norm of the residual h (redundantly,
//            same order, same result); its share of the shared expert's
//            gate/up rows; then the router: CTA rank r of each cluster
//            computes the logits of experts [r*E/8, (r+1)*E/8), the cluster
//            exchanges them through distributed shared memory, and every CTA
//            selects the top k itself -- no grid-wide step for routing.  Each
//            CTA then computes its share of the routed experts' gate/up rows
//            (a contiguous slice of the k*I (slot, row) pairs) and writes the
//            fp16 activations.
//   barrier  hierarchical grid barrier (cluster barrier, one atomic per
//            cluster, cluster barrier).
//   phase C  every CTA stages all activations (k*I + Is fp16) in shared
//            memory and computes its slice of output rows: per row the k
//            routed down dots and the shared down dot, combined in a fixed
//            order, y = sum_j g_j y_j + ysh; h += y.
//   barrier
// Memory traffic is driven by bulk L2 prefetches issued as soon as the
// addresses are known: after the top-k, a CTA prefetches its routed gate/up
// rows and its phase-C down rows; at the start of phase C it prefetches the
// next layer's routing-independent data (router slice, shared-expert rows)
// and slices of the experts most likely to be chosen (largest router bias),
// so HBM stays busy while the next layer waits for its routing.
// Every wait is bounded (about two seconds); a wait that runs out sets the
// device check word and the kernel runs on to its end.
#include <cooperative_groups.h>

namespace moe {

constexpr int DF_THREADS = 384;
constexpr int DF_WARPS = DF_THREADS / 32;
constexpr int DF_CLUSTER = 8;
constexpr int DF_MAX_LAYERS = 48;
constexpr int DF_MAX_H = 4096;
constexpr int DF_MAX_ACT = 16384;      // k*I + Is
constexpr int DF_MAX_ROWS = 64;        // output rows per CTA in phase C
constexpr int DF_MAX_UNITS = 16;       // down dots per output row (k + shared pieces)

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
  DfLayer layer[DF_MAX_LAYERS];
};

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

// L2 prefetch of [p, p + bytes): the 16-byte-aligned window around it (arrays
// handed to this kernel are 16-byte aligned with sizes that are multiples of
// 16, so the window stays inside them).
__device__ __forceinline__ void prefetch_l2(const void* p, size_t bytes) {
  if (bytes == 0) return;
  uintptr_t a = reinterpret_cast<uintptr_t>(p) & ~uintptr_t(15);
  uintptr_t e = (reinterpret_cast<uintptr_t>(p) + bytes + 15) & ~uintptr_t(15);
  while (a < e) {
    const uint32_t n = static_cast<uint32_t>((e - a) < 65536 ? (e - a) : 65536);
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a), "r"(n) : "memory");
    a += n;
  }
}

// Slice c of G of an array of `total` bytes (total a multiple of 16).
__device__ __forceinline__ void prefetch_slice(const void* base, size_t total, int c, int G) {
  const size_t b0 = total * c / G, b1 = total * (c + 1) / G;
  prefetch_l2(static_cast<const uint8_t*>(base) + b0, b1 - b0);
}

__device__ __forceinline__ uint4 ldcg_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}
__device__ __forceinline__ uint32_t ldg_nc_u32(const void* p) {
  uint32_t r;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}

// Hierarchical grid barrier: cluster barrier; one thread per cluster adds to
// the counter and waits for all clusters; cluster barrier.  `target` grows by
// the number of clusters at every barrier of the launch.
__device__ void df_grid_sync(cooperative_groups::cluster_group& cl, unsigned* ctr, unsigned target) {
  cl.sync();
  if (cl.block_rank() == 0 && threadIdx.x == 0) {
    __threadfence();
    red_release_gpu(ctr, 1u);
    const uint64_t t0 = df_clock();
    while (ld_acquire_gpu(ctr) < target) {
      if (df_clock() - t0 > 2000000000ull) { flag_check(CHECK_WAIT); break; }
    }
    __threadfence();
  }
  cl.sync();
  if (threadIdx.x == 0) __threadfence();
  __syncthreads();
}

// One row-pair (gate row i, up row i) against the register x; returns
// act = gelu_tanh(gate . x) * (up . x) in every lane.
template <int DF_CPL>
__device__ __forceinline__ float df_gateup_row(const uint8_t* gq, const uint16_t* gs, const uint16_t* gb,
                                               const uint8_t* uq, const uint16_t* us, const uint16_t* ub,
                                               int i, int K, int nch, const uint32_t (&xp)[DF_CPL][16],
                                               const float2 (&xst)[DF_CPL]) {
  const int lane = threadIdx.x & 31;
  const size_t rq = static_cast<size_t>(i) * (K / 2), rsb = static_cast<size_t>(i) * (K / 64);
  uint4 qg[DF_CPL], qu[DF_CPL];
  float sg[DF_CPL], bg[DF_CPL], su[DF_CPL], bu[DF_CPL];
#pragma unroll
  for (int j = 0; j < DF_CPL; ++j) {
    const int c = lane + 32 * j;
    if (c < nch) {
      qg[j] = ldg_nc_v4(gq + rq + 16 * c);
      qu[j] = ldg_nc_v4(uq + rq + 16 * c);
      sg[j] = bf16_to_f32(ldg_u16(gs + rsb + (c >> 1)));
      bg[j] = bf16_to_f32(ldg_u16(gb + rsb + (c >> 1)));
      su[j] = bf16_to_f32(ldg_u16(us + rsb + (c >> 1)));
      bu[j] = bf16_to_f32(ldg_u16(ub + rsb + (c >> 1)));
    }
  }
  float a = 0.f, u = 0.f;
#pragma unroll
  for (int j = 0; j < DF_CPL; ++j) {
    const int c = lane + 32 * j;
    if (c < nch) {
      const float dg = dot_chunk4(qg[j], xp[j]);
      const float du = dot_chunk4(qu[j], xp[j]);
      a += sg[j] * (dg - xst[j].x) + bg[j] * xst[j].y;
      u += su[j] * (du - xst[j].x) + bu[j] * xst[j].y;
    }
  }
  a = warp_sum(a);
  u = warp_sum(u);
  return gelu_tanh(a) * u;
}

template <int DF_CPL>
__global__ void __cluster_dims__(DF_CLUSTER, 1, 1) __launch_bounds__(DF_THREADS, 1)
k_decode_b1(const __grid_constant__ DfArgs a) {
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  extern __shared__ __align__(16) unsigned char smem[];
  const int H = a.H, I = a.I, Is = a.Is, E = a.E, k = a.k;
  const int G = gridDim.x, c = blockIdx.x;
  const int rank = static_cast<int>(cl.block_rank());
  const unsigned nclusters = G / DF_CLUSTER;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kI = k * I, nact = kI + Is;

  // shared memory
  float* xs = reinterpret_cast<float*>(smem);                          // [H] layer input (bf16 values)
  float* red = xs + DF_MAX_H;                                          // [32] reduction scratch
  float* lg_part = red + 32;                                           // [E/8] this CTA's logits
  float* lg_all = lg_part + 128;                                       // [E]
  int* sel_idx = reinterpret_cast<int*>(lg_all + 1024);                // [8]
  float* sel_g = reinterpret_cast<float*>(sel_idx + 8);                // [8]
  int* spec_ids = reinterpret_cast<int*>(sel_g + 8);                   // [8]
  float* part = reinterpret_cast<float*>(spec_ids + 8);                // [DF_MAX_ROWS][DF_MAX_UNITS]
  uint4* actP = reinterpret_cast<uint4*>(part + DF_MAX_ROWS * DF_MAX_UNITS);  // [nact/8] paired words
  float2* actS = reinterpret_cast<float2*>(actP + DF_MAX_ACT / 8);     // [nact/8] (off, sum) per word

  // static work split
  const int s0 = (int)((long)c * Is / G), s1 = (int)((long)(c + 1) * Is / G);        // shared gate/up pairs
  const int r0 = (int)((long)c * kI / G), r1 = (int)((long)(c + 1) * kI / G);        // routed (slot, row)
  const int o0 = (int)((long)c * H / G), o1 = (int)((long)(c + 1) * H / G);          // output rows
  const int nsub = (Is + I - 1) / I;                                                 // shared down pieces
  const int upr = k + nsub;                                                          // units per row
  const int nch = H / 32;
  const int epc = E / DF_CLUSTER;
  unsigned bar_target = 0;

  // prefetch the routing-independent data of layer l (and likely experts)
  auto prefetch_independent = [&](int l) {
    const DfLayer& W = a.layer[l];
    if (threadIdx.x == 0) {
      // router: 1/G slice of the whole matrix (every cluster reads all of it)
      prefetch_slice(W.rq, static_cast<size_t>(E) * H, c, G);
    } else if (threadIdx.x == 32) {
      prefetch_slice(W.rs, static_cast<size_t>(E) * (H / 64) * 2, c, G);
      prefetch_slice(W.rb, static_cast<size_t>(E) * (H / 64) * 2, c, G);
    } else if (threadIdx.x == 64) {
      for (int m = 0; m < 2; ++m) {
        prefetch_l2(reinterpret_cast<const uint8_t*>(W.sq[m]) + static_cast<size_t>(s0) * (H / 2),
                    static_cast<size_t>(s1 - s0) * (H / 2));
        prefetch_l2(W.ss[m] + static_cast<size_t>(s0) * (H / 64), static_cast<size_t>(s1 - s0) * (H / 64) * 2);
        prefetch_l2(W.sb[m] + static_cast<size_t>(s0) * (H / 64), static_cast<size_t>(s1 - s0) * (H / 64) * 2);
      }
    } else if (threadIdx.x == 96) {
      prefetch_l2(reinterpret_cast<const uint8_t*>(W.sq[2]) + static_cast<size_t>(o0) * (Is / 2),
                  static_cast<size_t>(o1 - o0) * (Is / 2));
      prefetch_l2(W.ss[2] + static_cast<size_t>(o0) * (Is / 64), static_cast<size_t>(o1 - o0) * (Is / 64) * 2);
      prefetch_l2(W.sb[2] + static_cast<size_t>(o0) * (Is / 64), static_cast<size_t>(o1 - o0) * (Is / 64) * 2);
    } else if (warp == 4 && W.bias != nullptr && a.spec > 0) {
      // the experts with the largest router bias, 1/G of each blob
      int bi[8];
      for (int j = 0; j < 8; ++j) bi[j] = 0;
      unsigned taken = 0;
      for (int r = 0; r < a.spec; ++r) {
        float v = -INFINITY;
        int id = 0x7fffffff;
        for (int s = 0, e = lane; e < E; ++s, e += 32) {
          if (taken & (1u << s)) continue;
          const float b = W.bias[e];
          if (b > v || (b == v && e < id)) { v = b; id = e; }
        }
        for (int o = 16; o > 0; o >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, v, o);
          const int oi = __shfl_xor_sync(0xffffffffu, id, o);
          if (ov > v || (ov == v && oi < id)) { v = ov; id = oi; }
        }
        if ((id & 31) == lane) taken |= 1u << (id >> 5);
        bi[r] = id;
      }
      if (lane < a.spec) {
        const size_t bb = a.off[8] + static_cast<size_t>(H) * (I / 64) * 2;   // blob bytes
        prefetch_slice(W.blobs[bi[lane]], bb, c, G);
      }
    }
  };

  prefetch_independent(0);

  for (int l = 0; l < a.L; ++l) {
    const DfLayer& W = a.layer[l];
    // ------------------------------------------------------------- A0: rms norm
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

    // ------------------------------------------------------ router (cluster)
    for (int el = warp; el < epc; el += DF_WARPS) {
      const int e = rank * epc + el;
      const uint8_t* qrow = reinterpret_cast<const uint8_t*>(W.rq) + static_cast<size_t>(e) * H;
      float acc = 0.f;
      for (int cc = lane; cc < H / 16; cc += 32) {
        const uint4 q = ldg_nc_v4(qrow + 16 * cc);
        const float sc = bf16_to_f32(ldg_u16(W.rs + static_cast<size_t>(e) * (H / 64) + (cc >> 2)));
        const float bi = bf16_to_f32(ldg_u16(W.rb + static_cast<size_t>(e) * (H / 64) + (cc >> 2)));
        const float* xv = xs + 16 * cc;
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
        float a0 = 0.f, a1 = 0.f, off = 0.f;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const uint32_t p[2] = {pack_half2(xv[4 * m], xv[4 * m + 2]), pack_half2(xv[4 * m + 1], xv[4 * m + 3])};
          dot_word8(w[m], p, a0, a1);
          const float2 f0 = unpack_half2(p[0]), f1 = unpack_half2(p[1]);
          off += (f0.x + f0.y) + (f1.x + f1.y);
        }
        acc += sc * ((a0 + a1) - 1024.f * off) + bi * off;
      }
      acc = warp_sum(acc);
      if (lane == 0) lg_part[el] = acc + (W.bias ? W.bias[e] : 0.f);
    }
    cl.sync();
    for (int e = threadIdx.x; e < E; e += DF_THREADS) {
      const float* src = cl.map_shared_rank(lg_part, e / epc);
      lg_all[e] = src[e % epc];
    }
    cl.sync();
    if (warp == 0) {
      unsigned taken = 0u;
      float sv[8];
      int si[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j >= k) break;
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        for (int s = 0, e = lane; e < E; ++s, e += 32) {
          if (taken & (1u << s)) continue;
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
      if (lane == 0) {
        float z[8], den = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) { z[j] = j < k ? expf(sv[j] - sv[0]) : 0.f; den += z[j]; }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (j >= k) break;
          sel_idx[j] = si[j];
          sel_g[j] = z[j] / den;
          if (c == 0 && a.idx_trace) a.idx_trace[static_cast<size_t>(l) * k + j] = si[j];
          if (c == 0 && a.gates_trace) a.gates_trace[static_cast<size_t>(l) * k + j] = z[j] / den;
        }
      }
    }
    __syncthreads();

    // prefetch this CTA's routed rows (gate/up slice and phase-C down rows)
    if (warp == 1) {
      for (int j = lane; j < k; j += 32) {
        const uint8_t* blob = static_cast<const uint8_t*>(W.blobs[sel_idx[j]]);
        prefetch_l2(blob + a.off[6] + static_cast<size_t>(o0) * (I / 2), static_cast<size_t>(o1 - o0) * (I / 2));
        prefetch_l2(blob + a.off[7] + static_cast<size_t>(o0) * (I / 64) * 2, static_cast<size_t>(o1 - o0) * (I / 64) * 2);
        prefetch_l2(blob + a.off[8] + static_cast<size_t>(o0) * (I / 64) * 2, static_cast<size_t>(o1 - o0) * (I / 64) * 2);
      }
    } else if (warp == 2 && lane < 2) {
      // gate/up slice [r0, r1) of the flattened (slot, row) list: at most a few slots
      for (int j = r0 / I; j <= (r1 - 1) / I && j < k; ++j) {
        const int i0 = max(r0 - j * I, 0), i1 = min(r1 - j * I, I);
        const uint8_t* blob = static_cast<const uint8_t*>(W.blobs[sel_idx[j]]);
        const int m = lane;   // 0 gate, 1 up
        prefetch_l2(blob + a.off[3 * m] + static_cast<size_t>(i0) * (H / 2), static_cast<size_t>(i1 - i0) * (H / 2));
        prefetch_l2(blob + a.off[3 * m + 1] + static_cast<size_t>(i0) * (H / 64) * 2, static_cast<size_t>(i1 - i0) * (H / 64) * 2);
        prefetch_l2(blob + a.off[3 * m + 2] + static_cast<size_t>(i0) * (H / 64) * 2, static_cast<size_t>(i1 - i0) * (H / 64) * 2);
      }
    }

    // register copy of x in the nibble-paired layout for this lane's chunks
    uint32_t xp[DF_CPL][16];
    float2 xst[DF_CPL];
#pragma unroll
    for (int j = 0; j < DF_CPL; ++j) {
      const int cc = lane + 32 * j;
      float off = 0.f, sum = 0.f;
      if (cc < nch) {
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          float v[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) v[t] = xs[32 * cc + 8 * m + t];
          uint32_t p[4];
          pair_word4(v, p);
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            xp[j][4 * m + t] = p[t];
            const float2 f = unpack_half2(p[t]);
            off += f.x + f.y;
          }
          const float2 f0 = unpack_half2(p[0]), f1 = unpack_half2(p[1]), f2 = unpack_half2(p[2]), f3 = unpack_half2(p[3]);
          sum += (f0.x + f0.y + f2.x + f2.y) + 16.f * (f1.x + f1.y + f3.x + f3.y);
        }
      } else {
#pragma unroll
        for (int t = 0; t < 16; ++t) xp[j][t] = 0u;
      }
      xst[j] = make_float2(1024.f * off, sum);
    }

    // ---------------------------------------------- shared-expert gate/up share
    for (int i = s0 + warp; i < s1; i += DF_WARPS) {
      const float v = df_gateup_row<DF_CPL>(reinterpret_cast<const uint8_t*>(W.sq[0]), W.ss[0], W.sb[0],
                                    reinterpret_cast<const uint8_t*>(W.sq[1]), W.ss[1], W.sb[1], i, H, nch, xp, xst);
      if (lane == 0) a.act[kI + i] = __float2half_rn(v);
    }

    // ------------------------------------------------- routed gate/up share
    for (int rr2 = r0 + warp; rr2 < r1; rr2 += DF_WARPS) {
      const int j = rr2 / I, i = rr2 - j * I;
      const uint8_t* blob = static_cast<const uint8_t*>(W.blobs[sel_idx[j]]);
      const float v = df_gateup_row<DF_CPL>(blob + a.off[0], reinterpret_cast<const uint16_t*>(blob + a.off[1]),
                                    reinterpret_cast<const uint16_t*>(blob + a.off[2]), blob + a.off[3],
                                    reinterpret_cast<const uint16_t*>(blob + a.off[4]),
                                    reinterpret_cast<const uint16_t*>(blob + a.off[5]), i, H, nch, xp, xst);
      if (lane == 0) a.act[rr2] = __float2half_rn(v);
    }

    bar_target += nclusters;
    df_grid_sync(cl, a.counter, bar_target);

    // ------------------------------------------------------------- phase C
    if (l + 1 < a.L) prefetch_independent(l + 1);
    // stage all activations (written by every CTA) in the nibble-paired layout
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
      for (int t = 0; t < 4; ++t) { const float2 f = unpack_half2(p[t]); off += f.x + f.y; }
      const float2 f0 = unpack_half2(p[0]), f1 = unpack_half2(p[1]), f2 = unpack_half2(p[2]), f3 = unpack_half2(p[3]);
      actS[w] = make_float2(1024.f * off, (f0.x + f0.y + f2.x + f2.y) + 16.f * (f1.x + f1.y + f3.x + f3.y));
    }
    __syncthreads();
    // units: (row o, piece u): u < k routed slot u (K = I); u >= k shared piece u-k
    const int nrow = o1 - o0;
    for (int un = warp; un < nrow * upr; un += DF_WARPS) {
      const int ro = un / upr, u = un - ro * upr, o = o0 + ro;
      const uint8_t* q;
      const uint16_t *sp, *bp;
      int wbase, nw;                   // first act word, words in this piece
      if (u < k) {
        const uint8_t* blob = static_cast<const uint8_t*>(W.blobs[sel_idx[u]]);
        q = blob + a.off[6] + static_cast<size_t>(o) * (I / 2);
        sp = reinterpret_cast<const uint16_t*>(blob + a.off[7]) + static_cast<size_t>(o) * (I / 64);
        bp = reinterpret_cast<const uint16_t*>(blob + a.off[8]) + static_cast<size_t>(o) * (I / 64);
        wbase = u * (I / 8);
        nw = I / 8;
      } else {
        const int pc = u - k;
        const int c0 = pc * I, c1 = min(Is, c0 + I);
        q = reinterpret_cast<const uint8_t*>(W.sq[2]) + static_cast<size_t>(o) * (Is / 2) + c0 / 2;
        sp = W.ss[2] + static_cast<size_t>(o) * (Is / 64) + c0 / 64;
        bp = W.sb[2] + static_cast<size_t>(o) * (Is / 64) + c0 / 64;
        wbase = (kI + c0) / 8;
        nw = (c1 - c0) / 8;
      }
      float acc = 0.f;
      for (int w = lane; w < nw; w += 32) {
        const uint32_t qw = ldg_nc_u32(q + 4 * w);
        const float sc = bf16_to_f32(ldg_u16(sp + (w >> 3)));
        const float bi = bf16_to_f32(ldg_u16(bp + (w >> 3)));
        const uint4 pp = actP[wbase + w];
        const uint32_t p[4] = {pp.x, pp.y, pp.z, pp.w};
        float a0 = 0.f, a1 = 0.f;
        dot_word4(qw, p, a0, a1);
        const float2 st = actS[wbase + w];
        acc += sc * ((a0 + a1) - st.x) + bi * st.y;
      }
      acc = warp_sum(acc);
      if (lane == 0) part[ro * DF_MAX_UNITS + u] = acc;
    }
    __syncthreads();
    for (int ro = threadIdx.x; ro < nrow; ro += DF_THREADS) {
      float y = 0.f;
      for (int j = 0; j < k; ++j) y = fmaf(sel_g[j], part[ro * DF_MAX_UNITS + j], y);
      float ys = 0.f;
      for (int pc = 0; pc < nsub; ++pc) ys += part[ro * DF_MAX_UNITS + k + pc];
      y += ys;
      const int o = o0 + ro;
      a.h[o] = __ldcg(a.h + o) + y;
      if (a.y_trace) a.y_trace[static_cast<size_t>(l) * H + o] = f32_to_bf16(y);
    }
    if (l + 1 < a.L) {
      bar_target += nclusters;
      df_grid_sync(cl, a.counter, bar_target);
    }
  }
}

size_t decode_fused_smem(int H, int nact) {
  (void)H; (void)nact;
  return (DF_MAX_H + 32 + 128 + 1024 + 24) * 4 + DF_MAX_ROWS * DF_MAX_UNITS * 4 +
         static_cast<size_t>(DF_MAX_ACT / 8) * (16 + 8) + 64;
}

}  // namespace moe
