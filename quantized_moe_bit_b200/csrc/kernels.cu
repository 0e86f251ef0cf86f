// CUDA-core kernels of the routed-MoE layer: RMS norm (A0), router + top-k
// (A1, A2), bucketing (A3), expert and shared-expert GEMVs (A4 - A6) and the
// combine (A7).
#include <cooperative_groups.h>

#include "gemv.cuh"
#include "kernels.cuh"

namespace cg = cooperative_groups;

namespace moe {


// ------------------------------------------------------------------------ A0
// One block per row; fixed-order fp32 sum of squares; x = bf16_rn(h / r).
__global__ void k_rmsnorm(const float* __restrict__ h, int H, float eps, uint16_t* __restrict__ x) {
  const int t = blockIdx.x;
  const float* row = h + static_cast<size_t>(t) * H;
  float ss = 0.f;
  for (int c = threadIdx.x; c < H; c += blockDim.x) ss = fmaf(row[c], row[c], ss);
  __shared__ float red[32];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    v = warp_sum(v);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float r = sqrtf(red[0] / static_cast<float>(H) + eps);
  for (int c = threadIdx.x; c < H; c += blockDim.x)
    x[static_cast<size_t>(t) * H + c] = f32_to_bf16(__fdiv_rn(row[c], r));
}

// --------------------------------------------------------------------- A1+A2
// Cluster of 8 CTAs per block of ROUTER_TB rows (tokens).  CTA rank r owns
// experts [r*E/8, (r+1)*E/8): its logits for those rows come from the tensor
// cores (mma.sync m16n8k16, fp16 operands, fp32 accumulate) and go into rank
// 0's shared memory; after the cluster barrier rank 0 selects the top k per
// row (one warp per row) and applies the softmax.
//
// Operands.  x is staged as "byte-paired" half2: word m of a chunk of 16
// elements (elements 4m..4m+3) holds P0 = (v0, v2), P1 = (v1, v3).  A lane
// (g, t) of an mma reads 16 code bytes of expert row g (and g+8): chunk
// 4 grp + t of the quantisation group; in k-step j it uses the bytes of word
// j, the even ones (1024 + b made exact fp16, minus 1024) as k-slots 2t, 2t+1
// and the odd ones as 2t+8, 2t+9 -- the order P0 / P1 of word j of the same
// chunk give the B fragment, so every product pairs a code with its own x
// value.  The four k-steps of a group (64 inputs) give the exact-product fp32
// dot d; then logit += S d + B sum(x of the group).
// Warps split the CTA's experts in m-tiles of 16 and the groups in slices;
// the slices' partial logits are added in slice order.
__device__ __forceinline__ void mma_16816_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// (1024 + b) as fp16 for bytes 0 and 2 (odd = false) or 1 and 3 of w, minus 1024: exact b
__device__ __forceinline__ uint32_t router_pair(uint32_t w, bool odd) {
  const uint32_t h = ((odd ? w >> 8 : w) & 0x00FF00FFu) | 0x64006400u;
  const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&h), __floats2half2_rn(1024.f, 1024.f));
  return *reinterpret_cast<const uint32_t*>(&r);
}

__global__ void __cluster_dims__(8, 1, 1) __launch_bounds__(ROUTER_THREADS)
k_router_topk(const uint16_t* __restrict__ x, int T, int H, const uint32_t* __restrict__ rq,
              const uint16_t* __restrict__ rs, const uint16_t* __restrict__ rb,
              const float* __restrict__ bias, int bias_per_row, int E, int k,
              int32_t* __restrict__ idx, float* __restrict__ gates, float* __restrict__ logits_out) {
  extern __shared__ __align__(16) unsigned char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int row0 = (blockIdx.x / 8) * ROUTER_TB;
  const int nrows = min(ROUTER_TB, T - row0);
  const int nch = H / 16, NG = H / 64;
  const RouterSmem L = router_smem_layout(H, E);
  cluster.barrier_arrive();       // waited on before the first write into rank 0's shared memory
  float* lg = reinterpret_cast<float*>(smem + L.lg);           // [TB][E] (rank 0's is the cluster's)
  unsigned char* xs = smem + L.xs;                             // per row: P uint2 [4][nch]
  float* xg = reinterpret_cast<float*>(smem + L.xg);           // [TB][NG] group sums of the staged x
  float* part = reinterpret_cast<float*>(smem + L.part);       // [8 warps][TB][16] partial logits
  const size_t row_bytes = L.row_bytes;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
  const int nwarp = blockDim.x >> 5;

  // this warp: m-tile mt of the CTA's experts, group slice ks; its first
  // batch of codes and scales is requested before x is staged
  const int epc = E / 8;
  const int nmt = (epc + 15) / 16, nks = (ROUTER_THREADS / 32) / nmt;
  const int mt = warp % nmt, ks = warp / nmt;
  const bool active_w = ks < nks;
  const int g0 = active_w ? ks * NG / nks : 0, g1 = active_w ? (ks + 1) * NG / nks : 0;
  const int ea = mt * 16 + gq, eb = ea + 8;               // the lane's two experts (CTA-local)
  const bool oka = ea < epc, okb = eb < epc;
  const int Ea = rank * epc + ea, Eb = rank * epc + eb;
  const uint8_t* qa = reinterpret_cast<const uint8_t*>(rq) + static_cast<size_t>(oka ? Ea : 0) * H + 16 * tq;
  const uint8_t* qb = reinterpret_cast<const uint8_t*>(rq) + static_cast<size_t>(okb ? Eb : 0) * H + 16 * tq;
  const uint16_t* sa = rs + static_cast<size_t>(oka ? Ea : 0) * NG;
  const uint16_t* ba = rb + static_cast<size_t>(oka ? Ea : 0) * NG;
  const uint16_t* sb = rs + static_cast<size_t>(okb ? Eb : 0) * NG;
  const uint16_t* bb = rb + static_cast<size_t>(okb ? Eb : 0) * NG;
  uint4 wa[ROUTER_GB], wb[ROUTER_GB];
  float s4[ROUTER_GB][4];
  auto load_batch = [&](int gb) {
#pragma unroll
    for (int u = 0; u < ROUTER_GB; ++u) {
      const int g = gb + u;
      const bool in = g < g1;
      wa[u] = (in && oka) ? ldg_nc_v4(qa + 64 * static_cast<size_t>(g)) : make_uint4(0u, 0u, 0u, 0u);
      wb[u] = (in && okb) ? ldg_nc_v4(qb + 64 * static_cast<size_t>(g)) : make_uint4(0u, 0u, 0u, 0u);
      s4[u][0] = (in && oka) ? bf16_to_f32(ldg_u16(sa + g)) : 0.f;
      s4[u][1] = (in && oka) ? bf16_to_f32(ldg_u16(ba + g)) : 0.f;
      s4[u][2] = (in && okb) ? bf16_to_f32(ldg_u16(sb + g)) : 0.f;
      s4[u][3] = (in && okb) ? bf16_to_f32(ldg_u16(bb + g)) : 0.f;
    }
  };
  load_batch(g0);

  // stage x rows (zeros past the last row), ROUTER_XB chunks per thread per batch
  const int nitems = ROUTER_TB * nch;
  for (int i0 = threadIdx.x; i0 < nitems; i0 += blockDim.x * ROUTER_XB) {
    uint4 u[ROUTER_XB][2];
#pragma unroll
    for (int j = 0; j < ROUTER_XB; ++j) {
      const int i = i0 + j * static_cast<int>(blockDim.x);
      u[j][0] = u[j][1] = make_uint4(0u, 0u, 0u, 0u);
      if (i < nitems && i / nch < nrows) {
        const int r = i / nch, c = i - r * nch;
        const uint16_t* src = x + static_cast<size_t>(row0 + r) * H + 16 * c;
        u[j][0] = *reinterpret_cast<const uint4*>(src);
        u[j][1] = *reinterpret_cast<const uint4*>(src + 8);
      }
    }
#pragma unroll
    for (int j = 0; j < ROUTER_XB; ++j) {
      const int i = i0 + j * static_cast<int>(blockDim.x);
      float sum = 0.f;
      if (i < nitems) {
        const int r = i / nch, c = i - r * nch;
        uint2* P = reinterpret_cast<uint2*>(xs + r * row_bytes);
        const uint32_t w[8] = {u[j][0].x, u[j][0].y, u[j][0].z, u[j][0].w, u[j][1].x, u[j][1].y, u[j][1].z, u[j][1].w};
#pragma unroll
        for (int m = 0; m < 4; ++m) {          // word m covers elements 4m..4m+3
          const float v0 = __uint_as_float(w[2 * m] << 16), v1 = __uint_as_float(w[2 * m] & 0xFFFF0000u);
          const float v2 = __uint_as_float(w[2 * m + 1] << 16), v3 = __uint_as_float(w[2 * m + 1] & 0xFFFF0000u);
          const uint32_t p0 = pack_half2(v0, v2), p1 = pack_half2(v1, v3);
          P[m * nch + c] = make_uint2(p0, p1);
          const float2 f0 = unpack_half2(p0), f1 = unpack_half2(p1);
          sum += (f0.x + f0.y) + (f1.x + f1.y);
        }
      }
      // a group's four chunks are items 4q .. 4q+3 of a row (nch % 4 == 0),
      // held by four consecutive lanes: their sums meet in the first
      sum += __shfl_down_sync(0xffffffffu, sum, 1);
      sum += __shfl_down_sync(0xffffffffu, sum, 2);
      if (i < nitems && (i % nch) % 4 == 0) xg[(i / nch) * NG + (i % nch) / 4] = sum;
    }
  }
  __syncthreads();

  if (active_w) {
    float acc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
    for (int gb = g0; gb < g1; gb += ROUTER_GB) {
      if (gb != g0) load_batch(gb);            // the first batch came before the staging
#pragma unroll
      for (int u = 0; u < ROUTER_GB; ++u) {
        const int g = gb + u;
        if (g < g1) {
          float d[2][4];
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) d[nt][i] = 0.f;
          const uint32_t qwa[4] = {wa[u].x, wa[u].y, wa[u].z, wa[u].w};
          const uint32_t qwb[4] = {wb[u].x, wb[u].y, wb[u].z, wb[u].w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t af[4] = {router_pair(qwa[j], false), router_pair(qwb[j], false),
                                    router_pair(qwa[j], true), router_pair(qwb[j], true)};
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
              const uint2 P = reinterpret_cast<const uint2*>(xs + (nt * 8 + gq) * row_bytes)[j * nch + 4 * g + tq];
              mma_16816_f16(d[nt], af, P.x, P.y);
            }
          }
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            const float xa = xg[(nt * 8 + 2 * tq) * NG + g], xb = xg[(nt * 8 + 2 * tq + 1) * NG + g];
            acc[nt][0] += s4[u][0] * d[nt][0] + s4[u][1] * xa;
            acc[nt][1] += s4[u][0] * d[nt][1] + s4[u][1] * xb;
            acc[nt][2] += s4[u][2] * d[nt][2] + s4[u][3] * xa;
            acc[nt][3] += s4[u][2] * d[nt][3] + s4[u][3] * xb;
          }
        }
      }
    }
    // partial logits of (row, expert) into the warp's slot
    float* pw = part + warp * (ROUTER_TB * 16);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int ra = nt * 8 + 2 * tq;
      pw[ra * 16 + gq] = acc[nt][0];
      pw[(ra + 1) * 16 + gq] = acc[nt][1];
      pw[ra * 16 + gq + 8] = acc[nt][2];
      pw[(ra + 1) * 16 + gq + 8] = acc[nt][3];
    }
  }
  __syncthreads();
  // the slices' sums, in slice order, plus the bias, into rank 0's logits
  // (every CTA of the cluster has started: the arrive above)
  cluster.barrier_wait();
  float* lg0 = cluster.map_shared_rank(lg, 0);
  for (int i = threadIdx.x; i < nmt * ROUTER_TB * 16; i += blockDim.x) {
    const int m = i / (ROUTER_TB * 16), rem = i - m * (ROUTER_TB * 16), r = rem / 16, el = rem % 16;
    const int e_loc = m * 16 + el;
    if (r < nrows && e_loc < epc) {
      float v = 0.f;
      for (int q = 0; q < nks; ++q) v += part[(q * nmt + m) * (ROUTER_TB * 16) + r * 16 + el];
      const int e = rank * epc + e_loc;
      float bbv = 0.f;
      if (bias != nullptr) bbv = bias_per_row ? bias[static_cast<size_t>(row0 + r) * E + e] : bias[e];
      lg0[r * E + e] = v + bbv;
    }
  }
  cluster.sync();
  if (rank != 0) return;

  // top-k + softmax, one warp per row
  for (int r = warp; r < nrows; r += nwarp) {
    const int t = row0 + r;
    const float* L = lg + r * E;
    if (logits_out != nullptr)
      for (int e = lane; e < E; e += 32) logits_out[static_cast<size_t>(t) * E + e] = L[e];
    // each lane holds experts lane, lane+32, ...; taken experts are marked in a bit mask
    unsigned taken = 0u;
    float sel[8];
    int sid[8];
    for (int j = 0; j < k; ++j) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
      for (int s = 0, e = lane; e < E; ++s, e += 32) {
        if (taken & (1u << s)) continue;
        const float v = L[e];
        if (v > bv || (v == bv && e < bi)) { bv = v; bi = e; }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
      }
      if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
      sel[j] = bv;
      sid[j] = bi;
    }
    if (lane == 0) {
      float z[8], den = 0.f;
      for (int j = 0; j < k; ++j) { z[j] = expf(sel[j] - sel[0]); den += z[j]; }
      for (int j = 0; j < k; ++j) {
        idx[static_cast<size_t>(t) * k + j] = sid[j];
        gates[static_cast<size_t>(t) * k + j] = z[j] / den;
      }
    }
  }
}

// ------------------------------------------------------------------------ A3
// One block of BUCKET_THREADS.  Warp w owns the pairs [w n / W, (w+1) n / W)
// (W warps): it counts them per expert (order-free shared atomics into its
// own histogram row), then, after an exclusive scan over (expert, warp),
// places them in index order from its own start offsets -- so the pairs of
// every expert come out in index order (stable) with all warps placing at
// once.  Pair indices are loaded BUCKET_B chunks of 32 at a time.
__global__ void __launch_bounds__(BUCKET_THREADS)
k_bucket(const int32_t* __restrict__ idx, int n, int E, int32_t* __restrict__ offsets,
         int32_t* __restrict__ pairs, int32_t* __restrict__ active, int32_t* __restrict__ n_active) {
  extern __shared__ int sh[];
  constexpr int W = BUCKET_THREADS / 32;
  int* hist = sh;           // [W][E]: counts, then start offsets
  int* tot = sh + W * E;    // [E]: counts, then expert offsets
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < W * E; i += BUCKET_THREADS) hist[i] = 0;
  __syncthreads();
  const int p0 = static_cast<int>(static_cast<long>(n) * warp / W);
  const int p1 = static_cast<int>(static_cast<long>(n) * (warp + 1) / W);
  int* h = hist + warp * E;
  for (int q0 = p0; q0 < p1; q0 += 32 * BUCKET_B) {
    int ev[BUCKET_B];
#pragma unroll
    for (int b = 0; b < BUCKET_B; ++b) {
      const int p = q0 + 32 * b + lane;
      ev[b] = p < p1 ? idx[p] : -1;
    }
#pragma unroll
    for (int b = 0; b < BUCKET_B; ++b) {
      const int p = q0 + 32 * b + lane;
      if (p < p1) {
        if (ev[b] >= 0 && ev[b] < E) atomicAdd(&h[ev[b]], 1);
        else flag_check(CHECK_EXPERT_ID);
      }
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += BUCKET_THREADS) {
    int c = 0;
    for (int w = 0; w < W; ++w) c += hist[w * E + e];
    tot[e] = c;
  }
  __syncthreads();
  if (warp == 0) {
    // warp scan over E in chunks of 32: expert offsets and the active list
    int base = 0, abase = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      const int v = e < E ? tot[e] : 0;
      const int a = v > 0 ? 1 : 0;
      int incl = v, ainc = a;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t1 = __shfl_up_sync(0xffffffffu, incl, o);
        const int t2 = __shfl_up_sync(0xffffffffu, ainc, o);
        if (lane >= o) { incl += t1; ainc += t2; }
      }
      if (e < E) {
        offsets[e] = base + incl - v;
        tot[e] = base + incl - v;
        if (a) active[abase + ainc - 1] = e;
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
      abase += __shfl_sync(0xffffffffu, ainc, 31);
    }
    if (lane == 0) {
      offsets[E] = base;
      *n_active = abase;
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += BUCKET_THREADS) {
    int s = tot[e];
    for (int w = 0; w < W; ++w) {
      const int c = hist[w * E + e];
      hist[w * E + e] = s;
      s += c;
    }
  }
  __syncthreads();
  for (int q0 = p0; q0 < p1; q0 += 32 * BUCKET_B) {
    int ev[BUCKET_B];
#pragma unroll
    for (int b = 0; b < BUCKET_B; ++b) {
      const int p = q0 + 32 * b + lane;
      ev[b] = p < p1 ? idx[p] : -1;
    }
#pragma unroll
    for (int b = 0; b < BUCKET_B; ++b) {
      const int p = q0 + 32 * b + lane;
      const int e = ev[b];
      const bool ok = p < p1 && e >= 0 && e < E;
      const unsigned m = __match_any_sync(0xffffffffu, ok ? e : -1);
      if (ok) pairs[h[e] + __popc(m & ((1u << lane) - 1u))] = p;
      __syncwarp();
      if (ok && (__ffs(m) - 1) == lane) h[e] += __popc(m);
      __syncwarp();
    }
  }
}

// ---------------------------------------------------------------- A4 / A6 up
// Gate/up projections + GeGLU for bucket rows, GEMV form.
// blockIdx.y = active-expert slot (routed) or 0 (shared); blockIdx.x = block
// of GEMV_ROWS intermediate rows.  Bucket rows are processed RG at a time from
// shared memory.  act[row] (fp16) is written at the bucket position.
__global__ void __launch_bounds__(256)
k_gateup_gemv(GateUpArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  int e = 0, pos0 = 0, cnt = a.T;
  const uint8_t *gq, *uq;
  const uint16_t *gs, *gb, *us, *ub;
  if (a.blob_ptrs != nullptr) {
    if (static_cast<int>(blockIdx.y) >= *a.n_active) return;
    e = a.active[blockIdx.y];
    if (e < 0 || e >= a.E) { flag_check(CHECK_EXPERT_ID); return; }
    pos0 = a.offsets[e];
    cnt = a.offsets[e + 1] - pos0;
    if (cnt > a.max_rows) return;
    const uint8_t* blob = static_cast<const uint8_t*>(a.blob_ptrs[e]);
    gq = blob + a.off[0]; gs = reinterpret_cast<const uint16_t*>(blob + a.off[1]);
    gb = reinterpret_cast<const uint16_t*>(blob + a.off[2]);
    uq = blob + a.off[3]; us = reinterpret_cast<const uint16_t*>(blob + a.off[4]);
    ub = reinterpret_cast<const uint16_t*>(blob + a.off[5]);
  } else {
    gq = reinterpret_cast<const uint8_t*>(a.gq); gs = a.gs; gb = a.gb;
    uq = reinterpret_cast<const uint8_t*>(a.uq); us = a.us; ub = a.ub;
  }
  const int K = a.H, nch = K / 32, N = a.I;
  float2* scratch = reinterpret_cast<float2*>(smem + GEMV_RG * staged_row_bytes(K));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarp = blockDim.x >> 5;
  const int i0 = blockIdx.x * GEMV_ROWS;
  for (int g0 = 0; g0 < cnt; g0 += GEMV_RG) {
    const int nr = min(GEMV_RG, cnt - g0);
    if (g0 > 0) __syncthreads();
    stage_rows4<uint16_t>(smem, scratch, K, nr, [&](int r) -> const uint16_t* {
      int tok;
      if (a.pairs != nullptr) {
        const int p = a.pairs[pos0 + g0 + r];
        tok = p / a.k;
      } else {
        tok = g0 + r;
      }
      if (tok < 0 || tok >= a.T) { flag_check(CHECK_PAIR_ID); return nullptr; }
      return a.x + static_cast<size_t>(tok) * K;
    });
    for (int i = i0 + warp; i < min(i0 + GEMV_ROWS, N); i += nwarp) {
      float av[GEMV_RG], uv[GEMV_RG];
      row_dot4<GEMV_RG>(gq + static_cast<size_t>(i) * (K / 2), gs + static_cast<size_t>(i) * (K / 64),
                        gb + static_cast<size_t>(i) * (K / 64), nch, smem, K, nr, av);
      row_dot4<GEMV_RG>(uq + static_cast<size_t>(i) * (K / 2), us + static_cast<size_t>(i) * (K / 64),
                        ub + static_cast<size_t>(i) * (K / 64), nch, smem, K, nr, uv);
      if (lane < nr) {
        float va = 0.f, vu = 0.f;
#pragma unroll
        for (int r = 0; r < GEMV_RG; ++r) if (r == lane) { va = av[r]; vu = uv[r]; }
        const float h = gelu_tanh(va) * vu;
        a.act[static_cast<size_t>(pos0 + g0 + lane) * N + i] = __float2half_rn(h);
      }
    }
  }
}

// ---------------------------------------------------------------- A5 / A6 down
// Down projection, GEMV form: y[dest(row)][o] = sum_i Wd[o, i] act[row][i].
// Routed: dest = pairs[pos] (row of y_pairs); shared: dest = row (ysh).
__global__ void __launch_bounds__(256)
k_down_gemv(DownArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  int e = 0, pos0 = 0, cnt = a.T;
  const uint8_t* dq;
  const uint16_t *ds, *db;
  if (a.blob_ptrs != nullptr) {
    if (static_cast<int>(blockIdx.y) >= *a.n_active) return;
    e = a.active[blockIdx.y];
    if (e < 0 || e >= a.E) { flag_check(CHECK_EXPERT_ID); return; }
    pos0 = a.offsets[e];
    cnt = a.offsets[e + 1] - pos0;
    if (cnt > a.max_rows) return;
    const uint8_t* blob = static_cast<const uint8_t*>(a.blob_ptrs[e]);
    dq = blob + a.off[6]; ds = reinterpret_cast<const uint16_t*>(blob + a.off[7]);
    db = reinterpret_cast<const uint16_t*>(blob + a.off[8]);
  } else {
    dq = reinterpret_cast<const uint8_t*>(a.dq); ds = a.ds; db = a.db;
  }
  const int K = a.I, nch = K / 32, N = a.H;
  float2* scratch = reinterpret_cast<float2*>(smem + GEMV_RG * staged_row_bytes(K));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarp = blockDim.x >> 5;
  const int o0 = blockIdx.x * GEMV_ROWS;
  for (int g0 = 0; g0 < cnt; g0 += GEMV_RG) {
    const int nr = min(GEMV_RG, cnt - g0);
    if (g0 > 0) __syncthreads();
    stage_rows4<__half>(smem, scratch, K, nr, [&](int r) -> const __half* {
      return a.act + static_cast<size_t>(pos0 + g0 + r) * K;
    });
    for (int o = o0 + warp; o < min(o0 + GEMV_ROWS, N); o += nwarp) {
      float yv[GEMV_RG];
      row_dot4<GEMV_RG>(dq + static_cast<size_t>(o) * (K / 2), ds + static_cast<size_t>(o) * (K / 64),
                        db + static_cast<size_t>(o) * (K / 64), nch, smem, K, nr, yv);
      if (lane < nr) {
        float v = 0.f;
#pragma unroll
        for (int r = 0; r < GEMV_RG; ++r) if (r == lane) v = yv[r];
        int dest = pos0 + g0 + lane;
        if (a.pairs != nullptr) dest = a.pairs[dest];
        a.y[static_cast<size_t>(dest) * N + o] = v;
      }
    }
  }
}

// ------------------------------------------------------------------------ A7
__global__ void k_combine(const float* __restrict__ yp, const float* __restrict__ gates,
                          const float* __restrict__ ysh, int H, int k, uint16_t* __restrict__ y,
                          const float* resid_in, float* resid_out) {
  const int t = blockIdx.y;
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= H) return;
  float g[8];
  for (int j = 0; j < k; ++j) g[j] = gates[static_cast<size_t>(t) * k + j];
  float acc = 0.f;
  for (int j = 0; j < k; ++j) acc = fmaf(g[j], yp[(static_cast<size_t>(t) * k + j) * H + c], acc);
  if (ysh != nullptr) acc += ysh[static_cast<size_t>(t) * H + c];
  if (y != nullptr) y[static_cast<size_t>(t) * H + c] = f32_to_bf16(acc);
  if (resid_out != nullptr) resid_out[static_cast<size_t>(t) * H + c] = resid_in[static_cast<size_t>(t) * H + c] + acc;
}

// (resid_out = resid_in + the sum: the residual add, in place when the two
// are the same array.)
// The same sum four columns per thread (16-byte aligned arrays, H % 4 == 0):
// the k pair rows are loaded before the fma chain, which runs in the same
// order (j = 0 .. k-1, then the shared row), so the result is bit-identical.
__global__ void __launch_bounds__(256)
k_combine4(const float* __restrict__ yp, const float* __restrict__ gates, const float* __restrict__ ysh, int H,
           int k, uint16_t* __restrict__ y, const float* resid_in, float* resid_out) {
  const int t = blockIdx.y;
  const int c = 4 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (c >= H) return;
  float g[8];
  float4 v[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j < k) {
      g[j] = gates[static_cast<size_t>(t) * k + j];
      v[j] = *reinterpret_cast<const float4*>(yp + (static_cast<size_t>(t) * k + j) * H + c);
    }
  }
  const float4 sh = ysh != nullptr ? *reinterpret_cast<const float4*>(ysh + static_cast<size_t>(t) * H + c)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j < k) {
      a0 = fmaf(g[j], v[j].x, a0);
      a1 = fmaf(g[j], v[j].y, a1);
      a2 = fmaf(g[j], v[j].z, a2);
      a3 = fmaf(g[j], v[j].w, a3);
    }
  }
  if (ysh != nullptr) {
    a0 += sh.x; a1 += sh.y; a2 += sh.z; a3 += sh.w;
  }
  const size_t o = static_cast<size_t>(t) * H + c;
  if (y != nullptr) {
    const uint2 pk = make_uint2(static_cast<uint32_t>(f32_to_bf16(a0)) | (static_cast<uint32_t>(f32_to_bf16(a1)) << 16),
                                static_cast<uint32_t>(f32_to_bf16(a2)) | (static_cast<uint32_t>(f32_to_bf16(a3)) << 16));
    *reinterpret_cast<uint2*>(y + o) = pk;
  }
  if (resid_out != nullptr) {
    float4 r = *reinterpret_cast<const float4*>(resid_in + o);
    r.x += a0; r.y += a1; r.z += a2; r.w += a3;
    *reinterpret_cast<float4*>(resid_out + o) = r;
  }
}

}  // namespace moe
