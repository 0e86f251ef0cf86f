// Dequant-fused grouped GEMM of the routed experts on the 5th-generation
// tensor cores (tcgen05 + TMEM), for buckets of several rows (prefill chunks,
// batched decode).
//
// Swap-AB: the weight rows are the MMA's M = 128 side and the bucket's tokens
// the N side (N <= 128, padded to a multiple of 16), so one expert's weights
// serve every row routed to it.  K runs in stages of 64 (one quantisation
// group, one 128-byte swizzle atom).  Per stage g:
//   producers (8 warps) copy the stage's packed 4-bit weights (16 B per
//     thread) and the bucket's fp16 activation rows (16-byte chunks placed
//     straight into the 128-byte-swizzled K-major layout) with cp.async into
//     a ring of RAW_STAGES slots, PK-1 stages ahead; when their own copies of
//     stage g have landed they dequantise w = S*q + B (half2 arithmetic: q is
//     exact, w is rounded once to fp16) into an A slot, fence the async proxy
//     and arrive on full[g];
//   one thread issues 4 tcgen05.mma (M=128, N, K=16) into a TMEM accumulator
//     and commits them to consumed[g] (frees the raw and A slots);
// after the last stage the 4 epilogue warps read TMEM (tcgen05.ld) and write
//   mode 0 (gate/up): A rows alternate gate/up of one intermediate index, so
//     act = gelu_tanh(gate) * up pairs up neighbouring lanes (fp16 out);
//   mode 1 (down):    y_pairs[pair][o] (fp32).
// Every mbarrier wait is bounded; a wait that runs out sets the device check
// word and the CTA skips its remaining work.
#include "tc_utils.cuh"

namespace moe {

constexpr int TC_BM = 128;
constexpr int TC_BK = 64;
constexpr int TC_PK = 6;                                  // raw ring (copy distance PK-1)
constexpr int TC_PA = 3;                                  // dequantised A ring (divides TC_PK)
constexpr int TC_NMAX = 128;
constexpr int TC_PRODUCER_WARPS = 8;
constexpr int TC_PRODUCERS = TC_PRODUCER_WARPS * 32;
constexpr int TC_THREADS = TC_PRODUCERS + 32;
constexpr int TC_ATOM = 128 * 128;                        // 128 rows x 128 B (64 fp16 of K)
constexpr int TC_RAW_A = TC_BM * TC_BK / 2;               // packed weights of one stage: 4 KB
constexpr int TC_RAW = TC_RAW_A + TC_ATOM;                // + activation tile
constexpr int TC_MAX_GROUPS = 64;                         // K <= 4096
constexpr size_t TC_SMEM = 1024 + TC_PK * TC_RAW + TC_PA * TC_ATOM +
                           static_cast<size_t>(TC_BM) * TC_MAX_GROUPS * 4 + 1024;
static_assert(TC_PK % TC_PA == 0, "A ring must divide the raw ring");
static_assert(TC_RAW % 1024 == 0, "swizzle atoms need 1024-byte alignment");

struct TcArgs {
  int mode;                       // 0 gate/up + GeGLU, 1 down
  const __half* xh;               // mode 0: fp16 [T, H] (the layer input, converted)
  const __half* act_in;           // mode 1: fp16 [T*k, I] (bucket order)
  int T, H, I, E, k;
  const void* const* blob_ptrs;   // routed: device [E] blob pointers (matrices at off[]); null: use mq/ms/mb
  const uint8_t* mq[3];           // one expert given as three q-matrices (gate, up, down), e.g. the shared expert
  const uint16_t* ms[3];
  const uint16_t* mb[3];
  const int32_t* offsets;
  const int32_t* pairs;
  const int32_t* active;
  const int32_t* n_active;
  int max_rows;                   // buckets with at most this many rows are left to the GEMV path
  size_t off[9];
  __half* act_out;                // mode 0
  float* y_out;                   // mode 1: fp32 [T*k, H]
};

// byte offset of (row r, 16-byte chunk c) inside one 128 x 128 B swizzled atom
__device__ __forceinline__ uint32_t sw128(int r, int c) {
  return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ __half2 as_h2(uint32_t v) { return *reinterpret_cast<__half2*>(&v); }
__device__ __forceinline__ uint32_t as_u32(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }

// 8 nibbles of one word -> 8 fp16 weights S*q + B in element order.
__device__ __forceinline__ uint4 dequant_word(uint32_t w, __half2 s2, __half2 b2) {
  const __half2 k1024 = __floats2half2_rn(1024.f, 1024.f);
  const __half2 k16 = __floats2half2_rn(0.0625f, 0.0625f);
  const __half2 k64 = __floats2half2_rn(-64.f, -64.f);
  const uint32_t w8 = w >> 8;
  const __half2 q04 = __hsub2(as_h2((w & 0x000F000Fu) | 0x64006400u), k1024);   // q0, q4
  const __half2 q15 = __hfma2(as_h2((w & 0x00F000F0u) | 0x64006400u), k16, k64);  // q1, q5
  const __half2 q26 = __hsub2(as_h2((w8 & 0x000F000Fu) | 0x64006400u), k1024);  // q2, q6
  const __half2 q37 = __hfma2(as_h2((w8 & 0x00F000F0u) | 0x64006400u), k16, k64); // q3, q7
  const uint32_t a = as_u32(__hfma2(q04, s2, b2)), b = as_u32(__hfma2(q15, s2, b2));
  const uint32_t c = as_u32(__hfma2(q26, s2, b2)), d = as_u32(__hfma2(q37, s2, b2));
  uint4 o;
  o.x = __byte_perm(a, b, 0x5410);   // w0 w1
  o.y = __byte_perm(c, d, 0x5410);   // w2 w3
  o.z = __byte_perm(a, b, 0x7632);   // w4 w5
  o.w = __byte_perm(c, d, 0x7632);   // w6 w7
  return o;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__global__ void k_to_f16(const uint16_t* __restrict__ x, size_t n8, __half* __restrict__ y) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint4 u = reinterpret_cast<const uint4*>(x)[i];
    uint4 o;
    o.x = pack_half2(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u));
    o.y = pack_half2(__uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u));
    o.z = pack_half2(__uint_as_float(u.z << 16), __uint_as_float(u.z & 0xFFFF0000u));
    o.w = pack_half2(__uint_as_float(u.w << 16), __uint_as_float(u.w & 0xFFFF0000u));
    reinterpret_cast<uint4*>(y)[i] = o;
  }
}

// The bucket list of one expert that serves all T rows: offsets {0, T},
// active {0}, n_active 1, pairs 0..T-1 (row t, pair width 1).
__global__ void k_one_bucket(int T, int32_t* offsets, int32_t* pairs, int32_t* active, int32_t* n_active) {
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < T; t += gridDim.x * blockDim.x) pairs[t] = t;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    offsets[0] = 0;
    offsets[1] = T;
    active[0] = 0;
    *n_active = 1;
  }
}

__global__ void __launch_bounds__(TC_THREADS, 1) k_expert_tc(TcArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sRaw = smem;                                       // [PK][TC_RAW]
  unsigned char* sA = sRaw + TC_PK * TC_RAW;                        // [PA][TC_ATOM]
  uint32_t* sSB = reinterpret_cast<uint32_t*>(sA + TC_PA * TC_ATOM);  // [128][groups] (S | B << 16)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sSB + TC_BM * TC_MAX_GROUPS);  // full[PK] consumed[PK] done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * TC_PK + 1);
  int* rowtab = reinterpret_cast<int*>(tmem_slot + 4);              // [TC_NMAX]

  if (static_cast<int>(blockIdx.y) >= *a.n_active) return;
  const int e = a.active[blockIdx.y];
  if (e < 0 || e >= a.E) { if (threadIdx.x == 0) flag_check(CHECK_EXPERT_ID); return; }
  const int pos0 = a.offsets[e];
  const int cnt = a.offsets[e + 1] - pos0;
  if (cnt <= a.max_rows) return;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = a.mode == 0 ? a.H : a.I;
  const int nkb = K / TC_BK;
  const uint8_t* blob = a.blob_ptrs ? static_cast<const uint8_t*>(a.blob_ptrs[e]) : nullptr;
  auto mat_q = [&](int mat) { return blob ? blob + a.off[3 * mat] : a.mq[mat]; };
  auto mat_s = [&](int mat) {
    return blob ? reinterpret_cast<const uint16_t*>(blob + a.off[3 * mat + 1]) : a.ms[mat];
  };
  auto mat_b = [&](int mat) {
    return blob ? reinterpret_cast<const uint16_t*>(blob + a.off[3 * mat + 2]) : a.mb[mat];
  };
  const int m0 = blockIdx.x * (a.mode == 0 ? 64 : 128);

  const uint32_t bar0 = tc::smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto cons_bar = [&](int s) { return bar0 + 8u * (TC_PK + s); };
  const uint32_t done_bar = bar0 + 8u * (2 * TC_PK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < TC_PK; ++s) {
      tc::mbar_init(full_bar(s), TC_PRODUCERS);
      tc::mbar_init(cons_bar(s), 1);
    }
    tc::mbar_init(done_bar, 1);
    tc::fence_mbar_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), TC_NMAX);
    tc::tmem_relinquish();
  }

  // Producer-side constants: thread t owns A row r (half h of the 64-element stage)
  const int t = threadIdx.x;
  const int r = t >> 1, h = t & 1;
  const uint8_t* qrow = nullptr;
  if (warp < TC_PRODUCER_WARPS) {
    int grow, mat;
    if (a.mode == 0) { mat = r & 1; grow = m0 + (r >> 1); }
    else { mat = 2; grow = m0 + r; }
    qrow = mat_q(mat) + static_cast<size_t>(grow) * (K / 2);
  }
  // S/B table of the tile: 128 rows x (K/64) groups, packed as S | B << 16
  for (int i = t; i < TC_BM * nkb; i += TC_THREADS) {
    const int rr = i / nkb, gg = i - rr * nkb;
    int grow, mat;
    if (a.mode == 0) { mat = rr & 1; grow = m0 + (rr >> 1); }
    else { mat = 2; grow = m0 + rr; }
    const uint16_t* sp = mat_s(mat) + static_cast<size_t>(grow) * nkb + gg;
    const uint16_t* bp = mat_b(mat) + static_cast<size_t>(grow) * nkb + gg;
    sSB[rr * TC_MAX_GROUPS + gg] = static_cast<uint32_t>(ldg_u16(sp)) | (static_cast<uint32_t>(ldg_u16(bp)) << 16);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;
  int gbase = 0;                 // global stage counter at the start of this n-tile
  int ntile = 0;

  for (int nt0 = 0; nt0 < cnt; nt0 += TC_NMAX, ++ntile, gbase += nkb) {
    const int N = min(TC_NMAX, cnt - nt0);
    const int Np = (N + 15) & ~15;
    if (t < TC_NMAX) {
      int v = -1;
      if (t < N) {
        const int p = pos0 + nt0 + t;
        if (a.mode == 0) {
          const int pr = a.pairs[p];
          v = pr / a.k;
          if (v < 0 || v >= a.T) { flag_check(CHECK_PAIR_ID); v = -1; }
        } else {
          v = a.pairs[p];
          if (v < 0 || v >= a.T * a.k) { flag_check(CHECK_PAIR_ID); v = -1; }
        }
      }
      rowtab[t] = v;
    }
    __syncthreads();

    if (warp < TC_PRODUCER_WARPS) {
      // ---------------------------------------------------------- producers
      auto issue = [&](int kb) {      // copies of local stage kb into raw slot (gbase+kb) % PK
        const int s = (gbase + kb) % TC_PK;
        const uint32_t raw = tc::smem_u32(sRaw + s * TC_RAW);
        cp_async16(raw + t * 16, qrow + kb * (TC_BK / 2) + 16 * h, 16);
        for (int q = t; q < Np * 8; q += TC_PRODUCERS) {
          const int n = q >> 3, c = q & 7;
          const __half* src;
          uint32_t bytes = 16;
          if (a.mode == 0) {
            const int row = rowtab[n];
            src = a.xh + static_cast<size_t>(row < 0 ? 0 : row) * K + kb * TC_BK + c * 8;
            if (row < 0) bytes = 0;
          } else {
            src = a.act_in + static_cast<size_t>(pos0 + nt0 + n) * K + kb * TC_BK + c * 8;
            if (n >= N) { src = a.act_in; bytes = 0; }
          }
          cp_async16(raw + TC_RAW_A + sw128(n, c), src, bytes);
        }
      };
      for (int p = 0; p < TC_PK - 1; ++p) {
        if (p < nkb) issue(p);
        cp_async_commit();
      }
      for (int kb = 0; kb < nkb && ok; ++kb) {
        const int g = gbase + kb;
        const int s = g % TC_PK;
        cp_async_wait<TC_PK - 2>();                         // own copies of stage kb landed
        if (g >= TC_PA) ok = tc::mbar_wait(cons_bar((g - TC_PA) % TC_PK), ((g - TC_PA) / TC_PK) & 1);
        if (!ok) break;
        const uint4 qq = *reinterpret_cast<const uint4*>(sRaw + s * TC_RAW + t * 16);
        const uint32_t sb = sSB[r * TC_MAX_GROUPS + kb];
        const float sf = bf16_to_f32(static_cast<uint16_t>(sb & 0xFFFF)), bf = bf16_to_f32(static_cast<uint16_t>(sb >> 16));
        const __half2 s2 = __floats2half2_rn(sf, sf), b2 = __floats2half2_rn(bf, bf);
        unsigned char* atom = sA + (g % TC_PA) * TC_ATOM;
        *reinterpret_cast<uint4*>(atom + sw128(r, 4 * h + 0)) = dequant_word(qq.x, s2, b2);
        *reinterpret_cast<uint4*>(atom + sw128(r, 4 * h + 1)) = dequant_word(qq.y, s2, b2);
        *reinterpret_cast<uint4*>(atom + sw128(r, 4 * h + 2)) = dequant_word(qq.z, s2, b2);
        *reinterpret_cast<uint4*>(atom + sw128(r, 4 * h + 3)) = dequant_word(qq.w, s2, b2);
        tc::fence_proxy_async_smem();
        tc::mbar_arrive(full_bar(s));
        if (kb + TC_PK - 1 < nkb) {
          // raw slot of stage g-1 is reused: wait until its MMAs are done
          if (g >= 1) ok = tc::mbar_wait(cons_bar((g - 1) % TC_PK), ((g - 1) / TC_PK) & 1);
          if (!ok) break;
          issue(kb + TC_PK - 1);
        }
        cp_async_commit();
      }
      cp_async_wait<0>();
    } else {
      // ------------------------------------------------------- MMA issuer
      const uint32_t idesc = tc::idesc_f16_f32(TC_BM, Np);
      for (int kb = 0; kb < nkb && ok; ++kb) {
        const int g = gbase + kb;
        const int s = g % TC_PK;
        ok = tc::mbar_wait(full_bar(s), (g / TC_PK) & 1);
        if (!ok) break;
        tc::tc_fence_after();
        if (lane == 0) {
          const uint32_t aBase = tc::smem_u32(sA + (g % TC_PA) * TC_ATOM);
          const uint32_t bBase = tc::smem_u32(sRaw + s * TC_RAW + TC_RAW_A);
#pragma unroll
          for (int kk = 0; kk < TC_BK / 16; ++kk)
            tc::umma_f16(tmem, tc::sdesc_k_sw128(aBase + kk * 32), tc::sdesc_k_sw128(bBase + kk * 32), idesc,
                         (kb > 0 || kk > 0) ? 1u : 0u);
          tc::umma_commit(cons_bar(s));
          if (kb == nkb - 1) tc::umma_commit(done_bar);
        }
        __syncwarp();
      }
    }

    // ------------------------------------------------------------ epilogue
    if (warp < 4) ok = __all_sync(0xffffffffu, ok);        // .aligned tcgen05.ld below: warp-uniform
    if (warp < 4 && ok) {
      ok = __all_sync(0xffffffffu, tc::mbar_wait(done_bar, ntile & 1));
      if (ok) {
        tc::tc_fence_after();
        const int row = 32 * warp + lane;
        for (int nc = 0; nc < Np; nc += 16) {
          float v[16];
          tc::tmem_ld16(tmem + (static_cast<uint32_t>(32 * warp) << 16) + nc, v);
          if (a.mode == 0) {
            const int i = m0 + (row >> 1);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float u = __shfl_xor_sync(0xffffffffu, v[j], 1);
              const int n = nc + j;
              if ((lane & 1) == 0 && n < N)
                a.act_out[static_cast<size_t>(pos0 + nt0 + n) * a.I + i] = __float2half_rn(gelu_tanh(v[j]) * u);
            }
          } else {
            const int o = m0 + row;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int n = nc + j;
              if (n < N) {
                const int dst = rowtab[n];
                if (dst >= 0) a.y_out[static_cast<size_t>(dst) * a.H + o] = v[j];
              }
            }
          }
        }
      }
    }
    tc::tc_fence_before();
    __syncthreads();        // TMEM read out (and rowtab used) before the next n-tile
    tc::tc_fence_after();
  }
  if (warp == 0) tc::tmem_dealloc(tmem, TC_NMAX);
}

}  // namespace moe
