// Decode-side building blocks: staging an activation row into the
// nibble-paired shared-memory layout, and the warp dot of one 4-bit weight
// row against several staged rows.
#pragma once
#include "common.cuh"

namespace moe {

// Shared-memory image of one activation row of length K (K % 32 == 0):
//   P   uint4 [4][nch]   P[m*nch + c] = the four half2 of word 4c+m (see
//                        pair_word4); word-major so that lane c of a warp
//                        reads 16 consecutive bytes (no bank conflicts)
//   st  float2 [nch]     (1024 * sum of stored halves, plain sum) per chunk c
// with nch = K / 32 chunks of 32 elements.
struct StagedRow {
  uint4* P;
  float2* st;
};

__host__ __device__ inline size_t staged_row_bytes(int K) {
  return static_cast<size_t>(K) / 2 * 4 + static_cast<size_t>(K) / 32 * sizeof(float2);
}

__device__ inline StagedRow staged_row_at(void* base, int K, int r) {
  char* p = static_cast<char*>(base) + static_cast<size_t>(r) * staged_row_bytes(K);
  StagedRow s;
  s.P = reinterpret_cast<uint4*>(p);
  s.st = reinterpret_cast<float2*>(p + static_cast<size_t>(K) / 2 * 4);
  return s;
}

// Load 8 consecutive activation values as fp32 from bf16 / fp16 / fp32 sources.
template <typename T> __device__ inline void load8(const T* src, float v[8]);
template <> __device__ inline void load8<uint16_t>(const uint16_t* src, float v[8]) {  // bf16
  uint4 u = *reinterpret_cast<const uint4*>(src);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
template <> __device__ inline void load8<__half>(const __half* src, float v[8]) {
  uint4 u = *reinterpret_cast<const uint4*>(src);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = unpack_half2(w[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
template <> __device__ inline void load8<float>(const float* src, float v[8]) {
  float4 a = *reinterpret_cast<const float4*>(src);
  float4 b = *reinterpret_cast<const float4*>(src + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// Stage `nrows` rows (row r read from src_row(r)) of length K into smem.
// All threads of the block take part; ends with __syncthreads().
// `scratch` holds nrows * (K/8) float2 of per-word partial sums.
template <typename T, typename RowFn>
__device__ void stage_rows4(void* smem, float2* scratch, int K, int nrows, RowFn src_row) {
  const int nw = K / 8, nch = K / 32;
  for (int i = threadIdx.x; i < nrows * nw; i += blockDim.x) {
    const int r = i / nw, w = i - r * nw;
    const T* src = src_row(r);
    float v[8];
    if (src != nullptr) {
      load8<T>(src + 8 * w, v);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = 0.f;
    }
    uint32_t p[4];
    pair_word4(v, p);
    StagedRow s = staged_row_at(smem, K, r);
    const int c = w >> 2, m = w & 3;
    s.P[m * nch + c] = make_uint4(p[0], p[1], p[2], p[3]);
    float off = 0.f, sum = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float2 f = unpack_half2(p[j]);
      off += f.x + f.y;
    }
    // plain sum uses the values as the dot sees them (fp16-rounded)
    float2 f0 = unpack_half2(p[0]), f1 = unpack_half2(p[1]);
    float2 f2 = unpack_half2(p[2]), f3 = unpack_half2(p[3]);
    sum = (f0.x + f0.y + f2.x + f2.y) + 16.f * (f1.x + f1.y + f3.x + f3.y);
    scratch[i] = make_float2(1024.f * off, sum);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < nrows * nch; i += blockDim.x) {
    const int r = i / nch, c = i - r * nch;
    const float2* sp = scratch + static_cast<size_t>(r) * nw + 4 * c;
    float2 a = sp[0], b = sp[1], cc = sp[2], d = sp[3];
    StagedRow s = staged_row_at(smem, K, r);
    s.st[c] = make_float2(((a.x + b.x) + cc.x) + d.x, ((a.y + b.y) + cc.y) + d.y);
  }
  __syncthreads();
}

// Warp dot products of one 4-bit weight row (K inputs, nch = K/32 chunks)
// with RG staged rows.  q: row start (bytes), s/b: the row's bf16 scale/bias.
// Result: out[r] = sum_c w[c] * v_r[c], full warp sum in every lane.
template <int RG>
__device__ __forceinline__ void row_dot4(const uint8_t* q, const uint16_t* s, const uint16_t* b,
                                         int nch, void* smem, int K, int nrows, float (&out)[RG]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int r = 0; r < RG; ++r) out[r] = 0.f;
  for (int c = lane; c < nch; c += 32) {
    const uint4 qq = ldg_nc_v4(q + static_cast<size_t>(c) * 16);
    const float sc = bf16_to_f32(ldg_u16(s + (c >> 1)));
    const float bi = bf16_to_f32(ldg_u16(b + (c >> 1)));
#pragma unroll
    for (int r = 0; r < RG; ++r) {
      if (r < nrows) {
        StagedRow sr = staged_row_at(smem, K, r);
        uint32_t p[16];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          uint4 u = sr.P[m * nch + c];
          p[4 * m + 0] = u.x; p[4 * m + 1] = u.y; p[4 * m + 2] = u.z; p[4 * m + 3] = u.w;
        }
        // word m's pairs are p[4m..4m+3]
        float a0 = 0.f, a1 = 0.f;
        dot_word4(qq.x, p + 0, a0, a1);
        dot_word4(qq.y, p + 4, a0, a1);
        dot_word4(qq.z, p + 8, a0, a1);
        dot_word4(qq.w, p + 12, a0, a1);
        const float2 st = sr.st[c];
        out[r] += sc * ((a0 + a1) - st.x) + bi * st.y;
      }
    }
  }
#pragma unroll
  for (int r = 0; r < RG; ++r) out[r] = warp_sum(out[r]);
}

}  // namespace moe
