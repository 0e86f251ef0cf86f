// Kernel declarations and launch-argument structs shared by the C-ABI layer.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int ROUTER_TB = 16;    // rows per router cluster (two mma n-tiles)
constexpr int ROUTER_THREADS = 512;   // 16 warps: m-tiles of 16 experts x slices of the groups
constexpr int ROUTER_XB = 6;     // x chunks a router thread loads before staging them
constexpr int ROUTER_GB = 3;     // groups of codes and scales a router lane loads before using them
constexpr int BUCKET_THREADS = 512;   // one block; each warp buckets a contiguous run of pairs
constexpr int BUCKET_B = 8;      // chunks of 32 pair indices a bucket warp loads at once
constexpr int GEMV_RG = 4;       // bucket rows staged at once by the GEMV kernels
constexpr int GEMV_ROWS = 32;    // output rows per GEMV block

struct GateUpArgs {
  const uint16_t* x;             // bf16 [T, H]
  int T, H, I, E, k;
  // routed mode (blob_ptrs != nullptr)
  const void* const* blob_ptrs;
  const int32_t* offsets;
  const int32_t* pairs;
  const int32_t* active;
  const int32_t* n_active;
  int max_rows;                  // buckets larger than this are skipped here
  size_t off[9];                 // byte offsets inside a blob
  // shared mode (blob_ptrs == nullptr; pairs == nullptr)
  const uint32_t* gq; const uint16_t* gs; const uint16_t* gb;
  const uint32_t* uq; const uint16_t* us; const uint16_t* ub;
  __half* act;                   // fp16 [rows, I]
};

struct DownArgs {
  const __half* act;             // fp16 [rows, I]
  int T, H, I, E, k;
  const void* const* blob_ptrs;
  const int32_t* offsets;
  const int32_t* pairs;
  const int32_t* active;
  const int32_t* n_active;
  int max_rows;
  size_t off[9];
  const uint32_t* dq; const uint16_t* ds; const uint16_t* db;
  float* y;                      // fp32 [dest rows, H]
};

__global__ void k_rmsnorm(const float* h, int H, float eps, uint16_t* x);
__global__ void k_router_topk(const uint16_t* x, int T, int H, const uint32_t* rq, const uint16_t* rs,
                              const uint16_t* rb, const float* bias, int bias_per_row, int E, int k,
                              int32_t* idx, float* gates, float* logits_out);
__global__ void k_bucket(const int32_t* idx, int n, int E, int32_t* offsets, int32_t* pairs,
                         int32_t* active, int32_t* n_active);
__global__ void k_gateup_gemv(GateUpArgs a);
__global__ void k_down_gemv(DownArgs a);
__global__ void k_combine(const float* yp, const float* gates, const float* ysh, int H, int k,
                          uint16_t* y, const float* resid_in, float* resid_out);
__global__ void k_combine4(const float* yp, const float* gates, const float* ysh, int H, int k,
                           uint16_t* y, const float* resid_in, float* resid_out);

// Shared memory of the router kernel: logits [TB][E] | staged x, per row the
// byte-paired words [4][H/16] (rows 32 bytes apart modulo 128, so the eight
// rows an mma reads fall in distinct banks) | group sums [TB][H/64] |
// partial logits [ROUTER_THREADS / 32 warps][TB][16].
struct RouterSmem {
  size_t lg, xs, row_bytes, xg, part, total;
};
__host__ __device__ inline RouterSmem router_smem_layout(int H, int E) {
  RouterSmem L;
  const size_t nch = static_cast<size_t>(H) / 16;
  L.lg = 0;
  L.xs = (static_cast<size_t>(ROUTER_TB) * E * sizeof(float) + 127) & ~size_t(127);
  L.row_bytes = nch * 4 * 8 + 32;
  L.xg = L.xs + ROUTER_TB * L.row_bytes;
  L.part = (L.xg + static_cast<size_t>(ROUTER_TB) * (H / 64) * sizeof(float) + 15) & ~size_t(15);
  L.total = L.part + static_cast<size_t>(ROUTER_THREADS / 32) * ROUTER_TB * 16 * sizeof(float);
  return L;
}
inline size_t router_smem_bytes(int H, int E) { return router_smem_layout(H, E).total; }

}  // namespace moe
