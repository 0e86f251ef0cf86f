// Kernel declarations and launch-argument structs shared by the C-ABI layer.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int ROUTER_TB = 8;     // rows per router cluster
constexpr int ROUTER_THREADS = 512;   // threads per router CTA (one warp per expert of the CTA's E/8)
constexpr int ROUTER_XB = 4;     // x chunks a router thread loads before staging them
constexpr int ROUTER_CB = 8;     // router chunks a lane loads before using them
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
                          uint16_t* y, float* resid);
__global__ void k_combine4(const float* yp, const float* gates, const float* ysh, int H, int k,
                           uint16_t* y, float* resid);

inline size_t router_smem_bytes(int H, int E) {
  const int nch = H / 16;
  return ROUTER_TB * E * sizeof(float) +
         ROUTER_TB * (static_cast<size_t>(nch) * 4 * 8 + nch * 8);
}

}  // namespace moe
