// Expert parallelism over G ranks (one process per GPU): rank d owns the
// routed experts [d E/G, (d+1) E/G); every rank keeps its own tokens, its
// router, its shared expert and its combine.  Per layer two exchanges move
// rows between ranks, each a kernel that stores straight into the peers'
// buffers (NVLink peer mappings, or this GPU's own memory for the rank
// itself), with no host round trip:
//   dispatch  the layer input row of every (token, slot) pair goes to the
//             owner of the pair's expert, at a row computed on the device
//             from every rank's bucket offsets;
//   return    the owner sends each expert output row back into the source
//             rank's y_pairs at the pair's own index, where the ordinary
//             combine reads it.
// Receiver layout (rank d): the rows of its experts in expert order; inside
// an expert, by source rank; inside a source, in that source's bucket order.
// With cnt(s, e) = off_s[e+1] - off_s[e], slot i of source s's bucket e
// (owner d = e / El) lands on row
//   base(e) + before(s, e) + (i - off_s[e]),
//   base(e)      = sum over e' in [d El, e) of sum over s' of cnt(s', e'),
//   before(s, e) = sum over s' < s of cnt(s', e),
// and the receiver's own bucket offsets are base(d El + j), j = 0 .. El.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int EP_MAX_G = 8;          // ranks
constexpr int EP_THREADS = 256;      // dispatch / return / plan

struct EpPeers {                     // by value: one device pointer per rank
  void* p[EP_MAX_G];
};

// Exclusive prefix sum of v[0..n) in place (n <= 1024, blockDim.x = EP_THREADS);
// returns the total.  sc: EP_THREADS / 32 + 1 ints of scratch.
__device__ int ep_block_exscan(int* v, int n, int* sc) {
  constexpr int PER = (1024 + EP_THREADS - 1) / EP_THREADS;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int b = threadIdx.x * PER;
  int loc[PER], s = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    loc[j] = b + j < n ? v[b + j] : 0;
    s += loc[j];
  }
  int incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) sc[warp] = incl;
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int w = 0; w < EP_THREADS / 32; ++w) {
      const int t = sc[w];
      sc[w] = run;
      run += t;
    }
    sc[EP_THREADS / 32] = run;
  }
  __syncthreads();
  int run = sc[warp] + incl - s;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    if (b + j < n) v[b + j] = run;
    run += loc[j];
  }
  const int total = sc[EP_THREADS / 32];
  __syncthreads();
  return total;
}

// tot[e] = sum over ranks of cnt(r, e) for e in [e0, e0 + n), and, when
// before is non-NULL, before[e - e0] = sum over r < s of cnt(r, e) - off_s[e].
__device__ void ep_counts(const int32_t* all_off, int G, int E, int s, int e0, int n, int* tot, int* before) {
  for (int j = threadIdx.x; j < n; j += blockDim.x) {
    const int e = e0 + j;
    int t = 0, b = 0;
    for (int r = 0; r < G; ++r) {
      const int c = all_off[r * (E + 1) + e + 1] - all_off[r * (E + 1) + e];
      t += c;
      if (r < s) b += c;
    }
    tot[j] = t;
    if (before) before[j] = b - all_off[s * (E + 1) + e];
  }
  __syncthreads();
}

// Source rank s: every bucketed slot's layer input row (bf16 [H]) and its
// (source, pair index) go to the owner of its expert.  One warp per slot.
__global__ void __launch_bounds__(EP_THREADS) k_ep_dispatch(const uint16_t* __restrict__ x, int H, int k,
                                                            const int32_t* __restrict__ idx,
                                                            const int32_t* __restrict__ pairs,
                                                            const int32_t* __restrict__ all_off, int G, int E, int s,
                                                            EpPeers recv_x, EpPeers recv_meta, int cap_rows) {
  extern __shared__ int ep_sm[];
  int* tot = ep_sm;              // [E] -> base (segmented scan, each owner's range from 0)
  int* pos0 = ep_sm + E;         // [E] before(s, e) - off_s[e]
  int* sc = ep_sm + 2 * E;
  const int El = E / G;
  ep_counts(all_off, G, E, s, 0, E, tot, pos0);
  // base(e): the scan over all experts minus its value at the owner's first expert
  int* scan = tot;
  ep_block_exscan(scan, E, sc);
  for (int e = threadIdx.x; e < E; e += blockDim.x) pos0[e] += scan[e] - scan[(e / El) * El];
  __syncthreads();
  const int n = all_off[s * (E + 1) + E];
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  const int nv = H / 8;                      // 16-byte vectors per row
  for (int i = blockIdx.x * wpb + (threadIdx.x >> 5); i < n; i += gridDim.x * wpb) {
    const int p = pairs[i];
    const int e = idx[p];
    if (e < 0 || e >= E) {
      if (lane == 0) flag_check(CHECK_EXPERT_ID);
      continue;
    }
    const int d = e / El;
    const int row = pos0[e] + i;
    if (row < 0 || row >= cap_rows) {
      if (lane == 0) flag_check(CHECK_EP_ROW);
      continue;
    }
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(p / k) * H);
    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(recv_x.p[d]) + static_cast<size_t>(row) * H);
    for (int v = lane; v < nv; v += 32) dst[v] = __ldg(src + v);
    if (lane == 0) static_cast<int2*>(recv_meta.p[d])[row] = make_int2(s, p);
  }
  __threadfence_system();
}

// Receiver rank d: its bucket offsets [El + 1] over the rows it received,
// the identity pair list of those rows, and the non-empty experts ascending
// with their count -- the inputs of the grouped expert GEMM with k = 1.
__global__ void __launch_bounds__(EP_THREADS) k_ep_recv_plan(const int32_t* __restrict__ all_off, int G, int E,
                                                             int d, int cap_rows, int32_t* __restrict__ offsets,
                                                             int32_t* __restrict__ pairs, int32_t* __restrict__ active,
                                                             int32_t* __restrict__ n_active) {
  extern __shared__ int ep_sm[];
  const int El = E / G;
  int* tot = ep_sm;              // [El + 1]
  int* flg = ep_sm + El + 1;     // [El + 1]
  int* sc = ep_sm + 2 * (El + 1);
  ep_counts(all_off, G, E, d, d * El, El, tot, nullptr);
  for (int j = threadIdx.x; j < El; j += blockDim.x) flg[j] = tot[j] > 0;
  __syncthreads();
  const int R = ep_block_exscan(tot, El, sc);
  const int na = ep_block_exscan(flg, El, sc);
  // offsets clamped to the capacity (rows past it were not stored; the
  // check word reports it)
  for (int j = threadIdx.x; j < El; j += blockDim.x) {
    offsets[j] = tot[j] < cap_rows ? tot[j] : cap_rows;
    const int nxt = j + 1 < El ? flg[j + 1] : na;
    if (nxt > flg[j]) active[flg[j]] = j;
  }
  if (threadIdx.x == 0) {
    offsets[El] = R < cap_rows ? R : cap_rows;
    n_active[0] = na;
    if (R > cap_rows) flag_check(CHECK_EP_ROW);
  }
  const int rows = R < cap_rows ? R : cap_rows;
  for (int r = threadIdx.x; r < rows; r += blockDim.x) pairs[r] = r;
}

// Receiver rank d: expert output row r (fp32 [H]) goes back to its source
// rank's y_pairs at the pair's index.  One warp per row.
__global__ void __launch_bounds__(EP_THREADS) k_ep_return(const float* __restrict__ y_rows, int H,
                                                          const int2* __restrict__ recv_meta,
                                                          const int32_t* __restrict__ offsets, int El, int G,
                                                          int n_pair_slots, int cap_rows, EpPeers y_pairs) {
  int R = offsets[El];
  if (R > cap_rows) R = cap_rows;
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  const int nv = H / 4;
  for (int r = blockIdx.x * wpb + (threadIdx.x >> 5); r < R; r += gridDim.x * wpb) {
    const int2 m = recv_meta[r];
    if (m.x < 0 || m.x >= G || m.y < 0 || m.y >= n_pair_slots) {
      if (lane == 0) flag_check(CHECK_PAIR_ID);
      continue;
    }
    const uint4* src = reinterpret_cast<const uint4*>(y_rows + static_cast<size_t>(r) * H);
    uint4* dst = reinterpret_cast<uint4*>(static_cast<float*>(y_pairs.p[m.x]) + static_cast<size_t>(m.y) * H);
    for (int v = lane; v < nv; v += 32) dst[v] = __ldg(src + v);
  }
  __threadfence_system();
}

}  // namespace moe

using namespace moe;

static int ep_check(int T, int H, int k, int E, int G, int rank, const char* who) {
  int st = check_dims(T, H, 64, E, k);
  if (st) return st;
  if (G < 1 || G > EP_MAX_G) return fail(MOE_ERR_INVALID_ARG, "%s: G must be in [1, %d] (got %d)", who, EP_MAX_G, G);
  if (E % G || (E / G) % 8)
    return fail(MOE_ERR_INVALID_ARG, "%s: E/G must be a whole multiple of 8 (E=%d, G=%d)", who, E, G);
  if (rank < 0 || rank >= G) return fail(MOE_ERR_INVALID_ARG, "%s: rank %d outside [0, %d)", who, rank, G);
  return MOE_OK;
}

static int ep_peers(void* const* in, int G, EpPeers* out, const char* who) {
  if (!in) return fail(MOE_ERR_INVALID_ARG, "%s: NULL peer table", who);
  for (int r = 0; r < EP_MAX_G; ++r) out->p[r] = nullptr;
  for (int r = 0; r < G; ++r) {
    if (!in[r] || !aligned16(in[r])) return fail(MOE_ERR_INVALID_ARG, "%s: peer buffer %d NULL or misaligned", who, r);
    out->p[r] = in[r];
  }
  return MOE_OK;
}

extern "C" {

int moe_ep_dispatch(const uint16_t* x, int T, int H, int k, int E, int G, int rank, const int32_t* idx,
                    const int32_t* pairs, const int32_t* all_offsets, void* const* recv_x, void* const* recv_meta,
                    int cap_rows, void* stream) {
  int st = ep_check(T, H, k, E, G, rank, "moe_ep_dispatch");
  if (st) return st;
  if (cap_rows < 0) return fail(MOE_ERR_INVALID_ARG, "moe_ep_dispatch: cap_rows < 0");
  if (!x || !idx || !pairs || !all_offsets) return fail(MOE_ERR_INVALID_ARG, "moe_ep_dispatch: NULL pointer");
  if (!aligned16(x)) return fail(MOE_ERR_INVALID_ARG, "moe_ep_dispatch: misaligned x");
  EpPeers px, pm;
  if ((st = ep_peers(recv_x, G, &px, "moe_ep_dispatch"))) return st;
  if ((st = ep_peers(recv_meta, G, &pm, "moe_ep_dispatch"))) return st;
  if (T == 0) return MOE_OK;
  const int slots = T * k, wpb = EP_THREADS / 32;
  int grid = (slots + wpb - 1) / wpb;
  if (grid > 4 * 148) grid = 4 * 148;
  const size_t smem = (2 * static_cast<size_t>(E) + EP_THREADS / 32 + 1) * sizeof(int);
  k_ep_dispatch<<<grid, EP_THREADS, smem, static_cast<cudaStream_t>(stream)>>>(x, H, k, idx, pairs, all_offsets, G, E,
                                                                                rank, px, pm, cap_rows);
  return launch_check("k_ep_dispatch");
}

int moe_ep_recv_plan(const int32_t* all_offsets, int G, int E, int rank, int cap_rows, int32_t* offsets,
                     int32_t* pairs, int32_t* active, int32_t* n_active, void* stream) {
  int st = ep_check(0, 64, 1, E, G, rank, "moe_ep_recv_plan");
  if (st) return st;
  if (cap_rows < 0) return fail(MOE_ERR_INVALID_ARG, "moe_ep_recv_plan: cap_rows < 0");
  if (!all_offsets || !offsets || !pairs || !active || !n_active)
    return fail(MOE_ERR_INVALID_ARG, "moe_ep_recv_plan: NULL pointer");
  const int El = E / G;
  const size_t smem = (2 * static_cast<size_t>(El + 1) + EP_THREADS / 32 + 1) * sizeof(int);
  k_ep_recv_plan<<<1, EP_THREADS, smem, static_cast<cudaStream_t>(stream)>>>(all_offsets, G, E, rank, cap_rows,
                                                                             offsets, pairs, active, n_active);
  return launch_check("k_ep_recv_plan");
}

int moe_ep_return(const float* y_rows, int H, int E, int G, int rank, const void* recv_meta, const int32_t* offsets,
                  int n_pair_slots, int cap_rows, void* const* y_pairs, void* stream) {
  int st = ep_check(0, H, 1, E, G, rank, "moe_ep_return");
  if (st) return st;
  if (cap_rows < 0 || n_pair_slots < 0) return fail(MOE_ERR_INVALID_ARG, "moe_ep_return: negative size");
  if (!y_rows || !recv_meta || !offsets) return fail(MOE_ERR_INVALID_ARG, "moe_ep_return: NULL pointer");
  if (!aligned16(y_rows) || (reinterpret_cast<uintptr_t>(recv_meta) & 7))
    return fail(MOE_ERR_INVALID_ARG, "moe_ep_return: misaligned pointer");
  EpPeers py;
  if ((st = ep_peers(y_pairs, G, &py, "moe_ep_return"))) return st;
  if (cap_rows == 0) return MOE_OK;
  const int wpb = EP_THREADS / 32;
  int grid = (cap_rows + wpb - 1) / wpb;
  if (grid > 4 * 148) grid = 4 * 148;
  k_ep_return<<<grid, EP_THREADS, 0, static_cast<cudaStream_t>(stream)>>>(
      y_rows, H, static_cast<const int2*>(recv_meta), offsets, E / G, G, n_pair_slots, cap_rows, py);
  return launch_check("k_ep_return");
}

int moe_device_alloc(size_t bytes, void** ptr) {
  if (!ptr) return fail(MOE_ERR_INVALID_ARG, "moe_device_alloc: NULL out pointer");
  *ptr = nullptr;
  if (bytes == 0) return fail(MOE_ERR_INVALID_ARG, "moe_device_alloc: zero bytes");
  return cuda_check(cudaMalloc(ptr, bytes), "moe_device_alloc");
}

int moe_device_free(void* ptr) { return ptr ? cuda_check(cudaFree(ptr), "moe_device_free") : MOE_OK; }

int moe_ipc_handle_bytes(void) { return static_cast<int>(sizeof(cudaIpcMemHandle_t)); }

int moe_ipc_get_handle(const void* ptr, void* handle_out) {
  if (!ptr || !handle_out) return fail(MOE_ERR_INVALID_ARG, "moe_ipc_get_handle: NULL pointer");
  cudaIpcMemHandle_t h;
  int st = cuda_check(cudaIpcGetMemHandle(&h, const_cast<void*>(ptr)), "moe_ipc_get_handle");
  if (st) return st;
  memcpy(handle_out, &h, sizeof(h));
  return MOE_OK;
}

int moe_ipc_open(const void* handle, void** ptr) {
  if (!handle || !ptr) return fail(MOE_ERR_INVALID_ARG, "moe_ipc_open: NULL pointer");
  *ptr = nullptr;
  cudaIpcMemHandle_t h;
  memcpy(&h, handle, sizeof(h));
  return cuda_check(cudaIpcOpenMemHandle(ptr, h, cudaIpcMemLazyEnablePeerAccess), "moe_ipc_open");
}

int moe_ipc_close(void* ptr) {
  if (!ptr) return fail(MOE_ERR_INVALID_ARG, "moe_ipc_close: NULL pointer");
  return cuda_check(cudaIpcCloseMemHandle(ptr), "moe_ipc_close");
}

}  // extern "C"
