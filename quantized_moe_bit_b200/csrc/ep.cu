// Expert parallelism over G ranks (one process per GPU): rank d owns the
// routed experts [d E/G, (d+1) E/G); every rank keeps its own tokens, its
// router, its shared expert and its combine.  Per layer two exchanges move
// rows between ranks, each a kernel that stores straight into the peers'
// buffers (NVLink peer mappings, or this GPU's own memory for the rank
// itself), with no host round trip.  The stores are complete when the kernel
// is (the end of a grid flushes its writes system-wide, as for mapped host
// memory), so a stream-ordered barrier across ranks after the kernel is what
// orders them before any peer reads them; no fence inside the kernel:
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
// A thread's loads of all ranks are issued together (one memory latency).
__device__ void ep_counts(const int32_t* __restrict__ all_off, int G, int E, int s, int e0, int n, int* tot,
                          int* before) {
  for (int j = threadIdx.x; j < n; j += blockDim.x) {
    const int e = e0 + j;
    int lo[EP_MAX_G], hi[EP_MAX_G];
#pragma unroll
    for (int r = 0; r < EP_MAX_G; ++r) {
      lo[r] = r < G ? __ldg(all_off + r * (E + 1) + e) : 0;
      hi[r] = r < G ? __ldg(all_off + r * (E + 1) + e + 1) : 0;
    }
    int t = 0, b = 0;
#pragma unroll
    for (int r = 0; r < EP_MAX_G; ++r) {
      t += hi[r] - lo[r];
      if (r < s) b += hi[r] - lo[r];
    }
    tot[j] = t;
    if (before) before[j] = b - __ldg(all_off + s * (E + 1) + e);
  }
  __syncthreads();
}

constexpr int EP_NV = 12;   // 16-byte vectors per lane in one warp copy step (a 6 KB bf16 row)

// One warp's copy step of vectors [b, b + 32 EP_NV) of a row: all loads of the
// step are issued before its stores.
__device__ __forceinline__ void ep_load(uint4 (&u)[EP_NV], const uint4* __restrict__ src, int n16, int b, int lane) {
#pragma unroll
  for (int j = 0; j < EP_NV; ++j) {
    const int v = b + lane + 32 * j;
    if (v < n16) u[j] = __ldg(src + v);
  }
}
__device__ __forceinline__ void ep_store(uint4* dst, const uint4 (&u)[EP_NV], int n16, int b, int lane) {
#pragma unroll
  for (int j = 0; j < EP_NV; ++j) {
    const int v = b + lane + 32 * j;
    if (v < n16) dst[v] = u[j];
  }
}

// Receiver plan of rank d, by one CTA: its bucket offsets [El + 1] over the
// rows it receives (clamped to the capacity), the identity pair list of
// those rows and the non-empty local experts ascending with their count --
// the inputs of the grouped expert GEMM with k = 1.  sm: 2 (El + 1) +
// EP_THREADS / 32 + 1 ints.
__device__ void ep_recv_plan_block(const int32_t* __restrict__ all_off, int G, int E, int d, int cap_rows,
                                   int32_t* __restrict__ offsets, int32_t* __restrict__ pairs,
                                   int32_t* __restrict__ active, int32_t* __restrict__ n_active, int* sm) {
  const int El = E / G;
  int* tot = sm;
  int* flg = sm + El + 1;
  int* sc = sm + 2 * (El + 1);
  ep_counts(all_off, G, E, d, d * El, El, tot, nullptr);
  for (int j = threadIdx.x; j < El; j += blockDim.x) flg[j] = tot[j] > 0;
  __syncthreads();
  const int R = ep_block_exscan(tot, El, sc);
  const int na = ep_block_exscan(flg, El, sc);
  for (int j = threadIdx.x; j < El; j += blockDim.x) {
    offsets[j] = tot[j] < cap_rows ? tot[j] : cap_rows;
    const int nxt = j + 1 < El ? flg[j + 1] : na;
    if (nxt > flg[j]) active[flg[j]] = j;
  }
  if (threadIdx.x == 0) {
    offsets[El] = R < cap_rows ? R : cap_rows;
    n_active[0] = na;
    if (R > cap_rows) flag_check(CHECK_EP_ROW);   // rows past the capacity were not stored
  }
  const int rows = R < cap_rows ? R : cap_rows;
  for (int r = threadIdx.x; r < rows; r += blockDim.x) pairs[r] = r;
}

// Source rank s: every bucketed slot's layer input row (bf16 [H]) and its
// (source, pair index) go to the owner of its expert, one warp per slot.  A
// warp's first row is loaded before the CTA builds its row table (the load
// does not depend on it).  The grid's last block writes rank s's own
// receiver plan meanwhile.
// sm: 2 (E + 1) + EP_THREADS / 32 + 1 ints.
__global__ void __launch_bounds__(EP_THREADS) k_ep_dispatch(const uint16_t* __restrict__ x, int H, int k,
                                                            const int32_t* __restrict__ idx,
                                                            const int32_t* __restrict__ pairs,
                                                            const int32_t* __restrict__ all_off, int G, int E, int s,
                                                            EpPeers recv_x, EpPeers recv_meta, int cap_rows,
                                                            int n_slots, int32_t* plan_offsets, int32_t* plan_pairs,
                                                            int32_t* plan_active, int32_t* plan_n_active) {
  extern __shared__ int ep_sm[];
  int* tot = ep_sm;              // [E] -> the scan of the totals
  int* pos0 = ep_sm + E + 1;     // [E] row of slot i of bucket e = pos0[e] + i
  int* sc = ep_sm + 2 * (E + 1);
  const int El = E / G;
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  const int nv = H / 8;          // 16-byte vectors per row
  int n = all_off[s * (E + 1) + E];
  if (n < 0 || n > n_slots) {
    if (blockIdx.x == 0 && threadIdx.x == 0) flag_check(CHECK_PAIR_ID);
    n = n < 0 ? 0 : n_slots;
  }
  if (blockIdx.x == gridDim.x - 1) {   // the plan block copies nothing
    ep_recv_plan_block(all_off, G, E, s, cap_rows, plan_offsets, plan_pairs, plan_active, plan_n_active, ep_sm);
    return;
  }
  const int ncopy = gridDim.x - 1;    // copying blocks
  int i = blockIdx.x * wpb + (threadIdx.x >> 5);
  uint4 u[EP_NV];
  int p0 = -1;
  if (i < n) {
    p0 = pairs[i];
    if (p0 >= 0 && p0 < n_slots) ep_load(u, reinterpret_cast<const uint4*>(x + static_cast<size_t>(p0 / k) * H), nv, 0, lane);
  }
  ep_counts(all_off, G, E, s, 0, E, tot, pos0);
  ep_block_exscan(tot, E, sc);   // base(e) = tot[e] - tot[first expert of e's owner]
  for (int e = threadIdx.x; e < E; e += blockDim.x) pos0[e] += tot[e] - tot[(e / El) * El];
  __syncthreads();
  for (bool first = true; i < n; i += ncopy * wpb, first = false) {
    const int p = first ? p0 : pairs[i];
    if (p < 0 || p >= n_slots) {
      if (lane == 0) flag_check(CHECK_PAIR_ID);
      continue;
    }
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
    int b = 0;
    if (first) {
      ep_store(dst, u, nv, 0, lane);
      b = 32 * EP_NV;
    }
    for (; b < nv; b += 32 * EP_NV) {
      ep_load(u, src, nv, b, lane);
      ep_store(dst, u, nv, b, lane);
    }
    if (lane == 0) static_cast<int2*>(recv_meta.p[d])[row] = make_int2(s, p);
  }
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
    uint4 u[EP_NV];
    for (int b = 0; b < nv; b += 32 * EP_NV) {
      ep_load(u, src, nv, b, lane);
      ep_store(dst, u, nv, b, lane);
    }
  }
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
                    int cap_rows, int32_t* plan_offsets, int32_t* plan_pairs, int32_t* plan_active,
                    int32_t* plan_n_active, void* stream) {
  int st = ep_check(T, H, k, E, G, rank, "moe_ep_dispatch");
  if (st) return st;
  if (cap_rows < 0) return fail(MOE_ERR_INVALID_ARG, "moe_ep_dispatch: cap_rows < 0");
  if (!x || !idx || !pairs || !all_offsets) return fail(MOE_ERR_INVALID_ARG, "moe_ep_dispatch: NULL pointer");
  if (!plan_offsets || !plan_pairs || !plan_active || !plan_n_active)
    return fail(MOE_ERR_INVALID_ARG, "moe_ep_dispatch: NULL plan output");
  if (!aligned16(x)) return fail(MOE_ERR_INVALID_ARG, "moe_ep_dispatch: misaligned x");
  EpPeers px, pm;
  if ((st = ep_peers(recv_x, G, &px, "moe_ep_dispatch"))) return st;
  if ((st = ep_peers(recv_meta, G, &pm, "moe_ep_dispatch"))) return st;
  // T = 0 still launches: the rank's receiver plan covers the rows other
  // ranks send it
  const int slots = T * k, wpb = EP_THREADS / 32;
  int grid = (slots + wpb - 1) / wpb;
  if (grid > 4 * 148) grid = 4 * 148;
  grid += 1;                            // the plan block
  const size_t smem = (2 * static_cast<size_t>(E + 1) + EP_THREADS / 32 + 1) * sizeof(int);
  k_ep_dispatch<<<grid, EP_THREADS, smem, static_cast<cudaStream_t>(stream)>>>(
      x, H, k, idx, pairs, all_offsets, G, E, rank, px, pm, cap_rows, slots, plan_offsets, plan_pairs, plan_active,
      plan_n_active);
  return launch_check("k_ep_dispatch");
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
