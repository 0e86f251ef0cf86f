// C-ABI of libmoe: argument checks, workspace carving and kernel launches.
#include <cstdarg>
#include <mutex>
#include <cstdio>
#include <cstring>

#include "gemv.cuh"
#include "kernels.cuh"
#include "tc_gemm.cu"
#include "decode_fused.cu"
#include "grouped_mma.cu"

namespace moe {

static thread_local char g_err[512] = "";
static int g_gemv_max_rows = 2;
static int g_grouped_mma = 0;            // buckets of 3..32 rows on the grouped mma.sync kernel (off: measured slower)

// Two library-owned streams per device for independent parts of a call (the
// shared expert, the GEMV buckets), forked from and joined back into the
// caller's stream with events, so a captured graph gets the same branches.
// Created on first use, kept until exit; the fork-launch-join sequence of a
// call holds g_fork_mu so that concurrent host threads do not mix events.
struct SideStreams {
  cudaStream_t st[2] = {nullptr, nullptr};
  cudaEvent_t ev[4] = {nullptr, nullptr, nullptr, nullptr};
};
static std::recursive_mutex g_fork_mu;
static SideStreams* side_streams() {
  static SideStreams per_dev[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  SideStreams& S = per_dev[dev];
  if (!S.st[0]) {
    for (int i = 0; i < 2; ++i)
      if (cudaStreamCreateWithFlags(&S.st[i], cudaStreamNonBlocking) != cudaSuccess) { cudaGetLastError(); return nullptr; }
    for (int i = 0; i < 4; ++i)
      if (cudaEventCreateWithFlags(&S.ev[i], cudaEventDisableTiming) != cudaSuccess) { cudaGetLastError(); return nullptr; }
  }
  return &S;
}
int cuda_check(cudaError_t e, const char* what);
// `to` waits for the work issued so far on `from` (event ev)
static int stream_after(cudaStream_t to, cudaStream_t from, cudaEvent_t ev) {
  int st = cuda_check(cudaEventRecord(ev, from), "cudaEventRecord");
  if (st) return st;
  return cuda_check(cudaStreamWaitEvent(to, ev, 0), "cudaStreamWaitEvent");
}

// CTAs of the persistent grouped kernel: one per SM (cached per device).
static int grouped_grid() {
  static int cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int nsm = 0;
    if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || nsm <= 0) nsm = 148;
    cached[dev] = nsm;
  }
  return cached[dev];
}
static int g_decode_fused = 1;
static int g_decode_spec = 0;
static int g_decode_prefetch = 0;
static unsigned long long* g_decode_stamps = nullptr;

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_check(cudaError_t e, const char* what) {
  if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return MOE_OK;
}

int launch_check(const char* what) { return cuda_check(cudaGetLastError(), what); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static size_t align_up(size_t n, size_t a = 256) { return (n + a - 1) / a * a; }

static void blob_offsets(int H, int I, size_t off[9]) {
  const size_t q = static_cast<size_t>(I) * H / 2, s = static_cast<size_t>(I) * (H / 64) * 2;
  size_t o = 0;
  for (int m = 0; m < 3; ++m) {
    off[3 * m + 0] = o; o += q;
    off[3 * m + 1] = o; o += s;
    off[3 * m + 2] = o; o += s;
  }
}

static int check_dims(int T, int H, int I, int E, int k) {
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T must be >= 0 (got %d)", T);
  if (H <= 0 || H % 64) return fail(MOE_ERR_INVALID_ARG, "H must be a positive multiple of 64 (got %d)", H);
  if (I <= 0 || I % 64) return fail(MOE_ERR_INVALID_ARG, "I must be a positive multiple of 64 (got %d)", I);
  if (E <= 0 || E % 8 || E > 1024) return fail(MOE_ERR_INVALID_ARG, "E must be a multiple of 8 in [8, 1024] (got %d)", E);
  if (k < 1 || k > 8 || k > E) return fail(MOE_ERR_INVALID_ARG, "k must be in [1, min(8, E)] (got %d)", k);
  return MOE_OK;
}

// Raise a kernel's dynamic shared-memory limit once per (device, kernel);
// later calls (also inside stream capture) find it done and make no API call.
static int set_smem(const void* fn, size_t bytes) {
  if (bytes <= 48 * 1024) return MOE_OK;
  struct Entry { const void* fn; int dev; size_t bytes; };
  static Entry table[64];
  static int n = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  for (int i = 0; i < n; ++i)
    if (table[i].fn == fn && table[i].dev == dev && table[i].bytes >= bytes) return MOE_OK;
  int st = cuda_check(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(bytes)),
                      "cudaFuncSetAttribute(smem)");
  if (st) return st;
  for (int i = 0; i < n; ++i)
    if (table[i].fn == fn && table[i].dev == dev) { table[i].bytes = bytes; return MOE_OK; }
  if (n < 64) table[n++] = Entry{fn, dev, bytes};
  return MOE_OK;
}

static size_t gemv_smem(int K) {
  return GEMV_RG * staged_row_bytes(K) + static_cast<size_t>(GEMV_RG) * (K / 8) * sizeof(float2);
}

}  // namespace moe

using namespace moe;

extern "C" {

const char* moe_last_error_string(void) { return g_err; }

int moe_version(void) { return 100; }

int moe_sync(void* stream) {
  int st = cuda_check(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)), "moe_sync");
  if (st) return st;
  unsigned int w = 0;
  st = cuda_check(cudaMemcpyFromSymbol(&w, g_check_word, sizeof(w)), "read check word");
  if (st) return st;
  if (w != 0) {
    unsigned int z = 0;
    cudaMemcpyToSymbol(g_check_word, &z, sizeof(z));
    return fail(MOE_ERR_DEVICE_CHECK, "device check word 0x%x (1: expert id, 2: pair id, 4: wait)", w);
  }
  return MOE_OK;
}

size_t moe_blob_bytes(int H, int I, size_t* offsets9) {
  if (H <= 0 || I <= 0 || H % 64 || I % 64) return 0;
  size_t off[9];
  blob_offsets(H, I, off);
  if (offsets9) memcpy(offsets9, off, sizeof(off));
  return 3 * (static_cast<size_t>(I) * H / 2 + static_cast<size_t>(I) * (H / 64) * 4);
}

int moe_set_grouped_mma(int enable) {
  g_grouped_mma = enable ? 1 : 0;
  return MOE_OK;
}

int moe_set_gemv_max_rows(int rows) {
  if (rows < 0) return fail(MOE_ERR_INVALID_ARG, "gemv_max_rows must be >= 0");
  g_gemv_max_rows = rows;
  return MOE_OK;
}

int moe_rmsnorm(const float* h, int T, int H, float eps, uint16_t* x, void* stream) {
  if (T < 0 || H <= 0 || H % 64) return fail(MOE_ERR_INVALID_ARG, "moe_rmsnorm: bad T/H");
  if (T == 0) return MOE_OK;
  if (!h || !x || !aligned16(h) || !aligned16(x)) return fail(MOE_ERR_INVALID_ARG, "moe_rmsnorm: bad pointer");
  k_rmsnorm<<<T, 256, 0, static_cast<cudaStream_t>(stream)>>>(h, H, eps, x);
  return launch_check("k_rmsnorm");
}

int moe_router_topk(const uint16_t* x, int T, int H, const moe_qmat* router, const float* bias,
                    int bias_per_row, int E, int k, int32_t* idx, float* gates, float* logits_opt,
                    void* stream) {
  int st = check_dims(T, H, 64, E, k);
  if (st) return st;
  if (T == 0) return MOE_OK;
  if (!x || !router || !idx || !gates || !router->q || !router->s || !router->b)
    return fail(MOE_ERR_INVALID_ARG, "moe_router_topk: NULL pointer");
  if (router->bits != 8 || router->out != E || router->in != H)
    return fail(MOE_ERR_INVALID_ARG, "moe_router_topk: router must be 8-bit [E=%d, H=%d]", E, H);
  if (!aligned16(x) || !aligned16(router->q)) return fail(MOE_ERR_INVALID_ARG, "moe_router_topk: misaligned");
  const size_t smem = router_smem_bytes(H, E);
  if (smem > 227 * 1024) return fail(MOE_ERR_UNSUPPORTED, "moe_router_topk: H=%d E=%d too large", H, E);
  st = set_smem(reinterpret_cast<const void*>(k_router_topk), smem);
  if (st) return st;
  const int nblk = (T + ROUTER_TB - 1) / ROUTER_TB;
  k_router_topk<<<nblk * 8, 256, smem, static_cast<cudaStream_t>(stream)>>>(
      x, T, H, router->q, router->s, router->b, bias, bias_per_row, E, k, idx, gates, logits_opt);
  return launch_check("k_router_topk");
}

int moe_bucket(const int32_t* idx, int T, int k, int E, int32_t* offsets, int32_t* pairs,
               int32_t* active, int32_t* n_active, void* stream) {
  int st = check_dims(T, 64, 64, E, k);
  if (st) return st;
  if (static_cast<long>(T) * k > 65536) return fail(MOE_ERR_UNSUPPORTED, "moe_bucket: T*k > 65536");
  if (!idx || !offsets || !pairs || !active || !n_active) return fail(MOE_ERR_INVALID_ARG, "moe_bucket: NULL pointer");
  k_bucket<<<1, 256, 2 * E * sizeof(int), static_cast<cudaStream_t>(stream)>>>(idx, T * k, E, offsets, pairs,
                                                                              active, n_active);
  return launch_check("k_bucket");
}

size_t moe_expert_workspace_size(int T, int H, int I, int k) {
  // fp16 activation between the projections + fp16 copy of x for the tensor-core path
  return align_up(static_cast<size_t>(T) * k * I * sizeof(__half)) + align_up(static_cast<size_t>(T) * H * sizeof(__half));
}

// Paired activation rows (x and the gate/up activation) for the grouped
// mma.sync kernel: fp16 pairs [rows, K] plus fp32 group sums [rows, K/64] x 2.
static size_t mma_extra_bytes(int T, int H, int I, int k) {
  const size_t tk = static_cast<size_t>(T) * k;
  return align_up(static_cast<size_t>(T) * H * 2) + align_up(static_cast<size_t>(T) * (H / 64) * 8) +
         align_up(tk * I * 2) + align_up(tk * (I / 64) * 8) + align_up(8);   // + the two work counters
}

size_t moe_expert_workspace_size_mma(int T, int H, int I, int k) {
  return moe_expert_workspace_size(T, H, I, k) + mma_extra_bytes(T, H, I, k);
}

int moe_expert_forward(const uint16_t* x, int T, int H, int I, int E, int k, const void* const* blob_ptrs,
                       const int32_t* offsets, const int32_t* pairs, const int32_t* active,
                       const int32_t* n_active, float* y_pairs, void* ws, size_t ws_bytes, void* stream) {
  int st = check_dims(T, H, I, E, k);
  if (st) return st;
  if (T == 0) return MOE_OK;
  if (!x || !blob_ptrs || !offsets || !pairs || !active || !n_active || !y_pairs || !ws)
    return fail(MOE_ERR_INVALID_ARG, "moe_expert_forward: NULL pointer");
  if (ws_bytes < moe_expert_workspace_size(T, H, I, k))
    return fail(MOE_ERR_INVALID_ARG, "moe_expert_forward: workspace too small");
  if (!aligned16(x) || !aligned16(ws) || !aligned16(y_pairs))
    return fail(MOE_ERR_INVALID_ARG, "moe_expert_forward: misaligned pointer");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  __half* act = static_cast<__half*>(ws);
  __half* xh = reinterpret_cast<__half*>(static_cast<char*>(ws) + align_up(static_cast<size_t>(T) * k * I * sizeof(__half)));
  const int maxA = T * k < E ? T * k : E;
  // Buckets of at most gemv_max_rows rows go to the GEMV kernels, larger ones
  // to the tensor-core kernel (shapes it supports: H % 128 == 0, H, I <= 4096);
  // with the larger workspace, buckets of up to GM_NMAX rows go to the grouped
  // mma.sync kernel instead.
  const bool tc = T > g_gemv_max_rows && H % 128 == 0 && H <= 4096 && I <= 4096;
  const int gemv_rows = tc ? g_gemv_max_rows : (1 << 30);
  const bool mma = tc && g_grouped_mma && grouped_mma_ok(H, I) &&
                   ws_bytes >= moe_expert_workspace_size_mma(T, H, I, k);
  const int tc_min = mma ? GM_NMAX : g_gemv_max_rows;     // the tensor-core kernel takes buckets above this
  char* xw = static_cast<char*>(ws) + moe_expert_workspace_size(T, H, I, k);
  uint4* xP = reinterpret_cast<uint4*>(xw);
  float2* xS = reinterpret_cast<float2*>(xw + align_up(static_cast<size_t>(T) * H * 2));
  uint4* aP = reinterpret_cast<uint4*>(xw + align_up(static_cast<size_t>(T) * H * 2) +
                                       align_up(static_cast<size_t>(T) * (H / 64) * 8));
  float2* aS = reinterpret_cast<float2*>(reinterpret_cast<char*>(aP) + align_up(static_cast<size_t>(T) * k * I * 2));
  unsigned* queues = reinterpret_cast<unsigned*>(reinterpret_cast<char*>(aS) +
                                                 align_up(static_cast<size_t>(T) * k * (I / 64) * 8));
  GmArgs gm{};
  if (mma) {
    const size_t gsm = grouped_mma_smem(H, I);
    if ((st = set_smem(reinterpret_cast<const void*>(k_group_mma), gsm))) return st;
    const long nw = static_cast<long>(T) * (H / 8);
    k_pair_rows<<<static_cast<int>((nw + 255) / 256 < 1024 ? (nw + 255) / 256 : 1024), 256, 0, s>>>(x, 1, T, H, xP, xS);
    if ((st = launch_check("k_pair_rows(x)"))) return st;
    gm.mode = 0; gm.P = xP; gm.S = xS; gm.T = T; gm.H = H; gm.I = I; gm.E = E; gm.k = k;
    gm.blob_ptrs = blob_ptrs; blob_offsets(H, I, gm.off);
    gm.offsets = offsets; gm.pairs = pairs; gm.active = active; gm.n_active = n_active;
    gm.lo = g_gemv_max_rows; gm.hi = GM_NMAX;
    gm.act_out = static_cast<__half*>(ws); gm.y_out = y_pairs;
    if ((st = cuda_check(cudaMemsetAsync(queues, 0, 8, s), "zero work counters"))) return st;
    gm.queue = queues;
    k_group_mma<<<grouped_grid(), GM_THREADS, gsm, s>>>(gm);
    if ((st = launch_check("k_group_mma(gate/up)"))) return st;
  }

  // with the tensor-core path, the GEMV buckets (disjoint rows of act and
  // y_pairs) run on a side stream alongside it
  std::unique_lock<std::recursive_mutex> fork_lock(g_fork_mu, std::defer_lock);
  SideStreams* side = tc ? side_streams() : nullptr;
  cudaStream_t gs = s;
  if (side) {
    fork_lock.lock();
    gs = side->st[1];
    if ((st = stream_after(gs, s, side->ev[2]))) return st;
  }
  GateUpArgs g{};
  g.x = x; g.T = T; g.H = H; g.I = I; g.E = E; g.k = k;
  g.blob_ptrs = blob_ptrs; g.offsets = offsets; g.pairs = pairs; g.active = active; g.n_active = n_active;
  g.max_rows = gemv_rows;
  blob_offsets(H, I, g.off);
  g.act = act;
  size_t sm = gemv_smem(H);
  if ((st = set_smem(reinterpret_cast<const void*>(k_gateup_gemv), sm))) return st;
  k_gateup_gemv<<<dim3((I + GEMV_ROWS - 1) / GEMV_ROWS, maxA), 256, sm, gs>>>(g);
  if ((st = launch_check("k_gateup_gemv"))) return st;

  TcArgs ta{};
  if (tc) {
    const size_t n8 = static_cast<size_t>(T) * H / 8;
    k_to_f16<<<static_cast<int>((n8 + 255) / 256 < 1024 ? (n8 + 255) / 256 : 1024), 256, 0, s>>>(x, n8, xh);
    if ((st = launch_check("k_to_f16"))) return st;
    ta.mode = 0; ta.xh = xh; ta.T = T; ta.H = H; ta.I = I; ta.E = E; ta.k = k;
    ta.blob_ptrs = blob_ptrs; ta.offsets = offsets; ta.pairs = pairs; ta.active = active; ta.n_active = n_active;
    ta.max_rows = tc_min;
    blob_offsets(H, I, ta.off);
    ta.act_out = act; ta.act_in = act; ta.y_out = y_pairs;
    if ((st = set_smem(reinterpret_cast<const void*>(k_expert_tc), TC_SMEM))) return st;
    k_expert_tc<<<dim3(I / 64, maxA), TC_THREADS, TC_SMEM, s>>>(ta);
    if ((st = launch_check("k_expert_tc(gate/up)"))) return st;
  }

  if (mma) {
    const long nw = static_cast<long>(T) * k * (I / 8);
    k_pair_rows<<<static_cast<int>((nw + 255) / 256 < 1024 ? (nw + 255) / 256 : 1024), 256, 0, s>>>(
        reinterpret_cast<const uint16_t*>(act), 0, T * k, I, aP, aS);
    if ((st = launch_check("k_pair_rows(act)"))) return st;
    gm.mode = 1; gm.P = aP; gm.S = aS; gm.queue = queues + 1;
    k_group_mma<<<grouped_grid(), GM_THREADS, grouped_mma_smem(H, I), s>>>(gm);
    if ((st = launch_check("k_group_mma(down)"))) return st;
  }
  DownArgs d{};
  d.act = act; d.T = T; d.H = H; d.I = I; d.E = E; d.k = k;
  d.blob_ptrs = blob_ptrs; d.offsets = offsets; d.pairs = pairs; d.active = active; d.n_active = n_active;
  d.max_rows = gemv_rows;
  blob_offsets(H, I, d.off);
  d.y = y_pairs;
  sm = gemv_smem(I);
  if ((st = set_smem(reinterpret_cast<const void*>(k_down_gemv), sm))) return st;
  k_down_gemv<<<dim3((H + GEMV_ROWS - 1) / GEMV_ROWS, maxA), 256, sm, gs>>>(d);
  if ((st = launch_check("k_down_gemv"))) return st;
  if (tc) {
    ta.mode = 1;
    k_expert_tc<<<dim3(H / 128, maxA), TC_THREADS, TC_SMEM, s>>>(ta);
    if ((st = launch_check("k_expert_tc(down)"))) return st;
  }
  if (side && (st = stream_after(s, gs, side->ev[3]))) return st;     // join
  return MOE_OK;
}

size_t moe_shared_workspace_size(int T, int H, int Is) {
  // fp16 activation [T, Is]; for the tensor-core path also fp16 x [T, H] and
  // the one-expert bucket list (offsets[2], active[1], n_active, pairs[T])
  return align_up(static_cast<size_t>(T) * Is * sizeof(__half)) + align_up(static_cast<size_t>(T) * H * sizeof(__half)) +
         3 * align_up(16) + align_up(static_cast<size_t>(T) * 4);
}

int moe_shared_forward(const uint16_t* x, int T, int H, int Is, const moe_qmat* sh, float* ysh, void* ws,
                       size_t ws_bytes, void* stream) {
  int st = check_dims(T, H, Is, 8, 1);
  if (st) return st;
  if (T == 0) return MOE_OK;
  if (!x || !sh || !ysh || !ws) return fail(MOE_ERR_INVALID_ARG, "moe_shared_forward: NULL pointer");
  for (int m = 0; m < 3; ++m) {
    const int out = m < 2 ? Is : H, in = m < 2 ? H : Is;
    if (!sh[m].q || !sh[m].s || !sh[m].b || sh[m].bits != 4 || sh[m].out != out || sh[m].in != in)
      return fail(MOE_ERR_INVALID_ARG, "moe_shared_forward: matrix %d must be 4-bit [%d, %d]", m, out, in);
    if (!aligned16(sh[m].q)) return fail(MOE_ERR_INVALID_ARG, "moe_shared_forward: misaligned weights");
  }
  if (ws_bytes < moe_shared_workspace_size(T, H, Is))
    return fail(MOE_ERR_INVALID_ARG, "moe_shared_forward: workspace too small");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  __half* act = static_cast<__half*>(ws);
  // several rows: the three matrices on the tensor cores as one expert whose
  // bucket is every row (same kernel and arithmetic as the routed buckets)
  if (T > g_gemv_max_rows && H % 128 == 0 && H <= 4096 && Is <= 4096) {
    char* p = static_cast<char*>(ws) + align_up(static_cast<size_t>(T) * Is * sizeof(__half));
    __half* xh = reinterpret_cast<__half*>(p);
    p += align_up(static_cast<size_t>(T) * H * sizeof(__half));
    int32_t* offsets = reinterpret_cast<int32_t*>(p); p += align_up(16);
    int32_t* active = reinterpret_cast<int32_t*>(p); p += align_up(16);
    int32_t* n_active = reinterpret_cast<int32_t*>(p); p += align_up(16);
    int32_t* pairs = reinterpret_cast<int32_t*>(p);
    k_one_bucket<<<(T + 255) / 256 < 64 ? (T + 255) / 256 : 64, 256, 0, s>>>(T, offsets, pairs, active, n_active);
    if ((st = launch_check("k_one_bucket"))) return st;
    const size_t n8 = static_cast<size_t>(T) * H / 8;
    k_to_f16<<<static_cast<int>((n8 + 255) / 256 < 1024 ? (n8 + 255) / 256 : 1024), 256, 0, s>>>(x, n8, xh);
    if ((st = launch_check("k_to_f16(shared)"))) return st;
    TcArgs ta{};
    ta.mode = 0; ta.xh = xh; ta.T = T; ta.H = H; ta.I = Is; ta.E = 1; ta.k = 1;
    ta.blob_ptrs = nullptr;
    for (int m = 0; m < 3; ++m) {
      ta.mq[m] = reinterpret_cast<const uint8_t*>(sh[m].q); ta.ms[m] = sh[m].s; ta.mb[m] = sh[m].b;
    }
    ta.offsets = offsets; ta.pairs = pairs; ta.active = active; ta.n_active = n_active;
    ta.max_rows = 0;
    ta.act_out = act; ta.act_in = act; ta.y_out = ysh;
    if ((st = set_smem(reinterpret_cast<const void*>(k_expert_tc), TC_SMEM))) return st;
    k_expert_tc<<<dim3(Is / 64, 1), TC_THREADS, TC_SMEM, s>>>(ta);
    if ((st = launch_check("k_expert_tc(shared gate/up)"))) return st;
    ta.mode = 1;
    k_expert_tc<<<dim3(H / 128, 1), TC_THREADS, TC_SMEM, s>>>(ta);
    return launch_check("k_expert_tc(shared down)");
  }
  GateUpArgs g{};
  g.x = x; g.T = T; g.H = H; g.I = Is; g.E = 1; g.k = 1; g.max_rows = 1 << 30;
  g.gq = sh[0].q; g.gs = sh[0].s; g.gb = sh[0].b;
  g.uq = sh[1].q; g.us = sh[1].s; g.ub = sh[1].b;
  g.act = act;
  size_t sm = gemv_smem(H);
  if ((st = set_smem(reinterpret_cast<const void*>(k_gateup_gemv), sm))) return st;
  k_gateup_gemv<<<dim3((Is + GEMV_ROWS - 1) / GEMV_ROWS, 1), 256, sm, s>>>(g);
  if ((st = launch_check("k_gateup_gemv(shared)"))) return st;
  DownArgs d{};
  d.act = act; d.T = T; d.H = H; d.I = Is; d.E = 1; d.k = 1; d.max_rows = 1 << 30;
  d.dq = sh[2].q; d.ds = sh[2].s; d.db = sh[2].b;
  d.y = ysh;
  sm = gemv_smem(Is);
  if ((st = set_smem(reinterpret_cast<const void*>(k_down_gemv), sm))) return st;
  k_down_gemv<<<dim3((H + GEMV_ROWS - 1) / GEMV_ROWS, 1), 256, sm, s>>>(d);
  return launch_check("k_down_gemv(shared)");
}

int moe_combine(const float* y_pairs, const float* gates, const float* ysh, int T, int H, int k, uint16_t* y,
                float* residual_inout, void* stream) {
  if (T < 0 || H <= 0 || k < 1 || k > 8) return fail(MOE_ERR_INVALID_ARG, "moe_combine: bad T/H/k");
  if (T == 0) return MOE_OK;
  if (!y_pairs || !gates) return fail(MOE_ERR_INVALID_ARG, "moe_combine: NULL pointer");
  k_combine<<<dim3((H + 255) / 256, T), 256, 0, static_cast<cudaStream_t>(stream)>>>(y_pairs, gates, ysh, H, k, y,
                                                                                 residual_inout);
  return launch_check("k_combine");
}

size_t moe_layer_workspace_size(int T, int H, int I, int Is, int E, int k) {
  size_t n = 0;
  n += align_up(static_cast<size_t>(T) * H * 2);        // x
  n += align_up(static_cast<size_t>(T) * k * 4) * 2;    // idx, gates
  n += align_up(static_cast<size_t>(E + 1) * 4);        // offsets
  n += align_up(static_cast<size_t>(T) * k * 4);        // pairs
  n += align_up(static_cast<size_t>(E) * 4);            // active
  n += align_up(4);                                     // n_active
  n += align_up(static_cast<size_t>(T) * k * H * 4);    // y_pairs
  n += align_up(static_cast<size_t>(T) * H * 4);        // ysh
  n += moe_expert_workspace_size_mma(T, H, I, k);
  n += moe_shared_workspace_size(T, H, Is);
  return n;
}

int moe_layer_forward(const float* h_in, float* h_out, const uint16_t* x_in, int T, int H, int I, int Is, int E,
                      int k, const moe_qmat* router, const float* bias, int bias_per_row,
                      const void* const* blob_ptrs, const moe_qmat* shared, uint16_t* x_out, uint16_t* y,
                      int32_t* idx_out, float* gates_out, void* ws, size_t ws_bytes, void* stream) {
  int st = check_dims(T, H, I, E, k);
  if (st) return st;
  if (T == 0) return MOE_OK;
  if (!x_in && !h_in) return fail(MOE_ERR_INVALID_ARG, "moe_layer_forward: need h_in or x_in");
  if (h_out && !h_in) return fail(MOE_ERR_INVALID_ARG, "moe_layer_forward: h_out needs h_in");
  if (!ws || ws_bytes < moe_layer_workspace_size(T, H, I, Is, E, k))
    return fail(MOE_ERR_INVALID_ARG, "moe_layer_forward: workspace too small");
  char* p = static_cast<char*>(ws);
  auto take = [&](size_t n) { char* q = p; p += align_up(n); return q; };
  uint16_t* x = reinterpret_cast<uint16_t*>(take(static_cast<size_t>(T) * H * 2));
  int32_t* idx = reinterpret_cast<int32_t*>(take(static_cast<size_t>(T) * k * 4));
  float* gates = reinterpret_cast<float*>(take(static_cast<size_t>(T) * k * 4));
  int32_t* offsets = reinterpret_cast<int32_t*>(take(static_cast<size_t>(E + 1) * 4));
  int32_t* pairs = reinterpret_cast<int32_t*>(take(static_cast<size_t>(T) * k * 4));
  int32_t* active = reinterpret_cast<int32_t*>(take(static_cast<size_t>(E) * 4));
  int32_t* n_active = reinterpret_cast<int32_t*>(take(4));
  float* y_pairs = reinterpret_cast<float*>(take(static_cast<size_t>(T) * k * H * 4));
  float* ysh = reinterpret_cast<float*>(take(static_cast<size_t>(T) * H * 4));
  const size_t ews = moe_expert_workspace_size_mma(T, H, I, k);
  void* ew = take(ews);
  const size_t sws = moe_shared_workspace_size(T, H, Is);
  void* sw = take(sws);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  const uint16_t* xin = x_in;
  if (!xin) {
    if ((st = moe_rmsnorm(h_in, T, H, 1e-6f, x, stream))) return st;
    xin = x;
  }
  if (x_out && (st = cuda_check(cudaMemcpyAsync(x_out, xin, static_cast<size_t>(T) * H * 2,
                                                cudaMemcpyDeviceToDevice, s), "copy x_out")))
    return st;
  // the shared expert needs only x: it runs on a side stream alongside the
  // router, the buckets and the routed experts (several rows only)
  std::unique_lock<std::recursive_mutex> fork_lock(g_fork_mu, std::defer_lock);
  SideStreams* side = T > g_gemv_max_rows ? side_streams() : nullptr;
  cudaStream_t shs = s;
  if (side) {
    fork_lock.lock();
    shs = side->st[0];
    if ((st = stream_after(shs, s, side->ev[0]))) return st;
  }
  if ((st = moe_shared_forward(xin, T, H, Is, shared, ysh, sw, sws, shs))) return st;
  if ((st = moe_router_topk(xin, T, H, router, bias, bias_per_row, E, k, idx, gates, nullptr, stream))) return st;
  if ((st = moe_bucket(idx, T, k, E, offsets, pairs, active, n_active, stream))) return st;
  if ((st = moe_expert_forward(xin, T, H, I, E, k, blob_ptrs, offsets, pairs, active, n_active, y_pairs, ew, ews,
                               stream)))
    return st;
  if (side && (st = stream_after(s, shs, side->ev[1]))) return st;   // join before the combine
  float* resid = nullptr;
  if (h_out) {
    if (h_out != h_in &&
        (st = cuda_check(cudaMemcpyAsync(h_out, h_in, static_cast<size_t>(T) * H * 4, cudaMemcpyDeviceToDevice, s),
                         "copy h")))
      return st;
    resid = h_out;
  }
  if ((st = moe_combine(y_pairs, gates, ysh, T, H, k, y, resid, stream))) return st;
  if (idx_out && (st = cuda_check(cudaMemcpyAsync(idx_out, idx, static_cast<size_t>(T) * k * 4,
                                                  cudaMemcpyDeviceToDevice, s), "copy idx")))
    return st;
  if (gates_out && (st = cuda_check(cudaMemcpyAsync(gates_out, gates, static_cast<size_t>(T) * k * 4,
                                                    cudaMemcpyDeviceToDevice, s), "copy gates")))
    return st;
  return MOE_OK;
}

// Shapes the fused batch-1 kernel serves.
static bool fused_ok(int T, int H, int I, int Is, int E, int k, int bias_per_row, int G) {
  if (!g_decode_fused || T != 1 || bias_per_row) return false;
  return df_fits(H, I, Is, E, k, G);
}

// CTAs of the fused kernel: one per SM when one CTA with the largest shared
// memory the kernel may ask for fits on an SM (cached per device).
static int fused_grid() {
  static int cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cached[dev]) return cached[dev];
  const void* fn = reinterpret_cast<const void*>(k_decode_b1);
  if (set_smem(fn, DF_SMEM_LIMIT)) return 0;
  int nsm = 0, per = 0;
  if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, fn, DF_THREADS, DF_SMEM_LIMIT) != cudaSuccess || per < 1) {
    cudaGetLastError();
    return 0;
  }
  cached[dev] = nsm;
  return cached[dev];
}

static size_t fused_ws(int I, int Is, int E, int k) {
  return align_up(static_cast<size_t>(k * I + Is) * 2) + align_up(static_cast<size_t>(E) * 8) + 256;
}

static int launch_fused(float* h, int H, int I, int Is, int E, int k, int L, const moe_qmat* routers,
                        const float* const* biases, const void* const* const* blob_tables, const moe_qmat* shared,
                        uint16_t* x_trace, uint16_t* y_trace, int32_t* idx_trace, float* gates_trace, void* ws,
                        int G, cudaStream_t s) {
  if (!aligned16(h)) return fail(MOE_ERR_INVALID_ARG, "moe_decode_forward: h must be 16-byte aligned");
  char* w = static_cast<char*>(ws);
  __half* act = reinterpret_cast<__half*>(w);
  unsigned long long* logits =
      reinterpret_cast<unsigned long long*>(w + align_up(static_cast<size_t>(k * I + Is) * 2));   // tagged
  unsigned* ctr = reinterpret_cast<unsigned*>(w + align_up(static_cast<size_t>(k * I + Is) * 2) +
                                              align_up(static_cast<size_t>(E) * 8));
  const size_t smem = decode_fused_smem(H, I, Is, E, k, G);
  int st;
  if ((st = set_smem(reinterpret_cast<const void*>(k_decode_b1), DF_SMEM_LIMIT))) return st;
  for (int l0 = 0; l0 < L; l0 += DF_MAX_LAYERS) {
    const int nl = L - l0 < DF_MAX_LAYERS ? L - l0 : DF_MAX_LAYERS;
    static DfArgs args;   // large parameter block; the launch copies it
    memset(&args, 0, sizeof(args));
    args.h = h; args.H = H; args.I = I; args.Is = Is; args.E = E; args.k = k; args.L = nl;
    blob_offsets(H, I, args.off);
    args.act = act; args.logits = logits; args.counter = ctr;
    const size_t TH = static_cast<size_t>(H), Tk = static_cast<size_t>(k);
    args.x_trace = x_trace ? x_trace + l0 * TH : nullptr;
    args.y_trace = y_trace ? y_trace + l0 * TH : nullptr;
    args.idx_trace = idx_trace ? idx_trace + l0 * Tk : nullptr;
    args.gates_trace = gates_trace ? gates_trace + l0 * Tk : nullptr;
    args.spec = g_decode_spec;
    args.prefetch = g_decode_prefetch;
    args.stamps = g_decode_stamps ? g_decode_stamps + static_cast<size_t>(l0) * G * 16 : nullptr;
    for (int l = 0; l < nl; ++l) {
      const moe_qmat& R = routers[l0 + l];
      DfLayer& d = args.layer[l];
      d.rq = R.q; d.rs = R.s; d.rb = R.b;
      d.bias = biases ? biases[l0 + l] : nullptr;
      d.blobs = blob_tables[l0 + l];
      for (int m = 0; m < 3; ++m) {
        const moe_qmat& S = shared[3 * (l0 + l) + m];
        d.sq[m] = S.q; d.ss[m] = S.s; d.sb[m] = S.b;
      }
    }
    if ((st = cuda_check(cudaMemsetAsync(ctr, 0, 256, s), "zero barrier counter and abort flag"))) return st;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(G, 1, 1);
    cfg.blockDim = dim3(DF_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeCooperative;
    at[0].val.cooperative = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if ((st = cuda_check(cudaLaunchKernelEx(&cfg, k_decode_b1, args), "k_decode_b1 launch"))) return st;
  }
  return MOE_OK;
}

int moe_set_decode_profile(unsigned long long* stamps) {
  g_decode_stamps = stamps;
  return MOE_OK;
}

int moe_decode_grid(void) { return fused_grid(); }

int moe_set_decode_prefetch(int flags) {
  if (flags < 0 || flags > 3) return fail(MOE_ERR_INVALID_ARG, "prefetch flags must be in [0, 3]");
  g_decode_prefetch = flags;
  return MOE_OK;
}

int moe_set_decode_fused(int enable, int spec_experts) {
  if (spec_experts < 0 || spec_experts > 8) return fail(MOE_ERR_INVALID_ARG, "spec_experts must be in [0, 8]");
  g_decode_fused = enable ? 1 : 0;
  g_decode_spec = spec_experts;
  return MOE_OK;
}

int moe_decode_launches(int T, int L) {
  if (T <= 0 || L <= 0) return 0;
  // fused batch-1 path: one kernel per DF_MAX_LAYERS layers; otherwise rmsnorm,
  // router, bucket, shared gate/up, shared down, expert gate/up, expert down and
  // combine per layer (plus the tensor-core kernels for multi-row buckets)
  if (T == 1 && g_decode_fused) return (L + DF_MAX_LAYERS - 1) / DF_MAX_LAYERS;
  return 8 * L;
}

size_t moe_decode_workspace_size(int T, int H, int I, int Is, int E, int k) {
  const size_t layered = moe_layer_workspace_size(T, H, I, Is, E, k);
  const size_t fused = fused_ws(I, Is, E, k);
  return layered > fused ? layered : fused;
}

int moe_decode_forward(float* h, int T, int H, int I, int Is, int E, int k, int L, const moe_qmat* routers,
                       const float* const* biases, int bias_per_row, const void* const* const* blob_tables,
                       const moe_qmat* shared, uint16_t* x_trace, uint16_t* y_trace, int32_t* idx_trace,
                       float* gates_trace, void* ws, size_t ws_bytes, void* stream) {
  int st = check_dims(T, H, I, E, k);
  if (st) return st;
  if (L < 0) return fail(MOE_ERR_INVALID_ARG, "moe_decode_forward: L < 0");
  if (T == 0 || L == 0) return MOE_OK;
  if (!h || !routers || !blob_tables || !shared) return fail(MOE_ERR_INVALID_ARG, "moe_decode_forward: NULL pointer");
  if (ws_bytes < moe_decode_workspace_size(T, H, I, Is, E, k))
    return fail(MOE_ERR_INVALID_ARG, "moe_decode_forward: workspace too small");
  const int G = (T == 1 && g_decode_fused) ? fused_grid() : 0;
  if (fused_ok(T, H, I, Is, E, k, bias_per_row, G))
    return launch_fused(h, H, I, Is, E, k, L, routers, biases, blob_tables, shared, x_trace, y_trace, idx_trace,
                        gates_trace, ws, G, static_cast<cudaStream_t>(stream));
  const size_t TH = static_cast<size_t>(T) * H, Tk = static_cast<size_t>(T) * k;
  for (int l = 0; l < L; ++l) {
    const float* b = biases ? biases[l] : nullptr;
    st = moe_layer_forward(h, h, nullptr, T, H, I, Is, E, k, &routers[l], b, bias_per_row, blob_tables[l],
                           &shared[3 * l], x_trace ? x_trace + l * TH : nullptr, y_trace ? y_trace + l * TH : nullptr,
                           idx_trace ? idx_trace + l * Tk : nullptr, gates_trace ? gates_trace + l * Tk : nullptr, ws,
                           ws_bytes, stream);
    if (st) return st;
  }
  return MOE_OK;
}

}  // extern "C"
