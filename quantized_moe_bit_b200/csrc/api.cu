// C-ABI of libmoe: argument checks, workspace carving and kernel launches.
#include <cstdarg>
#include <mutex>
#include <cstdio>
#include <cstring>

#include "gemv.cuh"
#include "kernels.cuh"
#include "moe_gemm.cu"
#include "decode_fused.cu"

namespace moe {

static thread_local char g_err[512] = "";
// phase timestamps of the persistent batch-1 kernel for this thread's calls (tracing aid)
static thread_local unsigned long long* g_decode_stamps = nullptr;

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

static int check_flags(int flags) {
  if (flags & ~(MOE_FLAG_GEMV | MOE_FLAG_TC | MOE_FLAG_LAYERED))
    return fail(MOE_ERR_INVALID_ARG, "unknown flag bits 0x%x", flags);
  if ((flags & MOE_FLAG_GEMV) && (flags & MOE_FLAG_TC))
    return fail(MOE_ERR_INVALID_ARG, "MOE_FLAG_GEMV and MOE_FLAG_TC exclude each other");
  return MOE_OK;
}

// Raise a kernel's dynamic shared-memory limit once per (device, kernel);
// later calls (also inside stream capture) find it done and make no API call.
static int set_smem(const void* fn, size_t bytes) {
  if (bytes <= 48 * 1024) return MOE_OK;
  struct Entry { const void* fn; int dev; size_t bytes; };
  static Entry table[64];
  static int n = 0;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
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

// SMs of the current device (cached per device): the persistent grids.
static int sm_count() {
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

// ------------------------------------------------------- tensor maps (TMA)
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

// The GM_NBOX activation tensor maps of one fp16 matrix [rows, cols]
// (row-major): boxes of 64 columns (128 bytes, 128-byte swizzle) by
// 16, 32, 64 or 128 rows; rows beyond the matrix read as zero.
static int make_act_maps(CUtensorMap* maps, const void* base, int rows, int cols) {
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  for (int i = 0; i < GM_NBOX; ++i) {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
    const cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(gm_box_rows(i))};
    const cuuint32_t es[2] = {1u, 1u};
    const CUresult r = enc(&maps[i], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                           es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  }
  return MOE_OK;
}

// The tensor map of a matrix's packed codes: uint8 [rows, row_bytes]
// (row-major), boxes of 128 bytes (256 4-bit values) by box_rows rows,
// 128-byte swizzle; bytes beyond a row's end read as zero.
static int make_code_map(CUtensorMap* map, const void* base, int rows, int row_bytes, int box_rows) {
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
  const cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t es[2] = {1u, 1u};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled (codes) failed (%d)", static_cast<int>(r));
  return MOE_OK;
}

// ------------------------------------------------------- expert path
// Which kernels serve the experts of a T-row call: the GEMV kernels for T <= 2
// (or MOE_FLAG_GEMV), the grouped GEMM otherwise (or MOE_FLAG_TC), when the
// shapes fit it.
static bool gemm_shapes_ok(int T, int H, int I, int Is, int E, int k) {
  if (H % GM_BM || H > GM_MAX_G * 64 || I > GM_MAX_G * 64 || Is > GM_MAX_G * 64) return false;
  const long P = static_cast<long>(T) * k;
  const long chunks = (E < P ? E : P) + (P + GM_NMAX - 1) / GM_NMAX + (T + GM_NMAX - 1) / GM_NMAX;
  return P < (1L << 24) && chunks <= GM_MAX_CHUNKS;
}
static bool use_gemm(int T, int H, int I, int Is, int E, int k, int flags) {
  if (flags & MOE_FLAG_GEMV) return false;
  if (!(flags & MOE_FLAG_TC) && T <= 2) return false;
  return gemm_shapes_ok(T, H, I, Is, E, k);
}

// Workspace carving of the expert calls (every region 256-byte aligned).
struct ExpertWs {      // routed experts
  GmPlan* plan;
  CUtensorMap* maps;   // [GM_MAX_CTAS][GM_MAP_RING][2] per-CTA patched code maps (grouped GEMM only)
  __half* act;         // [T*k, I] bucket order
  __half* xs;          // [T*k, H] the layer input gathered into bucket order (grouped GEMM only)
};
constexpr size_t GM_RING_BYTES = static_cast<size_t>(GM_MAX_CTAS) * GM_MAP_RING * 2 * sizeof(CUtensorMap);
static size_t expert_ws_bytes(int T, int H, int I, int k) {
  const size_t P = static_cast<size_t>(T) * k;
  return align_up(sizeof(GmPlan)) + align_up(GM_RING_BYTES) + align_up(P * I * 2) + align_up(P * H * 2);
}
static ExpertWs carve_expert(void* ws, int T, int H, int I, int k) {
  const size_t P = static_cast<size_t>(T) * k;
  char* p = static_cast<char*>(ws);
  ExpertWs w;
  w.plan = reinterpret_cast<GmPlan*>(p); p += align_up(sizeof(GmPlan));
  w.maps = reinterpret_cast<CUtensorMap*>(p); p += align_up(GM_RING_BYTES);
  w.act = reinterpret_cast<__half*>(p); p += align_up(P * I * 2);
  w.xs = reinterpret_cast<__half*>(p);
  (void)H;
  return w;
}
struct SharedWs {
  GmPlan* plan;
  __half* act;         // [T, Is]
  __half* xh;          // [T, H] the layer input as fp16 (grouped GEMM only)
};
static size_t shared_ws_bytes(int T, int H, int Is) {
  return align_up(sizeof(GmPlan)) + align_up(static_cast<size_t>(T) * Is * 2) + align_up(static_cast<size_t>(T) * H * 2);
}
static SharedWs carve_shared(void* ws, int T, int H, int Is) {
  char* p = static_cast<char*>(ws);
  SharedWs w;
  w.plan = reinterpret_cast<GmPlan*>(p); p += align_up(sizeof(GmPlan));
  w.act = reinterpret_cast<__half*>(p); p += align_up(static_cast<size_t>(T) * Is * 2);
  w.xh = reinterpret_cast<__half*>(p);
  (void)H;
  return w;
}

// The grouped GEMM over a routed segment (rt != null) and/or the shared
// expert (sh != null) of one T-row step: prep, gate/up, down.
struct RoutedIn {
  const void* const* blob_ptrs; const int32_t* offsets; const int32_t* pairs; const int32_t* active;
  const int32_t* n_active; float* y_pairs; int I, E, k;
};
struct SharedIn {
  const moe_qmat* m; float* ysh; int Is;
};
static int run_gemm(const uint16_t* x, int T, int H, const RoutedIn* rt, const SharedIn* sh, GmPlan* plan,
                    CUtensorMap* map_ring, __half* act_r, __half* xs, __half* act_s, __half* xh, cudaStream_t s) {
  int st;
  const int k = rt ? rt->k : 1;
  const long P = rt ? static_cast<long>(T) * k : 0;
  {
    const long rows = P + (sh ? T : 0);     // one row per block and step
    int blocks = static_cast<int>(rows < 4L * sm_count() ? rows : 4L * sm_count());
    blocks = blocks < 1 ? 1 : blocks;
    k_gm_prep<<<blocks, 256, 0, s>>>(x, T, H, k, rt ? rt->offsets : nullptr, rt ? rt->pairs : nullptr,
                                     rt ? rt->active : nullptr, rt ? rt->n_active : nullptr, rt ? rt->E : 0,
                                     rt ? 1 : 0, sh ? T : 0, xs, sh ? xh : nullptr, plan);
    if ((st = launch_check("k_gm_prep"))) return st;
  }
  if ((st = set_smem(reinterpret_cast<const void*>(k_moe_gemm), GM_SMEM))) return st;
  static thread_local GemmArgs g;       // large parameter block (tensor maps); the launch copies it
  memset(&g, 0, sizeof(g));
  g.H = H;
  g.plan = plan;
  if (rt) {
    g.I = rt->I; g.E = rt->E; g.k = rt->k;
    g.blob_ptrs = rt->blob_ptrs; g.pairs = rt->pairs; g.P = static_cast<int>(P);
    blob_offsets(H, rt->I, g.off);
    g.act_r = act_r; g.y_r = rt->y_pairs;
  }
  if (sh) {
    g.Is = sh->Is; g.Ts = T;
    for (int m = 0; m < 3; ++m) {
      g.sq[m] = reinterpret_cast<const uint8_t*>(sh->m[m].q); g.ss[m] = sh->m[m].s; g.sb[m] = sh->m[m].b;
    }
    g.act_s = act_s; g.y_s = sh->ysh;
  } else {
    g.Is = 64;   // unused (no shared chunks); keeps the m-tile count well defined
  }
  if (!rt) g.I = 64;
  const int grid = sm_count() < GM_MAX_CTAS ? sm_count() : GM_MAX_CTAS;
  g.map_ring = map_ring;
  for (int phase = 0; phase < 2; ++phase) {
    g.phase = phase;
    // code maps: the routed template (any valid address; replaced per item)
    // and the shared expert's matrices
    const int box_rows = phase == 0 ? 64 : GM_BM;
    if (rt && (st = make_code_map(&g.tmR, map_ring, phase == 0 ? rt->I : H, phase == 0 ? H / 2 : rt->I / 2, box_rows)))
      return st;
    if (sh) {
      if (phase == 0) {
        if ((st = make_code_map(&g.tmS[0], sh->m[0].q, sh->Is, H / 2, box_rows))) return st;
        if ((st = make_code_map(&g.tmS[1], sh->m[1].q, sh->Is, H / 2, box_rows))) return st;
      } else if ((st = make_code_map(&g.tmS[0], sh->m[2].q, H, sh->Is / 2, box_rows))) {
        return st;
      }
    }
    if (rt && (st = make_act_maps(g.tmB[1], phase == 0 ? static_cast<const void*>(xs) : act_r, static_cast<int>(P),
                                  phase == 0 ? H : rt->I)))
      return st;
    if (sh && (st = make_act_maps(g.tmB[0], phase == 0 ? static_cast<const void*>(xh) : act_s, T,
                                  phase == 0 ? H : sh->Is)))
      return st;
    k_moe_gemm<<<grid, GM_THREADS, GM_SMEM, s>>>(g);
    if ((st = launch_check(phase == 0 ? "k_moe_gemm(gate/up)" : "k_moe_gemm(down)"))) return st;
  }
  return MOE_OK;
}

static int check_shared_mats(const moe_qmat* sh, int H, int Is) {
  for (int m = 0; m < 3; ++m) {
    const int out = m < 2 ? Is : H, in = m < 2 ? H : Is;
    if (!sh[m].q || !sh[m].s || !sh[m].b || sh[m].bits != 4 || sh[m].out != out || sh[m].in != in)
      return fail(MOE_ERR_INVALID_ARG, "shared expert: matrix %d must be 4-bit [%d, %d]", m, out, in);
    if (!aligned16(sh[m].q) || !aligned16(sh[m].s) || !aligned16(sh[m].b))
      return fail(MOE_ERR_INVALID_ARG, "shared expert: matrix %d arrays must be 16-byte aligned", m);
  }
  return MOE_OK;
}

// GEMV path of the routed experts (every bucket): gate/up + GeGLU, then down.
static int run_routed_gemv(const uint16_t* x, int T, int H, int I, int E, int k, const void* const* blob_ptrs,
                           const int32_t* offsets, const int32_t* pairs, const int32_t* active,
                           const int32_t* n_active, float* y_pairs, __half* act, cudaStream_t s) {
  int st;
  const int maxA = T * k < E ? T * k : E;
  GateUpArgs g{};
  g.x = x; g.T = T; g.H = H; g.I = I; g.E = E; g.k = k;
  g.blob_ptrs = blob_ptrs; g.offsets = offsets; g.pairs = pairs; g.active = active; g.n_active = n_active;
  g.max_rows = 1 << 30;
  blob_offsets(H, I, g.off);
  g.act = act;
  size_t sm = gemv_smem(H);
  if ((st = set_smem(reinterpret_cast<const void*>(k_gateup_gemv), sm))) return st;
  k_gateup_gemv<<<dim3((I + GEMV_ROWS - 1) / GEMV_ROWS, maxA), 256, sm, s>>>(g);
  if ((st = launch_check("k_gateup_gemv"))) return st;
  DownArgs d{};
  d.act = act; d.T = T; d.H = H; d.I = I; d.E = E; d.k = k;
  d.blob_ptrs = blob_ptrs; d.offsets = offsets; d.pairs = pairs; d.active = active; d.n_active = n_active;
  d.max_rows = 1 << 30;
  blob_offsets(H, I, d.off);
  d.y = y_pairs;
  sm = gemv_smem(I);
  if ((st = set_smem(reinterpret_cast<const void*>(k_down_gemv), sm))) return st;
  k_down_gemv<<<dim3((H + GEMV_ROWS - 1) / GEMV_ROWS, maxA), 256, sm, s>>>(d);
  return launch_check("k_down_gemv");
}

// GEMV path of the shared expert.
static int run_shared_gemv(const uint16_t* x, int T, int H, int Is, const moe_qmat* sh, float* ysh, __half* act,
                           cudaStream_t s) {
  int st;
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
    return fail(MOE_ERR_DEVICE_CHECK, "device check word 0x%x (1: expert id, 2: pair id, 4: wait, 8: expert-parallel row past capacity)", w);
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
  k_router_topk<<<nblk * 8, ROUTER_THREADS, smem, static_cast<cudaStream_t>(stream)>>>(
      x, T, H, router->q, router->s, router->b, bias, bias_per_row, E, k, idx, gates, logits_opt);
  return launch_check("k_router_topk");
}

int moe_bucket(const int32_t* idx, int T, int k, int E, int32_t* offsets, int32_t* pairs,
               int32_t* active, int32_t* n_active, void* stream) {
  int st = check_dims(T, 64, 64, E, k);
  if (st) return st;
  if (static_cast<long>(T) * k > 65536) return fail(MOE_ERR_UNSUPPORTED, "moe_bucket: T*k > 65536");
  if (!idx || !offsets || !pairs || !active || !n_active) return fail(MOE_ERR_INVALID_ARG, "moe_bucket: NULL pointer");
  const size_t bsm = (BUCKET_THREADS / 32 + 1) * static_cast<size_t>(E) * sizeof(int);   // per-warp histograms
  if (bsm > 48 * 1024 && (st = set_smem(reinterpret_cast<const void*>(k_bucket), bsm))) return st;
  k_bucket<<<1, BUCKET_THREADS, bsm, static_cast<cudaStream_t>(stream)>>>(idx, T * k, E, offsets, pairs, active,
                                                                         n_active);
  return launch_check("k_bucket");
}

size_t moe_expert_workspace_size(int T, int H, int I, int k) {
  if (T < 0 || H <= 0 || I <= 0 || k <= 0) return 0;
  return expert_ws_bytes(T, H, I, k);
}

int moe_expert_forward(const uint16_t* x, int T, int H, int I, int E, int k, const void* const* blob_ptrs,
                       const int32_t* offsets, const int32_t* pairs, const int32_t* active,
                       const int32_t* n_active, float* y_pairs, void* ws, size_t ws_bytes, int flags, void* stream) {
  int st = check_dims(T, H, I, E, k);
  if (st) return st;
  if ((st = check_flags(flags))) return st;
  if (T == 0) return MOE_OK;
  if (!x || !blob_ptrs || !offsets || !pairs || !active || !n_active || !y_pairs || !ws)
    return fail(MOE_ERR_INVALID_ARG, "moe_expert_forward: NULL pointer");
  if (ws_bytes < moe_expert_workspace_size(T, H, I, k))
    return fail(MOE_ERR_INVALID_ARG, "moe_expert_forward: workspace too small");
  if (!aligned16(x) || !aligned16(ws) || !aligned16(y_pairs))
    return fail(MOE_ERR_INVALID_ARG, "moe_expert_forward: misaligned pointer");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  ExpertWs w = carve_expert(ws, T, H, I, k);
  if (!use_gemm(T, H, I, 64, E, k, flags)) {
    if (flags & MOE_FLAG_TC) return fail(MOE_ERR_UNSUPPORTED, "moe_expert_forward: shapes outside the grouped GEMM");
    return run_routed_gemv(x, T, H, I, E, k, blob_ptrs, offsets, pairs, active, n_active, y_pairs, w.act, s);
  }
  RoutedIn rt{blob_ptrs, offsets, pairs, active, n_active, y_pairs, I, E, k};
  return run_gemm(x, T, H, &rt, nullptr, w.plan, w.maps, w.act, w.xs, nullptr, nullptr, s);
}

size_t moe_shared_workspace_size(int T, int H, int Is) {
  if (T < 0 || H <= 0 || Is <= 0) return 0;
  return shared_ws_bytes(T, H, Is);
}

int moe_shared_forward(const uint16_t* x, int T, int H, int Is, const moe_qmat* sh, float* ysh, void* ws,
                       size_t ws_bytes, int flags, void* stream) {
  int st = check_dims(T, H, Is, 8, 1);
  if (st) return st;
  if ((st = check_flags(flags))) return st;
  if (T == 0) return MOE_OK;
  if (!x || !sh || !ysh || !ws) return fail(MOE_ERR_INVALID_ARG, "moe_shared_forward: NULL pointer");
  if ((st = check_shared_mats(sh, H, Is))) return st;
  if (ws_bytes < moe_shared_workspace_size(T, H, Is))
    return fail(MOE_ERR_INVALID_ARG, "moe_shared_forward: workspace too small");
  if (!aligned16(x) || !aligned16(ws) || !aligned16(ysh))
    return fail(MOE_ERR_INVALID_ARG, "moe_shared_forward: misaligned pointer");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  SharedWs w = carve_shared(ws, T, H, Is);
  if (!use_gemm(T, H, 64, Is, 8, 1, flags)) {
    if (flags & MOE_FLAG_TC) return fail(MOE_ERR_UNSUPPORTED, "moe_shared_forward: shapes outside the grouped GEMM");
    return run_shared_gemv(x, T, H, Is, sh, ysh, w.act, s);
  }
  SharedIn si{sh, ysh, Is};
  return run_gemm(x, T, H, nullptr, &si, w.plan, nullptr, nullptr, nullptr, w.act, w.xh, s);
}

// The combine with the residual add read from resid_in and written to
// resid_out (the same array for the in-place form).
static int launch_combine(const float* y_pairs, const float* gates, const float* ysh, int T, int H, int k, uint16_t* y,
                          const float* resid_in, float* resid_out, cudaStream_t cs) {
  const bool vec = H % 4 == 0 && aligned16(y_pairs) && (!ysh || aligned16(ysh)) &&
                   (!resid_out || (aligned16(resid_out) && aligned16(resid_in))) && (reinterpret_cast<uintptr_t>(y) & 7) == 0;
  if (vec) {
    k_combine4<<<dim3((H / 4 + 255) / 256, T), 256, 0, cs>>>(y_pairs, gates, ysh, H, k, y, resid_in, resid_out);
    return launch_check("k_combine4");
  }
  k_combine<<<dim3((H + 255) / 256, T), 256, 0, cs>>>(y_pairs, gates, ysh, H, k, y, resid_in, resid_out);
  return launch_check("k_combine");
}

int moe_combine(const float* y_pairs, const float* gates, const float* ysh, int T, int H, int k, uint16_t* y,
                float* residual_inout, void* stream) {
  if (T < 0 || H <= 0 || k < 1 || k > 8) return fail(MOE_ERR_INVALID_ARG, "moe_combine: bad T/H/k");
  if (T == 0) return MOE_OK;
  if (!y_pairs || !gates) return fail(MOE_ERR_INVALID_ARG, "moe_combine: NULL pointer");
  return launch_combine(y_pairs, gates, ysh, T, H, k, y, residual_inout, residual_inout,
                        static_cast<cudaStream_t>(stream));
}

// Workspace of one layer: routing buffers, y_pairs, ysh, then the expert and
// shared-expert regions (the grouped GEMM's plan is the expert region's).
struct LayerWs {
  uint16_t* x; int32_t* idx; float* gates; int32_t* offsets; int32_t* pairs; int32_t* active; int32_t* n_active;
  float* y_pairs; float* ysh; void* ew; size_t ews; void* sw; size_t sws;
};
static size_t layer_ws_bytes(int T, int H, int I, int Is, int E, int k) {
  size_t n = 0;
  n += align_up(static_cast<size_t>(T) * H * 2);        // x
  n += align_up(static_cast<size_t>(T) * k * 4) * 2;    // idx, gates
  n += align_up(static_cast<size_t>(E + 1) * 4);        // offsets
  n += align_up(static_cast<size_t>(T) * k * 4);        // pairs
  n += align_up(static_cast<size_t>(E) * 4);            // active
  n += align_up(4);                                     // n_active
  n += align_up(static_cast<size_t>(T) * k * H * 4);    // y_pairs
  n += align_up(static_cast<size_t>(T) * H * 4);        // ysh
  n += expert_ws_bytes(T, H, I, k);
  n += shared_ws_bytes(T, H, Is);
  return n;
}
static LayerWs carve_layer(void* ws, int T, int H, int I, int Is, int E, int k) {
  char* p = static_cast<char*>(ws);
  auto take = [&](size_t n) { char* q = p; p += align_up(n); return q; };
  LayerWs w;
  w.x = reinterpret_cast<uint16_t*>(take(static_cast<size_t>(T) * H * 2));
  w.idx = reinterpret_cast<int32_t*>(take(static_cast<size_t>(T) * k * 4));
  w.gates = reinterpret_cast<float*>(take(static_cast<size_t>(T) * k * 4));
  w.offsets = reinterpret_cast<int32_t*>(take(static_cast<size_t>(E + 1) * 4));
  w.pairs = reinterpret_cast<int32_t*>(take(static_cast<size_t>(T) * k * 4));
  w.active = reinterpret_cast<int32_t*>(take(static_cast<size_t>(E) * 4));
  w.n_active = reinterpret_cast<int32_t*>(take(4));
  w.y_pairs = reinterpret_cast<float*>(take(static_cast<size_t>(T) * k * H * 4));
  w.ysh = reinterpret_cast<float*>(take(static_cast<size_t>(T) * H * 4));
  w.ews = expert_ws_bytes(T, H, I, k);
  w.ew = p; p += w.ews;
  w.sws = shared_ws_bytes(T, H, Is);
  w.sw = p;
  return w;
}

size_t moe_layer_workspace_size(int T, int H, int I, int Is, int E, int k) {
  if (T < 0 || H <= 0 || I <= 0 || Is <= 0 || E <= 0 || k <= 0) return 0;
  return layer_ws_bytes(T, H, I, Is, E, k);
}

int moe_layer_forward(const float* h_in, float* h_out, const uint16_t* x_in, int T, int H, int I, int Is, int E,
                      int k, const moe_qmat* router, const float* bias, int bias_per_row,
                      const void* const* blob_ptrs, const moe_qmat* shared, uint16_t* x_out, uint16_t* y,
                      int32_t* idx_out, float* gates_out, void* ws, size_t ws_bytes, int flags, void* stream) {
  int st = check_dims(T, H, I, E, k);
  if (st) return st;
  if ((st = check_dims(T, H, Is, E, k))) return st;
  if ((st = check_flags(flags))) return st;
  if (T == 0) return MOE_OK;
  if (!x_in && !h_in) return fail(MOE_ERR_INVALID_ARG, "moe_layer_forward: need h_in or x_in");
  if (h_out && !h_in) return fail(MOE_ERR_INVALID_ARG, "moe_layer_forward: h_out needs h_in");
  if (!blob_ptrs || !shared || !router) return fail(MOE_ERR_INVALID_ARG, "moe_layer_forward: NULL pointer");
  if (!ws || !aligned16(ws) || ws_bytes < moe_layer_workspace_size(T, H, I, Is, E, k))
    return fail(MOE_ERR_INVALID_ARG, "moe_layer_forward: workspace too small or misaligned");
  if ((st = check_shared_mats(shared, H, Is))) return st;
  LayerWs w = carve_layer(ws, T, H, I, Is, E, k);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  const uint16_t* xin = x_in;
  if (!xin) {
    if ((st = moe_rmsnorm(h_in, T, H, 1e-6f, w.x, stream))) return st;
    xin = w.x;
  }
  if (x_out && (st = cuda_check(cudaMemcpyAsync(x_out, xin, static_cast<size_t>(T) * H * 2,
                                                cudaMemcpyDeviceToDevice, s), "copy x_out")))
    return st;
  if ((st = moe_router_topk(xin, T, H, router, bias, bias_per_row, E, k, w.idx, w.gates, nullptr, stream))) return st;
  if ((st = moe_bucket(w.idx, T, k, E, w.offsets, w.pairs, w.active, w.n_active, stream))) return st;
  const bool gemm = use_gemm(T, H, I, Is, E, k, flags);
  if (!gemm && (flags & MOE_FLAG_TC)) return fail(MOE_ERR_UNSUPPORTED, "moe_layer_forward: shapes outside the grouped GEMM");
  if (gemm) {
    // routed buckets and the shared expert in one persistent launch per projection
    if (!aligned16(xin)) return fail(MOE_ERR_INVALID_ARG, "moe_layer_forward: misaligned x_in");
    ExpertWs ew = carve_expert(w.ew, T, H, I, k);
    SharedWs sw = carve_shared(w.sw, T, H, Is);
    RoutedIn rt{blob_ptrs, w.offsets, w.pairs, w.active, w.n_active, w.y_pairs, I, E, k};
    SharedIn si{shared, w.ysh, Is};
    if ((st = run_gemm(xin, T, H, &rt, &si, ew.plan, ew.maps, ew.act, ew.xs, sw.act, sw.xh, s))) return st;
  } else {
    if ((st = moe_shared_forward(xin, T, H, Is, shared, w.ysh, w.sw, w.sws, flags, stream))) return st;
    if ((st = moe_expert_forward(xin, T, H, I, E, k, blob_ptrs, w.offsets, w.pairs, w.active, w.n_active, w.y_pairs,
                                 w.ew, w.ews, flags, stream)))
      return st;
  }
  // h_out = h_in + the layer's output (the combine reads one and writes the other)
  if ((st = launch_combine(w.y_pairs, w.gates, w.ysh, T, H, k, y, h_out ? h_in : nullptr, h_out, s))) return st;
  if (idx_out && (st = cuda_check(cudaMemcpyAsync(idx_out, w.idx, static_cast<size_t>(T) * k * 4,
                                                  cudaMemcpyDeviceToDevice, s), "copy idx")))
    return st;
  if (gates_out && (st = cuda_check(cudaMemcpyAsync(gates_out, w.gates, static_cast<size_t>(T) * k * 4,
                                                    cudaMemcpyDeviceToDevice, s), "copy gates")))
    return st;
  return MOE_OK;
}

// Shapes the fused batch-1 kernel serves.
static bool fused_ok(int T, int H, int I, int Is, int E, int k, int bias_per_row, int G, int flags) {
  if ((flags & MOE_FLAG_LAYERED) || T != 1 || bias_per_row) return false;
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
  for (int l = 0; l < L; ++l) {
    const moe_qmat& R = routers[l];
    if (!R.q || !R.s || !R.b || R.bits != 8 || R.out != E || R.in != H || !aligned16(R.q) || !aligned16(R.s) ||
        !aligned16(R.b))
      return fail(MOE_ERR_INVALID_ARG, "moe_decode_forward: router %d must be 8-bit [E, H] with 16-byte aligned arrays", l);
    int st = check_shared_mats(shared + 3 * l, H, Is);
    if (st) return st;
  }
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
    static thread_local DfArgs args;   // large parameter block; the launch copies it
    memset(&args, 0, sizeof(args));
    args.h = h; args.H = H; args.I = I; args.Is = Is; args.E = E; args.k = k; args.L = nl;
    blob_offsets(H, I, args.off);
    args.act = act; args.logits = logits; args.counter = ctr;
    const size_t TH = static_cast<size_t>(H), Tk = static_cast<size_t>(k);
    args.x_trace = x_trace ? x_trace + l0 * TH : nullptr;
    args.y_trace = y_trace ? y_trace + l0 * TH : nullptr;
    args.idx_trace = idx_trace ? idx_trace + l0 * Tk : nullptr;
    args.gates_trace = gates_trace ? gates_trace + l0 * Tk : nullptr;
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

int moe_decode_launches(int T, int L, int flags) {
  if (T <= 0 || L <= 0) return 0;
  // persistent batch-1 path: one kernel per DF_MAX_LAYERS layers.  Otherwise
  // per layer: rmsnorm, router, bucket, then either the grouped GEMM (prep,
  // gate/up, down) or the GEMV kernels (shared gate/up and down, routed
  // gate/up and down), and the combine.
  if (T == 1 && !(flags & MOE_FLAG_LAYERED)) return (L + DF_MAX_LAYERS - 1) / DF_MAX_LAYERS;
  const bool gemm = !(flags & MOE_FLAG_GEMV) && (T > 2 || (flags & MOE_FLAG_TC));
  return (gemm ? 7 : 8) * L;
}

size_t moe_decode_workspace_size(int T, int H, int I, int Is, int E, int k) {
  if (T < 0 || H <= 0 || I <= 0 || Is <= 0 || E <= 0 || k <= 0) return 0;
  const size_t layered = moe_layer_workspace_size(T, H, I, Is, E, k);
  const size_t fused = fused_ws(I, Is, E, k);
  return layered > fused ? layered : fused;
}

int moe_decode_forward(float* h, int T, int H, int I, int Is, int E, int k, int L, const moe_qmat* routers,
                       const float* const* biases, int bias_per_row, const void* const* const* blob_tables,
                       const moe_qmat* shared, uint16_t* x_trace, uint16_t* y_trace, int32_t* idx_trace,
                       float* gates_trace, void* ws, size_t ws_bytes, int flags, void* stream) {
  int st = check_dims(T, H, I, E, k);
  if (st) return st;
  if ((st = check_flags(flags))) return st;
  if (L < 0) return fail(MOE_ERR_INVALID_ARG, "moe_decode_forward: L < 0");
  if (T == 0 || L == 0) return MOE_OK;
  if (!h || !routers || !blob_tables || !shared) return fail(MOE_ERR_INVALID_ARG, "moe_decode_forward: NULL pointer");
  if (ws_bytes < moe_decode_workspace_size(T, H, I, Is, E, k))
    return fail(MOE_ERR_INVALID_ARG, "moe_decode_forward: workspace too small");
  const int G = (T == 1 && !(flags & MOE_FLAG_LAYERED)) ? fused_grid() : 0;
  if (fused_ok(T, H, I, Is, E, k, bias_per_row, G, flags))
    return launch_fused(h, H, I, Is, E, k, L, routers, biases, blob_tables, shared, x_trace, y_trace, idx_trace,
                        gates_trace, ws, G, static_cast<cudaStream_t>(stream));
  const size_t TH = static_cast<size_t>(T) * H, Tk = static_cast<size_t>(T) * k;
  for (int l = 0; l < L; ++l) {
    const float* b = biases ? biases[l] : nullptr;
    st = moe_layer_forward(h, h, nullptr, T, H, I, Is, E, k, &routers[l], b, bias_per_row, blob_tables[l],
                           &shared[3 * l], x_trace ? x_trace + l * TH : nullptr, y_trace ? y_trace + l * TH : nullptr,
                           idx_trace ? idx_trace + l * Tk : nullptr, gates_trace ? gates_trace + l * Tk : nullptr, ws,
                           ws_bytes, flags, stream);
    if (st) return st;
  }
  return MOE_OK;
}

// ------------------------------------------------------------ decode session
struct moe_decode_session {
  int H = 0;
  cudaStream_t stream = nullptr;
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  float* pin_in = nullptr;
  float* pin_out = nullptr;
};

int moe_decode_session_destroy(moe_decode_session* s) {
  if (!s) return MOE_OK;
  if (s->stream) cudaStreamSynchronize(s->stream);
  if (s->exec) cudaGraphExecDestroy(s->exec);
  if (s->graph) cudaGraphDestroy(s->graph);
  if (s->pin_in) cudaFreeHost(s->pin_in);
  if (s->pin_out) cudaFreeHost(s->pin_out);
  if (s->stream) cudaStreamDestroy(s->stream);
  delete s;
  return MOE_OK;
}

int moe_decode_session_create(float* h_dev, int H, int I, int Is, int E, int k, int L, const moe_qmat* routers,
                              const float* const* biases, int bias_per_row, const void* const* const* blob_tables,
                              const moe_qmat* shared, void* ws, size_t ws_bytes, int flags, moe_decode_session** out) {
  if (!out) return fail(MOE_ERR_INVALID_ARG, "moe_decode_session_create: NULL out");
  *out = nullptr;
  int st = check_dims(1, H, I, E, k);
  if (st) return st;
  if ((st = check_dims(1, H, Is, E, k))) return st;
  if ((st = check_flags(flags))) return st;
  if (L <= 0) return fail(MOE_ERR_INVALID_ARG, "moe_decode_session_create: L must be > 0");
  if (!h_dev || !routers || !blob_tables || !shared || !ws)
    return fail(MOE_ERR_INVALID_ARG, "moe_decode_session_create: NULL pointer");
  if (!aligned16(h_dev)) return fail(MOE_ERR_INVALID_ARG, "moe_decode_session_create: h_dev must be 16-byte aligned");
  if (ws_bytes < moe_decode_workspace_size(1, H, I, Is, E, k))
    return fail(MOE_ERR_INVALID_ARG, "moe_decode_session_create: workspace too small");
  for (int l = 0; l < L; ++l) {
    const moe_qmat& R = routers[l];
    if (!R.q || !R.s || !R.b || R.bits != 8 || R.out != E || R.in != H)
      return fail(MOE_ERR_INVALID_ARG, "moe_decode_session_create: router %d must be 8-bit [E, H]", l);
    if ((st = check_shared_mats(shared + 3 * l, H, Is))) return st;
  }
  moe_decode_session* s = new moe_decode_session();
  s->H = H;
  const size_t nb = static_cast<size_t>(H) * sizeof(float);
  if ((st = cuda_check(cudaStreamCreateWithFlags(&s->stream, cudaStreamNonBlocking), "session stream")) ||
      (st = cuda_check(cudaHostAlloc(reinterpret_cast<void**>(&s->pin_in), nb, cudaHostAllocDefault), "session pinned")) ||
      (st = cuda_check(cudaHostAlloc(reinterpret_cast<void**>(&s->pin_out), nb, cudaHostAllocDefault), "session pinned"))) {
    moe_decode_session_destroy(s);
    return st;
  }
  // the kernels load their code and attributes before the capture (on a
  // zero row: whatever h_dev held, the warm-up then routes validly)
  if ((st = cuda_check(cudaMemsetAsync(h_dev, 0, nb, s->stream), "session zero row")) ||
      (st = moe_decode_forward(h_dev, 1, H, I, Is, E, k, L, routers, biases, bias_per_row, blob_tables, shared,
                               nullptr, nullptr, nullptr, nullptr, ws, ws_bytes, flags, s->stream)) ||
      (st = cuda_check(cudaStreamSynchronize(s->stream), "session warm-up"))) {
    moe_decode_session_destroy(s);
    return st;
  }
  if ((st = cuda_check(cudaStreamBeginCapture(s->stream, cudaStreamCaptureModeThreadLocal), "session capture"))) {
    moe_decode_session_destroy(s);
    return st;
  }
  int cst = cuda_check(cudaMemcpyAsync(h_dev, s->pin_in, nb, cudaMemcpyHostToDevice, s->stream), "session copy in");
  if (!cst)
    cst = moe_decode_forward(h_dev, 1, H, I, Is, E, k, L, routers, biases, bias_per_row, blob_tables, shared,
                             nullptr, nullptr, nullptr, nullptr, ws, ws_bytes, flags, s->stream);
  if (!cst) cst = cuda_check(cudaMemcpyAsync(s->pin_out, h_dev, nb, cudaMemcpyDeviceToHost, s->stream), "session copy out");
  st = cuda_check(cudaStreamEndCapture(s->stream, &s->graph), "session end capture");
  if (cst || st) {
    moe_decode_session_destroy(s);
    return cst ? cst : st;
  }
  if ((st = cuda_check(cudaGraphInstantiate(&s->exec, s->graph, 0), "session instantiate"))) {
    moe_decode_session_destroy(s);
    return st;
  }
  *out = s;
  return MOE_OK;
}

int moe_decode_session_step(moe_decode_session* s, const float* h_in, float* h_out) {
  if (!s || !s->exec || !h_in || !h_out) return fail(MOE_ERR_INVALID_ARG, "moe_decode_session_step: NULL pointer");
  const size_t nb = static_cast<size_t>(s->H) * sizeof(float);
  memcpy(s->pin_in, h_in, nb);
  int st = cuda_check(cudaGraphLaunch(s->exec, s->stream), "session step launch");
  if (st) return st;
  if ((st = cuda_check(cudaStreamSynchronize(s->stream), "session step"))) return st;
  memcpy(h_out, s->pin_out, nb);
  return MOE_OK;
}

void* moe_decode_session_stream(moe_decode_session* s) { return s ? static_cast<void*>(s->stream) : nullptr; }

}  // extern "C"
