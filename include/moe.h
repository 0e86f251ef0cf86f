/*
 * libmoe — routed Mixture-of-Experts layer with MLX-style affine 4-bit experts
 * and an 8-bit router, for NVIDIA B200 (sm_100a).
 *
 * The layer (one step of a routed-MoE transformer block):
 *   A0  x = bf16( h / sqrt(mean(h^2) + eps) )            layer-input RMS norm
 *   A1  logits = W_r x + beta                             8-bit affine router
 *   A2  idx = top-k(logits), gates = softmax(logits[idx])
 *   A3  pairs (t, j) grouped by expert
 *   A4  act = gelu_tanh(W_g x) * (W_u x)                  per (token, expert) pair
 *   A5  y_pair = W_d act
 *   A6  ysh = W_sd (gelu_tanh(W_sg x) * (W_su x))         always-on shared expert
 *   A7  y = sum_j gates_j * y_pair_j + ysh                (then h += y between layers)
 *
 * Passages defining the operations:
 *   "TurboFieldfare: Gemma 4 26B on an 8 GB MacBook, in ~2 GB of RAM"
 *   (blog-mushroom.pages.dev), section "Why 26B Fits in 2 GB": 8 of 128 experts
 *   per token and layer; the shared-expert branch runs while expert blobs are
 *   fetched and the two outputs are merged; a 16-slot LFU per layer; prefill in
 *   chunks of up to 128 rows so that one expert blob serves the chunk.
 *   "TurboFieldfareとは｜26BのGemma 4を約2GBのRAMで動かすSwift製ランタイムの実像"
 *   (ai-heartland.com), section "TurboFieldfareとは": MLX affine 4-bit, group 64,
 *   bf16 scale and bias; 8-bit router; 4-bit shared and routed experts.
 *   The softmax over the top-k logits, the gelu_tanh GeGLU, the ungated
 *   shared expert and the eps = 1e-6 norm without weight are this library's
 *   definition of the layer; the pages do not state them.
 *
 * Conventions (every call):
 *   - Return an int status (moe_status).  No call aborts or exits.
 *     moe_last_error_string() gives detail for the calling thread.
 *   - Pointers documented "device" are CUDA device pointers owned by the
 *     caller; the library never allocates device memory in these calls.
 *     Scratch comes from caller workspaces sized by the *_workspace_size calls.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     asynchronous on it; errors of a kernel surface at a later call or at
 *     moe_sync().
 *   - bf16 / fp16 values are passed as uint16_t bit patterns.
 *   - Dimensions: H, I, Is multiples of 64; E a multiple of 8, E <= 1024;
 *     1 <= k <= 8 and k <= E.  Device pointers 16-byte aligned.
 *
 * Quantised matrix [out, in] (moe_qmat): w[r,c] = S[r,c/64] * q[r,c] + B[r,c/64]
 *   q  uint32 [out, in*bits/32], element c at bit bits*(c % (32/bits)) of word
 *      c / (32/bits) (low bits first)
 *   s  bf16   [out, in/64]    b  bf16 [out, in/64]
 *   bits = 4 for experts, 8 for the router.
 *
 * Expert blob (routed expert, bytes, contiguous, 16-byte aligned):
 *   gate.q gate.s gate.b | up.q up.s up.b | down.q down.s down.b
 *   with gate, up = [I, H] and down = [H, I], 4-bit; blob_bytes = 3*(I*H/2 + 4*I*H/64).
 *   A routed layer is given as a device array of E blob pointers, so blobs may
 *   live anywhere (one allocation with a fixed stride, or cache slots).
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* bad size, NULL pointer or misalignment; nothing launched */
  MOE_ERR_CUDA = 2,          /* a CUDA runtime call or launch failed */
  MOE_ERR_TIMEOUT = 3,       /* a bounded host wait ran out */
  MOE_ERR_DEVICE_CHECK = 4,  /* a kernel found an out-of-range index and skipped it */
  MOE_ERR_UNSUPPORTED = 5    /* valid request this build does not serve */
} moe_status;

typedef struct moe_qmat {
  const uint32_t* q;   /* device */
  const uint16_t* s;   /* device, bf16 */
  const uint16_t* b;   /* device, bf16 */
  int32_t out;
  int32_t in;
  int32_t bits;        /* 4 or 8 */
} moe_qmat;

/* Detail of the last non-OK status on this thread (static storage). */
MOE_API const char* moe_last_error_string(void);
/* Library version (major*10000 + minor*100 + patch). */
MOE_API int moe_version(void);
/* Synchronise `stream`, then report CUDA errors and the device check word
 * (MOE_ERR_DEVICE_CHECK if a kernel skipped an out-of-range index since the
 * last moe_sync; the word is cleared). */
MOE_API int moe_sync(void* stream);

/* Bytes of one expert blob and its offsets: offsets[9] receives the byte
 * offsets of gate.q gate.s gate.b up.q up.s up.b down.q down.s down.b. */
MOE_API size_t moe_blob_bytes(int H, int I, size_t* offsets9);

/* A0 — layer-input RMS norm.
 * Source: "drumih/turbo-fieldfare" (paperfeed.app), section "How it works":
 * each decode step walks the 30 transformer layers, so every layer's MoE input
 * is the running hidden state.  The pages do not give the norm; this library
 * defines it as an RMS norm with eps and no learned weight, the output rounded
 * to bf16 (the layer input of every routed-MoE call below).
 *   h  fp32 [T,H] (device, read)     x  bf16 [T,H] (device, written)
 * x = bf16_rn(h / sqrt(mean(h^2) + eps)), sum of squares in fp32, fixed order.
 * Errors: MOE_ERR_INVALID_ARG (T < 0, H not a positive multiple of 64, NULL or
 * misaligned pointer) before any launch; T = 0 is a no-op. */
MOE_API int moe_rmsnorm(const float* h, int T, int H, float eps, uint16_t* x, void* stream);

/* A1 + A2 — router and top-k.
 * Sources: "TurboFieldfare: Gemma 4 26B on an 8 GB MacBook, in ~2 GB of RAM"
 * (blog-mushroom.pages.dev), section "Why 26B Fits in 2 GB": the router picks
 * 8 of 128 experts per token in each layer; "TurboFieldfareとは｜26BのGemma 4
 * を約2GBのRAMで動かすSwift製ランタイムの実像" (ai-heartland.com), section
 * "TurboFieldfareとは：エキスパートをSSDに置いたままMoEを走らせる": the router
 * projection alone is 8-bit MLX affine (group 64, bf16 scale and bias).  The
 * softmax over the k selected logits is this library's definition.
 *   x       bf16 [T,H] (device)
 *   router  8-bit q-matrix [E,H] (host struct of device pointers)
 *   bias    fp32 [E] (bias_per_row = 0) or [T,E] (bias_per_row = 1) or NULL (device)
 *   idx     int32 [T,k] (device): the k largest logits, descending; an exact
 *           tie goes to the lower expert id
 *   gates   fp32 [T,k] (device): softmax over the k selected logits
 *   logits_opt fp32 [T,E] (device) or NULL: logits including the bias
 * Logits are accumulated in fp32.  Runs as clusters of 8 CTAs per block of
 * rows; the top-k reads the logits through distributed shared memory.
 * Errors: MOE_ERR_INVALID_ARG (dims, NULL pointer, router not 8-bit [E,H],
 * misaligned x or router codes), MOE_ERR_UNSUPPORTED (H, E too large for the
 * kernel's shared memory); nothing is launched on an error. */
MOE_API int moe_router_topk(const uint16_t* x, int T, int H, const moe_qmat* router,
                    const float* bias, int bias_per_row, int E, int k,
                    int32_t* idx, float* gates, float* logits_opt, void* stream);

/* A3 — bucketing (stable counting sort of the T*k pairs by expert).
 * Source: "TurboFieldfare: Gemma 4 26B on an 8 GB MacBook, in ~2 GB of RAM"
 * (blog-mushroom.pages.dev), section "Why 26B Fits in 2 GB": prefill chunks of
 * up to 128 tokens let one expert blob serve every row of the chunk routed to
 * it; the buckets are those row groups.
 *   idx      int32 [T,k] (device)
 *   offsets  int32 [E+1] (device): bucket e is pairs[offsets[e] .. offsets[e+1])
 *   pairs    int32 [T*k] (device): value t*k + j, t then j ascending inside a bucket
 *   active   int32 [E]   (device): experts with a non-empty bucket, ascending
 *   n_active int32 [1]   (device)
 * Requires T*k <= 65536 (else MOE_ERR_UNSUPPORTED).  Out-of-range ids are
 * skipped and flagged (MOE_ERR_DEVICE_CHECK at the next moe_sync). */
MOE_API int moe_bucket(const int32_t* idx, int T, int k, int E, int32_t* offsets,
               int32_t* pairs, int32_t* active, int32_t* n_active, void* stream);

/* Per-call path flags (bit set; 0 lets the library choose).  A flag changes
 * which kernels run, never the definition of the result; paths agree within
 * the output tolerance, not bit for bit. */
enum {
  MOE_FLAG_GEMV = 1,      /* every expert bucket and the shared expert on the CUDA-core GEMV kernels */
  MOE_FLAG_TC = 2,        /* every bucket (one row included) on the tensor-core grouped GEMM */
  MOE_FLAG_LAYERED = 4    /* moe_decode_forward at T = 1: the per-layer calls, not the persistent kernel */
};

/* A4 + A5 — routed experts for every pair.
 * Sources: "TurboFieldfareとは｜26BのGemma 4を約2GBのRAMで動かすSwift製ランタイム
 * の実像" (ai-heartland.com), section "TurboFieldfareとは：エキスパートをSSDに
 * 置いたままMoEを走らせる": routed experts are MLX affine 4-bit, group 64, bf16
 * scale and bias; "TurboFieldfare: Gemma 4 26B on an 8 GB MacBook, in ~2 GB
 * of RAM" (blog-mushroom.pages.dev), section "Why 26B Fits in 2 GB": each
 * expert is one ~3.3 MB blob.  The expert itself (gelu_tanh(W_g x) * W_u x,
 * then W_d) is this library's definition.
 *   x          bf16 [T,H] (device)
 *   blob_ptrs  device array [E] of device pointers to expert blobs
 *   offsets, pairs, active, n_active   from moe_bucket (device)
 *   y_pairs    fp32 [T*k, H] (device): row t*k + j = expert idx[t,j] applied to x[t]
 *   ws         device workspace of at least moe_expert_workspace_size(T,H,I,k) bytes
 *   flags      MOE_FLAG_* (0: the library's choice)
 * Path: with flags 0, T <= 2 runs the decode GEMV kernels (CUDA cores) and
 * larger T the tcgen05 grouped GEMM; MOE_FLAG_GEMV / MOE_FLAG_TC force one.
 * The choice depends on T and flags only, never on the data.  The
 * activation between the projections is fp16.
 * Errors: MOE_ERR_INVALID_ARG (dims, NULL or misaligned pointer, workspace too
 * small) before any launch; T = 0 is a no-op. */
MOE_API size_t moe_expert_workspace_size(int T, int H, int I, int k);
MOE_API int moe_expert_forward(const uint16_t* x, int T, int H, int I, int E, int k,
                       const void* const* blob_ptrs, const int32_t* offsets,
                       const int32_t* pairs, const int32_t* active,
                       const int32_t* n_active, float* y_pairs,
                       void* ws, size_t ws_bytes, int flags, void* stream);
/* moe_expert_forward without a workspace argument, for callers that cannot
 * allocate device memory where they run the experts (inside a CUDA graph
 * being captured, under a memory pool that must not be re-entered, or in an
 * embedder whose device memory is reserved up front).  The pages describe no
 * counterpart of this call; it is a convenience of this library.
 *   Arguments and results are those of moe_expert_forward with flags 0.
 *   Scratch: a static device array of MOE_NOALLOC_SCRATCH_BYTES (4 MiB) in
 *   the library image, one per GPU that loads the library, kept until exit.
 *   It must hold moe_expert_workspace_size(T,H,I,k) bytes (at H = 2816,
 *   I = 704, k = 8 that is T <= 70); larger requests return
 *   MOE_ERR_INVALID_ARG and launch nothing.
 *   Argument checks (sizes, NULL and misaligned pointers) come before any
 *   CUDA call.  Every call then looks up the array's device address on the
 *   current device (cudaGetSymbolAddress), so the address stays right after a
 *   device reset; the first call on a device may load the library's device
 *   code, so make it before any stream capture.
 *   Every call on a device shares the one array and leaves its contents
 *   behind; two calls whose kernels overlap on the GPU (different streams,
 *   no ordering between them) race on it.  Nothing in it needs to start at
 *   zero.  The call allocates no device memory. */
#define MOE_NOALLOC_SCRATCH_BYTES (4 * 1024 * 1024)
MOE_API int moe_expert_forward_noalloc(const uint16_t* x, int T, int H, int I, int E, int k,
                                       const void* const* blob_ptrs, const int32_t* offsets,
                                       const int32_t* pairs, const int32_t* active,
                                       const int32_t* n_active, float* y_pairs, void* stream);

/* A6 — shared expert on every row.
 * Sources: "TurboFieldfare: Gemma 4 26B on an 8 GB MacBook, in ~2 GB of RAM"
 * (blog-mushroom.pages.dev), section "Why 26B Fits in 2 GB": the shared-expert
 * branch runs while the routed blobs are fetched; "TurboFieldfareとは｜26Bの
 * Gemma 4を約2GBのRAMで動かすSwift製ランタイムの実像" (ai-heartland.com),
 * section "TurboFieldfareとは：エキスパートをSSDに置いたままMoEを走らせる": the
 * shared expert is 4-bit like the routed ones.  Ungated (added as is) by this
 * library's definition.
 *   shared  host array of 3 q-matrices: gate [Is,H], up [Is,H], down [H,Is]
 *   ysh     fp32 [T,H] (device)
 *   ws      device workspace of at least moe_shared_workspace_size(T,H,Is) bytes
 *   flags   MOE_FLAG_* (path as in moe_expert_forward: one expert whose
 *           bucket holds every row)
 * Errors: MOE_ERR_INVALID_ARG (dims, a matrix not 4-bit of the stated shape,
 * NULL or misaligned pointer, workspace too small) before any launch. */
MOE_API size_t moe_shared_workspace_size(int T, int H, int Is);
MOE_API int moe_shared_forward(const uint16_t* x, int T, int H, int Is, const moe_qmat* shared,
                       float* ysh, void* ws, size_t ws_bytes, int flags, void* stream);

/* A7 — combine.
 * Source: "TurboFieldfare: Gemma 4 26B on an 8 GB MacBook, in ~2 GB of RAM"
 * (blog-mushroom.pages.dev), section "Why 26B Fits in 2 GB": the routed and
 * the shared-expert outputs are merged.  The merge is this library's
 * definition: the gate-weighted sum of the k routed outputs plus the shared one,
 *   y[t] = sum_{j=0..k-1} gates[t,j] * y_pairs[t*k+j] + ysh[t],
 * summed in fp32 in that order; y bf16 [T,H] (device, may be NULL);
 * residual_inout fp32 [T,H] (device) or NULL: residual += the fp32 sum.
 * Errors: MOE_ERR_INVALID_ARG (T < 0, k outside 1..8, NULL y_pairs or gates). */
MOE_API int moe_combine(const float* y_pairs, const float* gates, const float* ysh,
                int T, int H, int k, uint16_t* y, float* residual_inout, void* stream);

/* One whole layer, A0 (optional) to A7: the calls above in order on `stream`.
 * Source: "drumih/turbo-fieldfare" (paperfeed.app), section "How it works":
 * per layer the router runs from resident weights, the routed experts the
 * step needs are applied and the shared-expert compute overlaps their fetch.
 *   h_in     fp32 [T,H] (device) residual stream or NULL; when x_in is NULL the
 *            layer input is its RMS norm (A0, eps = 1e-6)
 *   h_out    fp32 [T,H] (device) or NULL: receives h_in + y (fp32, before the
 *            bf16 rounding of y); may equal h_in
 *   x_in     bf16 [T,H] (device) layer input used instead of the norm of h_in
 *            when non-NULL
 *   x_out    bf16 [T,H] (device) or NULL: the layer input actually used
 *   y        bf16 [T,H] (device) or NULL: the layer output
 *   idx, gates  int32/fp32 [T,k] (device) or NULL: the routing used
 *   blob_ptrs   device array [E] of blob pointers
 *   ws       device workspace of at least moe_layer_workspace_size(...) bytes
 *   flags    MOE_FLAG_* for the routed and the shared experts
 * On the tensor-core path the routed buckets and the shared expert share one
 * persistent launch per projection (gate/up, then down), so the shared
 * expert's weights stream while the routed experts compute.
 * Errors: as the calls it makes; h_out without h_in, or neither h_in nor
 * x_in, is MOE_ERR_INVALID_ARG. */
MOE_API size_t moe_layer_workspace_size(int T, int H, int I, int Is, int E, int k);
MOE_API int moe_layer_forward(const float* h_in, float* h_out, const uint16_t* x_in, int T, int H,
                      int I, int Is, int E, int k, const moe_qmat* router,
                      const float* bias, int bias_per_row, const void* const* blob_ptrs,
                      const moe_qmat* shared, uint16_t* x_out, uint16_t* y,
                      int32_t* idx, float* gates, void* ws, size_t ws_bytes, int flags, void* stream);

/* A whole decode/prefill step through L stacked layers (A0 .. A7 per layer,
 * residual add between layers).
 * Source: "drumih/turbo-fieldfare" (paperfeed.app), section "How it works":
 * each decode step walks the 30 transformer layers.  For l = 0 .. L-1:
 *   x_l = rmsnorm(h); h += layer_l(x_l)
 *   h          fp32 [T,H] (device), updated in place (the step input on entry,
 *              the residual stream after the last layer on return)
 *   routers    host array [L] of 8-bit router q-matrices [E,H]
 *   biases     host array [L] of device fp32 pointers ([E] or, with
 *              bias_per_row, [T,E]) or NULL entries / NULL array for none
 *   blob_tables host array [L] of device arrays [E] of expert-blob pointers
 *   shared     host array [L*3] of shared-expert q-matrices
 *   x_trace, y_trace   bf16 [L,T,H] (device) or NULL: every layer's input/output
 *   idx_trace, gates_trace  int32/fp32 [L,T,k] (device) or NULL
 *   ws         device workspace of at least moe_decode_workspace_size(...) bytes
 *   flags      MOE_FLAG_*
 * Batch-1 steps (T = 1, per-expert or no bias) run as one persistent kernel
 * per up to 48 layers (one CTA per SM, cooperative launch) unless
 * MOE_FLAG_LAYERED is set; other shapes run moe_layer_forward per layer.
 * Layers run in order on `stream`.
 * Errors: MOE_ERR_INVALID_ARG (dims, L < 0, NULL arrays, workspace too small)
 * before any launch. */
MOE_API size_t moe_decode_workspace_size(int T, int H, int I, int Is, int E, int k);
/* Phase timestamps of the persistent batch-1 kernel (a tracing aid that never
 * changes results).  Applies to moe_decode_forward calls made later by the
 * calling thread: when `stamps` (device, [L][G][16] uint64, G =
 * moe_decode_grid()) is non-NULL, thread 0 of every CTA writes %globaltimer
 * (ns) at the phase boundaries of each layer (the points are listed in the
 * kernel's source).  NULL turns it off (default). */
MOE_API int moe_set_decode_profile(unsigned long long* stamps);
/* CTAs of the persistent batch-1 kernel on the current device (0: not available). */
MOE_API int moe_decode_grid(void);
/* Number of kernels one moe_decode_forward(T, L, flags) call launches. */
MOE_API int moe_decode_launches(int T, int L, int flags);
MOE_API int moe_decode_forward(float* h, int T, int H, int I, int Is, int E, int k, int L,
                               const moe_qmat* routers, const float* const* biases,
                               int bias_per_row, const void* const* const* blob_tables,
                               const moe_qmat* shared, uint16_t* x_trace, uint16_t* y_trace,
                               int32_t* idx_trace, float* gates_trace, void* ws,
                               size_t ws_bytes, int flags, void* stream);

/* Decode session: one batch-1 step per call from host memory to host memory,
 * the way a server calls the layer stack token by token.
 * Source: "drumih/turbo-fieldfare" (paperfeed.app), section "How it works":
 * each decode step walks the 30 layers; the step is moe_decode_forward's
 * (T = 1), the session only holds its arguments and the row copies.  Created once with
 * the arguments of moe_decode_forward (T = 1; checked once, here); every
 * step copies the token's residual row in, runs the L layers, copies the row
 * out and waits for it.  The copies and the launches are one CUDA graph
 * (instantiated at creation on the session's own stream) between two
 * pinned staging rows of the session.
 *   h_dev     fp32 [1,H] (device): the row the layers update (owned by the caller)
 *   routers .. ws, flags   as moe_decode_forward (they must stay valid for
 *             the session's life; the graph holds their addresses)
 *   out       receives the session handle
 * moe_decode_session_step:
 *   h_in      fp32 [H] host (any host memory): the step's input row
 *   h_out     fp32 [H] host: the residual row after the L layers (may equal h_in)
 *   returns after the row is back; a device check (bounded waits, ids) is
 *   reported by the next moe_sync
 * moe_decode_session_stream: the session's CUDA stream (for events).
 * A session is used by one thread at a time (its staging rows are shared
 * by its steps); creation runs one warm-up step on a zeroed h_dev.
 * Errors: creation fails with the codes of moe_decode_forward, before any
 * launch; a step fails with MOE_ERR_CUDA. */
typedef struct moe_decode_session moe_decode_session;
MOE_API int moe_decode_session_create(float* h_dev, int H, int I, int Is, int E, int k, int L,
                                      const moe_qmat* routers, const float* const* biases,
                                      int bias_per_row, const void* const* const* blob_tables,
                                      const moe_qmat* shared, void* ws, size_t ws_bytes, int flags,
                                      moe_decode_session** out);
MOE_API int moe_decode_session_step(moe_decode_session* s, const float* h_in, float* h_out);
MOE_API void* moe_decode_session_stream(moe_decode_session* s);
MOE_API int moe_decode_session_destroy(moe_decode_session* s);

/* ------------------------------------------------------------------------
 * Per-layer LFU expert-slot cache (routed experts streamed from pinned host
 * memory).  "TurboFieldfare: Gemma 4 26B on an 8 GB MacBook, in ~2 GB of
 * RAM" (blog-mushroom.pages.dev), section "Why 26B Fits in 2 GB": per token
 * the host checks the 8 selected ids against a 16-slot LFU cache of the
 * layer; hits reuse the resident copy, misses fetch the blob; the shared
 * expert runs while the fetches complete.
 * Policy (the pages say only "16-slot LFU"): counts live while an expert is
 * resident (insert 1, hit +1); in a step hits are taken first, then misses,
 * each in the step's order; a global tick advances per access; a miss fills
 * the lowest empty slot, else evicts, among slots not used by the step, the
 * smallest (count, last tick, slot index).  Every access is logged as
 * (layer, step, expert, hit, slot), `step` counting that layer's steps.
 * A handle is not thread-safe: one handle per pair of streams.
 */
typedef struct moe_lfu moe_lfu;
enum { MOE_LFU_FAULT_NONE = 0, MOE_LFU_FAULT_COPY_FAILS = 1, MOE_LFU_FAULT_SLOW_COPY = 2 };
/* host_blobs: host array [L*E] of pinned host pointers (blob of expert e of
 * layer l at index l*E + e), slot_pool: device memory of L*n_slots*slot_stride
 * bytes (caller-owned; slot s of layer l at (l*n_slots + s)*slot_stride).
 * Both NULL: a planning-only handle (moe_lfu_plan, moe_lfu_get_log). */
MOE_API int moe_lfu_create(int n_layers, int n_experts, int n_slots, size_t blob_bytes,
                           const void* const* host_blobs, void* slot_pool, size_t slot_stride,
                           moe_lfu** out);
/* Plan one step without copying: slots_out[i], hit_out[i] for ids[i]
 * (distinct, at most n_slots of them).  Updates the cache state and log. */
MOE_API int moe_lfu_plan(moe_lfu* h, int layer, const int32_t* ids, int n, int32_t* slots_out,
                         int32_t* hit_out);
/* One step: plan; on `side_stream` wait for `wait_event` (recorded by the
 * caller after the kernels that read this layer's slots; may be NULL), copy
 * each missed blob into its slot (one cudaMemcpyAsync per miss), update the
 * layer's device pointer table dev_table [E] for the step's ids, and record
 * `done_event`; the caller's compute stream waits on done_event before the
 * expert kernels.  Host waits are bounded by timeout_ms (MOE_ERR_TIMEOUT).
 * A step is all or nothing for the cache state: when any part of it fails
 * (a copy that cannot be issued, a wait that runs out) the layer's state and
 * log are restored to what they were before the call and the error is
 * returned; slots that copies issued by the failed call overwrite are marked,
 * and the next step that hits the expert such a slot holds copies its blob
 * again (logged as the hit the policy makes it).  Repeating the failed call
 * therefore plans exactly as the first attempt would have. */
MOE_API int moe_lfu_step(moe_lfu* h, int layer, const int32_t* ids, int n, void* side_stream,
                         void* wait_event, void* done_event, void** dev_table, int timeout_ms);
/* Poll an event until it completes or timeout_ms passes (MOE_ERR_TIMEOUT). */
MOE_API int moe_lfu_wait(void* event, int timeout_ms);
/* The access log: n_records records of 5 int32 (layer, step, expert, hit,
 * slot); up to cap_records are copied into buf (may be NULL). */
MOE_API int moe_lfu_get_log(moe_lfu* h, int32_t* buf, size_t cap_records, size_t* n_records);
MOE_API int moe_lfu_stats(moe_lfu* h, int64_t* hits, int64_t* misses, int64_t* bytes_copied);
/* Test hook: after `after_n` copies, every further copy fails before it is
 * issued (kind 1) or is delayed by 50 ms on the host (kind 2); kind 0 clears it. */
MOE_API int moe_lfu_set_fault(moe_lfu* h, int kind, int after_n);
/* Lookahead prefetch (f2; off by default): after each moe_streamed_layer_forward
 * call on a layer, stage up to per_call (0 .. n_slots) experts of that layer
 * ahead of their next use -- the non-resident experts accessed most often so
 * far in the run (ties to the lower id), each into the slot a miss would
 * take, only while that slot is empty or its resident's count is below the
 * candidate's access total; a prefetched expert enters with count 0, is one
 * more step of the layer and is logged with hit = 2 (moe_lfu_stats counts
 * such records neither as hits nor as misses).  The copies follow the
 * call's expert kernels on the side stream and belong to the call's
 * transaction.  The pages report speculative expert reads as measured and
 * rejected: "TurboFieldfareとは｜…の実像" (ai-heartland.com), section
 * "103件の実験記録が教える「効いたのに採用しなかった最適化」".
 * moe_lfu_plan_prefetch plans one such prefetch without copying (state and
 * log updated; ids_out / slots_out of capacity per_call; *n_out = count). */
MOE_API int moe_lfu_set_prefetch(moe_lfu* h, int per_call);
MOE_API int moe_lfu_plan_prefetch(moe_lfu* h, int layer, int per_call, int32_t* ids_out, int32_t* slots_out,
                                  int* n_out);
MOE_API int moe_lfu_destroy(moe_lfu* h);

/* One routed-MoE layer whose routed experts are streamed through the LFU
 * slots of layer `layer` (A0 .. A7 with the residual update of hres):
 * rms norm, router + top-k and bucketing on main_stream; the routing goes to
 * the host (bounded wait); the shared expert is queued on main_stream so it
 * runs while the misses are copied on side_stream; the layer's accesses are
 * cut into steps (T = 1: the token's k ids in selection order; T > 1: the
 * chunk's distinct experts, resident ones first, each group ascending, k per
 * step); per step moe_lfu_step stages the blobs and main_stream runs the
 * expert kernels for that step's experts through dev_table; then the combine
 * adds y into hres.  The per-pair arithmetic is that of moe_layer_forward
 * with the same flags, so the result equals the all-resident layer bit for bit.
 * Source: "TurboFieldfare: Gemma 4 26B on an 8 GB MacBook, in ~2 GB of RAM"
 * (blog-mushroom.pages.dev), section "Why 26B Fits in 2 GB" (hits reuse the
 * resident blob, misses fetch it, the shared expert runs meanwhile).
 *   dev_table  device [E] pointer table of this layer (updated per step)
 *   ws         device workspace >= moe_streamed_workspace_size(...)
 *   flags      MOE_FLAG_* as in moe_layer_forward
 * All the steps of one call form one transaction of the cache (see
 * moe_lfu_step): if the call fails after planning, the layer's cache state
 * and log are as before the call and hres is unchanged, so the caller may
 * repeat the call. */
MOE_API size_t moe_streamed_workspace_size(int T, int H, int I, int Is, int E, int k);
MOE_API int moe_streamed_layer_forward(moe_lfu* h, int layer, float* hres, int T, int H, int I, int Is,
                                       int E, int k, const moe_qmat* router, const float* bias,
                                       int bias_per_row, const moe_qmat* shared, void** dev_table,
                                       uint16_t* x_out, uint16_t* y_out, int32_t* idx_out, void* ws,
                                       size_t ws_bytes, int flags, void* main_stream, void* side_stream,
                                       int timeout_ms);

/* ---------------------------------------------------------------------------
 * Expert parallelism (one process per GPU, G ranks).  The pages run the
 * layer on one device; splitting its routed experts over ranks is this
 * library's extension of the same computation.  Per token only its top-k
 * routed experts are applied ("drumih/turbo-fieldfare" (paperfeed.app),
 * section "Why this is interesting"), each from its own 4-bit blob
 * ("TurboFieldfare: Gemma 4 26B on an 8 GB MacBook, in ~2 GB of RAM"
 * (blog-mushroom.pages.dev), section "Why 26B Fits in 2 GB"), so the experts
 * split into disjoint sets: rank d owns experts [d E/G, (d+1) E/G), and a
 * (token, slot) pair is computed where its expert lives.  Each rank keeps its
 * own tokens, router, shared expert and combine; results equal the one-GPU
 * layer's within the output tolerance (the grouped GEMM sees other bucket
 * sizes).
 *
 * Per layer, on each rank: norm, router, moe_bucket; all ranks' bucket
 * offsets gathered into all_offsets (int32 [G][E+1], rank r's row r, e.g. by
 * an all-gather); moe_ep_dispatch (which also writes the rank's receiver
 * plan); a barrier across ranks; moe_expert_forward over the received rows
 * (k = 1, E/G experts); moe_ep_return; a barrier; moe_combine of the rank's
 * own y_pairs.
 *
 * Receiver layout: rank d's received rows are ordered by its experts, then
 * by source rank, then by the source's bucket order.  With
 * cnt(s,e) = all_offsets[s][e+1] - all_offsets[s][e], slot i of source s's
 * bucket e lands on row base(e) + before(s,e) + (i - all_offsets[s][e]) of
 * rank e/(E/G), where base(e) sums cnt over all sources and the experts of
 * that rank below e, and before(s,e) sums cnt(s',e) over s' < s.
 *
 * Peer tables are host arrays of G device pointers, entry r being rank r's
 * buffer as this process maps it (its own buffer for r = this rank, an
 * moe_ipc_open mapping for the others); each must be 16-byte aligned.
 * Requirements: 1 <= G <= 8, E/G a whole multiple of 8, 0 <= rank < G.
 * Rows past a receiver's capacity are skipped and flagged (check word bit 8,
 * MOE_ERR_DEVICE_CHECK at the next moe_sync).  Errors otherwise as the other
 * calls: MOE_ERR_INVALID_ARG before any launch.
 * --------------------------------------------------------------------------- */

/* Dispatch (source rank `rank`): for each bucketed slot i < all_offsets[rank][E]
 * with pair p = pairs[i], copies x row p / k (bf16 [H]) to row
 * base(e) + before(rank,e) + (i - off[e]) of recv_x[e/(E/G)] (bf16 [cap_rows, H])
 * and writes (rank, p) to the same row of recv_meta[...] (int32 [cap_rows, 2]),
 * e = idx[p].  The same launch writes this rank's receiver plan (device):
 * plan_offsets int32 [E/G + 1] = base(rank*E/G + j) clamped to cap_rows
 * (plan_offsets[E/G] = rows received), plan_pairs int32 [cap_rows] = the
 * identity over the rows received, plan_active int32 [E/G] = the local
 * experts with rows, ascending, plan_n_active int32 [1]: the inputs of
 * moe_expert_forward over recv_x with T = cap_rows, k = 1, E = E/G and this
 * rank's blob table, once every rank's dispatch has completed.
 *   x        bf16 [T,H] (device): the layer input
 *   idx      int32 [T,k] (device) routing; pairs: from moe_bucket (device)
 *   all_offsets  int32 [G][E+1] (device)
 *   recv_x, recv_meta  host arrays [G] of peer device pointers
 * T = 0 still launches (the plan covers what the other ranks send).  The
 * stores are complete when the kernel is; a barrier across ranks ordered
 * after it on the stream makes them safe to read on the peers. */
MOE_API int moe_ep_dispatch(const uint16_t* x, int T, int H, int k, int E, int G, int rank,
                            const int32_t* idx, const int32_t* pairs, const int32_t* all_offsets,
                            void* const* recv_x, void* const* recv_meta, int cap_rows,
                            int32_t* plan_offsets, int32_t* plan_pairs, int32_t* plan_active,
                            int32_t* plan_n_active, void* stream);

/* Return (receiver rank `rank`): row r < offsets[E/G] of y_rows (fp32
 * [cap_rows, H], the expert outputs over the received rows) goes to row p of
 * y_pairs[s] (fp32 [n_pair_slots, H] on rank s), (s, p) = recv_meta[r].
 * Completion as for the dispatch. */
MOE_API int moe_ep_return(const float* y_rows, int H, int E, int G, int rank, const void* recv_meta,
                          const int32_t* offsets, int n_pair_slots, int cap_rows, void* const* y_pairs,
                          void* stream);

/* Device buffers that other processes may map: moe_device_alloc returns a
 * whole allocation of `bytes` (cudaMalloc) whose handle moe_ipc_get_handle
 * writes into moe_ipc_handle_bytes() bytes; another process on the same node
 * maps it with moe_ipc_open (peer access enabled on first use) and unmaps it
 * with moe_ipc_close.  A process cannot open its own handle. */
MOE_API int moe_device_alloc(size_t bytes, void** ptr);
MOE_API int moe_device_free(void* ptr);
MOE_API int moe_ipc_handle_bytes(void);
MOE_API int moe_ipc_get_handle(const void* ptr, void* handle_out);
MOE_API int moe_ipc_open(const void* handle, void** ptr);
MOE_API int moe_ipc_close(void* ptr);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H_ */
