// Routed-expert forward without a caller workspace.
//
// Some callers cannot allocate device memory at the point where they run the
// experts: code that runs inside a CUDA graph being captured, custom
// allocators or memory pools that must not be re-entered, and embedders whose
// device memory is fully reserved up front.  moe_expert_forward needs a
// workspace for the fp16 activations between the projections; this entry
// point takes that scratch from a fixed array that is part of the library
// image instead, so the caller passes only inputs and outputs.

namespace moe {

// The scratch: one array per GPU that loads the library, held until exit.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

// Host code must not use g_noalloc_scratch as an address: on the host it is a
// stand-in symbol.  Its device address is looked up on the current device at
// every call (a cheap host query), so a device reset, which reloads the
// library's device code at another address, cannot leave a stale pointer.
static int noalloc_scratch(void** out) {
  void* p = nullptr;
  int st = cuda_check(cudaGetSymbolAddress(&p, g_noalloc_scratch), "cudaGetSymbolAddress(scratch)");
  if (st) return st;
  *out = p;
  return MOE_OK;
}

}  // namespace moe

extern "C" int moe_expert_forward_noalloc(const uint16_t* x, int T, int H, int I, int E, int k,
                                          const void* const* blob_ptrs, const int32_t* offsets,
                                          const int32_t* pairs, const int32_t* active,
                                          const int32_t* n_active, float* y_pairs, void* stream) {
  using namespace moe;
  // every argument check of moe_expert_forward, before any CUDA call
  int st = check_dims(T, H, I, E, k);
  if (st) return st;
  const size_t need = moe_expert_workspace_size(T, H, I, k);
  if (need > static_cast<size_t>(MOE_NOALLOC_SCRATCH_BYTES))
    return fail(MOE_ERR_INVALID_ARG,
                "moe_expert_forward_noalloc: T=%d k=%d H=%d I=%d needs %zu bytes of scratch, more than the "
                "%d-byte static scratch; use moe_expert_forward with a workspace",
                T, k, H, I, need, MOE_NOALLOC_SCRATCH_BYTES);
  if (T == 0) return MOE_OK;
  if (!x || !blob_ptrs || !offsets || !pairs || !active || !n_active || !y_pairs)
    return fail(MOE_ERR_INVALID_ARG, "moe_expert_forward_noalloc: NULL pointer");
  if (!aligned16(x) || !aligned16(y_pairs))
    return fail(MOE_ERR_INVALID_ARG, "moe_expert_forward_noalloc: misaligned pointer");
  void* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch))) return st;
  // Every region of the scratch is written by the call's own kernels before
  // they read it (the chunk plan, the gathered input, the activations), so
  // nothing in it has to start at zero.
  return moe_expert_forward(x, T, H, I, E, k, blob_ptrs, offsets, pairs, active, n_active, y_pairs, scratch,
                            static_cast<size_t>(MOE_NOALLOC_SCRATCH_BYTES), 0, stream);
}
