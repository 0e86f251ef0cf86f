// Routed-expert forward without a caller workspace.
//
// Some callers cannot allocate device memory at the point where they run the
// experts: code that runs inside a CUDA graph being captured, custom
// allocators or memory pools that must not be re-entered, and embedders whose
// device memory is fully reserved up front.  moe_expert_forward needs a
// workspace for the fp16 activation between the gate/up and the down
// projections; this entry point takes that scratch from a fixed array that is
// part of the library image instead, so the caller passes only inputs and
// outputs.
#include <mutex>

namespace moe {

// The scratch: one array per GPU that loads the library, held until exit.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

// Host code must not use g_noalloc_scratch as an address: on the host it is a
// stand-in symbol.  Its device address is looked up once per device.
static void* g_noalloc_ptr[64];
static std::mutex g_noalloc_mu;

static int noalloc_scratch(void** out) {
  int dev = 0;
  int st = cuda_check(cudaGetDevice(&dev), "cudaGetDevice");
  if (st) return st;
  if (dev < 0 || dev >= 64) return fail(MOE_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    st = cuda_check(cudaGetSymbolAddress(&p, g_noalloc_scratch), "cudaGetSymbolAddress(scratch)");
    if (st) return st;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return MOE_OK;
}

}  // namespace moe

extern "C" int moe_expert_forward_noalloc(const uint16_t* x, int T, int H, int I, int E, int k,
                                          const void* const* blob_ptrs, const int32_t* offsets,
                                          const int32_t* pairs, const int32_t* active,
                                          const int32_t* n_active, float* y_pairs, void* stream) {
  using namespace moe;
  int st = check_dims(T, H, I, E, k);
  if (st) return st;
  const size_t need = moe_expert_workspace_size(T, H, I, k);
  if (need > static_cast<size_t>(MOE_NOALLOC_SCRATCH_BYTES))
    return fail(MOE_ERR_INVALID_ARG,
                "moe_expert_forward_noalloc: T=%d k=%d I=%d needs %zu bytes of scratch, more than the "
                "%d-byte static scratch; use moe_expert_forward with a workspace",
                T, k, I, need, MOE_NOALLOC_SCRATCH_BYTES);
  if (T == 0) return MOE_OK;
  void* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch))) return st;
  // The activation rows are written by the gate/up kernel before the down
  // kernel reads them, so nothing in the scratch has to start at zero.
  return moe_expert_forward(x, T, H, I, E, k, blob_ptrs, offsets, pairs, active, n_active, y_pairs, scratch,
                            static_cast<size_t>(MOE_NOALLOC_SCRATCH_BYTES), stream);
}
