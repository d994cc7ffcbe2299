// vsa_coarse_select_noalloc: the coarse stage for callers that cannot
// allocate device memory.
//
// vsa_coarse_select needs a caller-supplied workspace for the pooled q, k, v
// cubes.  Some callers cannot provide one: a plugin or extension loaded into a
// host application that owns every device allocation itself and offers no
// allocator to its plugins, or code that must not call cudaMalloc while work
// is in flight because cudaMalloc may synchronise the device.  This entry
// point serves them: its scratch is a fixed file-scope device array that
// exists in every GPU context that loads the library, from module load until
// the process exits.
//
// The array's host-side name is only a stand-in for the symbol, never a device
// address, so the device address is looked up with cudaGetSymbolAddress in the
// calling thread's current CUDA context and passed to the kernels.  The
// address belongs to that context, so it is cached per context (by the
// context's unique id): a context the caller made current, or the new primary
// context after cudaDeviceReset, gets its own lookup.  The first call in each
// context does that lookup.
#include "common.cuh"

namespace vsa {
namespace {

// 32 MiB: pooled q, k, v in float32, 3 * B * H * C * d * 4 bytes.
constexpr size_t kNoAllocScratchBytes = 32ull << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

CtxCache<void*> g_noalloc_ptr;

// Device address of the scratch array in the current context.
int noalloc_scratch(void** out) {
  const bool ok = g_noalloc_ptr.get(current_context_id(), [](void** p) {
    return cudaGetSymbolAddress(p, g_noalloc_scratch) == cudaSuccess && *p != nullptr;
  }, out);
  return ok ? VSA_OK : VSA_ERR_CUDA;
}

}  // namespace
}  // namespace vsa

using namespace vsa;

extern "C" int vsa_coarse_select_noalloc(const vsa_shape* shape, const void* q_tiled,
                                         const void* k_tiled, const void* v_tiled,
                                         const int32_t* cube_count, int topk, float* o_coarse,
                                         int32_t* sel_idx, float* coarse_logits,
                                         cudaStream_t stream) {
  const size_t need = vsa_workspace_bytes(shape, topk);
  if (need == 0) {
    // Shape or k invalid: let the workspace entry point classify the error
    // (it returns before any launch).
    return vsa_coarse_select(shape, q_tiled, k_tiled, v_tiled, cube_count, topk, o_coarse,
                             sel_idx, coarse_logits, nullptr, 0, stream);
  }
  if (need > kNoAllocScratchBytes) return VSA_ERR_TOO_LARGE;
  void* scratch = nullptr;
  const int rc = noalloc_scratch(&scratch);
  if (rc != VSA_OK) return rc;
  // Same validation and kernels as vsa_coarse_select, with the static scratch
  // as the workspace; the pooling pass overwrites every scratch element it
  // reads, so nothing needs clearing.
  return vsa_coarse_select(shape, q_tiled, k_tiled, v_tiled, cube_count, topk, o_coarse, sel_idx,
                           coarse_logits, scratch, kNoAllocScratchBytes, stream);
}
