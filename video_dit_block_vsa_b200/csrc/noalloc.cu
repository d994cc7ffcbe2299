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
// address, so the device address is looked up once per device with
// cudaGetSymbolAddress (with that device current) and passed to the kernels.
// The first call on each device does that lookup.
#include <mutex>

#include "common.cuh"

namespace vsa {
namespace {

// 32 MiB: pooled q, k, v in float32, 3 * B * H * C * d * 4 bytes.
constexpr size_t kNoAllocScratchBytes = 32ull << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDev = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDev];

// Device address of the scratch array on the current device (set up once).
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return VSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return VSA_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return VSA_OK;
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
