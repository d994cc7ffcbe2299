// extern "C" entry points of libvsa (declared in include/vsa.h): argument
// validation, per-device setup (architecture check, status word address),
// TMA tensor maps, and the kernel launches of the VSA forward path.
#include <cuda.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "common.cuh"
#include "fine.cuh"
#include "linear.cuh"

namespace vsa {

// Launchers (permute.cu, coarse.cu, fine.cu).
cudaError_t launch_tile_permute(const Geom&, const void*, void*, int32_t*, int, cudaStream_t);
cudaError_t launch_untile(const Geom&, const void*, void*, int, cudaStream_t);
cudaError_t launch_combine(const Geom&, const void*, const float*, const float*, const float*,
                           void*, int, cudaStream_t);
cudaError_t launch_coarse_select(const Geom&, const void*, const void*, const void*,
                                 const int32_t*, int, float*, int32_t*, float*, float*, int*,
                                 cudaStream_t, bool token_order);
cudaError_t launch_tile_pool(const Geom&, const void*, const void*, const void*, void*, void*,
                             void*, int32_t*, float*, int*, cudaStream_t);
cudaError_t launch_coarse_only(const Geom&, int, float*, int32_t*, float*, const float*,
                               cudaStream_t);
cudaError_t launch_block_sparse_fwd(const Geom&, const FineMaps&, const int32_t*, const int32_t*,
                                    int, void*, float*, const float*, const float*, const float*,
                                    bool, int*, int, cudaStream_t, const void*);
cudaError_t launch_debug_wait(uint64_t, int*, cudaStream_t);
cudaError_t launch_linear_branch(int bh, long long N, int d, const void* q, const void* k,
                                 void* out, uint8_t* ws, const LinearLayout& L,
                                 const CUtensorMap& fk_map, const CUtensorMap& v_map,
                                 const CUtensorMap& fq_map, const CUtensorMap& b_map, int* status,
                                 int sms, cudaStream_t s);
cudaError_t launch_projection(const Geom&, int, int, const CUtensorMap&, const CUtensorMap&, void*,
                              void*, void*, int32_t*, int*, int, cudaStream_t);
cudaError_t launch_select_transpose(int, int, int, const int32_t*, int32_t*, int32_t*, int32_t*,
                                    int*, int, cudaStream_t);
cudaError_t launch_backward_prep(const Geom&, const void*, const void*, const float*, const float*,
                                 const float*, void*, float*, float*, float*, float*, cudaStream_t);
cudaError_t launch_coarse_backward(int, int, int, const float*, const float*, const float*, float*,
                                   void*, size_t, cudaStream_t);
size_t coarse_backward_plane_bytes(int C);
cudaError_t launch_block_sparse_bwd(const Geom&, const BwdMaps&, int, const float*, const float*,
                                    const int32_t*, const int32_t*, const int32_t*, const float*,
                                    void*, void*, void*, int*, int, cudaStream_t, const void*,
                                    const void*);

// Device-side status word, one per device that loads the library.
__device__ int g_status;

namespace {

constexpr int kMaxDevices = 64;

// What the library needs per call on the current device: hardware facts (the
// same in every context on the device) and the status word's device address
// (valid only in the context it was looked up in).
struct DeviceState {
  int sms = 0;
  int* status = nullptr;
};

struct DeviceInfo {
  bool ready = false;
  int supported = 0;
  int sms = 0;
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
CtxCache<int*> g_status_ptr;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
std::once_flag g_ctx_fns_once;
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

template <typename Fn>
Fn driver_fn(const char* name) {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(fn);
}

// Per-call setup: architecture check (once per device) and the status word's
// device address in the current context (a host-side symbol is not a device
// pointer; the address is looked up once per context).
int device_state(DeviceState* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return VSA_ERR_CUDA;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceInfo& di = g_dev[dev];
    if (!di.ready) {
      int major = 0, minor = 0, sms = 0;
      if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return VSA_ERR_CUDA;
      di.supported = (major == 10 && minor == 0);
      di.sms = sms;
      di.ready = true;
    }
    if (!di.supported) return VSA_ERR_UNSUPPORTED;
    out->sms = di.sms;
  }
  const bool ok = g_status_ptr.get(current_context_id(), [](int** p) {
    void* a = nullptr;
    if (cudaGetSymbolAddress(&a, g_status) != cudaSuccess || a == nullptr) return false;
    *p = static_cast<int*>(a);
    return true;
  }, &out->status);
  return ok ? VSA_OK : VSA_ERR_CUDA;
}

int get_encoder() {
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_encode) return VSA_OK;
  g_encode = driver_fn<EncodeTiledFn>("cuTensorMapEncodeTiled");
  return g_encode ? VSA_OK : VSA_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Validates the shape and fills the geometry.  The tiled row count of all
// heads must fit a 32-bit TMA coordinate.
int make_geom(const vsa_shape* s, Geom* g) {
  if (s == nullptr) return VSA_ERR_INVALID_ARG;
  if (s->cube_t != 4 || s->cube_h != 4 || s->cube_w != 4) return VSA_ERR_UNSUPPORTED;
  if (s->head_dim != 64 && s->head_dim != 128) return VSA_ERR_UNSUPPORTED;
  if (s->batch < 1 || s->heads < 1 || s->grid_t < 1 || s->grid_h < 1 || s->grid_w < 1)
    return VSA_ERR_INVALID_ARG;
  g->B = s->batch;
  g->H = s->heads;
  g->d = s->head_dim;
  g->T = s->grid_t;
  g->Y = s->grid_h;
  g->X = s->grid_w;
  g->Ct = (g->T + 3) / 4;
  g->Cy = (g->Y + 3) / 4;
  g->Cx = (g->X + 3) / 4;
  const long long C = static_cast<long long>(g->Ct) * g->Cy * g->Cx;
  if (C > kMaxCubes) return VSA_ERR_UNSUPPORTED;
  g->C = static_cast<int>(C);
  g->N = static_cast<long long>(g->T) * g->Y * g->X;
  g->rows = C * kSlots;
  g->inv_cx = ((1ull << 32) + g->Cx - 1) / g->Cx;
  g->inv_cy = ((1ull << 32) + g->Cy - 1) / g->Cy;
  const long long all_rows = static_cast<long long>(g->B) * g->H * g->rows;
  if (all_rows >= (1ll << 31) || static_cast<long long>(g->B) * g->H >= 65536)
    return VSA_ERR_UNSUPPORTED;
  return VSA_OK;
}

int tiled_map(const Geom& g, const void* ptr, CUtensorMap* m, int box_rows = 64) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(g.d),
                              static_cast<cuuint64_t>(g.B) * g.H * g.rows};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(g.d) * 2};
  const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? VSA_OK : VSA_ERR_CUDA;
}

// The fine kernel's maps: q, k, v with one-cube boxes, k and v with 16-row boxes.
int fine_maps(const Geom& g, const void* q, const void* k, const void* v, FineMaps* m) {
  if (tiled_map(g, q, &m->q) != VSA_OK || tiled_map(g, k, &m->k) != VSA_OK ||
      tiled_map(g, v, &m->v) != VSA_OK || tiled_map(g, k, &m->k16, 16) != VSA_OK ||
      tiled_map(g, v, &m->v16, 16) != VSA_OK)
    return VSA_ERR_CUDA;
  return VSA_OK;
}

int cuda_rc(cudaError_t e) { return e == cudaSuccess ? VSA_OK : VSA_ERR_CUDA; }

}  // namespace
}  // namespace vsa

namespace vsa {

uint64_t current_context_id() {
  std::call_once(g_ctx_fns_once, [] {
    g_ctx_get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    g_ctx_get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  });
  if (g_ctx_get_current == nullptr || g_ctx_get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  if (g_ctx_get_current(&ctx) != CUDA_SUCCESS) return 0;
  if (ctx == nullptr) {
    // No context on this thread yet: make the current device's primary
    // context current, as the next runtime call would.
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess) return 0;
    if (g_ctx_get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  }
  unsigned long long id = 0;
  if (g_ctx_get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

}  // namespace vsa

using namespace vsa;

extern "C" {

int vsa_num_cubes(const vsa_shape* shape, int* num_cubes) {
  Geom g;
  if (num_cubes == nullptr) return VSA_ERR_INVALID_ARG;
  const int rc = make_geom(shape, &g);
  if (rc != VSA_OK) return rc;
  *num_cubes = g.C;
  return VSA_OK;
}

int vsa_topk_from_ratio(int num_cubes, float ratio, int* topk) {
  if (topk == nullptr || num_cubes < 1 || !(ratio > 0.0f) || ratio > 1.0f)
    return VSA_ERR_INVALID_ARG;
  long long k = static_cast<long long>(std::floor(static_cast<double>(ratio) * num_cubes + 0.5));
  if (k < 1) k = 1;
  if (k > num_cubes) k = num_cubes;
  *topk = static_cast<int>(k);
  return VSA_OK;
}

size_t vsa_workspace_bytes(const vsa_shape* shape, int topk) {
  Geom g;
  if (make_geom(shape, &g) != VSA_OK || topk < 1 || topk > g.C) return 0;
  const size_t bytes = 3ull * g.B * g.H * g.C * g.d * sizeof(float);
  return (bytes + 255) & ~static_cast<size_t>(255);
}

int vsa_tile_permute(const vsa_shape* shape, const void* x, void* x_tiled, int32_t* cube_count,
                     cudaStream_t stream) {
  Geom g;
  int rc = make_geom(shape, &g);
  if (rc != VSA_OK) return rc;
  if (!x || !x_tiled || !aligned16(x) || !aligned16(x_tiled) ||
      (cube_count && (reinterpret_cast<uintptr_t>(cube_count) & 3u)))
    return VSA_ERR_INVALID_ARG;
  DeviceState st;
  if ((rc = device_state(&st)) != VSA_OK) return rc;
  return cuda_rc(launch_tile_permute(g, x, x_tiled, cube_count, st.sms, stream));
}

size_t vsa_linear_workspace_bytes(const vsa_shape* shape) {
  Geom g;
  if (make_geom(shape, &g) != VSA_OK) return 0;
  return linear_layout(g.B * g.H, g.N, g.d).bytes;
}

// A bf16 tensor [planes][rows][cols] (cols contiguous) with 128-byte-swizzled
// boxes of 64 columns x box_rows rows x 1 plane.
int planes_map(const void* ptr, long long planes, long long rows, int cols, int box_rows,
               CUtensorMap* m) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(planes)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols) * 2,
                                 static_cast<cuuint64_t>(rows) * cols * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? VSA_OK : VSA_ERR_CUDA;
}

int matrix_map(const void* ptr, long long rows, long long cols, int box_rows, CUtensorMap* m);

int vsa_linear_branch_add(const vsa_shape* shape, const void* q, const void* k, const void* v,
                          void* out, void* workspace, size_t workspace_bytes,
                          cudaStream_t stream) {
  Geom g;
  int rc = make_geom(shape, &g);
  if (rc != VSA_OK) return rc;
  if (!q || !k || !v || !out || !workspace || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
      !aligned16(out) || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      workspace_bytes < vsa_linear_workspace_bytes(shape))
    return VSA_ERR_INVALID_ARG;
  DeviceState st;
  if ((rc = device_state(&st)) != VSA_OK) return rc;
  if ((rc = get_encoder()) != VSA_OK) return rc;
  const int bh = g.B * g.H;
  const LinearLayout L = linear_layout(bh, g.N, g.d);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  CUtensorMap fk_map, v_map, fq_map, b_map;
  if (planes_map(ws + L.fk, bh, g.N, g.d, 64, &fk_map) != VSA_OK ||
      planes_map(v, bh, g.N, g.d, 64, &v_map) != VSA_OK ||
      planes_map(ws + L.fq, bh, g.N, g.d, 128, &fq_map) != VSA_OK ||
      matrix_map(ws + L.bmat, static_cast<long long>(bh) * (g.d + 16), g.d, g.d + 16, &b_map) != VSA_OK)
    return VSA_ERR_CUDA;
  return cuda_rc(launch_linear_branch(bh, g.N, g.d, q, k, out, ws, L, fk_map, v_map, fq_map, b_map,
                                      st.status, st.sms, stream));
}

// A row-major bf16 matrix [rows, cols] with 128-byte-swizzled boxes of
// 64 columns x box_rows rows.
int matrix_map(const void* ptr, long long rows, long long cols, int box_rows, CUtensorMap* m) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? VSA_OK : VSA_ERR_CUDA;
}

int vsa_qkv_projection_tiled(const vsa_shape* shape, int hidden, const void* x, const void* w_qkv,
                             void* q_tiled, void* k_tiled, void* v_tiled, int32_t* cube_count,
                             cudaStream_t stream) {
  Geom g;
  int rc = make_geom(shape, &g);
  if (rc != VSA_OK) return rc;
  if (hidden < 64 || hidden % 64 != 0 || !x || !w_qkv || !q_tiled || !k_tiled || !v_tiled ||
      !aligned16(x) || !aligned16(w_qkv) || !aligned16(q_tiled) || !aligned16(k_tiled) ||
      !aligned16(v_tiled) || (cube_count && (reinterpret_cast<uintptr_t>(cube_count) & 3u)))
    return VSA_ERR_INVALID_ARG;
  const long long rows = static_cast<long long>(g.B) * g.N;
  if (rows >= (1ll << 31) || static_cast<long long>(hidden) * 3 * g.H * g.d >= (1ll << 40))
    return VSA_ERR_UNSUPPORTED;
  DeviceState st;
  if ((rc = device_state(&st)) != VSA_OK) return rc;
  if ((rc = get_encoder()) != VSA_OK) return rc;
  CUtensorMap amap, bmap;
  if (matrix_map(x, rows, hidden, 128, &amap) != VSA_OK ||
      matrix_map(w_qkv, 3ll * g.H * g.d, hidden, 256, &bmap) != VSA_OK)
    return VSA_ERR_CUDA;
  return cuda_rc(launch_projection(g, 0, hidden, amap, bmap, q_tiled, k_tiled, v_tiled, cube_count,
                                   st.status, st.sms, stream));
}

int vsa_out_projection_tiled(const vsa_shape* shape, int hidden, const void* o_tiled,
                             const void* w_o, void* y, cudaStream_t stream) {
  Geom g;
  int rc = make_geom(shape, &g);
  if (rc != VSA_OK) return rc;
  if (hidden < 64 || hidden % 64 != 0 || !o_tiled || !w_o || !y || !aligned16(o_tiled) ||
      !aligned16(w_o) || !aligned16(y))
    return VSA_ERR_INVALID_ARG;
  DeviceState st;
  if ((rc = device_state(&st)) != VSA_OK) return rc;
  if ((rc = get_encoder()) != VSA_OK) return rc;
  CUtensorMap amap, bmap;
  if (matrix_map(o_tiled, static_cast<long long>(g.B) * g.H * g.rows, g.d, 128, &amap) != VSA_OK ||
      matrix_map(w_o, hidden, static_cast<long long>(g.H) * g.d, 256, &bmap) != VSA_OK)
    return VSA_ERR_CUDA;
  return cuda_rc(launch_projection(g, 1, hidden, amap, bmap, y, nullptr, nullptr, nullptr,
                                   st.status, st.sms, stream));
}

int vsa_untile(const vsa_shape* shape, const void* x_tiled, void* x, cudaStream_t stream) {
  Geom g;
  int rc = make_geom(shape, &g);
  if (rc != VSA_OK) return rc;
  if (!x || !x_tiled || !aligned16(x) || !aligned16(x_tiled)) return VSA_ERR_INVALID_ARG;
  DeviceState st;
  if ((rc = device_state(&st)) != VSA_OK) return rc;
  return cuda_rc(launch_untile(g, x_tiled, x, st.sms, stream));
}

int vsa_combine(const vsa_shape* shape, const void* o_fine_tiled, const float* o_coarse,
                const float* g_fine, const float* g_coarse, void* out_tiled, cudaStream_t stream) {
  Geom g;
  int rc = make_geom(shape, &g);
  if (rc != VSA_OK) return rc;
  if (!o_fine_tiled || !out_tiled || !aligned16(o_fine_tiled) || !aligned16(out_tiled))
    return VSA_ERR_INVALID_ARG;
  if ((g_fine == nullptr) != (g_coarse == nullptr)) return VSA_ERR_INVALID_ARG;
  if (g_fine && (!o_coarse || !aligned16(o_coarse) ||
                 (reinterpret_cast<uintptr_t>(g_fine) & 3u) ||
                 (reinterpret_cast<uintptr_t>(g_coarse) & 3u)))
    return VSA_ERR_INVALID_ARG;
  DeviceState st;
  if ((rc = device_state(&st)) != VSA_OK) return rc;
  return cuda_rc(launch_combine(g, o_fine_tiled, o_coarse, g_fine, g_coarse, out_tiled, st.sms,
                                stream));
}

int vsa_coarse_select(const vsa_shape* shape, const void* q_tiled, const void* k_tiled,
                      const void* v_tiled, const int32_t* cube_count, int topk, float* o_coarse,
                      int32_t* sel_idx, float* coarse_logits, void* workspace,
                      size_t workspace_bytes, cudaStream_t stream) {
  Geom g;
  int rc = make_geom(shape, &g);
  if (rc != VSA_OK) return rc;
  if (topk < 1 || topk > g.C) return VSA_ERR_INVALID_ARG;
  if (!q_tiled || !k_tiled || !v_tiled || !cube_count || !sel_idx || !workspace)
    return VSA_ERR_INVALID_ARG;
  if (!aligned16(q_tiled) || !aligned16(k_tiled) || !aligned16(v_tiled) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      (reinterpret_cast<uintptr_t>(cube_count) & 3u) ||
      (reinterpret_cast<uintptr_t>(sel_idx) & 3u) || (o_coarse && !aligned16(o_coarse)) ||
      (coarse_logits && (reinterpret_cast<uintptr_t>(coarse_logits) & 3u)))
    return VSA_ERR_INVALID_ARG;
  if (workspace_bytes < vsa_workspace_bytes(shape, topk)) return VSA_ERR_INVALID_ARG;
  DeviceState st;
  if ((rc = device_state(&st)) != VSA_OK) return rc;
  return cuda_rc(launch_coarse_select(g, q_tiled, k_tiled, v_tiled, cube_count, topk, o_coarse,
                                      sel_idx, coarse_logits, static_cast<float*>(workspace),
                                      st.status, stream, false));
}

int vsa_tile_permute_pool(const vsa_shape* shape, const void* q, const void* k, const void* v,
                          void* q_tiled, void* k_tiled, void* v_tiled, int32_t* cube_count,
                          void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  Geom g;
  int rc = make_geom(shape, &g);
  if (rc != VSA_OK) return rc;
  if (!q || !k || !v || !q_tiled || !k_tiled || !v_tiled || !workspace) return VSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q_tiled) ||
      !aligned16(k_tiled) || !aligned16(v_tiled) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      (cube_count && (reinterpret_cast<uintptr_t>(cube_count) & 3u)))
    return VSA_ERR_INVALID_ARG;
  if (workspace_bytes < vsa_workspace_bytes(shape, 1)) return VSA_ERR_INVALID_ARG;
  DeviceState st;
  if ((rc = device_state(&st)) != VSA_OK) return rc;
  return cuda_rc(launch_tile_pool(g, q, k, v, q_tiled, k_tiled, v_tiled, cube_count,
                                  static_cast<float*>(workspace), st.status, stream));
}

int vsa_coarse_select_pooled(const vsa_shape* shape, int topk, float* o_coarse, int32_t* sel_idx,
                             float* coarse_logits, const void* workspace, size_t workspace_bytes,
                             cudaStream_t stream) {
  Geom g;
  int rc = make_geom(shape, &g);
  if (rc != VSA_OK) return rc;
  if (topk < 1 || topk > g.C) return VSA_ERR_INVALID_ARG;
  if (!sel_idx || !workspace) return VSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      (reinterpret_cast<uintptr_t>(sel_idx) & 3u) || (o_coarse && !aligned16(o_coarse)) ||
      (coarse_logits && (reinterpret_cast<uintptr_t>(coarse_logits) & 3u)))
    return VSA_ERR_INVALID_ARG;
  if (workspace_bytes < vsa_workspace_bytes(shape, topk)) return VSA_ERR_INVALID_ARG;
  DeviceState st;
  if ((rc = device_state(&st)) != VSA_OK) return rc;
  return cuda_rc(launch_coarse_only(g, topk, o_coarse, sel_idx, coarse_logits,
                                    static_cast<const float*>(workspace), stream));
}

int vsa_coarse_select_tokens(const vsa_shape* shape, const void* q, const void* k, const void* v,
                             int topk, float* o_coarse, int32_t* sel_idx, float* coarse_logits,
                             void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  Geom g;
  int rc = make_geom(shape, &g);
  if (rc != VSA_OK) return rc;
  if (topk < 1 || topk > g.C) return VSA_ERR_INVALID_ARG;
  if (!q || !k || !v || !sel_idx || !workspace) return VSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      (reinterpret_cast<uintptr_t>(sel_idx) & 3u) || (o_coarse && !aligned16(o_coarse)) ||
      (coarse_logits && (reinterpret_cast<uintptr_t>(coarse_logits) & 3u)))
    return VSA_ERR_INVALID_ARG;
  if (workspace_bytes < vsa_workspace_bytes(shape, topk)) return VSA_ERR_INVALID_ARG;
  DeviceState st;
  if ((rc = device_state(&st)) != VSA_OK) return rc;
  return cuda_rc(launch_coarse_select(g, q, k, v, nullptr, topk, o_coarse, sel_idx, coarse_logits,
                                      static_cast<float*>(workspace), st.status, stream, true));
}

int vsa_block_sparse_fwd(const vsa_shape* shape, const void* q_tiled, const void* k_tiled,
                         const void* v_tiled, const int32_t* cube_count, const int32_t* sel_idx,
                         int topk, void* o_fine_tiled, float* lse, cudaStream_t stream) {
  Geom g;
  int rc = make_geom(shape, &g);
  if (rc != VSA_OK) return rc;
  if (topk < 1 || topk > g.C) return VSA_ERR_INVALID_ARG;
  if (!q_tiled || !k_tiled || !v_tiled || !cube_count || !sel_idx || !o_fine_tiled)
    return VSA_ERR_INVALID_ARG;
  if (!aligned16(q_tiled) || !aligned16(k_tiled) || !aligned16(v_tiled) ||
      !aligned16(o_fine_tiled) || (reinterpret_cast<uintptr_t>(cube_count) & 3u) ||
      (reinterpret_cast<uintptr_t>(sel_idx) & 3u) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return VSA_ERR_INVALID_ARG;
  DeviceState st;
  if ((rc = device_state(&st)) != VSA_OK) return rc;
  if ((rc = get_encoder()) != VSA_OK) return rc;
  FineMaps maps;
  if (fine_maps(g, q_tiled, k_tiled, v_tiled, &maps) != VSA_OK) return VSA_ERR_CUDA;
  return cuda_rc(launch_block_sparse_fwd(g, maps, cube_count, sel_idx, topk, o_fine_tiled,
                                         lse, nullptr, nullptr, nullptr, false, st.status, st.sms,
                                         stream, q_tiled));
}

int vsa_block_sparse_fwd_out(const vsa_shape* shape, const void* q_tiled, const void* k_tiled,
                             const void* v_tiled, const int32_t* cube_count, const int32_t* sel_idx,
                             int topk, const float* o_coarse, const float* g_fine,
                             const float* g_coarse, void* out, float* lse, cudaStream_t stream) {
  Geom g;
  int rc = make_geom(shape, &g);
  if (rc != VSA_OK) return rc;
  if (topk < 1 || topk > g.C) return VSA_ERR_INVALID_ARG;
  if (!q_tiled || !k_tiled || !v_tiled || !cube_count || !sel_idx || !out)
    return VSA_ERR_INVALID_ARG;
  if ((g_fine == nullptr) != (g_coarse == nullptr)) return VSA_ERR_INVALID_ARG;
  if (g_fine && (!o_coarse || !aligned16(o_coarse) ||
                 (reinterpret_cast<uintptr_t>(g_fine) & 3u) ||
                 (reinterpret_cast<uintptr_t>(g_coarse) & 3u)))
    return VSA_ERR_INVALID_ARG;
  if (!aligned16(q_tiled) || !aligned16(k_tiled) || !aligned16(v_tiled) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(cube_count) & 3u) ||
      (reinterpret_cast<uintptr_t>(sel_idx) & 3u) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return VSA_ERR_INVALID_ARG;
  DeviceState st;
  if ((rc = device_state(&st)) != VSA_OK) return rc;
  if ((rc = get_encoder()) != VSA_OK) return rc;
  FineMaps maps;
  if (fine_maps(g, q_tiled, k_tiled, v_tiled, &maps) != VSA_OK) return VSA_ERR_CUDA;
  return cuda_rc(launch_block_sparse_fwd(g, maps, cube_count, sel_idx, topk, out, lse,
                                         g_fine ? o_coarse : nullptr, g_fine, g_coarse, true,
                                         st.status, st.sms, stream, q_tiled));
}

int vsa_select_transpose(const vsa_shape* shape, const int32_t* sel_idx, int topk,
                         int32_t* key_offsets, int32_t* query_lists, void* workspace,
                         size_t workspace_bytes, cudaStream_t stream) {
  Geom g;
  int rc = make_geom(shape, &g);
  if (rc != VSA_OK) return rc;
  if (topk < 1 || topk > g.C) return VSA_ERR_INVALID_ARG;
  if (!sel_idx || !key_offsets || !query_lists || !workspace) return VSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(sel_idx) & 3u) || (reinterpret_cast<uintptr_t>(key_offsets) & 3u) ||
      (reinterpret_cast<uintptr_t>(query_lists) & 3u) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return VSA_ERR_INVALID_ARG;
  const long long pairs = static_cast<long long>(g.B) * g.H * g.C * topk;
  if (static_cast<long long>(g.C) * topk >= (1ll << 31)) return VSA_ERR_UNSUPPORTED;
  if (workspace_bytes < static_cast<size_t>(pairs) * sizeof(int32_t)) return VSA_ERR_INVALID_ARG;
  DeviceState st;
  if ((rc = device_state(&st)) != VSA_OK) return rc;
  return cuda_rc(launch_select_transpose(g.B * g.H, g.C, topk, sel_idx, key_offsets, query_lists,
                                         static_cast<int32_t*>(workspace), st.status, st.sms, stream));
}

int vsa_backward_prep(const vsa_shape* shape, const void* dout, const void* o_fine_tiled,
                      const float* o_coarse, const float* g_fine, const float* g_coarse,
                      void* do_fine_tiled, float* delta, float* do_coarse, float* dg_fine,
                      float* dg_coarse, cudaStream_t stream) {
  Geom g;
  int rc = make_geom(shape, &g);
  if (rc != VSA_OK) return rc;
  if (!dout || !o_fine_tiled || !do_fine_tiled || !delta) return VSA_ERR_INVALID_ARG;
  if ((g_fine == nullptr) != (g_coarse == nullptr)) return VSA_ERR_INVALID_ARG;
  const bool gated = g_fine != nullptr;
  if (gated && (!o_coarse || !do_coarse || !dg_fine || !dg_coarse)) return VSA_ERR_INVALID_ARG;
  auto a4 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; };
  if (!aligned16(dout) || !aligned16(o_fine_tiled) || !aligned16(do_fine_tiled) || !a4(delta))
    return VSA_ERR_INVALID_ARG;
  if (gated && (!aligned16(o_coarse) || !aligned16(do_coarse) || !a4(g_fine) || !a4(g_coarse) ||
                !a4(dg_fine) || !a4(dg_coarse)))
    return VSA_ERR_INVALID_ARG;
  DeviceState st;
  if ((rc = device_state(&st)) != VSA_OK) return rc;
  return cuda_rc(launch_backward_prep(g, dout, o_fine_tiled, gated ? o_coarse : nullptr,
                                      g_fine, g_coarse, do_fine_tiled, delta,
                                      gated ? do_coarse : nullptr, gated ? dg_fine : nullptr,
                                      gated ? dg_coarse : nullptr, stream));
}

size_t vsa_coarse_backward_workspace_bytes(const vsa_shape* shape) {
  Geom g;
  if (make_geom(shape, &g) != VSA_OK) return 0;
  return static_cast<size_t>(g.B) * g.H * coarse_backward_plane_bytes(g.C);
}

int vsa_coarse_backward(const vsa_shape* shape, const float* pooled, const float* o_coarse,
                        const float* do_coarse, float* d_pooled, void* workspace,
                        size_t workspace_bytes, cudaStream_t stream) {
  Geom g;
  int rc = make_geom(shape, &g);
  if (rc != VSA_OK) return rc;
  if (!pooled || !o_coarse || !do_coarse || !d_pooled || !workspace) return VSA_ERR_INVALID_ARG;
  if (!aligned16(pooled) || !aligned16(o_coarse) || !aligned16(do_coarse) || !aligned16(d_pooled) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return VSA_ERR_INVALID_ARG;
  const long long bh = static_cast<long long>(g.B) * g.H;
  if (bh > 65535) return VSA_ERR_UNSUPPORTED;  // (b, h) is a grid index
  if (workspace_bytes < coarse_backward_plane_bytes(g.C)) return VSA_ERR_INVALID_ARG;
  DeviceState st;
  if ((rc = device_state(&st)) != VSA_OK) return rc;
  return cuda_rc(launch_coarse_backward(static_cast<int>(bh), g.C, g.d, pooled, o_coarse, do_coarse,
                                        d_pooled, workspace, workspace_bytes, stream));
}

int vsa_block_sparse_bwd(const vsa_shape* shape, const void* q_tiled, const void* k_tiled,
                         const void* v_tiled, const int32_t* sel_idx, int topk,
                         const int32_t* key_offsets, const int32_t* query_lists, const float* lse,
                         const void* do_fine_tiled, const float* delta, const float* d_pooled,
                         void* dq, void* dk, void* dv, cudaStream_t stream) {
  Geom g;
  int rc = make_geom(shape, &g);
  if (rc != VSA_OK) return rc;
  if (topk < 1 || topk > g.C) return VSA_ERR_INVALID_ARG;
  if (!q_tiled || !k_tiled || !v_tiled || !sel_idx || !key_offsets || !query_lists || !lse ||
      !do_fine_tiled || !delta || !dq || !dk || !dv)
    return VSA_ERR_INVALID_ARG;
  auto a4 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; };
  if (!aligned16(q_tiled) || !aligned16(k_tiled) || !aligned16(v_tiled) ||
      !aligned16(do_fine_tiled) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      (d_pooled && !aligned16(d_pooled)) || !a4(sel_idx) || !a4(key_offsets) ||
      !a4(query_lists) || !aligned16(lse) || !aligned16(delta))
    return VSA_ERR_INVALID_ARG;
  DeviceState st;
  if ((rc = device_state(&st)) != VSA_OK) return rc;
  if ((rc = get_encoder()) != VSA_OK) return rc;
  BwdMaps maps;
  if (tiled_map(g, q_tiled, &maps.q) != VSA_OK || tiled_map(g, k_tiled, &maps.k) != VSA_OK ||
      tiled_map(g, v_tiled, &maps.v) != VSA_OK || tiled_map(g, do_fine_tiled, &maps.dO) != VSA_OK)
    return VSA_ERR_CUDA;
  return cuda_rc(launch_block_sparse_bwd(g, maps, topk, lse, delta, sel_idx, key_offsets,
                                         query_lists, d_pooled, dq, dk, dv, st.status, st.sms,
                                         stream, q_tiled, do_fine_tiled));
}

int vsa_get_status(cudaStream_t stream) {
  DeviceState st;
  int rc = device_state(&st);
  if (rc != VSA_OK) return rc;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return VSA_ERR_CUDA;
  int value = 0;
  const int zero = 0;
  if (cudaMemcpy(&value, st.status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemcpy(st.status, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
    return VSA_ERR_CUDA;
  return value;
}

int vsa_debug_wait_timeout(uint64_t timeout_ns, cudaStream_t stream) {
  if (timeout_ns < 1000ull || timeout_ns > 1000000000ull) return VSA_ERR_INVALID_ARG;
  DeviceState st;
  const int rc = device_state(&st);
  if (rc != VSA_OK) return rc;
  return cuda_rc(launch_debug_wait(timeout_ns, st.status, stream));
}

const char* vsa_strerror(int code) {
  switch (code) {
    case VSA_OK: return "ok";
    case VSA_ERR_INVALID_ARG: return "invalid argument";
    case VSA_ERR_UNSUPPORTED: return "unsupported shape or device";
    case VSA_ERR_CUDA: return "CUDA runtime error";
    case VSA_ERR_TIMEOUT: return "device wait timed out";
    case VSA_ERR_BAD_INDEX: return "inconsistent cube_count or sel_idx entry";
    case VSA_ERR_TOO_LARGE: return "problem exceeds the fixed scratch of vsa_coarse_select_noalloc";
    default: return "unknown status";
  }
}

}  // extern "C"
