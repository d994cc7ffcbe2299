// vsa_forward_host: the whole forward path from HOST buffers.  The (b, h)
// planes are independent, so they are processed in chunks: while one chunk
// computes on the caller's stream, the next chunk's q, k, v (and gates) are
// copied in on one internal stream and the previous chunk's output is copied
// out on another, so PCIe transfers in both directions overlap the kernels.
// Every stage runs through the library's own entry points: tiling and pooling
// in one pass, the coarse stage, and the fine stage writing the final output
// (gated combine and untile in its epilogue).
#include <cuda_runtime.h>

#include <cstdint>

#include "common.cuh"

namespace vsa {
namespace {

constexpr int kBufs = 2;  // chunk buffers in flight

struct CopyStreams {
  cudaStream_t h2d = nullptr;
  cudaStream_t d2h = nullptr;
};

CtxCache<CopyStreams> g_streams;

// Two non-blocking copy streams per CUDA context, created on first use in
// that context and kept for the life of the process (a stream belongs to the
// context it was created in).
int copy_streams(CopyStreams* out) {
  const bool ok = g_streams.get(current_context_id(), [](CopyStreams* cs) {
    if (cudaStreamCreateWithFlags(&cs->h2d, cudaStreamNonBlocking) != cudaSuccess) return false;
    if (cudaStreamCreateWithFlags(&cs->d2h, cudaStreamNonBlocking) != cudaSuccess) {
      cudaStreamDestroy(cs->h2d);
      return false;
    }
    return true;
  }, out);
  return ok ? VSA_OK : VSA_ERR_CUDA;
}

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Byte offsets of one chunk buffer inside the workspace.
struct ChunkLayout {
  size_t x[3], g[2], xt[3], out, oc, sel, pool, counts, total;
};

ChunkLayout chunk_layout(int C, long long N, int d, int topk, int hc, bool gated) {
  ChunkLayout L{};
  const size_t tok = static_cast<size_t>(hc) * N * d * 2;           // bf16 [hc, N, d]
  const size_t til = static_cast<size_t>(hc) * 64 * C * d * 2;       // bf16 [hc, 64C, d]
  size_t off = 0;
  for (int i = 0; i < 3; ++i) { L.x[i] = off; off += round256(tok); }
  for (int i = 0; i < 2; ++i) {
    L.g[i] = off;
    if (gated) off += round256(static_cast<size_t>(hc) * N * 4);
  }
  for (int i = 0; i < 3; ++i) { L.xt[i] = off; off += round256(til); }
  L.out = off; off += round256(tok);
  L.oc = off; if (gated) off += round256(static_cast<size_t>(hc) * C * d * 4);
  L.sel = off; off += round256(static_cast<size_t>(hc) * C * topk * 4);
  L.pool = off; off += round256(3ull * hc * C * d * 4);
  L.counts = off; off += round256(static_cast<size_t>(C) * 4);
  L.total = off;
  return L;
}

bool shape_ok(const vsa_shape* s, int topk, int* C, long long* N) {
  if (s == nullptr) return false;
  if (vsa_num_cubes(s, C) != VSA_OK) return false;
  if (topk < 1 || topk > *C) return false;
  *N = static_cast<long long>(s->grid_t) * s->grid_h * s->grid_w;
  return true;
}

int chunk_heads(const vsa_shape* s, int heads_per_chunk) {
  const int bh = s->batch * s->heads;
  int hc = heads_per_chunk > 0 ? heads_per_chunk : 2;
  return hc < bh ? hc : bh;
}

}  // namespace
}  // namespace vsa

using namespace vsa;

extern "C" {

size_t vsa_forward_host_workspace_bytes(const vsa_shape* shape, int topk, int heads_per_chunk,
                                        int gated) {
  int C = 0;
  long long N = 0;
  if (!shape_ok(shape, topk, &C, &N) || heads_per_chunk < 0) return 0;
  const int hc = chunk_heads(shape, heads_per_chunk);
  return kBufs * chunk_layout(C, N, shape->head_dim, topk, hc, gated != 0).total;
}

int vsa_forward_host(const vsa_shape* shape, int topk, const void* q, const void* k,
                     const void* v, const float* g_fine, const float* g_coarse, void* out,
                     void* workspace, size_t workspace_bytes, int heads_per_chunk,
                     cudaStream_t stream) {
  int C = 0;
  long long N = 0;
  if (!shape_ok(shape, topk, &C, &N) || heads_per_chunk < 0) return VSA_ERR_INVALID_ARG;
  if (!q || !k || !v || !out || !workspace) return VSA_ERR_INVALID_ARG;
  if ((g_fine == nullptr) != (g_coarse == nullptr)) return VSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return VSA_ERR_INVALID_ARG;
  const bool gated = g_fine != nullptr;
  const int d = shape->head_dim;
  const int bh_total = shape->batch * shape->heads;
  const int hc = chunk_heads(shape, heads_per_chunk);
  const ChunkLayout L = chunk_layout(C, N, d, topk, hc, gated);
  if (workspace_bytes < kBufs * L.total) return VSA_ERR_INVALID_ARG;
  // The shape itself (and the sub-shapes below) go through the full checks.
  vsa_shape sub = *shape;
  sub.batch = 1;
  sub.heads = hc;
  int rc = vsa_num_cubes(&sub, &C);
  if (rc != VSA_OK) return rc;

  CopyStreams cs;
  if ((rc = copy_streams(&cs)) != VSA_OK) return rc;
  cudaEvent_t ev_entry, ev_in[kBufs], ev_done[kBufs], ev_out[kBufs];
  cudaEvent_t* all[1 + 3 * kBufs] = {&ev_entry};
  for (int b = 0; b < kBufs; ++b) {
    all[1 + b] = &ev_in[b];
    all[1 + kBufs + b] = &ev_done[b];
    all[1 + 2 * kBufs + b] = &ev_out[b];
  }
  int made = 0;
  for (; made < 1 + 3 * kBufs; ++made)
    if (cudaEventCreateWithFlags(all[made], cudaEventDisableTiming) != cudaSuccess) break;
  auto finish = [&](int code) {
    for (int i = 0; i < made; ++i) cudaEventDestroy(*all[i]);  // released once their work ends
    return code;
  };
  if (made != 1 + 3 * kBufs) return finish(VSA_ERR_CUDA);

  // Earlier work on `stream` may still use the workspace.
  if (cudaEventRecord(ev_entry, stream) != cudaSuccess ||
      cudaStreamWaitEvent(cs.h2d, ev_entry, 0) != cudaSuccess ||
      cudaStreamWaitEvent(cs.d2h, ev_entry, 0) != cudaSuccess)
    return finish(VSA_ERR_CUDA);

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t plane_tok = static_cast<size_t>(N) * d * 2;
  const size_t plane_gate = static_cast<size_t>(N) * 4;
  const void* src[3] = {q, k, v};
  const float* gsrc[2] = {g_fine, g_coarse};
  const int nchunks = (bh_total + hc - 1) / hc;
  for (int ci = 0; ci < nchunks; ++ci) {
    const int b = ci % kBufs;
    uint8_t* base = ws + b * L.total;
    const int h0 = ci * hc;
    const int n = (bh_total - h0) < hc ? (bh_total - h0) : hc;
    sub.heads = n;
    // inputs: wait until the chunk that last used this buffer has computed
    if (ci >= kBufs && cudaStreamWaitEvent(cs.h2d, ev_done[b], 0) != cudaSuccess)
      return finish(VSA_ERR_CUDA);
    for (int t = 0; t < 3; ++t)
      if (cudaMemcpyAsync(base + L.x[t], static_cast<const uint8_t*>(src[t]) + h0 * plane_tok,
                          n * plane_tok, cudaMemcpyHostToDevice, cs.h2d) != cudaSuccess)
        return finish(VSA_ERR_CUDA);
    if (gated)
      for (int t = 0; t < 2; ++t)
        if (cudaMemcpyAsync(base + L.g[t], reinterpret_cast<const uint8_t*>(gsrc[t]) + h0 * plane_gate,
                            n * plane_gate, cudaMemcpyHostToDevice, cs.h2d) != cudaSuccess)
          return finish(VSA_ERR_CUDA);
    if (cudaEventRecord(ev_in[b], cs.h2d) != cudaSuccess) return finish(VSA_ERR_CUDA);
    // compute: after the inputs landed and the buffer's previous output left
    if (cudaStreamWaitEvent(stream, ev_in[b], 0) != cudaSuccess) return finish(VSA_ERR_CUDA);
    if (ci >= kBufs && cudaStreamWaitEvent(stream, ev_out[b], 0) != cudaSuccess)
      return finish(VSA_ERR_CUDA);
    int32_t* counts = reinterpret_cast<int32_t*>(base + L.counts);
    int32_t* sel = reinterpret_cast<int32_t*>(base + L.sel);
    float* oc = gated ? reinterpret_cast<float*>(base + L.oc) : nullptr;
    const size_t pool_bytes = vsa_workspace_bytes(&sub, topk);
    if ((rc = vsa_tile_permute_pool(&sub, base + L.x[0], base + L.x[1], base + L.x[2],
                                    base + L.xt[0], base + L.xt[1], base + L.xt[2], counts,
                                    base + L.pool, pool_bytes, stream)) != VSA_OK ||
        (rc = vsa_coarse_select_pooled(&sub, topk, oc, sel, nullptr, base + L.pool, pool_bytes,
                                       stream)) != VSA_OK ||
        (rc = vsa_block_sparse_fwd_out(
             &sub, base + L.xt[0], base + L.xt[1], base + L.xt[2], counts, sel, topk, oc,
             gated ? reinterpret_cast<const float*>(base + L.g[0]) : nullptr,
             gated ? reinterpret_cast<const float*>(base + L.g[1]) : nullptr, base + L.out,
             nullptr, stream)) != VSA_OK)
      return finish(rc);
    if (cudaEventRecord(ev_done[b], stream) != cudaSuccess) return finish(VSA_ERR_CUDA);
    // output
    if (cudaStreamWaitEvent(cs.d2h, ev_done[b], 0) != cudaSuccess ||
        cudaMemcpyAsync(static_cast<uint8_t*>(out) + h0 * plane_tok, base + L.out, n * plane_tok,
                        cudaMemcpyDeviceToHost, cs.d2h) != cudaSuccess ||
        cudaEventRecord(ev_out[b], cs.d2h) != cudaSuccess)
      return finish(VSA_ERR_CUDA);
  }
  // `stream` completes only after the last output copy.
  for (int b = 0; b < kBufs && b < nchunks; ++b)
    if (cudaStreamWaitEvent(stream, ev_out[b], 0) != cudaSuccess) return finish(VSA_ERR_CUDA);
  return finish(VSA_OK);
}

}  // extern "C"
