// Backward of the coarse attention O_c = softmax(qbar kbar^T / sqrt(d)) vbar
// (float32, per (b, h), over the C pooled vectors): the coarse branch of a VSA
// backward pass.  With P the softmax, dO_c the incoming gradient and
// scale = 1/sqrt(d):
//   D_i   = <dO_c[i], O_c[i]>
//   dS_ij = P_ij (dP_ij - D_i),   dP = dO_c vbar^T
//   dqbar = scale dS kbar,   dkbar = scale dS^T qbar,   dvbar = P^T dO_c
//
// C is at most 8192 (1440 for a 720p video), so the C x C matrices are kept in
// a workspace (row stride ldc = C rounded up to 64, pad columns zero):
//   logits  (64 x 64 tiles)  S = scale qbar kbar^T into buffer 0, dP into buffer 1
//   softmax (a warp per row) P over buffer 0, dS over buffer 1, D from O_c
//   grads   (64 x d tiles)   dqbar, dkbar, dvbar: products over the C rows
// The two tile kernels are register-tiled SIMT GEMMs: 256 threads, 32-deep
// k chunks staged k-major in shared memory, each thread 4 rows x (BN/16)
// columns.  Float32 throughout: the sums are those of the definition, in
// float32 order.  The (b, h) planes run in chunks as large as the workspace.
#include <cmath>

#include "common.cuh"
#include "simt_tile.cuh"

namespace vsa {

namespace {

using simt::kChunk;
using simt::kThreads;
using simt::kTileM;
using simt::chunk_fma;
using simt::stage;
using simt::tile_col;

// out[i][j] = mul * sum_e A[i][e] B[j][e] for a 64 x 64 tile (A, B rows of d floats).
template <int D>
__device__ __forceinline__ void logits_tile(const float* __restrict__ A, const float* __restrict__ B,
                                            int C, int ldc, int i0, int j0, float mul,
                                            float* __restrict__ out, float* As, float* Bs) {
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int e0 = 0; e0 < D; e0 += kChunk) {
    __syncthreads();  // the previous chunk (or tile) is no longer read
    stage<kTileM, true>(As, A, D, i0, C, e0, D);
    stage<kTileM, true>(Bs, B, D, j0, C, e0, D);
    __syncthreads();
    chunk_fma<64>(As, Bs, tx, ty, acc);
  }
  // rows i < C; columns j0..j0+63 lie inside the padded row (j >= C are 0:
  // their operand rows were staged as zeros)
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int i = i0 + ty * 4 + r;
    if (i >= C) continue;
    float* row = out + static_cast<long long>(i) * ldc + j0 + tx * 4;
    *reinterpret_cast<float4*>(row) =
        make_float4(acc[r][0] * mul, acc[r][1] * mul, acc[r][2] * mul, acc[r][3] * mul);
  }
}

// grid (ldc/64 key tiles, ldc/64 query tiles, planes of this chunk).
template <int D>
__global__ void __launch_bounds__(kThreads) coarse_bwd_logits(
    int C, int ldc, const float* __restrict__ qb, const float* __restrict__ kb,
    const float* __restrict__ vb, const float* __restrict__ doc, float* __restrict__ sbuf,
    float* __restrict__ dpbuf) {
  __shared__ __align__(16) float As[kChunk * kTileM];
  __shared__ __align__(16) float Bs[kChunk * kTileM];
  const long long bh = blockIdx.z;
  const long long plane = bh * C * D;
  const long long mat = bh * C * static_cast<long long>(ldc);
  const int i0 = blockIdx.y * kTileM, j0 = blockIdx.x * kTileM;
  const float scale = 1.0f / sqrtf(static_cast<float>(D));
  logits_tile<D>(qb + plane, kb + plane, C, ldc, i0, j0, scale, sbuf + mat, As, Bs);
  logits_tile<D>(doc + plane, vb + plane, C, ldc, i0, j0, 1.0f, dpbuf + mat, As, Bs);
}

// grid (ceil(C/8), planes): one warp per row i.  Turns the row of S into P and
// the row of dP into dS in place; pad columns stay 0.
__global__ void __launch_bounds__(kThreads) coarse_bwd_softmax(
    int C, int ldc, int d, const float* __restrict__ oc, const float* __restrict__ doc,
    float* __restrict__ sbuf, float* __restrict__ dpbuf) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * (kThreads / 32) + warp;
  if (i >= C) return;  // whole warp
  const long long bh = blockIdx.y;
  const long long r = (bh * C + i) * static_cast<long long>(ldc);
  float* s = sbuf + r;
  float* dp = dpbuf + r;
  // online max and sum per lane, then merged across the warp
  float m = -INFINITY, z = 0.f;
  for (int j = lane; j < C; j += 32) {
    const float x = s[j];
    if (x > m) {
      z = z * expf(m - x) + 1.0f;  // m = -inf on the first element: z = 0 * 0 + 1
      m = x;
    } else {
      z += expf(x - m);
    }
  }
  for (int off = 16; off; off >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, off);
    const float z2 = __shfl_xor_sync(0xffffffffu, z, off);
    const float mn = fmaxf(m, m2);
    // a lane that saw no element has m = -inf, z = 0 and contributes nothing
    const float a = (m == -INFINITY) ? 0.f : z * expf(m - mn);
    const float b = (m2 == -INFINITY) ? 0.f : z2 * expf(m2 - mn);
    z = a + b;
    m = mn;
  }
  const long long orow = (bh * C + i) * static_cast<long long>(d);
  float D = 0.f;
  for (int e = lane; e < d; e += 32) D = fmaf(doc[orow + e], oc[orow + e], D);
  for (int off = 16; off; off >>= 1) D += __shfl_xor_sync(0xffffffffu, D, off);
  const float rz = 1.0f / z;
  for (int j = lane; j < C; j += 32) {
    const float p = expf(s[j] - m) * rz;
    const float g = p * (dp[j] - D);
    s[j] = p;
    dp[j] = g;
  }
}

// grid (ldc/64 row tiles, planes, 3): which = 0 dqbar = scale dS kbar,
// 1 dkbar = scale dS^T qbar, 2 dvbar = P^T dO_c; each a 64 x D tile summed over
// the C rows of the products' inner index.
template <int D>
__global__ void __launch_bounds__(kThreads) coarse_bwd_grads(
    int C, int ldc, const float* __restrict__ qb, const float* __restrict__ kb,
    const float* __restrict__ doc, const float* __restrict__ pbuf,
    const float* __restrict__ dsbuf, float* __restrict__ dq, float* __restrict__ dk,
    float* __restrict__ dv) {
  __shared__ __align__(16) float As[kChunk * kTileM];
  __shared__ __align__(16) float Bs[kChunk * D];
  const int which = blockIdx.z;
  const long long bh = blockIdx.y;
  const long long plane = bh * C * D;
  const long long mat = bh * C * static_cast<long long>(ldc);
  const int m0 = blockIdx.x * kTileM;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const float scale = 1.0f / sqrtf(static_cast<float>(D));
  const float* A = (which == 2 ? pbuf : dsbuf) + mat;
  const float* B = (which == 0 ? kb : which == 1 ? qb : doc) + plane;
  float* out = (which == 0 ? dq : which == 1 ? dk : dv) + plane;
  const float mul = which == 2 ? 1.0f : scale;
  float acc[4][D / 16] = {};
  for (int k0 = 0; k0 < C; k0 += kChunk) {
    __syncthreads();
    if (which == 0)  // A[i][j] = dS[i][j]: rows i, k = j contiguous (pads are 0)
      stage<kTileM, true>(As, A, ldc, m0, C, k0, C);
    else  // A[j][i] = dS[i][j] or P[i][j]: k = i indexes the rows
      stage<kTileM, false>(As, A, ldc, m0, C, k0, C);
    stage<D, false>(Bs, B, D, 0, D, k0, C);
    __syncthreads();
    chunk_fma<D>(As, Bs, tx, ty, acc);
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int m = m0 + ty * 4 + r;
    if (m >= C) continue;
    float* row = out + static_cast<long long>(m) * D;
#pragma unroll
    for (int g = 0; g < D / 64; ++g)
      *reinterpret_cast<float4*>(row + tile_col(tx, 4 * g)) =
          make_float4(acc[r][4 * g] * mul, acc[r][4 * g + 1] * mul, acc[r][4 * g + 2] * mul,
                      acc[r][4 * g + 3] * mul);
  }
}

template <int D>
cudaError_t run_chunk(int nbh, int C, int ldc, const float* qb, const float* kb, const float* vb,
                      const float* oc, const float* doc, float* dq, float* dk, float* dv,
                      float* sbuf, float* dpbuf, cudaStream_t s) {
  const int tiles = ldc / kTileM;
  coarse_bwd_logits<D><<<dim3(tiles, tiles, nbh), kThreads, 0, s>>>(C, ldc, qb, kb, vb, doc, sbuf,
                                                                   dpbuf);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  coarse_bwd_softmax<<<dim3((C + 7) / 8, nbh), kThreads, 0, s>>>(C, ldc, D, oc, doc, sbuf, dpbuf);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  coarse_bwd_grads<D><<<dim3(tiles, nbh, 3), kThreads, 0, s>>>(C, ldc, qb, kb, doc, sbuf, dpbuf,
                                                               dq, dk, dv);
  return cudaGetLastError();
}

}  // namespace

// Row stride of the workspace matrices and the bytes one (b, h) plane needs.
int coarse_backward_ldc(int C) { return (C + kTileM - 1) / kTileM * kTileM; }

size_t coarse_backward_plane_bytes(int C) {
  return 2ull * static_cast<size_t>(C) * coarse_backward_ldc(C) * sizeof(float);
}

cudaError_t launch_coarse_backward(int BH, int C, int d, const float* pooled, const float* oc,
                                   const float* doc, float* dpooled, void* workspace,
                                   size_t workspace_bytes, cudaStream_t s) {
  const int ldc = coarse_backward_ldc(C);
  const size_t per = coarse_backward_plane_bytes(C);
  const long long fit = static_cast<long long>(workspace_bytes / per);
  const int chunk = static_cast<int>(fit < BH ? fit : BH);
  if (chunk < 1) return cudaErrorInvalidValue;
  const long long plane = static_cast<long long>(BH) * C * d;
  for (int b0 = 0; b0 < BH; b0 += chunk) {
    const int nbh = BH - b0 < chunk ? BH - b0 : chunk;
    const long long off = static_cast<long long>(b0) * C * d;
    float* sbuf = static_cast<float*>(workspace);
    float* dpbuf = sbuf + static_cast<long long>(nbh) * C * ldc;
    const float* qb = pooled + off;
    const float* kb = pooled + plane + off;
    const float* vb = pooled + 2 * plane + off;
    float* dq = dpooled + off;
    float* dk = dpooled + plane + off;
    float* dv = dpooled + 2 * plane + off;
    cudaError_t err =
        d == 64 ? run_chunk<64>(nbh, C, ldc, qb, kb, vb, oc + off, doc + off, dq, dk, dv, sbuf, dpbuf, s)
                : run_chunk<128>(nbh, C, ldc, qb, kb, vb, oc + off, doc + off, dq, dk, dv, sbuf, dpbuf, s);
    if (err != cudaSuccess) return err;
  }
  return cudaSuccess;
}

}  // namespace vsa
