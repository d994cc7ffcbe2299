// Register-tiled float32 SIMT products shared by the backward kernels: a CTA
// of 256 threads computes a 64 x BN tile, each thread 4 rows x (BN/16)
// columns, summing over k in 32-deep chunks staged k-major in shared memory
// (dst[k][m], m contiguous) so every inner-loop read is a float4 that a
// quarter warp takes from 128 contiguous bytes or as a broadcast.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace vsa {
namespace simt {

constexpr int kThreads = 256;
constexpr int kTileM = 64;  // rows of an output tile
constexpr int kChunk = 32;  // k per staged chunk

// Four consecutive elements as floats (16-byte load of float, 8-byte load of bf16).
__device__ __forceinline__ float4 load4(const float* p) {
  return __ldg(reinterpret_cast<const float4*>(p));
}
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
  const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                     __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u));
}

// One operand chunk into shared memory, k-major: dst[k][m] for k < 32, m < W.
// kKContig: element (m, k) at src[m * ld + k]  (valid while m0 + m < mlim;
//           k stays inside the row by construction)
// else:     element (m, k) at src[k * ld + m]  (valid while k0 + k < klim)
// Invalid elements load as 0.  Every vector read is aligned: ld, the chunk
// start and the tile start are multiples of 4 elements.
template <int W, bool kKContig, typename T>
__device__ __forceinline__ void stage(float* dst, const T* __restrict__ src, int ld, int m0,
                                      int mlim, int k0, int klim) {
  if constexpr (kKContig) {
    // W rows x 8 groups of 4 k; consecutive threads take consecutive rows so
    // the transposed shared-memory stores hit consecutive banks
    for (int idx = threadIdx.x; idx < W * (kChunk / 4); idx += kThreads) {
      const int m = idx % W, kq = idx / W;
      float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
      if (m0 + m < mlim) x = load4(src + static_cast<long long>(m0 + m) * ld + k0 + 4 * kq);
      dst[(4 * kq + 0) * W + m] = x.x;
      dst[(4 * kq + 1) * W + m] = x.y;
      dst[(4 * kq + 2) * W + m] = x.z;
      dst[(4 * kq + 3) * W + m] = x.w;
    }
  } else {
    // 32 rows of k x W/4 groups of m: coalesced reads, float4 stores
    for (int idx = threadIdx.x; idx < kChunk * (W / 4); idx += kThreads) {
      const int m4 = idx % (W / 4), k = idx / (W / 4);
      float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
      if (k0 + k < klim) x = load4(src + static_cast<long long>(k0 + k) * ld + m0 + 4 * m4);
      *reinterpret_cast<float4*>(&dst[k * W + 4 * m4]) = x;
    }
  }
}

// A whole 64-row operand of width K (k = 0 .. K-1) into dst[k][m], k-major:
// element (m, k) at src[(m0 + m) * ld + k], rows m0 + m >= mlim as 0.
template <typename T>
__device__ __forceinline__ void stage_rows_t(float* dst, const T* __restrict__ src, int ld,
                                             int m0, int mlim, int K) {
  for (int idx = threadIdx.x; idx < kTileM * (K / 4); idx += kThreads) {
    const int m = idx % kTileM, kq = idx / kTileM;
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (m0 + m < mlim) x = load4(src + static_cast<long long>(m0 + m) * ld + 4 * kq);
    dst[(4 * kq + 0) * kTileM + m] = x.x;
    dst[(4 * kq + 1) * kTileM + m] = x.y;
    dst[(4 * kq + 2) * kTileM + m] = x.z;
    dst[(4 * kq + 3) * kTileM + m] = x.w;
  }
}

// Column of the c-th accumulator of thread tx in a BN-wide tile: two float4
// groups 64 apart when BN = 128, so a quarter warp reads 128 contiguous bytes.
__device__ __forceinline__ int tile_col(int tx, int c) { return (c >> 2) * 64 + tx * 4 + (c & 3); }

// acc[r][c] += sum over the chunk of As[k][ty*4 + r] * Bs[k][tile_col(tx, c)],
// As with row stride lda (kTileM unless given), Bs with row stride BN.
template <int BN>
__device__ __forceinline__ void chunk_fma(const float* As, const float* Bs, int tx, int ty,
                                          float (&acc)[4][BN / 16], int lda = kTileM) {
#pragma unroll 8
  for (int k = 0; k < kChunk; ++k) {
    const float4 a = *reinterpret_cast<const float4*>(&As[k * lda + ty * 4]);
    const float av[4] = {a.x, a.y, a.z, a.w};
    float bv[BN / 16];
#pragma unroll
    for (int g = 0; g < BN / 64; ++g) {
      const float4 b = *reinterpret_cast<const float4*>(&Bs[k * BN + g * 64 + tx * 4]);
      bv[4 * g] = b.x; bv[4 * g + 1] = b.y; bv[4 * g + 2] = b.z; bv[4 * g + 3] = b.w;
    }
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < BN / 16; ++c) acc[r][c] = fmaf(av[r], bv[c], acc[r][c]);
  }
}

}  // namespace simt
}  // namespace vsa
