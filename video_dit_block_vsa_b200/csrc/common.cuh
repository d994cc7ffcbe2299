// Shared device/host helpers of the VSA library: cube geometry, status word
// reporting and the bounded barrier wait every kernel uses.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "ctx_cache.h"
#include "vsa.h"

namespace vsa {

constexpr int kSlots = 64;          // tokens per 4x4x4 cube
constexpr int kMaxCubes = 8192;     // coarse stage keeps one logits row per query cube in smem
constexpr uint64_t kWaitNs = 4000000000ull;  // bound on any in-kernel wait (4 s)

// Geometry of the cube tiling, passed by value to every kernel.
struct Geom {
  int B, H, d;
  int T, Y, X;       // grid
  int Ct, Cy, Cx;    // cubes per axis
  int C;             // cubes
  long long N;       // tokens
  long long rows;    // 64*C tiled rows per (b, h)
  uint64_t inv_cx;   // ceil(2^32 / Cx): for n, Cx < 2^16, n / Cx == (n * inv_cx) >> 32
  uint64_t inv_cy;   // ceil(2^32 / Cy)
};

// Division by a runtime divisor below 2^16 for dividends below 2^16, with the
// precomputed reciprocal inv = ceil(2^32 / d): n * inv / 2^32 = n / d + n e / (d 2^32)
// with 0 <= e < d, and the second term stays below 1/d when n e < 2^32.
__host__ __device__ inline uint32_t div_small(uint32_t n, uint64_t inv) {
  return static_cast<uint32_t>((static_cast<uint64_t>(n) * inv) >> 32);
}

// Valid tokens of cube c along each axis and in total.
__host__ __device__ inline void cube_extent(const Geom& g, int c, int& nt, int& ny, int& nx,
                                            int& t0, int& y0, int& x0) {
  // c < kMaxCubes < 2^16, so the divisions by Cx and Cy use the reciprocals
  const int r = static_cast<int>(div_small(static_cast<uint32_t>(c), g.inv_cx));
  const int cx = c - r * g.Cx;
  const int ct = static_cast<int>(div_small(static_cast<uint32_t>(r), g.inv_cy));
  const int cy = r - ct * g.Cy;
  t0 = ct * 4; y0 = cy * 4; x0 = cx * 4;
  nt = min(4, g.T - t0);
  ny = min(4, g.Y - y0);
  nx = min(4, g.X - x0);
}

__host__ __device__ inline int cube_valid(const Geom& g, int c) {
  int nt, ny, nx, t0, y0, x0;
  cube_extent(g, c, nt, ny, nx, t0, y0, x0);
  return nt * ny * nx;
}

// Token index held by slot s of cube c, or -1 for a pad slot.
__device__ __forceinline__ long long slot_token(const Geom& g, int c, int s) {
  int nt, ny, nx, t0, y0, x0;
  cube_extent(g, c, nt, ny, nx, t0, y0, x0);
  int lt, ly, lx;
  if ((nt & ny & nx) == 4) {  // full cube: slot s = 16 lt + 4 ly + lx
    lt = s >> 4;
    ly = (s >> 2) & 3;
    lx = s & 3;
  } else {
    const int nyx = ny * nx;
    if (s >= nt * nyx) return -1;
    lt = s / nyx;
    const int rem = s - lt * nyx;
    ly = rem / nx;
    lx = rem - ly * nx;
  }
  return (static_cast<long long>(t0 + lt) * g.Y + (y0 + ly)) * g.X + (x0 + lx);
}

// Unique id of the CUDA context current on this thread; if none is current,
// the current device's primary context is made current first.  0 if it
// cannot be determined.  Values cached per context (CtxCache) use it as key.
uint64_t current_context_id();

// Raises a kernel's dynamic shared-memory limit once per CUDA context, so
// that later launches, including launches made while a stream is being
// captured into a CUDA graph, only launch.  The attribute belongs to the
// context, so a new context (after cudaDeviceReset, or one the caller made
// current) gets it raised again.
template <typename Kernel>
inline cudaError_t smem_limit_once(Kernel kernel, int bytes, CtxCache<char>* done) {
  cudaError_t err = cudaSuccess;
  char ok = 0;
  const bool got = done->get(current_context_id(), [&](char* v) {
    err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    *v = 1;
    return err == cudaSuccess;
  }, &ok);
  if (got) return cudaSuccess;
  return err != cudaSuccess ? err : cudaErrorInvalidValue;
}

// Record a device-side condition in the status word (first one wins).
__device__ inline void report(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ inline uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

}  // namespace vsa
