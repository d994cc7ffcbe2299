// Shared device/host helpers of the VSA library: cube geometry, status word
// reporting and the bounded barrier wait every kernel uses.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

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
};

// Valid tokens of cube c along each axis and in total.
__host__ __device__ inline void cube_extent(const Geom& g, int c, int& nt, int& ny, int& nx,
                                            int& t0, int& y0, int& x0) {
  int cx = c % g.Cx;
  int r = c / g.Cx;
  int cy = r % g.Cy;
  int ct = r / g.Cy;
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
