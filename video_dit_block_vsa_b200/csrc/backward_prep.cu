// First pass of a VSA backward: the gradient of the gated combine, taken to
// the layouts the attention backward kernels read, in one pass over dout.
//
// For out[n] = g_f[n] O_f[n] + g_c[n] O_c[cube(n)] (or out = O_f ungated):
//   dO_f[r]  = bf16(g_f[n] dout[n])  tiled (pad rows 0)   - fine-branch gradient
//   D[r]     = sum_e dO_f[r, e] O_f[r, e]  (float32)      - softmax backward term
//   dO_c[c]  = sum over the cube's valid rows of g_c[n] dout[n]
//   dg_f[n]  = <dout[n], O_f[r]>,  dg_c[n] = <dout[n], O_c[c]>
// where r is the tiled row of token n and c its cube.  The selection is held
// fixed, as in the forward (a discrete choice passes no gradient).
//
// One warp per (b*h, cube), as the pooling pass: a row of d bf16 is d/8
// 16-byte chunks, the warp covers 32/(d/8) rows per step, row sums reduce
// over the lanes of a row and the dO_c sums over the rows at the end.
#include "common.cuh"

namespace vsa {

namespace {

__device__ __forceinline__ float lo_bf16(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_bf16(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&p);
}

__global__ void __launch_bounds__(256) backward_prep_kernel(
    Geom g, const uint4* __restrict__ dout, const uint4* __restrict__ of,
    const float* __restrict__ oc, const float* __restrict__ gf, const float* __restrict__ gc,
    uint4* __restrict__ dof, float* __restrict__ delta, float* __restrict__ doc,
    float* __restrict__ dgf, float* __restrict__ dgc) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long item = static_cast<long long>(blockIdx.x) * 8 + warp;  // (b*h, cube)
  if (item >= static_cast<long long>(g.B) * g.H * g.C) return;
  const long long bh = item / g.C;
  const int c = static_cast<int>(item - bh * g.C);
  const int n_c = cube_valid(g, c);
  const int chunks = g.d >> 3;            // 8 or 16 chunks of 8 values per row
  const int rows_per_step = 32 / chunks;  // 4 or 2
  const int ch = lane % chunks;
  const int r0 = lane / chunks;
  const bool gated = gf != nullptr;
  const long long row_base = bh * g.rows + static_cast<long long>(c) * kSlots;

  float occ[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // this lane's slice of O_c[c]
  if (gated) {
    const float4* src = reinterpret_cast<const float4*>(oc + (bh * g.C + c) * g.d + ch * 8);
    const float4 a = __ldg(&src[0]), b = __ldg(&src[1]);
    occ[0] = a.x; occ[1] = a.y; occ[2] = a.z; occ[3] = a.w;
    occ[4] = b.x; occ[5] = b.y; occ[6] = b.z; occ[7] = b.w;
  }
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // dO_c partial sums
  // every lane runs the same number of steps (the shuffles below need the
  // whole warp); pad rows take zero values and write zeros
  for (int r = r0; r < kSlots; r += rows_per_step) {
    const long long row = row_base + r;
    const bool valid = r < n_c;
    long long tok = 0;
    uint32_t wu[4] = {0u, 0u, 0u, 0u}, ou[4] = {0u, 0u, 0u, 0u};
    float wf = 1.f, wc = 0.f;
    if (valid) {
      tok = bh * g.N + slot_token(g, c, r);
      const uint4 w = __ldg(&dout[tok * chunks + ch]);
      const uint4 o = __ldg(&of[row * chunks + ch]);
      wu[0] = w.x; wu[1] = w.y; wu[2] = w.z; wu[3] = w.w;
      ou[0] = o.x; ou[1] = o.y; ou[2] = o.z; ou[3] = o.w;
      if (gated) {
        wf = __ldg(&gf[tok]);
        wc = __ldg(&gc[tok]);
      }
    }
    uint32_t du[4];
    float dsum = 0.f, fsum = 0.f, csum = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float d0 = lo_bf16(wu[e]), d1 = hi_bf16(wu[e]);
      const float o0 = lo_bf16(ou[e]), o1 = hi_bf16(ou[e]);
      du[e] = gated ? pack_bf16x2(wf * d0, wf * d1) : wu[e];
      dsum = fmaf(lo_bf16(du[e]), o0, fmaf(hi_bf16(du[e]), o1, dsum));
      fsum = fmaf(d0, o0, fmaf(d1, o1, fsum));
      csum = fmaf(d0, occ[2 * e], fmaf(d1, occ[2 * e + 1], csum));
      acc[2 * e] = fmaf(wc, d0, acc[2 * e]);
      acc[2 * e + 1] = fmaf(wc, d1, acc[2 * e + 1]);
    }
    dof[row * chunks + ch] = make_uint4(du[0], du[1], du[2], du[3]);
    // row sums over the `chunks` lanes of this row (they are adjacent lanes)
    for (int off = 1; off < chunks; off <<= 1) {
      dsum += __shfl_xor_sync(0xffffffffu, dsum, off);
      fsum += __shfl_xor_sync(0xffffffffu, fsum, off);
      csum += __shfl_xor_sync(0xffffffffu, csum, off);
    }
    if (ch == 0) {
      delta[row] = dsum;  // 0 on pad rows
      if (gated && valid) {
        dgf[tok] = fsum;
        dgc[tok] = csum;
      }
    }
  }
  if (!gated) return;
  for (int off = chunks; off < 32; off <<= 1) {  // over the row groups
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
  }
  if (r0 == 0) {
    float4* dst = reinterpret_cast<float4*>(doc + (bh * g.C + c) * g.d + ch * 8);
    dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
}

}  // namespace

cudaError_t launch_backward_prep(const Geom& g, const void* dout, const void* of,
                                 const float* oc, const float* gf, const float* gc, void* dof,
                                 float* delta, float* doc, float* dgf, float* dgc,
                                 cudaStream_t s) {
  const long long items = static_cast<long long>(g.B) * g.H * g.C;
  backward_prep_kernel<<<static_cast<unsigned>((items + 7) / 8), 256, 0, s>>>(
      g, static_cast<const uint4*>(dout), static_cast<const uint4*>(of), oc, gf, gc,
      static_cast<uint4*>(dof), delta, doc, dgf, dgc);
  return cudaGetLastError();
}

}  // namespace vsa
