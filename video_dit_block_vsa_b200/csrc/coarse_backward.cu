// Backward of the coarse attention O_c = softmax(qbar kbar^T / sqrt(d)) vbar
// (float32, per (b, h), over the C pooled vectors): the coarse branch of a VSA
// backward pass.  With P the softmax, dO_c the incoming gradient and
// scale = 1/sqrt(d):
//   D_i   = <dO_c[i], O_c[i]>
//   dS_ij = P_ij (<dO_c[i], vbar[j]> - D_i)
//   dqbar[i] = scale sum_j dS_ij kbar[j]
//   dkbar[j] = scale sum_i dS_ij qbar[i],   dvbar[j] = sum_i P_ij dO_c[i]
//
// Two passes, no C x C matrix in memory:
//   rows    (one CTA per query cube i): the row of logits in shared memory,
//           its max m_i and 1/z_i, D_i, the row of dS, then dqbar[i];
//           m, 1/z and D go to a 3*B*H*C float scratch.
//   columns (one CTA per key cube j): recomputes column j of P from the saved
//           m and 1/z with the same float arithmetic (so P is bit-identical
//           to the rows pass), forms column j of dS, then dkbar[j], dvbar[j].
// Each thread takes whole dot products of length d (float4 loads of one row);
// the weighted sums over rows run with consecutive threads on consecutive
// elements of a row, so those loads are coalesced.
#include <cmath>

#include "common.cuh"

namespace vsa {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float block_reduce(float v, float* red, bool is_max) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int off = 16; off; off >>= 1) {
    const float o = __shfl_xor_sync(0xffffffffu, v, off);
    v = is_max ? fmaxf(v, o) : v + o;
  }
  __syncthreads();  // red[] may still be read from the previous reduction
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = red[0];
  for (int w = 1; w < kThreads / 32; ++w) r = is_max ? fmaxf(r, red[w]) : r + red[w];
  return r;
}

// <a, row> over d elements: a in shared memory, row in global memory (16-byte aligned).
__device__ __forceinline__ float dot_row(const float* a, const float* __restrict__ row, int d) {
  const float4* r4 = reinterpret_cast<const float4*>(row);
  float s = 0.f;
  for (int e = 0; e < (d >> 2); ++e) {
    const float4 x = __ldg(&r4[e]);
    s = fmaf(a[4 * e], x.x, s);
    s = fmaf(a[4 * e + 1], x.y, s);
    s = fmaf(a[4 * e + 2], x.z, s);
    s = fmaf(a[4 * e + 3], x.w, s);
  }
  return s;
}

// out[e] = mul * sum_{r < n} w[r] M[r, e] for e < d (w in shared memory, M global
// [n][d]).  kThreads/d row groups sum interleaved rows; part[] combines them.
// Must be called by the whole block; out is written by threads e < d.
__device__ __forceinline__ void weighted_rows(const float* w, const float* __restrict__ M, int n,
                                              int d, float mul, float* part,
                                              float* __restrict__ out) {
  const int groups = kThreads / d;
  const int e = threadIdx.x % d, grp = threadIdx.x / d;
  float acc = 0.f;
  if (grp < groups)
    for (int r = grp; r < n; r += groups) acc = fmaf(w[r], __ldg(&M[static_cast<long long>(r) * d + e]), acc);
  __syncthreads();  // part[] may still be read from the previous call
  part[threadIdx.x] = acc;
  __syncthreads();
  if (threadIdx.x < d) {
    float s = 0.f;
    for (int g = 0; g < groups; ++g) s += part[g * d + threadIdx.x];
    out[threadIdx.x] = s * mul;
  }
}

// grid (C, B*H).  Dynamic smem: qbar[i], dO_c[i] (d floats each), w[C].
__global__ void __launch_bounds__(kThreads) coarse_bwd_rows(
    int C, int d, const float* __restrict__ qb, const float* __restrict__ kb,
    const float* __restrict__ vb, const float* __restrict__ oc, const float* __restrict__ doc,
    float* __restrict__ dqb, float* __restrict__ row_max, float* __restrict__ row_rz,
    float* __restrict__ row_D) {
  extern __shared__ float sm[];
  float* qi = sm;
  float* gi = sm + d;
  float* w = sm + 2 * d;
  __shared__ float red[kThreads / 32];
  __shared__ float part[kThreads];
  const int i = blockIdx.x;
  const long long bh = blockIdx.y;
  const long long base = bh * C * static_cast<long long>(d);
  const long long row_i = base + static_cast<long long>(i) * d;
  const float scale = 1.0f / sqrtf(static_cast<float>(d));
  float dpart = 0.f;
  for (int e = threadIdx.x; e < d; e += kThreads) {
    qi[e] = qb[row_i + e];
    gi[e] = doc[row_i + e];
    dpart = fmaf(gi[e], oc[row_i + e], dpart);
  }
  const float D = block_reduce(dpart, red, false);  // its barriers publish qi, gi
  float mx = -INFINITY;
  for (int j = threadIdx.x; j < C; j += kThreads) {
    const float s = dot_row(qi, kb + base + static_cast<long long>(j) * d, d) * scale;
    w[j] = s;
    mx = fmaxf(mx, s);
  }
  mx = block_reduce(mx, red, true);
  float z = 0.f;
  for (int j = threadIdx.x; j < C; j += kThreads) {
    const float p = expf(w[j] - mx);
    w[j] = p;
    z += p;
  }
  z = block_reduce(z, red, false);
  const float rz = 1.0f / z;
  for (int j = threadIdx.x; j < C; j += kThreads) {
    const float p = w[j] * rz;
    const float dp = dot_row(gi, vb + base + static_cast<long long>(j) * d, d);
    w[j] = p * (dp - D);  // dS_ij
  }
  __syncthreads();
  weighted_rows(w, kb + base, C, d, scale, part, dqb + row_i);
  if (threadIdx.x == 0) {
    const long long r = bh * C + i;
    row_max[r] = mx;
    row_rz[r] = rz;
    row_D[r] = D;
  }
}

// grid (C, B*H).  Dynamic smem: kbar[j], vbar[j] (d floats each), p[C], ds[C].
__global__ void __launch_bounds__(kThreads) coarse_bwd_cols(
    int C, int d, const float* __restrict__ qb, const float* __restrict__ kb,
    const float* __restrict__ vb, const float* __restrict__ doc, const float* __restrict__ row_max,
    const float* __restrict__ row_rz, const float* __restrict__ row_D, float* __restrict__ dkb,
    float* __restrict__ dvb) {
  extern __shared__ float sm[];
  float* kj = sm;
  float* vj = sm + d;
  float* p = sm + 2 * d;
  float* ds = p + C;
  __shared__ float part[kThreads];
  const int j = blockIdx.x;
  const long long bh = blockIdx.y;
  const long long base = bh * C * static_cast<long long>(d);
  const long long row_j = base + static_cast<long long>(j) * d;
  const float scale = 1.0f / sqrtf(static_cast<float>(d));
  for (int e = threadIdx.x; e < d; e += kThreads) {
    kj[e] = kb[row_j + e];
    vj[e] = vb[row_j + e];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < C; i += kThreads) {
    const long long r = bh * C + i;
    // same operands and order as the rows pass: fmaf(a, b, c) == fmaf(b, a, c)
    const float s = dot_row(kj, qb + base + static_cast<long long>(i) * d, d) * scale;
    const float pij = expf(s - row_max[r]) * row_rz[r];
    const float dp = dot_row(vj, doc + base + static_cast<long long>(i) * d, d);
    p[i] = pij;
    ds[i] = pij * (dp - row_D[r]);
  }
  __syncthreads();
  weighted_rows(ds, qb + base, C, d, scale, part, dkb + row_j);
  weighted_rows(p, doc + base, C, d, 1.0f, part, dvb + row_j);
}

}  // namespace

size_t coarse_backward_smem_bytes(int C, int d) {
  return static_cast<size_t>(2 * d + 2 * C) * sizeof(float);
}

cudaError_t launch_coarse_backward(int BH, int C, int d, const float* pooled, const float* oc,
                                   const float* doc, float* dpooled, float* stats,
                                   cudaStream_t s) {
  static unsigned long long rows_set = 0, cols_set = 0;
  const int most = static_cast<int>(coarse_backward_smem_bytes(kMaxCubes, 128));
  cudaError_t err = smem_limit_once(coarse_bwd_rows, most, &rows_set);
  if (err != cudaSuccess) return err;
  err = smem_limit_once(coarse_bwd_cols, most, &cols_set);
  if (err != cudaSuccess) return err;
  const long long plane = static_cast<long long>(BH) * C * d;
  const float* qb = pooled;
  const float* kb = pooled + plane;
  const float* vb = pooled + 2 * plane;
  float* row_max = stats;
  float* row_rz = stats + static_cast<long long>(BH) * C;
  float* row_D = stats + 2 * static_cast<long long>(BH) * C;
  const dim3 grid(C, BH);
  const size_t rows_smem = static_cast<size_t>(2 * d + C) * sizeof(float);
  coarse_bwd_rows<<<grid, kThreads, rows_smem, s>>>(C, d, qb, kb, vb, oc, doc, dpooled, row_max,
                                                    row_rz, row_D);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  coarse_bwd_cols<<<grid, kThreads, coarse_backward_smem_bytes(C, d), s>>>(
      C, d, qb, kb, vb, doc, row_max, row_rz, row_D, dpooled + plane, dpooled + 2 * plane);
  return cudaGetLastError();
}

}  // namespace vsa
