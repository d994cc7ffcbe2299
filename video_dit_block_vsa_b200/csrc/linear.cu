// Low-rank linear compensation branch summed with the block-sparse output
// (the sparse + linear variant: the SparkDiffusion page's RoLA, a block-sparse
// branch plus a low-rank linear branch that keeps the global context; the
// TurboDiffusion review's sparse-linear attention).  Reading taken: linear
// attention over every token of the (b, h) sequence with the positive feature
// map phi(x) = elu(x) + 1,
//   O_lin[r] = phi(q_r)^T KV / phi(q_r)^T z,  KV = sum_t phi(k_t) v_t^T,
//   z = sum_t phi(k_t),
// added to the block-sparse output in token order.
//
// Three passes, all float32, deterministic (fixed summation order):
//   1. linear_kv_kernel      grid (S, B*H): partial KV and z over one of S
//                            token chunks of a sequence (64 x d register
//                            tiles of phi(K_chunk)^T V_chunk, both halves of
//                            KV's rows for d = 128);
//   2. linear_reduce_kernel  grid (B*H): the S partials summed in order;
//   3. linear_apply_kernel   grid (ceil(N/64), B*H): 64 tokens x d outputs of
//                            phi(Q) KV, divided by phi(Q) z, added to out.
// The products are the register-tiled float32 products of simt_tile.cuh over
// 32-deep chunks staged in shared memory.
#include "common.cuh"
#include "simt_tile.cuh"

namespace vsa {

namespace {

using simt::kChunk;
using simt::kThreads;
using simt::kTileM;
using simt::chunk_fma;
using simt::load4;
using simt::tile_col;
using bf16 = __nv_bfloat16;

__device__ __forceinline__ float phi(float x) { return x > 0.f ? x + 1.f : __expf(x); }

// rows [t0, t0 + kChunk) of a [N, D] bf16 sequence into dst[t][e] (row-major,
// D floats per row), phi applied if kPhi; rows at or past N are zero.
template <int D, bool kPhi>
__device__ __forceinline__ void stage_rows(float* dst, const bf16* __restrict__ src, long long N,
                                           long long t0) {
  for (int idx = threadIdx.x; idx < kChunk * (D / 4); idx += kThreads) {
    const int t = idx / (D / 4), e4 = idx - t * (D / 4);
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    const long long row = t0 + t;
    if (row < N) {
      x = load4(src + row * D + 4 * e4);
      if (kPhi) {
        x.x = phi(x.x);
        x.y = phi(x.y);
        x.z = phi(x.z);
        x.w = phi(x.w);
      }
    }
    *reinterpret_cast<float4*>(&dst[t * D + 4 * e4]) = x;
  }
}

// Partials of one token chunk: ws[(bh * S + s)] holds KV (D x D, row a =
// feature of phi(k), column e = value dim) then z (D).
template <int D>
__global__ void __launch_bounds__(kThreads) linear_kv_kernel(long long N, int S,
                                                             const bf16* __restrict__ k,
                                                             const bf16* __restrict__ v,
                                                             float* __restrict__ ws) {
  __shared__ __align__(16) float fk[kChunk * D];  // phi(k) rows: fk[t][a]
  __shared__ __align__(16) float vs[kChunk * D];  // v rows:      vs[t][e]
  const int s = blockIdx.x;
  const long long bh = blockIdx.y;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const long long per = (N + S - 1) / S;
  const long long lo = min(N, s * per), hi = min(N, lo + per);
  const bf16* kb = k + bh * N * D;
  const bf16* vb = v + bh * N * D;
  constexpr int kRowTiles = D / kTileM;  // 64-row tiles of KV
  float acc[kRowTiles][4][D / 16] = {};
  float zacc = 0.f;  // z[threadIdx.x] for threads < D
  for (long long t0 = lo; t0 < hi; t0 += kChunk) {
    __syncthreads();  // previous chunk consumed
    stage_rows<D, true>(fk, kb, hi, t0);
    stage_rows<D, false>(vs, vb, hi, t0);
    __syncthreads();
    // KV[a][e] += sum_t fk[t][a] vs[t][e]: As = fk (k-major over t, a contiguous)
#pragma unroll
    for (int rt = 0; rt < kRowTiles; ++rt) chunk_fma<D>(fk + rt * kTileM, vs, tx, ty, acc[rt], D);
    if (threadIdx.x < D) {
#pragma unroll 8
      for (int t = 0; t < kChunk; ++t) zacc += fk[t * D + threadIdx.x];
    }
  }
  float* out = ws + (bh * S + s) * (static_cast<long long>(D) * D + D);
#pragma unroll
  for (int rt = 0; rt < kRowTiles; ++rt)
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < D / 16; ++c)
        out[static_cast<long long>(rt * kTileM + ty * 4 + r) * D + tile_col(tx, c)] = acc[rt][r][c];
  if (threadIdx.x < D) out[static_cast<long long>(D) * D + threadIdx.x] = zacc;
}

// kv[bh] = sum over s = 0 .. S-1 of the partials, in that order.
template <int D>
__global__ void __launch_bounds__(kThreads) linear_reduce_kernel(int S, const float* __restrict__ ws,
                                                                 float* __restrict__ kv) {
  constexpr long long kPer = static_cast<long long>(D) * D + D;
  const long long bh = blockIdx.x;
  const float* src = ws + bh * S * kPer;
  float* dst = kv + bh * kPer;
  for (long long e = threadIdx.x; e < kPer; e += blockDim.x) {
    float t = 0.f;
    for (int s = 0; s < S; ++s) t += src[s * kPer + e];
    dst[e] = t;
  }
}

// out[r] = bf16(out[r] + phi(q_r)^T KV / phi(q_r)^T z) for 64 tokens of one (b, h).
template <int D>
__global__ void __launch_bounds__(kThreads) linear_apply_kernel(long long N,
                                                                const bf16* __restrict__ q,
                                                                const float* __restrict__ kv,
                                                                bf16* __restrict__ out) {
  __shared__ __align__(16) float fq[kChunk * kTileM];  // phi(q) chunk, k-major: fq[a][r]
  __shared__ __align__(16) float ks[kChunk * D];       // KV rows a of the chunk: ks[a][e]
  __shared__ __align__(16) float zs[D];
  const long long bh = blockIdx.y;
  const long long r0 = static_cast<long long>(blockIdx.x) * kTileM;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const bf16* qb = q + bh * N * D;
  const float* kvb = kv + bh * (static_cast<long long>(D) * D + D);
  if (threadIdx.x < D) zs[threadIdx.x] = kvb[static_cast<long long>(D) * D + threadIdx.x];
  float acc[4][D / 16] = {};
  float den[4] = {0.f, 0.f, 0.f, 0.f};
  for (int a0 = 0; a0 < D; a0 += kChunk) {
    __syncthreads();  // previous chunk consumed (and zs written)
    // phi(q) rows r0 .. r0+63, features a0 .. a0+31, transposed to fq[a][r]
    for (int idx = threadIdx.x; idx < kTileM * (kChunk / 4); idx += kThreads) {
      const int r = idx % kTileM, a4 = idx / kTileM;
      float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r0 + r < N) {
        x = load4(qb + (r0 + r) * D + a0 + 4 * a4);
        x.x = phi(x.x);
        x.y = phi(x.y);
        x.z = phi(x.z);
        x.w = phi(x.w);
      }
      fq[(4 * a4 + 0) * kTileM + r] = x.x;
      fq[(4 * a4 + 1) * kTileM + r] = x.y;
      fq[(4 * a4 + 2) * kTileM + r] = x.z;
      fq[(4 * a4 + 3) * kTileM + r] = x.w;
    }
    for (int idx = threadIdx.x; idx < kChunk * (D / 4); idx += kThreads) {
      const int a = idx / (D / 4), e4 = idx - a * (D / 4);
      *reinterpret_cast<float4*>(&ks[a * D + 4 * e4]) =
          *reinterpret_cast<const float4*>(&kvb[static_cast<long long>(a0 + a) * D + 4 * e4]);
    }
    __syncthreads();
    chunk_fma<D>(fq, ks, tx, ty, acc);
#pragma unroll 8
    for (int a = 0; a < kChunk; ++a) {
      const float4 f = *reinterpret_cast<const float4*>(&fq[a * kTileM + ty * 4]);
      const float za = zs[a0 + a];
      den[0] = fmaf(f.x, za, den[0]);
      den[1] = fmaf(f.y, za, den[1]);
      den[2] = fmaf(f.z, za, den[2]);
      den[3] = fmaf(f.w, za, den[3]);
    }
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const long long row = r0 + ty * 4 + r;
    if (row >= N) continue;
    const float inv = 1.0f / den[r];
    bf16* o = out + (bh * N + row) * D;
#pragma unroll
    for (int grp = 0; grp < D / 64; ++grp) {
      const int col = tile_col(tx, 4 * grp);
      const uint2 old = *reinterpret_cast<const uint2*>(o + col);
      const float f[4] = {__uint_as_float(old.x << 16), __uint_as_float(old.x & 0xFFFF0000u),
                          __uint_as_float(old.y << 16), __uint_as_float(old.y & 0xFFFF0000u)};
      __nv_bfloat162 lo2 = __floats2bfloat162_rn(fmaf(acc[r][4 * grp + 0], inv, f[0]),
                                                 fmaf(acc[r][4 * grp + 1], inv, f[1]));
      __nv_bfloat162 hi2 = __floats2bfloat162_rn(fmaf(acc[r][4 * grp + 2], inv, f[2]),
                                                 fmaf(acc[r][4 * grp + 3], inv, f[3]));
      *reinterpret_cast<uint2*>(o + col) =
          make_uint2(*reinterpret_cast<uint32_t*>(&lo2), *reinterpret_cast<uint32_t*>(&hi2));
    }
  }
}

}  // namespace

// Token chunks per sequence for the partial sums: about 296 CTAs in all (two
// per SM of a B200), at least 256 tokens per chunk.  Fixed, so that the
// workspace size does not depend on the device.
int linear_splits(int bh, long long N) {
  long long S = (296ll + bh - 1) / bh;
  S = S < 1 ? 1 : S;
  const long long most = (N + 255) / 256;
  if (S > most) S = most;
  return static_cast<int>(S < 1 ? 1 : S);
}

size_t linear_workspace_floats(int bh, long long N, int d) {
  const long long per = static_cast<long long>(d) * d + d;
  return static_cast<size_t>(bh) * (linear_splits(bh, N) + 1) * per;
}

cudaError_t launch_linear_branch(int bh, long long N, int d, const void* q, const void* k,
                                 const void* v, void* out, float* ws, cudaStream_t s) {
  const int S = linear_splits(bh, N);
  const long long per = static_cast<long long>(d) * d + d;
  float* partial = ws;
  float* kv = ws + static_cast<long long>(bh) * S * per;
  auto b = [](const void* p) { return static_cast<const bf16*>(p); };
  const dim3 apply_grid(static_cast<unsigned>((N + kTileM - 1) / kTileM), bh);
  if (d == 128) {
    linear_kv_kernel<128><<<dim3(S, bh), kThreads, 0, s>>>(N, S, b(k), b(v), partial);
    linear_reduce_kernel<128><<<bh, kThreads, 0, s>>>(S, partial, kv);
    linear_apply_kernel<128><<<apply_grid, kThreads, 0, s>>>(N, b(q), kv, static_cast<bf16*>(out));
  } else {
    linear_kv_kernel<64><<<dim3(S, bh), kThreads, 0, s>>>(N, S, b(k), b(v), partial);
    linear_reduce_kernel<64><<<bh, kThreads, 0, s>>>(S, partial, kv);
    linear_apply_kernel<64><<<apply_grid, kThreads, 0, s>>>(N, b(q), kv, static_cast<bf16*>(out));
  }
  return cudaGetLastError();
}

}  // namespace vsa
