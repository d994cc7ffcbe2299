// Backward of the fine block-sparse attention, with the pooling and untile
// steps of the backward folded into the epilogues.  For query cube i, its
// selected key cubes j (the forward's selection, held fixed) and
// scale = 1/sqrt(d), per 64 x 64 block (rows r of cube i, keys c of cube j):
//   P  = exp(scale Q_i K_j^T - lse_i)      (the forward's natural-log LSE;
//                                            0 on pad rows and pad keys)
//   dP = dO_i V_j^T,   dS = P (dP - D_i)   (dO_i = tiled dO_f, D = rowsum(dO_f O_f),
//                                            both from the combine-gradient pass)
//   dQ_i += scale dS K_j,   dK_j += scale dS^T Q_i,   dV_j += P^T dO_i
// and the gradient of the cube means reaches every valid row of the cube:
//   dq[r] = dQ_i[r] + dqbar[i] / n_i   (same for k and v with dkbar, dvbar).
//
// Two kernels, neither with atomics (results are deterministic):
//   fine_bwd_dq    one CTA per query cube, walking its selected key cubes
//   fine_bwd_dkdv  one CTA per key cube, walking the query cubes that
//                  selected it (the CSR lists of the selection transpose)
// Each 64 x 64 and 64 x d product is the register-tiled float32 SIMT product
// of simt_tile.cuh; the cube's own operands stay in shared memory, the other
// side's are staged in 32-deep chunks.  bf16 in, float32 arithmetic, bf16
// gradients out in token order.
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
using simt::stage_rows_t;
using simt::tile_col;
using bf16 = __nv_bfloat16;

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&p);
}

// Writes rows m < n (rows of cube `cube`) of a 64 x D float32 tile to their
// tokens as bf16: out[token] = acc * mul + bar[cube] * rn (bar may be null).
template <int D>
__device__ __forceinline__ void store_tokens(const Geom& g, long long bh, int cube, int n,
                                             const float (&acc)[4][D / 16], float mul,
                                             const float* __restrict__ bar, float rn,
                                             bf16* __restrict__ out) {
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const float* b = bar ? bar + (bh * g.C + cube) * D : nullptr;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int m = ty * 4 + r;
    if (m >= n) continue;
    const long long tok = bh * g.N + slot_token(g, cube, m);
    bf16* row = out + tok * D;
#pragma unroll
    for (int grp = 0; grp < D / 64; ++grp) {
      const int col = tile_col(tx, 4 * grp);
      float v[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        v[q] = acc[r][4 * grp + q] * mul;
        if (b) v[q] = fmaf(b[col + q], rn, v[q]);
      }
      *reinterpret_cast<uint2*>(row + col) = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
    }
  }
}

// Dynamic shared memory of each kernel (floats).
template <int D>
constexpr int dq_smem_floats() { return 2 * D * kTileM + kChunk * D + kTileM * kTileM; }
template <int D>
constexpr int dkdv_smem_floats() { return 2 * D * kTileM + kChunk * D + 2 * kTileM * kTileM; }

// grid (C, B*H): dq of query cube i.
// smem: Qt, Gt [D][64] (Q_i^T, dO_i^T), Bs [32][D] (staged chunk), Ss [64][64] (dS^T).
template <int D>
__global__ void __launch_bounds__(kThreads, 1) fine_bwd_dq(
    Geom g, int topk, const bf16* __restrict__ qt, const bf16* __restrict__ kt,
    const bf16* __restrict__ vt, const bf16* __restrict__ dot, const float* __restrict__ lse,
    const float* __restrict__ delta, const int32_t* __restrict__ sel,
    const float* __restrict__ dqbar, bf16* __restrict__ dq, int* status) {
  extern __shared__ __align__(16) float sm[];
  float* Qt = sm;
  float* Gt = Qt + D * kTileM;
  float* Bs = Gt + D * kTileM;
  float* Ss = Bs + kChunk * D;
  __shared__ float lse_s[kTileM], D_s[kTileM];
  const int i = blockIdx.x;
  const long long bh = blockIdx.y;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int n_i = cube_valid(g, i);
  const long long qrow0 = bh * g.rows + static_cast<long long>(i) * kSlots;
  const float scale = 1.0f / sqrtf(static_cast<float>(D));
  stage_rows_t(Qt, qt + qrow0 * D, D, 0, kTileM, D);
  stage_rows_t(Gt, dot + qrow0 * D, D, 0, kTileM, D);
  if (threadIdx.x < kTileM) {
    lse_s[threadIdx.x] = lse[qrow0 + threadIdx.x];
    D_s[threadIdx.x] = delta[qrow0 + threadIdx.x];
  }
  float acc[4][D / 16] = {};
  const int32_t* my_sel = sel + (bh * g.C + i) * topk;
  for (int t = 0; t < topk; ++t) {
    const int j = my_sel[t];
    if (j < 0 || j >= g.C) {  // the same entry for every thread: a uniform skip
      if (threadIdx.x == 0) report(status, VSA_ERR_BAD_INDEX);
      continue;
    }
    const int n_j = cube_valid(g, j);
    const bf16* kj = kt + (bh * g.rows + static_cast<long long>(j) * kSlots) * D;
    const bf16* vj = vt + (bh * g.rows + static_cast<long long>(j) * kSlots) * D;
    // S = Q_i K_j^T and dP = dO_i V_j^T (rows r = ty*4+a, keys c = tx*4+b)
    float s[4][4] = {}, dp[4][4] = {};
    for (int e0 = 0; e0 < D; e0 += kChunk) {
      __syncthreads();  // Bs (and, on the first chunk, Ss of the last block) no longer read
      stage<kTileM, true>(Bs, kj, D, 0, kTileM, e0, D);
      __syncthreads();
      chunk_fma<64>(Qt + e0 * kTileM, Bs, tx, ty, s);
      __syncthreads();
      stage<kTileM, true>(Bs, vj, D, 0, kTileM, e0, D);
      __syncthreads();
      chunk_fma<64>(Gt + e0 * kTileM, Bs, tx, ty, dp);
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int r = ty * 4 + a;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int c = tx * 4 + b;
        const float p = (r < n_i && c < n_j) ? expf(fmaf(s[a][b], scale, -lse_s[r])) : 0.f;
        Ss[c * kTileM + r] = p * (dp[a][b] - D_s[r]);
      }
    }
    // dQ_i += dS K_j over the 64 keys, two chunks of 32
    for (int c0 = 0; c0 < kTileM; c0 += kChunk) {
      __syncthreads();  // Ss complete; Bs no longer read
      stage<D, false>(Bs, kj, D, 0, D, c0, kTileM);
      __syncthreads();
      chunk_fma<D>(Ss + c0 * kTileM, Bs, tx, ty, acc);
    }
  }
  store_tokens<D>(g, bh, i, n_i, acc, scale, dqbar, 1.0f / static_cast<float>(n_i), dq);
}

// grid (C, B*H): dk, dv of key cube j.
// smem: Kt, Vt [D][64] (K_j^T, V_j^T), Bs [32][D], Ps, Ss [64][64] (P, dS as [r][c]).
template <int D>
__global__ void __launch_bounds__(kThreads, 1) fine_bwd_dkdv(
    Geom g, int topk, const bf16* __restrict__ qt, const bf16* __restrict__ kt,
    const bf16* __restrict__ vt, const bf16* __restrict__ dot, const float* __restrict__ lse,
    const float* __restrict__ delta, const int32_t* __restrict__ key_offsets,
    const int32_t* __restrict__ query_lists, const float* __restrict__ dkbar,
    const float* __restrict__ dvbar, bf16* __restrict__ dk, bf16* __restrict__ dv, int* status) {
  extern __shared__ __align__(16) float sm[];
  float* Kt = sm;
  float* Vt = Kt + D * kTileM;
  float* Bs = Vt + D * kTileM;
  float* Ps = Bs + kChunk * D;
  float* Ss = Ps + kTileM * kTileM;
  __shared__ float lse_s[kTileM], D_s[kTileM];
  const int j = blockIdx.x;
  const long long bh = blockIdx.y;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int n_j = cube_valid(g, j);
  const long long krow0 = bh * g.rows + static_cast<long long>(j) * kSlots;
  const float scale = 1.0f / sqrtf(static_cast<float>(D));
  stage_rows_t(Kt, kt + krow0 * D, D, 0, kTileM, D);
  stage_rows_t(Vt, vt + krow0 * D, D, 0, kTileM, D);
  float acc_k[4][D / 16] = {}, acc_v[4][D / 16] = {};
  const int32_t* offs = key_offsets + bh * (g.C + 1);
  const int32_t* list = query_lists + bh * static_cast<long long>(g.C) * topk;
  const int p0 = offs[j], p1 = offs[j + 1];
  for (int p = p0; p < p1; ++p) {
    const int i = list[p];
    if (i < 0 || i >= g.C) {  // uniform skip
      if (threadIdx.x == 0) report(status, VSA_ERR_BAD_INDEX);
      continue;
    }
    const int n_i = cube_valid(g, i);
    const long long qrow0 = bh * g.rows + static_cast<long long>(i) * kSlots;
    const bf16* qi = qt + qrow0 * D;
    const bf16* gi = dot + qrow0 * D;
    __syncthreads();  // lse_s, D_s, Ps, Ss and Bs of the previous query cube no longer read
    if (threadIdx.x < kTileM) {
      lse_s[threadIdx.x] = lse[qrow0 + threadIdx.x];
      D_s[threadIdx.x] = delta[qrow0 + threadIdx.x];
    }
    // S^T = K_j Q_i^T and dP^T = V_j dO_i^T (keys c = ty*4+a, rows r = tx*4+b)
    float s[4][4] = {}, dp[4][4] = {};
    for (int e0 = 0; e0 < D; e0 += kChunk) {
      stage<kTileM, true>(Bs, qi, D, 0, kTileM, e0, D);
      __syncthreads();
      chunk_fma<64>(Kt + e0 * kTileM, Bs, tx, ty, s);
      __syncthreads();
      stage<kTileM, true>(Bs, gi, D, 0, kTileM, e0, D);
      __syncthreads();
      chunk_fma<64>(Vt + e0 * kTileM, Bs, tx, ty, dp);
      __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int c = ty * 4 + a;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int r = tx * 4 + b;
        const float pr = (r < n_i && c < n_j) ? expf(fmaf(s[a][b], scale, -lse_s[r])) : 0.f;
        Ps[r * kTileM + c] = pr;
        Ss[r * kTileM + c] = pr * (dp[a][b] - D_s[r]);
      }
    }
    // dV_j += P^T dO_i and dK_j += dS^T Q_i over the 64 rows, two chunks of 32
    for (int r0 = 0; r0 < kTileM; r0 += kChunk) {
      __syncthreads();  // Ps, Ss complete; Bs no longer read
      stage<D, false>(Bs, gi, D, 0, D, r0, kTileM);
      __syncthreads();
      chunk_fma<D>(Ps + r0 * kTileM, Bs, tx, ty, acc_v);
      __syncthreads();
      stage<D, false>(Bs, qi, D, 0, D, r0, kTileM);
      __syncthreads();
      chunk_fma<D>(Ss + r0 * kTileM, Bs, tx, ty, acc_k);
    }
  }
  const float rn = 1.0f / static_cast<float>(n_j);
  store_tokens<D>(g, bh, j, n_j, acc_k, scale, dkbar, rn, dk);
  store_tokens<D>(g, bh, j, n_j, acc_v, 1.0f, dvbar, rn, dv);
}

template <int D>
cudaError_t run(const Geom& g, int topk, const bf16* qt, const bf16* kt, const bf16* vt,
                const bf16* dot, const float* lse, const float* delta, const int32_t* sel,
                const int32_t* key_offsets, const int32_t* query_lists, const float* dpooled,
                bf16* dq, bf16* dk, bf16* dv, int* status, cudaStream_t s) {
  static CtxCache<char> dq_set, dkdv_set;
  const int dq_bytes = dq_smem_floats<D>() * static_cast<int>(sizeof(float));
  const int dkdv_bytes = dkdv_smem_floats<D>() * static_cast<int>(sizeof(float));
  cudaError_t err = smem_limit_once(fine_bwd_dq<D>, dq_bytes, &dq_set);
  if (err != cudaSuccess) return err;
  if ((err = smem_limit_once(fine_bwd_dkdv<D>, dkdv_bytes, &dkdv_set)) != cudaSuccess) return err;
  const long long plane = static_cast<long long>(g.B) * g.H * g.C * D;
  const float* dqbar = dpooled;
  const float* dkbar = dpooled ? dpooled + plane : nullptr;
  const float* dvbar = dpooled ? dpooled + 2 * plane : nullptr;
  const dim3 grid(g.C, g.B * g.H);
  fine_bwd_dq<D><<<grid, kThreads, dq_bytes, s>>>(g, topk, qt, kt, vt, dot, lse, delta, sel, dqbar,
                                                  dq, status);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  fine_bwd_dkdv<D><<<grid, kThreads, dkdv_bytes, s>>>(g, topk, qt, kt, vt, dot, lse, delta,
                                                      key_offsets, query_lists, dkbar, dvbar, dk,
                                                      dv, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_block_sparse_bwd(const Geom& g, int topk, const void* qt, const void* kt,
                                    const void* vt, const void* dot, const float* lse,
                                    const float* delta, const int32_t* sel,
                                    const int32_t* key_offsets, const int32_t* query_lists,
                                    const float* dpooled, void* dq, void* dk, void* dv,
                                    int* status, cudaStream_t s) {
  auto b = [](const void* p) { return static_cast<const bf16*>(p); };
  auto w = [](void* p) { return static_cast<bf16*>(p); };
  if (g.d == 64)
    return run<64>(g, topk, b(qt), b(kt), b(vt), b(dot), lse, delta, sel, key_offsets,
                   query_lists, dpooled, w(dq), w(dk), w(dv), status, s);
  return run<128>(g, topk, b(qt), b(kt), b(vt), b(dot), lse, delta, sel, key_offsets, query_lists,
                  dpooled, w(dq), w(dk), w(dv), status, s);
}

}  // namespace vsa
