// Coarse stage of VSA (FastWan article "单块 H200 ... 5 秒即生一个 5 秒视频",
// section "一张卡，秒生视频", Fig. 5 paragraph; dynamic key selection in
// section "传统零散郑重力，为何会在蒸馏中失效？").
//
// 1. pool_kernel: qbar, kbar, vbar = mean of each cube's n_c valid rows
//    (float32), an HBM-bound pass over the three tiled tensors.
// 2. coarse_kernel: for a tile of R query cubes of one (b, h):
//      S_c[i, :] = qbar_i kbar^T / sqrt(d)       (float32, row kept in smem)
//      sel[i]    = top-k of S_c[i, :], ties to the lower index, ascending
//      O_c[i]    = softmax(S_c[i, :]) vbar
//    The per-row top-k is a warp-level MSB-first radix select on the
//    order-preserving integer image of the float logits, followed by one
//    ballot-compaction pass in index order (so the output is ascending and
//    equal logits are taken lowest index first).
#include <cmath>

#include "common.cuh"

namespace vsa {

namespace {

constexpr int kCoarseThreads = 256;
constexpr int kLogitBudgetBytes = 132 * 1024;

// ------------------------------------------------------------------ pooling
// One warp per (tensor, b*h, cube).  A row of d bf16 is d/8 16-byte chunks;
// the warp covers 32/(d/8) rows per step and reduces across row groups at the end.
__global__ void __launch_bounds__(256) pool_kernel(Geom g, const uint4* __restrict__ q,
                                                   const uint4* __restrict__ k,
                                                   const uint4* __restrict__ v,
                                                   const int32_t* __restrict__ counts,
                                                   float* __restrict__ ws, int* status) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long item = static_cast<long long>(blockIdx.x) * 8 + warp;  // (b*h, cube)
  const long long items = static_cast<long long>(g.B) * g.H * g.C;
  if (item >= items) return;
  const int which = blockIdx.y;  // 0 q, 1 k, 2 v
  const uint4* src = which == 0 ? q : (which == 1 ? k : v);
  const long long bh = item / g.C;
  const int c = static_cast<int>(item - bh * g.C);
  const int n = cube_valid(g, c);
  if (which == 0 && lane == 0 && counts[c] != n) report(status, VSA_ERR_BAD_INDEX);

  const int chunks = g.d >> 3;         // 8 or 16
  const int rows_per_step = 32 / chunks;  // 4 or 2
  const int ch = lane % chunks;
  const int r0 = lane / chunks;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  const uint4* base = src + (bh * g.rows + static_cast<long long>(c) * kSlots) * chunks;
  for (int r = r0; r < n; r += rows_per_step) {
    const uint4 w = __ldg(&base[static_cast<long long>(r) * chunks + ch]);
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[2 * e] += __uint_as_float(u[e] << 16);
      acc[2 * e + 1] += __uint_as_float(u[e] & 0xFFFF0000u);
    }
  }
  for (int off = chunks; off < 32; off <<= 1) {
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
  }
  if (r0 == 0) {
    float* dst = ws + (static_cast<long long>(which) * g.B * g.H * g.C + item) * g.d + ch * 8;
    const float inv_n = 1.0f / static_cast<float>(n);
    float4 a = make_float4(acc[0] * inv_n, acc[1] * inv_n, acc[2] * inv_n, acc[3] * inv_n);
    float4 b = make_float4(acc[4] * inv_n, acc[5] * inv_n, acc[6] * inv_n, acc[7] * inv_n);
    reinterpret_cast<float4*>(dst)[0] = a;
    reinterpret_cast<float4*>(dst)[1] = b;
  }
}

// ------------------------------------------------------------------ top-k
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f + 0.0f);  // -0 -> +0 so they tie
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Writes the indices of the k largest of row[0..C) (ties: lower index first)
// in ascending order to out[0..k).  Executed by one full warp; hist is a
// warp-private 256-entry smem array.
__device__ void warp_topk(const float* row, int C, int k, int* hist, int32_t* out) {
  const int lane = threadIdx.x & 31;
  uint32_t prefix = 0u, mask = 0u;
  int remaining = k;  // rank of the wanted key among the keys matching the prefix
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = lane; b < 256; b += 32) hist[b] = 0;
    __syncwarp();
    for (int j = lane; j < C; j += 32) {
      const uint32_t key = order_key(row[j]);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
    }
    __syncwarp();
    // lane l owns bins 255-8l .. 248-8l (descending); inclusive scan over lanes
    int cnt[8];
    int own = 0;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      cnt[t] = hist[255 - 8 * lane - t];
      own += cnt[t];
    }
    int incl = own;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    const unsigned hit = __ballot_sync(0xffffffffu, incl >= remaining);
    const int src = __ffs(hit) - 1;  // first lane whose cumulative count reaches `remaining`
    int digit = 0, above = 0;
    if (lane == src) {
      int run = incl - own;  // keys in higher bins of earlier lanes
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        if (run + cnt[t] >= remaining) {
          digit = 255 - 8 * lane - t;
          above = run;
          break;
        }
        run += cnt[t];
      }
    }
    digit = __shfl_sync(0xffffffffu, digit, src);
    above = __shfl_sync(0xffffffffu, above, src);
    remaining -= above;
    prefix |= static_cast<uint32_t>(digit) << shift;
    mask |= 255u << shift;
    __syncwarp();
  }
  // prefix = key of the k-th largest; take all keys above it and the first
  // `remaining` keys equal to it, in index order.
  const unsigned lt = (1u << lane) - 1u;
  int pos = 0, eq_seen = 0;
  for (int j0 = 0; j0 < C; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t key = j < C ? order_key(row[j]) : 0u;
    const bool gt = j < C && key > prefix;
    const bool eq = j < C && key == prefix;
    const unsigned eqm = __ballot_sync(0xffffffffu, eq);
    const bool take = gt || (eq && eq_seen + __popc(eqm & lt) < remaining);
    const unsigned tm = __ballot_sync(0xffffffffu, take);
    if (take) out[pos + __popc(tm & lt)] = j;
    pos += __popc(tm);
    eq_seen += __popc(eqm);
  }
}

// ------------------------------------------------------------------ coarse
// grid (ceil(C/R), B*H), 256 threads, R <= 16 query cubes per CTA.
// smem: S [R][Cp] f32 (Cp = C rounded up to 4) | qT [d][16] | staging
// [32][260] (key slices, then value chunks) | hist [8][256].
//
// Logits: a 16-row x 256-key tile per pass; thread t owns rows 4*(t/64)..+3
// and keys 4*(t%64)..+3 (16 accumulators), over head-dim slices of 32
// staged transposed in smem, so each step is two 128-bit smem loads for 16
// FMAs.  O_c: thread t owns rows 2*(t/32), +1 and d/32 columns.
constexpr int kTileKeys = 256;
constexpr int kSlice = 32;
constexpr int kStagePitch = kTileKeys + 4;

__global__ void __launch_bounds__(kCoarseThreads) coarse_kernel(
    Geom g, int R, int topk, const float* __restrict__ ws, float* __restrict__ o_coarse,
    int32_t* __restrict__ sel, float* __restrict__ logits_out) {
  extern __shared__ __align__(16) float sm[];
  const int C = g.C, d = g.d;
  const int Cp = (C + 3) & ~3;
  float* S = sm;                                     // [R][Cp]
  float* qT = S + static_cast<size_t>(R) * Cp;       // [d][16]
  float* stage = qT + static_cast<size_t>(d) * 16;   // [32][kStagePitch]
  int* hist = reinterpret_cast<int*>(stage + kSlice * kStagePitch);  // [8][256]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y;
  const int i0 = blockIdx.x * R;
  const int rows = min(R, C - i0);
  const long long plane = static_cast<long long>(g.B) * g.H * C * d;
  const float* qbar = ws + (static_cast<long long>(bh) * C) * d;
  const float* kbar = ws + plane + (static_cast<long long>(bh) * C) * d;
  const float* vbar = ws + 2 * plane + (static_cast<long long>(bh) * C) * d;
  const float scale = 1.0f / sqrtf(static_cast<float>(d));

  for (int e = tid; e < 16 * d; e += kCoarseThreads) {  // qT[col][row]
    const int r = e & 15, col = e >> 4;
    qT[e] = r < rows ? qbar[static_cast<long long>(i0 + r) * d + col] : 0.f;
  }
  // ---- logits
  const int rg = tid >> 6, kg = tid & 63;
  for (int j0 = 0; j0 < C; j0 += kTileKeys) {
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
    for (int e0 = 0; e0 < d; e0 += kSlice) {
      __syncthreads();
      // stage keys j0..j0+255, dims e0..e0+31, transposed: stage[dim][key]
      for (int idx = tid; idx < kTileKeys * (kSlice / 4); idx += kCoarseThreads) {
        const int jj = idx >> 3, q4 = idx & 7;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (j0 + jj < C)
          v = *reinterpret_cast<const float4*>(kbar + static_cast<long long>(j0 + jj) * d + e0 + 4 * q4);
        stage[(4 * q4 + 0) * kStagePitch + jj] = v.x;
        stage[(4 * q4 + 1) * kStagePitch + jj] = v.y;
        stage[(4 * q4 + 2) * kStagePitch + jj] = v.z;
        stage[(4 * q4 + 3) * kStagePitch + jj] = v.w;
      }
      __syncthreads();
#pragma unroll 8
      for (int ee = 0; ee < kSlice; ++ee) {
        const float4 qv = *reinterpret_cast<const float4*>(qT + (e0 + ee) * 16 + 4 * rg);
        const float4 kv = *reinterpret_cast<const float4*>(stage + ee * kStagePitch + 4 * kg);
        const float qa[4] = {qv.x, qv.y, qv.z, qv.w};
        const float ka[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(qa[a], ka[b], acc[a][b]);
      }
    }
    const int jb = j0 + 4 * kg;
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int r = 4 * rg + a;
      if (r >= rows) continue;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int j = jb + b;
        if (j < C) {
          const float s = acc[a][b] * scale;
          S[static_cast<size_t>(r) * Cp + j] = s;
          if (logits_out != nullptr)
            logits_out[(static_cast<long long>(bh) * C + i0 + r) * C + j] = s;
        }
      }
    }
  }
  __syncthreads();
  // ---- top-k on the logits, then softmax in place (one warp per row)
  for (int r = warp; r < rows; r += 8) {
    float* row = S + static_cast<size_t>(r) * Cp;
    warp_topk(row, C, topk, hist + warp * 256,
              sel + (static_cast<long long>(bh) * C + i0 + r) * topk);
    float mx = -INFINITY;
    for (int j = lane; j < C; j += 32) mx = fmaxf(mx, row[j]);
    for (int off = 16; off; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    float z = 0.f;
    for (int j = lane; j < C; j += 32) {
      const float p = expf(row[j] - mx);
      row[j] = p;
      z += p;
    }
    for (int off = 16; off; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
    const float inv = 1.0f / z;
    __syncwarp();
    for (int j = lane; j < Cp; j += 32) row[j] = j < C ? row[j] * inv : 0.f;
  }
  if (o_coarse == nullptr) return;
  // ---- O_c = P vbar: rows 2*(t/32), +1; columns cpt*(t%32) .. +cpt-1
  const int cpt = d / 32;  // 4 (d=128) or 2 (d=64)
  const int r0 = 2 * (tid >> 5), c0 = cpt * (tid & 31);
  float o0[4] = {0.f, 0.f, 0.f, 0.f}, o1[4] = {0.f, 0.f, 0.f, 0.f};
  const int vchunk = (kSlice * kStagePitch) / d & ~3;  // value rows per staged chunk
  for (int j0 = 0; j0 < C; j0 += vchunk) {
    __syncthreads();
    const int nk = min(vchunk, C - j0);
    for (int idx = tid; idx < vchunk * d / 4; idx += kCoarseThreads) {
      const int jj = idx / (d / 4), q4 = idx - jj * (d / 4);
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (jj < nk) v = *reinterpret_cast<const float4*>(vbar + static_cast<long long>(j0 + jj) * d + 4 * q4);
      reinterpret_cast<float4*>(stage)[idx] = v;
    }
    __syncthreads();
    if (r0 < rows) {
      const float* p0 = S + static_cast<size_t>(r0) * Cp + j0;
      const float* p1 = p0 + Cp;
      for (int jj = 0; jj < nk; jj += 4) {
        const float4 pa = *reinterpret_cast<const float4*>(p0 + jj);
        const float4 pb = *reinterpret_cast<const float4*>(p1 + jj);
        const float pav[4] = {pa.x, pa.y, pa.z, pa.w};
        const float pbv[4] = {pb.x, pb.y, pb.z, pb.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float* vrow = stage + (jj + u) * d + c0;
          if (cpt == 4) {
            const float4 v = *reinterpret_cast<const float4*>(vrow);
            o0[0] = fmaf(pav[u], v.x, o0[0]); o0[1] = fmaf(pav[u], v.y, o0[1]);
            o0[2] = fmaf(pav[u], v.z, o0[2]); o0[3] = fmaf(pav[u], v.w, o0[3]);
            o1[0] = fmaf(pbv[u], v.x, o1[0]); o1[1] = fmaf(pbv[u], v.y, o1[1]);
            o1[2] = fmaf(pbv[u], v.z, o1[2]); o1[3] = fmaf(pbv[u], v.w, o1[3]);
          } else {
            const float2 v = *reinterpret_cast<const float2*>(vrow);
            o0[0] = fmaf(pav[u], v.x, o0[0]); o0[1] = fmaf(pav[u], v.y, o0[1]);
            o1[0] = fmaf(pbv[u], v.x, o1[0]); o1[1] = fmaf(pbv[u], v.y, o1[1]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    if (c >= cpt) break;
    if (r0 < rows) o_coarse[(static_cast<long long>(bh) * C + i0 + r0) * d + c0 + c] = o0[c];
    if (r0 + 1 < rows) o_coarse[(static_cast<long long>(bh) * C + i0 + r0 + 1) * d + c0 + c] = o1[c];
  }
}

}  // namespace

// Rows of query cubes per coarse CTA: 16, or fewer when a [R][C] float32
// logits block would not fit next to the staging buffers.
int coarse_rows_per_cta(int C, int d) {
  (void)d;
  const int Cp = (C + 3) & ~3;
  int R = 16;
  while (R > 4 && static_cast<long long>(R) * Cp * 4 > kLogitBudgetBytes) R >>= 1;
  return R;
}

size_t coarse_smem_bytes(int C, int d, int R) {
  const size_t Cp = (static_cast<size_t>(C) + 3) & ~static_cast<size_t>(3);
  return (R * Cp + static_cast<size_t>(d) * 16 + static_cast<size_t>(kSlice) * kStagePitch) *
             sizeof(float) + 8 * 256 * sizeof(int);
}

cudaError_t launch_coarse_select(const Geom& g, const void* qt, const void* kt, const void* vt,
                                 const int32_t* counts, int topk, float* o_coarse,
                                 int32_t* sel, float* logits, float* ws, int* status,
                                 cudaStream_t s) {
  const long long items = static_cast<long long>(g.B) * g.H * g.C;
  dim3 pg(static_cast<unsigned>((items + 7) / 8), 3);
  pool_kernel<<<pg, 256, 0, s>>>(g, static_cast<const uint4*>(qt), static_cast<const uint4*>(kt),
                                 static_cast<const uint4*>(vt), counts, ws, status);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const int R = coarse_rows_per_cta(g.C, g.d);
  const size_t smem = coarse_smem_bytes(g.C, g.d, R);
  err = cudaFuncSetAttribute(coarse_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  dim3 cg(static_cast<unsigned>((g.C + R - 1) / R), static_cast<unsigned>(g.B * g.H));
  coarse_kernel<<<cg, kCoarseThreads, smem, s>>>(g, R, topk, ws, o_coarse, sel, logits);
  return cudaGetLastError();
}

}  // namespace vsa
