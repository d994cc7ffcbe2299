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
constexpr int kKeyChunk = 32;
constexpr int kLogitBudgetBytes = 160 * 1024;

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
// grid (ceil(C/R), B*H); R query cubes per CTA; 256 threads.
// smem: logits [R][C] f32 | q rows [R][d] | key/value chunk [32][d+1] | hist [8][256]
__global__ void __launch_bounds__(kCoarseThreads) coarse_kernel(
    Geom g, int R, int topk, const float* __restrict__ ws, float* __restrict__ o_coarse,
    int32_t* __restrict__ sel, float* __restrict__ logits_out) {
  extern __shared__ float sm[];
  const int C = g.C, d = g.d, dp = g.d + 1;
  float* S = sm;                                   // [R][C]
  float* qs = S + static_cast<size_t>(R) * C;      // [R][d]
  float* ks = qs + static_cast<size_t>(R) * d;     // [32][d+1]
  int* hist = reinterpret_cast<int*>(ks + kKeyChunk * dp);  // [8][256]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y;
  const int i0 = blockIdx.x * R;
  const int rows = min(R, C - i0);
  const long long plane = static_cast<long long>(g.B) * g.H * C * d;
  const float* qbar = ws + (static_cast<long long>(bh) * C) * d;
  const float* kbar = ws + plane + (static_cast<long long>(bh) * C) * d;
  const float* vbar = ws + 2 * plane + (static_cast<long long>(bh) * C) * d;
  const float scale = 1.0f / sqrtf(static_cast<float>(d));

  for (int e = tid; e < R * d; e += kCoarseThreads) {
    const int r = e / d;
    qs[e] = r < rows ? qbar[static_cast<long long>(i0 + r) * d + (e - r * d)] : 0.f;
  }
  // ---- logits: thread -> key jj = lane of the chunk, rows warp, warp+8, ...
  for (int j0 = 0; j0 < C; j0 += kKeyChunk) {
    __syncthreads();
    const int nk = min(kKeyChunk, C - j0);
    for (int e = tid; e < kKeyChunk * d; e += kCoarseThreads) {
      const int jj = e / d, col = e - jj * d;
      ks[jj * dp + col] = jj < nk ? kbar[static_cast<long long>(j0 + jj) * d + col] : 0.f;
    }
    __syncthreads();
    if (lane < nk) {
      for (int r = warp; r < rows; r += 8) {
        const float* qr = qs + r * d;
        const float* kr = ks + lane * dp;
        float acc = 0.f;
        for (int e = 0; e < d; ++e) acc = fmaf(qr[e], kr[e], acc);
        const float s = acc * scale;
        S[static_cast<size_t>(r) * C + j0 + lane] = s;
        if (logits_out != nullptr)
          logits_out[(static_cast<long long>(bh) * C + i0 + r) * C + j0 + lane] = s;
      }
    }
  }
  __syncthreads();
  // ---- top-k on the logits, then softmax in place (one warp per row)
  for (int r = warp; r < rows; r += 8) {
    float* row = S + static_cast<size_t>(r) * C;
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
    for (int j = lane; j < C; j += 32) row[j] *= inv;
  }
  if (o_coarse == nullptr) return;
  // ---- O_c = P vbar: thread -> column e = tid % d, rows tid / d + G*m
  const int G = kCoarseThreads / d;  // 2 (d=128) or 4 (d=64)
  const int e = tid % d, rg = tid / d;
  float acc[16];
#pragma unroll
  for (int m = 0; m < 16; ++m) acc[m] = 0.f;
  for (int j0 = 0; j0 < C; j0 += kKeyChunk) {
    __syncthreads();
    const int nk = min(kKeyChunk, C - j0);
    for (int t = tid; t < kKeyChunk * d; t += kCoarseThreads) {
      const int jj = t / d, col = t - jj * d;
      ks[jj * dp + col] = jj < nk ? vbar[static_cast<long long>(j0 + jj) * d + col] : 0.f;
    }
    __syncthreads();
    for (int jj = 0; jj < nk; ++jj) {
      const float vv = ks[jj * dp + e];
#pragma unroll
      for (int m = 0; m < 16; ++m) {
        const int r = rg + G * m;
        if (r < rows) acc[m] = fmaf(S[static_cast<size_t>(r) * C + j0 + jj], vv, acc[m]);
      }
    }
  }
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    const int r = rg + G * m;
    if (r < rows) o_coarse[(static_cast<long long>(bh) * C + i0 + r) * d + e] = acc[m];
  }
}

}  // namespace

// Rows of query cubes per coarse CTA: as many as the smem logits budget
// allows, at most 16 (the O_c accumulation keeps 16 rows per thread for d=64
// and 8 for d=128).
int coarse_rows_per_cta(int C, int d) {
  int R = kLogitBudgetBytes / (C * 4);
  const int cap = (d == 128) ? 16 : 16;
  if (R > cap) R = cap;
  if (R < 1) R = 1;
  return R;
}

size_t coarse_smem_bytes(int C, int d, int R) {
  return (static_cast<size_t>(R) * C + static_cast<size_t>(R) * d +
          static_cast<size_t>(kKeyChunk) * (d + 1)) * sizeof(float) + 8 * 256 * sizeof(int);
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
