// Transpose of the top-k selection: for every key cube, the query cubes that
// selected it, in ascending order (a CSR list per (b, h)).  The key-stationary
// half of a backward pass (dK, dV of one key cube accumulated over the query
// cubes that attended to it) walks these lists.
//
// The query cubes of each (b, h) are split into G groups of consecutive cubes,
// one CTA per (group, b, h), in three passes:
//   1. count: per group and key cube, how many of the group's query cubes
//      selected it (shared-memory counters, written to the workspace);
//   2. scan: per (b, h), the CSR offsets, and for each group the first slot
//      of its entries in every key cube's segment (groups in query order);
//   3. scatter: each group walks its query cubes in ascending order and puts
//      query i at its key cubes' cursors.  A query cube selects a key cube at
//      most once, so the k entries of one query cube touch distinct cursors
//      and can go in parallel; query cubes go one after another, so every
//      segment ends up ascending with no sorting and the result is
//      deterministic.
#include "common.cuh"

namespace vsa {

namespace {

constexpr int kThreads = 256;

// Query cubes [lo, hi) of group g of C cubes split into G groups.
__device__ __forceinline__ void group_range(int C, int G, int g, int& lo, int& hi) {
  const int per = (C + G - 1) / G;
  lo = min(C, g * per);
  hi = min(C, lo + per);
}

// grid (G, B*H): counts[bh][g][j] = #query cubes of group g that selected j.
__global__ void __launch_bounds__(kThreads) transpose_count_kernel(
    int C, int topk, int G, const int32_t* __restrict__ sel, int32_t* __restrict__ counts,
    int* status) {
  extern __shared__ int32_t cnt[];  // C counters
  const int g = blockIdx.x;
  const long long bh = blockIdx.y;
  for (int j = threadIdx.x; j < C; j += blockDim.x) cnt[j] = 0;
  __syncthreads();
  int lo, hi;
  group_range(C, G, g, lo, hi);
  const int32_t* s = sel + bh * C * topk;
  const long long p0 = static_cast<long long>(lo) * topk, p1 = static_cast<long long>(hi) * topk;
  for (long long p = p0 + threadIdx.x; p < p1; p += blockDim.x) {
    const int j = __ldg(&s[p]);
    if (j < 0 || j >= C) {
      report(status, VSA_ERR_BAD_INDEX);
      continue;
    }
    atomicAdd(&cnt[j], 1);
  }
  __syncthreads();
  int32_t* out = counts + (bh * G + g) * C;
  for (int j = threadIdx.x; j < C; j += blockDim.x) out[j] = cnt[j];
}

// grid (B*H): offsets[bh][j] (exclusive scan over key cubes of the group
// totals) and, in place of counts[bh][g][j], the first slot of group g in
// key cube j's segment.
__global__ void __launch_bounds__(kThreads) transpose_scan_kernel(int C, int G,
                                                                  int32_t* __restrict__ counts,
                                                                  int32_t* __restrict__ offsets) {
  extern __shared__ int32_t tot[];  // C totals, then their exclusive scan
  __shared__ int32_t warp_sum[kThreads / 32];
  const long long bh = blockIdx.x;
  int32_t* cg = counts + bh * G * C;
  for (int j = threadIdx.x; j < C; j += blockDim.x) {
    int t = 0;
    for (int g = 0; g < G; ++g) t += cg[static_cast<long long>(g) * C + j];
    tot[j] = t;
  }
  __syncthreads();
  // exclusive scan of tot[0..C): each thread scans a contiguous run
  const int per = (C + kThreads - 1) / kThreads;
  const int lo = min(C, static_cast<int>(threadIdx.x) * per), hi = min(C, lo + per);
  int run = 0;
  for (int j = lo; j < hi; ++j) run += tot[j];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = run;
  for (int d = 1; d < 32; d <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += o;
  }
  if (lane == 31) warp_sum[warp] = incl;
  __syncthreads();
  int before = 0;
  for (int w = 0; w < warp; ++w) before += warp_sum[w];
  int base = before + incl - run;
  __syncthreads();  // every thread has read its run of tot before it is overwritten
  int32_t* off = offsets + bh * (C + 1);
  for (int j = lo; j < hi; ++j) {
    const int t = tot[j];
    off[j] = base;
    tot[j] = base;
    base += t;
  }
  if (threadIdx.x == kThreads - 1) off[C] = base;
  __syncthreads();
  // first slot of each group in each segment: groups follow query order
  for (int j = threadIdx.x; j < C; j += blockDim.x) {
    int slot = tot[j];
    for (int g = 0; g < G; ++g) {
      const long long e = static_cast<long long>(g) * C + j;
      const int c = cg[e];
      cg[e] = slot;
      slot += c;
    }
  }
}

// grid (G, B*H): query cubes of group g, in ascending order, into their key
// cubes' segments.
__global__ void __launch_bounds__(kThreads) transpose_scatter_kernel(
    int C, int topk, int G, const int32_t* __restrict__ sel, const int32_t* __restrict__ starts,
    int32_t* __restrict__ queries) {
  extern __shared__ int32_t cur[];  // C cursors
  const int g = blockIdx.x;
  const long long bh = blockIdx.y;
  const int32_t* st = starts + (bh * G + g) * C;
  for (int j = threadIdx.x; j < C; j += blockDim.x) cur[j] = st[j];
  __syncthreads();
  int lo, hi;
  group_range(C, G, g, lo, hi);
  const int32_t* s = sel + bh * C * topk;
  int32_t* out = queries + bh * C * topk;
  for (int i = lo; i < hi; ++i) {
    // the k entries of query cube i name distinct key cubes: no two threads
    // of this pass share a cursor
    for (int t = threadIdx.x; t < topk; t += blockDim.x) {
      const int j = __ldg(&s[static_cast<long long>(i) * topk + t]);
      if (j < 0 || j >= C) continue;  // reported by the count pass
      out[cur[j]++] = i;
    }
    __syncthreads();
  }
}

}  // namespace

// Groups per (b, h): enough CTAs to fill the GPU, and the workspace of
// B*H*C*k int32 holds the B*H*G*C group counters while G <= k.
int transpose_groups(int bh, int C, int topk, int sms) {
  int G = (2 * sms + bh - 1) / bh;
  G = min(G, 64);
  G = min(G, topk);
  G = min(G, C);
  return max(G, 1);
}

cudaError_t launch_select_transpose(int bh, int C, int topk, const int32_t* sel, int32_t* offsets,
                                    int32_t* queries, int32_t* scratch, int* status, int sms,
                                    cudaStream_t s) {
  const int G = transpose_groups(bh, C, topk, sms);
  const size_t smem = static_cast<size_t>(C) * sizeof(int32_t);
  transpose_count_kernel<<<dim3(G, bh), kThreads, smem, s>>>(C, topk, G, sel, scratch, status);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  transpose_scan_kernel<<<bh, kThreads, smem, s>>>(C, G, scratch, offsets);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  transpose_scatter_kernel<<<dim3(G, bh), kThreads, smem, s>>>(C, topk, G, sel, scratch, queries);
  return cudaGetLastError();
}

}  // namespace vsa
