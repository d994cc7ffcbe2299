// Transpose of the top-k selection: for every key cube, the query cubes that
// selected it, in ascending order (a CSR list per (b, h)).  The key-stationary
// half of a backward pass (dK, dV of one key cube accumulated over the query
// cubes that attended to it) walks these lists.
//
// One CTA per (b, h):
//   1. count, per key cube, how many query cubes selected it (shared atomics);
//   2. exclusive scan of the counts -> offsets;
//   3. scatter every (query i, key j) pair into j's segment at a claimed slot;
//   4. order each segment: a query cube selects a key cube at most once, so
//      the query indices of a segment are distinct and each one's position is
//      its rank among them (computed directly, no data-dependent swaps).
#include "common.cuh"

namespace vsa {

namespace {

constexpr int kTransposeThreads = 1024;

__global__ void __launch_bounds__(kTransposeThreads) select_transpose_kernel(
    int C, int topk, const int32_t* __restrict__ sel, int32_t* __restrict__ offsets,
    int32_t* __restrict__ queries, int32_t* __restrict__ scratch, int* status) {
  extern __shared__ int32_t cnt[];  // C + 1 counters, then reused as cursors
  const long long bh = blockIdx.x;
  const int32_t* s = sel + bh * C * topk;
  int32_t* off = offsets + bh * (C + 1);
  int32_t* out = queries + bh * C * topk;
  int32_t* tmp = scratch + bh * C * topk;
  const int tid = threadIdx.x;
  const long long pairs = static_cast<long long>(C) * topk;

  for (int j = tid; j <= C; j += blockDim.x) cnt[j] = 0;
  __syncthreads();
  for (long long p = tid; p < pairs; p += blockDim.x) {
    const int j = s[p];
    if (j < 0 || j >= C) {
      report(status, VSA_ERR_BAD_INDEX);
      continue;
    }
    atomicAdd(&cnt[j], 1);
  }
  __syncthreads();
  // exclusive scan of cnt[0..C) by one warp: each lane scans a contiguous run
  if (tid < 32) {
    const int per = (C + 31) / 32;
    const int lo = min(C, tid * per), hi = min(C, lo + per);
    int run = 0;
    for (int j = lo; j < hi; ++j) run += cnt[j];
    int incl = run;
    for (int d = 1; d < 32; d <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, d);
      if (tid >= d) incl += o;
    }
    int base = incl - run;
    for (int j = lo; j < hi; ++j) {
      const int c = cnt[j];
      off[j] = base;
      cnt[j] = base;  // becomes the segment's fill cursor
      base += c;
    }
    if (tid == 31) off[C] = incl;
  }
  __syncthreads();
  // scatter query indices into their key segments (order inside a segment arbitrary)
  for (long long p = tid; p < pairs; p += blockDim.x) {
    const int j = s[p];
    if (j < 0 || j >= C) continue;
    const int slot = atomicAdd(&cnt[j], 1);
    tmp[slot] = static_cast<int32_t>(p / topk);
  }
  __syncthreads();
  // order each segment by rank: entry e of segment [a, b) goes to a + #{smaller}
  const int total = off[C];  // pairs with a valid key index
  for (int e = tid; e < total; e += blockDim.x) {
    const int q = tmp[e];
    // the segment holding e: off[lo] <= e < off[lo + 1] (off is non-decreasing,
    // so the binary search lands on the non-empty segment)
    int lo = 0, hi = C;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (off[mid] <= e) lo = mid; else hi = mid;
    }
    const int a = off[lo], b = off[lo + 1];
    int rank = 0;
    for (int f = a; f < b; ++f) rank += tmp[f] < q ? 1 : 0;
    out[a + rank] = q;
  }
}

}  // namespace

cudaError_t launch_select_transpose(int bh, int C, int topk, const int32_t* sel, int32_t* offsets,
                                    int32_t* queries, int32_t* scratch, int* status,
                                    cudaStream_t s) {
  const size_t smem = static_cast<size_t>(C + 1) * sizeof(int32_t);
  select_transpose_kernel<<<bh, kTransposeThreads, smem, s>>>(C, topk, sel, offsets, queries,
                                                                scratch, status);
  return cudaGetLastError();
}

}  // namespace vsa
