// Coarse stage of VSA (FastWan article "单块 H200 ... 5 秒即生一个 5 秒视频",
// section "一张卡，秒生视频", Fig. 5 paragraph; dynamic key selection in
// section "传统零散郑重力，为何会在蒸馏中失效？").
//
// 1. pool_kernel: qbar, kbar, vbar = mean of each cube's n_c valid rows
//    (float32), an HBM-bound pass over the three tiled tensors, or over the
//    token-order tensors (so the coarse stage need not wait for the tiling).
// 2. coarse_kernel: for a tile of R query cubes of one (b, h):
//      S_c[i, :] = qbar_i kbar^T / sqrt(d)       (float32, row kept in smem)
//      sel[i]    = top-k of S_c[i, :], ties to the lower index, ascending
//      O_c[i]    = softmax(S_c[i, :]) vbar
//    The per-row top-k is a warp-level MSB-first radix select on the
//    order-preserving integer image of the float logits (kept in registers
//    for rows of up to 1536 cubes), followed by one ballot-compaction pass in
//    index order (so the output is ascending and equal logits are taken
//    lowest index first).
#include <cmath>

#include "common.cuh"

namespace vsa {

namespace {

constexpr int kCoarseThreads = 256;
constexpr int kLogitBudgetBytes = 132 * 1024;

// ------------------------------------------------------------------ pooling
// One warp per (tensor, b*h, cube).  A row of d bf16 is d/8 16-byte chunks;
// the warp covers 32/(d/8) rows per step and reduces across row groups at the end.
// With token-order input and tiled outputs given, the same pass also writes the
// tiled tensors (valid rows copied, pad rows zero) and the cube counts: the
// tiling and the pooling then cost one read of q, k, v.
__global__ void __launch_bounds__(256) pool_kernel(Geom g, const uint4* __restrict__ q,
                                                   const uint4* __restrict__ k,
                                                   const uint4* __restrict__ v,
                                                   const int32_t* __restrict__ counts,
                                                   float* __restrict__ ws, int* status,
                                                   bool token_order, uint4* __restrict__ qt,
                                                   uint4* __restrict__ kt,
                                                   uint4* __restrict__ vt,
                                                   int32_t* __restrict__ counts_out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long item = static_cast<long long>(blockIdx.x) * 8 + warp;  // (b*h, cube)
  const long long items = static_cast<long long>(g.B) * g.H * g.C;
  if (item >= items) return;
  const int which = blockIdx.y;  // 0 q, 1 k, 2 v
  const uint4* src = which == 0 ? q : (which == 1 ? k : v);
  const long long bh = item / g.C;
  const int c = static_cast<int>(item - bh * g.C);
  const int n = cube_valid(g, c);
  if (which == 0 && lane == 0 && counts != nullptr && counts[c] != n)
    report(status, VSA_ERR_BAD_INDEX);

  const int chunks = g.d >> 3;         // 8 or 16
  const int rows_per_step = 32 / chunks;  // 4 or 2
  const int ch = lane % chunks;
  const int r0 = lane / chunks;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  // tiled input: the cube's valid rows are its first n rows; token-order input:
  // row r of the cube is token slot_token(c, r) of the (b, h) plane
  const uint4* base = token_order ? src + bh * g.N * chunks
                                  : src + (bh * g.rows + static_cast<long long>(c) * kSlots) * chunks;
  uint4* tiled = which == 0 ? qt : (which == 1 ? kt : vt);
  if (tiled != nullptr) tiled += (bh * g.rows + static_cast<long long>(c) * kSlots) * chunks;
  if (counts_out != nullptr && which == 0 && bh == 0 && lane == 0) counts_out[c] = n;
#pragma unroll 4
  for (int r = r0; r < n; r += rows_per_step) {
    const long long row = token_order ? slot_token(g, c, r) : r;
    const uint4 w = __ldg(&base[row * chunks + ch]);
    if (tiled != nullptr) tiled[r * chunks + ch] = w;
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[2 * e] += __uint_as_float(u[e] << 16);
      acc[2 * e + 1] += __uint_as_float(u[e] & 0xFFFF0000u);
    }
  }
  if (tiled != nullptr) {  // pad rows of the tiled copy
    for (int r = r0; r < kSlots; r += rows_per_step)
      if (r >= n) tiled[r * chunks + ch] = make_uint4(0u, 0u, 0u, 0u);
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

// Keys of a row cached in registers per lane (rows of up to 32 * kTopkRegs
// cubes never re-read shared memory during the selection).
constexpr int kTopkRegs = 48;

// Writes the indices of the k largest of row[0..C) (ties: lower index first)
// to out[0..k): first the key cubes holding more than 16 valid tokens, then
// the others, each group in ascending order.  Executed by one full warp; hist
// is a warp-private 256-entry smem array.  Most-significant-digit-first radix
// select over the order-preserving integer image of the floats, 8 bits per
// pass, then one ballot-compaction pass in index order.
__device__ void warp_topk(const Geom& g, const float* row, int C, int k, int* hist,
                          int32_t* out) {
  const int lane = threadIdx.x & 31;
  uint32_t kc[kTopkRegs];
#pragma unroll
  for (int u = 0; u < kTopkRegs; ++u) {
    const int j = lane + 32 * u;
    kc[u] = j < C ? order_key(row[j]) : 0u;
  }
  uint32_t prefix = 0u, mask = 0u;
  int remaining = k;  // rank of the wanted key among the keys matching the prefix
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = lane; b < 256; b += 32) hist[b] = 0;
    __syncwarp();
#pragma unroll
    for (int u = 0; u < kTopkRegs; ++u) {
      const int j = lane + 32 * u;
      if (j < C && (kc[u] & mask) == prefix) atomicAdd(&hist[(kc[u] >> shift) & 255u], 1);
    }
    for (int j = lane + 32 * kTopkRegs; j < C; j += 32) {
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
  // `remaining` keys equal to it in index order.  One pass in index order
  // writes the taken key cubes with more than 16 valid tokens from the front
  // of out[] and the others from the back; reversing the back part then
  // leaves both groups ascending, wide ones first (the order the fine kernel
  // packs key rows in).
  const unsigned lt = (1u << lane) - 1u;
  int pos_w = 0, pos_n = 0, eq_seen = 0;
  auto take_window = [&](int j, uint32_t key) {
    const bool gt = j < C && key > prefix;
    const bool eq = j < C && key == prefix;
    const unsigned eqm = __ballot_sync(0xffffffffu, eq);
    const bool take = gt || (eq && eq_seen + __popc(eqm & lt) < remaining);
    const bool wide = cube_valid(g, j < C ? j : 0) > 16;
    const unsigned wm = __ballot_sync(0xffffffffu, take && wide);
    const unsigned nm = __ballot_sync(0xffffffffu, take && !wide);
    if (take && wide) out[pos_w + __popc(wm & lt)] = j;
    if (take && !wide) out[k - 1 - (pos_n + __popc(nm & lt))] = j;
    pos_w += __popc(wm);
    pos_n += __popc(nm);
    eq_seen += __popc(eqm);
  };
#pragma unroll
  for (int u = 0; u < kTopkRegs; ++u) take_window(lane + 32 * u, kc[u]);
  for (int j0 = 32 * kTopkRegs; j0 < C; j0 += 32) {
    const int j = j0 + lane;
    take_window(j, j < C ? order_key(row[j]) : 0u);
  }
  __syncwarp();
  // out[pos_w .. k) holds the narrow cubes in descending order: reverse it
  for (int a = lane; a < pos_n / 2; a += 32) {
    const int x = out[pos_w + a], y = out[k - 1 - a];
    out[pos_w + a] = y;
    out[k - 1 - a] = x;
  }
}

// ------------------------------------------------------------------ coarse
// grid (ceil(C/R), B*H), 256 threads, R <= 16 query cubes per CTA.
// smem: S [R][Cp] f32 (Cp = C rounded up to 4) | qT [d][16] | staging
// (key slices [512][33], then value chunks [132][d]) | hist [8][256].
//
// Logits: a 16-row x 512-key tile per pass; thread t owns rows 8*(t/128)..+7
// and keys (t%128) + 128*b, b < 4 (32 accumulators), over head-dim slices of
// 32 staged row-major at a pitch of 33 floats: the four key loads of a step
// hit 32 distinct banks per warp, the eight query values are two broadcast
// 128-bit loads, so a step is six smem wavefronts per warp for 32 FMAs, and
// the staging stores are conflict-free too.
// O_c: thread t owns rows 4*(t/64)..+3 and d/64 adjacent columns.
constexpr int kTileKeys = 512;
constexpr int kSlice = 32;
constexpr int kStagePitch = kSlice + 1;
constexpr int kStageFloats = kTileKeys * kStagePitch;

__global__ void __launch_bounds__(kCoarseThreads) coarse_kernel(
    Geom g, int R, int topk, const float* __restrict__ ws, float* __restrict__ o_coarse,
    int32_t* __restrict__ sel, float* __restrict__ logits_out) {
  extern __shared__ __align__(16) float sm[];
  const int C = g.C, d = g.d;
  const int Cp = (C + 3) & ~3;
  float* S = sm;                                     // [R][Cp]
  float* qT = S + static_cast<size_t>(R) * Cp;       // [d][16]
  float* stage = qT + static_cast<size_t>(d) * 16;   // kStageFloats
  int* hist = reinterpret_cast<int*>(stage + kStageFloats);  // [8][256]

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
  const int rg = tid >> 7, kg = tid & 127;
  for (int j0 = 0; j0 < C; j0 += kTileKeys) {
    float acc[8][4];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
    for (int e0 = 0; e0 < d; e0 += kSlice) {
      __syncthreads();
      // stage keys j0..j0+511, dims e0..e0+31: stage[key][dim], pitch 33
      for (int idx = tid; idx < kTileKeys * (kSlice / 4); idx += kCoarseThreads) {
        const int jj = idx >> 3, q4 = idx & 7;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (j0 + jj < C)
          v = *reinterpret_cast<const float4*>(kbar + static_cast<long long>(j0 + jj) * d + e0 + 4 * q4);
        float* dst = stage + jj * kStagePitch + 4 * q4;
        dst[0] = v.x;
        dst[1] = v.y;
        dst[2] = v.z;
        dst[3] = v.w;
      }
      __syncthreads();
      const float* qcol = qT + e0 * 16 + 8 * rg;
      const float* krow = stage + kg * kStagePitch;
#pragma unroll 4
      for (int ee = 0; ee < kSlice; ++ee) {
        const float4 qa = *reinterpret_cast<const float4*>(qcol + ee * 16);
        const float4 qb = *reinterpret_cast<const float4*>(qcol + ee * 16 + 4);
        const float qv[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
        float kv[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) kv[b] = krow[b * 128 * kStagePitch + ee];
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(qv[a], kv[b], acc[a][b]);
      }
    }
#pragma unroll
    for (int a = 0; a < 8; ++a) {
      const int r = 8 * rg + a;
      if (r >= rows) continue;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int j = j0 + kg + 128 * b;
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
    warp_topk(g, row, C, topk, hist + warp * 256,
              sel + (static_cast<long long>(bh) * C + i0 + r) * topk);
    float mx = -INFINITY;
#pragma unroll 8
    for (int j = lane; j < C; j += 32) mx = fmaxf(mx, row[j]);
    for (int off = 16; off; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    float z = 0.f;
#pragma unroll 8
    for (int j = lane; j < C; j += 32) {
      const float p = expf(row[j] - mx);
      row[j] = p;
      z += p;
    }
    for (int off = 16; off; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
    const float inv = 1.0f / z;
    __syncwarp();
#pragma unroll 8
    for (int j = lane; j < Cp; j += 32) row[j] = j < C ? row[j] * inv : 0.f;
  }
  if (o_coarse == nullptr) return;
  // ---- O_c = P vbar: rows 4*(t/64)..+3; columns cpt*(t%64) .. +cpt-1
  const int cpt = d / 64;  // 2 (d=128) or 1 (d=64)
  const int r0 = 4 * (tid >> 6), c0 = cpt * (tid & 63);
  float o[4][2] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
  const int vchunk = (kStageFloats / d) & ~3;  // value rows per staged chunk
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
      for (int jj = 0; jj < nk; jj += 4) {
        float pv[4][4];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          const float4 p = *reinterpret_cast<const float4*>(p0 + a * Cp + jj);
          pv[a][0] = p.x; pv[a][1] = p.y; pv[a][2] = p.z; pv[a][3] = p.w;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float* vrow = stage + (jj + u) * d + c0;
          if (cpt == 2) {
            const float2 v = *reinterpret_cast<const float2*>(vrow);
#pragma unroll
            for (int a = 0; a < 4; ++a) {
              o[a][0] = fmaf(pv[a][u], v.x, o[a][0]);
              o[a][1] = fmaf(pv[a][u], v.y, o[a][1]);
            }
          } else {
            const float v = *vrow;
#pragma unroll
            for (int a = 0; a < 4; ++a) o[a][0] = fmaf(pv[a][u], v, o[a][0]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    if (r0 + a >= rows) break;
    float* dst = o_coarse + (static_cast<long long>(bh) * C + i0 + r0 + a) * d + c0;
    if (cpt == 2)
      *reinterpret_cast<float2*>(dst) = make_float2(o[a][0], o[a][1]);
    else
      *dst = o[a][0];
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
  return (R * Cp + static_cast<size_t>(d) * 16 + static_cast<size_t>(kStageFloats)) *
             sizeof(float) + 8 * 256 * sizeof(int);
}

cudaError_t launch_coarse_only(const Geom& g, int topk, float* o_coarse, int32_t* sel,
                               float* logits, const float* ws, cudaStream_t s);

cudaError_t launch_coarse_select(const Geom& g, const void* qt, const void* kt, const void* vt,
                                 const int32_t* counts, int topk, float* o_coarse,
                                 int32_t* sel, float* logits, float* ws, int* status,
                                 cudaStream_t s, bool token_order) {
  const long long items = static_cast<long long>(g.B) * g.H * g.C;
  dim3 pg(static_cast<unsigned>((items + 7) / 8), 3);
  pool_kernel<<<pg, 256, 0, s>>>(g, static_cast<const uint4*>(qt), static_cast<const uint4*>(kt),
                                 static_cast<const uint4*>(vt), counts, ws, status, token_order,
                                 nullptr, nullptr, nullptr, nullptr);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  return launch_coarse_only(g, topk, o_coarse, sel, logits, ws, s);
}

cudaError_t launch_tile_pool(const Geom& g, const void* q, const void* k, const void* v,
                             void* qt, void* kt, void* vt, int32_t* counts, float* ws,
                             int* status, cudaStream_t s) {
  const long long items = static_cast<long long>(g.B) * g.H * g.C;
  dim3 pg(static_cast<unsigned>((items + 7) / 8), 3);
  pool_kernel<<<pg, 256, 0, s>>>(g, static_cast<const uint4*>(q), static_cast<const uint4*>(k),
                                 static_cast<const uint4*>(v), nullptr, ws, status, true,
                                 static_cast<uint4*>(qt), static_cast<uint4*>(kt),
                                 static_cast<uint4*>(vt), counts);
  return cudaGetLastError();
}

cudaError_t launch_coarse_only(const Geom& g, int topk, float* o_coarse, int32_t* sel,
                               float* logits, const float* ws, cudaStream_t s) {
  cudaError_t err;
  const int R = coarse_rows_per_cta(g.C, g.d);
  const size_t smem = coarse_smem_bytes(g.C, g.d, R);
  // the limit is raised once per device to the largest block any accepted
  // shape needs: the logits block never exceeds kLogitBudgetBytes, plus qT
  // for d = 128, the staging buffer and the top-k histograms
  static CtxCache<char> limit_set;
  const size_t most = kLogitBudgetBytes + (static_cast<size_t>(128) * 16 + kStageFloats) * sizeof(float) +
                      8 * 256 * sizeof(int);
  err = smem_limit_once(coarse_kernel, static_cast<int>(most), &limit_set);
  if (err != cudaSuccess) return err;
  if (smem > most) return cudaErrorInvalidValue;
  dim3 cg(static_cast<unsigned>((g.C + R - 1) / R), static_cast<unsigned>(g.B * g.H));
  coarse_kernel<<<cg, kCoarseThreads, smem, s>>>(g, R, topk, ws, o_coarse, sel, logits);
  return cudaGetLastError();
}

}  // namespace vsa
