// Projections of a DiT attention block with VSA's layout changes fused in
// (FastWan news article "单块 H200 ... 5 秒即生一个 5 秒视频", section
// "一张卡，秒生视频": the end-to-end figures come from whole DiT blocks, where
// VSA sits between the QKV projection and the output projection):
//   qkv  [q | k | v] = x W_qkv^T, written straight into the tiled layout: the
//        product's row for token n of batch b goes to tiled row
//        64 cube(n) + slot(n) of (b, h) in q_t, k_t or v_t (the tile
//        permutation in the epilogue);
//   out  y = o W_o^T with o read from the tiled layout (rows cube-major, the
//        K blocks walking the heads), each row written to its token (the
//        untile in the epilogue; pad rows are skipped).
// One tcgen05 GEMM kernel serves both: 128 x 256 output tiles, K in blocks
// of 64 (one 128-byte swizzle atom) through a 4-stage TMA ring, one thread
// issuing M = 128, N = 256, K = 16 MMAs, the accumulator double-buffered in
// TMEM (2 x 256 columns) so that the four epilogue warps drain one tile while
// the next one accumulates.  Persistent CTAs walk the tiles in bands of 16
// row tiles (all column tiles of a band before the next band), so a band's
// activations and the weight tiles in flight stay in L2.  Every wait is
// bounded (4 s); on a timeout the CTA records VSA_ERR_TIMEOUT and stops.
#include <cuda.h>

#include "common.cuh"
#include "ptx.cuh"

namespace vsa {

namespace {

using namespace ptx;
using bf16 = __nv_bfloat16;

constexpr int kThreads = 256;
constexpr int kProducerWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kEpiWarp0 = 4;
constexpr int kTileM = 128, kTileN = 256, kTileK = 64;
constexpr int kStages = 4;
constexpr int kBand = 16;                                   // row tiles per band
constexpr uint32_t kABytes = kTileM * kTileK * 2;           // 16 KB
constexpr uint32_t kBBytes = kTileN * kTileK * 2;           // 32 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t kBarOff = kStages * kStageBytes;
constexpr size_t kSmem = 1024 + kBarOff + 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kIdesc = idesc_bf16_f32(kTileM, kTileN, false, false);

struct ProjMaps {
  CUtensorMap a;  // activations: x [B N, hidden] (qkv) or tiled o [B H 64C, d] (out)
  CUtensorMap b;  // weights [out features, in features]
};

struct ProjArgs {
  Geom g;
  int mode;          // 0: qkv (scatter to the tiled layout), 1: out (gather from it)
  int hidden;
  int m_tiles;       // row tiles per batch (qkv: over all B N rows, one "batch")
  int batches;       // 1 (qkv) or B (out)
  int n_tiles;
  int k_blocks;
  int n_out;         // output features: 3 H d (qkv) or hidden (out)
  bf16* out0;        // qkv: q_t, k_t, v_t; out: y
  bf16* out1;
  bf16* out2;
  int* status;
};

struct Tile {
  int b, mt, nt;
};

__device__ __forceinline__ Tile tile_of(const ProjArgs& a, int t) {
  // bands of kBand row tiles; inside a band, column tiles outer
  const int per_batch = a.m_tiles * a.n_tiles;
  Tile r;
  r.b = t / per_batch;
  int rem = t - r.b * per_batch;
  const int band = rem / (kBand * a.n_tiles);
  const int band0 = band * kBand;
  const int rows_in_band = min(kBand, a.m_tiles - band0);
  rem -= band * kBand * a.n_tiles;
  r.nt = rem / rows_in_band;
  r.mt = band0 + (rem - r.nt * rows_in_band);
  return r;
}

// Row of the A tensor map for row tile mt, K block kb.
__device__ __forceinline__ int a_row(const ProjArgs& a, const Tile& tl, int kb) {
  if (a.mode == 0) return tl.mt * kTileM;
  const int per_head = a.g.d / kTileK;  // K blocks per head
  const int h = kb / per_head;
  return static_cast<int>((static_cast<long long>(tl.b) * a.g.H + h) * a.g.rows) + tl.mt * kTileM;
}

__device__ __forceinline__ int a_col(const ProjArgs& a, int kb) {
  if (a.mode == 0) return kb * kTileK;
  return (kb % (a.g.d / kTileK)) * kTileK;
}

__device__ __forceinline__ void proj_fail(volatile int* abort_flag, int* status) {
  report(status, VSA_ERR_TIMEOUT);
  *abort_flag = 1;
}

// Tiled row (64 cube + slot) of token n of a (b, h) sequence.
__device__ __forceinline__ long long tiled_row(const Geom& g, long long n) {
  const long long yx = static_cast<long long>(g.Y) * g.X;
  const int t = static_cast<int>(n / yx);
  const int rem = static_cast<int>(n - t * yx);
  const int y = rem / g.X, x = rem - y * g.X;
  const int c = ((t >> 2) * g.Cy + (y >> 2)) * g.Cx + (x >> 2);
  const int ny = min(4, g.Y - (y & ~3)), nx = min(4, g.X - (x & ~3));
  const int slot = ((t & 3) * ny + (y & 3)) * nx + (x & 3);
  return static_cast<long long>(c) * kSlots + slot;
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&p);
}

__global__ void __launch_bounds__(kThreads, 1) proj_kernel(const __grid_constant__ ProjMaps maps,
                                                           const ProjArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOff);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* acc_full = bars + 2 * kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&maps.a);
    prefetch_tmap(&maps.b);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int tiles = a.batches * a.m_tiles * a.n_tiles;

  if (warp == kProducerWarp) {
    uint32_t it = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
      if (*abort_flag) break;
      const Tile tl = tile_of(a, t);
      for (int kb = 0; kb < a.k_blocks; ++kb, ++it) {
        const int s = static_cast<int>(it % kStages);
        const uint32_t round = it / kStages;
        int ok = 1;
        if (lane == 0) ok = mbar_wait(&empty[s], (round & 1u) ^ 1u) ? 1 : 0;
        if (!__shfl_sync(0xffffffffu, ok, 0)) {
          if (lane == 0) proj_fail(abort_flag, a.status);
          break;
        }
        if (lane == 0) mbar_arrive_expect_tx(&full[s], kStageBytes);
        __syncwarp();
        uint8_t* st = smem + s * kStageBytes;
        if (lane == 0) tma_load_2d(st, &maps.a, &full[s], a_col(a, kb), a_row(a, tl, kb));
        if (lane == 1) tma_load_2d(st + kABytes, &maps.b, &full[s], kb * kTileK, tl.nt * kTileN);
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      uint32_t it = 0;
      int u = 0;
      const uint32_t base = smem_u32(smem);
      for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++u) {
        if (*abort_flag) break;
        const int buf = u & 1;
        if (!mbar_wait(&acc_empty[buf], ((u >> 1) & 1) ^ 1)) {
          proj_fail(abort_flag, a.status);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + buf * kTileN;
        bool ok = true;
        for (int kb = 0; kb < a.k_blocks; ++kb, ++it) {
          const int s = static_cast<int>(it % kStages);
          const uint32_t round = it / kStages;
          if (!mbar_wait(&full[s], round & 1u)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = base + s * kStageBytes;
          const uint64_t adesc = sdesc_sw128(sa, 16, 1024);
          const uint64_t bdesc = sdesc_sw128(sa + kABytes, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < kTileK / 16; ++kk)
            umma_ss(d_tmem, adesc + kk * 2, bdesc + kk * 2, kIdesc, (kb > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&empty[s]);
        }
        if (!ok) {
          proj_fail(abort_flag, a.status);
          break;
        }
        umma_commit(&acc_full[buf]);
      }
    }
  } else if (warp >= kEpiWarp0) {
    const int wq = warp & 3;
    const int row = wq * 32 + lane;  // TMEM lane = row of the tile
    const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
    const Geom& g = a.g;
    int u = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++u) {
      if (*abort_flag) break;
      const Tile tl = tile_of(a, t);
      const int buf = u & 1;
      if (!mbar_wait(&acc_full[buf], (u >> 1) & 1)) {
        proj_fail(abort_flag, a.status);
        break;
      }
      tc_fence_after();
      // destination of this thread's row
      bool valid;
      long long m = static_cast<long long>(tl.mt) * kTileM + row;
      long long b = 0, trow = 0, tok = 0;
      if (a.mode == 0) {
        valid = m < static_cast<long long>(g.B) * g.N;
        if (valid) {
          b = m / g.N;
          trow = tiled_row(g, m - b * g.N);
        }
      } else {
        valid = m < g.rows;
        if (valid) {
          const int c = static_cast<int>(m >> 6);
          const long long n = slot_token(g, c, static_cast<int>(m & 63));
          valid = n >= 0;
          tok = static_cast<long long>(tl.b) * g.N + n;
        }
      }
#pragma unroll 1
      for (int ch = 0; ch < kTileN / 32; ++ch) {
        float v[16];
        uint32_t w[16];
        float v2[16];
        tmem_ld16(tmem + lane_addr + buf * kTileN + ch * 32, v);
        tmem_ld16(tmem + lane_addr + buf * kTileN + ch * 32 + 16, v2);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          w[e] = pack2(v[2 * e], v[2 * e + 1]);
          w[8 + e] = pack2(v2[2 * e], v2[2 * e + 1]);
        }
        const int col = tl.nt * kTileN + ch * 32;  // first output feature of the chunk
        if (!valid || col >= a.n_out) continue;
        bf16* dst;
        if (a.mode == 0) {
          const int hd = g.H * g.d;
          const int part = col / hd, rem = col - part * hd;
          const int h = rem / g.d, e0 = rem - h * g.d;
          bf16* t0 = part == 0 ? a.out0 : (part == 1 ? a.out1 : a.out2);
          dst = t0 + ((b * g.H + h) * g.rows + trow) * g.d + e0;
        } else {
          dst = a.out0 + tok * a.hidden + col;
        }
        uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
        for (int q = 0; q < 4; ++q) d4[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

// Zeroes the pad rows of the tiled q, k, v (cubes with fewer than 64 tokens)
// and writes the cube counts.  One warp per (cube, tensor) of a (b, h).
__global__ void __launch_bounds__(256) pad_rows_kernel(Geom g, uint4* __restrict__ q,
                                                       uint4* __restrict__ k,
                                                       uint4* __restrict__ v,
                                                       int32_t* __restrict__ counts) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x * 8 + warp;
  if (c >= g.C) return;
  const long long bh = blockIdx.y;
  const int which = blockIdx.z;
  const int n = cube_valid(g, c);
  if (counts != nullptr && bh == 0 && which == 0 && lane == 0) counts[c] = n;
  if (n == kSlots) return;
  uint4* t = which == 0 ? q : (which == 1 ? k : v);
  const int per_row = g.d / 8;  // 16-byte chunks per row
  uint4* base = t + (bh * g.rows + static_cast<long long>(c) * kSlots) * per_row;
  for (int i = n * per_row + lane; i < kSlots * per_row; i += 32) base[i] = make_uint4(0u, 0u, 0u, 0u);
}

}  // namespace

size_t proj_smem_bytes() { return kSmem; }

cudaError_t launch_projection(const Geom& g, int mode, int hidden, const CUtensorMap& amap,
                              const CUtensorMap& bmap, void* out0, void* out1, void* out2,
                              int32_t* counts, int* status, int sms, cudaStream_t s) {
  static CtxCache<char> limit_set;
  cudaError_t err = smem_limit_once(proj_kernel, static_cast<int>(kSmem), &limit_set);
  if (err != cudaSuccess) return err;
  ProjMaps maps{amap, bmap};
  ProjArgs a{};
  a.g = g;
  a.mode = mode;
  a.hidden = hidden;
  if (mode == 0) {
    const long long M = static_cast<long long>(g.B) * g.N;
    a.m_tiles = static_cast<int>((M + kTileM - 1) / kTileM);
    a.batches = 1;
    a.n_out = 3 * g.H * g.d;
    a.k_blocks = (hidden + kTileK - 1) / kTileK;
  } else {
    a.m_tiles = static_cast<int>((g.rows + kTileM - 1) / kTileM);
    a.batches = g.B;
    a.n_out = hidden;
    a.k_blocks = g.H * (g.d / kTileK);
  }
  a.n_tiles = (a.n_out + kTileN - 1) / kTileN;
  a.out0 = static_cast<bf16*>(out0);
  a.out1 = static_cast<bf16*>(out1);
  a.out2 = static_cast<bf16*>(out2);
  a.status = status;
  if (mode == 0) {
    dim3 pg(static_cast<unsigned>((g.C + 7) / 8), static_cast<unsigned>(g.B * g.H), 3);
    pad_rows_kernel<<<pg, 256, 0, s>>>(g, static_cast<uint4*>(out0), static_cast<uint4*>(out1),
                                       static_cast<uint4*>(out2), counts);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  const long long tiles = static_cast<long long>(a.batches) * a.m_tiles * a.n_tiles;
  const int grid = static_cast<int>(tiles < sms ? tiles : sms);
  proj_kernel<<<grid, kThreads, kSmem, s>>>(maps, a);
  return cudaGetLastError();
}

}  // namespace vsa
