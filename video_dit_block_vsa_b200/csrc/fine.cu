// Fine stage of VSA: exact attention of each 64-token query cube over the
// valid tokens of its k selected key cubes (FastWan article "单块 H200 ...
// 5 秒即生一个 5 秒视频", section "一张卡，秒生视频": the fine block-sparse
// kernel over a 64x64 block mask).
//
// One CTA per (query cube, b*h); 4 warps.  Tiles move by TMA (128-byte
// swizzle) into shared memory; S = Q K^T and O += P V run on the tcgen05
// tensor cores (M = 64 rows, bf16 operands, float32 accumulators in TMEM);
// the online softmax reads S from TMEM (one query row per thread), writes
// P as bf16 into a swizzled smem tile for the second MMA and rescales O in
// TMEM when the running row maximum grows.
//
// TMEM layout for M = 64 (cta_group::1): row m of a 64-row accumulator sits
// in lane (m % 16) + 32 * (m / 16), i.e. lanes 0..15 of each warp's
// 32-lane sub-partition; thread `lane < 16` of warp w owns row 16w + lane.
//
// Every wait is bounded (4 s of wall time); on a timeout the CTA records
// VSA_ERR_TIMEOUT, skips the remaining work, frees its TMEM and exits.
#include <cuda.h>

#include "common.cuh"
#include "ptx.cuh"

namespace vsa {

namespace {

using namespace ptx;

constexpr int kThreads = 128;
constexpr uint32_t kHalfTile = 64 * 128;  // one [64 rows x 64 bf16] swizzled half tile, bytes
constexpr uint32_t kTmemCols = 256;       // S: cols [0, 64); O: cols [128, 128 + d)
constexpr uint32_t kColO = 128;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ uint32_t pack2_bf16(float a, float b) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&p);
}

template <int D>
__global__ void __launch_bounds__(kThreads) fine_fwd_kernel(
    const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
    const __grid_constant__ CUtensorMap tv, Geom g, const int32_t* __restrict__ counts,
    const int32_t* __restrict__ sel, int topk, __nv_bfloat16* __restrict__ out,
    float* __restrict__ lse, int* status) {
  constexpr int kHalves = D / 64;
  constexpr uint32_t kTile = kHalves * kHalfTile;
  constexpr uint32_t kIdescQK = idesc_bf16_f32(64, 64, false, false);  // Q K-major, K K-major
  constexpr uint32_t kIdescPV = idesc_bf16_f32(64, D, false, true);    // P K-major, V MN-major

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* Qs = smem;
  uint8_t* Ks = Qs + kTile;
  uint8_t* Vs = Ks + kTile;
  uint8_t* Ps = Vs + kTile;  // [64 rows x 64 keys] bf16, one half tile
  uint64_t* bars = reinterpret_cast<uint64_t*>(Ps + kHalfTile);  // q, kv, mma
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int i = blockIdx.x;
  const int bh = blockIdx.y;
  const int row = warp * 16 + lane;  // query row owned by this thread (lane < 16)
  const bool has_row = lane < 16;

  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 32) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    mbar_init(&bars[2], 1);
    fence_barrier_init();
    prefetch_tmap(&tq);
    prefetch_tmap(&tk);
    prefetch_tmap(&tv);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t tS = tmem + lane_off;
  const uint32_t tO = tmem + lane_off + kColO;

  const int row0 = bh * static_cast<int>(g.rows);  // first tiled row of this (b, h)
  const int ni = cube_valid(g, i);
  if (tid == 0 && counts[i] != ni) report(status, VSA_ERR_BAD_INDEX);
  const int32_t* my_sel = sel + (static_cast<long long>(bh) * g.C + i) * topk;

  if (tid == 0) {
    mbar_arrive_expect_tx(&bars[0], kTile);
#pragma unroll
    for (int h = 0; h < kHalves; ++h) tma_load_2d(Qs + h * kHalfTile, &tq, &bars[0], h * 64, row0 + i * 64);
  }
  bool timed_out = !mbar_wait(&bars[0], 0);

  const float sl2 = kLog2e / sqrtf(static_cast<float>(D));  // scores -> log2 units
  float m_run = -INFINITY, l_run = 0.f;
  uint32_t kv_phase = 0, mma_phase = 0;
  int prev = -1;

  for (int jj = 0; jj < topk && !__syncthreads_or(timed_out); ++jj) {
    int j = __ldg(&my_sel[jj]);
    if (j < 0 || j >= g.C || j <= prev) {
      if (tid == 0) report(status, VSA_ERR_BAD_INDEX);
      j = j < 0 ? 0 : (j >= g.C ? g.C - 1 : j);
    }
    prev = j;
    const int nj = cube_valid(g, j);

    // ---- K_j, V_j -> smem
    if (tid == 0) {
      mbar_arrive_expect_tx(&bars[1], 2 * kTile);
#pragma unroll
      for (int h = 0; h < kHalves; ++h) {
        tma_load_2d(Ks + h * kHalfTile, &tk, &bars[1], h * 64, row0 + j * 64);
        tma_load_2d(Vs + h * kHalfTile, &tv, &bars[1], h * 64, row0 + j * 64);
      }
    }
    timed_out |= !mbar_wait(&bars[1], kv_phase);
    kv_phase ^= 1u;
    if (__syncthreads_or(timed_out)) break;

    // ---- S = Q K^T  (M=64, N=64, K=D)
    if (tid == 0) {
      tc_fence_after();
      const uint32_t qa = smem_u32(Qs), ka = smem_u32(Ks);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * kHalfTile + (kk & 3) * 32;
        umma_ss(tmem, sdesc_sw128(qa + off, 16, 1024), sdesc_sw128(ka + off, 16, 1024),
                kIdescQK, kk > 0 ? 1u : 0u);
      }
      umma_commit(&bars[2]);
    }
    timed_out |= !mbar_wait(&bars[2], mma_phase);
    mma_phase ^= 1u;
    if (__syncthreads_or(timed_out)) break;
    tc_fence_after();

    // ---- online softmax on this thread's row
    float s[64];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float t[16];
      tmem_ld16(tS + c * 16, t);
#pragma unroll
      for (int e = 0; e < 16; ++e) s[c * 16 + e] = t[e];
    }
    float mx = -INFINITY;
#pragma unroll
    for (int e = 0; e < 64; ++e) {
      if (e >= nj) s[e] = -INFINITY;  // pad key slots
      mx = fmaxf(mx, s[e]);
    }
    const float m_new = fmaxf(m_run, mx * sl2);
    const float alpha = exp2f(m_run - m_new);
    float sum = 0.f;
#pragma unroll
    for (int e = 0; e < 64; ++e) {
      s[e] = exp2f(fmaf(s[e], sl2, -m_new));
      sum += s[e];
    }
    l_run = l_run * alpha + sum;
    m_run = m_new;
    if (has_row) {
      uint8_t* prow = Ps + row * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint4 w;
        w.x = pack2_bf16(s[8 * c + 0], s[8 * c + 1]);
        w.y = pack2_bf16(s[8 * c + 2], s[8 * c + 3]);
        w.z = pack2_bf16(s[8 * c + 4], s[8 * c + 5]);
        w.w = pack2_bf16(s[8 * c + 6], s[8 * c + 7]);
        *reinterpret_cast<uint4*>(prow + ((c ^ (row & 7)) << 4)) = w;
      }
    }
    if (jj > 0) {  // O *= alpha before accumulating this block
#pragma unroll
      for (int c = 0; c < D / 16; ++c) {
        float o[16];
        tmem_ld16(tO + c * 16, o);
#pragma unroll
        for (int e = 0; e < 16; ++e) o[e] *= alpha;
        tmem_st16(tO + c * 16, o);
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- O += P V  (M=64, N=D, K=64)
    if (tid == 0) {
      tc_fence_after();
      const uint32_t pa = smem_u32(Ps), va = smem_u32(Vs);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        umma_ss(tmem + kColO, sdesc_sw128(pa + kk * 32, 16, 1024),
                sdesc_sw128(va + kk * 2048, kHalfTile, 1024), kIdescPV,
                (jj > 0 || kk > 0) ? 1u : 0u);
      }
      umma_commit(&bars[2]);
    }
    timed_out |= !mbar_wait(&bars[2], mma_phase);
    mma_phase ^= 1u;
    tc_fence_after();
  }

  if (__syncthreads_or(timed_out)) {
    if (tid == 0) report(status, VSA_ERR_TIMEOUT);
  } else {
    // ---- epilogue: O / l -> bf16, pad rows -> 0
    const bool valid = row < ni;
    const float inv = valid ? 1.0f / l_run : 0.f;
    __nv_bfloat16* orow = out + (static_cast<long long>(row0) + i * 64 + row) * D;
#pragma unroll
    for (int c = 0; c < D / 16; ++c) {
      float o[16];
      tmem_ld16(tO + c * 16, o);
      if (!valid) {
#pragma unroll
        for (int e = 0; e < 16; ++e) o[e] = 0.f;
      }
      if (has_row) {
        uint4 w0, w1;
        w0.x = pack2_bf16(o[0] * inv, o[1] * inv);
        w0.y = pack2_bf16(o[2] * inv, o[3] * inv);
        w0.z = pack2_bf16(o[4] * inv, o[5] * inv);
        w0.w = pack2_bf16(o[6] * inv, o[7] * inv);
        w1.x = pack2_bf16(o[8] * inv, o[9] * inv);
        w1.y = pack2_bf16(o[10] * inv, o[11] * inv);
        w1.z = pack2_bf16(o[12] * inv, o[13] * inv);
        w1.w = pack2_bf16(o[14] * inv, o[15] * inv);
        reinterpret_cast<uint4*>(orow + c * 16)[0] = w0;
        reinterpret_cast<uint4*>(orow + c * 16)[1] = w1;
      }
    }
    if (lse != nullptr && has_row) {
      lse[static_cast<long long>(row0) + i * 64 + row] =
          valid ? (m_run + log2f(l_run)) * kLn2 : -INFINITY;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

// Shared memory request: the tiles plus alignment slack, raised to 100 KB so
// that at most two CTAs share an SM and their TMEM (2 x 256 columns) fits.
size_t fine_smem_bytes(int d) {
  const size_t need = 1024 /* alignment slack */ + 3 * (d / 64) * kHalfTile + kHalfTile + 64;
  return need > 100 * 1024 ? need : 100 * 1024;
}

cudaError_t launch_block_sparse_fwd(const Geom& g, const CUtensorMap& tq, const CUtensorMap& tk,
                                    const CUtensorMap& tv, const int32_t* counts,
                                    const int32_t* sel, int topk, void* out, float* lse,
                                    int* status, cudaStream_t s) {
  const size_t smem = fine_smem_bytes(g.d);
  dim3 grid(static_cast<unsigned>(g.C), static_cast<unsigned>(g.B * g.H));
  cudaError_t err;
  if (g.d == 128) {
    err = cudaFuncSetAttribute(fine_fwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    fine_fwd_kernel<128><<<grid, kThreads, smem, s>>>(tq, tk, tv, g, counts, sel, topk,
                                                       static_cast<__nv_bfloat16*>(out), lse, status);
  } else {
    err = cudaFuncSetAttribute(fine_fwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    fine_fwd_kernel<64><<<grid, kThreads, smem, s>>>(tq, tk, tv, g, counts, sel, topk,
                                                      static_cast<__nv_bfloat16*>(out), lse, status);
  }
  return cudaGetLastError();
}

// Diagnostic kernel: waits on a barrier nothing arrives at, with the same
// bounded wait as the fine kernel, and records the timeout.
__global__ void debug_wait_kernel(uint64_t limit_ns, int* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (!mbar_wait(&bar, 0, limit_ns) && threadIdx.x == 0) report(status, VSA_ERR_TIMEOUT);
}

cudaError_t launch_debug_wait(uint64_t limit_ns, int* status, cudaStream_t s) {
  debug_wait_kernel<<<1, 32, 0, s>>>(limit_ns, status);
  return cudaGetLastError();
}

}  // namespace vsa
