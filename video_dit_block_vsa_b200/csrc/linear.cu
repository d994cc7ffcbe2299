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
// On the tensor cores, four passes, deterministic (fixed summation order):
//   1. linear_phi_kernel   phi(q), phi(k) rounded to bf16 (the MMA operands);
//   2. linear_gemm<KV>     per (b, h) and token chunk: [KV | z] as one
//                          product phi(K_chunk)^T [V_chunk | 1] (M = 128
//                          features, N = d + 16: the appended column of ones
//                          gives z, the rest of that 16-column block is 0;
//                          both operands MN-major, K = tokens), float32
//                          partials;
//   3. linear_reduce_kernel the chunk partials summed in order and stored as
//                          the bf16 matrix B = [KV^T ; z^T ; 0] (d + 16 rows);
//   4. linear_gemm<APPLY>  per (b, h) and 128 tokens: phi(Q) B^T, whose
//                          column d is the denominator phi(q) . z; the
//                          epilogue adds num / den to the output.
// The GEMM kernel: one TMA producer warp, one MMA-issuing thread, four
// epilogue warps, a 4-stage ring, the accumulator double-buffered in TMEM.
// bf16 operands (phi(k), phi(q), KV and z rounded to bf16), float32
// accumulation.  Every wait is bounded (4 s); on a timeout the CTA records
// VSA_ERR_TIMEOUT and stops.
#include <cuda.h>

#include "common.cuh"
#include "linear.cuh"
#include "ptx.cuh"

namespace vsa {

namespace {

using namespace ptx;
using bf16 = __nv_bfloat16;

constexpr int kThreads = 256;
constexpr int kProducerWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kEpiWarp0 = 4;
constexpr int kStages = 4;
constexpr uint32_t kAtom = 64 * 128;                  // 64 rows x 128 B (SW128)
constexpr uint32_t kStageBytes = 40 * 1024;           // A 16 KB, then B (+ the ones atom)
constexpr uint32_t kBOff = 16 * 1024;
constexpr uint32_t kBarOff = kStages * kStageBytes;
constexpr size_t kSmem = 1024 + kBarOff + 256;
constexpr uint32_t kTmemCols = 512;
constexpr int kApplyRows = 128;                       // tokens per apply tile
constexpr int kChunkAlign = 64;                       // tokens per K block of the KV product

struct LinMaps {
  CUtensorMap a;  // KV: phi(k) [bh][N][d] 3-D; APPLY: phi(q) [bh][N][d] 3-D
  CUtensorMap b;  // KV: v [bh][N][d] 3-D; APPLY: B [bh (d+16)][d] 2-D
};

struct LinArgs {
  int d, bh, splits, per, m_tiles;
  long long N;
  float* partial;  // KV: [bh][splits][128][d + 16] float32
  bf16* out;       // APPLY: [bh][N][d], read and written
  int* status;
};

__device__ __forceinline__ void lin_fail(volatile int* abort_flag, int* status) {
  report(status, VSA_ERR_TIMEOUT);
  *abort_flag = 1;
}

__device__ __forceinline__ float phi(float x) { return x > 0.f ? x + 1.f : __expf(x); }

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&p);
}

// phi(x) for 8 bf16 values in a 16-byte word, rounded back to bf16.
__device__ __forceinline__ uint4 phi8(uint4 u) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    o[i] = pack2(phi(__uint_as_float(w[i] << 16)), phi(__uint_as_float(w[i] & 0xFFFF0000u)));
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// 1. phi(q), phi(k) as bf16, 8 values per thread step.
__global__ void __launch_bounds__(256) linear_phi_kernel(long long n8, const uint4* __restrict__ q,
                                                         const uint4* __restrict__ k,
                                                         uint4* __restrict__ fq,
                                                         uint4* __restrict__ fk) {
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    fq[i] = phi8(__ldg(&q[i]));
    fk[i] = phi8(__ldg(&k[i]));
  }
}

// 3. B[bh] = [KV^T ; z^T ; 0]: row e < d holds KV[:, e], row d holds z, rows
//    d+1 .. d+15 are zero; the chunk partials are summed in chunk order.
__global__ void __launch_bounds__(256) linear_reduce_kernel(int d, int splits,
                                                            const float* __restrict__ partial,
                                                            bf16* __restrict__ bmat) {
  const long long bh = blockIdx.x;
  const int pitch = d + 16;
  const float* src = partial + bh * splits * 128ll * pitch;
  bf16* dst = bmat + bh * static_cast<long long>(pitch) * d;
  for (int idx = threadIdx.x; idx < pitch * d; idx += blockDim.x) {
    const int row = idx / d, a = idx - row * d;  // output column `row`, feature a
    float t = 0.f;
    if (row <= d)
      for (int s = 0; s < splits; ++s) t += src[(static_cast<long long>(s) * 128 + a) * pitch + row];
    dst[idx] = __float2bfloat16_rn(t);
  }
}

// 2 and 4: the two products.  kApply = false: tile = (bh, chunk), C =
// phi(K)^T [V | 1] over the chunk's tokens; kApply = true: tile = (bh, 128
// tokens), C = phi(Q) B^T added to the output as num / den.
template <bool kApply>
__global__ void __launch_bounds__(kThreads, 1) linear_gemm(const __grid_constant__ LinMaps maps,
                                                           const LinArgs a) {
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
  const int d = a.d;
  const int n_cols = d + 16;
  const int atoms = d / 64;

  if (!kApply && warp >= kEpiWarp0) {
    // the ones atom of every stage: row t (a token) = [1, 0, ..., 0] in the
    // 128-byte-swizzled layout (16-byte chunk 0 of row t sits at chunk t % 8)
    for (int i = threadIdx.x - kEpiWarp0 * 32; i < kStages * 64 * 8; i += 128) {
      const int s = i / 512, r = (i / 8) % 64, c = i % 8;
      uint4* dst = reinterpret_cast<uint4*>(smem + s * kStageBytes + kBOff + atoms * kAtom + r * 128 +
                                            c * 16);
      const bool one = c == (r & 7);
      *dst = make_uint4(one ? 0x3F80u : 0u, 0u, 0u, 0u);
    }
    fence_async_smem();
  }
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
  const int tiles = kApply ? a.bh * a.m_tiles : a.bh * a.splits;
  // K blocks of a tile
  auto k_blocks = [&](int t) -> int {
    if (kApply) return atoms;
    const int s = t % a.splits;
    const long long t0 = static_cast<long long>(s) * a.per;
    const long long len = min(static_cast<long long>(a.per), a.N - t0);
    return len <= 0 ? 0 : static_cast<int>((len + kChunkAlign - 1) / kChunkAlign);
  };
  const uint32_t a_bytes = kApply ? 16u * 1024u : 2u * kAtom;
  const uint32_t b_bytes = kApply ? static_cast<uint32_t>(n_cols) * 128u : atoms * kAtom;

  if (warp == kProducerWarp) {
    uint32_t it = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
      if (*abort_flag) break;
      const int nk = k_blocks(t);
      const int bh = kApply ? t / a.m_tiles : t / a.splits;
      const int part = kApply ? t % a.m_tiles : t % a.splits;
      bool ok = true;
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int s = static_cast<int>(it % kStages);
        const uint32_t round = it / kStages;
        int w = 1;
        if (lane == 0) w = mbar_wait(&empty[s], (round & 1u) ^ 1u) ? 1 : 0;
        if (!__shfl_sync(0xffffffffu, w, 0)) {
          ok = false;
          break;
        }
        if (lane == 0) mbar_arrive_expect_tx(&full[s], a_bytes + b_bytes);
        __syncwarp();
        uint8_t* st = smem + s * kStageBytes;
        if (kApply) {
          // phi(Q) rows part*128 .., features kb*64 ..; B rows of bh, features kb*64 ..
          if (lane == 0) tma_load_3d(st, &maps.a, &full[s], kb * 64, part * kApplyRows, bh);
          if (lane == 1) tma_load_2d(st + kBOff, &maps.b, &full[s], kb * 64, bh * n_cols);
        } else {
          // tokens t0 .. t0+63 of the chunk: phi(K) features 0..127 (two atoms;
          // the second is all fill for d = 64), V features in d/64 atoms
          const int t0 = part * a.per + kb * kChunkAlign;
          if (lane < 2) tma_load_3d(st + lane * kAtom, &maps.a, &full[s], lane * 64, t0, bh);
          else if (lane < 2 + atoms)
            tma_load_3d(st + kBOff + (lane - 2) * kAtom, &maps.b, &full[s], (lane - 2) * 64, t0, bh);
        }
      }
      if (!ok) {
        if (lane == 0) lin_fail(abort_flag, a.status);
        break;
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      const uint32_t idesc = kApply ? idesc_bf16_f32(128, n_cols, false, false)
                                    : idesc_bf16_f32(128, n_cols, true, true);
      uint32_t it = 0;
      int u = 0;
      const uint32_t base = smem_u32(smem);
      for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++u) {
        if (*abort_flag) break;
        const int nk = k_blocks(t);
        const int buf = u & 1;
        if (!mbar_wait(&acc_empty[buf], ((u >> 1) & 1) ^ 1)) {
          lin_fail(abort_flag, a.status);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + buf * 256;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = static_cast<int>(it % kStages);
          const uint32_t round = it / kStages;
          if (!mbar_wait(&full[s], round & 1u)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = base + s * kStageBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            uint64_t ad, bd;
            if (kApply) {  // K-major: 16 features = 32 bytes along the row
              ad = sdesc_sw128(sa, 16, 1024) + kk * 2;
              bd = sdesc_sw128(sa + kBOff, 16, 1024) + kk * 2;
            } else {       // MN-major: 16 tokens = 16 rows of 128 bytes
              ad = sdesc_sw128(sa, kAtom, 1024) + kk * 128;
              bd = sdesc_sw128(sa + kBOff, kAtom, 1024) + kk * 128;
            }
            umma_ss(d_tmem, ad, bd, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty[s]);
        }
        if (!ok) {
          lin_fail(abort_flag, a.status);
          break;
        }
        umma_commit(&acc_full[buf]);
      }
    }
  } else if (warp >= kEpiWarp0) {
    const int wq = warp & 3;
    const int row = wq * 32 + lane;  // TMEM lane = row of the tile
    const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
    int u = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++u) {
      if (*abort_flag) break;
      const int buf = u & 1;
      const uint32_t acc = tmem + lane_addr + buf * 256;
      if (!mbar_wait(&acc_full[buf], (u >> 1) & 1)) {
        lin_fail(abort_flag, a.status);
        break;
      }
      tc_fence_after();
      if (!kApply) {
        // row = feature a: KV[a][0..d), z[a] (and the 15 zero columns)
        float* dst = a.partial + (static_cast<long long>(t) * 128 + row) * n_cols;
        for (int c = 0; c < n_cols; c += 16) {
          float v[16];
          tmem_ld16(acc + c, v);
          float4* d4 = reinterpret_cast<float4*>(dst + c);
#pragma unroll
          for (int q = 0; q < 4; ++q) d4[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
      } else {
        const int bh = t / a.m_tiles, m = t % a.m_tiles;
        const long long tok = static_cast<long long>(m) * kApplyRows + row;
        float z[16];
        tmem_ld16(acc + d, z);  // column d: phi(q) . z
        const float inv = 1.0f / z[0];
        for (int c = 0; c < d; c += 16) {
          float v[16];
          tmem_ld16(acc + c, v);
          if (tok < a.N) {
            uint4* o = reinterpret_cast<uint4*>(a.out + (static_cast<long long>(bh) * a.N + tok) * d + c);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint4 old = o[h];
              const uint32_t w[4] = {old.x, old.y, old.z, old.w};
              uint32_t nw[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int e = 8 * h + 2 * i;
                nw[i] = pack2(fmaf(v[e], inv, __uint_as_float(w[i] << 16)),
                              fmaf(v[e + 1], inv, __uint_as_float(w[i] & 0xFFFF0000u)));
              }
              o[h] = make_uint4(nw[0], nw[1], nw[2], nw[3]);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

// Token chunks per sequence for the KV product: about 296 CTAs in all (two
// per SM of a B200), at least 512 tokens per chunk; each chunk a multiple of
// 64 tokens.  Fixed, so that the workspace size does not depend on the device.
void linear_split(int bh, long long N, int* splits, int* per) {
  long long S = (296ll + bh - 1) / bh;
  const long long most = (N + 511) / 512;
  if (S > most) S = most;
  if (S < 1) S = 1;
  long long p = (N + S - 1) / S;
  p = (p + kChunkAlign - 1) / kChunkAlign * kChunkAlign;
  *per = static_cast<int>(p);
  *splits = static_cast<int>((N + p - 1) / p);
}

// Workspace: phi(q), phi(k) (bf16), the KV partials (float32), B (bf16),
// each 256-byte aligned.
LinearLayout linear_layout(int bh, long long N, int d) {
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  LinearLayout L;
  linear_split(bh, N, &L.splits, &L.per);
  const size_t act = up(static_cast<size_t>(bh) * N * d * 2);
  L.fq = 0;
  L.fk = act;
  L.partial = 2 * act;
  L.bmat = L.partial + up(static_cast<size_t>(bh) * L.splits * 128 * (d + 16) * 4);
  L.bytes = L.bmat + up(static_cast<size_t>(bh) * (d + 16) * d * 2);
  return L;
}

size_t linear_smem_bytes() { return kSmem; }

cudaError_t launch_linear_branch(int bh, long long N, int d, const void* q, const void* k,
                                 void* out, uint8_t* ws, const LinearLayout& L,
                                 const CUtensorMap& fk_map, const CUtensorMap& v_map,
                                 const CUtensorMap& fq_map, const CUtensorMap& b_map, int* status,
                                 int sms, cudaStream_t s) {
  static CtxCache<char> kv_set, apply_set;
  cudaError_t err = smem_limit_once(linear_gemm<false>, static_cast<int>(kSmem), &kv_set);
  if (err != cudaSuccess) return err;
  if ((err = smem_limit_once(linear_gemm<true>, static_cast<int>(kSmem), &apply_set)) != cudaSuccess)
    return err;
  const long long n8 = static_cast<long long>(bh) * N * d / 8;
  const int pgrid = static_cast<int>(min(n8 / 256 + 1, static_cast<long long>(sms) * 8));
  linear_phi_kernel<<<pgrid, 256, 0, s>>>(n8, static_cast<const uint4*>(q),
                                          static_cast<const uint4*>(k),
                                          reinterpret_cast<uint4*>(ws + L.fq),
                                          reinterpret_cast<uint4*>(ws + L.fk));
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  LinArgs a{};
  a.d = d;
  a.bh = bh;
  a.splits = L.splits;
  a.per = L.per;
  a.N = N;
  a.m_tiles = static_cast<int>((N + kApplyRows - 1) / kApplyRows);
  a.partial = reinterpret_cast<float*>(ws + L.partial);
  a.out = static_cast<bf16*>(out);
  a.status = status;
  const long long kv_tiles = static_cast<long long>(bh) * L.splits;
  linear_gemm<false><<<static_cast<int>(kv_tiles < sms ? kv_tiles : sms), kThreads, kSmem, s>>>(
      LinMaps{fk_map, v_map}, a);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  linear_reduce_kernel<<<bh, 256, 0, s>>>(d, L.splits, a.partial,
                                          reinterpret_cast<bf16*>(ws + L.bmat));
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  const long long ap_tiles = static_cast<long long>(bh) * a.m_tiles;
  linear_gemm<true><<<static_cast<int>(ap_tiles < sms ? ap_tiles : sms), kThreads, kSmem, s>>>(
      LinMaps{fq_map, b_map}, a);
  return cudaGetLastError();
}

}  // namespace vsa
