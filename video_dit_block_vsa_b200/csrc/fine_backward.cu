// Backward of the fine block-sparse attention on the tensor cores, with the
// pooling and untile steps of the backward folded into the epilogues.  For
// query cube i, its selected key cubes j (the forward's selection, held
// fixed) and scale = 1/sqrt(d), per 64 x 64 block (rows r of cube i, keys c
// of cube j):
//   P  = exp(scale Q_i K_j^T - lse_i)      (the forward's natural-log LSE;
//                                            0 on pad rows and pad keys)
//   dP = dO_i V_j^T,   dS = P (dP - D_i)   (dO_i = tiled dO_f, D = rowsum(dO_f O_f),
//                                            both from the combine-gradient pass)
//   dQ_i += scale dS K_j,   dK_j += scale dS^T Q_i,   dV_j += P^T dO_i
// and the gradient of the cube means reaches every valid row of the cube:
//   dq[r] = dQ_i[r] + dqbar[i] / n_i   (same for k and v with dkbar, dvbar).
// (FastWan news article "单块 H200 ... 5 秒即生一个 5 秒视频", section
// "传统零散郑重力，为何会在蒸馏中失效？": VSA is trained as a drop-in for
// FlashAttention, so the fine stage needs this backward.)
//
// Two persistent kernels (one CTA per SM), neither with atomics, so the
// results are deterministic:
//   dq    an item is one query cube i; the steps are its k selected key
//         cubes.  Per step S = Q_i K_j^T and dP = dO_i V_j^T (M = 64, N = 64,
//         K = d, both operands in shared memory), dS on the CUDA cores, then
//         dQ += dS K_j with dS read from TMEM as the A operand.
//   dkdv  an item is one key cube j; the steps are the query cubes that
//         selected it (the selection transpose's CSR list).  Per step
//         S^T = K_j Q_i^T and dP^T = V_j dO_i^T, P^T and dS^T on the CUDA
//         cores, then dV += P^T dO_i and dK += dS^T Q_i (P^T, dS^T from TMEM).
// Warp roles as in the forward: warp 0 feeds shared memory with TMA (the
// item's stationary pair once, the streamed pair of every step through a
// 4-slot ring), one thread of warp 1 issues every MMA, warps 4-7 do the
// elementwise work and the epilogue; each of them owns the 16 TMEM lanes of
// its sub-partition that an M = 64 accumulator occupies.  S and dP are
// double-buffered in TMEM, so the tensor core computes step e+1's products
// while the elementwise warps work on step e.  P and dS enter the MMAs as
// bf16 (as in a bf16 training step); accumulation is float32.  Every wait is
// bounded (4 s); on a timeout the CTA records VSA_ERR_TIMEOUT and every role
// stops.
#include <cuda.h>

#include "common.cuh"
#include "fine.cuh"
#include "ptx.cuh"

namespace vsa {

namespace {

using namespace ptx;
using bf16 = __nv_bfloat16;

constexpr int kThreads = 256;
constexpr int kProducerWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kEwWarp0 = 4;       // warps 4-7: elementwise + epilogue
constexpr int kEwThreads = 128;
constexpr int kRing = 4;          // streamed-pair slots
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct BCfg {
  static constexpr int kHalves = D / 64;                   // 128-byte atoms per row
  static constexpr uint32_t kHalf = 64 * 128;              // one cube x 64 columns (SW128)
  static constexpr uint32_t kTile = kHalves * kHalf;       // one cube x D
  static constexpr uint32_t kStat = 2 * kTile;             // the item's stationary pair
  static constexpr uint32_t kRows = 2 * kTile;             // lse, delta rows inside a slot
  static constexpr uint32_t kSlot = 2 * kTile + 1024;      // streamed pair + lse, delta rows
  static constexpr uint32_t kRingOff = 2 * kStat;          // two stationary buffers first
  static constexpr uint32_t kBarOff = kRingOff + kRing * kSlot;
  static constexpr size_t kSmem = 1024 + kBarOff + 256;
  // TMEM: S, dP of buffer b at columns 128 b and 128 b + 64; accumulators after
  static constexpr uint32_t kAcc0 = 256;                   // dQ (dq) or dK (dkdv)
  static constexpr uint32_t kAcc1 = 256 + D;               // dV (dkdv)
  static constexpr uint32_t kColQ = 256 + D;               // dq: Q_i, the A operand of S
  static constexpr uint32_t kColG = 256 + D + D / 2;       // dq: dO_i, the A operand of dP
  static constexpr uint32_t kIdescS = idesc_bf16_f32(64, 64, false, false);
  static constexpr uint32_t kIdescAcc = idesc_bf16_f32(64, D, false, true);
};

__device__ __forceinline__ uint32_t col_s(int b) { return 128u * static_cast<uint32_t>(b); }
__device__ __forceinline__ uint32_t col_p(int b) { return 128u * static_cast<uint32_t>(b) + 64u; }

struct BwdShared {
  uint64_t* stat_full;   // [2]
  uint64_t* stat_empty;  // [2]
  uint64_t* ring_full;   // [kRing]
  uint64_t* ring_empty;  // [kRing]
  uint64_t* s_full;      // [2] S, dP of buffer b computed
  uint64_t* ds_full;     // [2] dS (and P^T) of buffer b written to TMEM
  uint64_t* acc_full;    // item's accumulators complete
  uint64_t* acc_empty;   // epilogue has read them
  volatile int* abort_flag;
  uint8_t* base;
};

struct BwdArgs {
  Geom g;
  int topk;
  const int32_t* sel;          // dq: the forward's selection [B, H, C, k]
  const int32_t* key_offsets;  // dkdv: CSR offsets [B, H, C+1]
  const int32_t* query_lists;  // dkdv: CSR lists [B, H, C*k]
  const float* lse;            // [B, H, 64C] natural log
  const float* delta;          // [B, H, 64C]
  const float* bar0;           // dq: dqbar; dkdv: dkbar  ([B, H, C, d] or null)
  const float* bar1;           // dkdv: dvbar
  bf16* out0;                  // dq: dq; dkdv: dk  (token order)
  bf16* out1;                  // dkdv: dv
  const bf16* qt;              // dq: tiled q (rows copied into TMEM)
  const bf16* dot;             // dq: tiled dO_f
  int* status;
};

__device__ __forceinline__ void bwd_fail(const BwdShared& sh, int* status) {
  report(status, VSA_ERR_TIMEOUT);
  *sh.abort_flag = 1;
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack2_bf16(float a, float b) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&p);
}

// The steps of an item: the selection row of query cube `cube` (dq) or the
// CSR list of key cube `cube` (dkdv).  Offsets that do not describe a list
// inside the CSR array are reported and give an empty list.
template <bool kDq>
__device__ __forceinline__ int item_list(const BwdArgs& a, int bh, int cube, const int32_t** list) {
  const Geom& g = a.g;
  if (kDq) {
    *list = a.sel + (static_cast<long long>(bh) * g.C + cube) * a.topk;
    return a.topk;
  }
  const int32_t* offs = a.key_offsets + static_cast<long long>(bh) * (g.C + 1);
  const int p0 = __ldg(&offs[cube]), p1 = __ldg(&offs[cube + 1]);
  const long long cap = static_cast<long long>(g.C) * a.topk;
  if (p0 < 0 || p1 < p0 || p1 > cap) {
    report(a.status, VSA_ERR_BAD_INDEX);
    *list = a.query_lists;
    return 0;
  }
  *list = a.query_lists + static_cast<long long>(bh) * cap + p0;
  return p1 - p0;
}

// Entries of a list read 32 at a time, one per lane, the next window loaded
// while the current one is used.  Warp-collective; get() with e = 0, 1, ...
struct ListWindow {
  const int32_t* list;
  int n, cur, nxt;
  __device__ __forceinline__ void init(const int32_t* l, int n_, int lane) {
    list = l;
    n = n_;
    cur = lane < n ? __ldg(&l[lane]) : 0;
    nxt = 32 + lane < n ? __ldg(&l[32 + lane]) : 0;
  }
  __device__ __forceinline__ int get(int e, int lane) {
    if (e > 0 && (e & 31) == 0) {
      cur = nxt;
      nxt = e + 32 + lane < n ? __ldg(&list[e + 32 + lane]) : 0;
    }
    return __shfl_sync(0xffffffffu, cur, e & 31);
  }
};

// A list entry as a cube index, clamped into [0, C); bad entries are reported.
__device__ __forceinline__ int entry_cube(const Geom& g, int raw, int* status) {
  if (raw < 0 || raw >= g.C) {
    if (status != nullptr && (threadIdx.x & 31) == 0) report(status, VSA_ERR_BAD_INDEX);
    return raw < 0 ? 0 : g.C - 1;
  }
  return raw;
}

// ------------------------------------------------------------------ producer
template <int D, bool kDq>
__device__ void bwd_producer(const BwdShared& sh, const BwdArgs& a, const BwdMaps& maps) {
  using Cf = BCfg<D>;
  const Geom& g = a.g;
  const int lane = threadIdx.x & 31;
  const int items = g.B * g.H * g.C;
  uint32_t ring = 0;
  int u = 0;  // items with at least one step
  auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
    int ok = 1;
    if (lane == 0) ok = mbar_wait(bar, parity) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
  };
  for (int item = blockIdx.x; item < items; item += gridDim.x) {
    if (*sh.abort_flag) return;
    const int bh = item / g.C, cube = item - bh * g.C;
    const int32_t* list;
    const int n = item_list<kDq>(a, bh, cube, &list);
    if (n == 0) continue;
    const int row0 = bh * static_cast<int>(g.rows);
    if (!kDq) {
      // the stationary pair K_j, V_j (the dq kernel's Q_i, dO_i go to TMEM
      // through the elementwise warps)
      const int sb = u & 1;
      if (!wait_all(&sh.stat_empty[sb], ((u >> 1) & 1) ^ 1)) return bwd_fail(sh, a.status);
      ++u;
      uint8_t* stat = sh.base + sb * Cf::kStat;
      if (lane == 0) mbar_arrive_expect_tx(&sh.stat_full[sb], Cf::kStat);
      __syncwarp();
      if (lane < 2 * Cf::kHalves) {
        const int which = lane / Cf::kHalves, h = lane - which * Cf::kHalves;
        tma_load_2d(stat + which * Cf::kTile + h * Cf::kHalf, which ? &maps.v : &maps.k,
                    &sh.stat_full[sb], h * 64, row0 + cube * 64);
      }
    }
    // the streamed pair of every step: K_j, V_j (dq) or Q_i, dO_i and the
    // lse and delta rows of query cube i (dkdv)
    ListWindow win;
    win.init(list, n, lane);
    for (int e = 0; e < n; ++e) {
      const int other = entry_cube(g, win.get(e, lane), a.status);
      const int slot = static_cast<int>(ring % kRing);
      const uint32_t round = ring / kRing;
      ++ring;
      if (!wait_all(&sh.ring_empty[slot], (round & 1u) ^ 1u)) return bwd_fail(sh, a.status);
      uint8_t* dst = sh.base + Cf::kRingOff + slot * Cf::kSlot;
      if (lane == 0) mbar_arrive_expect_tx(&sh.ring_full[slot], 2 * Cf::kTile + (kDq ? 0u : 512u));
      __syncwarp();
      const int orow = row0 + other * 64;
      if (lane < 2 * Cf::kHalves) {
        const int which = lane / Cf::kHalves, h = lane - which * Cf::kHalves;
        const CUtensorMap* m = kDq ? (which ? &maps.v : &maps.k) : (which ? &maps.dO : &maps.q);
        tma_load_2d(dst + which * Cf::kTile + h * Cf::kHalf, m, &sh.ring_full[slot], h * 64, orow);
      } else if (!kDq && lane < 2 * Cf::kHalves + 2) {
        const int which = lane - 2 * Cf::kHalves;  // 0: lse row, 1: delta row (64 floats each)
        bulk_load(dst + Cf::kRows + which * 256, (which ? a.delta : a.lse) + orow, 256u,
                  &sh.ring_full[slot]);
      }
    }
  }
}

// ------------------------------------------------------------------ MMA issuer
template <int D, bool kDq>
__device__ void bwd_mma(const BwdShared& sh, const BwdArgs& a, uint32_t tmem) {
  using Cf = BCfg<D>;
  constexpr int kK = D / 16;
  const Geom& g = a.g;
  const int items = g.B * g.H * g.C;
  const uint32_t base = smem_u32(sh.base);
  uint32_t ring = 0, ds_ph0 = 0u, ds_ph1 = 0u;
  int u = 0;
  for (int item = blockIdx.x; item < items; item += gridDim.x) {
    if (*sh.abort_flag) return;
    const int bh = item / g.C, cube = item - bh * g.C;
    const int32_t* list;
    const int n = item_list<kDq>(a, bh, cube, &list);
    if (n == 0) continue;
    const int sb = u & 1;
    if (!mbar_wait(&sh.stat_full[sb], (u >> 1) & 1)) return bwd_fail(sh, a.status);
    tc_fence_after();
    const uint32_t stat = base + sb * Cf::kStat;
    // A operands of S and dP: Q_i and dO_i (dq), K_j and V_j (dkdv), K-major
    const uint64_t a0 = sdesc_sw128(stat, 16, 1024);
    const uint64_t a1 = sdesc_sw128(stat + Cf::kTile, 16, 1024);
    int slot_of[2] = {0, 0};
    // S and dP of step e into buffer e & 1
    auto sdp = [&](int e) -> bool {
      const int b = e & 1;
      const int slot = static_cast<int>(ring % kRing);
      const uint32_t round = ring / kRing;
      ++ring;
      if (!mbar_wait(&sh.ring_full[slot], round & 1u)) return false;
      tc_fence_after();
      slot_of[b] = slot;
      const uint32_t sa = base + Cf::kRingOff + slot * Cf::kSlot;
      const uint64_t b0 = sdesc_sw128(sa, 16, 1024);              // K_j (dq) or Q_i (dkdv)
      const uint64_t b1 = sdesc_sw128(sa + Cf::kTile, 16, 1024);  // V_j (dq) or dO_i (dkdv)
#pragma unroll
      for (int kk = 0; kk < kK; ++kk) {
        const uint64_t o = ((kk >> 2) * Cf::kHalf + (kk & 3) * 32) >> 4;
        if (kDq)  // Q_i from TMEM: 16 features = 8 packed columns per k-step
          umma_ts(tmem + col_s(b), tmem + Cf::kColQ + kk * 8, b0 + o, Cf::kIdescS, kk > 0 ? 1u : 0u);
        else
          umma_ss(tmem + col_s(b), a0 + o, b0 + o, Cf::kIdescS, kk > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int kk = 0; kk < kK; ++kk) {
        const uint64_t o = ((kk >> 2) * Cf::kHalf + (kk & 3) * 32) >> 4;
        if (kDq)
          umma_ts(tmem + col_p(b), tmem + Cf::kColG + kk * 8, b1 + o, Cf::kIdescS, kk > 0 ? 1u : 0u);
        else
          umma_ss(tmem + col_p(b), a1 + o, b1 + o, Cf::kIdescS, kk > 0 ? 1u : 0u);
      }
      umma_commit(&sh.s_full[b]);
      return true;
    };
    if (!sdp(0)) return bwd_fail(sh, a.status);
    for (int e = 0; e < n; ++e) {
      const int b = e & 1;
      // the next step's products run while the elementwise warps work on this one
      if (e + 1 < n && !sdp(e + 1)) return bwd_fail(sh, a.status);
      if (e == 0) {  // the previous item's epilogue has read the accumulators
        if (!mbar_wait(sh.acc_empty, (u & 1) ^ 1)) return bwd_fail(sh, a.status);
        tc_fence_after();
      }
      uint32_t& ph = b ? ds_ph1 : ds_ph0;
      if (!mbar_wait(&sh.ds_full[b], ph)) return bwd_fail(sh, a.status);
      ph ^= 1u;
      tc_fence_after();
      const uint32_t sa = base + Cf::kRingOff + slot_of[b] * Cf::kSlot;
      // the streamed tiles as [64 rows (K) x D (N)] MN-major B operands
      const uint64_t m0 = sdesc_sw128(sa, Cf::kHalf, 1024);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t acc = (e > 0 || kk > 0) ? 1u : 0u;
        if (kDq) {
          // dQ += dS K_j
          umma_ts(tmem + Cf::kAcc0, tmem + col_s(b) + kk * 8, m0 + kk * 128, Cf::kIdescAcc, acc);
        } else {
          const uint64_t m1 = sdesc_sw128(sa + Cf::kTile, Cf::kHalf, 1024);
          // dV += P^T dO_i, dK += dS^T Q_i
          umma_ts(tmem + Cf::kAcc1, tmem + col_s(b) + kk * 8, m1 + kk * 128, Cf::kIdescAcc, acc);
          umma_ts(tmem + Cf::kAcc0, tmem + col_p(b) + kk * 8, m0 + kk * 128, Cf::kIdescAcc, acc);
        }
      }
      umma_commit(&sh.ring_empty[slot_of[b]]);
    }
    umma_commit(sh.acc_full);
    umma_commit(&sh.stat_empty[sb]);
    ++u;
  }
}

// ------------------------------------------------------------------ elementwise + epilogue
// Writes the valid row r of the item's cube: out[token] = bf16(acc * mul +
// bar[cube] / n), for this thread's half of the columns (acc may be null: 0).
template <int D>
__device__ __forceinline__ void write_row(const Geom& g, int bh, int cube, int r, int h,
                                          const uint32_t* acc, float mul, const float* bar,
                                          float rn, bf16* out) {
  constexpr int kOH = D / 2;
  const long long tok = static_cast<long long>(bh) * g.N + slot_token(g, cube, r);
  uint4* orow = reinterpret_cast<uint4*>(out + tok * D + h * kOH);
  const float4* b4 = bar ? reinterpret_cast<const float4*>(
                               bar + (static_cast<long long>(bh) * g.C + cube) * D + h * kOH)
                         : nullptr;
#pragma unroll
  for (int q8 = 0; q8 < kOH / 8; ++q8) {
    float v[8];
#pragma unroll
    for (int x = 0; x < 8; ++x) v[x] = acc ? __uint_as_float(acc[q8 * 8 + x]) * mul : 0.f;
    if (b4) {
      const float4 c0 = __ldg(&b4[2 * q8]), c1 = __ldg(&b4[2 * q8 + 1]);
      v[0] = fmaf(c0.x, rn, v[0]);
      v[1] = fmaf(c0.y, rn, v[1]);
      v[2] = fmaf(c0.z, rn, v[2]);
      v[3] = fmaf(c0.w, rn, v[3]);
      v[4] = fmaf(c1.x, rn, v[4]);
      v[5] = fmaf(c1.y, rn, v[5]);
      v[6] = fmaf(c1.z, rn, v[6]);
      v[7] = fmaf(c1.w, rn, v[7]);
    }
    orow[q8] = make_uint4(pack2_bf16(v[0], v[1]), pack2_bf16(v[2], v[3]), pack2_bf16(v[4], v[5]),
                          pack2_bf16(v[6], v[7]));
  }
}

template <int D>
__device__ __forceinline__ void ld_half_row(uint32_t taddr, uint32_t (&v)[D / 2]) {
  if constexpr (D == 128) {
    tmem_ld_16x32bx2_x64(taddr, v);
  } else {
    tmem_ld_16x32bx2_x32(taddr, v);
  }
}

template <int D, bool kDq>
__device__ void bwd_elementwise(const BwdShared& sh, const BwdArgs& a, uint32_t tmem) {
  using Cf = BCfg<D>;
  const Geom& g = a.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wq = warp & 3;              // TMEM sub-partition
  const int h = lane >> 4;              // which 32 of the 64 columns this thread holds
  const int r = wq * 16 + (lane & 15);  // row of the item's cube (query row or key row)
  const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
  const float sl2 = kLog2e * rsqrtf(static_cast<float>(D));
  const float scale = rsqrtf(static_cast<float>(D));
  const int items = g.B * g.H * g.C;
  uint32_t ring = 0, s_ph0 = 0u, s_ph1 = 0u;
  int u = 0;
  for (int item = blockIdx.x; item < items; item += gridDim.x) {
    if (*sh.abort_flag) return;
    const int bh = item / g.C, cube = item - bh * g.C;
    const int32_t* list;
    const int n = item_list<kDq>(a, bh, cube, &list);
    const int nc = cube_valid(g, cube);
    const bool row_ok = r < nc;
    const float rn = 1.0f / static_cast<float>(nc);
    if (n > 0) {
      float lse2 = 0.f, dlt = 0.f;  // dq: this query row's lse (log2 units) and D
      if (kDq && row_ok) {
        const long long row = static_cast<long long>(bh) * g.rows + cube * 64 + r;
        lse2 = __ldg(&a.lse[row]) * kLog2e;
        dlt = __ldg(&a.delta[row]);
      }
      if (kDq) {
        // Q_i and dO_i rows into TMEM as the A operands of S and dP: this
        // thread's row r, features D/2 h .. D/2 h + D/2 - 1 (two per column).
        // The previous item's products have completed: its accumulator was
        // waited for.
        const long long row = static_cast<long long>(bh) * g.rows + cube * 64 + r;
#pragma unroll
        for (int which = 0; which < 2; ++which) {
          const uint4* src = reinterpret_cast<const uint4*>((which ? a.dot : a.qt) + row * D + h * (D / 2));
          const uint32_t col = which ? Cf::kColG : Cf::kColQ;
          if constexpr (D == 128) {
            uint32_t w[32];
#pragma unroll
            for (int x = 0; x < 8; ++x) {
              const uint4 v4 = __ldg(&src[x]);
              w[4 * x] = v4.x;
              w[4 * x + 1] = v4.y;
              w[4 * x + 2] = v4.z;
              w[4 * x + 3] = v4.w;
            }
            tmem_st_16x32bx2_x32(tmem + lane_addr + col, w);
          } else {
            uint32_t w[16];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              const uint4 v4 = __ldg(&src[x]);
              w[4 * x] = v4.x;
              w[4 * x + 1] = v4.y;
              w[4 * x + 2] = v4.z;
              w[4 * x + 3] = v4.w;
            }
            tmem_st_16x32bx2_x16(tmem + lane_addr + col, w);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&sh.stat_full[u & 1]);
      }
      ListWindow win;
      win.init(list, n, lane);
      for (int e = 0; e < n; ++e) {
        const int b = e & 1;
        const int other = entry_cube(g, win.get(e, lane), nullptr);
        const int no = cube_valid(g, other);  // valid keys (dq) or query rows (dkdv)
        const int slot = static_cast<int>(ring % kRing);
        const uint32_t round = ring / kRing;
        ++ring;
        uint32_t& sp = b ? s_ph1 : s_ph0;
        if (!mbar_wait(&sh.s_full[b], sp)) return bwd_fail(sh, a.status);
        sp ^= 1u;
        tc_fence_after();
        uint32_t sv[32], pv[32];
        tmem_ld_16x32bx2_x32(tmem + lane_addr + col_s(b), sv);
        tmem_ld_16x32bx2_x32(tmem + lane_addr + col_p(b), pv);
        if (kDq) {
          // columns: keys 32 h + x of key cube `other`
          uint32_t pk[16];
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            float ds[2];
#pragma unroll
            for (int y = 0; y < 2; ++y) {
              const int c = 32 * h + 2 * x + y;
              const bool ok = row_ok && c < no;
              const float p = fast_exp2(fmaf(__uint_as_float(sv[2 * x + y]), sl2, -lse2));
              ds[y] = ok ? p * (__uint_as_float(pv[2 * x + y]) - dlt) : 0.f;
            }
            pk[x] = pack2_bf16(ds[0], ds[1]);
          }
          tmem_st_16x32bx2_x16(tmem + lane_addr + col_s(b), pk);  // dS over S
        } else {
          // columns: query rows 32 h + x of query cube `other`; their lse and
          // D came with the step's tiles
          if (!mbar_wait(&sh.ring_full[slot], round & 1u)) return bwd_fail(sh, a.status);
          const float4* rows = reinterpret_cast<const float4*>(sh.base + Cf::kRingOff +
                                                               slot * Cf::kSlot + Cf::kRows);
          uint32_t pp[16], pd[16];
#pragma unroll
          for (int x4 = 0; x4 < 8; ++x4) {
            const float4 l4 = rows[8 * h + x4];       // lse[32 h + 4 x4 ..]
            const float4 d4 = rows[16 + 8 * h + x4];  // delta[32 h + 4 x4 ..]
            const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
            const float dv[4] = {d4.x, d4.y, d4.z, d4.w};
            float p[4], ds[4];
#pragma unroll
            for (int y = 0; y < 4; ++y) {
              const int q = 32 * h + 4 * x4 + y;
              const int x = 4 * x4 + y;
              const bool ok = row_ok && q < no;
              const float e2 = fast_exp2(fmaf(__uint_as_float(sv[x]), sl2, -lv[y] * kLog2e));
              p[y] = ok ? e2 : 0.f;
              ds[y] = ok ? e2 * (__uint_as_float(pv[x]) - dv[y]) : 0.f;
            }
            pp[2 * x4] = pack2_bf16(p[0], p[1]);
            pp[2 * x4 + 1] = pack2_bf16(p[2], p[3]);
            pd[2 * x4] = pack2_bf16(ds[0], ds[1]);
            pd[2 * x4 + 1] = pack2_bf16(ds[2], ds[3]);
          }
          tmem_st_16x32bx2_x16(tmem + lane_addr + col_s(b), pp);  // P^T over S^T
          tmem_st_16x32bx2_x16(tmem + lane_addr + col_p(b), pd);  // dS^T over dP^T
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&sh.ds_full[b]);
      }
      // ---- epilogue: accumulators -> token-order bf16 rows (+ the pooled term)
      if (!mbar_wait(sh.acc_full, u & 1)) return bwd_fail(sh, a.status);
      tc_fence_after();
      ++u;
      uint32_t acc[D / 2];
      ld_half_row<D>(tmem + lane_addr + Cf::kAcc0, acc);
      if (kDq) {
        tc_fence_before();
        mbar_arrive(sh.acc_empty);
        if (row_ok) write_row<D>(g, bh, cube, r, h, acc, scale, a.bar0, rn, a.out0);
      } else {
        if (row_ok) write_row<D>(g, bh, cube, r, h, acc, scale, a.bar0, rn, a.out0);
        ld_half_row<D>(tmem + lane_addr + Cf::kAcc1, acc);
        tc_fence_before();
        mbar_arrive(sh.acc_empty);
        if (row_ok) write_row<D>(g, bh, cube, r, h, acc, 1.0f, a.bar1, rn, a.out1);
      }
    } else if (row_ok) {
      // a key cube no query cube selected: only the pooled term (or zero)
      write_row<D>(g, bh, cube, r, h, nullptr, 0.f, a.bar0, rn, a.out0);
      if (!kDq) write_row<D>(g, bh, cube, r, h, nullptr, 0.f, a.bar1, rn, a.out1);
    }
  }
}

template <int D, bool kDq>
__global__ void __launch_bounds__(kThreads, 1) fine_bwd_kernel(const __grid_constant__ BwdMaps maps,
                                                               const BwdArgs a) {
  using Cf = BCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cf::kBarOff);
  BwdShared sh;
  sh.base = smem;
  sh.stat_full = bars;
  sh.stat_empty = bars + 2;
  sh.ring_full = bars + 4;
  sh.ring_empty = bars + 4 + kRing;
  sh.s_full = bars + 4 + 2 * kRing;
  sh.ds_full = sh.s_full + 2;
  sh.acc_full = sh.s_full + 4;
  sh.acc_empty = sh.s_full + 5;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sh.s_full + 6);
  sh.abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    for (int q = 0; q < 2; ++q) {
      mbar_init(&sh.stat_full[q], kDq ? kEwThreads : 1);
      mbar_init(&sh.stat_empty[q], 1);
      mbar_init(&sh.s_full[q], 1);
      mbar_init(&sh.ds_full[q], kEwThreads);
    }
    for (int s = 0; s < kRing; ++s) {
      mbar_init(&sh.ring_full[s], 1);
      mbar_init(&sh.ring_empty[s], 1);
    }
    mbar_init(sh.acc_full, 1);
    mbar_init(sh.acc_empty, kEwThreads);
    *sh.abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&maps.q);
    prefetch_tmap(&maps.k);
    prefetch_tmap(&maps.v);
    prefetch_tmap(&maps.dO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kProducerWarp) {
    bwd_producer<D, kDq>(sh, a, maps);
  } else if (warp == kMmaWarp) {
    if (lane == 0) bwd_mma<D, kDq>(sh, a, tmem);
  } else if (warp >= kEwWarp0) {
    bwd_elementwise<D, kDq>(sh, a, tmem);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

template <int D>
cudaError_t run(const BwdMaps& maps, const BwdArgs& base, const float* dpooled, bf16* dq, bf16* dk,
                bf16* dv, int sms, cudaStream_t s) {
  static CtxCache<char> dq_set, dkdv_set;
  constexpr int kBytes = static_cast<int>(BCfg<D>::kSmem);
  cudaError_t err = smem_limit_once(fine_bwd_kernel<D, true>, kBytes, &dq_set);
  if (err != cudaSuccess) return err;
  if ((err = smem_limit_once(fine_bwd_kernel<D, false>, kBytes, &dkdv_set)) != cudaSuccess) return err;
  const Geom& g = base.g;
  const long long plane = static_cast<long long>(g.B) * g.H * g.C * D;
  const long long items = static_cast<long long>(g.B) * g.H * g.C;
  const int grid = static_cast<int>(items < sms ? items : sms);
  BwdArgs qa = base;
  qa.bar0 = dpooled;
  qa.bar1 = nullptr;
  qa.out0 = dq;
  qa.out1 = nullptr;
  fine_bwd_kernel<D, true><<<grid, kThreads, kBytes, s>>>(maps, qa);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  BwdArgs ka = base;
  ka.bar0 = dpooled ? dpooled + plane : nullptr;
  ka.bar1 = dpooled ? dpooled + 2 * plane : nullptr;
  ka.out0 = dk;
  ka.out1 = dv;
  fine_bwd_kernel<D, false><<<grid, kThreads, kBytes, s>>>(maps, ka);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_block_sparse_bwd(const Geom& g, const BwdMaps& maps, int topk,
                                    const float* lse, const float* delta, const int32_t* sel,
                                    const int32_t* key_offsets, const int32_t* query_lists,
                                    const float* dpooled, void* dq, void* dk, void* dv,
                                    int* status, int sms, cudaStream_t s, const void* q_tiled,
                                    const void* do_tiled) {
  BwdArgs a{};
  a.qt = static_cast<const bf16*>(q_tiled);
  a.dot = static_cast<const bf16*>(do_tiled);
  a.g = g;
  a.topk = topk;
  a.sel = sel;
  a.key_offsets = key_offsets;
  a.query_lists = query_lists;
  a.lse = lse;
  a.delta = delta;
  a.status = status;
  auto w = [](void* p) { return static_cast<bf16*>(p); };
  if (g.d == 64) return run<64>(maps, a, dpooled, w(dq), w(dk), w(dv), sms, s);
  return run<128>(maps, a, dpooled, w(dq), w(dk), w(dv), sms, s);
}

}  // namespace vsa
