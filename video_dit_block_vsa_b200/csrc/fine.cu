// Fine stage of VSA: exact attention of each 64-token query cube over the
// valid tokens of its k selected key cubes (FastWan article "单块 H200 ...
// 5 秒即生一个 5 秒视频", section "一张卡，秒生视频": the fine block-sparse
// kernel over a 64x64 block mask).
//
// Design (sm_100a):
//  * Persistent CTAs, one per SM, walk work items head-major; an item is a
//    pair of query cubes (A, B) of one (b, h).  Each cube has its own key
//    list, so every MMA has M = 64 rows (one cube); the two cubes ping-pong
//    so that the tensor core works on one while the other's softmax runs.
//  * Warp roles: warp 0 = TMA producer, warp 1 = MMA issuer (one thread),
//    warps 4-7 = softmax of cube A, warps 8-11 = softmax of cube B.
//  * Key packing: each selected key cube is "wide" (more than 16 valid tokens:
//    one 64-row group of four 16-row chunks) or "narrow" (at most 16 valid
//    tokens, packed to the front of the cube: one 16-row chunk).  A selection
//    row lists its wide cubes first (the coarse stage writes them that way), so
//    a cube's key rows are a sequence of T = 4 W + (k - W) chunks and step j
//    holds chunks 8j .. 8j+7: 128 key rows, one N = 128 MMA.  The partial
//    cubes of a ragged grid so cost a quarter of a full cube.  The last step
//    of a cube may hold fewer chunks: its Q K^T uses N = 16 x chunks and its
//    P V that many 16-key slices.  The two cubes of an item may have
//    different step counts.
//  * Keys and values stream through a ring of 128-key smem slots (128-byte
//    swizzle, TMA-filled) in exactly the order the MMA issuer consumes them:
//    K_A0 K_B0 | V_A0 K_A1 V_B0 K_B1 | ...
//  * TMEM: an M = 64 accumulator occupies 16 lanes of each warp's 32-lane
//    sub-partition, so the two cubes share columns: cube A in lanes 0-15,
//    cube B in lanes 16-31.  Columns: S [0,128), O [128,128+d), Q
//    [128+d, 128+3d/2).  The softmax warps write their cube's query rows into
//    TMEM at the start of an item, and Q K^T reads Q as the TMEM A operand
//    (no shared-memory operand reads for Q, and shared memory holds only the
//    K/V ring: 7 slots at d = 128).  The softmax writes P (bf16 pairs) over
//    the first 64 columns of its S, and O += P V reads P from TMEM as well, so
//    P never touches shared memory.  MMAs issued by one thread execute in
//    order, so the next S = Q K^T cannot overwrite P before the P V that
//    reads it.
//  * The softmax reads S with the 16-lane .16x32bx2 shape: thread t holds row
//    16*(warp%4) + t%16, columns [64*(t/16), +64) of the step, i.e. exactly
//    one key cube's 64 keys.
//  * Online softmax in log2 units with conditional rescaling: the running
//    reference max only moves (and O, l are rescaled) when a row's max grows
//    by more than 2^8, so most steps skip the O round trip through registers.
//  * Every wait is bounded (4 s); on a timeout the CTA records
//    VSA_ERR_TIMEOUT, every role stops, TMEM is freed and the CTA exits.
#include <cuda.h>

#include <type_traits>

#include "common.cuh"
#include "fine.cuh"
#include "ptx.cuh"

namespace vsa {

namespace {

using namespace ptx;

constexpr int kWarps = 12;
constexpr int kThreads = kWarps * 32;
constexpr int kProducerWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kSoftmaxWarp0 = 4;  // warps 4..7: cube A, 8..11: cube B
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 8.0f;  // rescale only when a row max grows by > 2^8
constexpr int kWideMin = 17;          // a key cube with this many valid tokens or more is wide

template <int D>
struct Cfg {
  static constexpr int kHalves = D / 64;                       // 128-byte atoms per row
  static constexpr uint32_t kQHalf = 64 * 128;                 // [64 rows x 128 B]
  static constexpr uint32_t kQBytes = kHalves * kQHalf;        // one query cube tile
  static constexpr uint32_t kKVHalf = 128 * 128;               // [128 rows x 128 B]
  static constexpr uint32_t kSlotBytes = kHalves * kKVHalf;    // 128 keys x D
  static constexpr int kSlots = D == 128 ? 7 : 14;             // the ring fills shared memory
  static constexpr uint32_t kRingOff = 0;
  static constexpr uint32_t kBarOff = kRingOff + kSlots * kSlotBytes;
  static constexpr size_t kSmem = 1024 + kBarOff + 512;
  // TMEM columns; cube A uses lanes 0-15 of every sub-partition, cube B lanes 16-31
  static constexpr uint32_t kColS = 0;            // S (P over its first 64 columns)
  static constexpr uint32_t kColO = 128;          // O
  static constexpr uint32_t kColQ = 128 + D;      // Q, the A operand of Q K^T (D/2 columns)
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(64, D, false, true);  // P (TMEM), V MN-major
};

// Where the epilogue writes O / l: the tiled bf16 tensor, or (token_order)
// the final bf16 output in token order, optionally as the gated sum
// g_f * bf16(O / l) + g_c * O_c of the combine step.
struct OutSpec {
  __nv_bfloat16* out;
  float* lse;
  const float* o_coarse;
  const float* g_fine;
  const float* g_coarse;
  int token_order;
};

struct Shared {
  volatile int* chunks;  // [2 Q buffers][2 cubes]: 16-row key chunks, producer -> MMA thread
  uint64_t* q_full;
  uint64_t* q_empty;
  uint64_t* q_ready;  // [2] a cube's query rows are in TMEM
  uint64_t* kv_full;
  uint64_t* kv_empty;
  uint64_t* s_full;
  uint64_t* p_full;
  uint64_t* o_full;
  volatile int* abort_flag;
  uint8_t* base;
};

// TMEM lane offset of cube c's accumulators and operands.
__device__ __forceinline__ uint32_t cube_lanes(int c) { return static_cast<uint32_t>(16 * c) << 16; }

struct Item {
  int bh, i0, i1, row0;
  bool has_b;
};

__device__ __forceinline__ Item decode(const Geom& g, int item, int pairs) {
  Item it;
  it.bh = item / pairs;
  const int pr = item - it.bh * pairs;
  it.i0 = 2 * pr;
  it.i1 = it.i0 + 1;
  it.has_b = it.i1 < g.C;
  it.row0 = it.bh * static_cast<int>(g.rows);
  return it;
}

__device__ __forceinline__ void fail(const Shared& sh, int* status) {
  report(status, VSA_ERR_TIMEOUT);
  *sh.abort_flag = 1;
}

// 2^x with one MUFU operation (ex2.approx, flushes subnormal results to 0;
// 2^-inf = 0).  The probabilities it feeds are rounded to bf16 afterwards.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack2_bf16(float a, float b) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&p);
}

__device__ __forceinline__ int clamp_cube(const Geom& g, int x) {
  return x < 0 ? 0 : (x >= g.C ? g.C - 1 : x);
}

// ------------------------------------------------------------------ key plan
// A selection row lists its W wide key cubes first, then its k - W narrow
// ones (each group ascending, as the coarse stage writes it).  The cube's key
// rows are a sequence of T = 4 W + (k - W) chunks of 16 rows; step j holds
// chunks 8j .. 8j+7, half h of it the four chunks from cb = 8j + 4h, which are
// either one wide cube (cb < 4W) or up to four narrow ones.

// What half-step from chunk cb holds: 0 nothing, 1 one wide cube, 2 narrow cubes.
__device__ __forceinline__ int half_kind(int cb, int W, int T) {
  return cb >= T ? 0 : (cb < 4 * W ? 1 : 2);
}

// List entry of chunk slot q (0..3) of the half-step from chunk cb, or -1
// (the three continuation slots of a wide cube and slots past the end).
__device__ __forceinline__ int half_entry(int cb, int q, int W, int topk) {
  if (cb < 4 * W) return q == 0 ? cb >> 2 : -1;
  const int e = W + (cb - 4 * W) + q;
  return e < topk ? e : -1;
}

// Wide entries of a list (warp-collective).  With `status`, also checks the
// list: entries in [0, C), wide cubes before narrow ones, each group strictly
// ascending; a violation is recorded as VSA_ERR_BAD_INDEX.  The loads of up
// to eight 32-entry windows are issued before any of them is used.
__device__ __forceinline__ int count_wide(const Geom& g, const int32_t* list, int topk, int lane,
                                          int* status) {
  int wide = 0;
  int prev_last = -1;
  bool prev_wide_last = true;
  bool bad = false;
  for (int b0 = 0; b0 < topk; b0 += 256) {
    int raws[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = b0 + 32 * u + lane;
      raws[u] = i < topk ? __ldg(&list[i]) : 0;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int b = b0 + 32 * u;
      if (b >= topk) break;
      const bool in = b + lane < topk;
      const int raw = raws[u];
      const bool w = in && cube_valid(g, clamp_cube(g, raw)) >= kWideMin;
      wide += __popc(__ballot_sync(0xffffffffu, w));
      if (status != nullptr) {
        int prev = __shfl_up_sync(0xffffffffu, raw, 1);
        bool prev_w = __shfl_up_sync(0xffffffffu, w, 1);
        if (lane == 0) {
          prev = prev_last;
          prev_w = prev_wide_last;
        }
        if (in) {
          bad |= raw < 0 || raw >= g.C;
          if (b + lane > 0) bad |= (w && !prev_w) || (w == prev_w && raw <= prev);
        }
        prev_last = __shfl_sync(0xffffffffu, raw, 31);
        prev_wide_last = __shfl_sync(0xffffffffu, w, 31);
      }
    }
  }
  if (status != nullptr && __any_sync(0xffffffffu, bad) && lane == 0)
    report(status, VSA_ERR_BAD_INDEX);
  return wide;
}

// A list entry fetched ahead of its use: the load is issued now and the value
// (clamped into [0, C)) is only read by `cube_of` later, so the load's latency
// overlaps other work.
struct Ahead {
  int raw;
  bool present;
};

__device__ __forceinline__ Ahead fetch_entry(const int32_t* list, int e) {
  Ahead a;
  a.present = e >= 0;
  a.raw = a.present ? __ldg(&list[e]) : 0;
  return a;
}

__device__ __forceinline__ int cube_of(const Geom& g, const Ahead& a) {
  return a.present ? clamp_cube(g, a.raw) : -1;
}

// ------------------------------------------------------------------ producer
// Run by the whole producer warp; lane 0 issues the barrier and TMA operations.
template <int D>
__device__ void producer(const Shared& sh, const Geom& g, const FineMaps& maps,
                         const int32_t* __restrict__ counts, const int32_t* __restrict__ sel,
                         int topk, int* status) {
  using Cf = Cfg<D>;
  const int lane = threadIdx.x & 31;
  const bool leader = lane == 0;
  const int pairs = (g.C + 1) / 2;
  const int items = g.B * g.H * pairs;
  uint32_t ring = 0;
  int t = 0;
  // lane 0 waits; the verdict is broadcast so the warp leaves together
  auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
    int ok = 1;
    if (leader) ok = mbar_wait(bar, parity) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
  };
  for (int item = blockIdx.x; item < items; item += gridDim.x, ++t) {
    if (*sh.abort_flag) return;
    const Item it = decode(g, item, pairs);
    if (leader && (__ldg(&counts[it.i0]) != cube_valid(g, it.i0) ||
                   (it.has_b && __ldg(&counts[it.i1]) != cube_valid(g, it.i1))))
      report(status, VSA_ERR_BAD_INDEX);
    const int32_t* list[2];
    list[0] = sel + (static_cast<long long>(it.bh) * g.C + it.i0) * topk;
    list[1] = list[0] + topk;
    int W[2], T[2], n[2];
    W[0] = count_wide(g, list[0], topk, lane, status);
    W[1] = it.has_b ? count_wide(g, list[1], topk, lane, status) : 0;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      T[c] = 3 * W[c] + topk;
      n[c] = (T[c] + 7) / 8;
    }
    if (!it.has_b) T[1] = n[1] = 0;  // no cube B: nothing to plan or fetch
    // ---- the item's chunk counts
    const int qb = t & 1;
    if (!wait_all(&sh.q_empty[qb], ((t >> 1) & 1) ^ 1)) return fail(sh, status);
    if (leader) {
      sh.chunks[2 * qb] = T[0];  // published to the MMA thread by the q_full arrive
      sh.chunks[2 * qb + 1] = it.has_b ? T[1] : 0;
      mbar_arrive(&sh.q_full[qb]);  // the query rows go to TMEM through the softmax warps
    }
    // ---- key / value slots, in the MMA issuer's order: K_A0 K_B0, then per
    // step j: V_Aj K_A(j+1) V_Bj K_B(j+1), skipping steps a cube does not have.
    // Lane q < 8 owns chunk slot q: its list entry for the next K load of each
    // cube is fetched one K load ahead, and a V load reuses the entries of the
    // K load of the same step.  Each cube's lookahead lives in its own
    // variables and every slot is emitted by code specialised for its cube and
    // kind, so no instruction that picks one cube's entry also waits for the
    // other cube's load still in flight.
    auto lookup = [&](int c, int j) -> Ahead {
      const int Wc = c ? W[1] : W[0], Tc = c ? T[1] : T[0];
      const int cb = 8 * j + 4 * (lane >> 2);
      int e = -1;
      if (lane < 8 && half_kind(cb, Wc, Tc) != 0) e = half_entry(cb, lane & 3, Wc, topk);
      return fetch_entry(c ? list[1] : list[0], e);
    };
    Ahead next_k0 = lookup(0, 0), next_k1 = lookup(1, 0);
    Ahead last_k0 = next_k0, last_k1 = next_k1;
    // one slot: 0 = issued, 1 = abort seen, 2 = a wait timed out
    auto emit = [&](auto cube, auto value, int j) -> int {
      constexpr int c = decltype(cube)::value;
      constexpr bool is_v = decltype(value)::value;
      Ahead& next_k = c ? next_k1 : next_k0;
      Ahead& last_k = c ? last_k1 : last_k0;
      if (*sh.abort_flag) return 1;
      const int slot = static_cast<int>(ring % Cf::kSlots);
      const uint32_t round = ring / Cf::kSlots;
      ++ring;
      // this step's chunk slots: lane q < 8 loads slot q's key cube
      const int Wc = W[c], Tc = T[c];
      const int cb0 = 8 * j;
      const bool wide = half_kind(cb0 + 4 * (lane >> 2), Wc, Tc) == 1;
      int mine;
      if constexpr (is_v) {
        mine = cube_of(g, last_k);
      } else {
        mine = cube_of(g, next_k);
        last_k = next_k;
        next_k = lookup(c, j + 1);
      }
      const int nc = min(8, Tc - cb0);
      if (!wait_all(&sh.kv_empty[slot], (round & 1u) ^ 1u)) return 2;
      // the step's key rows: 64 per wide cube, 16 per narrow cube
      if (leader) mbar_arrive_expect_tx(&sh.kv_full[slot], static_cast<uint32_t>(nc) * 16u * D * 2u);
      __syncwarp();
      if (mine >= 0) {
        uint8_t* dst = sh.base + Cf::kRingOff + slot * Cf::kSlotBytes + (lane >> 2) * 8192 +
                       (lane & 3) * 2048;
        const CUtensorMap* m = is_v ? (wide ? &maps.v : &maps.v16) : (wide ? &maps.k : &maps.k16);
#pragma unroll
        for (int dh = 0; dh < Cf::kHalves; ++dh)
          tma_load_2d(dst + dh * Cf::kKVHalf, m, &sh.kv_full[slot], dh * 64, it.row0 + mine * 64);
      }
      return 0;
    };
    using A = std::integral_constant<int, 0>;
    using B = std::integral_constant<int, 1>;
    using K = std::false_type;
    using V = std::true_type;
    int rc = emit(A{}, K{}, 0);
    if (rc == 0 && n[1] > 0) rc = emit(B{}, K{}, 0);
    const int nmax = max(n[0], n[1]);
    for (int js = 0; rc == 0 && js < nmax; ++js) {
      if (js < n[0]) {
        rc = emit(A{}, V{}, js);
        if (rc == 0 && js + 1 < n[0]) rc = emit(A{}, K{}, js + 1);
      }
      if (rc == 0 && js < n[1]) {
        rc = emit(B{}, V{}, js);
        if (rc == 0 && js + 1 < n[1]) rc = emit(B{}, K{}, js + 1);
      }
    }
    if (rc == 1) return;
    if (rc == 2) return fail(sh, status);
  }
}

// ------------------------------------------------------------------ MMA issuer
// One thread issues every MMA.  Its own instruction latency must stay far
// below the 64 cycles an M = 64, N = 128, K = 16 MMA occupies the tensor
// pipe, so descriptors are built once per operand tile and each k-step only
// adds a compile-time offset to the start-address field (the 14-bit field
// holds smem byte address / 16, which cannot carry for a 227 KB window), and
// every group of MMAs is fully unrolled.
template <int D>
__device__ void mma_issuer(const Shared& sh, const Geom& g, uint32_t tmem, int topk,
                           int* status) {
  using Cf = Cfg<D>;
  constexpr int kK = D / 16;  // k-steps of Q K^T
  const int pairs = (g.C + 1) / 2;
  const int items = g.B * g.H * pairs;
  constexpr uint32_t kIdescQK = idesc_bf16_f32(64, 128, false, false);
  const uint32_t ring_base = smem_u32(sh.base + Cf::kRingOff);
  // Ring position kept as (slot, phase) and advanced incrementally; the K and
  // V descriptors of slot 0 are built once and a slot adds its byte offset / 16
  // to the start-address field.
  uint32_t slot_c = 0, phase_c = 0;
  const uint64_t kdesc_base = sdesc_sw128(ring_base, 16, 1024);
  const uint64_t vdesc_base = sdesc_sw128(ring_base, Cf::kKVHalf, 1024);
  uint32_t p_phase0 = 0u, p_phase1 = 0u, q_phase0 = 0u, q_phase1 = 0u;
  int t = 0;
  for (int item = blockIdx.x; item < items; item += gridDim.x, ++t) {
    if (*sh.abort_flag) return;
    const Item it = decode(g, item, pairs);
    const int qb = t & 1;
    if (!mbar_wait(&sh.q_full[qb], (t >> 1) & 1)) return fail(sh, status);
    tc_fence_after();
    // steps and last-step chunks of both cubes (the producer's chunk counts)
    int n[2], last[2];
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int T = sh.chunks[2 * qb + c];
      n[c] = (T + 7) / 8;
      last[c] = T - 8 * (n[c] - 1);
    }
    auto next_slot = [&](uint32_t& slot) -> bool {
      slot = slot_c;
      if (!mbar_wait(&sh.kv_full[slot], phase_c)) return false;
      if (++slot_c == Cf::kSlots) {
        slot_c = 0;
        phase_c ^= 1u;
      }
      tc_fence_after();
      return true;
    };
    // S_c = Q_c K^T over one step's keys; Q_c read from TMEM
    auto qk = [&](int c, int j) -> bool {
      if (j == 0) {  // the cube's query rows are in TMEM
        uint32_t& qp = c == 0 ? q_phase0 : q_phase1;
        if (!mbar_wait(&sh.q_ready[c], qp)) return false;
        qp ^= 1u;
        tc_fence_after();
      }
      uint32_t slot;
      if (!next_slot(slot)) return false;
      const uint64_t b0 = kdesc_base + (slot * Cf::kSlotBytes >> 4);
      const int nc = j == (c ? n[1] : n[0]) - 1 ? (c ? last[1] : last[0]) : 8;
      const uint32_t idesc = (kIdescQK & ~(0x3Fu << 17)) | (static_cast<uint32_t>(2 * nc) << 17);
      const uint32_t dS = tmem + cube_lanes(c) + Cf::kColS;
      const uint32_t aQ = tmem + cube_lanes(c) + Cf::kColQ;
#pragma unroll
      for (int kk = 0; kk < kK; ++kk) {
        const uint64_t bo = ((kk >> 2) * Cf::kKVHalf + (kk & 3) * 32) >> 4;
        umma_ts(dS, aQ + kk * 8, b0 + bo, idesc, kk > 0 ? 1u : 0u);
      }
      umma_commit(&sh.kv_empty[slot]);
      umma_commit(&sh.s_full[c]);
      return true;
    };
    // O_c += P_c V over one step's keys; P_c read from TMEM
    auto pv = [&](int c, int j) -> bool {
      uint32_t& ph = c == 0 ? p_phase0 : p_phase1;
      if (!mbar_wait(&sh.p_full[c], ph)) return false;
      ph ^= 1u;
      tc_fence_after();
      uint32_t slot;
      if (!next_slot(slot)) return false;
      const uint64_t v0 = vdesc_base + (slot * Cf::kSlotBytes >> 4);
      const uint32_t dO = tmem + cube_lanes(c) + Cf::kColO;
      const uint32_t aP = tmem + cube_lanes(c) + Cf::kColS;
      const int nsteps = c ? n[1] : n[0];
      const int nc = j == nsteps - 1 ? (c ? last[1] : last[0]) : 8;
      const uint32_t acc0 = j > 0 ? 1u : 0u;
      umma_ts(dO, aP, v0, Cf::kIdescPV, acc0);
      if (nc == 8) {
#pragma unroll
        for (int kk = 1; kk < 8; ++kk)
          umma_ts(dO, aP + kk * 8, v0 + (kk * 2048 >> 4), Cf::kIdescPV, 1u);
      } else {
        for (int kk = 1; kk < nc; ++kk)
          umma_ts(dO, aP + kk * 8, v0 + (kk * 2048 >> 4), Cf::kIdescPV, 1u);
      }
      umma_commit(&sh.kv_empty[slot]);
      if (j == nsteps - 1) umma_commit(&sh.o_full[c]);
      return true;
    };
    if (!qk(0, 0)) return fail(sh, status);
    if (n[1] > 0 && !qk(1, 0)) return fail(sh, status);
    // No abort check inside the item: a failed role stops feeding this
    // thread, whose next bounded wait then ends the item.
    const int nmax = max(n[0], n[1]);
    for (int j = 0; j < nmax; ++j) {
      if (j < n[0]) {
        if (!pv(0, j)) return fail(sh, status);
        if (j + 1 < n[0] && !qk(0, j + 1)) return fail(sh, status);
      }
      if (j < n[1]) {
        if (!pv(1, j)) return fail(sh, status);
        if (j + 1 < n[1] && !qk(1, j + 1)) return fail(sh, status);
      }
    }
    umma_commit(&sh.q_empty[qb]);  // Q buffer free once this item's MMAs complete
  }
}

// ------------------------------------------------------------------ softmax
template <int D, bool kTokenOut>
__device__ void softmax_wg(const Shared& sh, const Geom& g, uint32_t tmem, int c,
                           const int32_t* __restrict__ sel, int topk, const OutSpec os,
                           int* status, const int32_t* __restrict__ counts,
                           const __nv_bfloat16* __restrict__ q_tiled) {
  __nv_bfloat16* __restrict__ out = os.out;
  float* __restrict__ lse = os.lse;
  using Cf = Cfg<D>;
  constexpr int kOH = D / 2;  // O columns per thread (half a row)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wq = warp & 3;              // TMEM sub-partition of this warp
  const int hh = lane >> 4;             // which 64-key half of a step this thread holds
  const int r = wq * 16 + (lane & 15);  // query row of the cube
  const uint32_t lane_addr = (static_cast<uint32_t>(wq * 32) << 16) + cube_lanes(c);
  const uint32_t tS = tmem + lane_addr + Cf::kColS;
  const uint32_t tO = tmem + lane_addr + Cf::kColO;
  const uint32_t tQ = tmem + lane_addr + Cf::kColQ;
  const float sl2 = kLog2e * rsqrtf(static_cast<float>(D));
  const int pairs = (g.C + 1) / 2;
  const int items = g.B * g.H * pairs;
  uint32_t s_phase = 0u, o_phase = 0u;

  for (int item = blockIdx.x; item < items; item += gridDim.x) {
    if (*sh.abort_flag) return;
    const Item it = decode(g, item, pairs);
    if (c == 1 && !it.has_b) continue;
    const int i = c == 0 ? it.i0 : it.i1;
    const int ni = cube_valid(g, i);
    const int32_t* list = sel + (static_cast<long long>(it.bh) * g.C + i) * topk;
    {
      // the cube's query rows into TMEM as the A operand of Q K^T (features
      // 2 col, 2 col + 1 packed in column col): this thread's row r, features
      // D/2 hh .. D/2 hh + D/2 - 1.  The previous item's products of this cube
      // have completed: its last S and O were waited for.
      const uint4* qrow = reinterpret_cast<const uint4*>(
          q_tiled + (static_cast<long long>(it.row0) + i * 64 + r) * D + hh * (D / 2));
      if constexpr (D == 128) {
        uint32_t qw[32];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint4 x = __ldg(&qrow[u]);
          qw[4 * u] = x.x;
          qw[4 * u + 1] = x.y;
          qw[4 * u + 2] = x.z;
          qw[4 * u + 3] = x.w;
        }
        tmem_st_16x32bx2_x32(tQ, qw);
      } else {
        uint32_t qw[16];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint4 x = __ldg(&qrow[u]);
          qw[4 * u] = x.x;
          qw[4 * u + 1] = x.y;
          qw[4 * u + 2] = x.z;
          qw[4 * u + 3] = x.w;
        }
        tmem_st_16x32bx2_x16(tQ, qw);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sh.q_ready[c]);
    }
    float m_ref = -INFINITY, l_part = 0.f;
    const int W = count_wide(g, list, topk, lane, nullptr);
    const int T = 3 * W + topk;  // 16-row key chunks of the cube
    // list entries of this thread's four chunks (the half-step from chunk
    // 8j + 4hh), fetched one step ahead
    auto fetch = [&](int j, Ahead (&a)[4]) {
      const int cb = 8 * j + 4 * hh;
      const int kind = half_kind(cb, W, T);
#pragma unroll
      for (int q = 0; q < 4; ++q) a[q] = fetch_entry(list, kind == 0 ? -1 : half_entry(cb, q, W, topk));
    };
    Ahead ahead[4];
    fetch(0, ahead);
    for (int j = 0; 8 * j < T; ++j) {
      // valid key rows of this thread's four chunks, from the cube_count table
      // (checked against the grid by the producer; a mismatch is reported as
      // VSA_ERR_BAD_INDEX, and since counts only set masks, never addresses,
      // it cannot make the kernel read or write out of bounds)
      const bool wide = half_kind(8 * j + 4 * hh, W, T) == 1;
      int vc[4];
      if (wide) {
        const int n = __ldg(&counts[cube_of(g, ahead[0])]);
#pragma unroll
        for (int q = 0; q < 4; ++q) vc[q] = min(16, max(0, n - 16 * q));
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int cq = cube_of(g, ahead[q]);
          vc[q] = cq >= 0 ? __ldg(&counts[cq]) : 0;
        }
      }
      fetch(j + 1, ahead);
      if (!mbar_wait(&sh.s_full[c], s_phase)) return fail(sh, status);
      s_phase ^= 1u;
      tc_fence_after();
      uint32_t sv[64];
      tmem_ld_16x32bx2_x64(tS, sv);
      if ((vc[0] & vc[1] & vc[2] & vc[3]) != 16) {  // mask pad and absent key rows
#pragma unroll
        for (int e = 0; e < 64; ++e)
          if ((e & 15) >= vc[e >> 4]) sv[e] = __float_as_uint(-INFINITY);
      }
      float mx8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mx8[u] = __uint_as_float(sv[u]);
#pragma unroll
      for (int e = 8; e < 64; ++e) mx8[e & 7] = fmaxf(mx8[e & 7], __uint_as_float(sv[e]));
      float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                       fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const float mx2 = mx * sl2;
      float alpha = 1.f;
      bool need = false;
      if (j == 0) {
        m_ref = mx2;
      } else if (mx2 > m_ref + kRescaleLog2) {
        alpha = exp2f(m_ref - mx2);
        m_ref = mx2;
        need = true;
      }
      if (__any_sync(0xffffffffu, need)) {  // the previous P V has completed
        uint32_t ov[kOH];
        if constexpr (kOH == 64) {
          tmem_ld_16x32bx2_x64(tO, ov);
        } else {
          tmem_ld_16x32bx2_x32(tO, ov);
        }
#pragma unroll
        for (int e = 0; e < kOH; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
        if constexpr (kOH == 64) {
          tmem_st_16x32bx2_x64(tO, ov);
        } else {
          tmem_st_16x32bx2_x32(tO, ov);
        }
      }
      l_part *= alpha;
      float sum8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      uint32_t pk[32];
      const float neg_m = -m_ref;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float p0 = fast_exp2(fmaf(__uint_as_float(sv[2 * e]), sl2, neg_m));
        const float p1 = fast_exp2(fmaf(__uint_as_float(sv[2 * e + 1]), sl2, neg_m));
        sum8[e & 7] += p0 + p1;
        pk[e] = pack2_bf16(p0, p1);
      }
      l_part += ((sum8[0] + sum8[1]) + (sum8[2] + sum8[3])) + ((sum8[4] + sum8[5]) + (sum8[6] + sum8[7]));
      tmem_st_16x32bx2_x32(tS, pk);  // P over the first 64 columns of S
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sh.p_full[c]);
    }
    // ---- epilogue: O / l -> bf16; pad rows -> 0 (tiled) or no write (token order)
    const bool valid = r < ni;
    // token-order output: the row's token and gates, ahead of the O load so
    // they are not live beside its registers
    long long tok = 0;
    float wf = 0.f, wc = 0.f;
    if (kTokenOut && valid) {
      tok = static_cast<long long>(it.bh) * g.N + slot_token(g, i, r);
      if (os.g_fine != nullptr) {
        wf = __ldg(&os.g_fine[tok]);
        wc = __ldg(&os.g_coarse[tok]);
      }
    }
    if (!mbar_wait(&sh.o_full[c], o_phase)) return fail(sh, status);
    o_phase ^= 1u;
    tc_fence_after();
    uint32_t ov[kOH];
    if constexpr (kOH == 64) {
      tmem_ld_16x32bx2_x64(tO, ov);
    } else {
      tmem_ld_16x32bx2_x32(tO, ov);
    }
    const float l = l_part + __shfl_xor_sync(0xffffffffu, l_part, 16);
    const float inv = 1.0f / l;
    if (!kTokenOut) {
      uint4* orow = reinterpret_cast<uint4*>(
          out + (static_cast<long long>(it.row0) + i * 64 + r) * D + hh * kOH);
#pragma unroll
      for (int q8 = 0; q8 < kOH / 8; ++q8) {
        uint4 w = make_uint4(0u, 0u, 0u, 0u);
        if (valid) {
          w.x = pack2_bf16(__uint_as_float(ov[q8 * 8 + 0]) * inv, __uint_as_float(ov[q8 * 8 + 1]) * inv);
          w.y = pack2_bf16(__uint_as_float(ov[q8 * 8 + 2]) * inv, __uint_as_float(ov[q8 * 8 + 3]) * inv);
          w.z = pack2_bf16(__uint_as_float(ov[q8 * 8 + 4]) * inv, __uint_as_float(ov[q8 * 8 + 5]) * inv);
          w.w = pack2_bf16(__uint_as_float(ov[q8 * 8 + 6]) * inv, __uint_as_float(ov[q8 * 8 + 7]) * inv);
        }
        orow[q8] = w;
      }
    } else if (valid) {
      // pad rows have no token and write nothing
      uint4* orow = reinterpret_cast<uint4*>(out + tok * D + hh * kOH);
      const bool gated = os.g_fine != nullptr;
      const float4* oc = reinterpret_cast<const float4*>(
          os.o_coarse + (static_cast<long long>(it.bh) * g.C + i) * D + hh * kOH);
#pragma unroll
      for (int q8 = 0; q8 < kOH / 8; ++q8) {
        uint32_t f[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          f[e] = pack2_bf16(__uint_as_float(ov[q8 * 8 + 2 * e]) * inv,
                            __uint_as_float(ov[q8 * 8 + 2 * e + 1]) * inv);
        if (gated) {  // the combine step's arithmetic on the bf16 fine output
          const float4 c0 = __ldg(&oc[2 * q8]);
          const float4 c1 = __ldg(&oc[2 * q8 + 1]);
          const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
          for (int e = 0; e < 4; ++e)
            f[e] = pack2_bf16(fmaf(wf, __uint_as_float(f[e] << 16), wc * cv[2 * e]),
                              fmaf(wf, __uint_as_float(f[e] & 0xFFFF0000u), wc * cv[2 * e + 1]));
        }
        orow[q8] = make_uint4(f[0], f[1], f[2], f[3]);
      }
    }
    if (lse != nullptr && hh == 0)
      lse[static_cast<long long>(it.row0) + i * 64 + r] =
          valid ? (m_ref + log2f(l)) * kLn2 : -INFINITY;
  }
}

template <int D, bool kTokenOut>
__global__ void __launch_bounds__(kThreads, 1) fine_fwd_kernel(
    const __grid_constant__ FineMaps maps, Geom g, const int32_t* __restrict__ counts,
    const int32_t* __restrict__ sel, int topk, const OutSpec os, int* status,
    const __nv_bfloat16* __restrict__ q_tiled) {
  using Cf = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cf::kBarOff);
  Shared sh;
  sh.base = smem;
  sh.q_full = bars;
  sh.q_empty = bars + 2;
  sh.kv_full = bars + 4;
  sh.kv_empty = bars + 4 + Cf::kSlots;
  sh.s_full = bars + 4 + 2 * Cf::kSlots;
  sh.p_full = sh.s_full + 2;
  sh.o_full = sh.s_full + 4;
  sh.q_ready = sh.s_full + 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sh.q_ready + 2);
  sh.abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  sh.chunks = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    for (int q = 0; q < 2; ++q) {
      mbar_init(&sh.q_full[q], 1);
      mbar_init(&sh.q_empty[q], 1);
      mbar_init(&sh.s_full[q], 1);
      mbar_init(&sh.p_full[q], 128);
      mbar_init(&sh.o_full[q], 1);
      mbar_init(&sh.q_ready[q], 128);
    }
    for (int s = 0; s < Cf::kSlots; ++s) {
      mbar_init(&sh.kv_full[s], 1);
      mbar_init(&sh.kv_empty[s], 1);
    }
    *sh.abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&maps.q);
    prefetch_tmap(&maps.k);
    prefetch_tmap(&maps.v);
    prefetch_tmap(&maps.k16);
    prefetch_tmap(&maps.v16);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kProducerWarp) {
    producer<D>(sh, g, maps, counts, sel, topk, status);
  } else if (warp == kMmaWarp) {
    if (lane == 0) mma_issuer<D>(sh, g, tmem, topk, status);
  } else if (warp >= kSoftmaxWarp0) {
    softmax_wg<D, kTokenOut>(sh, g, tmem, (warp - kSoftmaxWarp0) >> 2, sel, topk, os, status, counts,
                             q_tiled);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

size_t fine_smem_bytes(int d) { return d == 128 ? Cfg<128>::kSmem : Cfg<64>::kSmem; }

cudaError_t launch_block_sparse_fwd(const Geom& g, const FineMaps& maps, const int32_t* counts,
                                    const int32_t* sel, int topk, void* out, float* lse,
                                    const float* o_coarse, const float* g_fine,
                                    const float* g_coarse, bool token_order, int* status, int sms,
                                    cudaStream_t s, const void* q_tiled) {
  const long long items = static_cast<long long>(g.B) * g.H * ((g.C + 1) / 2);
  const int grid = static_cast<int>(items < sms ? items : sms);
  const size_t smem = fine_smem_bytes(g.d);
  const OutSpec os{static_cast<__nv_bfloat16*>(out), lse, o_coarse, g_fine, g_coarse,
                   token_order ? 1 : 0};
  cudaError_t err;
  // one kernel per head dim and output form; each raises its smem limit once
  static CtxCache<char> limit_set[4];
  auto run = [&](auto kernel, int which) -> cudaError_t {
    cudaError_t e = smem_limit_once(kernel, static_cast<int>(smem), &limit_set[which]);
    if (e != cudaSuccess) return e;
    kernel<<<grid, kThreads, smem, s>>>(maps, g, counts, sel, topk, os, status,
                                        static_cast<const __nv_bfloat16*>(q_tiled));
    return cudaSuccess;
  };
  if (g.d == 128)
    err = token_order ? run(fine_fwd_kernel<128, true>, 0) : run(fine_fwd_kernel<128, false>, 1);
  else
    err = token_order ? run(fine_fwd_kernel<64, true>, 2) : run(fine_fwd_kernel<64, false>, 3);
  if (err != cudaSuccess) return err;
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
