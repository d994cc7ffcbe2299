// Token <-> cube permutation and the gated combine: HBM-bound passes that
// move 16-byte chunks (8 bf16) with one thread per chunk of the written
// tensor, so every store is a coalesced 128-bit store.
//
// Tiling (FastWan article "单块 H200 ... 5 秒即生一个 5 秒视频", section
// "一张卡，秒生视频": 64-token blocks of the 64x64 block-sparse mask): the
// latent grid is cut into 4x4x4 cubes in row-major cube order; a cube's valid
// tokens fill its first n_c slots in row-major local (t, y, x) order and the
// other slots are zero.  Because the valid tokens of a partial cube form the
// sub-box [0,nt) x [0,ny) x [0,nx) of the cube, slot s holds local offset
// (s / (ny*nx), (s / nx) % ny, s % nx).
#include "common.cuh"

namespace vsa {

namespace {

__global__ void __launch_bounds__(256) tile_permute_kernel(Geom g, const uint4* __restrict__ x,
                                                           uint4* __restrict__ xt,
                                                           int32_t* __restrict__ counts) {
  // All row indices fit in 32 bits (the host rejects B*H*64*C >= 2^31), so
  // the per-chunk divisions are 32-bit; only byte offsets are 64-bit.
  const int lg_ch = (g.d == 128) ? 4 : 3;  // 16-byte chunks per row: d/8
  const unsigned rows = static_cast<unsigned>(g.rows);
  const unsigned total_rows = static_cast<unsigned>(g.B * g.H) * rows;
  const unsigned rows_per_pass = (gridDim.x * blockDim.x) >> lg_ch;
  const int ch = threadIdx.x & ((1 << lg_ch) - 1);
  for (unsigned row = (blockIdx.x * blockDim.x + threadIdx.x) >> lg_ch; row < total_rows;
       row += rows_per_pass) {
    const unsigned bh = row / rows;
    const unsigned r = row - bh * rows;
    const long long n = slot_token(g, static_cast<int>(r >> 6), static_cast<int>(r & 63));
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (n >= 0) v = __ldg(&x[((static_cast<long long>(bh) * g.N + n) << lg_ch) + ch]);
    xt[(static_cast<long long>(row) << lg_ch) + ch] = v;
  }
  if (counts != nullptr && blockIdx.x == 0) {
    for (int c = threadIdx.x; c < g.C; c += blockDim.x) counts[c] = cube_valid(g, c);
  }
}

__global__ void __launch_bounds__(256) untile_kernel(Geom g, const uint4* __restrict__ xt,
                                                     uint4* __restrict__ x) {
  const int lg_ch = (g.d == 128) ? 4 : 3;
  const unsigned N = static_cast<unsigned>(g.N);
  const unsigned total_tok = static_cast<unsigned>(g.B * g.H) * N;
  const unsigned tok_per_pass = (gridDim.x * blockDim.x) >> lg_ch;
  const int ch = threadIdx.x & ((1 << lg_ch) - 1);
  for (unsigned tok = (blockIdx.x * blockDim.x + threadIdx.x) >> lg_ch; tok < total_tok;
       tok += tok_per_pass) {
    const unsigned bh = tok / N;
    const unsigned n = tok - bh * N;
    const unsigned ty = n / static_cast<unsigned>(g.X);
    const int xg = static_cast<int>(n - ty * static_cast<unsigned>(g.X));
    const unsigned tg_u = ty / static_cast<unsigned>(g.Y);
    const int yg = static_cast<int>(ty - tg_u * static_cast<unsigned>(g.Y));
    const int tg = static_cast<int>(tg_u);
    const int c = ((tg >> 2) * g.Cy + (yg >> 2)) * g.Cx + (xg >> 2);
    int nt, ny, nx, t0, y0, x0;
    cube_extent(g, c, nt, ny, nx, t0, y0, x0);
    const int s = ((tg - t0) * ny + (yg - y0)) * nx + (xg - x0);
    x[(static_cast<long long>(tok) << lg_ch) + ch] =
        __ldg(&xt[((static_cast<long long>(bh) * g.rows + c * kSlots + s) << lg_ch) + ch]);
  }
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&p);
}

// `of` and `out` may alias (in-place combine): each element is read and then
// written by the same thread, so no restrict / read-only-cache loads on them.
__global__ void __launch_bounds__(256) combine_kernel(Geom g, const uint4* of,
                                                      const float4* __restrict__ oc,
                                                      const float* __restrict__ gf,
                                                      const float* __restrict__ gc,
                                                      uint4* out) {
  const int lg_ch = (g.d == 128) ? 4 : 3;
  const unsigned rows = static_cast<unsigned>(g.rows);
  const unsigned total_rows = static_cast<unsigned>(g.B * g.H) * rows;
  const unsigned rows_per_pass = (gridDim.x * blockDim.x) >> lg_ch;
  const int ch = threadIdx.x & ((1 << lg_ch) - 1);
  for (unsigned row_u = (blockIdx.x * blockDim.x + threadIdx.x) >> lg_ch; row_u < total_rows;
       row_u += rows_per_pass) {
    const long long o = (static_cast<long long>(row_u) << lg_ch) + ch;
    const long long bh = row_u / rows;
    const int r = static_cast<int>(row_u - static_cast<unsigned>(bh) * rows);
    const int c = r >> 6;
    const long long n = slot_token(g, c, r & 63);
    uint4 res = make_uint4(0u, 0u, 0u, 0u);
    if (n >= 0 && gf == nullptr) {
      res = of[o];  // ungated: out = O_f
    } else if (n >= 0) {
      const float wf = __ldg(&gf[bh * g.N + n]);
      const float wc = __ldg(&gc[bh * g.N + n]);
      const uint4 f = of[o];
      const long long cb = ((bh * g.C + c) * g.d + ch * 8) >> 2;  // float4 index
      const float4 c0 = __ldg(&oc[cb]);
      const float4 c1 = __ldg(&oc[cb + 1]);
      res.x = pack_bf16(fmaf(wf, bf16_lo(f.x), wc * c0.x), fmaf(wf, bf16_hi(f.x), wc * c0.y));
      res.y = pack_bf16(fmaf(wf, bf16_lo(f.y), wc * c0.z), fmaf(wf, bf16_hi(f.y), wc * c0.w));
      res.z = pack_bf16(fmaf(wf, bf16_lo(f.z), wc * c1.x), fmaf(wf, bf16_hi(f.z), wc * c1.y));
      res.w = pack_bf16(fmaf(wf, bf16_lo(f.w), wc * c1.z), fmaf(wf, bf16_hi(f.w), wc * c1.w));
    }
    out[o] = res;
  }
}

int stream_grid(long long chunks, int sms) {
  const long long want = (chunks + 255) / 256;
  const long long cap = static_cast<long long>(sms) * 16;  // 16 resident 256-thread CTAs per SM
  return static_cast<int>(want < cap ? (want > 0 ? want : 1) : cap);
}

}  // namespace

cudaError_t launch_tile_permute(const Geom& g, const void* x, void* xt, int32_t* counts,
                                int sms, cudaStream_t s) {
  const long long chunks = static_cast<long long>(g.B) * g.H * g.rows * (g.d / 8);
  tile_permute_kernel<<<stream_grid(chunks, sms), 256, 0, s>>>(
      g, static_cast<const uint4*>(x), static_cast<uint4*>(xt), counts);
  return cudaGetLastError();
}

cudaError_t launch_untile(const Geom& g, const void* xt, void* x, int sms, cudaStream_t s) {
  const long long chunks = static_cast<long long>(g.B) * g.H * g.N * (g.d / 8);
  untile_kernel<<<stream_grid(chunks, sms), 256, 0, s>>>(g, static_cast<const uint4*>(xt),
                                                         static_cast<uint4*>(x));
  return cudaGetLastError();
}

cudaError_t launch_combine(const Geom& g, const void* of, const float* oc, const float* gf,
                           const float* gc, void* out, int sms, cudaStream_t s) {
  const long long chunks = static_cast<long long>(g.B) * g.H * g.rows * (g.d / 8);
  if (gf == nullptr && out == of) return cudaSuccess;  // ungated and in place: nothing to do
  combine_kernel<<<stream_grid(chunks, sms), 256, 0, s>>>(
      g, static_cast<const uint4*>(of), reinterpret_cast<const float4*>(oc), gf, gc,
      static_cast<uint4*>(out));
  return cudaGetLastError();
}

}  // namespace vsa
