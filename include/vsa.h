/*
 * vsa.h -- C ABI of the B200 (sm_100a) video sparse attention (VSA) forward path.
 *
 * VSA is the trainable, dynamic block-sparse attention of FastWan ("单块 H200
 * ... 5 秒即生一个 5 秒视频", section "一张卡，秒生视频"; restated in
 * "超越Sora：FastWan如何以“稀疏蒸馏”重塑实时AI视频生成范式", section
 * "技术原理与创新点解析").  A coarse stage looks at the whole sequence at
 * block granularity and picks, for every query block, the key blocks that
 * matter; a fine block-sparse kernel then runs exact attention over those
 * 64x64 blocks only.  The pages name the stages but print no formula; the
 * readings taken here are stated with each call.
 *
 * Terms
 *   B       batch, H heads, d head dim (64 or 128)
 *   grid    latent token grid T x Hg x Wg; N = T*Hg*Wg tokens in row-major
 *           (t, y, x) order, token n = (t*Hg + y)*Wg + x
 *   cube    4x4x4 block of the grid = 64 token slots.  Cube c = (ct*Cy+cy)*Cx+cx
 *           with Ct = ceil(T/4), Cy = ceil(Hg/4), Cx = ceil(Wg/4), C = Ct*Cy*Cx.
 *           Edge cubes of a grid whose sides are not multiples of 4 are
 *           partial: they hold n_c < 64 tokens.
 *   tiled   [B, H, 64*C, d] layout: cube c owns rows 64c .. 64c+63; its n_c
 *           tokens fill the first n_c rows in row-major local (t, y, x)
 *           order; the remaining rows are zero padding.
 *   k       number of key cubes each query cube attends to (1 <= k <= C).
 *
 * Conventions (every call)
 *   - Tensor pointers are DEVICE pointers owned by the caller, contiguous
 *     row-major, 16-byte aligned.  bf16 tensors are IEEE bfloat16 bit
 *     patterns.  The library allocates no device memory; scratch comes from
 *     the caller's workspace (vsa_coarse_select).
 *   - Every call is asynchronous on `stream`.  A call returns VSA_OK after a
 *     successful launch; argument errors are reported before any launch and
 *     nothing is written.
 *   - Device-side conditions (a bounded wait that ran out, an inconsistent
 *     cube_count / sel_idx entry) are recorded in a status word of the
 *     current CUDA context, read and cleared by vsa_get_status().  Kernels
 *     never trap.
 *   - Calls work in whatever CUDA context is current on the calling thread
 *     (the device's primary context by default); values the library keeps
 *     per context (the status word's address, raised kernel limits, the host
 *     path's copy streams) are looked up again in a new context.
 *   - Calls on one device from several host threads are safe; calls that
 *     overlap on the GPU and write the same output race, as any CUDA kernel.
 */
#ifndef VSA_H_
#define VSA_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

enum vsa_status_code {
  VSA_OK = 0,
  VSA_ERR_INVALID_ARG = 1,  /* null / misaligned pointer, bad size, k not in [1, C] */
  VSA_ERR_UNSUPPORTED = 2,  /* cube not 4x4x4, d not in {64, 128}, device not sm_100 */
  VSA_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
  VSA_ERR_TIMEOUT = 4,      /* device: a bounded wait ran out (status word) */
  VSA_ERR_BAD_INDEX = 5,    /* device: cube_count or sel_idx entry inconsistent (status word) */
  VSA_ERR_TOO_LARGE = 6     /* problem needs more scratch than vsa_coarse_select_noalloc holds */
};

typedef struct vsa_shape {
  int batch;                       /* B >= 1 */
  int heads;                       /* H >= 1 */
  int head_dim;                    /* d: 64 or 128 */
  int grid_t, grid_h, grid_w;      /* latent token grid, each >= 1 */
  int cube_t, cube_h, cube_w;      /* must be 4, 4, 4 */
} vsa_shape;

/* Host-only helper: C = ceil(T/4)*ceil(Hg/4)*ceil(Wg/4).  No GPU work. */
int vsa_num_cubes(const vsa_shape* shape, int* num_cubes);

/* Host-only helper: k from a top-k ratio r of the C cubes,
 * k = max(1, floor(r*C + 0.5)).  A ratio of 0.1 is the 90 % attention
 * sparsity of the TurboDiffusion review (section "評估 / 設置"); 0.125 is the
 * 87.5 % sparsity of the FastWan scaling experiment.  r must be in (0, 1]. */
int vsa_topk_from_ratio(int num_cubes, float ratio, int* topk);

/* Bytes of device workspace vsa_coarse_select needs for this shape and k
 * (pooled q, k, v in float32: 3*B*H*C*d*4 bytes, rounded up to 256). */
size_t vsa_workspace_bytes(const vsa_shape* shape, int topk);

/* Token -> cube permutation (the 4x4x4 tiling the coarse and fine stages
 * work on; 64-token blocks are the 64x64 blocks of the fine kernel).
 *   x          bf16 [B, H, N, d], token order           (read)
 *   x_tiled    bf16 [B, H, 64*C, d], tiled; pad rows 0  (written)
 *   cube_count int32 [C] valid tokens per cube, or NULL (written)
 * One call per tensor (q, k, v). */
int vsa_tile_permute(const vsa_shape* shape, const void* x, void* x_tiled,
                     int32_t* cube_count, cudaStream_t stream);

/* Coarse stage (FastWan article, section "一张卡，秒生视频", Fig. 5
 * paragraph: the block-sparse attention the coarse stage produces is highly
 * dynamic).  Reading taken: each cube is mean-pooled over its n_c valid
 * tokens (qbar, kbar, vbar); coarse attention over the C pooled vectors with
 * scale 1/sqrt(d) gives the coarse output O_c = softmax(qbar kbar^T/sqrt(d)) vbar;
 * for each query cube the k key cubes with the largest coarse logits are
 * selected, ties to the lower index.  Each row lists the selected key cubes
 * that hold more than 16 valid tokens first, then the others, each group in
 * ascending index order (the order in which the fine stage packs key rows:
 * a cube of at most 16 tokens costs it a quarter of a full cube; on a grid
 * whose sides are multiples of 4 every cube is full and the order is plain
 * ascending).  Logits are computed in float32.
 *   q_tiled, k_tiled, v_tiled  bf16 [B, H, 64*C, d] from vsa_tile_permute
 *   cube_count   int32 [C] as written by vsa_tile_permute for this shape
 *                (checked against the grid; a mismatch is recorded as
 *                VSA_ERR_BAD_INDEX and the grid's count is used)
 *   topk         k, 1 <= k <= C
 *   o_coarse     float32 [B, H, C, d] coarse output, or NULL
 *   sel_idx      int32 [B, H, C, k] selected key cubes (written)
 *   coarse_logits float32 [B, H, C, C] scaled logits, or NULL (diagnostics)
 *   workspace    device scratch of at least vsa_workspace_bytes(shape, k)
 *                bytes, 256-byte aligned; contents on entry are ignored */
int vsa_coarse_select(const vsa_shape* shape, const void* q_tiled, const void* k_tiled,
                      const void* v_tiled, const int32_t* cube_count, int topk,
                      float* o_coarse, int32_t* sel_idx, float* coarse_logits,
                      void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Tiling and pooling in one pass over q, k, v: writes q_tiled, k_tiled,
 * v_tiled and cube_count exactly as three vsa_tile_permute calls, and the
 * per-cube means (float32, the first 3*B*H*C*d*4 bytes of the workspace, in
 * the layout vsa_coarse_select uses) exactly as vsa_coarse_select's pooling,
 * so each input tensor is read once.  The pages have no counterpart: this is
 * the coarse stage's pooling fused into the tiling pass.
 *   q, k, v          bf16 [B, H, N, d] token order
 *   *_tiled          bf16 [B, H, 64*C, d] (written)
 *   cube_count       int32 [C] or NULL (written)
 *   workspace        >= vsa_workspace_bytes(shape, 1) bytes, 256-byte aligned */
int vsa_tile_permute_pool(const vsa_shape* shape, const void* q, const void* k, const void* v,
                          void* q_tiled, void* k_tiled, void* v_tiled, int32_t* cube_count,
                          void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* The coarse stage after vsa_tile_permute_pool: coarse attention, top-k and
 * O_c from the cube means already in `workspace` (same outputs, bit for bit,
 * as vsa_coarse_select on the tiled tensors).  Arguments as vsa_coarse_select
 * minus the tensors. */
int vsa_coarse_select_pooled(const vsa_shape* shape, int topk, float* o_coarse, int32_t* sel_idx,
                             float* coarse_logits, const void* workspace, size_t workspace_bytes,
                             cudaStream_t stream);

/* vsa_coarse_select on the TOKEN-ORDER tensors: the same result (pooled
 * vectors, logits, selection, O_c) without waiting for vsa_tile_permute, so a
 * caller can run the coarse stage on a second stream while q, k, v are tiled
 * for the fine stage.  The pages have no counterpart: this is a scheduling
 * convenience; the cube means are summed in the same row order as
 * vsa_coarse_select, so both calls return identical bits.
 *   q, k, v      bf16 [B, H, N, d] in token order
 *   other arguments as vsa_coarse_select (no cube_count input) */
int vsa_coarse_select_tokens(const vsa_shape* shape, const void* q, const void* k, const void* v,
                             int topk, float* o_coarse, int32_t* sel_idx, float* coarse_logits,
                             void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* vsa_coarse_select for callers that cannot allocate device memory.  The
 * pages have no counterpart: this is a library convenience.  Some callers own
 * no device allocator (a plugin inside a host application that manages all
 * device memory itself) or must not call cudaMalloc while work is in flight
 * (it may synchronise the device); they cannot provide the workspace that
 * vsa_coarse_select needs.  This variant takes the same arguments minus the
 * workspace and computes the same result with the same kernels, using a
 * fixed 32 MiB device array inside the library as its scratch.
 *   - Limit: 3*B*H*C*d*4 bytes of pooled q, k, v must fit in 32 MiB, i.e.
 *     B*H*C*d <= 2,796,202 (e.g. 12 heads x 1440 cubes x d=128 fits; 40 heads
 *     of the 21x45x80 grid do not).  Larger problems return VSA_ERR_TOO_LARGE
 *     before any launch; use vsa_coarse_select with a workspace for them.
 *   - Every GPU context that loads the library holds the 32 MiB from module
 *     load until the process exits.
 *   - The first call in each CUDA context (the device's primary context, a
 *     context the caller made current, or the new primary context after
 *     cudaDeviceReset) looks up the array's device address in that context;
 *     make that first call before any stream capture.
 *   - All calls on a device share the one array: calls that overlap on the
 *     GPU (different streams, no ordering between them) race on it.  Calls
 *     ordered on one stream are safe.  The array keeps the last call's
 *     pooled vectors; every call overwrites what it reads.
 *   - Allocates nothing: no cudaMalloc / cudaFree or allocating library call. */
int vsa_coarse_select_noalloc(const vsa_shape* shape, const void* q_tiled, const void* k_tiled,
                              const void* v_tiled, const int32_t* cube_count, int topk,
                              float* o_coarse, int32_t* sel_idx, float* coarse_logits,
                              cudaStream_t stream);

/* Fine stage: block-sparse attention over the selected 64x64 blocks (FastWan
 * article, section "一张卡，秒生视频": the fine block-sparse kernel, 64x64
 * block mask).  For every valid query token r of cube i:
 *   O_f[r] = softmax_t(q_r . k_t / sqrt(d)) v_t  over the valid tokens t of
 * the cubes in sel_idx[b, h, i, :].  Pad key slots are masked out; pad query
 * rows are written as 0.  bf16 in, float32 accumulation, bf16 out.
 *   q_tiled, k_tiled, v_tiled  bf16 [B, H, 64*C, d]
 *   cube_count   int32 [C] (checked as in vsa_coarse_select)
 *   sel_idx      int32 [B, H, C, k], entries in [0, C), each row in the
 *                order vsa_coarse_select writes: key cubes with more than 16
 *                valid tokens first, then the others, each group strictly
 *                ascending (an entry out of range or out of order is recorded
 *                as VSA_ERR_BAD_INDEX; out-of-range entries are clamped)
 * The kernel packs the key rows of a query cube's selection into 128-row
 * steps: a cube of more than 16 tokens takes 64 rows, one of at most 16 takes
 * 16 rows, so the partial cubes at the edges of a ragged grid cost a quarter
 * of a full cube.
 *   o_fine_tiled bf16 [B, H, 64*C, d] (written)
 *   lse          float32 [B, H, 64*C] natural-log log-sum-exp of each valid
 *                row's scaled scores (-inf for pad rows), or NULL */
int vsa_block_sparse_fwd(const vsa_shape* shape, const void* q_tiled, const void* k_tiled,
                         const void* v_tiled, const int32_t* cube_count,
                         const int32_t* sel_idx, int topk, void* o_fine_tiled,
                         float* lse, cudaStream_t stream);

/* vsa_block_sparse_fwd whose epilogue writes the FINAL output: each valid row
 * of O_f goes straight to its token in `out` (token order, as vsa_untile
 * would put it), and with gates the row is first combined exactly as
 * vsa_combine does (g_fine * bf16(O_f) + g_coarse * O_c, rounded to bf16).
 * Same bits as vsa_block_sparse_fwd + vsa_combine + vsa_untile; the pages have
 * no counterpart: this is the combine and untile steps fused into the fine
 * kernel, which saves two passes over the output.
 *   q/k/v_tiled, cube_count, sel_idx, topk, lse   as vsa_block_sparse_fwd
 *   o_coarse     float32 [B, H, C, d] (may be NULL when the gates are NULL)
 *   g_fine, g_coarse float32 [B, H, N] in token order, or both NULL
 *   out          bf16 [B, H, N, d] token order (written) */
int vsa_block_sparse_fwd_out(const vsa_shape* shape, const void* q_tiled, const void* k_tiled,
                             const void* v_tiled, const int32_t* cube_count, const int32_t* sel_idx,
                             int topk, const float* o_coarse, const float* g_fine,
                             const float* g_coarse, void* out, float* lse, cudaStream_t stream);

/* Optional per-token gated sum of the fine and coarse outputs, in tiled order:
 *   out[r] = g_fine[n] * O_f[r] + g_coarse[n] * O_c[cube of r]
 * where n is the token held by tiled row r.  With g_fine == g_coarse == NULL,
 * out = O_f (a copy).  Either both gates are given or neither.
 *   o_fine_tiled bf16 [B, H, 64*C, d]
 *   o_coarse     float32 [B, H, C, d] (may be NULL when the gates are NULL)
 *   g_fine, g_coarse float32 [B, H, N] in TOKEN order, or both NULL
 *   out_tiled    bf16 [B, H, 64*C, d]; pad rows 0 (may alias o_fine_tiled) */
int vsa_combine(const vsa_shape* shape, const void* o_fine_tiled, const float* o_coarse,
                const float* g_fine, const float* g_coarse, void* out_tiled,
                cudaStream_t stream);

/* Inverse of vsa_tile_permute: bf16 [B, H, 64*C, d] -> bf16 [B, H, N, d];
 * pad rows are dropped. */
int vsa_untile(const vsa_shape* shape, const void* x_tiled, void* x, cudaStream_t stream);

/* Bytes of device workspace vsa_linear_branch_add needs for this shape
 * (phi(q) and phi(k) as bf16, per-chunk float32 partial sums of KV and z, and
 * the bf16 [KV^T ; z^T] matrix of every (b, h)), or 0 for an invalid shape. */
size_t vsa_linear_workspace_bytes(const vsa_shape* shape);

/* Low-rank linear compensation branch, added to an output in place (the
 * sparse + linear variant: the SparkDiffusion page, RoLA paragraph, pairs a
 * block-sparse branch with a low-rank linear branch that keeps the global
 * context at 97 % sparsity; the TurboDiffusion review names trainable
 * sparse-linear attention).  The pages print no formula; reading taken: for
 * every token r of each (b, h) sequence,
 *   out[r] += phi(q_r)^T KV / (phi(q_r)^T z),
 *   KV = sum over all tokens t of phi(k_t) v_t^T,  z = sum_t phi(k_t),
 * with phi(x) = elu(x) + 1 (positive, so the divisor never vanishes); the
 * N x N attention matrix of this branch has rank at most d.  Run after the
 * block-sparse forward (for example vsa_block_sparse_fwd_out) to get
 * out = O_block_sparse + O_linear.  The two products run on the tensor cores
 * with bf16 operands (phi(q), phi(k), KV and z rounded to bf16) and float32
 * accumulation, in a fixed summation order (deterministic); the sum is
 * rounded to bf16.  On a wait that exceeds its bound the kernels record
 * VSA_ERR_TIMEOUT and stop.
 *   q, k, v   bf16 [B, H, N, d] token order (read)
 *   out       bf16 [B, H, N, d] token order (read and written)
 *   workspace device scratch of at least vsa_linear_workspace_bytes(shape)
 *             bytes, 256-byte aligned; contents on entry are ignored */
int vsa_linear_branch_add(const vsa_shape* shape, const void* q, const void* k, const void* v,
                          void* out, void* workspace, size_t workspace_bytes,
                          cudaStream_t stream);

/* QKV projection of a DiT attention block with the tile permutation in its
 * epilogue (FastWan news article, section "一张卡，秒生视频": VSA runs inside
 * whole DiT blocks, between the QKV and the output projection; the pages give
 * no formula, reading: the linear-layer convention, no bias):
 *   [q | k | v] = x W_qkv^T, the 3 H d output features ordered q heads, k
 *   heads, v heads (head h = features h d .. h d + d - 1),
 * written straight into the tiled layout vsa_tile_permute produces (pad rows
 * zero), plus the cube counts; bf16 operands, float32 accumulation on the
 * tensor cores, bf16 results.
 *   hidden        input features, a positive multiple of 64
 *   x             bf16 [B, N, hidden] token order (read)
 *   w_qkv         bf16 [3*H*d, hidden] (read)
 *   q/k/v_tiled   bf16 [B, H, 64*C, d] (written, pad rows included)
 *   cube_count    int32 [C] (written) or NULL
 * Pointers 16-byte aligned.  On a wait that exceeds its bound the kernel
 * records VSA_ERR_TIMEOUT and stops. */
int vsa_qkv_projection_tiled(const vsa_shape* shape, int hidden, const void* x, const void* w_qkv,
                             void* q_tiled, void* k_tiled, void* v_tiled, int32_t* cube_count,
                             cudaStream_t stream);

/* Output projection of a DiT attention block reading the attention output in
 * the tiled layout, with the untile step in its epilogue:
 *   y[b, n] = concat over heads h of o[b, h, n] times W_o^T
 * where o[b, h, n] is the tiled row of token n (pad rows are read but never
 * written anywhere).
 *   hidden    output features, a positive multiple of 64
 *   o_tiled   bf16 [B, H, 64*C, d], e.g. vsa_block_sparse_fwd's or
 *             vsa_combine's output (read)
 *   w_o       bf16 [hidden, H*d] (read)
 *   y         bf16 [B, N, hidden] token order (written)
 * Pointers 16-byte aligned. */
int vsa_out_projection_tiled(const vsa_shape* shape, int hidden, const void* o_tiled,
                             const void* w_o, void* y, cudaStream_t stream);

/* Bytes of device workspace vsa_forward_host needs: two chunk buffers, each
 * holding heads_per_chunk (b, h) planes of the inputs, their tiled copies,
 * the final output and the coarse-stage scratch.  heads_per_chunk
 * 0 means 2; gated is 0 or 1.  Returns 0 for an invalid shape or k. */
size_t vsa_forward_host_workspace_bytes(const vsa_shape* shape, int topk, int heads_per_chunk,
                                        int gated);

/* The whole forward path (tile, coarse stage, fine stage, gated combine,
 * untile) from HOST buffers, for callers whose tensors live in host memory.
 * The pages give no such call; it composes the calls above.
 *   q, k, v   bf16 [B, H, N, d] in token order, HOST memory (read)
 *   g_fine, g_coarse float32 [B, H, N] HOST memory, or both NULL (ungated)
 *   out       bf16 [B, H, N, d] HOST memory (written)
 *   workspace DEVICE memory, 256-byte aligned, of at least
 *             vsa_forward_host_workspace_bytes(shape, topk, heads_per_chunk, gated)
 * The B*H planes are processed in chunks of heads_per_chunk (0: 2): while one
 * chunk computes on `stream`, the library copies the next chunk in and the
 * previous chunk's output out on two copy streams of its own (created once
 * per device), so both PCIe directions overlap the kernels.  Host buffers
 * should be page-locked (cudaHostAlloc / cudaHostRegister); pageable memory
 * works but its copies do not overlap.  The call returns once everything is
 * enqueued: `out` is complete when `stream` is (for example after
 * cudaStreamSynchronize(stream) or vsa_get_status(stream)), and earlier work
 * on `stream` finishes before the workspace is touched.  Argument errors are
 * reported before any copy; a failure after some chunks were enqueued
 * returns its code with those chunks still in flight. */
int vsa_forward_host(const vsa_shape* shape, int topk, const void* q, const void* k,
                     const void* v, const float* g_fine, const float* g_coarse, void* out,
                     void* workspace, size_t workspace_bytes, int heads_per_chunk,
                     cudaStream_t stream);

/* Transpose of a selection, for the key-stationary side of a backward pass:
 * for every key cube j of every (b, h), the query cubes i with j in
 * sel_idx[b, h, i, :], in ascending order, as a CSR list.  The pages have no
 * counterpart (they describe no backward kernel); it is a building block.
 *   sel_idx      int32 [B, H, C, k], rows without repeats, in any order (for
 *                example as vsa_coarse_select writes them); an index outside
 *                [0, C) is recorded as VSA_ERR_BAD_INDEX and left out
 *   key_offsets  int32 [B, H, C + 1] (written): key cube j's list is
 *                query_lists[b, h, key_offsets[b, h, j] .. key_offsets[b, h, j + 1])
 *   query_lists  int32 [B, H, C * k] (written)
 *   workspace    device scratch of at least B*H*C*k*4 bytes, 256-byte aligned */
int vsa_select_transpose(const vsa_shape* shape, const int32_t* sel_idx, int topk,
                         int32_t* key_offsets, int32_t* query_lists, void* workspace,
                         size_t workspace_bytes, cudaStream_t stream);

/* First pass of a backward: the gradient of the gated combine, in the layouts
 * the attention backward reads, in one pass over dout (selection held fixed;
 * the pages describe no backward, this follows from differentiating the
 * forward).  With out = g_f O_f + g_c O_c[cube] (or out = O_f ungated):
 *   do_fine_tiled bf16 [B, H, 64*C, d] (written): bf16(g_f * dout), tiled, pad rows 0
 *   delta         float32 [B, H, 64*C] (written): sum over d of do_fine * O_f, pad rows 0
 *   do_coarse     float32 [B, H, C, d] (written, gated only): sum over the cube's
 *                 valid tokens of g_c * dout
 *   dg_fine, dg_coarse float32 [B, H, N] (written, gated only): <dout, O_f>, <dout, O_c[cube]>
 * Inputs: dout bf16 [B, H, N, d] token order; o_fine_tiled bf16 [B, H, 64*C, d]
 * (the forward's O_f); o_coarse float32 [B, H, C, d] and the gates as in
 * vsa_combine, all three NULL when ungated. */
int vsa_backward_prep(const vsa_shape* shape, const void* dout, const void* o_fine_tiled,
                      const float* o_coarse, const float* g_fine, const float* g_coarse,
                      void* do_fine_tiled, float* delta, float* do_coarse, float* dg_fine,
                      float* dg_coarse, cudaStream_t stream);

/* Bytes of workspace vsa_coarse_backward needs to process all B*H planes in
 * one pass: B*H * 2*C*ldc*4, ldc = C rounded up to a multiple of 64 (two C x C
 * float32 matrices per plane).  0 for an invalid shape. */
size_t vsa_coarse_backward_workspace_bytes(const vsa_shape* shape);

/* Backward of the coarse attention O_c = softmax(qbar kbar^T / sqrt(d)) vbar
 * (the coarse stage of vsa_coarse_select; the pages describe no backward, this
 * differentiates that forward exactly, in float32):
 *   pooled    float32 [3, B, H, C, d]: qbar, kbar, vbar, the layout
 *             vsa_tile_permute_pool / vsa_coarse_select leave at the start of
 *             their workspace (read)
 *   o_coarse  float32 [B, H, C, d]: the forward's O_c (read)
 *   do_coarse float32 [B, H, C, d]: gradient of O_c, e.g. from vsa_backward_prep (read)
 *   d_pooled  float32 [3, B, H, C, d]: dqbar, dkbar, dvbar (written)
 *   workspace device scratch, 256-byte aligned, holding P and dS of as many
 *             planes as fit: at least one plane's share of
 *             vsa_coarse_backward_workspace_bytes (2*C*ldc*4 bytes); with less
 *             than the full size the planes are processed in chunks
 * All float pointers 16-byte aligned; B*H at most 65535. */
int vsa_coarse_backward(const vsa_shape* shape, const float* pooled, const float* o_coarse,
                        const float* do_coarse, float* d_pooled, void* workspace,
                        size_t workspace_bytes, cudaStream_t stream);

/* Backward of the fine block-sparse attention with the selection held fixed
 * (the pages describe no backward; this differentiates vsa_block_sparse_fwd
 * exactly), plus the last steps of the whole backward: the gradient of the
 * cube means reaches every valid token of its cube, and dq, dk, dv are
 * written in token order.  With scale = 1/sqrt(d), per query cube i and
 * selected key cube j: P = exp(scale Q_i K_j^T - lse_i) (0 on pad rows and
 * keys), dS = P (dO_i V_j^T - delta_i), dQ_i += scale dS K_j,
 * dK_j += scale dS^T Q_i, dV_j += P^T dO_i; then for a valid row r of cube c
 * dq[token(r)] = dQ[r] + dqbar[c] / n_c (k and v alike).
 *   q/k/v_tiled   bf16 [B, H, 64*C, d], the forward's tiled inputs
 *   sel_idx       int32 [B, H, C, k], the forward's selection
 *   key_offsets, query_lists  the selection's transpose (vsa_select_transpose)
 *   lse           float32 [B, H, 64*C] from vsa_block_sparse_fwd
 *   do_fine_tiled, delta  from vsa_backward_prep
 *   d_pooled      float32 [3, B, H, C, d] from vsa_coarse_backward, or NULL
 *                 (ungated: the coarse output does not reach the result)
 *   dq, dk, dv    bf16 [B, H, N, d] token order (written, every token)
 * The products run on the tensor cores (tcgen05, bf16 operands, float32
 * accumulation): P and dS are rounded to bf16 before they enter the dV, dQ
 * and dK products, as in a bf16 training step.  No atomics: a query cube's
 * dq is accumulated over its key cubes by one CTA, a key cube's dk, dv over
 * the query cubes that selected it by one CTA, so the result is
 * deterministic.  An index outside [0, C) in sel_idx or query_lists is
 * recorded as VSA_ERR_BAD_INDEX and clamped into range; key_offsets that do
 * not describe a list inside the CSR array are recorded the same way and the
 * key cube is treated as selected by no query cube.  The tiled tensors, lse,
 * delta, d_pooled and dq, dk, dv 16-byte aligned; on a wait that exceeds its
 * bound the kernels record VSA_ERR_TIMEOUT and stop. */
int vsa_block_sparse_bwd(const vsa_shape* shape, const void* q_tiled, const void* k_tiled,
                         const void* v_tiled, const int32_t* sel_idx, int topk,
                         const int32_t* key_offsets, const int32_t* query_lists, const float* lse,
                         const void* do_fine_tiled, const float* delta, const float* d_pooled,
                         void* dq, void* dk, void* dv, cudaStream_t stream);

/* Synchronises `stream`, then returns and clears the status word of the
 * current device: VSA_OK, VSA_ERR_TIMEOUT or VSA_ERR_BAD_INDEX recorded by a
 * kernel since the last call, or VSA_ERR_CUDA if the synchronisation failed. */
int vsa_get_status(cudaStream_t stream);

/* Diagnostic: launches one kernel that waits on a barrier nothing arrives at,
 * for at most timeout_ns nanoseconds (1e3 .. 1e9), with the same bounded wait
 * the fine kernel uses; it then records VSA_ERR_TIMEOUT in the status word and
 * returns, leaving the context usable.  Used by the tests to exercise the
 * timeout path without faulting the GPU. */
int vsa_debug_wait_timeout(uint64_t timeout_ns, cudaStream_t stream);

/* Static text for a status code. */
const char* vsa_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* VSA_H_ */
