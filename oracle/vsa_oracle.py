"""Float64 NumPy oracle for the video sparse attention (VSA) forward path.

TEST INFRASTRUCTURE ONLY: imported by the tests, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the CUDA library.

Sources (web pages on FastWan / VSA; cited by title and section):
  [news]   FastWan news article "单块 H200 ... 5 秒即生一个 5 秒视频",
           section "一张卡，秒生视频": the 410M-parameter scaling DiT on a
           (16, 32, 32) latent, 87.5 % sparsity with 8x fewer attention
           FLOPs, the fine block-sparse kernel, the coarse stage and the
           64x64 block size (FlexAttention comparison paragraph), Fig. 5
           (the block-sparse attention chosen by the coarse stage is dynamic).
  [news-2] same article, section "传统零散郑重力，为何会在蒸馏中失效？":
           VSA identifies the key tokens of the sequence dynamically and is a
           trainable drop-in replacement for FlashAttention.
  [neican] "超越Sora：FastWan如何以“稀疏蒸馏”重塑实时AI视频生成范式",
           section "技术原理与创新点解析": restates the above.
  [turbo]  TurboDiffusion review, section "評估 / 設置": a top-k *ratio*
           of 0.1 corresponds to 90 % attention sparsity.

The pages name the stages but print no formula.  This module takes the
plainest reading of each stage that the pages support:

  1. tile      The (T, H, W) latent token grid is cut into 4x4x4 cubes
               (64 tokens = one 64-row block of the 64x64 block mask
               [news]).  Cubes are ordered row-major over (t, y, x) cube
               coordinates; inside a cube the in-grid tokens are listed
               row-major over the local (t, y, x) offsets and packed to the
               front of the cube's 64 slots.  Edge cubes of a grid whose
               sides are not multiples of 4 are partial: they hold n_c < 64
               tokens and their remaining slots are zero padding.
  2. pool      Coarse stage [news]: each cube is summarised by the mean of
               its n_c valid tokens, separately for q, k and v.
  3. coarse    Attention over the C pooled vectors, scaled by 1/sqrt(d):
               S_c = qbar kbar^T / sqrt(d), P_c = softmax_row(S_c),
               O_c = P_c vbar.  Blocks are not weighted by n_c.
  4. top-k     For each query cube, the k key cubes with the largest coarse
               logits S_c (not the probabilities), ties to the lower index,
               returned in ascending index order [news-2: dynamic selection
               of key tokens].  k may come from a ratio r of the C cubes as
               max(1, floor(r C + 0.5)) [turbo].
  5. fine      Exact softmax attention of each valid query token of cube i
               over the valid key tokens of its k selected cubes, scaled by
               1/sqrt(d) [news: fine block-sparse kernel over 64x64 blocks].
               Pad query slots produce zero rows.  The log-sum-exp of each
               valid row's scaled scores is returned as well.
  6. combine   Optional per-token gated sum out = g_f * O_f + g_c * O_c[cube]
               with two gate tensors in token order; without gates out = O_f.
  7. untile    Inverse of step 1; pad slots are dropped.

Every floating-point step is float64.  bf16 inputs are widened exactly.

Parity status: every function below is pinned by tests that do not re-type
its formula (brute-force enumeration, a loop-only restatement, closed forms,
and library routines for dense attention and logsumexp).  None is "parity
unpinned"; the end-to-end numbers of the pages are not reproducible from the
pages (they print no worked example), so only the FLOP accounting (8x fewer
attention FLOPs at 87.5 % sparsity [news]) is pinned against them.
"""

from __future__ import annotations

import math

import numpy as np

CUBE = (4, 4, 4)
SLOTS = CUBE[0] * CUBE[1] * CUBE[2]


# ----------------------------------------------------------------------------
# dtype helpers
# ----------------------------------------------------------------------------

def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) exactly to float64."""
    u32 = bits.astype(np.uint32) << np.uint32(16)
    return u32.view(np.float32).astype(np.float64)


# ----------------------------------------------------------------------------
# 1. tile permutation  (step "tile" in the module header)
# ----------------------------------------------------------------------------

def cube_grid(grid, cube=CUBE):
    """Number of cubes along (t, y, x): ceil(side / cube side)."""
    return tuple(-(-g // c) for g, c in zip(grid, cube))


def cube_permutation(grid, cube=CUBE):
    """Token index held by every cube slot, and the valid-token count per cube.

    Returns ``(slot_token, counts)``: ``slot_token`` is int64 [C, 64] with the
    flat token index n = (t*H + y)*W + x of each slot, or -1 for a pad slot;
    ``counts`` is int64 [C].  Cube c = (ct*Cy + cy)*Cx + cx.
    """
    T, H, W = grid
    ct_, cy_, cx_ = cube
    Ct, Cy, Cx = cube_grid(grid, cube)
    C = Ct * Cy * Cx
    slots = ct_ * cy_ * cx_
    slot_token = np.full((C, slots), -1, dtype=np.int64)
    counts = np.zeros(C, dtype=np.int64)
    c = 0
    for a in range(Ct):
        for b in range(Cy):
            for e in range(Cx):
                s = 0
                for lt in range(ct_):
                    for ly in range(cy_):
                        for lx in range(cx_):
                            t, y, x = a * ct_ + lt, b * cy_ + ly, e * cx_ + lx
                            if t < T and y < H and x < W:
                                slot_token[c, s] = (t * H + y) * W + x
                                s += 1
                counts[c] = s
                c += 1
    return slot_token, counts


def tile_permute(x: np.ndarray, grid, cube=CUBE):
    """[B, Hh, N, d] token order -> [B, Hh, 64*C, d] cube order, zero pad."""
    slot_token, counts = cube_permutation(grid, cube)
    C, S = slot_token.shape
    B, Hh, N, d = x.shape
    assert N == grid[0] * grid[1] * grid[2]
    out = np.zeros((B, Hh, C * S, d), dtype=x.dtype)
    flat = slot_token.reshape(-1)
    valid = flat >= 0
    out[:, :, valid, :] = x[:, :, flat[valid], :]
    return out, counts


def untile(xt: np.ndarray, grid, cube=CUBE):
    """Inverse of :func:`tile_permute`: [B, Hh, 64*C, d] -> [B, Hh, N, d]."""
    slot_token, _ = cube_permutation(grid, cube)
    B, Hh, _, d = xt.shape
    N = grid[0] * grid[1] * grid[2]
    out = np.zeros((B, Hh, N, d), dtype=xt.dtype)
    flat = slot_token.reshape(-1)
    valid = flat >= 0
    out[:, :, flat[valid], :] = xt[:, :, valid, :]
    return out


# ----------------------------------------------------------------------------
# 2. pooling  (coarse stage, [news])
# ----------------------------------------------------------------------------

def pool(xt: np.ndarray, counts: np.ndarray) -> np.ndarray:
    """Mean of the valid tokens of every cube: [B, Hh, 64*C, d] -> [B, Hh, C, d]."""
    B, Hh, R, d = xt.shape
    C = counts.shape[0]
    S = R // C
    out = np.zeros((B, Hh, C, d), dtype=np.float64)
    for c in range(C):
        n = int(counts[c])
        out[:, :, c, :] = xt[:, :, c * S:c * S + n, :].sum(axis=2) / n
    return out


# ----------------------------------------------------------------------------
# 3. coarse attention  ([news], Fig. 5 paragraph)
# ----------------------------------------------------------------------------

def coarse_attention(qb: np.ndarray, kb: np.ndarray, vb: np.ndarray):
    """Attention over pooled cubes.  Returns (S_c logits, O_c output).

    S_c = qbar kbar^T / sqrt(d); O_c = softmax_row(S_c) vbar.
    """
    d = qb.shape[-1]
    S = np.matmul(qb, np.swapaxes(kb, -1, -2)) / math.sqrt(d)
    m = S.max(axis=-1, keepdims=True)
    e = np.exp(S - m)
    P = e / e.sum(axis=-1, keepdims=True)
    O = np.matmul(P, vb)
    return S, O


# ----------------------------------------------------------------------------
# 4. top-k selection  ([news-2]: dynamic identification of key tokens)
# ----------------------------------------------------------------------------

def topk_from_ratio(C: int, ratio: float) -> int:
    """k = max(1, floor(ratio * C + 0.5)) ([turbo]: top-k ratio 0.1 = 90 %)."""
    return max(1, int(math.floor(ratio * C + 0.5)))


def topk_select(S: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest entries of every row of S.

    Ties go to the lower index; each row's indices are returned ascending.
    """
    C = S.shape[-1]
    flat = S.reshape(-1, C)
    out = np.empty((flat.shape[0], k), dtype=np.int64)
    for r in range(flat.shape[0]):
        order = np.argsort(-flat[r], kind="stable")  # equal scores keep index order
        out[r] = np.sort(order[:k])
    return out.reshape(S.shape[:-1] + (k,))


# ----------------------------------------------------------------------------
# 5. fine block-sparse attention  ([news]: fine kernel, 64x64 blocks)
# ----------------------------------------------------------------------------

def block_sparse_attention(qt, kt, vt, counts, sel, query_cubes=None, heads=None):
    """Exact attention of each query cube over its selected key cubes.

    qt, kt, vt : [B, Hh, 64*C, d] tiled tensors (float64).
    sel        : [B, Hh, C, k] selected key-cube indices.
    query_cubes: optional iterable of query cube indices to evaluate
                 (others are left as zero); default all.
    heads      : optional iterable of (b, h) pairs; default all.
    Returns (O_f [B, Hh, 64*C, d], lse [B, Hh, 64*C]); pad query rows and
    unevaluated rows are 0 (lse: -inf).
    """
    B, Hh, R, d = qt.shape
    C = counts.shape[0]
    S = R // C
    scale = 1.0 / math.sqrt(d)
    out = np.zeros((B, Hh, R, d), dtype=np.float64)
    lse = np.full((B, Hh, R), -np.inf, dtype=np.float64)
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(Hh)]
    cubes = range(C) if query_cubes is None else query_cubes
    for b, h in heads:
        for i in cubes:
            ni = int(counts[i])
            rows = slice(i * S, i * S + ni)
            keys = np.concatenate([np.arange(j * S, j * S + int(counts[j]))
                                   for j in sel[b, h, i]])
            Q = qt[b, h, rows]
            K = kt[b, h, keys]
            V = vt[b, h, keys]
            logits = (Q @ K.T) * scale
            m = logits.max(axis=1, keepdims=True)
            e = np.exp(logits - m)
            z = e.sum(axis=1, keepdims=True)
            out[b, h, rows] = (e / z) @ V
            lse[b, h, rows] = (m + np.log(z))[:, 0]
    return out, lse


# ----------------------------------------------------------------------------
# 6. gated combine
# ----------------------------------------------------------------------------

def combine(of_t, oc, counts, grid, g_f=None, g_c=None, cube=CUBE):
    """out = g_f * O_f + g_c * O_c[cube of the slot] in tiled order.

    g_f, g_c are [B, Hh, N] in token order; with both None, out = O_f.
    Pad slots are 0.
    """
    if g_f is None and g_c is None:
        return of_t.copy()
    slot_token, _ = cube_permutation(grid, cube)
    C, S = slot_token.shape
    out = np.zeros_like(of_t)
    for c in range(C):
        for s in range(int(counts[c])):
            n = slot_token[c, s]
            r = c * S + s
            out[:, :, r, :] = (g_f[:, :, n, None] * of_t[:, :, r, :]
                               + g_c[:, :, n, None] * oc[:, :, c, :])
    return out


# ----------------------------------------------------------------------------
# whole forward path
# ----------------------------------------------------------------------------

def vsa_forward(q, k, v, grid, topk, g_f=None, g_c=None, cube=CUBE):
    """The whole VSA forward path on float64 arrays [B, Hh, N, d].

    Returns a dict with every intermediate: counts, q_t, k_t, v_t, qbar,
    kbar, vbar, S_c, O_c, sel, O_f (tiled), lse, out_t (tiled), out.
    """
    q_t, counts = tile_permute(q, grid, cube)
    k_t, _ = tile_permute(k, grid, cube)
    v_t, _ = tile_permute(v, grid, cube)
    qb, kb, vb = pool(q_t, counts), pool(k_t, counts), pool(v_t, counts)
    S_c, O_c = coarse_attention(qb, kb, vb)
    sel = topk_select(S_c, topk)
    O_f, lse = block_sparse_attention(q_t, k_t, v_t, counts, sel)
    out_t = combine(O_f, O_c, counts, grid, g_f, g_c, cube)
    out = untile(out_t, grid, cube)
    return dict(counts=counts, q_t=q_t, k_t=k_t, v_t=v_t, qbar=qb, kbar=kb,
                vbar=vb, S_c=S_c, O_c=O_c, sel=sel, O_f=O_f, lse=lse,
                out_t=out_t, out=out)
