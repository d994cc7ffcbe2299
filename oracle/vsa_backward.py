"""Float64 backward of the VSA forward path: the gradients a training step needs.

TEST INFRASTRUCTURE ONLY: imported by the tests; never by the CUDA library,
and it shares no code with it.

Sources: the pages present VSA as trainable, a drop-in replacement for
FlashAttention in training ([news-2]: FastWan news article, section
"传统零散郑重力，为何会在蒸馏中失效？"); they print no backward pass.

Reading taken (the plainest one the forward supports):
  * The top-k selection is a discrete choice and passes no gradient: the
    selected key cubes are held fixed, as for any block-sparse mask.
  * Every other step is differentiated exactly, and the gradients of the
    fine and the coarse branch add:
      out[r]  = g_f[r] O_f[r] + g_c[r] O_c[cube(r)]
                -> dO_f[r] = g_f[r] dout[r]
                   dO_c[c] = sum over the valid rows r of cube c of g_c[r] dout[r]
                   dg_f[r] = <dout[r], O_f[r]>,  dg_c[r] = <dout[r], O_c[cube(r)]>
                   (no gates: out = O_f, so dO_f = dout and O_c receives nothing)
      O       = softmax(Q K^T / sqrt(d)) V  (fine: Q one query cube, K and V
                the valid rows of its selected cubes; coarse: the pooled
                vectors)
                -> P = softmax(.), D_r = <dO_r, O_r>,
                   dV = P^T dO,  dS = P * (dO V^T - D),
                   dQ = dS K / sqrt(d),  dK = dS^T Q / sqrt(d)
      xbar[c] = mean of the n_c valid rows of cube c
                -> every valid row of cube c receives dxbar[c] / n_c
      tile / untile are permutations (pad slots carry nothing), so a
      gradient goes back through them by the inverse permutation.

Parity status: pinned in tests/test_oracle_backward.py against torch
autograd of a differently written (dense, masked, token-order) forward,
against central finite differences, and, for k = C, against the backward of
torch's dense scaled-dot-product attention.
"""

from __future__ import annotations

import math

import numpy as np

from .vsa_oracle import (CUBE, block_sparse_attention, coarse_attention, cube_permutation,
                         pool, tile_permute, topk_select, untile)


def attention_backward(Q, K, V, dO, scale):
    """Gradients of O = softmax(Q K^T * scale) V for one dense block (float64)."""
    S = (Q @ K.T) * scale
    S = S - S.max(axis=1, keepdims=True)
    E = np.exp(S)
    P = E / E.sum(axis=1, keepdims=True)
    O = P @ V
    D = np.sum(dO * O, axis=1, keepdims=True)
    dV = P.T @ dO
    dS = P * (dO @ V.T - D)
    dQ = (dS @ K) * scale
    dK = (dS.T @ Q) * scale
    return dQ, dK, dV


def attention_backward_from_lse(Q, K, V, O, dO, lse, scale):
    """The same gradients written the way a kernel that saved the forward's
    natural-log log-sum-exp computes them: P = exp(S - lse), D = rowsum(dO * O),
    with O the forward output (no second softmax normalisation)."""
    P = np.exp((Q @ K.T) * scale - lse[:, None])
    D = np.sum(dO * O, axis=1, keepdims=True)
    dV = P.T @ dO
    dS = P * (dO @ V.T - D)
    return (dS @ K) * scale, (dS.T @ Q) * scale, dV


def select_transpose(sel, C):
    """For every key cube, the query cubes that selected it, ascending.

    sel: [..., C, k] selections (each row ascending, no repeats).  Returns
    (offsets [..., C + 1], queries [..., C * k]): the query cubes of key cube j
    are queries[..., offsets[j]:offsets[j + 1]].  The dK/dV side of a backward
    walks these lists.
    """
    lead = sel.shape[:-2]
    k = sel.shape[-1]
    flat = sel.reshape(-1, C, k)
    offs = np.zeros((flat.shape[0], C + 1), dtype=np.int64)
    qs = np.zeros((flat.shape[0], C * k), dtype=np.int64)
    for p in range(flat.shape[0]):
        lists = [[] for _ in range(C)]
        for i in range(C):  # ascending query cubes keep each list ascending
            for j in flat[p, i]:
                lists[int(j)].append(i)
        offs[p, 1:] = np.cumsum([len(l) for l in lists])
        qs[p] = np.concatenate([np.asarray(l, dtype=np.int64) for l in lists])
    return offs.reshape(lead + (C + 1,)), qs.reshape(lead + (C * k,))


def block_sparse_attention_backward(qt, kt, vt, counts, sel, dof_t):
    """Gradients of the fine stage w.r.t. the tiled q, k, v.

    qt, kt, vt, dof_t: [B, Hh, 64*C, d] float64; sel [B, Hh, C, k].
    Pad rows of the results are 0.
    """
    B, Hh, R, d = qt.shape
    C = counts.shape[0]
    S = R // C
    scale = 1.0 / math.sqrt(d)
    dq = np.zeros_like(qt)
    dk = np.zeros_like(kt)
    dv = np.zeros_like(vt)
    for b in range(B):
        for h in range(Hh):
            for i in range(C):
                ni = int(counts[i])
                rows = slice(i * S, i * S + ni)
                keys = np.concatenate([np.arange(j * S, j * S + int(counts[j]))
                                       for j in sel[b, h, i]])
                gq, gk, gv = attention_backward(qt[b, h, rows], kt[b, h, keys], vt[b, h, keys],
                                                dof_t[b, h, rows], scale)
                dq[b, h, rows] += gq
                np.add.at(dk[b, h], keys, gk)
                np.add.at(dv[b, h], keys, gv)
    return dq, dk, dv


def coarse_attention_backward(qb, kb, vb, doc):
    """Gradients of O_c = softmax(qbar kbar^T / sqrt(d)) vbar w.r.t. the pooled vectors."""
    B, Hh, C, d = qb.shape
    scale = 1.0 / math.sqrt(d)
    dqb = np.zeros_like(qb)
    dkb = np.zeros_like(kb)
    dvb = np.zeros_like(vb)
    for b in range(B):
        for h in range(Hh):
            dqb[b, h], dkb[b, h], dvb[b, h] = attention_backward(qb[b, h], kb[b, h], vb[b, h],
                                                                  doc[b, h], scale)
    return dqb, dkb, dvb


def pool_backward(dxb, counts, rows_per_cube=64):
    """Gradient of the cube means w.r.t. the tiled rows: dxbar[c] / n_c on each valid row."""
    B, Hh, C, d = dxb.shape
    dx = np.zeros((B, Hh, C * rows_per_cube, d), dtype=np.float64)
    for c in range(C):
        n = int(counts[c])
        dx[:, :, c * rows_per_cube:c * rows_per_cube + n, :] = dxb[:, :, c:c + 1, :] / n
    return dx


def combine_backward(dout_t, of_t, oc, counts, grid, g_f=None, g_c=None, cube=CUBE):
    """Gradients of the gated combine (tiled order in, gates in token order).

    Returns (dO_f tiled, dO_c [B, Hh, C, d], dg_f, dg_c [B, Hh, N] or None).
    """
    if g_f is None and g_c is None:
        return dout_t.copy(), np.zeros_like(oc), None, None
    slot_token, _ = cube_permutation(grid, cube)
    C, S = slot_token.shape
    B, Hh, N = g_f.shape
    dof = np.zeros_like(dout_t)
    doc = np.zeros_like(oc)
    dgf = np.zeros((B, Hh, N), dtype=np.float64)
    dgc = np.zeros((B, Hh, N), dtype=np.float64)
    for c in range(C):
        for s in range(int(counts[c])):
            n = slot_token[c, s]
            r = c * S + s
            g = dout_t[:, :, r, :]
            dof[:, :, r, :] = g_f[:, :, n, None] * g
            doc[:, :, c, :] += g_c[:, :, n, None] * g
            dgf[:, :, n] = np.sum(g * of_t[:, :, r, :], axis=-1)
            dgc[:, :, n] = np.sum(g * oc[:, :, c, :], axis=-1)
    return dof, doc, dgf, dgc


def vsa_backward(q, k, v, grid, topk, dout, g_f=None, g_c=None, cube=CUBE, sel=None):
    """Gradients of <dout, out> for the whole path on float64 arrays [B, Hh, N, d].

    Returns dict(dq, dk, dv [B, Hh, N, d], dg_f, dg_c [B, Hh, N] or None, sel,
    S_c) with the selection held at the forward's choice.  ``sel`` replaces
    that choice with another valid one (a top-k set of S_c up to ties); the
    arithmetic is the same.
    """
    q_t, counts = tile_permute(q, grid, cube)
    k_t, _ = tile_permute(k, grid, cube)
    v_t, _ = tile_permute(v, grid, cube)
    qb, kb, vb = pool(q_t, counts), pool(k_t, counts), pool(v_t, counts)
    S_c, O_c = coarse_attention(qb, kb, vb)
    if sel is None:
        sel = topk_select(S_c, topk)
    O_f, _ = block_sparse_attention(q_t, k_t, v_t, counts, sel)
    dout_t, _ = tile_permute(dout, grid, cube)
    dof, doc, dgf, dgc = combine_backward(dout_t, O_f, O_c, counts, grid, g_f, g_c, cube)
    dq_t, dk_t, dv_t = block_sparse_attention_backward(q_t, k_t, v_t, counts, sel, dof)
    dqb, dkb, dvb = coarse_attention_backward(qb, kb, vb, doc)
    S = q_t.shape[2] // counts.shape[0]
    dq_t += pool_backward(dqb, counts, S)
    dk_t += pool_backward(dkb, counts, S)
    dv_t += pool_backward(dvb, counts, S)
    return dict(dq=untile(dq_t, grid, cube), dk=untile(dk_t, grid, cube),
                dv=untile(dv_t, grid, cube), dg_f=dgf, dg_c=dgc, sel=sel, S_c=S_c)


__all__ = ["attention_backward", "attention_backward_from_lse", "select_transpose",
           "block_sparse_attention_backward", "coarse_attention_backward", "pool_backward",
           "combine_backward", "vsa_backward"]
