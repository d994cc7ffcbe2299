"""Float64 NumPy oracle for the low-rank linear compensation branch summed with
the block-sparse output (the sparse + linear variant of VSA).

TEST INFRASTRUCTURE ONLY: imported by the tests, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the CUDA library.

Sources (web pages, cited by title and section):
  [spark]  dgnews.ru page on SparkDiffusion (Peking University, Tsinghua,
           Alibaba), third paragraph: at 97 % attention sparsity the model is
           adapted with RoLA, an attention module that pairs a block-sparse
           branch with a low-rank linear branch which keeps the global
           context.
  [turbo]  TurboDiffusion review, sections "注意力加速" and the technical
           overview: trainable sparse-linear attention (SLA) combines sparse
           attention with linear attention.

Neither page prints a formula.  The plainest reading both support, taken
here:

  linear   A linear-attention branch over every valid token of the (b, h)
           sequence (global context):
               O_lin[r] = phi(q_r)^T KV / (phi(q_r)^T z),
               KV = sum_t phi(k_t) v_t^T,   z = sum_t phi(k_t),
           with the positive feature map phi(x) = elu(x) + 1 applied
           elementwise (x + 1 for x > 0, exp(x) otherwise), so every weight
           phi(q_r) . phi(k_t) is positive and the denominator never vanishes.
           The rank of the branch's N x N attention matrix is at most d: the
           low-rank part.  No scale is applied inside phi.
  sum      out = O_block_sparse + O_lin, the block-sparse branch being the
           whole VSA forward (fine stage, with the gated combine when gates
           are given).  The pages name no weight for either branch.

Every floating-point step is float64; bf16 inputs are widened exactly.

Parity status: pinned by tests that do not re-type the formula: the dense
N x N form of the same attention (phi(Q) phi(K)^T normalised by rows, times
V), closed forms (equal keys give the mean of the values, v = 1 gives 1),
invariance under a permutation of the tokens, and a loop-only restatement on
a tiny grid.
"""

from __future__ import annotations

import numpy as np

from . import vsa_oracle as vo


def feature_map(x: np.ndarray) -> np.ndarray:
    """phi(x) = elu(x) + 1: x + 1 for x > 0, exp(x) for x <= 0 (float64)."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(x > 0.0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def linear_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """Linear attention of every token over all tokens of its (b, h) sequence.

    q, k, v: [..., N, d] in token order (every token valid).  Returns
    [..., N, d]: phi(q_r)^T KV / phi(q_r)^T z with KV = sum_t phi(k_t) v_t^T and
    z = sum_t phi(k_t) [spark: low-rank linear branch for global context]."""
    fq, fk = feature_map(q), feature_map(k)
    v = np.asarray(v, dtype=np.float64)
    kv = np.einsum("...td,...te->...de", fk, v)   # [..., d, d]
    z = fk.sum(axis=-2)                            # [..., d]
    num = np.einsum("...rd,...de->...re", fq, kv)
    den = np.einsum("...rd,...d->...r", fq, z)
    return num / den[..., None]


def sparse_linear_forward(q, k, v, grid, topk, g_f=None, g_c=None):
    """The block-sparse VSA forward plus the linear branch, token order.

    Returns the VSA forward's dict with two more entries: "lin" (the linear
    branch [B, H, N, d]) and "out_sparse_linear" = out + lin [spark, turbo]."""
    ref = vo.vsa_forward(q, k, v, grid, topk, g_f, g_c)
    lin = linear_attention(q, k, v)
    ref["lin"] = lin
    ref["out_sparse_linear"] = ref["out"] + lin
    return ref
