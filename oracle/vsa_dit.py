"""Float64 NumPy oracle for the projections around VSA in a DiT attention
block: the QKV projection before the attention and the output projection
after it.

TEST INFRASTRUCTURE ONLY: imported by the tests, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the CUDA library.

Sources (web pages, cited by title and section):
  [news]  FastWan news article "单块 H200 ... 5 秒即生一个 5 秒视频", section
          "一张卡，秒生视频": the end-to-end Wan-1.3B / HunyuanVideo figures
          come from whole DiT blocks, where VSA replaces the attention between
          the QKV projection and the output projection.

The page prints no formula for the block.  The plainest reading, taken here:

  qkv   y = x W_qkv^T (the linear-layer convention, W [out, in]; no bias, the
        page names none), x [B, N, hidden] in token order; the 3 H d output
        features are q heads 0..H-1, then k heads, then v heads, head h of q
        being features h d .. h d + d - 1.
  out   y = o W_o^T with o the attention output [B, H, N, d] concatenated
        over heads in head order (feature h d + e = head h, feature e),
        W_o [hidden, H d].
  block out(vsa_forward(qkv(x))) with the VSA forward of ``vsa_oracle``.

Every step is float64; a matrix product is the library primitive
(``numpy.matmul``), used as one step with no blocking or reordering.

Parity status: pinned by tests that do not re-type the formula: a loop-only
restatement on tiny sizes, identity and scaled-identity weights (the
projection then only splits or concatenates heads), the round trip of the two
projections with identity weights, and linearity in the weights.
"""

from __future__ import annotations

import numpy as np

from . import vsa_oracle as vo


def qkv_projection(x: np.ndarray, w_qkv: np.ndarray, heads: int, head_dim: int):
    """x [B, N, hidden], w_qkv [3 H d, hidden] -> (q, k, v), each [B, H, N, d]."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w_qkv, dtype=np.float64)
    B, N, _ = x.shape
    y = np.matmul(x, w.T)                                    # [B, N, 3 H d]
    y = y.reshape(B, N, 3, heads, head_dim).transpose(2, 0, 3, 1, 4)
    return y[0], y[1], y[2]


def out_projection(o: np.ndarray, w_o: np.ndarray) -> np.ndarray:
    """o [B, H, N, d], w_o [hidden, H d] -> [B, N, hidden]."""
    o = np.asarray(o, dtype=np.float64)
    B, H, N, d = o.shape
    cat = o.transpose(0, 2, 1, 3).reshape(B, N, H * d)      # heads concatenated
    return np.matmul(cat, np.asarray(w_o, dtype=np.float64).T)


def attention_block(x, w_qkv, w_o, heads, head_dim, grid, topk, g_f=None, g_c=None):
    """QKV projection, VSA forward, output projection.  Returns the VSA
    forward's dict with q, k, v and y (the block output [B, N, hidden])."""
    q, k, v = qkv_projection(x, w_qkv, heads, head_dim)
    ref = vo.vsa_forward(q, k, v, grid, topk, g_f, g_c)
    ref.update(q=q, k=k, v=v, y=out_projection(ref["out"], w_o))
    return ref
