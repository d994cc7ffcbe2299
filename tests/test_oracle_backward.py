"""Pins of the float64 VSA backward (oracle/vsa_backward.py), all on the CPU.

The backward is checked against three things it does not share code with:
torch autograd of a dense, masked, token-order forward written here from the
definitions; central finite differences of <dout, out> through the oracle's
forward; and, with every cube selected and the coarse branch gated off, the
backward of torch's dense scaled-dot-product attention."""

import math

import numpy as np
import pytest
import torch

from oracle import vsa_backward as vb
from oracle import vsa_oracle as vo

GRIDS = [(4, 8, 8), (5, 6, 7), (3, 5, 9)]


def cube_of_tokens(grid):
    """Cube index of every token n = (t*Y + y)*X + x, from the 4x4x4 tiling."""
    T, Y, X = grid
    Cy, Cx = -(-Y // 4), -(-X // 4)
    t, y, x = np.meshgrid(np.arange(T), np.arange(Y), np.arange(X), indexing="ij")
    return (((t // 4) * Cy + y // 4) * Cx + x // 4).reshape(-1)


def dense_forward(q, k, v, grid, sel, g_f, g_c):
    """out in token order, written as dense masked attention plus a pooling matrix."""
    cube = torch.from_numpy(cube_of_tokens(grid))
    C = int(cube.max()) + 1
    B, H, N, d = q.shape
    scale = 1.0 / math.sqrt(d)
    # allowed[b, h, query token, key token]: the key's cube is selected by the query's cube
    chosen = torch.zeros(B, H, C, C, dtype=torch.bool)
    chosen.scatter_(3, torch.from_numpy(sel), True)
    allowed = chosen[:, :, cube][:, :, :, cube]
    logits = (q @ k.transpose(-1, -2)) * scale
    o_f = torch.softmax(logits.masked_fill(~allowed, float("-inf")), dim=-1) @ v
    member = (cube[None, :] == torch.arange(C)[:, None]).double()
    pool_mat = member / member.sum(dim=1, keepdim=True)          # [C, N]: mean over a cube
    qb, kb, vbar = pool_mat @ q, pool_mat @ k, pool_mat @ v
    o_c = torch.softmax((qb @ kb.transpose(-1, -2)) * scale, dim=-1) @ vbar
    if g_f is None:
        return o_f
    return g_f[..., None] * o_f + g_c[..., None] * o_c[:, :, cube]


def inputs(grid, B=2, H=2, d=8, seed=0, gated=True):
    rng = np.random.default_rng(seed)
    N = math.prod(grid)
    q, k, v, dout = (rng.standard_normal((B, H, N, d)) for _ in range(4))
    g_f = rng.random((B, H, N)) if gated else None
    g_c = rng.random((B, H, N)) if gated else None
    return q, k, v, dout, g_f, g_c


@pytest.mark.parametrize("grid", GRIDS)
@pytest.mark.parametrize("gated", [True, False])
def test_backward_equals_autograd_of_dense_masked_forward(grid, gated):
    q, k, v, dout, g_f, g_c = inputs(grid, gated=gated)
    C = math.prod(-(-s // 4) for s in grid)
    topk = max(1, C // 3)
    got = vb.vsa_backward(q, k, v, grid, topk, dout, g_f, g_c)
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    tgf = torch.tensor(g_f, requires_grad=True) if gated else None
    tgc = torch.tensor(g_c, requires_grad=True) if gated else None
    out = dense_forward(tq, tk, tv, grid, got["sel"], tgf, tgc)
    (out * torch.from_numpy(dout)).sum().backward()
    for name, t in (("dq", tq), ("dk", tk), ("dv", tv)):
        np.testing.assert_allclose(got[name], t.grad.numpy(), rtol=0, atol=1e-10, err_msg=name)
    if gated:
        np.testing.assert_allclose(got["dg_f"], tgf.grad.numpy(), rtol=0, atol=1e-10)
        np.testing.assert_allclose(got["dg_c"], tgc.grad.numpy(), rtol=0, atol=1e-10)
    else:
        assert got["dg_f"] is None and got["dg_c"] is None


def test_backward_matches_finite_differences():
    grid = (5, 6, 7)
    q, k, v, dout, g_f, g_c = inputs(grid, B=1, H=1, d=4, seed=3)
    topk = 3
    got = vb.vsa_backward(q, k, v, grid, topk, dout, g_f, g_c)
    args = dict(q=q, k=k, v=v, g_f=g_f, g_c=g_c)

    def loss(a):
        fw = vo.vsa_forward(a["q"], a["k"], a["v"], grid, topk, a["g_f"], a["g_c"])
        return float(np.sum(fw["out"] * dout)), fw["sel"]

    rng = np.random.default_rng(11)
    eps = 1e-6
    grads = dict(q=got["dq"], k=got["dk"], v=got["dv"], g_f=got["dg_f"], g_c=got["dg_c"])
    for name in args:
        u = rng.standard_normal(args[name].shape)
        plus = dict(args, **{name: args[name] + eps * u})
        minus = dict(args, **{name: args[name] - eps * u})
        lp, sp = loss(plus)
        lm, sm = loss(minus)
        assert np.array_equal(sp, got["sel"]) and np.array_equal(sm, got["sel"])  # selection held
        fd = (lp - lm) / (2 * eps)
        an = float(np.sum(grads[name] * u))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


@pytest.mark.parametrize("grid", [(4, 8, 8), (5, 6, 7)])
def test_all_cubes_selected_and_coarse_off_is_dense_attention_backward(grid):
    q, k, v, dout, _, _ = inputs(grid, seed=5, gated=False)
    C = math.prod(-(-s // 4) for s in grid)
    B, H, N, d = q.shape
    ones, zeros = np.ones((B, H, N)), np.zeros((B, H, N))
    got = vb.vsa_backward(q, k, v, grid, C, dout, ones, zeros)
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)
    (out * torch.from_numpy(dout)).sum().backward()
    for name, t in (("dq", tq), ("dk", tk), ("dv", tv)):
        np.testing.assert_allclose(got[name], t.grad.numpy(), rtol=0, atol=1e-10, err_msg=name)
    # dg_f = <dout, O_f> with O_f the dense attention output
    np.testing.assert_allclose(got["dg_f"], np.sum(dout * out.detach().numpy(), axis=-1),
                               rtol=0, atol=1e-10)


def test_pool_backward_spreads_the_mean_gradient_over_valid_rows():
    grid = (5, 6, 7)
    counts = vo.cube_permutation(grid)[1]
    C = counts.shape[0]
    rng = np.random.default_rng(2)
    dxb = rng.standard_normal((1, 1, C, 3))
    dx = vb.pool_backward(dxb, counts)
    for c in range(C):
        n = int(counts[c])
        block = dx[0, 0, 64 * c:64 * (c + 1)]
        np.testing.assert_allclose(block[:n].sum(axis=0), dxb[0, 0, c], atol=1e-12)
        assert np.all(block[n:] == 0)


def test_backward_from_saved_lse_equals_recomputed_softmax():
    # the recipe a kernel with the forward's LSE follows gives the same gradients
    grid = (5, 6, 7)
    q, k, v, dout, _, _ = inputs(grid, B=1, H=1, d=8, seed=7, gated=False)
    q_t, counts = vo.tile_permute(q, grid)
    k_t, _ = vo.tile_permute(k, grid)
    v_t, _ = vo.tile_permute(v, grid)
    do_t, _ = vo.tile_permute(dout, grid)
    C = counts.shape[0]
    sel = np.stack([np.arange(C)[::2][:3]] * C).reshape(1, 1, C, 3)
    O, lse = vo.block_sparse_attention(q_t, k_t, v_t, counts, sel)
    scale = 1.0 / math.sqrt(q.shape[-1])
    for i in range(C):
        rows = slice(64 * i, 64 * i + int(counts[i]))
        keys = np.concatenate([np.arange(64 * j, 64 * j + int(counts[j])) for j in sel[0, 0, i]])
        a = vb.attention_backward(q_t[0, 0, rows], k_t[0, 0, keys], v_t[0, 0, keys], do_t[0, 0, rows], scale)
        b = vb.attention_backward_from_lse(q_t[0, 0, rows], k_t[0, 0, keys], v_t[0, 0, keys],
                                           O[0, 0, rows], do_t[0, 0, rows], lse[0, 0, rows], scale)
        for x, y in zip(a, b):
            np.testing.assert_allclose(x, y, rtol=0, atol=1e-12)


def test_select_transpose_is_the_inverse_incidence():
    rng = np.random.default_rng(4)
    C, k = 11, 4
    sel = np.stack([np.sort(rng.choice(C, k, replace=False)) for _ in range(2 * C)]).reshape(2, C, k)
    offs, qs = vb.select_transpose(sel, C)
    for p in range(2):
        assert offs[p, 0] == 0 and offs[p, -1] == C * k
        for j in range(C):
            got = qs[p, offs[p, j]:offs[p, j + 1]]
            want = [i for i in range(C) if j in sel[p, i]]  # brute force
            assert list(got) == want
