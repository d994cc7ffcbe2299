"""Pins for the CPU oracle, checked against things other than itself.

Each test ties one oracle stage to an independent fact: brute-force
enumeration, a loop-only restatement, a hand-derived fixture, a closed form,
or a library routine (torch's scaled_dot_product_attention / logsumexp in
float64 on the CPU).  A plausible slip in the oracle (a dropped 1/sqrt(d), a
wrong sign, a transposed operand, dividing a partial cube by 64, the wrong tie
direction) fails at least one of them.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import vsa_oracle as vo
from oracle.vsa_loops import _slot_of_token, vsa_forward_loops
from video_dit_block_vsa_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "cube_counts.json")

RAGGED_GRIDS = [(4, 8, 8), (5, 5, 5), (1, 1, 1), (3, 7, 9), (6, 4, 5), (2, 9, 4)]


def sdpa(q, k, v):
    """Dense softmax attention by the library routine (scale 1/sqrt(d))."""
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    return torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v)).numpy()


# --------------------------------------------------------------------------
# tile permutation
# --------------------------------------------------------------------------

@pytest.mark.parametrize("grid", RAGGED_GRIDS)
def test_permutation_matches_token_walk(grid):
    slot_token, counts = vo.cube_permutation(grid)
    slot, counts_loop, C = _slot_of_token(grid, (4, 4, 4))
    assert C == slot_token.shape[0]
    assert list(counts) == counts_loop
    for n, (c, r) in slot.items():
        assert slot_token[c, r] == n
    flat = slot_token.reshape(-1)
    valid = flat[flat >= 0]
    N = grid[0] * grid[1] * grid[2]
    assert sorted(valid.tolist()) == list(range(N))  # every token exactly once
    # valid slots are packed to the front of each cube
    for c in range(C):
        assert np.all(slot_token[c, :counts[c]] >= 0)
        assert np.all(slot_token[c, counts[c]:] == -1)


def test_cube_counts_golden():
    data = json.load(open(GOLDEN))
    for g in data["grids"]:
        grid = tuple(g["grid"])
        assert vo.cube_grid(grid) == tuple(g["cubes"])
        slot_token, counts = vo.cube_permutation(grid)
        assert counts.shape[0] == g["C"]
        assert int(counts.sum()) == g["N"]
        if "histogram" in g:
            vals, freq = np.unique(counts, return_counts=True)
            assert {str(a): int(b) for a, b in zip(vals, freq)} == g["histogram"]
        if "counts_in_cube_order" in g:
            assert counts.tolist() == g["counts_in_cube_order"]
            assert slot_token[1, :16].tolist() == g["cube1_tokens"]


@pytest.mark.parametrize("grid", RAGGED_GRIDS)
def test_tile_untile_roundtrip_and_zero_pad(grid):
    rng = np.random.default_rng(7)
    N = grid[0] * grid[1] * grid[2]
    x = rng.standard_normal((2, 3, N, 5))
    xt, counts = vo.tile_permute(x, grid)
    assert np.array_equal(vo.untile(xt, grid), x)
    for c in range(counts.shape[0]):
        assert np.all(xt[:, :, c * 64 + counts[c]:(c + 1) * 64] == 0)


# --------------------------------------------------------------------------
# pooling
# --------------------------------------------------------------------------

@pytest.mark.parametrize("grid", [(5, 5, 5), (3, 7, 9), (4, 8, 8)])
def test_pool_equals_brute_force_average(grid):
    rng = np.random.default_rng(1)
    N = grid[0] * grid[1] * grid[2]
    x = rng.standard_normal((1, 2, N, 4))
    xt, counts = vo.tile_permute(x, grid)
    got = vo.pool(xt, counts)
    slot, _, C = _slot_of_token(grid, (4, 4, 4))
    for c in range(C):
        toks = [n for n, (cc, _) in slot.items() if cc == c]
        for b in range(1):
            for h in range(2):
                acc = [0.0] * 4
                for n in toks:
                    for e in range(4):
                        acc[e] += x[b, h, n, e]
                want = [a / len(toks) for a in acc]
                assert np.allclose(got[b, h, c], want, rtol=0, atol=1e-12)


def test_pool_constant_cube_is_the_constant():
    grid = (5, 6, 7)
    N = 5 * 6 * 7
    x = np.full((1, 1, N, 3), 2.5)
    xt, counts = vo.tile_permute(x, grid)
    assert np.all(vo.pool(xt, counts) == 2.5)  # a /64 slip on partial cubes fails here


# --------------------------------------------------------------------------
# coarse attention and top-k
# --------------------------------------------------------------------------

def test_coarse_attention_equals_library_sdpa():
    rng = np.random.default_rng(2)
    qb, kb, vb = (rng.standard_normal((2, 3, 17, 16)) for _ in range(3))
    S, O = vo.coarse_attention(qb, kb, vb)
    assert np.allclose(O, sdpa(qb, kb, vb), rtol=0, atol=1e-12)
    # logits: closed form on aligned vectors, q = a e1, k_j = b_j e1
    d = 16
    q = np.zeros((1, 1, 1, d)); q[..., 0] = 3.0
    k = np.zeros((1, 1, 4, d)); k[0, 0, :, 0] = [1.0, -2.0, 0.5, 4.0]
    S2, _ = vo.coarse_attention(q, k, np.ones((1, 1, 4, d)))
    assert np.allclose(S2[0, 0, 0], np.array([3.0, -6.0, 1.5, 12.0]) / 4.0, atol=1e-15)


def test_coarse_uniform_keys_average_values():
    rng = np.random.default_rng(3)
    qb = rng.standard_normal((1, 1, 6, 8))
    kb = np.tile(rng.standard_normal((1, 1, 1, 8)), (1, 1, 6, 1))
    vb = rng.standard_normal((1, 1, 6, 8))
    _, O = vo.coarse_attention(qb, kb, vb)
    assert np.allclose(O, np.broadcast_to(vb.mean(axis=2, keepdims=True), O.shape), atol=1e-12)


def test_topk_brute_force_and_ties():
    rng = np.random.default_rng(4)
    S = rng.standard_normal((3, 2, 11, 11))
    S[0, 0, 0, [2, 5, 7]] = 9.0  # a three-way tie at the top
    for k in (1, 3, 5, 11):
        sel = vo.topk_select(S, k)
        for idx in np.ndindex(S.shape[:-1]):
            row = S[idx].tolist()
            want = sorted(sorted(range(11), key=lambda j: (-row[j], j))[:k])
            assert sel[idx].tolist() == want
    assert vo.topk_select(S, 2)[0, 0, 0].tolist() == [2, 5]  # ties to the lower index
    flat = np.zeros((1, 9))
    assert vo.topk_select(flat, 4)[0].tolist() == [0, 1, 2, 3]
    desc = -np.arange(9, dtype=float)[None]
    assert vo.topk_select(desc, 3)[0].tolist() == [0, 1, 2]
    assert vo.topk_select(-desc, 3)[0].tolist() == [6, 7, 8]


def test_topk_from_ratio_page_values():
    # top-k ratio 0.1 of the TurboDiffusion review; 0.125 = 87.5 % sparsity
    assert vo.topk_from_ratio(624, 0.1) == 62
    assert vo.topk_from_ratio(1440, 0.125) == 180
    assert vo.topk_from_ratio(1440, 0.03) == 43
    assert vo.topk_from_ratio(256, 0.125) == 32
    assert vo.topk_from_ratio(10, 0.01) == 1


# --------------------------------------------------------------------------
# fine block-sparse attention
# --------------------------------------------------------------------------

@pytest.mark.parametrize("grid", [(4, 8, 8), (5, 5, 5), (3, 7, 9)])
def test_fine_all_blocks_equals_dense_sdpa(grid):
    rng = np.random.default_rng(5)
    N = grid[0] * grid[1] * grid[2]
    d = 16
    q, k, v = (rng.standard_normal((1, 2, N, d)) for _ in range(3))
    qt, counts = vo.tile_permute(q, grid)
    kt, _ = vo.tile_permute(k, grid)
    vt, _ = vo.tile_permute(v, grid)
    C = counts.shape[0]
    sel = np.broadcast_to(np.arange(C), (1, 2, C, C))
    O_t, lse_t = vo.block_sparse_attention(qt, kt, vt, counts, sel)
    O = vo.untile(O_t, grid)
    assert np.allclose(O, sdpa(q, k, v), rtol=0, atol=1e-12)
    # log-sum-exp against the library routine on the dense scaled scores
    scores = torch.from_numpy(q) @ torch.from_numpy(k).transpose(-1, -2) / math.sqrt(d)
    want_lse = torch.logsumexp(scores, dim=-1).numpy()
    lse = vo.untile(lse_t[..., None], grid)[..., 0]
    assert np.allclose(lse, want_lse, rtol=0, atol=1e-12)


def test_fine_one_hot_equals_single_block_attention():
    grid = (5, 5, 5)
    rng = np.random.default_rng(6)
    d = 8
    q, k, v = (rng.standard_normal((1, 1, 125, d)) for _ in range(3))
    qt, counts = vo.tile_permute(q, grid)
    kt, _ = vo.tile_permute(k, grid)
    vt, _ = vo.tile_permute(v, grid)
    C = counts.shape[0]
    for j in range(C):
        sel = np.full((1, 1, C, 1), j)
        O_t, _ = vo.block_sparse_attention(qt, kt, vt, counts, sel)
        kj = kt[:, :, j * 64:j * 64 + counts[j]]
        vj = vt[:, :, j * 64:j * 64 + counts[j]]
        for i in range(C):
            qi = qt[:, :, i * 64:i * 64 + counts[i]]
            assert np.allclose(O_t[:, :, i * 64:i * 64 + counts[i]], sdpa(qi, kj, vj), atol=1e-12)
            assert np.all(O_t[:, :, i * 64 + counts[i]:(i + 1) * 64] == 0)


def test_fine_equal_keys_give_mean_value_and_rows_normalised():
    grid = (4, 8, 8)
    rng = np.random.default_rng(8)
    d = 8
    q = rng.standard_normal((1, 1, 256, d))
    k = np.tile(rng.standard_normal((1, 1, 1, d)), (1, 1, 256, 1))
    v = rng.standard_normal((1, 1, 256, d))
    qt, counts = vo.tile_permute(q, grid)
    kt, _ = vo.tile_permute(k, grid)
    vt, _ = vo.tile_permute(v, grid)
    sel = np.array([[[[0, 3], [1, 2], [0, 1], [2, 3]]]])
    O_t, _ = vo.block_sparse_attention(qt, kt, vt, counts, sel)
    for i in range(4):
        keys = np.concatenate([vt[0, 0, j * 64:(j + 1) * 64] for j in sel[0, 0, i]])
        assert np.allclose(O_t[0, 0, i * 64:(i + 1) * 64], keys.mean(axis=0), atol=1e-12)
    ones = np.ones_like(vt)
    O1, _ = vo.block_sparse_attention(qt, kt, ones, counts, sel)
    assert np.allclose(O1, 1.0, atol=1e-12)  # softmax rows sum to one


# --------------------------------------------------------------------------
# combine and the whole path
# --------------------------------------------------------------------------

def test_combine_closed_forms():
    grid = (5, 5, 5)
    rng = np.random.default_rng(9)
    slot_token, counts = vo.cube_permutation(grid)
    of_t = rng.standard_normal((1, 2, 8 * 64, 4))
    for c in range(8):
        of_t[:, :, c * 64 + counts[c]:(c + 1) * 64] = 0
    oc = rng.standard_normal((1, 2, 8, 4))
    one, zero = np.ones((1, 2, 125)), np.zeros((1, 2, 125))
    assert np.allclose(vo.combine(of_t, oc, counts, grid, one, zero), of_t)
    got = vo.combine(of_t, oc, counts, grid, zero, one)
    for c in range(8):
        assert np.allclose(got[:, :, c * 64:c * 64 + counts[c]], oc[:, :, c:c + 1])
    assert np.array_equal(vo.combine(of_t, oc, counts, grid), of_t)


def _nested(a):
    return a.tolist()


@pytest.mark.parametrize("grid,d,k,gated", [((4, 8, 8), 64, 2, True), ((5, 6, 7), 8, 3, True),
                                             ((3, 5, 9), 8, 2, False)])
def test_whole_path_matches_loop_restatement(grid, d, k, gated):
    rng = np.random.default_rng(10)
    N = grid[0] * grid[1] * grid[2]
    Hh = 2 if d == 64 else 1
    q, kk, v = (rng.standard_normal((1, Hh, N, d)) for _ in range(3))
    g_f = rng.random((1, Hh, N)) if gated else None
    g_c = rng.random((1, Hh, N)) if gated else None
    ref = vo.vsa_forward(q, kk, v, grid, k, g_f, g_c)
    lp = vsa_forward_loops(_nested(q), _nested(kk), _nested(v), grid, k,
                           None if g_f is None else _nested(g_f),
                           None if g_c is None else _nested(g_c))
    assert np.allclose(ref["S_c"], np.array(lp["S_c"]), atol=1e-12)
    assert ref["sel"].tolist() == lp["sel"]
    assert np.allclose(ref["O_c"], np.array(lp["O_c"]), atol=1e-12)
    assert np.allclose(vo.untile(ref["O_f"], grid), np.array(lp["O_f_tokens"]), atol=1e-12)
    assert np.allclose(ref["out"], np.array(lp["out"]), atol=1e-12)


def test_tiny_workload_dense_topk_equals_dense_attention():
    w = wl.WORKLOADS["tiny_dense"]
    x = wl.make_inputs(w)
    q, k, v = (vo.bf16_bits_to_f64(x[n]) for n in ("q", "k", "v"))
    ref = vo.vsa_forward(q, k, v, w.grid, w.topk)
    O_f = vo.untile(ref["O_f"], w.grid)
    assert np.allclose(O_f, sdpa(q, k, v), atol=1e-12)


def test_bf16_widening_exact():
    bits = np.array([0x3F80, 0xBF80, 0x4049, 0x0000, 0x8000, 0x7F7F, 0x0001], dtype=np.uint16)
    want = [1.0, -1.0, 3.140625, 0.0, -0.0, 3.3895313892515355e38, 9.183549615799121e-41]
    assert vo.bf16_bits_to_f64(bits).tolist() == want


def test_input_rounding_is_nearest_even():
    x = np.array([1.0, 1.00390625, 1.01171875, -2.5, 1.0 + 2 ** -8 + 2 ** -20], dtype=np.float32)
    got = vo.bf16_bits_to_f64(wl.f32_to_bf16_bits(x))
    # 1+2^-8 is a tie -> even (1.0); 1+3*2^-8 tie -> even (1+2^-6); above a tie rounds up
    assert got.tolist() == [1.0, 1.0, 1.015625, -2.5, 1.0078125]
