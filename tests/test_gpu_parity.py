"""GPU parity: every C-ABI call against the float64 oracle on the same seeded
inputs.  Integer work (permutation, counts, selection) is compared exactly
(selection up to coarse-logit ties within 1e-4); floating-point outputs within
max-abs 2e-2 / mean-abs 2e-3 for bf16 in, float32 accumulation."""

import math

import numpy as np
import pytest
import torch

from oracle import vsa_oracle as vo
from video_dit_block_vsa_b200 import workloads as wl
from tests.vsa_checks import (assert_close, bf16_dev_bits, bf16_dev_to_f64, check_selection, wide_first,
                              to_dev_bf16)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vsa():
    from video_dit_block_vsa_b200 import build
    build.build()
    from video_dit_block_vsa_b200 import vsa as mod
    assert mod.vsa_get_status() == 0
    return mod


def rand_bits(shape, seed):
    rng = np.random.default_rng(seed)
    return wl.f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32))


SHAPES = [  # (B, H, d, grid)
    (1, 2, 64, (4, 8, 8)),
    (1, 3, 128, (5, 5, 5)),
    (2, 2, 64, (3, 7, 9)),
    (1, 1, 64, (1, 1, 1)),
    (1, 2, 128, (21, 30, 52)),
    (1, 1, 128, (21, 45, 80)),
]


# --------------------------------------------------------------------------
# tile permute / untile: bit-exact
# --------------------------------------------------------------------------

@pytest.mark.parametrize("B,H,d,grid", SHAPES)
def test_tile_permute_and_untile_bit_exact(vsa, B, H, d, grid):
    N = math.prod(grid)
    bits = rand_bits((B, H, N, d), 11)
    shape = vsa.make_shape(B, H, d, grid)
    C = vsa.vsa_num_cubes(shape)
    x = to_dev_bf16(bits)
    xt = torch.full((B, H, 64 * C, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    counts = torch.full((C,), -7, dtype=torch.int32, device="cuda")
    vsa.vsa_tile_permute(shape, x, xt, counts)
    back = torch.empty_like(x)
    vsa.vsa_untile(shape, xt, back)
    torch.cuda.synchronize()
    ref_t, ref_counts = vo.tile_permute(bits, grid)
    assert np.array_equal(bf16_dev_bits(xt), ref_t)
    assert np.array_equal(counts.cpu().numpy(), ref_counts)
    assert np.array_equal(bf16_dev_bits(back), bits)
    assert vsa.vsa_get_status() == 0


# --------------------------------------------------------------------------
# coarse select: pooling, logits, top-k, coarse output
# --------------------------------------------------------------------------

COARSE = [  # (B, H, d, grid, k)
    (1, 2, 64, (4, 8, 8), 2),
    (1, 2, 64, (4, 8, 8), 4),
    (1, 2, 128, (5, 6, 7), 3),
    (2, 3, 128, (9, 10, 11), 1),
    (1, 2, 128, (21, 30, 52), 62),
    (1, 1, 128, (21, 45, 80), 180),
    (1, 1, 64, (16, 32, 32), 256),
    (1, 1, 64, (48, 48, 48), 200),   # C = 1728: rows longer than the register-cached part
    (1, 1, 64, (36, 64, 64), 300),   # C = 2304: 8 query cubes per coarse CTA
]


def coarse_run(vsa, B, H, d, grid, k, seed=5, cube_mean=0.5):
    w = wl.Workload("t", B, H, d, grid, k, seed, cube_mean, False)
    x = wl.make_inputs(w)
    shape = vsa.make_shape(B, H, d, grid)
    C = vsa.vsa_num_cubes(shape)
    bufs = vsa.VsaBuffers(shape, k, want_coarse=True)
    for name, t in (("q", bufs.q_t), ("k", bufs.k_t), ("v", bufs.v_t)):
        vsa.vsa_tile_permute(shape, to_dev_bf16(x[name]), t, bufs.counts if name == "q" else None)
    logits = torch.empty(B, H, C, C, dtype=torch.float32, device="cuda")
    vsa.vsa_coarse_select(shape, bufs.q_t, bufs.k_t, bufs.v_t, bufs.counts, k, bufs.sel,
                          bufs.workspace, o_coarse=bufs.o_c, coarse_logits=logits)
    torch.cuda.synchronize()
    return w, x, shape, C, bufs, logits


@pytest.mark.parametrize("B,H,d,grid,k", COARSE)
def test_coarse_select(vsa, B, H, d, grid, k):
    w, x, shape, C, bufs, logits = coarse_run(vsa, B, H, d, grid, k)
    q, kk, v = (vo.bf16_bits_to_f64(x[n]) for n in ("q", "k", "v"))
    q_t, counts = vo.tile_permute(q, grid)
    k_t, _ = vo.tile_permute(kk, grid)
    v_t, _ = vo.tile_permute(v, grid)
    qb, kb, vb = vo.pool(q_t, counts), vo.pool(k_t, counts), vo.pool(v_t, counts)
    S, O_c = vo.coarse_attention(qb, kb, vb)
    ws = bufs.workspace.view(torch.float32)[: 3 * B * H * C * d].view(3, B, H, C, d).cpu().numpy()
    assert_close(ws[0], qb, "qbar", 1e-5, 1e-6)
    assert_close(ws[1], kb, "kbar", 1e-5, 1e-6)
    assert_close(ws[2], vb, "vbar", 1e-5, 1e-6)
    assert_close(logits.cpu().numpy(), S, "coarse logits", 2e-5, 2e-6)
    equal, swapped = check_selection(bufs.sel.cpu().numpy(), S, k, counts)
    assert equal + swapped == B * H * C
    assert_close(bufs.o_c.cpu().numpy(), O_c, "coarse output", 1e-4, 1e-5)
    assert vsa.vsa_get_status() == 0


@pytest.mark.parametrize("B,H,d,grid,k", [(1, 2, 64, (4, 8, 8), 2), (2, 3, 128, (9, 10, 11), 5),
                                           (1, 2, 128, (21, 30, 52), 62)])
def test_coarse_select_tokens_equals_tiled_call(vsa, B, H, d, grid, k):
    # pooling straight from token order sums each cube's rows in the same order
    w, x, shape, C, bufs, logits = coarse_run(vsa, B, H, d, grid, k)
    sel = torch.empty_like(bufs.sel)
    o_c = torch.empty_like(bufs.o_c)
    lg = torch.empty_like(logits)
    ws = torch.empty_like(bufs.workspace)
    vsa.vsa_coarse_select_tokens(shape, to_dev_bf16(x["q"]), to_dev_bf16(x["k"]), to_dev_bf16(x["v"]),
                                 k, sel, ws, o_coarse=o_c, coarse_logits=lg)
    torch.cuda.synchronize()
    assert vsa.vsa_get_status() == 0
    n = 3 * B * H * C * d * 4
    assert torch.equal(ws[:n], bufs.workspace[:n])
    assert torch.equal(lg, logits)
    assert torch.equal(sel, bufs.sel)
    assert torch.equal(o_c, bufs.o_c)


@pytest.mark.parametrize("B,H,d,grid,k", [(1, 2, 64, (4, 8, 8), 2), (2, 3, 128, (9, 10, 11), 5),
                                           (1, 2, 128, (21, 30, 52), 62), (1, 1, 64, (1, 1, 1), 1)])
def test_fused_tile_pool_equals_separate_calls(vsa, B, H, d, grid, k):
    # one pass that tiles q, k, v and pools them gives the same bits as the
    # three tiling calls plus the coarse call's own pooling
    w, x, shape, C, bufs, logits = coarse_run(vsa, B, H, d, grid, k)
    qt, kt, vt = (torch.full_like(bufs.q_t, 7.0) for _ in range(3))  # pads must be overwritten
    counts = torch.full_like(bufs.counts, -1)
    ws = torch.empty_like(bufs.workspace)
    vsa.vsa_tile_permute_pool(shape, to_dev_bf16(x["q"]), to_dev_bf16(x["k"]), to_dev_bf16(x["v"]),
                              qt, kt, vt, ws, counts)
    sel = torch.empty_like(bufs.sel)
    o_c = torch.empty_like(bufs.o_c)
    lg = torch.empty_like(logits)
    vsa.vsa_coarse_select_pooled(shape, k, sel, ws, o_coarse=o_c, coarse_logits=lg)
    torch.cuda.synchronize()
    assert vsa.vsa_get_status() == 0
    for got, want in ((qt, bufs.q_t), (kt, bufs.k_t), (vt, bufs.v_t)):
        assert torch.equal(got.view(torch.int16), want.view(torch.int16))
    assert torch.equal(counts, bufs.counts)
    n = 3 * B * H * C * d * 4
    assert torch.equal(ws[:n], bufs.workspace[:n])
    assert torch.equal(lg, logits)
    assert torch.equal(sel, bufs.sel)
    assert torch.equal(o_c, bufs.o_c)


@pytest.mark.parametrize("name", ["tiny_k2", "wan1.3b_ft_16x28x52", "wan1.3b_480p_21x30x52"])
def test_fine_with_fused_combine_untile_equals_separate_calls(vsa, name):
    # the fine kernel writing the final token-order output (gated sum applied
    # when the workload has gates) gives the same bits as fwd + combine + untile
    w = wl.WORKLOADS[name]
    x = wl.make_inputs(w)
    shape = vsa.make_shape(w.batch, w.heads, w.head_dim, w.grid)
    q, k, v = (to_dev_bf16(x[n]) for n in ("q", "k", "v"))
    g_f = torch.from_numpy(x["g_f"]).cuda() if w.gated else None
    g_c = torch.from_numpy(x["g_c"]).cuda() if w.gated else None
    want = torch.empty_like(q)
    bufs = vsa.vsa_forward(shape, q, k, v, w.topk, want, g_f, g_c)
    got = torch.full_like(q, 3.0)
    lse = torch.empty(w.batch, w.heads, 64 * w.cubes, dtype=torch.float32, device="cuda")
    vsa.vsa_block_sparse_fwd_out(shape, bufs.q_t, bufs.k_t, bufs.v_t, bufs.counts, bufs.sel, w.topk,
                                 got, bufs.o_c if w.gated else None, g_f, g_c, lse=lse)
    lse_want = torch.empty_like(lse)
    vsa.vsa_block_sparse_fwd(shape, bufs.q_t, bufs.k_t, bufs.v_t, bufs.counts, bufs.sel, w.topk,
                             bufs.o_f, lse_want)
    torch.cuda.synchronize()
    assert vsa.vsa_get_status() == 0
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))
    assert torch.equal(lse, lse_want)


@pytest.mark.parametrize("grid,k", [((8, 8, 8), 3), ((48, 48, 48), 1700)])
def test_topk_ties_go_to_lower_index(vsa, grid, k):
    # identical k vectors in every cube -> all coarse logits of a row tie
    B, H, d = 1, 1, 64
    N = math.prod(grid)
    shape = vsa.make_shape(B, H, d, grid)
    C = vsa.vsa_num_cubes(shape)
    rng = np.random.default_rng(3)
    kv = np.tile(wl.f32_to_bf16_bits(rng.standard_normal((1, 1, 1, d), dtype=np.float32)), (B, H, N, 1))
    bufs = vsa.VsaBuffers(shape, k)
    vsa.vsa_tile_permute(shape, to_dev_bf16(rand_bits((B, H, N, d), 4)), bufs.q_t, bufs.counts)
    vsa.vsa_tile_permute(shape, to_dev_bf16(kv), bufs.k_t)
    vsa.vsa_tile_permute(shape, to_dev_bf16(kv), bufs.v_t)
    vsa.vsa_coarse_select(shape, bufs.q_t, bufs.k_t, bufs.v_t, bufs.counts, k, bufs.sel, bufs.workspace)
    sel = bufs.sel.cpu().numpy()
    # the k lowest indices, listed wide cubes first (each group ascending)
    assert np.all(sel == wide_first(np.arange(k), vo.cube_permutation(grid)[1]))


# --------------------------------------------------------------------------
# fine block-sparse attention
# --------------------------------------------------------------------------

def fine_case(vsa, B, H, d, grid, sel_np, seed=9, lse=True):
    N = math.prod(grid)
    x = {n: rand_bits((B, H, N, d), seed + i) for i, n in enumerate("qkv")}
    shape = vsa.make_shape(B, H, d, grid)
    C = vsa.vsa_num_cubes(shape)
    k = sel_np.shape[-1]
    bufs = vsa.VsaBuffers(shape, k, want_lse=lse)
    for n, t in (("q", bufs.q_t), ("k", bufs.k_t), ("v", bufs.v_t)):
        vsa.vsa_tile_permute(shape, to_dev_bf16(x[n]), t, bufs.counts if n == "q" else None)
    _, grid_counts = vo.cube_permutation(grid)
    sel_np = wide_first(sel_np, grid_counts)  # the fine kernel's row order
    bufs.sel.copy_(torch.from_numpy(sel_np.astype(np.int32)))
    bufs.o_f.fill_(float("nan"))
    vsa.vsa_block_sparse_fwd(shape, bufs.q_t, bufs.k_t, bufs.v_t, bufs.counts, bufs.sel, k,
                             bufs.o_f, bufs.lse)
    torch.cuda.synchronize()
    q_t, counts = vo.tile_permute(vo.bf16_bits_to_f64(x["q"]), grid)
    k_t, _ = vo.tile_permute(vo.bf16_bits_to_f64(x["k"]), grid)
    v_t, _ = vo.tile_permute(vo.bf16_bits_to_f64(x["v"]), grid)
    ref, ref_lse = vo.block_sparse_attention(q_t, k_t, v_t, counts, sel_np)
    return bufs, ref, ref_lse, counts


def valid_rows(counts):
    return np.concatenate([np.arange(c * 64, c * 64 + n) for c, n in enumerate(counts)])


FINE = [  # (B, H, d, grid, k)
    (1, 2, 64, (4, 8, 8), 2),
    (1, 2, 64, (4, 8, 8), 4),
    (1, 2, 128, (4, 8, 8), 3),
    (1, 3, 128, (5, 5, 5), 8),   # includes a one-token cube
    (2, 2, 64, (3, 7, 9), 5),
    (1, 2, 128, (9, 13, 8), 7),
    (1, 1, 128, (16, 16, 16), 64),
]


@pytest.mark.parametrize("B,H,d,grid,k", FINE)
def test_block_sparse_fwd_random_selection(vsa, B, H, d, grid, k):
    C = math.prod(-(-g // 4) for g in grid)
    rng = np.random.default_rng(17)
    sel = np.stack([np.sort(rng.choice(C, k, replace=False)) for _ in range(B * H * C)])
    sel = sel.reshape(B, H, C, k)
    bufs, ref, ref_lse, counts = fine_case(vsa, B, H, d, grid, sel)
    got = bf16_dev_to_f64(bufs.o_f)
    rows = valid_rows(counts)
    assert_close(got[:, :, rows], ref[:, :, rows], "O_f")
    pad = np.setdiff1d(np.arange(64 * C), rows)
    assert np.all(got[:, :, pad] == 0)
    lse = bufs.lse.cpu().numpy()
    assert_close(lse[:, :, rows], ref_lse[:, :, rows], "lse", 1e-3, 1e-4)
    assert np.all(np.isneginf(lse[:, :, pad]))
    assert vsa.vsa_get_status() == 0


def test_block_sparse_fwd_one_hot(vsa):
    B, H, d, grid = 1, 2, 128, (5, 9, 9)
    C = math.prod(-(-g // 4) for g in grid)
    sel = np.broadcast_to(((np.arange(C) + 1) % C)[:, None], (B, H, C, 1)).copy()
    bufs, ref, _, counts = fine_case(vsa, B, H, d, grid, sel, lse=False)
    rows = valid_rows(counts)
    assert_close(bf16_dev_to_f64(bufs.o_f)[:, :, rows], ref[:, :, rows], "O_f one-hot")


def test_block_sparse_fwd_deterministic(vsa):
    B, H, d, grid, k = 1, 4, 128, (16, 16, 16), 8
    C = 64
    rng = np.random.default_rng(2)
    sel = np.stack([np.sort(rng.choice(C, k, replace=False)) for _ in range(B * H * C)]).reshape(B, H, C, k)
    bufs, _, _, _ = fine_case(vsa, B, H, d, grid, sel, lse=False)
    first = bufs.o_f.clone()
    for _ in range(2):
        vsa.vsa_block_sparse_fwd(bufs.shape, bufs.q_t, bufs.k_t, bufs.v_t, bufs.counts, bufs.sel, k, bufs.o_f)
        torch.cuda.synchronize()
        assert torch.equal(first.view(torch.int16), bufs.o_f.view(torch.int16))


# --------------------------------------------------------------------------
# combine
# --------------------------------------------------------------------------

@pytest.mark.parametrize("B,H,d,grid", [(1, 2, 64, (4, 8, 8)), (1, 2, 128, (5, 6, 7)),
                                        (2, 1, 128, (21, 30, 52))])
def test_combine(vsa, B, H, d, grid):
    N = math.prod(grid)
    shape = vsa.make_shape(B, H, d, grid)
    C = vsa.vsa_num_cubes(shape)
    rng = np.random.default_rng(21)
    of_bits, counts = vo.tile_permute(rand_bits((B, H, N, d), 3), grid)
    o_f = to_dev_bf16(of_bits)
    o_c = torch.from_numpy(rng.standard_normal((B, H, C, d)).astype(np.float32)).cuda()
    g_f = torch.from_numpy(rng.random((B, H, N), dtype=np.float32)).cuda()
    g_c = torch.from_numpy(rng.random((B, H, N), dtype=np.float32)).cuda()
    out = torch.full_like(o_f, float("nan"))
    vsa.vsa_combine(shape, o_f, out, o_c, g_f, g_c)
    torch.cuda.synchronize()
    ref = vo.combine(vo.bf16_bits_to_f64(of_bits), o_c.double().cpu().numpy(), counts, grid,
                     g_f.double().cpu().numpy(), g_c.double().cpu().numpy())
    got = bf16_dev_to_f64(out)
    # bf16 rounding of the result (half an ulp <= 2^-8 relative) plus the
    # float32 evaluation of g_f*O_f + g_c*O_c (~1e-7 absolute for O(1) terms,
    # visible only where the two terms nearly cancel)
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-6)
    # ungated: a copy; in place: nothing to do
    out2 = torch.full_like(o_f, float("nan"))
    vsa.vsa_combine(shape, o_f, out2)
    torch.cuda.synchronize()
    assert torch.equal(out2.view(torch.int16), o_f.view(torch.int16))
    # in-place gated
    o_f2 = o_f.clone()
    vsa.vsa_combine(shape, o_f2, o_f2, o_c, g_f, g_c)
    torch.cuda.synchronize()
    assert torch.equal(o_f2.view(torch.int16), out.view(torch.int16))


# --------------------------------------------------------------------------
# whole path on the workloads, through the public forward call
# --------------------------------------------------------------------------

def sampled_cubes(counts, n, seed):
    C = counts.shape[0]
    rng = np.random.default_rng(seed)
    picks = {0, C - 1, int(np.argmin(counts))}
    partial = np.flatnonzero(counts < 64)
    if partial.size:
        picks.update(rng.choice(partial, min(4, partial.size), replace=False).tolist())
    picks.update(rng.choice(C, min(n, C), replace=False).tolist())
    return sorted(picks)


def check_workload(vsa, w, head_sample=None, cube_sample=None):
    """Runs the workload through both forms of the public forward call and
    checks them against the oracle:
      - the three launches the benchmark times (``vsa_forward_fused``: tiling
        with pooling, coarse stage from the means, fine kernel writing the gated
        token-order output), on every head: tiled q, k, v bit-exact, selection
        tie-aware; the output on the sampled heads and query cubes;
      - the five separate calls (``vsa_forward``): selection and output
        bit-identical to the fused form on every head."""
    x = wl.make_inputs(w)
    shape = vsa.make_shape(w.batch, w.heads, w.head_dim, w.grid)
    q, k, v = (to_dev_bf16(x[n]) for n in ("q", "k", "v"))
    g_f = torch.from_numpy(x["g_f"]).cuda() if w.gated else None
    g_c = torch.from_numpy(x["g_c"]).cuda() if w.gated else None
    out = torch.empty_like(q)
    bufs = vsa.vsa_forward_fused(shape, q, k, v, w.topk, out, g_f, g_c)
    torch.cuda.synchronize()
    assert vsa.vsa_get_status() == 0
    # the separate calls: same selection and output bits as the fused form
    out_calls = torch.empty_like(q)
    bufs_calls = vsa.vsa_forward(shape, q, k, v, w.topk, out_calls, g_f, g_c)
    torch.cuda.synchronize()
    assert vsa.vsa_get_status() == 0
    assert torch.equal(bufs_calls.sel, bufs.sel), f"{w.name}: selections of the two forms differ"
    assert torch.equal(out_calls.view(torch.int16), out.view(torch.int16)), \
        f"{w.name}: outputs of the two forms differ"
    del bufs_calls, out_calls
    sel_gpu = bufs.sel.cpu().numpy()
    heads = [(b, h) for b in range(w.batch) for h in range(w.heads)]
    sampled = set(heads)
    if head_sample is not None:
        rng = np.random.default_rng(w.seed)
        idx = sorted(rng.choice(len(heads), head_sample, replace=False).tolist())
        sampled = {heads[i] for i in idx}
    slot_token, counts = vo.cube_permutation(w.grid)
    assert np.array_equal(bufs.counts.cpu().numpy(), counts)
    for b, h in heads:
        tiled = {}
        for n, dev_t in (("q", bufs.q_t), ("k", bufs.k_t), ("v", bufs.v_t)):
            ref_bits, _ = vo.tile_permute(x[n][b:b + 1, h:h + 1], w.grid)
            assert np.array_equal(bf16_dev_bits(dev_t[b, h]), ref_bits[0, 0]), \
                f"{w.name}: tiled {n} differs (b={b}, h={h})"
            tiled[n] = vo.bf16_bits_to_f64(ref_bits)
        q_t, k_t, v_t = tiled["q"], tiled["k"], tiled["v"]
        S, O_c = vo.coarse_attention(vo.pool(q_t, counts), vo.pool(k_t, counts), vo.pool(v_t, counts))
        sel = sel_gpu[b:b + 1, h:h + 1]
        check_selection(sel, S, w.topk, counts)  # selection up to ties; outputs use the GPU's choice
        if (b, h) not in sampled:
            continue
        gf = x["g_f"][b:b + 1, h:h + 1].astype(np.float64) if w.gated else None
        gc = x["g_c"][b:b + 1, h:h + 1].astype(np.float64) if w.gated else None
        cubes = None if cube_sample is None else sampled_cubes(counts, cube_sample, w.seed + h)
        O_f, _ = vo.block_sparse_attention(q_t, k_t, v_t, counts, sel, query_cubes=cubes)
        ref = vo.untile(vo.combine(O_f, O_c, counts, w.grid, gf, gc), w.grid)[0, 0]
        cube_list = range(counts.shape[0]) if cubes is None else cubes
        toks = np.concatenate([slot_token[c, :counts[c]] for c in cube_list])
        got = bf16_dev_to_f64(out[b, h])
        assert_close(got[toks], ref[toks], f"{w.name} out (b={b}, h={h})")


def test_largest_cube_count(vsa):
    """C = 8192 cubes, the most a coarse row holds (32 x 128 x 128 latents, one
    head, d = 64): the whole path against the oracle, selection on every row."""
    w = wl.Workload("max_cubes_32x128x128", 1, 1, 64, (32, 128, 128), 8, 41, 0.5, False)
    check_workload(vsa, w, cube_sample=12)


@pytest.mark.parametrize("name", ["tiny_k2", "tiny_dense"])
def test_workload_tiny_full(vsa, name):
    check_workload(vsa, wl.WORKLOADS[name])


@pytest.mark.parametrize("name", ["scaling_16x32x32", "wan1.3b_ft_16x28x52", "wan1.3b_480p_21x30x52"])
def test_workload_sampled(vsa, name):
    check_workload(vsa, wl.WORKLOADS[name], head_sample=3, cube_sample=24)


@pytest.mark.parametrize("name", ["wan14b_720p_21x45x80_k180", "wan14b_720p_21x45x80_k43",
                                  "wan14b_720p_21x45x80_dense"])
def test_workload_720p_full_size_sampled(vsa, name):
    check_workload(vsa, wl.WORKLOADS[name], head_sample=2, cube_sample=12)


# --------------------------------------------------------------------------
# status word: timeouts and bad indices are reported, the context survives
# --------------------------------------------------------------------------

def test_bounded_wait_times_out_and_context_survives(vsa):
    vsa.vsa_debug_wait_timeout(2_000_000)  # 2 ms on a barrier nothing arrives at
    assert vsa.vsa_get_status() == vsa.VSA_ERR_TIMEOUT
    assert vsa.vsa_get_status() == 0  # cleared
    check_workload(vsa, wl.WORKLOADS["tiny_k2"])


def test_inconsistent_indices_are_reported(vsa):
    B, H, d, grid, k = 1, 1, 64, (5, 5, 5), 2
    C = 8
    sel = np.broadcast_to(np.array([0, 1]), (B, H, C, k)).copy()
    bufs, _, _, _ = fine_case(vsa, B, H, d, grid, sel, lse=False)
    assert vsa.vsa_get_status() == 0
    bufs.sel[..., 0] = 3  # not ascending
    vsa.vsa_block_sparse_fwd(bufs.shape, bufs.q_t, bufs.k_t, bufs.v_t, bufs.counts, bufs.sel, k, bufs.o_f)
    assert vsa.vsa_get_status() == vsa.VSA_ERR_BAD_INDEX
    bufs.sel[..., 1] = 99  # out of range: clamped, reported
    vsa.vsa_block_sparse_fwd(bufs.shape, bufs.q_t, bufs.k_t, bufs.v_t, bufs.counts, bufs.sel, k, bufs.o_f)
    assert vsa.vsa_get_status() == vsa.VSA_ERR_BAD_INDEX
    bufs.counts.fill_(64)  # not this grid's counts
    bufs.sel.copy_(torch.from_numpy(sel.astype(np.int32)))
    vsa.vsa_block_sparse_fwd(bufs.shape, bufs.q_t, bufs.k_t, bufs.v_t, bufs.counts, bufs.sel, k, bufs.o_f)
    assert vsa.vsa_get_status() == vsa.VSA_ERR_BAD_INDEX
    assert vsa.vsa_get_status() == 0
