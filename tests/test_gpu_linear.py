"""GPU parity of the low-rank linear compensation branch (vsa_linear_branch_add)
against the float64 oracle (oracle/vsa_linear.py): the branch alone (added to a
zero output) and the whole sparse + linear forward (the block-sparse forward
the benchmark runs, then the branch added in place).  Tolerances as for every
bf16 output: max-abs 2e-2, mean-abs 2e-3."""

import numpy as np
import pytest
import torch

from oracle import vsa_linear as vl
from oracle import vsa_oracle as vo
from video_dit_block_vsa_b200 import workloads as wl
from tests.vsa_checks import assert_close, bf16_dev_to_f64, check_selection, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vsa():
    from video_dit_block_vsa_b200 import build
    build.build()
    from video_dit_block_vsa_b200 import vsa as mod
    assert mod.vsa_get_status() == 0
    return mod


def rand_bits(shape, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return wl.f32_to_bf16_bits(scale * rng.standard_normal(shape, dtype=np.float32))


@pytest.mark.parametrize("B,H,d,grid", [(1, 2, 64, (4, 8, 8)), (2, 3, 128, (5, 7, 9)),
                                        (1, 2, 128, (21, 30, 52)), (1, 1, 64, (1, 1, 1))])
def test_linear_branch_alone(vsa, B, H, d, grid):
    N = int(np.prod(grid))
    shape = vsa.make_shape(B, H, d, grid)
    x = {n: rand_bits((B, H, N, d), 31 + i, 1.5) for i, n in enumerate("qkv")}
    q, k, v = (to_dev_bf16(x[n]) for n in "qkv")
    out = torch.zeros_like(q)
    ws = torch.empty(vsa.vsa_linear_workspace_bytes(shape), dtype=torch.uint8, device="cuda")
    vsa.vsa_linear_branch_add(shape, q, k, v, out, ws)
    torch.cuda.synchronize()
    assert vsa.vsa_get_status() == 0
    f64 = lambda n: vo.bf16_bits_to_f64(x[n])
    ref = vl.linear_attention(f64("q"), f64("k"), f64("v"))
    assert_close(bf16_dev_to_f64(out), ref, f"linear branch {grid}")
    # deterministic: a second call on a zero output gives the same bits
    out2 = torch.zeros_like(q)
    vsa.vsa_linear_branch_add(shape, q, k, v, out2, ws)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))


def sampled_cubes(counts, n, seed):
    """The first, last and smallest cube, a few partial ones and n random ones."""
    C = counts.shape[0]
    rng = np.random.default_rng(seed)
    picks = {0, C - 1, int(np.argmin(counts))}
    partial = np.flatnonzero(counts < 64)
    if partial.size:
        picks.update(rng.choice(partial, min(4, partial.size), replace=False).tolist())
    picks.update(rng.choice(C, min(n, C), replace=False).tolist())
    return sorted(picks)


@pytest.mark.parametrize("name,heads,cube_sample", [("tiny_k2", None, None),
                                                    ("wan1.3b_ft_16x28x52", 2, 24),
                                                    ("wan14b_720p_21x45x80_k43", 1, 16)])
def test_sparse_plus_linear_forward(vsa, name, heads, cube_sample):
    """The three-launch block-sparse forward, then the branch added in place:
    out = O_sparse + O_lin against the oracle's sum, on every head's selection
    (tie-aware) and the sampled query cubes' tokens."""
    w = wl.WORKLOADS[name]
    H = w.heads if heads is None else heads
    x = wl.make_inputs(w, heads=H)
    shape = vsa.make_shape(w.batch, H, w.head_dim, w.grid)
    q, k, v = (to_dev_bf16(x[n]) for n in ("q", "k", "v"))
    g_f = torch.from_numpy(x["g_f"]).cuda() if w.gated else None
    g_c = torch.from_numpy(x["g_c"]).cuda() if w.gated else None
    out = torch.empty_like(q)
    bufs = vsa.vsa_forward_fused(shape, q, k, v, w.topk, out, g_f, g_c)
    ws = torch.empty(vsa.vsa_linear_workspace_bytes(shape), dtype=torch.uint8, device="cuda")
    vsa.vsa_linear_branch_add(shape, q, k, v, out, ws)
    torch.cuda.synchronize()
    assert vsa.vsa_get_status() == 0
    sel_gpu = bufs.sel.cpu().numpy()
    slot_token, counts = vo.cube_permutation(w.grid)
    for b in range(w.batch):
        for h in range(H):
            f64 = {n: vo.bf16_bits_to_f64(x[n][b:b + 1, h:h + 1]) for n in "qkv"}
            tiled = {n: vo.tile_permute(f64[n], w.grid)[0] for n in "qkv"}
            S, O_c = vo.coarse_attention(*(vo.pool(tiled[n], counts) for n in "qkv"))
            sel = sel_gpu[b:b + 1, h:h + 1]
            check_selection(sel, S, w.topk, counts)  # outputs use the GPU's (tie-checked) choice
            cubes = None if cube_sample is None else sampled_cubes(counts, cube_sample, w.seed + h)
            O_f, _ = vo.block_sparse_attention(tiled["q"], tiled["k"], tiled["v"], counts, sel,
                                               query_cubes=cubes)
            gf = x["g_f"][b:b + 1, h:h + 1].astype(np.float64) if w.gated else None
            gc = x["g_c"][b:b + 1, h:h + 1].astype(np.float64) if w.gated else None
            sparse = vo.untile(vo.combine(O_f, O_c, counts, w.grid, gf, gc), w.grid)
            want = (sparse + vl.linear_attention(f64["q"], f64["k"], f64["v"]))[0, 0]
            cube_list = range(counts.shape[0]) if cubes is None else cubes
            toks = np.concatenate([slot_token[c, :counts[c]] for c in cube_list])
            got = bf16_dev_to_f64(out[b, h])
            assert_close(got[toks], want[toks], f"{name} sparse + linear (b={b}, h={h})")


def test_linear_branch_rejects_bad_arguments(vsa):
    shape = vsa.make_shape(1, 1, 64, (4, 4, 4))
    N = 64
    q = torch.zeros(1, 1, N, 64, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(vsa.vsa_linear_workspace_bytes(shape), dtype=torch.uint8, device="cuda")
    with pytest.raises(vsa.VsaError):
        vsa.vsa_linear_branch_add(shape, q, q, q, q, ws[:16])  # workspace too small
