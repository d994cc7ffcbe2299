"""GPU parity of the DiT-block projections with the layout changes fused in
(vsa_qkv_projection_tiled, vsa_out_projection_tiled) and of the whole block
(vsa.vsa_attention_block) against the float64 oracle (oracle/vsa_dit.py).

The products run on the tensor cores with bf16 operands and float32
accumulation, then round to bf16: a result is within half a bf16 ulp of the
exact value (at most 2^-8 of its magnitude) plus the float32 accumulation
error, which is absolute (partial sums are as large as the result's scale)
and grows with the reduction length: at K = 5120 it measured ~2e-6 of the
largest result, as for a float32 GEMM on the CUDA cores.  Each element must
lie within 2^-8 of its own magnitude plus 2^-14 of the largest magnitude.  The
whole block compares y with the oracle's block run on the GPU's own q, k, v
(the selection checked tie-aware), at 1e-2 (max) / 1e-3 (mean) of max |y|."""

import numpy as np
import pytest
import torch

from oracle import vsa_dit as vd
from oracle import vsa_oracle as vo
from video_dit_block_vsa_b200 import workloads as wl
from tests.vsa_checks import bf16_dev_to_f64, check_selection, to_dev_bf16

pytestmark = pytest.mark.gpu

REL = 2.0 ** -8


@pytest.fixture(scope="module")
def vsa():
    from video_dit_block_vsa_b200 import build
    build.build()
    from video_dit_block_vsa_b200 import vsa as mod
    assert mod.vsa_get_status() == 0
    return mod


def bits(shape, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return wl.f32_to_bf16_bits((scale * rng.standard_normal(shape, dtype=np.float32)).astype(np.float32))


def close_elementwise(got, ref, what):
    err = np.abs(got - ref)
    bound = REL * np.abs(ref) + 2.0 ** -14 * np.abs(ref).max()
    bad = err > bound
    assert not bad.any(), f"{what}: {bad.sum()} elements off, worst {err.max():.3e}"


CASES = [(1, 2, 64, (4, 8, 8), 128), (2, 2, 128, (5, 7, 9), 192), (1, 3, 64, (6, 5, 10), 256),
         (1, 2, 128, (16, 28, 52), 256)]


@pytest.mark.parametrize("B,H,d,grid,hidden", CASES)
def test_qkv_projection_tiled(vsa, B, H, d, grid, hidden):
    N = int(np.prod(grid))
    shape = vsa.make_shape(B, H, d, grid)
    C = vsa.vsa_num_cubes(shape)
    xb = bits((B, N, hidden), 1)
    wb = bits((3 * H * d, hidden), 2, hidden ** -0.5)
    q_t, k_t, v_t = (torch.full((B, H, 64 * C, d), float("nan"), dtype=torch.bfloat16, device="cuda")
                     for _ in range(3))
    counts = torch.full((C,), -1, dtype=torch.int32, device="cuda")
    vsa.vsa_qkv_projection_tiled(shape, hidden, to_dev_bf16(xb), to_dev_bf16(wb), q_t, k_t, v_t, counts)
    torch.cuda.synchronize()
    assert vsa.vsa_get_status() == 0
    refs = vd.qkv_projection(vo.bf16_bits_to_f64(xb), vo.bf16_bits_to_f64(wb), H, d)
    _, cnt = vo.cube_permutation(grid)
    assert np.array_equal(counts.cpu().numpy(), cnt)
    for name, t, ref in zip("qkv", (q_t, k_t, v_t), refs):
        ref_t, _ = vo.tile_permute(ref, grid)  # pad rows 0
        close_elementwise(bf16_dev_to_f64(t), ref_t, f"{name}_tiled {grid}")


@pytest.mark.parametrize("B,H,d,grid,hidden", CASES)
def test_out_projection_tiled(vsa, B, H, d, grid, hidden):
    N = int(np.prod(grid))
    shape = vsa.make_shape(B, H, d, grid)
    C = vsa.vsa_num_cubes(shape)
    ob = bits((B, H, 64 * C, d), 3)  # pad rows hold values too: they must not reach y
    wb = bits((hidden, H * d), 4, (H * d) ** -0.5)
    y = torch.full((B, N, hidden), float("nan"), dtype=torch.bfloat16, device="cuda")
    vsa.vsa_out_projection_tiled(shape, hidden, to_dev_bf16(ob), to_dev_bf16(wb), y)
    torch.cuda.synchronize()
    assert vsa.vsa_get_status() == 0
    ref = vd.out_projection(vo.untile(vo.bf16_bits_to_f64(ob), grid), vo.bf16_bits_to_f64(wb))
    close_elementwise(bf16_dev_to_f64(y), ref, f"y {grid}")


@pytest.mark.parametrize("name,heads,hidden", [("tiny_k2", None, 128), ("wan1.3b_ft_16x28x52", 2, 256),
                                               ("wan1.3b_480p_21x30x52", 1, 128)])
def test_attention_block(vsa, name, heads, hidden):
    w = wl.WORKLOADS[name]
    H = w.heads if heads is None else heads
    B, N, d = w.batch, w.tokens, w.head_dim
    shape = vsa.make_shape(B, H, d, w.grid)
    x = wl.make_inputs(w, heads=H)
    xb = bits((B, N, hidden), w.seed + 10)
    wq = bits((3 * H * d, hidden), w.seed + 11, hidden ** -0.5)
    wo = bits((hidden, H * d), w.seed + 12, (H * d) ** -0.5)
    g_f = torch.from_numpy(x["g_f"]).cuda() if w.gated else None
    g_c = torch.from_numpy(x["g_c"]).cuda() if w.gated else None
    y = torch.empty(B, N, hidden, dtype=torch.bfloat16, device="cuda")
    bufs = vsa.vsa_attention_block(shape, hidden, to_dev_bf16(xb), to_dev_bf16(wq), to_dev_bf16(wo),
                                   w.topk, y, g_f, g_c)
    torch.cuda.synchronize()
    assert vsa.vsa_get_status() == 0
    # the oracle's block on the GPU's own (bf16) q, k, v
    q_t, k_t, v_t = (bf16_dev_to_f64(t) for t in (bufs.q_t, bufs.k_t, bufs.v_t))
    _, counts = vo.cube_permutation(w.grid)
    S, O_c = vo.coarse_attention(vo.pool(q_t, counts), vo.pool(k_t, counts), vo.pool(v_t, counts))
    sel = bufs.sel.cpu().numpy()
    check_selection(sel, S, w.topk, counts)
    O_f, _ = vo.block_sparse_attention(q_t, k_t, v_t, counts, sel)
    gf = x["g_f"].astype(np.float64) if w.gated else None
    gc = x["g_c"].astype(np.float64) if w.gated else None
    o = vo.untile(vo.combine(O_f, O_c, counts, w.grid, gf, gc), w.grid)
    ref = vd.out_projection(o, vo.bf16_bits_to_f64(wo))
    got = bf16_dev_to_f64(y)
    m = np.abs(ref).max()
    e = np.abs(got - ref)
    assert e.max() <= 1e-2 * m, f"{name} y: max err {e.max():.3e} vs max |y| {m:.3e}"
    assert e.mean() <= 1e-3 * m, f"{name} y: mean err {e.mean():.3e} vs max |y| {m:.3e}"
    # q, k, v themselves against the oracle's projection
    refs = vd.qkv_projection(vo.bf16_bits_to_f64(xb), vo.bf16_bits_to_f64(wq), H, d)
    for n_, t, r in zip("qkv", (q_t, k_t, v_t), refs):
        close_elementwise(t, vo.tile_permute(r, w.grid)[0], f"{name} {n_}_tiled")


def test_projections_full_size_sampled(vsa):
    """Wan-14B at 720p: hidden 5120, 40 heads x 128, 75.6k tokens (the sizes a
    720p block runs); sampled tokens checked row by row for both projections."""
    w = wl.WORKLOADS["wan14b_720p_21x45x80_k180"]
    B, H, d, N, hidden = w.batch, w.heads, w.head_dim, w.tokens, 5120
    shape = vsa.make_shape(B, H, d, w.grid)
    C = vsa.vsa_num_cubes(shape)
    xb = bits((B, N, hidden), 21)
    wq = bits((3 * H * d, hidden), 22, hidden ** -0.5)
    q_t, k_t, v_t = (torch.empty(B, H, 64 * C, d, dtype=torch.bfloat16, device="cuda") for _ in range(3))
    vsa.vsa_qkv_projection_tiled(shape, hidden, to_dev_bf16(xb), to_dev_bf16(wq), q_t, k_t, v_t)
    torch.cuda.synchronize()
    assert vsa.vsa_get_status() == 0
    slot_token, counts = vo.cube_permutation(w.grid)
    rng = np.random.default_rng(23)
    toks = np.unique(np.concatenate([rng.choice(N, 48, replace=False), [0, N - 1],
                                     slot_token[int(np.argmin(counts)), :1]]))
    tiled_row = np.empty(N, dtype=np.int64)
    for c in range(C):
        for s in range(int(counts[c])):
            tiled_row[slot_token[c, s]] = 64 * c + s
    xs = vo.bf16_bits_to_f64(xb[:, toks])
    refs = vd.qkv_projection(xs, vo.bf16_bits_to_f64(wq), H, d)  # [B, H, len(toks), d]
    rows = torch.from_numpy(tiled_row[toks]).cuda()
    for n_, t, r in zip("qkv", (q_t, k_t, v_t), refs):
        close_elementwise(bf16_dev_to_f64(t[:, :, rows]), r, f"720p {n_}_tiled")
    del q_t, k_t, v_t
    # output projection from a tiled o
    ob = bits((B, H, 64 * C, d), 24)
    wo = bits((hidden, H * d), 25, (H * d) ** -0.5)
    y = torch.empty(B, N, hidden, dtype=torch.bfloat16, device="cuda")
    vsa.vsa_out_projection_tiled(shape, hidden, to_dev_bf16(ob), to_dev_bf16(wo), y)
    torch.cuda.synchronize()
    assert vsa.vsa_get_status() == 0
    o_s = vo.bf16_bits_to_f64(ob[:, :, tiled_row[toks]])  # [B, H, len(toks), d]
    ref = vd.out_projection(o_s, vo.bf16_bits_to_f64(wo))
    close_elementwise(bf16_dev_to_f64(y[:, torch.from_numpy(toks).cuda()]), ref, "720p y")


def test_projection_rejects_bad_hidden(vsa):
    shape = vsa.make_shape(1, 2, 64, (4, 8, 8))
    C = vsa.vsa_num_cubes(shape)
    x = torch.zeros(1, 256, 96, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(3 * 2 * 64, 96, dtype=torch.bfloat16, device="cuda")
    q = torch.zeros(1, 2, 64 * C, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(vsa.VsaError):
        vsa.vsa_qkv_projection_tiled(shape, 96, x, w, q, q, q)  # hidden not a multiple of 64
