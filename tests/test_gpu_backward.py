"""The whole backward on the GPU (vsa_backward: combine gradient, coarse
backward, selection transpose, fine backward with the pooling and untile steps)
against the oracle's vsa_backward, which differentiates the float64 forward
with the selection held at its choice.

The GPU rounds where a bf16 training step would: O_f and the gated dO_f are
bf16, P and dS are computed in float32 and enter the tensor-core products as
bf16, the products accumulate in float32, dq, dk, dv are bf16.  A CPU
emulation of those roundings lands within 5.6e-3 (max) and 3e-4 (mean) of
the largest gradient on these cases; the bounds below leave 1.8x and 3x of
room.  A wrong index, a transposed operand or a dropped term is off by the
gradient's own size.

"""

import numpy as np
import pytest
import torch

from oracle import vsa_backward as vb
from oracle import vsa_oracle as vo
from video_dit_block_vsa_b200 import workloads as wl
from tests.vsa_checks import bf16_dev_to_f64, check_selection, to_dev_bf16

pytestmark = pytest.mark.gpu

MAX_REL = 1e-2   # max |got - ref| / max |ref|, per gradient
MEAN_REL = 1e-3  # mean |got - ref| / max |ref|


@pytest.fixture(scope="module")
def vsa():
    from video_dit_block_vsa_b200 import build
    build.build()
    from video_dit_block_vsa_b200 import vsa as mod
    assert mod.vsa_get_status() == 0
    return mod


def check(got, ref, what):
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    m = np.abs(ref).max()
    e = np.abs(got - ref)
    assert e.max() <= MAX_REL * m, f"{what}: max err {e.max():.3e} vs max |ref| {m:.3e}"
    assert e.mean() <= MEAN_REL * m, f"{what}: mean err {e.mean():.3e} vs max |ref| {m:.3e}"


def run_backward(vsa, w, heads, seed_offset=400):
    H = w.heads if heads is None else heads
    B, N, d = w.batch, w.tokens, w.head_dim
    x = wl.make_inputs(w, heads=H)
    shape = vsa.make_shape(B, H, d, w.grid)
    q, k, v = (to_dev_bf16(x[n]) for n in ("q", "k", "v"))
    g_f = torch.from_numpy(x["g_f"]).cuda() if w.gated else None
    g_c = torch.from_numpy(x["g_c"]).cuda() if w.gated else None
    out = torch.empty_like(q)
    bufs = vsa.VsaBuffers(shape, w.topk, want_coarse=w.gated, want_lse=True)
    vsa.vsa_forward(shape, q, k, v, w.topk, out, g_f, g_c, bufs=bufs)
    rng = np.random.default_rng(w.seed + seed_offset)
    dout_bits = wl.f32_to_bf16_bits(rng.standard_normal((B, H, N, d), dtype=np.float32))
    dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
    dgf = torch.empty(B, H, N, dtype=torch.float32, device="cuda") if w.gated else None
    dgc = torch.empty_like(dgf) if w.gated else None
    vsa.vsa_backward(shape, bufs, to_dev_bf16(dout_bits), dq, dk, dv, g_f, g_c, dgf, dgc)
    torch.cuda.synchronize()
    assert vsa.vsa_get_status() == 0
    return x, dout_bits, bufs, (dq, dk, dv, dgf, dgc)


CASES = [
    (wl.WORKLOADS["tiny_k2"], None),                                           # gated, d = 64, C = 4
    (wl.Workload("ragged_gated", 2, 2, 128, (5, 7, 9), 3, 21, 0.5, True), None),  # B = 2, partial cubes
    (wl.Workload("ragged_ungated", 1, 2, 64, (6, 5, 10), 4, 22, 0.5, False), None),
    (wl.WORKLOADS["wan1.3b_ft_16x28x52"], 1),                                  # C = 364, k = 46, gated
]


@pytest.mark.parametrize("w,heads", CASES, ids=[c[0].name for c in CASES])
def test_backward_matches_oracle(vsa, w, heads):
    x, dout_bits, bufs, (dq, dk, dv, dgf, dgc) = run_backward(vsa, w, heads)
    f64 = lambda n: vo.bf16_bits_to_f64(x[n])
    gf = x["g_f"].astype(np.float64) if w.gated else None
    gc = x["g_c"].astype(np.float64) if w.gated else None
    args = (f64("q"), f64("k"), f64("v"), w.grid, w.topk, vo.bf16_bits_to_f64(dout_bits), gf, gc)
    ref = vb.vsa_backward(*args)
    sel = bufs.sel.cpu().numpy().astype(np.int64)
    counts = vo.cube_permutation(w.grid)[1]
    equal, swapped = check_selection(sel, ref["S_c"], w.topk, counts)  # a top-k set up to the tie band
    if swapped:  # gradients of the GPU's (equally valid) selection
        ref = vb.vsa_backward(*args, sel=sel)
    check(bf16_dev_to_f64(dq), ref["dq"], "dq")
    check(bf16_dev_to_f64(dk), ref["dk"], "dk")
    check(bf16_dev_to_f64(dv), ref["dv"], "dv")
    if w.gated:
        check(dgf.double().cpu().numpy(), ref["dg_f"], "dg_f")
        check(dgc.double().cpu().numpy(), ref["dg_c"], "dg_c")


def test_backward_is_deterministic(vsa):
    w = wl.Workload("ragged_gated", 2, 2, 128, (5, 7, 9), 3, 21, 0.5, True)
    first = run_backward(vsa, w, None)[3]
    second = run_backward(vsa, w, None)[3]
    for a, b in zip(first, second):
        assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a,
                           b.view(torch.int16) if b.dtype == torch.bfloat16 else b)


def test_fine_backward_alone_on_a_random_selection(vsa):
    # vsa_block_sparse_bwd on a selection the coarse stage did not make (key
    # cubes chosen by no query cube get zero gradient), ungated (no pooled term)
    B, H, d, grid, k = 1, 2, 64, (10, 14, 15), 2
    shape = vsa.make_shape(B, H, d, grid)
    C = vsa.vsa_num_cubes(shape)
    N = int(np.prod(grid))
    rng = np.random.default_rng(77)
    bits = {n: wl.f32_to_bf16_bits(rng.standard_normal((B, H, N, d), dtype=np.float32)) for n in "qkv"}
    sel = np.stack([np.sort(rng.choice(C, k, replace=False)) for _ in range(B * H * C)]).reshape(B, H, C, k)
    f64 = {n: vo.bf16_bits_to_f64(b) for n, b in bits.items()}
    qt, counts = vo.tile_permute(f64["q"], grid)
    kt, _ = vo.tile_permute(f64["k"], grid)
    vt, _ = vo.tile_permute(f64["v"], grid)
    of, lse = vo.block_sparse_attention(qt, kt, vt, counts, sel)
    dof_bits = wl.f32_to_bf16_bits(rng.standard_normal((B, H, 64 * C, d), dtype=np.float32))
    dof_bits, _ = vo.tile_permute(vo.untile(dof_bits, grid), grid)  # pad rows 0
    dof = vo.bf16_bits_to_f64(dof_bits)
    of_bits = wl.f32_to_bf16_bits(of.astype(np.float32))
    delta = np.sum(dof * vo.bf16_bits_to_f64(of_bits), axis=-1).astype(np.float32)
    ref_q, ref_k, ref_v = vb.block_sparse_attention_backward(qt, kt, vt, counts, sel, dof)

    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    tiled = {n: dev(vo.tile_permute(bits[n], grid)[0].view(np.int16)).view(torch.bfloat16) for n in "qkv"}
    d_sel = dev(sel.astype(np.int32))
    offs = torch.empty(B, H, C + 1, dtype=torch.int32, device="cuda")
    lists = torch.empty(B, H, C * k, dtype=torch.int32, device="cuda")
    ws = torch.empty(B * H * C * k * 4, dtype=torch.uint8, device="cuda")
    vsa.vsa_select_transpose(shape, d_sel, k, offs, lists, ws)
    dq, dk, dv = (torch.full((B, H, N, d), float("nan"), dtype=torch.bfloat16, device="cuda")
                  for _ in range(3))
    vsa.vsa_block_sparse_bwd(shape, tiled["q"], tiled["k"], tiled["v"], d_sel, k, offs, lists,
                             dev(lse.astype(np.float32)), to_dev_bf16(dof_bits), dev(delta),
                             dq, dk, dv)
    torch.cuda.synchronize()
    assert vsa.vsa_get_status() == 0
    check(bf16_dev_to_f64(dq), vo.untile(ref_q, grid), "dq")
    check(bf16_dev_to_f64(dk), vo.untile(ref_k, grid), "dk")
    check(bf16_dev_to_f64(dv), vo.untile(ref_v, grid), "dv")
    chosen = np.zeros((B, H, C), dtype=bool)
    for b in range(B):
        for h in range(H):
            chosen[b, h, np.unique(sel[b, h])] = True
    slot_token, _ = vo.cube_permutation(grid)
    got_k = bf16_dev_to_f64(dk)
    for b in range(B):
        for h in range(H):
            for c in np.flatnonzero(~chosen[b, h]):
                toks = slot_token[c, :int(counts[c])]
                assert np.all(got_k[b, h, toks] == 0)
