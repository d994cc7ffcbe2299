"""vsa_coarse_backward (gradient of the coarse attention w.r.t. the pooled
vectors) against the oracle's coarse_attention_backward.

Inputs come from the seeded generator and the oracle: qbar, kbar, vbar are the
oracle's cube means of the workload's q, k, v rounded to float32, O_c the
oracle's coarse output from them, dO_c a seeded normal draw.  The kernel works
in float32 with sums over up to C terms, so the bound is relative to each
gradient's largest magnitude (a wrong index or a dropped term is O(1) off).
One more case feeds the forward's own workspace (through pooled_view) and
coarse output to the call, to check that the layouts compose."""

import numpy as np
import pytest
import torch

from oracle import vsa_backward as vb
from oracle import vsa_oracle as vo
from video_dit_block_vsa_b200 import workloads as wl
from tests.vsa_checks import to_dev_bf16

pytestmark = pytest.mark.gpu

MAX_REL = 1e-4   # max |got - ref| / max |ref|, per gradient
MEAN_REL = 1e-5  # mean |got - ref| / max |ref|


@pytest.fixture(scope="module")
def vsa():
    from video_dit_block_vsa_b200 import build
    build.build()
    from video_dit_block_vsa_b200 import vsa as mod
    assert mod.vsa_get_status() == 0
    return mod


def oracle_pooled(w, heads):
    x = wl.make_inputs(w, heads=heads)
    out = []
    for n in ("q", "k", "v"):
        t, counts = vo.tile_permute(vo.bf16_bits_to_f64(x[n]), w.grid)
        out.append(vo.pool(t, counts))
    return x, out


def check(got, refs, what):
    for name, g, r in zip(("dqbar", "dkbar", "dvbar"), got, refs):
        assert np.all(np.isfinite(g)), f"{what} {name}: non-finite values"
        m = np.abs(r).max()
        e = np.abs(g - r)
        assert e.max() <= MAX_REL * m, f"{what} {name}: max err {e.max():.3e} vs max |ref| {m:.3e}"
        assert e.mean() <= MEAN_REL * m, f"{what} {name}: mean err {e.mean():.3e}"


CASES = [  # (workload, heads, one plane of workspace)
    (wl.WORKLOADS["tiny_k2"], 2, None),                                        # C = 4, d = 64
    (wl.Workload("ragged_d64", 2, 2, 64, (16, 36, 36), 8, 31, 0.5, False), None, True),  # C = 324
    (wl.Workload("odd_c27", 1, 3, 128, (9, 10, 11), 5, 32, 0.5, False), None, None),  # C = 27
    (wl.WORKLOADS["wan1.3b_ft_16x28x52"], 2, None),                            # C = 364, d = 128
    (wl.WORKLOADS["wan14b_720p_21x45x80_k180"], 2, True),                      # C = 1440
]


@pytest.mark.parametrize("w,heads,chunked", CASES,
                         ids=[c[0].name + ("-chunked" if c[2] else "") for c in CASES])
def test_coarse_backward_matches_oracle(vsa, w, heads, chunked):
    H = w.heads if heads is None else heads
    B, d = w.batch, w.head_dim
    _, pooled = oracle_pooled(w, H)
    p32 = [p.astype(np.float32) for p in pooled]
    p64 = [p.astype(np.float64) for p in p32]
    C = p32[0].shape[2]
    _, oc = vo.coarse_attention(*p64)
    oc32 = oc.astype(np.float32)
    rng = np.random.default_rng(w.seed + 200)
    doc32 = rng.standard_normal((B, H, C, d), dtype=np.float32)
    refs = vb.coarse_attention_backward(*p64, doc32.astype(np.float64))

    shape = vsa.make_shape(B, H, d, w.grid)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    d_pooled = torch.full((3, B, H, C, d), float("nan"), dtype=torch.float32, device="cuda")
    full = vsa.vsa_coarse_backward_workspace_bytes(shape)
    # the whole workspace, or one plane's share (the planes then run in chunks)
    ws = torch.empty(full if chunked is None else full // (B * H), dtype=torch.uint8, device="cuda")
    vsa.vsa_coarse_backward(shape, dev(np.stack(p32)), dev(oc32), dev(doc32), d_pooled, ws)
    torch.cuda.synchronize()
    assert vsa.vsa_get_status() == 0
    check(d_pooled.cpu().numpy(), refs, w.name)


def test_coarse_backward_on_the_forward_workspace(vsa):
    w = wl.WORKLOADS["wan1.3b_480p_21x30x52"]  # ragged grid, C = 624
    H, B, d = 2, w.batch, w.head_dim
    x, pooled = oracle_pooled(w, H)
    C = pooled[0].shape[2]
    refs_rng = np.random.default_rng(w.seed + 300)
    doc32 = refs_rng.standard_normal((B, H, C, d), dtype=np.float32)
    refs = vb.coarse_attention_backward(*pooled, doc32.astype(np.float64))

    shape = vsa.make_shape(B, H, d, w.grid)
    bufs = vsa.VsaBuffers(shape, w.topk)
    q, k, v = (to_dev_bf16(x[n]) for n in ("q", "k", "v"))
    vsa.vsa_tile_permute_pool(shape, q, k, v, bufs.q_t, bufs.k_t, bufs.v_t, bufs.workspace,
                              bufs.counts)
    vsa.vsa_coarse_select_pooled(shape, w.topk, bufs.sel, bufs.workspace, o_coarse=bufs.o_c)
    d_pooled = torch.full((3, B, H, C, d), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(vsa.vsa_coarse_backward_workspace_bytes(shape), dtype=torch.uint8, device="cuda")
    vsa.vsa_coarse_backward(shape, vsa.pooled_view(shape, bufs.workspace), bufs.o_c,
                            torch.from_numpy(doc32).cuda(), d_pooled, ws)
    torch.cuda.synchronize()
    assert vsa.vsa_get_status() == 0
    check(d_pooled.cpu().numpy(), refs, "forward workspace")
