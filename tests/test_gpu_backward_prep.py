"""vsa_backward_prep (gradient of the gated combine, first pass of a backward)
against the oracle's combine_backward on the same bf16 inputs (the forward's
O_f and O_c taken from the oracle): the fine-branch
gradient within bf16 rounding, the float32 row sums, gate gradients and the
coarse-branch gradient within float32 accumulation, pad rows exactly zero."""

import numpy as np
import pytest
import torch

from oracle import vsa_backward as vb
from oracle import vsa_oracle as vo
from video_dit_block_vsa_b200 import workloads as wl
from tests.vsa_checks import bf16_dev_to_f64, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vsa():
    from video_dit_block_vsa_b200 import build
    build.build()
    from video_dit_block_vsa_b200 import vsa as mod
    assert mod.vsa_get_status() == 0
    return mod


CASES = [wl.WORKLOADS["tiny_k2"], wl.Workload("ragged_gated", 2, 2, 128, (5, 7, 9), 3, 21, 0.5, True),
         wl.Workload("ragged_ungated", 1, 2, 64, (6, 5, 10), 4, 22, 0.5, False)]


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_backward_prep_matches_combine_backward(vsa, w):
    x = wl.make_inputs(w)
    shape = vsa.make_shape(w.batch, w.heads, w.head_dim, w.grid)
    B, H, N, d, C = w.batch, w.heads, w.tokens, w.head_dim, w.cubes
    # the forward's O_f and O_c come from the oracle (rounded to the types the
    # kernel reads), so no input of the check is produced by the CUDA path
    f64 = lambda n: vo.bf16_bits_to_f64(x[n])
    q_t, counts = vo.tile_permute(f64("q"), w.grid)
    k_t, _ = vo.tile_permute(f64("k"), w.grid)
    v_t, _ = vo.tile_permute(f64("v"), w.grid)
    S_c, oc_ref = vo.coarse_attention(vo.pool(q_t, counts), vo.pool(k_t, counts), vo.pool(v_t, counts))
    of_ref, _ = vo.block_sparse_attention(q_t, k_t, v_t, counts, vo.topk_select(S_c, w.topk))
    of_bits = wl.f32_to_bf16_bits(of_ref.astype(np.float32))
    o_f = to_dev_bf16(of_bits)
    oc32 = oc_ref.astype(np.float32)
    o_c = torch.from_numpy(oc32).cuda() if w.gated else None
    g_f = torch.from_numpy(x["g_f"]).cuda() if w.gated else None
    g_c = torch.from_numpy(x["g_c"]).cuda() if w.gated else None
    rng = np.random.default_rng(w.seed + 100)
    dout_bits = wl.f32_to_bf16_bits(rng.standard_normal((B, H, N, d), dtype=np.float32))
    dout = to_dev_bf16(dout_bits)
    dof = torch.full_like(o_f, 5.0)
    delta = torch.full((B, H, 64 * C), 5.0, dtype=torch.float32, device="cuda")
    doc = torch.empty(B, H, C, d, dtype=torch.float32, device="cuda") if w.gated else None
    dgf = torch.empty(B, H, N, dtype=torch.float32, device="cuda") if w.gated else None
    dgc = torch.empty_like(dgf) if w.gated else None
    vsa.vsa_backward_prep(shape, dout, o_f, dof, delta, o_c, g_f, g_c, doc, dgf, dgc)
    torch.cuda.synchronize()
    assert vsa.vsa_get_status() == 0

    of = vo.bf16_bits_to_f64(of_bits)
    oc = oc32.astype(np.float64) if w.gated else np.zeros((B, H, C, d))
    dout64 = vo.bf16_bits_to_f64(dout_bits)
    dout_t, _ = vo.tile_permute(dout64, w.grid)
    gf64 = x["g_f"].astype(np.float64) if w.gated else None
    gc64 = x["g_c"].astype(np.float64) if w.gated else None
    dof_ref, doc_ref, dgf_ref, dgc_ref = vb.combine_backward(dout_t, of, oc, counts, w.grid, gf64, gc64)

    got_dof = bf16_dev_to_f64(dof)
    assert np.all(np.abs(got_dof - dof_ref) <= np.abs(dof_ref) * 2.0 ** -8 + 1e-30)
    valid = np.zeros(64 * C, dtype=bool)
    for c in range(C):
        valid[64 * c:64 * c + int(counts[c])] = True
    assert np.all(got_dof[:, :, ~valid] == 0)
    got_delta = delta.cpu().numpy()
    ref_delta = np.sum(got_dof * of, axis=-1)  # D is formed from the bf16 gradient the kernel wrote
    tol = 1e-5 * np.sum(np.abs(got_dof * of), axis=-1) + 1e-6
    assert np.all(np.abs(got_delta - ref_delta) <= tol)
    assert np.all(got_delta[:, :, ~valid] == 0)
    if w.gated:
        prod = np.abs(dout64)
        tol_gf = 1e-5 * np.sum(prod * np.abs(vo.untile(of, w.grid)), axis=-1) + 1e-6
        assert np.all(np.abs(dgf.cpu().numpy() - dgf_ref) <= tol_gf)
        assert np.all(np.abs(dgc.cpu().numpy() - dgc_ref) <= 1e-5 * np.abs(dgc_ref) + 1e-4)
        np.testing.assert_allclose(doc.cpu().numpy(), doc_ref, rtol=1e-5, atol=1e-5)
