"""The head-sharded forward on one GPU (a world of one rank: no exchange): its
default attention is the CUDA path, so the output must be the fused forward's
bits.  The exchanges themselves are covered on the CPU with gloo ranks
(tests/test_head_parallel_cpu.py)."""

import pytest
import torch

from video_dit_block_vsa_b200 import workloads as wl
from tests.vsa_checks import to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vsa():
    from video_dit_block_vsa_b200 import build
    build.build()
    from video_dit_block_vsa_b200 import vsa as mod
    assert mod.vsa_get_status() == 0
    return mod


@pytest.mark.parametrize("name,heads", [("tiny_k2", None), ("wan1.3b_ft_16x28x52", 2)])
def test_one_rank_is_the_fused_forward(vsa, name, heads):
    from video_dit_block_vsa_b200 import head_parallel as hp
    w = wl.WORKLOADS[name]
    H = w.heads if heads is None else heads
    x = wl.make_inputs(w, heads=H)
    q, k, v = (to_dev_bf16(x[n]) for n in "qkv")
    g_f = torch.from_numpy(x["g_f"]).cuda() if w.gated else None
    g_c = torch.from_numpy(x["g_c"]).cuda() if w.gated else None
    shape = vsa.make_shape(w.batch, H, w.head_dim, w.grid)
    ref = torch.empty_like(q)
    vsa.vsa_forward_fused(shape, q, k, v, w.topk, ref, g_f, g_c)
    out = hp.vsa_forward_head_parallel(w.grid, w.topk, q, k, v, g_f, g_c)
    torch.cuda.synchronize()
    assert vsa.vsa_get_status() == 0
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
