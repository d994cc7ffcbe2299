"""vsa_select_transpose against the oracle's selection transpose, bit for bit
(integer work): random ascending selections, the oracle's coarse-stage
selection on a ragged workload, every cube selected, and one key cube selected by all."""

import numpy as np
import pytest
import torch

from oracle import vsa_backward as vb
from oracle import vsa_oracle as vo
from video_dit_block_vsa_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vsa():
    from video_dit_block_vsa_b200 import build
    build.build()
    from video_dit_block_vsa_b200 import vsa as mod
    assert mod.vsa_get_status() == 0
    return mod


def run(vsa, shape, sel):
    B, H, C, k = sel.shape
    d_sel = torch.from_numpy(sel.astype(np.int32)).cuda()
    offs = torch.full((B, H, C + 1), -1, dtype=torch.int32, device="cuda")
    lists = torch.full((B, H, C * k), -1, dtype=torch.int32, device="cuda")
    ws = torch.empty(B * H * C * k * 4 + 256, dtype=torch.uint8, device="cuda")
    vsa.vsa_select_transpose(shape, d_sel, k, offs, lists, ws)
    torch.cuda.synchronize()
    assert vsa.vsa_get_status() == 0
    want_offs, want_lists = vb.select_transpose(sel, C)
    assert np.array_equal(offs.cpu().numpy(), want_offs)
    assert np.array_equal(lists.cpu().numpy(), want_lists)


@pytest.mark.parametrize("B,H,grid,k", [(2, 3, (5, 7, 9), 4), (1, 2, (21, 30, 52), 62),
                                         (1, 1, (4, 8, 8), 4), (1, 1, (1, 1, 1), 1)])
def test_random_selections(vsa, B, H, grid, k):
    shape = vsa.make_shape(B, H, 64, grid)
    C = vsa.vsa_num_cubes(shape)
    rng = np.random.default_rng(C + k)
    sel = np.stack([np.sort(rng.choice(C, k, replace=False)) for _ in range(B * H * C)])
    run(vsa, shape, sel.reshape(B, H, C, k))


def test_one_key_cube_chosen_by_every_query(vsa):
    B, H, grid, k = 1, 2, (8, 12, 16), 3
    shape = vsa.make_shape(B, H, 64, grid)
    C = vsa.vsa_num_cubes(shape)
    sel = np.tile(np.array([0, C // 2, C - 1]), (B, H, C, 1))
    run(vsa, shape, sel)


def test_coarse_stage_selection(vsa):
    """A selection with the structure the coarse stage gives (the oracle's own
    top-k on a ragged 480p grid): the lists' lengths spread unevenly."""
    w = wl.WORKLOADS["wan1.3b_480p_21x30x52"]
    x = wl.make_inputs(w, heads=2)
    shape = vsa.make_shape(w.batch, 2, w.head_dim, w.grid)
    pooled = []
    for n in ("q", "k", "v"):
        t, counts = vo.tile_permute(vo.bf16_bits_to_f64(x[n]), w.grid)
        pooled.append(vo.pool(t, counts))
    S_c, _ = vo.coarse_attention(*pooled)
    run(vsa, shape, vo.topk_select(S_c, w.topk))
