"""The head-sharded forward's exchanges (video_dit_block_vsa_b200/head_parallel.py)
on the CPU with gloo ranks: each rank holds a token shard of q, k, v (and the
gates), the all-to-all turns the shards into head shards, the oracle's VSA
forward runs on each head shard in place of the CUDA kernels, and the second
all-to-all returns the output shards.  Put back together, they must equal the
oracle's forward on the whole tensors: the exchanges move data only.  Uneven
token shards (N not a multiple of the ranks) are covered."""

import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CASES = {
    "tiny_gated": dict(B=1, H=2, d=64, grid=(4, 8, 8), topk=2, gated=True, seed=3),
    "ragged": dict(B=2, H=4, d=64, grid=(5, 7, 9), topk=3, gated=False, seed=4),
    "ragged_gated": dict(B=1, H=6, d=64, grid=(6, 5, 10), topk=4, gated=True, seed=5),
}


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(c):
    rng = np.random.default_rng(c["seed"])
    N = int(np.prod(c["grid"]))
    shp = (c["B"], c["H"], N, c["d"])
    q, k, v = (rng.standard_normal(shp) for _ in range(3))
    g = (rng.random((c["B"], c["H"], N)), rng.random((c["B"], c["H"], N))) if c["gated"] else (None, None)
    return q, k, v, g[0], g[1]


def _oracle_attention(batch, heads, d, grid, topk, q, k, v, g_f, g_c):
    import torch
    from oracle import vsa_oracle as vo
    n = lambda t: None if t is None else t.numpy()
    return torch.from_numpy(vo.vsa_forward(n(q), n(k), n(v), grid, topk, n(g_f), n(g_c))["out"])


def _rank_main(rank, world, port, name, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch
    from video_dit_block_vsa_b200 import dist as vdist
    from video_dit_block_vsa_b200 import head_parallel as hp
    info = vdist.init("gloo", timeout_s=60)
    c = CASES[name]
    q, k, v, g_f, g_c = _inputs(c)
    N = int(np.prod(c["grid"]))
    s, e = hp.token_shards(N, world)[rank]
    shard = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a[:, :, s:e]))
    o = hp.vsa_forward_head_parallel(c["grid"], c["topk"], shard(q), shard(k), shard(v),
                                     shard(g_f), shard(g_c), attention=_oracle_attention)
    out.put((rank, s, e, o.numpy()))
    vdist.shutdown(info)


@pytest.mark.parametrize("name,world", [("tiny_gated", 2), ("ragged", 2), ("ragged_gated", 3)])
def test_head_parallel_forward_equals_the_whole(name, world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, name, out)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted((out.get(timeout=180) for _ in range(world)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    sys.path.insert(0, ROOT)
    from oracle import vsa_oracle as vo
    c = CASES[name]
    q, k, v, g_f, g_c = _inputs(c)
    want = vo.vsa_forward(q, k, v, c["grid"], c["topk"], g_f, g_c)["out"]
    got = np.concatenate([o for _, _, _, o in results], axis=2)
    assert [r[1] for r in results] == sorted(r[1] for r in results)
    assert got.shape == want.shape
    assert np.allclose(got, want, rtol=0, atol=1e-12)


def test_token_shards_cover_the_sequence():
    sys.path.insert(0, ROOT)
    from video_dit_block_vsa_b200 import head_parallel as hp
    for n, w in ((315, 2), (256, 3), (7, 8), (75600, 8)):
        sh = hp.token_shards(n, w)
        assert sh[0][0] == 0 and sh[-1][1] == n
        assert all(a[1] == b[0] for a, b in zip(sh, sh[1:]))
        sizes = [e - s for s, e in sh]
        assert max(sizes) - min(sizes) <= 1


def test_heads_must_split_over_the_ranks():
    sys.path.insert(0, ROOT)
    import torch
    from video_dit_block_vsa_b200 import head_parallel as hp
    # one rank: no exchange, the attention runs on everything
    x = torch.zeros(1, 3, 256, 64, dtype=torch.float64)
    seen = {}

    def attn(batch, heads, d, grid, topk, q, k, v, g_f, g_c):
        seen["shape"] = tuple(q.shape)
        return q + 1

    o = hp.vsa_forward_head_parallel((4, 8, 8), 2, x, x, x, attention=attn)
    assert seen["shape"] == (1, 3, 256, 64) and torch.equal(o, x + 1)
