"""vsa_forward_host: the whole path from host buffers, processed in chunks of
(b, h) planes with the copies overlapping the kernels.  Each chunk runs the
same kernels as the device-buffer path, so the output must equal that path's
bit for bit (the device path itself is checked against the oracle in
test_gpu_parity.py); chunk sizes that do not divide B*H, and chunks that
cross a batch boundary, are covered.  The device-buffer path is also replayed
from a captured CUDA graph."""

import numpy as np
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


def host_bf16(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).pin_memory()


def device_path(vsa, w, x, shape):
    q, k, v = (to_dev_bf16(x[n]) for n in ("q", "k", "v"))
    g_f = torch.from_numpy(x["g_f"]).cuda() if w.gated else None
    g_c = torch.from_numpy(x["g_c"]).cuda() if w.gated else None
    out = torch.empty_like(q)
    vsa.vsa_forward(shape, q, k, v, w.topk, out, g_f, g_c)
    torch.cuda.synchronize()
    assert vsa.vsa_get_status() == 0
    return out.cpu()


def host_path(vsa, w, x, shape, heads_per_chunk, repeats=1):
    hq, hk, hv = (host_bf16(x[n]) for n in ("q", "k", "v"))
    hgf = torch.from_numpy(x["g_f"]).pin_memory() if w.gated else None
    hgc = torch.from_numpy(x["g_c"]).pin_memory() if w.gated else None
    hout = torch.empty(hq.shape, dtype=torch.bfloat16).pin_memory()
    nbytes = vsa.vsa_forward_host_workspace_bytes(shape, w.topk, heads_per_chunk, w.gated)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(repeats):
        hout.fill_(0)
        vsa.vsa_forward_host(shape, w.topk, hq, hk, hv, hout, ws, hgf, hgc, heads_per_chunk)
        torch.cuda.synchronize()
        assert vsa.vsa_get_status() == 0
        outs.append(hout.clone())
    return outs


CASES = [
    (wl.WORKLOADS["tiny_k2"], 1),                # 2 planes, one per chunk
    (wl.WORKLOADS["wan1.3b_ft_16x28x52"], 5),    # gated, 12 planes: chunks 5, 5, 2
    (wl.WORKLOADS["scaling_16x32x32"], 0),       # ungated, default chunk of 2: six chunks
    (wl.Workload("b2_ragged", 2, 3, 64, (5, 7, 9), 3, 11, 0.5, True), 4),  # chunk crosses b
    (wl.Workload("b3_one_chunk", 3, 1, 128, (6, 6, 10), 4, 12, 0.5, False), 16),
]


@pytest.mark.parametrize("w,heads_per_chunk", CASES, ids=[c[0].name for c in CASES])
def test_host_path_equals_device_path(vsa, w, heads_per_chunk):
    x = wl.make_inputs(w)
    shape = vsa.make_shape(w.batch, w.heads, w.head_dim, w.grid)
    want = device_path(vsa, w, x, shape).view(torch.int16)
    got = host_path(vsa, w, x, shape, heads_per_chunk)[0].view(torch.int16)
    assert torch.equal(got, want)


def test_host_path_reuses_its_workspace(vsa):
    w = wl.WORKLOADS["wan1.3b_ft_16x28x52"]
    x = wl.make_inputs(w)
    shape = vsa.make_shape(w.batch, w.heads, w.head_dim, w.grid)
    a, b = host_path(vsa, w, x, shape, 4, repeats=2)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_device_path_replays_from_a_cuda_graph(vsa):
    # after one eager call the path only launches kernels, so a stream capture
    # of it replays to the same bits
    w = wl.WORKLOADS["wan1.3b_ft_16x28x52"]
    x = wl.make_inputs(w)
    shape = vsa.make_shape(w.batch, w.heads, w.head_dim, w.grid)
    q, k, v = (to_dev_bf16(x[n]) for n in ("q", "k", "v"))
    g_f = torch.from_numpy(x["g_f"]).cuda()
    g_c = torch.from_numpy(x["g_c"]).cuda()
    out_eager = torch.empty_like(q)
    bufs = vsa.vsa_forward(shape, q, k, v, w.topk, out_eager, g_f, g_c)
    torch.cuda.synchronize()
    out_graph = torch.zeros_like(q)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            vsa.vsa_forward(shape, q, k, v, w.topk, out_graph, g_f, g_c, bufs=bufs)
    for _ in range(2):
        out_graph.zero_()
        graph.replay()
    torch.cuda.synchronize()
    assert vsa.vsa_get_status() == 0
    assert torch.equal(out_graph.view(torch.int16), out_eager.view(torch.int16))
    del graph
