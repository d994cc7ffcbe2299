"""The Python binding's marshalling, on a host without a GPU.

The library's compute calls are replaced by a recorder that checks each call
against the argument count its ctypes signature declares and returns VSA_OK;
the host-only helpers (cube count, workspace sizes) stay real.  Tensors are
CPU tensors with the device checks bypassed, so the composed calls (the
forward convenience and the four-call backward) can be followed argument by
argument: which buffer each call reads and writes, in which order."""

import ctypes

import pytest
import torch

from video_dit_block_vsa_b200 import build

build.build()
from video_dit_block_vsa_b200 import vsa as V  # noqa: E402

HOST_ONLY = {"vsa_num_cubes", "vsa_topk_from_ratio", "vsa_workspace_bytes",
             "vsa_forward_host_workspace_bytes", "vsa_coarse_backward_workspace_bytes",
             "vsa_linear_workspace_bytes", "vsa_strerror"}


class Recorder:
    def __init__(self, real):
        self.real = real
        self.calls = []

    def __getattr__(self, name):
        if name in HOST_ONLY:
            return getattr(self.real, name)
        nargs = len(V._sig[name][1])

        def call(*args):
            assert len(args) == nargs, f"{name}: {len(args)} arguments, signature has {nargs}"
            self.calls.append((name, args))
            return V.VSA_OK
        return call

    def names(self):
        return [n for n, _ in self.calls]


@pytest.fixture
def lib(monkeypatch):
    rec = Recorder(V._lib)
    monkeypatch.setattr(V, "_lib", rec)
    monkeypatch.setattr(V, "_stream", lambda s: ctypes.c_void_p(0))

    def expect(t, dtype, shape, name):  # dtype and shape, not the device
        assert t.dtype == dtype, (name, t.dtype, dtype)
        assert tuple(t.shape) == tuple(shape), (name, tuple(t.shape), tuple(shape))
    monkeypatch.setattr(V, "_expect", expect)
    monkeypatch.setattr(V, "_expect_device", lambda t, name: None)
    return rec


def addr(a):
    return None if a is None else a.value


def ptr(t):
    return t.data_ptr()


def setup(gated):
    shape = V.make_shape(1, 2, 64, (4, 8, 8))
    B, H, N, d, topk = 1, 2, 256, 64, 2
    bf = dict(dtype=torch.bfloat16)
    q, k, v, out, dout = (torch.zeros(B, H, N, d, **bf) for _ in range(5))
    g_f = torch.zeros(B, H, N) if gated else None
    g_c = torch.zeros(B, H, N) if gated else None
    bufs = V.VsaBuffers(shape, topk, device="cpu", want_coarse=gated, want_lse=True)
    return shape, topk, (q, k, v, out, dout, g_f, g_c), bufs


def test_forward_calls_in_order(lib):
    shape, topk, (q, k, v, out, _, g_f, g_c), bufs = setup(gated=True)
    V.vsa_forward(shape, q, k, v, topk, out, g_f, g_c, bufs=bufs)
    assert lib.names() == ["vsa_tile_permute"] * 3 + ["vsa_coarse_select", "vsa_block_sparse_fwd",
                                                      "vsa_combine", "vsa_untile"]
    fwd = lib.calls[4][1]
    # (shape, q_t, k_t, v_t, counts, sel, k, o_f, lse, stream)
    assert addr(fwd[7]) == ptr(bufs.o_f) and addr(fwd[8]) == ptr(bufs.lse)


@pytest.mark.parametrize("gated", [True, False])
def test_backward_wiring(lib, gated):
    shape, topk, (q, k, v, out, dout, g_f, g_c), bufs = setup(gated)
    B, H, N, d = 1, 2, 256, 64
    dq, dk, dv = (torch.zeros(B, H, N, d, dtype=torch.bfloat16) for _ in range(3))
    dgf = torch.zeros(B, H, N) if gated else None
    dgc = torch.zeros(B, H, N) if gated else None
    grads = V.VsaGradBuffers(shape, topk, gated, device="cpu")
    V.vsa_backward(shape, bufs, dout, dq, dk, dv, g_f, g_c, dgf, dgc, grads=grads)
    expect = ["vsa_backward_prep"] + (["vsa_coarse_backward"] if gated else []) + \
             ["vsa_select_transpose", "vsa_block_sparse_bwd"]
    assert lib.names() == expect
    calls = dict(lib.calls)

    # prep: (shape, dout, o_f, o_c, g_f, g_c, do_f, delta, do_c, dg_f, dg_c, stream)
    a = calls["vsa_backward_prep"]
    assert addr(a[1]) == ptr(dout) and addr(a[2]) == ptr(bufs.o_f)
    assert addr(a[6]) == ptr(grads.do_f) and addr(a[7]) == ptr(grads.delta)
    if gated:
        assert addr(a[3]) == ptr(bufs.o_c) and addr(a[4]) == ptr(g_f) and addr(a[5]) == ptr(g_c)
        assert addr(a[8]) == ptr(grads.do_c) and addr(a[9]) == ptr(dgf) and addr(a[10]) == ptr(dgc)
        # coarse: (shape, pooled, o_c, do_c, d_pooled, workspace, bytes, stream); the pooled
        # means are the first bytes of the forward's workspace
        c = calls["vsa_coarse_backward"]
        assert addr(c[1]) == ptr(bufs.workspace) and addr(c[2]) == ptr(bufs.o_c)
        assert addr(c[3]) == ptr(grads.do_c) and addr(c[4]) == ptr(grads.d_pooled)
        assert addr(c[5]) == ptr(grads.coarse_ws) and c[6] == grads.coarse_ws.numel()
    else:
        assert all(addr(a[i]) is None for i in (3, 4, 5, 8, 9, 10))
    # transpose: (shape, sel, k, offsets, lists, workspace, bytes, stream)
    t = calls["vsa_select_transpose"]
    assert addr(t[1]) == ptr(bufs.sel) and t[2] == topk
    assert addr(t[3]) == ptr(grads.key_offsets) and addr(t[4]) == ptr(grads.query_lists)
    assert addr(t[5]) == ptr(grads.transpose_ws)
    # fine: (shape, q_t, k_t, v_t, sel, k, offsets, lists, lse, do_f, delta, d_pooled, dq, dk, dv, stream)
    f = calls["vsa_block_sparse_bwd"]
    assert [addr(f[i]) for i in (1, 2, 3, 4)] == [ptr(bufs.q_t), ptr(bufs.k_t), ptr(bufs.v_t),
                                                   ptr(bufs.sel)]
    assert f[5] == topk
    assert addr(f[6]) == ptr(grads.key_offsets) and addr(f[7]) == ptr(grads.query_lists)
    assert addr(f[8]) == ptr(bufs.lse) and addr(f[9]) == ptr(grads.do_f)
    assert addr(f[10]) == ptr(grads.delta)
    assert addr(f[11]) == (ptr(grads.d_pooled) if gated else None)
    assert [addr(f[i]) for i in (12, 13, 14)] == [ptr(dq), ptr(dk), ptr(dv)]


def test_backward_needs_the_forward_lse(lib):
    shape, topk, (q, k, v, out, dout, g_f, g_c), _ = setup(gated=False)
    bufs = V.VsaBuffers(shape, topk, device="cpu", want_coarse=False, want_lse=False)
    dq, dk, dv = (torch.zeros_like(q) for _ in range(3))
    with pytest.raises(ValueError, match="LSE"):
        V.vsa_backward(shape, bufs, dout, dq, dk, dv)
    assert lib.calls == []


def test_device_buffers_are_checked():
    # unpatched: a host tensor where a device buffer belongs is refused in
    # Python, before any pointer reaches the library
    with pytest.raises(ValueError, match="CUDA"):
        V._expect_device(torch.zeros(16, dtype=torch.uint8), "workspace")
    with pytest.raises(ValueError, match="CUDA"):
        V._expect(torch.zeros(4, dtype=torch.int32), torch.int32, (4,), "cube_count")
    with pytest.raises(ValueError, match="contiguous"):
        V._ptr(torch.zeros(4, 4).t())


@pytest.mark.parametrize("gated", [True, False])
def test_attention_block_wiring(lib, gated):
    """QKV projection into the tiled buffers, coarse stage and fine stage on
    them, the combine when gated, and the output projection reading the tiled
    attention output (the combined one when gated)."""
    shape, topk, (_, _, _, _, _, g_f, g_c), bufs = setup(gated)
    hidden = 128
    x = torch.zeros(1, 256, hidden, dtype=torch.bfloat16)
    w_qkv = torch.zeros(3 * 2 * 64, hidden, dtype=torch.bfloat16)
    w_o = torch.zeros(hidden, 2 * 64, dtype=torch.bfloat16)
    y = torch.zeros(1, 256, hidden, dtype=torch.bfloat16)
    V.vsa_attention_block(shape, hidden, x, w_qkv, w_o, topk, y, g_f, g_c, bufs=bufs)
    expect = ["vsa_qkv_projection_tiled", "vsa_coarse_select", "vsa_block_sparse_fwd"] + \
             (["vsa_combine"] if gated else []) + ["vsa_out_projection_tiled"]
    assert lib.names() == expect
    calls = dict(lib.calls)
    qkv = calls["vsa_qkv_projection_tiled"]  # (shape, hidden, x, w, q_t, k_t, v_t, counts, stream)
    assert qkv[1] == hidden
    assert [addr(a) for a in qkv[4:8]] == [ptr(bufs.q_t), ptr(bufs.k_t), ptr(bufs.v_t), ptr(bufs.counts)]
    outp = calls["vsa_out_projection_tiled"]  # (shape, hidden, o_t, w_o, y, stream)
    assert addr(outp[2]) == ptr(bufs.out_t if gated else bufs.o_f)
    assert addr(outp[4]) == ptr(y)


def test_linear_branch_marshalling(lib):
    shape, _, (q, k, v, out, _, _, _), _ = setup(False)
    ws = torch.zeros(V.vsa_linear_workspace_bytes(shape), dtype=torch.uint8)
    V.vsa_linear_branch_add(shape, q, k, v, out, ws)
    (name, args), = lib.calls
    assert name == "vsa_linear_branch_add"
    assert [addr(a) for a in args[1:6]] == [ptr(q), ptr(k), ptr(v), ptr(out), ptr(ws)]
    assert args[6] == ws.numel()


def test_head_parallel_one_rank_runs_the_fused_forward(lib):
    from video_dit_block_vsa_b200 import head_parallel as hp
    _, topk, (q, k, v, _, _, g_f, g_c), _ = setup(True)
    hp.vsa_forward_head_parallel((4, 8, 8), topk, q, k, v, g_f, g_c)
    assert lib.names() == ["vsa_tile_permute_pool", "vsa_coarse_select_pooled",
                           "vsa_block_sparse_fwd_out"]

