"""vsa_coarse_select_noalloc: the coarse stage for callers that cannot
allocate device memory (for example a plugin inside an application that owns
every device allocation, or code that must not call cudaMalloc while work is
in flight).  It must give the same result as vsa_coarse_select, which takes a
caller-allocated workspace, and reject problems larger than its fixed scratch.

Called through the C ABI directly (ctypes on libvsa.so), twice in a row, and
compared with the workspace entry point: the selection must be identical and
the coarse output and logits equal within the coarse-stage tolerances of the
parity tests.  This file sorts last so that a run stopping at the first
failure has already run every other test; it also passes on its own in a
fresh process.
"""

import ctypes
import math

import numpy as np
import pytest
import torch

from video_dit_block_vsa_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vsa():
    from video_dit_block_vsa_b200 import build
    build.build()
    from video_dit_block_vsa_b200 import vsa as mod
    assert mod.vsa_get_status() == 0
    return mod


def _tiled_inputs(vsa, w):
    x = wl.make_inputs(w)
    shape = vsa.make_shape(w.batch, w.heads, w.head_dim, w.grid)
    bufs = vsa.VsaBuffers(shape, w.topk, want_coarse=True)
    to_dev = lambda b: torch.from_numpy(b.view(np.int16)).cuda().view(torch.bfloat16)
    vsa.vsa_tile_permute(shape, to_dev(x["q"]), bufs.q_t, bufs.counts)
    vsa.vsa_tile_permute(shape, to_dev(x["k"]), bufs.k_t)
    vsa.vsa_tile_permute(shape, to_dev(x["v"]), bufs.v_t)
    return shape, bufs


def _noalloc_call(vsa, shape, bufs, topk, sel, o_c, logits):
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return vsa._lib.vsa_coarse_select_noalloc(
        ctypes.byref(shape), p(bufs.q_t), p(bufs.k_t), p(bufs.v_t), p(bufs.counts), topk,
        p(o_c), p(sel), p(logits), stream)


@pytest.mark.parametrize("name", ["wan1.3b_480p_21x30x52", "tiny_k2"])
def test_noalloc_matches_workspace_entry_point_twice(vsa, name):
    w = wl.WORKLOADS[name]
    shape, bufs = _tiled_inputs(vsa, w)
    C = vsa.vsa_num_cubes(shape)
    B, H, d, k = w.batch, w.heads, w.head_dim, w.topk
    ref_logits = torch.empty(B, H, C, C, dtype=torch.float32, device="cuda")
    vsa.vsa_coarse_select(shape, bufs.q_t, bufs.k_t, bufs.v_t, bufs.counts, k, bufs.sel,
                          bufs.workspace, o_coarse=bufs.o_c, coarse_logits=ref_logits)
    torch.cuda.synchronize()
    for call in range(2):
        sel = torch.full_like(bufs.sel, -1)
        o_c = torch.full_like(bufs.o_c, float("nan"))
        logits = torch.full_like(ref_logits, float("nan"))
        rc = _noalloc_call(vsa, shape, bufs, k, sel, o_c, logits)
        assert rc == vsa.VSA_OK, vsa.vsa_strerror(rc)
        torch.cuda.synchronize()
        assert vsa.vsa_get_status() == 0
        assert torch.equal(sel, bufs.sel), f"call {call}: selection differs"
        assert torch.allclose(o_c, bufs.o_c, rtol=0, atol=1e-4), f"call {call}: coarse output"
        assert torch.allclose(logits, ref_logits, rtol=0, atol=2e-5), f"call {call}: logits"


def test_noalloc_rejects_problems_beyond_its_scratch(vsa):
    w = wl.WORKLOADS["wan14b_720p_21x45x80_k180"]  # 40 heads: 88 MB of pooled vectors
    shape = vsa.make_shape(w.batch, w.heads, w.head_dim, w.grid)
    assert 3 * w.batch * w.heads * w.cubes * w.head_dim * 4 > 32 << 20
    dummy = ctypes.c_void_p(0x10000)
    rc = vsa._lib.vsa_coarse_select_noalloc(ctypes.byref(shape), dummy, dummy, dummy, dummy,
                                            w.topk, None, dummy, None, None)
    assert rc == vsa.VSA_ERR_TOO_LARGE
    assert "scratch" in vsa.vsa_strerror(rc)
    assert vsa.vsa_get_status() == 0


def test_noalloc_under_a_second_context(vsa):
    """The entry point called while a second CUDA context, made with the driver
    API as a host application might, is current: the library looks up its
    scratch array and status word for that context, so the result equals the
    primary context's bit for bit, and the primary context still works after
    the second one is gone."""
    from cuda.bindings import driver as drv

    w = wl.WORKLOADS["tiny_k2"]
    shape, bufs = _tiled_inputs(vsa, w)
    C = vsa.vsa_num_cubes(shape)
    B, H, d, k = w.batch, w.heads, w.head_dim, w.topk
    sel_ref = torch.empty(B, H, C, k, dtype=torch.int32, device="cuda")
    oc_ref = torch.empty(B, H, C, d, dtype=torch.float32, device="cuda")
    lg_ref = torch.empty(B, H, C, C, dtype=torch.float32, device="cuda")
    assert _noalloc_call(vsa, shape, bufs, k, sel_ref, oc_ref, lg_ref) == 0
    torch.cuda.synchronize()
    host = [t.cpu().numpy() for t in (bufs.q_t.view(torch.int16), bufs.k_t.view(torch.int16),
                                      bufs.v_t.view(torch.int16), bufs.counts)]
    ok = drv.CUresult.CUDA_SUCCESS
    err, dev = drv.cuDeviceGet(torch.cuda.current_device())
    assert err == ok
    err, ctx = drv.cuCtxCreate(0, dev)
    assert err == ok
    try:
        ptrs = []

        def alloc(nbytes):
            e, p = drv.cuMemAlloc(nbytes)
            assert e == ok
            ptrs.append(p)
            return p

        dins = []
        for a in host:
            p = alloc(a.nbytes)
            assert drv.cuMemcpyHtoD(p, a, a.nbytes)[0] == ok
            dins.append(p)
        sel = np.empty((B, H, C, k), np.int32)
        oc = np.empty((B, H, C, d), np.float32)
        lg = np.empty((B, H, C, C), np.float32)
        sel_p, oc_p, lg_p = alloc(sel.nbytes), alloc(oc.nbytes), alloc(lg.nbytes)
        vp = lambda p: ctypes.c_void_p(int(p))
        rc = vsa._lib.vsa_coarse_select_noalloc(ctypes.byref(shape), vp(dins[0]), vp(dins[1]),
                                                vp(dins[2]), vp(dins[3]), k, vp(oc_p), vp(sel_p),
                                                vp(lg_p), None)
        assert rc == 0
        assert drv.cuCtxSynchronize()[0] == ok
        assert vsa._lib.vsa_get_status(None) == 0
        for a, p in ((sel, sel_p), (oc, oc_p), (lg, lg_p)):
            assert drv.cuMemcpyDtoH(a, p, a.nbytes)[0] == ok
        for p in ptrs:
            assert drv.cuMemFree(p)[0] == ok
    finally:
        drv.cuCtxPopCurrent()
        drv.cuCtxDestroy(ctx)
    assert np.array_equal(sel, sel_ref.cpu().numpy())
    assert np.array_equal(oc, oc_ref.cpu().numpy())
    assert np.array_equal(lg, lg_ref.cpu().numpy())
    # back in the primary context
    sel2 = torch.empty_like(sel_ref)
    assert _noalloc_call(vsa, shape, bufs, k, sel2, torch.empty_like(oc_ref), torch.empty_like(lg_ref)) == 0
    torch.cuda.synchronize()
    assert vsa.vsa_get_status() == 0
    assert torch.equal(sel2, sel_ref)
