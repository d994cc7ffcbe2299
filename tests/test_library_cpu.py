"""libvsa on a machine without a GPU: the library builds, loads, exports every
symbol include/vsa.h declares, and its host-only helpers and argument checks
work (no call here launches GPU work)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "vsa.h")


@pytest.fixture(scope="module")
def vsa():
    from video_dit_block_vsa_b200 import build
    build.build()
    from video_dit_block_vsa_b200 import vsa as mod
    return mod


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:int|size_t|const char\*)\s+(vsa_\w+)\s*\(", text, re.M)))


def test_header_declares_the_path():
    names = declared_functions()
    for n in ("vsa_tile_permute", "vsa_coarse_select", "vsa_block_sparse_fwd", "vsa_combine",
              "vsa_untile"):
        assert n in names


def test_library_exports_every_declared_symbol(vsa):
    lib = ctypes.CDLL(vsa._LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), n
    assert set(declared_functions()) == set(vsa.EXPORTED)


def test_num_cubes_and_ratio(vsa):
    s = vsa.make_shape(1, 40, 128, (21, 45, 80))
    assert vsa.vsa_num_cubes(s) == 1440
    assert vsa.vsa_num_cubes(vsa.make_shape(1, 12, 128, (21, 30, 52))) == 624
    assert vsa.vsa_topk_from_ratio(624, 0.1) == 62
    assert vsa.vsa_topk_from_ratio(1440, 0.125) == 180
    assert vsa.vsa_topk_from_ratio(1440, 0.03) == 43
    assert vsa.vsa_topk_from_ratio(1440, 1.0) == 1440
    with pytest.raises(vsa.VsaError):
        vsa.vsa_topk_from_ratio(1440, 0.0)
    with pytest.raises(vsa.VsaError):
        vsa.vsa_topk_from_ratio(0, 0.5)


def test_workspace_bytes(vsa):
    s = vsa.make_shape(1, 40, 128, (21, 45, 80))
    assert vsa.vsa_workspace_bytes(s, 180) == 3 * 40 * 1440 * 128 * 4
    assert vsa.vsa_workspace_bytes(s, 0) == 0
    assert vsa.vsa_workspace_bytes(s, 1441) == 0


def test_unsupported_shapes_rejected_before_launch(vsa):
    lib = vsa._lib
    c = ctypes.c_int()
    bad_cube = vsa.VsaShape(1, 1, 128, 8, 8, 8, 2, 4, 4)
    assert lib.vsa_num_cubes(ctypes.byref(bad_cube), ctypes.byref(c)) == vsa.VSA_ERR_UNSUPPORTED
    bad_d = vsa.make_shape(1, 1, 96, (8, 8, 8))
    assert lib.vsa_num_cubes(ctypes.byref(bad_d), ctypes.byref(c)) == vsa.VSA_ERR_UNSUPPORTED
    bad_b = vsa.make_shape(0, 1, 128, (8, 8, 8))
    assert lib.vsa_num_cubes(ctypes.byref(bad_b), ctypes.byref(c)) == vsa.VSA_ERR_INVALID_ARG
    assert lib.vsa_num_cubes(None, ctypes.byref(c)) == vsa.VSA_ERR_INVALID_ARG
    # the most cubes a coarse row holds: 8192 accepted, more rejected
    at_max = vsa.make_shape(1, 1, 64, (32, 128, 128))
    assert lib.vsa_num_cubes(ctypes.byref(at_max), ctypes.byref(c)) == 0 and c.value == 8192
    too_many = vsa.make_shape(1, 1, 64, (36, 128, 128))
    assert lib.vsa_num_cubes(ctypes.byref(too_many), ctypes.byref(c)) == vsa.VSA_ERR_UNSUPPORTED


def test_null_and_misaligned_pointers_rejected_before_launch(vsa):
    lib = vsa._lib
    s = vsa.make_shape(1, 2, 64, (4, 8, 8))
    p = ctypes.c_void_p(0x1000)
    odd = ctypes.c_void_p(0x1008)
    assert lib.vsa_tile_permute(ctypes.byref(s), None, p, None, None) == vsa.VSA_ERR_INVALID_ARG
    assert lib.vsa_tile_permute(ctypes.byref(s), odd, p, None, None) == vsa.VSA_ERR_INVALID_ARG
    assert lib.vsa_untile(ctypes.byref(s), p, None, None) == vsa.VSA_ERR_INVALID_ARG
    # k outside [1, C]
    assert lib.vsa_block_sparse_fwd(ctypes.byref(s), p, p, p, p, p, 0, p, None, None) == vsa.VSA_ERR_INVALID_ARG
    assert lib.vsa_block_sparse_fwd(ctypes.byref(s), p, p, p, p, p, 5, p, None, None) == vsa.VSA_ERR_INVALID_ARG
    assert lib.vsa_coarse_select(ctypes.byref(s), p, p, p, p, 5, None, p, None, p, 1 << 20, None) == vsa.VSA_ERR_INVALID_ARG
    # workspace too small
    assert lib.vsa_coarse_select(ctypes.byref(s), p, p, p, p, 2, None, p, None, p, 16, None) == vsa.VSA_ERR_INVALID_ARG
    # one gate without the other
    assert lib.vsa_combine(ctypes.byref(s), p, p, p, None, p, None) == vsa.VSA_ERR_INVALID_ARG
    # token-order coarse stage: k out of range, missing output, small or misaligned workspace
    tok = lib.vsa_coarse_select_tokens
    assert tok(ctypes.byref(s), p, p, p, 5, None, p, None, p, 1 << 20, None) == vsa.VSA_ERR_INVALID_ARG
    assert tok(ctypes.byref(s), p, p, p, 2, None, None, None, p, 1 << 20, None) == vsa.VSA_ERR_INVALID_ARG
    assert tok(ctypes.byref(s), p, p, p, 2, None, p, None, p, 16, None) == vsa.VSA_ERR_INVALID_ARG
    assert tok(ctypes.byref(s), odd, p, p, 2, None, p, None, p, 1 << 20, None) == vsa.VSA_ERR_INVALID_ARG
    # fused tiling + pooling, and the coarse stage from pooled means
    tp = lib.vsa_tile_permute_pool
    assert tp(ctypes.byref(s), p, p, p, p, p, None, None, p, 1 << 20, None) == vsa.VSA_ERR_INVALID_ARG
    assert tp(ctypes.byref(s), p, p, p, p, p, p, None, p, 16, None) == vsa.VSA_ERR_INVALID_ARG
    assert tp(ctypes.byref(s), p, odd, p, p, p, p, None, p, 1 << 20, None) == vsa.VSA_ERR_INVALID_ARG
    fo = lib.vsa_block_sparse_fwd_out
    assert fo(ctypes.byref(s), p, p, p, p, p, 5, None, None, None, p, None, None) == vsa.VSA_ERR_INVALID_ARG
    assert fo(ctypes.byref(s), p, p, p, p, p, 2, None, None, None, None, None, None) == vsa.VSA_ERR_INVALID_ARG
    assert fo(ctypes.byref(s), p, p, p, p, p, 2, None, p, None, p, None, None) == vsa.VSA_ERR_INVALID_ARG
    assert fo(ctypes.byref(s), p, p, p, p, p, 2, None, p, p, p, None, None) == vsa.VSA_ERR_INVALID_ARG
    assert fo(ctypes.byref(s), p, p, p, p, p, 2, None, None, None, odd, None, None) == vsa.VSA_ERR_INVALID_ARG
    st = lib.vsa_select_transpose
    assert st(ctypes.byref(s), p, 5, p, p, p, 1 << 20, None) == vsa.VSA_ERR_INVALID_ARG
    assert st(ctypes.byref(s), p, 2, None, p, p, 1 << 20, None) == vsa.VSA_ERR_INVALID_ARG
    assert st(ctypes.byref(s), p, 2, p, p, p, 16, None) == vsa.VSA_ERR_INVALID_ARG
    assert st(ctypes.byref(s), p, 2, p, p, ctypes.c_void_p(0x100010), 1 << 20, None) == vsa.VSA_ERR_INVALID_ARG
    bp = lib.vsa_backward_prep
    assert bp(ctypes.byref(s), None, p, None, None, None, p, p, None, None, None, None) == vsa.VSA_ERR_INVALID_ARG
    assert bp(ctypes.byref(s), p, p, None, p, None, p, p, None, None, None, None) == vsa.VSA_ERR_INVALID_ARG
    assert bp(ctypes.byref(s), p, p, None, p, p, p, p, p, p, p, None) == vsa.VSA_ERR_INVALID_ARG
    assert bp(ctypes.byref(s), odd, p, None, None, None, p, p, None, None, None, None) == vsa.VSA_ERR_INVALID_ARG
    cp = lib.vsa_coarse_select_pooled
    assert cp(ctypes.byref(s), 5, None, p, None, p, 1 << 20, None) == vsa.VSA_ERR_INVALID_ARG
    assert cp(ctypes.byref(s), 2, None, None, None, p, 1 << 20, None) == vsa.VSA_ERR_INVALID_ARG
    assert cp(ctypes.byref(s), 2, None, p, None, p, 16, None) == vsa.VSA_ERR_INVALID_ARG
    cb = lib.vsa_coarse_backward
    assert cb(ctypes.byref(s), None, p, p, p, p, 1 << 20, None) == vsa.VSA_ERR_INVALID_ARG
    assert cb(ctypes.byref(s), p, p, p, None, p, 1 << 20, None) == vsa.VSA_ERR_INVALID_ARG
    assert cb(ctypes.byref(s), p, p, odd, p, p, 1 << 20, None) == vsa.VSA_ERR_INVALID_ARG
    assert cb(ctypes.byref(s), p, p, p, p, ctypes.c_void_p(0x100010), 1 << 20, None) == vsa.VSA_ERR_INVALID_ARG
    # less than one plane's P and dS (C = 4, row stride 64): 2 * 4 * 64 * 4 bytes
    assert cb(ctypes.byref(s), p, p, p, p, p, 2 * 4 * 64 * 4 - 1, None) == vsa.VSA_ERR_INVALID_ARG
    assert vsa.vsa_coarse_backward_workspace_bytes(s) == 2 * (2 * 4 * 64 * 4)
    big = vsa.make_shape(1, 40, 128, (21, 45, 80))  # C = 1440, row stride 1472
    assert vsa.vsa_coarse_backward_workspace_bytes(big) == 40 * 2 * 1440 * 1472 * 4
    fb = lib.vsa_block_sparse_bwd
    two = ctypes.c_void_p(0x1002)
    assert fb(ctypes.byref(s), p, p, p, p, 5, p, p, p, p, p, None, p, p, p, None) == vsa.VSA_ERR_INVALID_ARG
    assert fb(ctypes.byref(s), p, p, p, p, 2, p, p, p, p, p, None, None, p, p, None) == vsa.VSA_ERR_INVALID_ARG
    assert fb(ctypes.byref(s), odd, p, p, p, 2, p, p, p, p, p, None, p, p, p, None) == vsa.VSA_ERR_INVALID_ARG
    assert fb(ctypes.byref(s), p, p, p, p, 2, p, p, two, p, p, None, p, p, p, None) == vsa.VSA_ERR_INVALID_ARG
    assert fb(ctypes.byref(s), p, p, p, p, 2, p, p, p, p, p, odd, p, p, p, None) == vsa.VSA_ERR_INVALID_ARG
    assert lib.vsa_debug_wait_timeout(10, None) == vsa.VSA_ERR_INVALID_ARG
    # linear branch: small or misaligned workspace, misaligned tensors
    lb = lib.vsa_linear_branch_add
    need = vsa.vsa_linear_workspace_bytes(s)
    assert need > 0
    ws = ctypes.c_void_p(0x100000)
    assert lb(ctypes.byref(s), p, p, p, p, ws, need - 1, None) == vsa.VSA_ERR_INVALID_ARG
    assert lb(ctypes.byref(s), p, p, p, p, ctypes.c_void_p(0x100010), need, None) == vsa.VSA_ERR_INVALID_ARG
    assert lb(ctypes.byref(s), p, odd, p, p, ws, need, None) == vsa.VSA_ERR_INVALID_ARG
    # projections: hidden must be a positive multiple of 64; pointers checked
    qp, op_ = lib.vsa_qkv_projection_tiled, lib.vsa_out_projection_tiled
    assert qp(ctypes.byref(s), 96, p, p, p, p, p, None, None) == vsa.VSA_ERR_INVALID_ARG
    assert qp(ctypes.byref(s), 0, p, p, p, p, p, None, None) == vsa.VSA_ERR_INVALID_ARG
    assert qp(ctypes.byref(s), 128, p, None, p, p, p, None, None) == vsa.VSA_ERR_INVALID_ARG
    assert qp(ctypes.byref(s), 128, odd, p, p, p, p, None, None) == vsa.VSA_ERR_INVALID_ARG
    assert qp(ctypes.byref(s), 128, p, p, p, p, p, two, None) == vsa.VSA_ERR_INVALID_ARG
    assert op_(ctypes.byref(s), 96, p, p, p, None) == vsa.VSA_ERR_INVALID_ARG
    assert op_(ctypes.byref(s), 128, p, p, None, None) == vsa.VSA_ERR_INVALID_ARG
    assert op_(ctypes.byref(s), 128, p, odd, p, None) == vsa.VSA_ERR_INVALID_ARG


def test_strerror(vsa):
    assert vsa.vsa_strerror(0) == "ok"
    assert "timed out" in vsa.vsa_strerror(vsa.VSA_ERR_TIMEOUT)
    assert vsa.vsa_strerror(99) == "unknown status"


def test_forward_host_workspace_and_argument_checks(vsa):
    lib = vsa._lib
    s = vsa.make_shape(1, 40, 128, (21, 45, 80))
    C, N, d = 1440, 21 * 45 * 80, 128
    per_chunk_ungated = (3 * 8 * N * d * 2 + 3 * 8 * 64 * C * d * 2 + 8 * N * d * 2
                         + 8 * C * 180 * 4 + 3 * 8 * C * d * 4 + C * 4)
    got = vsa.vsa_forward_host_workspace_bytes(s, 180, 8, gated=False)
    assert per_chunk_ungated * 2 <= got <= per_chunk_ungated * 2 + 2 * 16 * 256
    gated = vsa.vsa_forward_host_workspace_bytes(s, 180, 8, gated=True)
    assert gated - got >= 2 * (2 * 8 * N * 4 + 8 * C * d * 4)
    # 0 means 2 planes per chunk
    assert vsa.vsa_forward_host_workspace_bytes(s, 180, 0) == vsa.vsa_forward_host_workspace_bytes(s, 180, 2)
    assert vsa.vsa_forward_host_workspace_bytes(s, 180, 2) < got
    assert vsa.vsa_forward_host_workspace_bytes(s, 0, 8) == 0
    assert vsa.vsa_forward_host_workspace_bytes(s, 180, -1) == 0
    # a chunk never exceeds B*H planes
    small = vsa.make_shape(1, 2, 64, (4, 8, 8))
    assert (vsa.vsa_forward_host_workspace_bytes(small, 2, 8)
            == vsa.vsa_forward_host_workspace_bytes(small, 2, 2))

    p = ctypes.c_void_p(0x1000)
    ws = ctypes.c_void_p(0x100000)
    big = ctypes.c_size_t(1 << 40)
    call = lambda *a: lib.vsa_forward_host(ctypes.byref(small), *a)
    ok_args = [2, p, p, p, None, None, p, ws, big, 0, None]
    a = list(ok_args); a[1] = None                       # q missing
    assert call(*a) == vsa.VSA_ERR_INVALID_ARG
    a = list(ok_args); a[4] = p                          # one gate without the other
    assert call(*a) == vsa.VSA_ERR_INVALID_ARG
    a = list(ok_args); a[7] = ctypes.c_void_p(0x100010)  # workspace not 256-byte aligned
    assert call(*a) == vsa.VSA_ERR_INVALID_ARG
    a = list(ok_args); a[8] = ctypes.c_size_t(1024)      # workspace too small
    assert call(*a) == vsa.VSA_ERR_INVALID_ARG
    a = list(ok_args); a[0] = 5                          # k > C
    assert call(*a) == vsa.VSA_ERR_INVALID_ARG
    a = list(ok_args); a[9] = -2                         # negative chunk
    assert call(*a) == vsa.VSA_ERR_INVALID_ARG


def test_header_compiles_as_c_and_a_c_program_links_the_library(vsa, tmp_path):
    # the boundary is a C ABI: a plain C translation unit includes the header,
    # links libvsa.so and calls the host-only entry points (no GPU needed)
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    cuda_inc = "/usr/local/cuda/include"
    if gcc is None or not os.path.exists(os.path.join(cuda_inc, "cuda_runtime_api.h")):
        pytest.skip("gcc or the CUDA headers are not available")
    src = tmp_path / "abi.c"
    src.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "vsa.h"
int main(void) {
  vsa_shape s = {1, 40, 128, 21, 45, 80, 4, 4, 4};
  int c = 0, k = 0;
  if (vsa_num_cubes(&s, &c) != VSA_OK || c != 1440) return 1;
  if (vsa_topk_from_ratio(c, 0.125f, &k) != VSA_OK || k != 180) return 2;
  if (vsa_workspace_bytes(&s, k) != (size_t)3 * 40 * 1440 * 128 * 4) return 3;
  if (strcmp(vsa_strerror(VSA_OK), "ok") != 0) return 4;
  if (vsa_tile_permute(&s, NULL, NULL, NULL, 0) != VSA_ERR_INVALID_ARG) return 5;
  /* two C x C float32 matrices per (b, h), rows padded to 1472 */
  if (vsa_coarse_backward_workspace_bytes(&s) != (size_t)40 * 2 * 1440 * 1472 * 4) return 6;
  if (vsa_block_sparse_bwd(&s, NULL, NULL, NULL, NULL, k, NULL, NULL, NULL, NULL, NULL, NULL,
                           NULL, NULL, NULL, 0) != VSA_ERR_INVALID_ARG) return 7;
  printf("c abi ok\n");
  return 0;
}
''')
    exe = tmp_path / "abi"
    libdir = os.path.dirname(vsa._LIB_PATH)
    res = subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-x", "c", str(src), "-o", str(exe),
                          f"-I{os.path.join(ROOT, 'include')}", f"-I{cuda_inc}", f"-L{libdir}",
                          "-lvsa", f"-Wl,-rpath,{libdir}"], capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, (run.returncode, run.stderr)
    assert "c abi ok" in run.stdout
