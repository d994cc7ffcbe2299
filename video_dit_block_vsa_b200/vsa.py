"""Python binding of libvsa (the C ABI in include/vsa.h).

Argument marshalling only: every function forwards torch tensors' device
pointers and the current CUDA stream to the C entry point of the same name and
raises ``VsaError`` on a non-zero status.  Every step of the path runs in the
library's CUDA kernels; there is no fallback.  Importing this module loads
``libvsa.so`` and raises if it has not been built
(``python -m video_dit_block_vsa_b200.build``).
"""

from __future__ import annotations

import ctypes
import math
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libvsa.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"{_LIB_PATH} is missing: build the CUDA library first "
        "(python -m video_dit_block_vsa_b200.build)")
_lib = ctypes.CDLL(_LIB_PATH)

VSA_OK = 0
VSA_ERR_INVALID_ARG = 1
VSA_ERR_UNSUPPORTED = 2
VSA_ERR_CUDA = 3
VSA_ERR_TIMEOUT = 4
VSA_ERR_BAD_INDEX = 5
VSA_ERR_TOO_LARGE = 6

EXPORTED = ("vsa_num_cubes", "vsa_topk_from_ratio", "vsa_workspace_bytes", "vsa_tile_permute",
            "vsa_coarse_select", "vsa_coarse_select_tokens", "vsa_tile_permute_pool",
            "vsa_coarse_select_pooled", "vsa_coarse_select_noalloc",
            "vsa_block_sparse_fwd", "vsa_block_sparse_fwd_out",
            "vsa_combine", "vsa_untile", "vsa_forward_host_workspace_bytes", "vsa_forward_host",
            "vsa_select_transpose", "vsa_backward_prep", "vsa_coarse_backward_workspace_bytes", "vsa_coarse_backward",
            "vsa_block_sparse_bwd", "vsa_linear_workspace_bytes", "vsa_linear_branch_add",
            "vsa_qkv_projection_tiled", "vsa_out_projection_tiled",
            "vsa_get_status", "vsa_debug_wait_timeout",
            "vsa_strerror")


class VsaShape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("grid_t", ctypes.c_int), ("grid_h", ctypes.c_int), ("grid_w", ctypes.c_int),
                ("cube_t", ctypes.c_int), ("cube_h", ctypes.c_int), ("cube_w", ctypes.c_int)]


class VsaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {vsa_strerror(code)} (code {code})")


_P = ctypes.c_void_p
_SP = ctypes.POINTER(VsaShape)
_sig = {
    "vsa_num_cubes": (ctypes.c_int, [_SP, ctypes.POINTER(ctypes.c_int)]),
    "vsa_topk_from_ratio": (ctypes.c_int, [ctypes.c_int, ctypes.c_float, ctypes.POINTER(ctypes.c_int)]),
    "vsa_workspace_bytes": (ctypes.c_size_t, [_SP, ctypes.c_int]),
    "vsa_tile_permute": (ctypes.c_int, [_SP, _P, _P, _P, _P]),
    "vsa_coarse_select": (ctypes.c_int, [_SP, _P, _P, _P, _P, ctypes.c_int, _P, _P, _P, _P,
                                         ctypes.c_size_t, _P]),
    "vsa_coarse_select_tokens": (ctypes.c_int, [_SP, _P, _P, _P, ctypes.c_int, _P, _P, _P, _P,
                                                ctypes.c_size_t, _P]),
    "vsa_tile_permute_pool": (ctypes.c_int, [_SP, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "vsa_coarse_select_pooled": (ctypes.c_int, [_SP, ctypes.c_int, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "vsa_coarse_select_noalloc": (ctypes.c_int, [_SP, _P, _P, _P, _P, ctypes.c_int, _P, _P, _P, _P]),
    "vsa_block_sparse_fwd": (ctypes.c_int, [_SP, _P, _P, _P, _P, _P, ctypes.c_int, _P, _P, _P]),
    "vsa_block_sparse_fwd_out": (ctypes.c_int, [_SP, _P, _P, _P, _P, _P, ctypes.c_int, _P, _P, _P,
                                                _P, _P, _P]),
    "vsa_combine": (ctypes.c_int, [_SP, _P, _P, _P, _P, _P, _P]),
    "vsa_untile": (ctypes.c_int, [_SP, _P, _P, _P]),
    "vsa_linear_workspace_bytes": (ctypes.c_size_t, [_SP]),
    "vsa_linear_branch_add": (ctypes.c_int, [_SP, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "vsa_qkv_projection_tiled": (ctypes.c_int, [_SP, ctypes.c_int, _P, _P, _P, _P, _P, _P, _P]),
    "vsa_out_projection_tiled": (ctypes.c_int, [_SP, ctypes.c_int, _P, _P, _P, _P]),
    "vsa_forward_host_workspace_bytes": (ctypes.c_size_t, [_SP, ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "vsa_forward_host": (ctypes.c_int, [_SP, ctypes.c_int, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t,
                                        ctypes.c_int, _P]),
    "vsa_select_transpose": (ctypes.c_int, [_SP, _P, ctypes.c_int, _P, _P, _P, ctypes.c_size_t, _P]),
    "vsa_backward_prep": (ctypes.c_int, [_SP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "vsa_coarse_backward_workspace_bytes": (ctypes.c_size_t, [_SP]),
    "vsa_coarse_backward": (ctypes.c_int, [_SP, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "vsa_block_sparse_bwd": (ctypes.c_int, [_SP, _P, _P, _P, _P, ctypes.c_int, _P, _P, _P, _P, _P,
                                            _P, _P, _P, _P, _P]),
    "vsa_get_status": (ctypes.c_int, [_P]),
    "vsa_debug_wait_timeout": (ctypes.c_int, [ctypes.c_uint64, _P]),
    "vsa_strerror": (ctypes.c_char_p, [ctypes.c_int]),
}
for _name, (_res, _args) in _sig.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


def vsa_strerror(code: int) -> str:
    return _lib.vsa_strerror(code).decode()


def make_shape(batch, heads, head_dim, grid, cube=(4, 4, 4)) -> VsaShape:
    return VsaShape(batch, heads, head_dim, grid[0], grid[1], grid[2], *cube)


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(rc: int, where: str):
    if rc != VSA_OK:
        raise VsaError(rc, where)


def _expect_device(t, name):
    """A caller-supplied device buffer (workspace): a CUDA tensor."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name}: expected a CUDA tensor")


def _expect(t, dtype, shape, name):
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_cuda:
        raise ValueError(f"{name}: expected a CUDA tensor")


# --------------------------------------------------------------------------
# host-only helpers
# --------------------------------------------------------------------------

def vsa_num_cubes(shape: VsaShape) -> int:
    c = ctypes.c_int(0)
    _check(_lib.vsa_num_cubes(ctypes.byref(shape), ctypes.byref(c)), "vsa_num_cubes")
    return c.value


def vsa_topk_from_ratio(num_cubes: int, ratio: float) -> int:
    k = ctypes.c_int(0)
    _check(_lib.vsa_topk_from_ratio(num_cubes, ratio, ctypes.byref(k)), "vsa_topk_from_ratio")
    return k.value


def vsa_workspace_bytes(shape: VsaShape, topk: int) -> int:
    return int(_lib.vsa_workspace_bytes(ctypes.byref(shape), topk))


# --------------------------------------------------------------------------
# the five calls of the path (device tensors)
# --------------------------------------------------------------------------

def _dims(shape: VsaShape):
    C = vsa_num_cubes(shape)
    N = shape.grid_t * shape.grid_h * shape.grid_w
    return shape.batch, shape.heads, N, shape.head_dim, C


def vsa_tile_permute(shape, x, x_tiled, cube_count=None, stream=None):
    B, H, N, d, C = _dims(shape)
    _expect(x, torch.bfloat16, (B, H, N, d), "x")
    _expect(x_tiled, torch.bfloat16, (B, H, 64 * C, d), "x_tiled")
    if cube_count is not None:
        _expect(cube_count, torch.int32, (C,), "cube_count")
    _check(_lib.vsa_tile_permute(ctypes.byref(shape), _ptr(x), _ptr(x_tiled), _ptr(cube_count),
                                 _stream(stream)), "vsa_tile_permute")


def vsa_coarse_select(shape, q_tiled, k_tiled, v_tiled, cube_count, topk, sel_idx, workspace,
                      o_coarse=None, coarse_logits=None, stream=None):
    B, H, N, d, C = _dims(shape)
    for n, t in (("q_tiled", q_tiled), ("k_tiled", k_tiled), ("v_tiled", v_tiled)):
        _expect(t, torch.bfloat16, (B, H, 64 * C, d), n)
    _expect(cube_count, torch.int32, (C,), "cube_count")
    _expect(sel_idx, torch.int32, (B, H, C, topk), "sel_idx")
    if o_coarse is not None:
        _expect(o_coarse, torch.float32, (B, H, C, d), "o_coarse")
    if coarse_logits is not None:
        _expect(coarse_logits, torch.float32, (B, H, C, C), "coarse_logits")
    _expect_device(workspace, "workspace")
    _check(_lib.vsa_coarse_select(ctypes.byref(shape), _ptr(q_tiled), _ptr(k_tiled), _ptr(v_tiled),
                                  _ptr(cube_count), topk, _ptr(o_coarse), _ptr(sel_idx),
                                  _ptr(coarse_logits), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream(stream)),
           "vsa_coarse_select")


def vsa_coarse_select_tokens(shape, q, k, v, topk, sel_idx, workspace, o_coarse=None,
                             coarse_logits=None, stream=None):
    """vsa_coarse_select on the token-order q, k, v (no tiling needed first)."""
    B, H, N, d, C = _dims(shape)
    for n, t in (("q", q), ("k", k), ("v", v)):
        _expect(t, torch.bfloat16, (B, H, N, d), n)
    _expect(sel_idx, torch.int32, (B, H, C, topk), "sel_idx")
    if o_coarse is not None:
        _expect(o_coarse, torch.float32, (B, H, C, d), "o_coarse")
    if coarse_logits is not None:
        _expect(coarse_logits, torch.float32, (B, H, C, C), "coarse_logits")
    _expect_device(workspace, "workspace")
    _check(_lib.vsa_coarse_select_tokens(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), topk,
                                         _ptr(o_coarse), _ptr(sel_idx), _ptr(coarse_logits),
                                         _ptr(workspace), workspace.numel() * workspace.element_size(),
                                         _stream(stream)), "vsa_coarse_select_tokens")


def vsa_tile_permute_pool(shape, q, k, v, q_tiled, k_tiled, v_tiled, workspace, cube_count=None,
                          stream=None):
    """Tiles q, k, v and writes their cube means into ``workspace`` in one pass."""
    B, H, N, d, C = _dims(shape)
    for n, t in (("q", q), ("k", k), ("v", v)):
        _expect(t, torch.bfloat16, (B, H, N, d), n)
    for n, t in (("q_tiled", q_tiled), ("k_tiled", k_tiled), ("v_tiled", v_tiled)):
        _expect(t, torch.bfloat16, (B, H, 64 * C, d), n)
    if cube_count is not None:
        _expect(cube_count, torch.int32, (C,), "cube_count")
    _expect_device(workspace, "workspace")
    _check(_lib.vsa_tile_permute_pool(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(q_tiled),
                                      _ptr(k_tiled), _ptr(v_tiled), _ptr(cube_count), _ptr(workspace),
                                      workspace.numel() * workspace.element_size(), _stream(stream)),
           "vsa_tile_permute_pool")


def vsa_coarse_select_pooled(shape, topk, sel_idx, workspace, o_coarse=None, coarse_logits=None,
                             stream=None):
    """The coarse stage from the cube means vsa_tile_permute_pool left in ``workspace``."""
    B, H, N, d, C = _dims(shape)
    _expect(sel_idx, torch.int32, (B, H, C, topk), "sel_idx")
    if o_coarse is not None:
        _expect(o_coarse, torch.float32, (B, H, C, d), "o_coarse")
    if coarse_logits is not None:
        _expect(coarse_logits, torch.float32, (B, H, C, C), "coarse_logits")
    _expect_device(workspace, "workspace")
    _check(_lib.vsa_coarse_select_pooled(ctypes.byref(shape), topk, _ptr(o_coarse), _ptr(sel_idx),
                                         _ptr(coarse_logits), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(), _stream(stream)),
           "vsa_coarse_select_pooled")


def vsa_coarse_select_noalloc(shape, q_tiled, k_tiled, v_tiled, cube_count, topk, sel_idx,
                              o_coarse=None, coarse_logits=None, stream=None):
    """vsa_coarse_select without a workspace, for callers that cannot
    allocate device memory; its scratch is a fixed 32 MiB array inside the
    library (see include/vsa.h for the limit and the sharing rules)."""
    B, H, N, d, C = _dims(shape)
    for n, t in (("q_tiled", q_tiled), ("k_tiled", k_tiled), ("v_tiled", v_tiled)):
        _expect(t, torch.bfloat16, (B, H, 64 * C, d), n)
    _expect(cube_count, torch.int32, (C,), "cube_count")
    _expect(sel_idx, torch.int32, (B, H, C, topk), "sel_idx")
    if o_coarse is not None:
        _expect(o_coarse, torch.float32, (B, H, C, d), "o_coarse")
    if coarse_logits is not None:
        _expect(coarse_logits, torch.float32, (B, H, C, C), "coarse_logits")
    _check(_lib.vsa_coarse_select_noalloc(ctypes.byref(shape), _ptr(q_tiled), _ptr(k_tiled),
                                          _ptr(v_tiled), _ptr(cube_count), topk, _ptr(o_coarse),
                                          _ptr(sel_idx), _ptr(coarse_logits), _stream(stream)),
           "vsa_coarse_select_noalloc")


def vsa_block_sparse_fwd(shape, q_tiled, k_tiled, v_tiled, cube_count, sel_idx, topk,
                         o_fine_tiled, lse=None, stream=None):
    B, H, N, d, C = _dims(shape)
    for n, t in (("q_tiled", q_tiled), ("k_tiled", k_tiled), ("v_tiled", v_tiled),
                 ("o_fine_tiled", o_fine_tiled)):
        _expect(t, torch.bfloat16, (B, H, 64 * C, d), n)
    _expect(cube_count, torch.int32, (C,), "cube_count")
    _expect(sel_idx, torch.int32, (B, H, C, topk), "sel_idx")
    if lse is not None:
        _expect(lse, torch.float32, (B, H, 64 * C), "lse")
    _check(_lib.vsa_block_sparse_fwd(ctypes.byref(shape), _ptr(q_tiled), _ptr(k_tiled),
                                     _ptr(v_tiled), _ptr(cube_count), _ptr(sel_idx), topk,
                                     _ptr(o_fine_tiled), _ptr(lse), _stream(stream)),
           "vsa_block_sparse_fwd")


def vsa_block_sparse_fwd_out(shape, q_tiled, k_tiled, v_tiled, cube_count, sel_idx, topk, out,
                             o_coarse=None, g_fine=None, g_coarse=None, lse=None, stream=None):
    """Fine stage writing the final token-order output (gated combine and untile fused)."""
    B, H, N, d, C = _dims(shape)
    for n, t in (("q_tiled", q_tiled), ("k_tiled", k_tiled), ("v_tiled", v_tiled)):
        _expect(t, torch.bfloat16, (B, H, 64 * C, d), n)
    _expect(cube_count, torch.int32, (C,), "cube_count")
    _expect(sel_idx, torch.int32, (B, H, C, topk), "sel_idx")
    _expect(out, torch.bfloat16, (B, H, N, d), "out")
    if g_fine is not None:
        _expect(g_fine, torch.float32, (B, H, N), "g_fine")
        _expect(g_coarse, torch.float32, (B, H, N), "g_coarse")
        _expect(o_coarse, torch.float32, (B, H, C, d), "o_coarse")
    if lse is not None:
        _expect(lse, torch.float32, (B, H, 64 * C), "lse")
    _check(_lib.vsa_block_sparse_fwd_out(ctypes.byref(shape), _ptr(q_tiled), _ptr(k_tiled),
                                         _ptr(v_tiled), _ptr(cube_count), _ptr(sel_idx), topk,
                                         _ptr(o_coarse), _ptr(g_fine), _ptr(g_coarse), _ptr(out),
                                         _ptr(lse), _stream(stream)), "vsa_block_sparse_fwd_out")


def vsa_combine(shape, o_fine_tiled, out_tiled, o_coarse=None, g_fine=None, g_coarse=None,
                stream=None):
    B, H, N, d, C = _dims(shape)
    _expect(o_fine_tiled, torch.bfloat16, (B, H, 64 * C, d), "o_fine_tiled")
    _expect(out_tiled, torch.bfloat16, (B, H, 64 * C, d), "out_tiled")
    if g_fine is not None:
        _expect(g_fine, torch.float32, (B, H, N), "g_fine")
        _expect(g_coarse, torch.float32, (B, H, N), "g_coarse")
        _expect(o_coarse, torch.float32, (B, H, C, d), "o_coarse")
    _check(_lib.vsa_combine(ctypes.byref(shape), _ptr(o_fine_tiled), _ptr(o_coarse),
                            _ptr(g_fine), _ptr(g_coarse), _ptr(out_tiled), _stream(stream)),
           "vsa_combine")


def vsa_untile(shape, x_tiled, x, stream=None):
    B, H, N, d, C = _dims(shape)
    _expect(x_tiled, torch.bfloat16, (B, H, 64 * C, d), "x_tiled")
    _expect(x, torch.bfloat16, (B, H, N, d), "x")
    _check(_lib.vsa_untile(ctypes.byref(shape), _ptr(x_tiled), _ptr(x), _stream(stream)),
           "vsa_untile")


def vsa_linear_workspace_bytes(shape) -> int:
    return int(_lib.vsa_linear_workspace_bytes(ctypes.byref(shape)))


def vsa_linear_branch_add(shape, q, k, v, out, workspace, stream=None):
    """Adds the low-rank linear branch to ``out`` in place (see vsa.h)."""
    B, H, N, d, C = _dims(shape)
    for n, t in (("q", q), ("k", k), ("v", v), ("out", out)):
        _expect(t, torch.bfloat16, (B, H, N, d), n)
    _expect_device(workspace, "workspace")
    _check(_lib.vsa_linear_branch_add(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                      _ptr(workspace), workspace.numel() * workspace.element_size(),
                                      _stream(stream)), "vsa_linear_branch_add")


def vsa_qkv_projection_tiled(shape, hidden, x, w_qkv, q_t, k_t, v_t, counts=None, stream=None):
    """[q | k | v] = x W_qkv^T written straight into the tiled layout (see vsa.h)."""
    B, H, N, d, C = _dims(shape)
    _expect(x, torch.bfloat16, (B, N, hidden), "x")
    _expect(w_qkv, torch.bfloat16, (3 * H * d, hidden), "w_qkv")
    for n, t in (("q_t", q_t), ("k_t", k_t), ("v_t", v_t)):
        _expect(t, torch.bfloat16, (B, H, 64 * C, d), n)
    if counts is not None:
        _expect(counts, torch.int32, (C,), "counts")
    _check(_lib.vsa_qkv_projection_tiled(ctypes.byref(shape), int(hidden), _ptr(x), _ptr(w_qkv),
                                         _ptr(q_t), _ptr(k_t), _ptr(v_t), _ptr(counts),
                                         _stream(stream)), "vsa_qkv_projection_tiled")


def vsa_out_projection_tiled(shape, hidden, o_t, w_o, y, stream=None):
    """y = o W_o^T from the tiled attention output, written in token order (see vsa.h)."""
    B, H, N, d, C = _dims(shape)
    _expect(o_t, torch.bfloat16, (B, H, 64 * C, d), "o_t")
    _expect(w_o, torch.bfloat16, (hidden, H * d), "w_o")
    _expect(y, torch.bfloat16, (B, N, hidden), "y")
    _check(_lib.vsa_out_projection_tiled(ctypes.byref(shape), int(hidden), _ptr(o_t), _ptr(w_o),
                                         _ptr(y), _stream(stream)), "vsa_out_projection_tiled")


def vsa_attention_block(shape, hidden, x, w_qkv, w_o, topk, y, g_fine=None, g_coarse=None,
                        bufs=None, stream=None):
    """A DiT attention block around VSA with the layout changes fused into the
    projections: the QKV projection writes q, k, v tiled (and the cube
    counts), the coarse stage pools them, the fine stage writes its output
    tiled (combined with the coarse output when gated), and the output
    projection reads it tiled and writes ``y`` in token order.  Returns the
    buffers."""
    if bufs is None:
        bufs = VsaBuffers(shape, topk, device=x.device, want_coarse=g_fine is not None)
    vsa_qkv_projection_tiled(shape, hidden, x, w_qkv, bufs.q_t, bufs.k_t, bufs.v_t, bufs.counts,
                             stream)
    vsa_coarse_select(shape, bufs.q_t, bufs.k_t, bufs.v_t, bufs.counts, topk, bufs.sel,
                      bufs.workspace, o_coarse=bufs.o_c, stream=stream)
    vsa_block_sparse_fwd(shape, bufs.q_t, bufs.k_t, bufs.v_t, bufs.counts, bufs.sel, topk,
                         bufs.o_f, stream=stream)
    o = bufs.o_f
    if g_fine is not None:
        vsa_combine(shape, bufs.o_f, bufs.out_t, bufs.o_c, g_fine, g_coarse, stream=stream)
        o = bufs.out_t
    vsa_out_projection_tiled(shape, hidden, o, w_o, y, stream)
    return bufs


def _expect_host(t, dtype, shape, name):
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.is_cuda:
        raise ValueError(f"{name}: expected a host (CPU) tensor")


def vsa_forward_host_workspace_bytes(shape, topk, heads_per_chunk=0, gated=False) -> int:
    return int(_lib.vsa_forward_host_workspace_bytes(ctypes.byref(shape), topk, heads_per_chunk,
                                                     1 if gated else 0))


def vsa_forward_host(shape, topk, q, k, v, out, workspace, g_fine=None, g_coarse=None,
                     heads_per_chunk=0, stream=None):
    """The whole path from host tensors (pinned for overlap): q, k, v, out bf16
    [B, H, N, d] and optional gates float32 [B, H, N] on the CPU; workspace is a
    device uint8 tensor of vsa_forward_host_workspace_bytes.  Asynchronous on
    ``stream``; ``out`` is complete when the stream is."""
    B, H, N, d, C = _dims(shape)
    for n, t in (("q", q), ("k", k), ("v", v), ("out", out)):
        _expect_host(t, torch.bfloat16, (B, H, N, d), n)
    if (g_fine is None) != (g_coarse is None):
        raise ValueError("give both gates or neither")
    if g_fine is not None:
        _expect_host(g_fine, torch.float32, (B, H, N), "g_fine")
        _expect_host(g_coarse, torch.float32, (B, H, N), "g_coarse")
    if not workspace.is_cuda:
        raise ValueError("workspace: expected a CUDA tensor")
    _check(_lib.vsa_forward_host(ctypes.byref(shape), topk, _ptr(q), _ptr(k), _ptr(v), _ptr(g_fine),
                                 _ptr(g_coarse), _ptr(out), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), heads_per_chunk,
                                 _stream(stream)), "vsa_forward_host")


def vsa_select_transpose(shape, sel_idx, topk, key_offsets, query_lists, workspace, stream=None):
    """For every key cube, the query cubes that selected it (ascending), as CSR."""
    B, H, N, d, C = _dims(shape)
    _expect(sel_idx, torch.int32, (B, H, C, topk), "sel_idx")
    _expect(key_offsets, torch.int32, (B, H, C + 1), "key_offsets")
    _expect(query_lists, torch.int32, (B, H, C * topk), "query_lists")
    _expect_device(workspace, "workspace")
    _check(_lib.vsa_select_transpose(ctypes.byref(shape), _ptr(sel_idx), topk, _ptr(key_offsets),
                                     _ptr(query_lists), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _stream(stream)),
           "vsa_select_transpose")


def vsa_backward_prep(shape, dout, o_fine_tiled, do_fine_tiled, delta, o_coarse=None, g_fine=None,
                      g_coarse=None, do_coarse=None, dg_fine=None, dg_coarse=None, stream=None):
    """Gradient of the gated combine, ready for the attention backward (see vsa.h)."""
    B, H, N, d, C = _dims(shape)
    _expect(dout, torch.bfloat16, (B, H, N, d), "dout")
    _expect(o_fine_tiled, torch.bfloat16, (B, H, 64 * C, d), "o_fine_tiled")
    _expect(do_fine_tiled, torch.bfloat16, (B, H, 64 * C, d), "do_fine_tiled")
    _expect(delta, torch.float32, (B, H, 64 * C), "delta")
    if g_fine is not None:
        for n, t, shp in (("o_coarse", o_coarse, (B, H, C, d)), ("do_coarse", do_coarse, (B, H, C, d)),
                          ("g_fine", g_fine, (B, H, N)), ("g_coarse", g_coarse, (B, H, N)),
                          ("dg_fine", dg_fine, (B, H, N)), ("dg_coarse", dg_coarse, (B, H, N))):
            _expect(t, torch.float32, shp, n)
    _check(_lib.vsa_backward_prep(ctypes.byref(shape), _ptr(dout), _ptr(o_fine_tiled), _ptr(o_coarse),
                                  _ptr(g_fine), _ptr(g_coarse), _ptr(do_fine_tiled), _ptr(delta),
                                  _ptr(do_coarse), _ptr(dg_fine), _ptr(dg_coarse), _stream(stream)),
           "vsa_backward_prep")


def vsa_coarse_backward_workspace_bytes(shape) -> int:
    return int(_lib.vsa_coarse_backward_workspace_bytes(ctypes.byref(shape)))


def vsa_coarse_backward(shape, pooled, o_coarse, do_coarse, d_pooled, workspace, stream=None):
    """Gradients of the coarse attention w.r.t. the pooled vectors (see vsa.h)."""
    B, H, N, d, C = _dims(shape)
    _expect(pooled, torch.float32, (3, B, H, C, d), "pooled")
    _expect(o_coarse, torch.float32, (B, H, C, d), "o_coarse")
    _expect(do_coarse, torch.float32, (B, H, C, d), "do_coarse")
    _expect(d_pooled, torch.float32, (3, B, H, C, d), "d_pooled")
    _expect_device(workspace, "workspace")
    _check(_lib.vsa_coarse_backward(ctypes.byref(shape), _ptr(pooled), _ptr(o_coarse), _ptr(do_coarse),
                                    _ptr(d_pooled), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream)),
           "vsa_coarse_backward")


def vsa_block_sparse_bwd(shape, q_tiled, k_tiled, v_tiled, sel_idx, topk, key_offsets, query_lists,
                         lse, do_fine_tiled, delta, dq, dk, dv, d_pooled=None, stream=None):
    """Fine-stage backward, pooling backward and untile: dq, dk, dv in token order (see vsa.h)."""
    B, H, N, d, C = _dims(shape)
    for n, t in (("q_tiled", q_tiled), ("k_tiled", k_tiled), ("v_tiled", v_tiled),
                 ("do_fine_tiled", do_fine_tiled)):
        _expect(t, torch.bfloat16, (B, H, 64 * C, d), n)
    for n, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _expect(t, torch.bfloat16, (B, H, N, d), n)
    _expect(sel_idx, torch.int32, (B, H, C, topk), "sel_idx")
    _expect(key_offsets, torch.int32, (B, H, C + 1), "key_offsets")
    _expect(query_lists, torch.int32, (B, H, C * topk), "query_lists")
    _expect(lse, torch.float32, (B, H, 64 * C), "lse")
    _expect(delta, torch.float32, (B, H, 64 * C), "delta")
    if d_pooled is not None:
        _expect(d_pooled, torch.float32, (3, B, H, C, d), "d_pooled")
    _check(_lib.vsa_block_sparse_bwd(ctypes.byref(shape), _ptr(q_tiled), _ptr(k_tiled), _ptr(v_tiled),
                                     _ptr(sel_idx), topk, _ptr(key_offsets), _ptr(query_lists), _ptr(lse),
                                     _ptr(do_fine_tiled), _ptr(delta), _ptr(d_pooled), _ptr(dq), _ptr(dk),
                                     _ptr(dv), _stream(stream)), "vsa_block_sparse_bwd")


def pooled_view(shape, workspace):
    """The pooled qbar, kbar, vbar [3, B, H, C, d] float32 at the start of a
    vsa_tile_permute_pool / vsa_coarse_select workspace (a view, no copy)."""
    B, H, N, d, C = _dims(shape)
    n = 3 * B * H * C * d
    return workspace.view(torch.uint8)[: 4 * n].view(torch.float32).view(3, B, H, C, d)


def vsa_get_status(stream=None) -> int:
    return int(_lib.vsa_get_status(_stream(stream)))


def vsa_debug_wait_timeout(timeout_ns: int, stream=None):
    _check(_lib.vsa_debug_wait_timeout(timeout_ns, _stream(stream)), "vsa_debug_wait_timeout")


# --------------------------------------------------------------------------
# convenience: the whole path with torch-allocated buffers
# --------------------------------------------------------------------------

class VsaBuffers:
    """Device buffers for one shape and k, allocated once with torch."""

    def __init__(self, shape: VsaShape, topk: int, device="cuda", want_coarse=True, want_lse=False):
        B, H, N, d, C = _dims(shape)
        self.shape, self.topk = shape, topk
        bf = dict(dtype=torch.bfloat16, device=device)
        self.q_t = torch.empty(B, H, 64 * C, d, **bf)
        self.k_t = torch.empty(B, H, 64 * C, d, **bf)
        self.v_t = torch.empty(B, H, 64 * C, d, **bf)
        self.o_f = torch.empty(B, H, 64 * C, d, **bf)
        self.out_t = torch.empty(B, H, 64 * C, d, **bf)
        self.counts = torch.empty(C, dtype=torch.int32, device=device)
        self.sel = torch.empty(B, H, C, topk, dtype=torch.int32, device=device)
        self.o_c = torch.empty(B, H, C, d, dtype=torch.float32, device=device) if want_coarse else None
        self.lse = torch.empty(B, H, 64 * C, dtype=torch.float32, device=device) if want_lse else None
        ws = vsa_workspace_bytes(shape, topk)
        self.workspace = torch.empty(ws, dtype=torch.uint8, device=device)


def vsa_forward(shape, q, k, v, topk, out, g_fine=None, g_coarse=None, bufs=None, stream=None):
    """Runs the whole path: tile q/k/v, coarse select, fine attention,
    combine, untile into ``out`` ([B, H, N, d] bf16).  Returns the buffers."""
    if bufs is None:
        bufs = VsaBuffers(shape, topk, device=q.device, want_coarse=g_fine is not None)
    vsa_tile_permute(shape, q, bufs.q_t, bufs.counts, stream)
    vsa_tile_permute(shape, k, bufs.k_t, None, stream)
    vsa_tile_permute(shape, v, bufs.v_t, None, stream)
    vsa_coarse_select(shape, bufs.q_t, bufs.k_t, bufs.v_t, bufs.counts, topk, bufs.sel,
                      bufs.workspace, o_coarse=bufs.o_c, stream=stream)
    vsa_block_sparse_fwd(shape, bufs.q_t, bufs.k_t, bufs.v_t, bufs.counts, bufs.sel, topk,
                         bufs.o_f, bufs.lse, stream)
    if g_fine is not None:
        vsa_combine(shape, bufs.o_f, bufs.out_t, bufs.o_c, g_fine, g_coarse, stream)
        vsa_untile(shape, bufs.out_t, out, stream)
    else:
        vsa_untile(shape, bufs.o_f, out, stream)
    return bufs


def vsa_forward_fused(shape, q, k, v, topk, out, g_fine=None, g_coarse=None, bufs=None,
                      stream=None):
    """The whole path in the three launches the benchmark times: tiling with
    the cube means in one pass, the coarse stage from those means, and the
    fine kernel whose epilogue applies the gated combine and writes ``out``
    in token order.  Same bits as ``vsa_forward``.  Returns the buffers."""
    if bufs is None:
        bufs = VsaBuffers(shape, topk, device=q.device, want_coarse=g_fine is not None)
    vsa_tile_permute_pool(shape, q, k, v, bufs.q_t, bufs.k_t, bufs.v_t, bufs.workspace,
                          bufs.counts, stream)
    vsa_coarse_select_pooled(shape, topk, bufs.sel, bufs.workspace, o_coarse=bufs.o_c,
                             stream=stream)
    vsa_block_sparse_fwd_out(shape, bufs.q_t, bufs.k_t, bufs.v_t, bufs.counts, bufs.sel, topk,
                             out, bufs.o_c if g_fine is not None else None, g_fine, g_coarse,
                             stream=stream)
    return bufs


class VsaGradBuffers:
    """Device scratch of one backward call, allocated once with torch."""

    def __init__(self, shape: VsaShape, topk: int, gated: bool, device="cuda"):
        B, H, N, d, C = _dims(shape)
        f32 = dict(dtype=torch.float32, device=device)
        self.do_f = torch.empty(B, H, 64 * C, d, dtype=torch.bfloat16, device=device)
        self.delta = torch.empty(B, H, 64 * C, **f32)
        self.key_offsets = torch.empty(B, H, C + 1, dtype=torch.int32, device=device)
        self.query_lists = torch.empty(B, H, C * topk, dtype=torch.int32, device=device)
        self.transpose_ws = torch.empty(B * H * C * topk * 4, dtype=torch.uint8, device=device)
        self.do_c = torch.empty(B, H, C, d, **f32) if gated else None
        self.d_pooled = torch.empty(3, B, H, C, d, **f32) if gated else None
        self.coarse_ws = (torch.empty(vsa_coarse_backward_workspace_bytes(shape), dtype=torch.uint8,
                                      device=device) if gated else None)


def vsa_backward(shape, bufs, dout, dq, dk, dv, g_fine=None, g_coarse=None, dg_fine=None,
                 dg_coarse=None, grads=None, stream=None):
    """Gradients of the whole path for the forward ``bufs`` left (a
    ``vsa_forward`` with ``VsaBuffers(..., want_lse=True)``): dq, dk, dv
    ([B, H, N, d] bf16) and, when gated, dg_fine, dg_coarse ([B, H, N] float32).
    Four library calls: the combine gradient, the coarse backward (gated only),
    the selection transpose and the fine backward.  Returns the scratch."""
    if bufs.lse is None:
        raise ValueError("the forward must keep its LSE (VsaBuffers(..., want_lse=True))")
    gated = g_fine is not None
    if grads is None:
        grads = VsaGradBuffers(shape, bufs.topk, gated, device=dout.device)
    vsa_backward_prep(shape, dout, bufs.o_f, grads.do_f, grads.delta, bufs.o_c if gated else None,
                      g_fine, g_coarse, grads.do_c, dg_fine, dg_coarse, stream)
    if gated:
        vsa_coarse_backward(shape, pooled_view(shape, bufs.workspace), bufs.o_c, grads.do_c,
                            grads.d_pooled, grads.coarse_ws, stream)
    vsa_select_transpose(shape, bufs.sel, bufs.topk, grads.key_offsets, grads.query_lists,
                         grads.transpose_ws, stream)
    vsa_block_sparse_bwd(shape, bufs.q_t, bufs.k_t, bufs.v_t, bufs.sel, bufs.topk, grads.key_offsets,
                         grads.query_lists, bufs.lse, grads.do_f, grads.delta, dq, dk, dv,
                         grads.d_pooled if gated else None, stream)
    return grads
