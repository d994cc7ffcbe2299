"""Pins for the DiT-block projections of the oracle (oracle/vsa_dit.py),
checked against things other than their own formula: explicit loops on tiny
sizes, identity weights (the projections then only split or concatenate
heads), the round trip of the two projections, and linearity.  A transposed
weight, a wrong head order or a q/k/v swap fails at least one."""

import numpy as np
import pytest

from oracle import vsa_dit as vd
from oracle import vsa_oracle as vo


def rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_qkv_projection_loops():
    B, N, H, d, hid = 2, 5, 2, 3, 4
    x, w = rand((B, N, hid), 1), rand((3 * H * d, hid), 2)
    q, k, v = vd.qkv_projection(x, w, H, d)
    for b in range(B):
        for n in range(N):
            for part, t in enumerate((q, k, v)):
                for h in range(H):
                    for e in range(d):
                        row = (part * H + h) * d + e
                        want = sum(x[b, n, i] * w[row, i] for i in range(hid))
                        assert abs(t[b, h, n, e] - want) < 1e-12


def test_out_projection_loops():
    B, N, H, d, hid = 1, 4, 3, 2, 5
    o, w = rand((B, H, N, d), 3), rand((hid, H * d), 4)
    y = vd.out_projection(o, w)
    for n in range(N):
        for j in range(hid):
            want = sum(o[0, h, n, e] * w[j, h * d + e] for h in range(H) for e in range(d))
            assert abs(y[0, n, j] - want) < 1e-12


def test_identity_weights_split_and_round_trip():
    B, N, H, d = 2, 7, 3, 4
    hid = H * d
    x = rand((B, N, hid), 5)
    eye = np.eye(hid)
    q, k, v = vd.qkv_projection(x, np.concatenate([eye, 2 * eye, 3 * eye]), H, d)
    for h in range(H):
        assert np.array_equal(q[:, h], x[:, :, h * d:(h + 1) * d])
    assert np.allclose(k, 2 * q) and np.allclose(v, 3 * q)
    assert np.allclose(vd.out_projection(q, eye), x, atol=0)


def test_linearity_in_the_weights():
    B, N, H, d, hid = 1, 6, 2, 4, 8
    x = rand((B, N, hid), 6)
    w1, w2 = rand((3 * H * d, hid), 7), rand((3 * H * d, hid), 8)
    a = vd.qkv_projection(x, w1 + 2 * w2, H, d)
    b1, b2 = vd.qkv_projection(x, w1, H, d), vd.qkv_projection(x, w2, H, d)
    for t, t1, t2 in zip(a, b1, b2):
        assert np.allclose(t, t1 + 2 * t2, atol=1e-12)


def test_attention_block_composes_the_forward():
    grid, H, d, hid, topk = (4, 8, 8), 2, 8, 12, 2
    N = int(np.prod(grid))
    x, wq, wo = rand((1, N, hid), 9), rand((3 * H * d, hid), 10), rand((hid, H * d), 11)
    ref = vd.attention_block(x, wq, wo, H, d, grid, topk)
    fwd = vo.vsa_forward(ref["q"], ref["k"], ref["v"], grid, topk)
    assert np.allclose(ref["y"], vd.out_projection(fwd["out"], wo), atol=1e-12)
