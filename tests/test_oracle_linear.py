"""Pins for the linear compensation branch of the oracle (oracle/vsa_linear.py),
checked against things other than its own formula: the dense N x N form of the
same attention computed by torch on the CPU, closed forms, token-permutation
invariance, and a loop-only restatement.  A plausible slip (KV transposed, the
normaliser left out or taken over the wrong axis, phi applied to v, the
feature map's branch flipped, the branch not added) fails at least one."""

import math

import numpy as np
import pytest
import torch

from oracle import vsa_linear as vl
from oracle import vsa_oracle as vo


def dense_linear(q, k, v):
    """phi(Q) phi(K)^T, each row divided by its sum, times V: the quadratic
    form of linear attention, with torch's elu as the feature map."""
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))
    fq = torch.nn.functional.elu(t(q)) + 1.0
    fk = torch.nn.functional.elu(t(k)) + 1.0
    w = fq @ fk.transpose(-1, -2)
    return ((w / w.sum(dim=-1, keepdim=True)) @ t(v)).numpy()


def rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_feature_map_closed_forms():
    x = np.array([-50.0, -1.0, -1e-12, 0.0, 1e-12, 0.5, 3.0])
    got = vl.feature_map(x)
    want = np.array([math.exp(-50.0), math.exp(-1.0), math.exp(-1e-12), 1.0, 1.0 + 1e-12, 1.5, 4.0])
    assert np.allclose(got, want, rtol=1e-15, atol=0.0)
    assert np.all(got > 0.0)


@pytest.mark.parametrize("shape", [(1, 1, 7, 4), (2, 3, 50, 16), (1, 2, 200, 64)])
def test_equals_dense_quadratic_form(shape):
    q, k, v = rand(shape, 1), rand(shape, 2), rand(shape, 3)
    assert np.allclose(vl.linear_attention(q, k, v), dense_linear(q, k, v), rtol=1e-12, atol=1e-12)


def test_equal_keys_give_mean_of_values():
    q, v = rand((1, 2, 30, 8), 4), rand((1, 2, 30, 8), 5)
    k = np.broadcast_to(rand((1, 2, 1, 8), 6), (1, 2, 30, 8))
    got = vl.linear_attention(q, k, v)
    assert np.allclose(got, np.broadcast_to(v.mean(axis=-2, keepdims=True), got.shape), atol=1e-13)


def test_unit_values_give_one():
    q, k = rand((2, 1, 40, 8), 7) * 3.0, rand((2, 1, 40, 8), 8) * 3.0
    got = vl.linear_attention(q, k, np.ones((2, 1, 40, 8)))
    assert np.allclose(got, 1.0, atol=1e-13)


def test_token_permutation_invariance():
    q, k, v = rand((1, 1, 60, 8), 9), rand((1, 1, 60, 8), 10), rand((1, 1, 60, 8), 11)
    perm = np.random.default_rng(12).permutation(60)
    base = vl.linear_attention(q, k, v)
    moved = vl.linear_attention(q[:, :, perm], k[:, :, perm], v[:, :, perm])
    assert np.allclose(moved, base[:, :, perm], atol=1e-13)
    # keys and values permuted alone: a global sum, so nothing changes
    assert np.allclose(vl.linear_attention(q, k[:, :, perm], v[:, :, perm]), base, atol=1e-13)


def test_loop_restatement_tiny():
    B, H, N, d = 1, 2, 9, 3
    q, k, v = rand((B, H, N, d), 13), rand((B, H, N, d), 14), rand((B, H, N, d), 15)
    phi = lambda x: x + 1.0 if x > 0.0 else math.exp(x)
    want = np.zeros((B, H, N, d))
    for b in range(B):
        for h in range(H):
            for r in range(N):
                num = [0.0] * d
                den = 0.0
                for t in range(N):
                    w = sum(phi(q[b, h, r, a]) * phi(k[b, h, t, a]) for a in range(d))
                    den += w
                    for e in range(d):
                        num[e] += w * v[b, h, t, e]
                for e in range(d):
                    want[b, h, r, e] = num[e] / den
    assert np.allclose(vl.linear_attention(q, k, v), want, rtol=1e-13, atol=1e-14)


def test_sparse_linear_forward_adds_the_branch():
    grid, topk = (4, 8, 8), 2
    N, d = 256, 16
    q, k, v = rand((1, 2, N, d), 16), rand((1, 2, N, d), 17), rand((1, 2, N, d), 18)
    ref = vl.sparse_linear_forward(q, k, v, grid, topk)
    assert np.allclose(ref["out_sparse_linear"], vo.vsa_forward(q, k, v, grid, topk)["out"]
                       + dense_linear(q, k, v), atol=1e-12)
