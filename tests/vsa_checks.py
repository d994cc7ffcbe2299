"""Helpers shared by the GPU parity tests: moving seeded inputs to the device,
and the comparison rules (tie-aware selection, output tolerances)."""

from __future__ import annotations

import numpy as np
import torch

from oracle import vsa_oracle as vo

# Output tolerances for bf16 inputs with float32 accumulation.
MAX_ABS = 2e-2
MEAN_ABS = 2e-3
# Coarse logits within this band of the k-th largest count as ties.
TIE_BAND = 1e-4


def to_dev_bf16(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def bf16_dev_to_f64(t: torch.Tensor) -> np.ndarray:
    bits = t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return vo.bf16_bits_to_f64(bits)


def bf16_dev_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def check_selection(sel_gpu: np.ndarray, logits_ref: np.ndarray, k: int):
    """Accepts the GPU's per-row selection if it is a top-k set of the
    reference logits up to the tie band.  Returns (rows_equal, rows_tie_swapped).
    Raises AssertionError with the first offending row otherwise."""
    C = logits_ref.shape[-1]
    flat_sel = sel_gpu.reshape(-1, k)
    flat_s = logits_ref.reshape(-1, C)
    equal = swapped = 0
    ref_sel = vo.topk_select(flat_s, k)
    for r in range(flat_sel.shape[0]):
        g = flat_sel[r]
        assert np.all(np.diff(g) > 0), f"row {r}: selection not strictly ascending: {g}"
        assert g.min() >= 0 and g.max() < C, f"row {r}: index out of range"
        if np.array_equal(g, ref_sel[r]):
            equal += 1
            continue
        tau = np.sort(flat_s[r])[::-1][k - 1]
        inside = np.zeros(C, bool)
        inside[g] = True
        ok = np.all(flat_s[r][inside] >= tau - TIE_BAND) and np.all(flat_s[r][~inside] <= tau + TIE_BAND)
        assert ok, f"row {r}: selection {g} is not a top-{k} set (ref {ref_sel[r]})"
        swapped += 1
    return equal, swapped


def assert_close(got: np.ndarray, want: np.ndarray, what: str, max_abs=MAX_ABS, mean_abs=MEAN_ABS):
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = np.abs(got - want)
    mx, mn = float(err.max()) if err.size else 0.0, float(err.mean()) if err.size else 0.0
    assert mx <= max_abs and mn <= mean_abs, f"{what}: max-abs {mx:.3g} (<= {max_abs}), mean-abs {mn:.3g} (<= {mean_abs})"
    return mx, mn
