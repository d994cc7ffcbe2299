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


def wide_first(sel: np.ndarray, counts: np.ndarray) -> np.ndarray:
    """The library's order of a selection row: key cubes with more than 16
    valid tokens first, then the others, each group ascending (the order the
    fine kernel packs key rows in).  Same set, rows reordered."""
    sel = np.asarray(sel)
    narrow = (np.asarray(counts)[sel] <= 16).astype(np.int64)
    order = np.lexsort((sel, narrow), axis=-1)
    return np.take_along_axis(sel, order, axis=-1)


def check_selection(sel_gpu: np.ndarray, logits_ref: np.ndarray, k: int, counts=None):
    """Accepts the GPU's per-row selection if it is a top-k set of the
    reference logits up to the tie band, listed in the library's order (wide
    key cubes first, each group ascending; with counts None every cube counts
    as wide, i.e. plain ascending).  Returns (rows_equal, rows_tie_swapped).
    Raises AssertionError with the first offending row otherwise."""
    C = logits_ref.shape[-1]
    if counts is None:
        counts = np.full(C, 64)
    flat_sel = sel_gpu.reshape(-1, k)
    flat_s = logits_ref.reshape(-1, C)
    equal = swapped = 0
    ref_sel = wide_first(vo.topk_select(flat_s, k), counts)
    for r in range(flat_sel.shape[0]):
        g = flat_sel[r]
        assert g.min() >= 0 and g.max() < C, f"row {r}: index out of range"
        assert np.array_equal(g, wide_first(g, counts)), f"row {r}: not in wide-first ascending order: {g}"
        assert np.unique(g).size == k, f"row {r}: repeated index: {g}"
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
