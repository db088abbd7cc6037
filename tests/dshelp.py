"""Helpers shared by the GPU tests: host <-> device marshalling, and the
parity criteria of the decode step (scores within 1e-3 relative, selection
exact outside a 1e-4 tie band around the k-th score, output within 2e-3)."""

from __future__ import annotations

import numpy as np

import oracle
import synth

SCORE_RTOL = 1e-3
TIE_BAND = 1e-4
OUT_ATOL = 2e-3


def to_dev(x: np.ndarray, dtype: str):
    import torch
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def to_host(t, dtype: str) -> np.ndarray:
    import torch
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    if t.dtype == torch.int16:
        return t.cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def check_scores(s_gpu: np.ndarray, s_ref: np.ndarray):
    """|s_gpu - s_ref| <= 1e-3 * max(|s_ref|, mean_t |s_ref|) per row."""
    floor = np.abs(s_ref).mean(axis=-1, keepdims=True)
    tol = SCORE_RTOL * np.maximum(np.abs(s_ref), floor)
    bad = np.abs(s_gpu.astype(np.float64) - s_ref) > tol
    assert not bad.any(), f"{bad.sum()} scores out of tolerance; worst " \
        f"{np.max(np.abs(s_gpu - s_ref) / np.maximum(tol, 1e-300))} x tol"


def check_selection(sel_gpu: np.ndarray, sel_ref: np.ndarray, s_ref: np.ndarray, k: int, s: int):
    """sel arrays [rows, k]; s_ref [rows, s]. The GPU set must be valid and
    differ from the oracle's only at tokens within the tie band of the k-th
    oracle score."""
    rows = sel_ref.shape[0]
    m = min(k, s)
    for r in range(rows):
        g = sel_gpu[r]
        assert np.all(g[m:] == -1), "padding"
        gg = g[:m]
        assert np.all(np.diff(gg) > 0), "ascending, no duplicates"
        assert gg.min() >= 0 and gg.max() < s
        ref = sel_ref[r, :m]
        diff = np.setxor1d(gg, ref)
        if diff.size:
            kth = np.sort(s_ref[r])[::-1][m - 1]
            band = TIE_BAND * abs(kth)
            far = diff[np.abs(s_ref[r, diff] - kth) > band]
            assert far.size == 0, f"row {r}: tokens {far[:8]} differ outside the tie band"


def oracle_row_slices(k, v, q, label, label_dtype, b, g, G):
    """Contiguous single-(b, g) views for running the oracle on one row."""
    ks = k[b:b + 1, g:g + 1]
    vs = v[b:b + 1, g:g + 1]
    qs = q[b:b + 1, g * G:(g + 1) * G]
    if label_dtype == "int4":
        lab = tuple(x[b:b + 1, g:g + 1] for x in label)
    else:
        lab = label[b:b + 1, g:g + 1]
    return qs, ks, vs, lab
