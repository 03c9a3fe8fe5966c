"""Acceptance checks of a candidate result against the oracle -- test infrastructure.

The bar (stated as the acceptance contract of this build):

* sign planes bit-exact, except an entry whose oracle residual |R_{k-1}[i,j]|
  is at most 1e-6 * alpha_k[i,g] may flip at path k; once it flipped, later
  planes at the same (i, j) may differ too (the residual there has the same
  magnitude either way, only its sign moved). The number of such entries must
  stay below 1e-6 * M * K; any other mismatch fails.
* scales within 1e-6 relative of the oracle's fp64 value.
* fp16 scale copies equal to round-to-nearest-even of the oracle value, except
  within 1e-6 relative of an fp16 rounding midpoint, where either neighbour
  is accepted.
* outputs within 1e-3 * sum_k sum_j |alpha_k x_j| of the oracle, per element.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass
class PlaneReport:
    entries: int
    flipped: int      # entries that differ, all within the near-zero allowance
    bad: int          # entries that differ outside the allowance
    max_flip_frac: float = 1e-6

    @property
    def ok(self) -> bool:
        return self.bad == 0 and self.flipped < self.max_flip_frac * self.entries


def _bits(planes: np.ndarray) -> np.ndarray:
    """[N, M, K/32] uint32 -> [N, M, K] 0/1, bit j of word w = column 32w + j."""
    b = np.ascontiguousarray(planes, dtype="<u4").view(np.uint8)
    return np.unpackbits(b, axis=-1, bitorder="little").reshape(planes.shape[0], planes.shape[1], -1)


def compare_planes(cand: np.ndarray, ref: np.ndarray, rabs: np.ndarray,
                   alpha: np.ndarray, rel: float = 1e-6) -> PlaneReport:
    N, M, W = ref.shape
    K = W * 32
    G = K // alpha.shape[2]
    cb, rb = _bits(cand), _bits(ref)
    diff = cb != rb                                    # [N, M, K]
    entries = M * K
    if not diff.any():
        return PlaneReport(entries, 0, 0)
    first = np.argmax(diff, axis=0)                    # first differing path per entry
    any_diff = diff.any(axis=0)
    ii, jj = np.nonzero(any_diff)
    kk = first[ii, jj]
    a = alpha[kk, ii, jj // G]
    allowed = rabs[kk, ii, jj] <= rel * a
    return PlaneReport(entries, int(allowed.sum()), int((~allowed).sum()))


def compare_scales(cand: np.ndarray, ref: np.ndarray, rel: float = 1e-6):
    cand = np.asarray(cand, dtype=np.float64)
    err = np.abs(cand - ref)
    lim = rel * np.abs(ref)
    bad = err > lim
    worst = float(np.max(err / np.maximum(np.abs(ref), 1e-300))) if ref.size else 0.0
    return int(bad.sum()), worst


def compare_scales_f16(cand16: np.ndarray, ref: np.ndarray, rel: float = 1e-6) -> int:
    """Number of fp16 scales that are neither RN(ref) nor, near a midpoint, the other neighbour."""
    ref = np.asarray(ref, dtype=np.float64)
    c = np.asarray(cand16, dtype=np.float16)
    rn = ref.astype(np.float16)
    ok = c == rn
    if ok.all():
        return 0
    lo = np.nextafter(rn, np.float16(-np.inf))
    hi = np.nextafter(rn, np.float16(np.inf))
    mid_lo = (rn.astype(np.float64) + lo.astype(np.float64)) / 2
    mid_hi = (rn.astype(np.float64) + hi.astype(np.float64)) / 2
    near_lo = np.abs(ref - mid_lo) <= rel * np.abs(ref)
    near_hi = np.abs(ref - mid_hi) <= rel * np.abs(ref)
    ok |= (near_lo & (c == lo)) | (near_hi & (c == hi))
    return int((~ok).sum())


def compare_outputs(cand: np.ndarray, ref: np.ndarray, denom: np.ndarray, tol: float = 1e-3):
    """Returns (number of elements over tolerance, worst |diff| / denom)."""
    cand = np.asarray(cand, dtype=np.float64)
    err = np.abs(cand - ref)
    lim = tol * denom
    ratio = err / np.maximum(denom, 1e-300)
    return int((err > lim).sum()), float(ratio.max()) if ratio.size else 0.0
