"""Comparison of the CUDA path's outputs with the oracle's, under the parity rule:

  * codes and scales must match bit for bit, except on the flagged set F: elements whose
    exact |y|/S lies within 1e-5 (relative) of an E2M1 rounding midpoint, and whole groups
    whose exact amax (or NV block-scale quotient) lies within 1e-5 of the scale rule's
    boundary;
  * at most 1e-4 of the elements may differ (a group whose scale differs counts whole);
  * two codes of magnitude zero are equal whatever their sign bits (+0 and -0 encode the
    same value; the sign of a cancelled fp32 butterfly sum is not the sign of the exact sum);
  * rotated values: |y_gpu - y_exact| <= 1e-5 * ||x_block||_2 for every element.
"""

from __future__ import annotations

import dataclasses

import numpy as np

import oracle as o

REL_TOL = 1e-5
MAX_MISMATCH_FRACTION = 1e-4


@dataclasses.dataclass
class ParityReport:
    n: int
    code_mismatch: int
    scale_mismatch_groups: int
    unflagged_code_mismatch: int
    unflagged_scale_mismatch: int
    flagged_elements: int
    flagged_groups: int
    mismatch_elements: int

    def ok(self, count_bound: bool = True) -> bool:
        subset = self.unflagged_code_mismatch == 0 and self.unflagged_scale_mismatch == 0
        if not count_bound:
            return subset
        return subset and self.mismatch_elements <= MAX_MISMATCH_FRACTION * max(self.n, 1)


def compare(res: dict, codes_gpu: np.ndarray, scales_gpu: np.ndarray, tol: float = REL_TOL) -> ParityReport:
    codes_gpu = np.asarray(codes_gpu, np.uint8)
    scales_gpu = np.asarray(scales_gpu, np.uint8)
    assert codes_gpu.shape == res["codes"].shape, (codes_gpu.shape, res["codes"].shape)
    assert scales_gpu.shape == res["scales"].shape
    g = res["group"]
    qo = o.unpack_nibbles(res["codes"])
    qg = o.unpack_nibbles(codes_gpu)
    M, K = qo.shape
    both_zero = ((qo & 7) == 0) & ((qg & 7) == 0)
    diff = (qo != qg) & ~both_zero
    sdiff = res["scales"] != scales_gpu
    el, gr = o.flags(res, tol)
    gr_el = np.repeat(gr, g, axis=1)
    sd_el = np.repeat(sdiff, g, axis=1)
    unflagged_codes = diff & ~(el | gr_el) & ~sd_el
    unflagged_scales = sdiff & ~gr
    mismatch_el = diff | sd_el
    return ParityReport(
        n=M * K,
        code_mismatch=int(diff.sum()),
        scale_mismatch_groups=int(sdiff.sum()),
        unflagged_code_mismatch=int(unflagged_codes.sum()),
        unflagged_scale_mismatch=int(unflagged_scales.sum()),
        flagged_elements=int(el.sum()),
        flagged_groups=int(gr.sum()),
        mismatch_elements=int(mismatch_el.sum()),
    )


def assert_parity(res: dict, codes_gpu, scales_gpu, label: str = "", count_bound: bool = True) -> ParityReport:
    """count_bound=False keeps only "every mismatch is flagged": for inputs built to sit on
    ties (exact midpoints, powers of two), where near-ties are dense by construction."""
    rep = compare(res, codes_gpu, scales_gpu)
    assert rep.ok(count_bound), f"{label}: {rep}"
    return rep


def rotated_value_error(y_gpu: np.ndarray, res: dict) -> float:
    """max over elements of |y_gpu - y64| / ||block||_2 (0 for all-zero blocks)."""
    y64 = res["y64"]
    M, K = y64.shape
    b = res["block"]
    nb = np.linalg.norm(y64.reshape(M, K // b, b), axis=2)
    err = np.abs(np.asarray(y_gpu, np.float64) - y64).reshape(M, K // b, b)
    rel = np.where(nb[..., None] > 0, err / np.where(nb > 0, nb, 1.0)[..., None], err)
    return float(rel.max()) if rel.size else 0.0
