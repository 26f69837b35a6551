"""The parity rule: how the CUDA path's codes and scales are compared with the oracle's.

TEST INFRASTRUCTURE, like the rest of ``oracle/``: only ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline leg use it.

  * codes and scales must match bit for bit, except on the flagged set F: elements whose
    exact |y|/S lies within 1e-5 (relative) of an E2M1 rounding midpoint, and whole groups
    whose exact amax (or NV block-scale quotient, or MBS macro mantissa) lies within 1e-5 of
    the scale rule's boundary (``fp4q_oracle.boundary_distance``);
  * at most 1e-4 of the elements may differ (a group whose scale differs counts whole);
  * a code of magnitude zero may differ from the oracle's in its sign bit only where the
    exact rotated value itself is within the rotated-value tolerance of zero,
    |y64| <= 1e-5 * ||block||_2: there the kernel's fp32 sum may cancel to a zero of either
    sign (or a tiny value of the other sign), and +0 and -0 encode the same value.
    Elsewhere the sign bit of a zero code is the sign of y and must match;
  * rotated values: |y_gpu - y_exact| <= 1e-5 * ||x_block||_2 for every element.

Each comparison is recorded (``REPORTS``) with its mismatch counts and a histogram of the
mismatches' distances to their boundary; the test session prints them at the end.
"""

from __future__ import annotations

import dataclasses

import numpy as np

from . import fp4q_oracle as o

REL_TOL = 1e-5
MAX_MISMATCH_FRACTION = 1e-4

# distance-to-boundary histogram: decades below the tolerance, then "above it" (unflagged)
HIST_EDGES = (0.0, 1e-9, 1e-8, 1e-7, 1e-6, REL_TOL)
HIST_LABELS = ("<1e-9", "1e-9..1e-8", "1e-8..1e-7", "1e-7..1e-6", "1e-6..1e-5", ">1e-5")

REPORTS: list = []


@dataclasses.dataclass
class ParityReport:
    label: str
    n: int
    code_mismatch: int
    scale_mismatch_groups: int
    unflagged_code_mismatch: int
    unflagged_scale_mismatch: int
    flagged_elements: int
    flagged_groups: int
    mismatch_elements: int
    zero_sign_forgiven: int
    hist_elements: tuple
    hist_groups: tuple

    def ok(self, count_bound: bool = True) -> bool:
        subset = self.unflagged_code_mismatch == 0 and self.unflagged_scale_mismatch == 0
        if not count_bound:
            return subset
        return subset and self.mismatch_elements <= MAX_MISMATCH_FRACTION * max(self.n, 1)

    def merge(self, other: "ParityReport") -> "ParityReport":
        """The report of two disjoint parts of one tensor (row chunks) taken together."""
        add = lambda a, b: tuple(x + y for x, y in zip(a, b))
        return ParityReport(
            label=self.label, n=self.n + other.n,
            code_mismatch=self.code_mismatch + other.code_mismatch,
            scale_mismatch_groups=self.scale_mismatch_groups + other.scale_mismatch_groups,
            unflagged_code_mismatch=self.unflagged_code_mismatch + other.unflagged_code_mismatch,
            unflagged_scale_mismatch=self.unflagged_scale_mismatch + other.unflagged_scale_mismatch,
            flagged_elements=self.flagged_elements + other.flagged_elements,
            flagged_groups=self.flagged_groups + other.flagged_groups,
            mismatch_elements=self.mismatch_elements + other.mismatch_elements,
            zero_sign_forgiven=self.zero_sign_forgiven + other.zero_sign_forgiven,
            hist_elements=add(self.hist_elements, other.hist_elements),
            hist_groups=add(self.hist_groups, other.hist_groups))

    def line(self) -> str:
        he = " ".join(f"{l}:{c}" for l, c in zip(HIST_LABELS, self.hist_elements) if c)
        hg = " ".join(f"{l}:{c}" for l, c in zip(HIST_LABELS, self.hist_groups) if c)
        exact = "bit-exact" if self.mismatch_elements == 0 and self.zero_sign_forgiven == 0 else \
            f"{self.mismatch_elements} elements differ ({self.mismatch_elements / max(self.n, 1):.2e})"
        return (f"{self.label}: n={self.n} {exact}; codes {self.code_mismatch} (unflagged "
                f"{self.unflagged_code_mismatch}), scale groups {self.scale_mismatch_groups} (unflagged "
                f"{self.unflagged_scale_mismatch}); |F| {self.flagged_elements} el + {self.flagged_groups} gr; "
                f"zero-sign forgiven {self.zero_sign_forgiven}"
                + (f"; element distances [{he}]" if he else "") + (f"; group distances [{hg}]" if hg else ""))


def _histogram(d: np.ndarray) -> tuple:
    d = np.asarray(d, np.float64).reshape(-1)
    counts = [int(np.sum((d >= lo) & (d < hi))) for lo, hi in zip(HIST_EDGES[:-1], HIST_EDGES[1:])]
    counts[-1] += int(np.sum(d == REL_TOL))
    counts.append(int(np.sum(d > REL_TOL)))
    return tuple(counts)


def small_zero(res: dict, tol: float = REL_TOL) -> np.ndarray:
    """Elements whose exact rotated value lies within the rotated-value tolerance of zero:
    |y64| <= tol * ||block||_2 (the Hadamard block's norm; for b = 1 only y64 = 0 itself)."""
    y64 = res["y64"]
    M, K = y64.shape
    b = res["block"]
    nb = np.linalg.norm(y64.reshape(M, K // b, b), axis=2)
    return (np.abs(y64).reshape(M, K // b, b) <= tol * nb[..., None]).reshape(M, K)


def compare(res: dict, codes_gpu: np.ndarray, scales_gpu: np.ndarray, tol: float = REL_TOL,
            label: str = "", macro_gpu=None) -> ParityReport:
    """Apply the parity rule to one result.  A group whose scale byte (or, for MBS, macro
    byte: pass ``macro_gpu``) differs from the oracle's is judged as a whole by its group
    distance; inside a group whose scale agrees, the divisor is the same on both sides, so
    every differing code must be flagged on its own.  (An MBS result compared without
    ``macro_gpu`` cannot tell, and lets a flagged group forgive its codes.)"""
    codes_gpu = np.asarray(codes_gpu, np.uint8)
    scales_gpu = np.asarray(scales_gpu, np.uint8)
    assert codes_gpu.shape == res["codes"].shape, (codes_gpu.shape, res["codes"].shape)
    assert scales_gpu.shape == res["scales"].shape
    g = res["group"]
    qo = o.unpack_nibbles(res["codes"])
    qg = o.unpack_nibbles(codes_gpu)
    M, K = qo.shape
    zero_pair = ((qo & 7) == 0) & ((qg & 7) == 0) & (qo != qg)
    forgiven = zero_pair & small_zero(res, tol)
    diff = (qo != qg) & ~forgiven
    d_el, d_gr = o.boundary_distance(res)
    el, gr = d_el <= tol, d_gr <= tol
    changed = res["scales"] != scales_gpu          # groups whose divisor differs
    unflagged_macro = 0
    mbs = res["fmt"] == o.MXFP4_MBS
    if mbs and macro_gpu is not None:
        macro_gpu = np.asarray(macro_gpu, np.uint8)
        assert macro_gpu.shape == res["macro"].shape
        mdiff = res["macro"] != macro_gpu
        unflagged_macro = int((mdiff & ~(o.mbs_macro_distance(res) <= tol)).sum())
        changed = changed | np.repeat(mdiff, o.MBS_MACRO // g, axis=1)
    ch_el = np.repeat(changed, g, axis=1)
    gr_el = np.repeat(gr, g, axis=1)
    if mbs and macro_gpu is None:
        unflagged_codes = diff & ~(el | gr_el) & ~ch_el
    else:
        unflagged_codes = diff & ~el & ~ch_el
    unflagged_scales = int((changed & ~gr).sum()) + unflagged_macro
    mismatch_el = diff | ch_el
    return ParityReport(
        label=label,
        n=M * K,
        code_mismatch=int(diff.sum()),
        scale_mismatch_groups=int(changed.sum()),
        unflagged_code_mismatch=int(unflagged_codes.sum()),
        unflagged_scale_mismatch=unflagged_scales,
        flagged_elements=int(el.sum()),
        flagged_groups=int(gr.sum()),
        mismatch_elements=int(mismatch_el.sum()),
        zero_sign_forgiven=int(forgiven.sum()),
        hist_elements=_histogram(d_el[diff & ~ch_el]),
        hist_groups=_histogram(d_gr[changed]),
    )


def assert_parity(res: dict, codes_gpu, scales_gpu, label: str = "", count_bound: bool = True,
                  macro_gpu=None) -> ParityReport:
    """count_bound=False keeps only "every mismatch is flagged": for inputs built to sit on
    ties (exact midpoints, powers of two), where near-ties are dense by construction."""
    rep = compare(res, codes_gpu, scales_gpu, label=label, macro_gpu=macro_gpu)
    REPORTS.append(rep)
    assert rep.ok(count_bound), rep.line()
    return rep


def record(rep: ParityReport, count_bound: bool = True) -> ParityReport:
    """Record a report made elsewhere (a merged, row-chunked one) and apply the rule to it."""
    REPORTS.append(rep)
    assert rep.ok(count_bound), rep.line()
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
