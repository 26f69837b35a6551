"""Pins of the parity rule's flagged set F (oracle.boundary_distance / oracle.flags) and of
the comparison itself (oracle.parity.compare), against hand-placed values.

F decides which mismatches the GPU path is forgiven, so it is pinned on both sides of
every edge: an element or group placed 5e-6 (relative) from a boundary is flagged, one
placed 2e-5 away is not, for every E2M1 midpoint and every scale rule's boundary.  The
boundaries come from the definitions, not from the oracle's code:
  * E2M1 codes change at the midpoints between neighbouring magnitudes of
    {0, .5, 1, 1.5, 2, 3, 4, 6} ("TORQ", 1. Problemstellung: the e2m1 codebook);
  * the floor (OCP) exponent floor(log2 A) - 2 steps where A crosses a power of two;
  * the ceil exponent ceil(log2(A / 6)) steps where A crosses 6 * 2^j = 1.5 * 2^(j + 2)
    ("Unveiling the Potential of Quantization with MXFP4", Methodologie 1: the standard
    rule maps the block maximum into (3, 6]);
  * OAS also steps where A / X crosses 3.5, i.e. A = 1.75 * 2^k (same section: [3, 3.5] is
    pushed to [6, 7]);
  * an E4M3 block scale steps halfway between two neighbouring E4M3 values;
  * an MBS macro byte ceil(256 f) steps where 256 f crosses an integer.
test_oracle_mutations.py plants mistakes in F (a wider or shifted window, a lost
boundary, the wrong divisor) and shows these pins catch each."""

import numpy as np
import pytest

import oracle as o
from oracle import parity

NEAR = 5e-6       # inside the 1e-5 window
FAR = 2e-5        # outside it


def mx_res(y_rows, S_rows, rule=o.SCALE_FLOOR_OCP, fmt=o.MXFP4, group=32, macro=None):
    """A hand-made oracle result: y64 (M, K) and the per-group divisor S64 (M, K/group)."""
    y = np.asarray(y_rows, np.float64)
    res = {"y64": y, "group": group, "block": 1, "S64": np.asarray(S_rows, np.float64), "rule": rule,
           "fmt": fmt, "tensor_scale": None}
    if macro is not None:
        res["macro"] = np.asarray(macro, np.uint8)
    return res


def nv_res(y_rows, S_rows, s_g):
    y = np.asarray(y_rows, np.float64)
    return {"y64": y, "group": 16, "block": 1, "S64": np.asarray(S_rows, np.float64), "rule": o.SCALE_NV_STATIC,
            "fmt": o.NVFP4, "tensor_scale": np.float32(s_g)}


def element_row(values, S=1.0, group=32):
    """One group: the probe values in its first slots and an amax of 6 S (so the floor scale
    is S), the rest 0."""
    row = np.zeros(group)
    row[:len(values)] = values
    row[-1] = 6.0 * S
    return row


MIDPOINTS = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]


@pytest.mark.parametrize("S", [1.0, 0.125, 64.0])
def test_element_flags_at_every_midpoint(S):
    probes = []
    for mp in MIDPOINTS:
        probes += [mp, mp * (1 + NEAR), mp * (1 - NEAR), mp * (1 + FAR), mp * (1 - FAR)]
    rows = []
    for i in range(0, len(probes), 5):
        rows.append(element_row([p * S for p in probes[i:i + 5]], S))
    res = mx_res(rows, np.full((len(rows), 1), S))
    el, gr = o.flags(res)
    for r in range(len(rows)):
        assert list(el[r, :5]) == [True, True, True, False, False], (S, MIDPOINTS[r], el[r, :5])
        assert el[r, 5:31].sum() == 0           # zeros: no boundary
    # the negative side is the same
    neg = mx_res([-r for r in rows], np.full((len(rows), 1), S))
    assert np.array_equal(o.flags(neg)[0], el)


def test_element_flags_use_the_group_divisor():
    """A value on a midpoint of y itself, but not of y / S, is not flagged (and vice versa)."""
    S = 0.125
    res = mx_res([element_row([0.25, 0.25 * S, 5.0, 5.0 * S * (1 + NEAR)], S)], [[S]])
    el, _ = o.flags(res)
    assert list(el[0, :4]) == [False, True, False, True]


def test_values_between_midpoints_are_not_flagged():
    vals = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, 0.6, 2.2, 4.4, 5.9, 7.5, 100.0]
    res = mx_res([element_row(vals)], [[1.0]])
    el, _ = o.flags(res)
    assert not el[0, :len(vals)].any()


def group_rows(amaxes, group=32):
    """One group per amax: the amax in slot 0, a small value elsewhere."""
    rows = np.zeros((len(amaxes), group))
    rows[:, 0] = amaxes
    rows[:, 1] = np.asarray(amaxes) * 0.3
    return rows


def group_flags(rule, amaxes):
    rows = group_rows(amaxes)
    e = o.mx_scale_exponent(np.max(np.abs(rows), axis=1, keepdims=True).astype(np.float32), rule)
    return o.flags(mx_res(rows, np.ldexp(1.0, e), rule=rule))[1][:, 0]


def edges(base, k):
    a = base * 2.0 ** k
    return [a, a * (1 + NEAR), a * (1 - NEAR), a * (1 + FAR), a * (1 - FAR)]


EXPECT = [True, True, True, False, False]


@pytest.mark.parametrize("k", [-10, -1, 0, 3, 20])
def test_group_flags_floor(k):
    assert list(group_flags(o.SCALE_FLOOR_OCP, edges(1.0, k))) == EXPECT
    assert not group_flags(o.SCALE_FLOOR_OCP, edges(1.5, k)[:3]).any()
    assert not group_flags(o.SCALE_FLOOR_OCP, edges(1.75, k)[:3]).any()


@pytest.mark.parametrize("k", [-10, -1, 0, 3, 20])
def test_group_flags_ceil(k):
    assert list(group_flags(o.SCALE_CEIL_NOCLIP, edges(1.5, k))) == EXPECT
    assert not group_flags(o.SCALE_CEIL_NOCLIP, edges(1.0, k)[:3]).any()
    assert not group_flags(o.SCALE_CEIL_NOCLIP, edges(1.75, k)[:3]).any()


@pytest.mark.parametrize("k", [-10, -1, 0, 3, 20])
def test_group_flags_oas(k):
    assert list(group_flags(o.SCALE_OAS, edges(1.75, k))) == EXPECT
    assert list(group_flags(o.SCALE_OAS, edges(1.5, k))) == EXPECT
    assert not group_flags(o.SCALE_OAS, edges(1.0, k)[:3]).any()


def test_the_ceil_boundary_is_where_the_exponent_steps():
    """Independent of F: the scale byte really does change across each rule's boundary (and
    nowhere in between), so F's places are the right ones."""
    for rule, base in ((o.SCALE_FLOOR_OCP, 1.0), (o.SCALE_CEIL_NOCLIP, 1.5), (o.SCALE_OAS, 1.75)):
        for k in (-3, 0, 5):
            a = base * 2.0 ** k
            lo = o.mx_scale_exponent(np.float32([a * (1 - FAR)]), rule)[0]
            hi = o.mx_scale_exponent(np.float32([a * (1 + FAR)]), rule)[0]
            assert hi != lo, (rule, k)


def test_zero_group_has_no_flags():
    res = mx_res([np.zeros(32)], [[2.0 ** -127]])
    el, gr = o.flags(res)
    assert not el.any() and not gr.any()


E4M3_MIDPOINTS = [1.0625, 1.5 * 2.0 ** -9, 416.0 + 16.0, 0.5 * (0.875 + 0.9375)]


@pytest.mark.parametrize("s_g", [1.0, 0.5, 3.0e-3])
def test_nv_group_flags_at_e4m3_midpoints(s_g):
    """s_b = A / (6 s_g): flagged within 1e-5 of a midpoint between E4M3 neighbours (1.0625 between
    1 and 1.125; 1.5 * 2^-9 between the first two subnormals; 432 between 416 and 448;
    0.90625 between 0.875 and 0.9375), not at an E4M3 value itself."""
    amaxes = []
    for m in E4M3_MIDPOINTS:
        amaxes += [6.0 * s_g * v for v in (m, m * (1 + NEAR), m * (1 - NEAR), m * (1 + FAR), m * (1 - FAR))]
    amaxes += [6.0 * s_g * v for v in (1.0, 1.125, 448.0, 2.0 ** -9)]
    rows = group_rows(amaxes, 16)
    s_b = (np.max(np.abs(rows), axis=1) / (6.0 * s_g)).astype(np.float32)
    S = o.e4m3_decode(o.e4m3_encode(s_b)) * s_g
    gr = o.flags(nv_res(rows, S[:, None], s_g))[1][:, 0]
    assert list(gr[:20]) == EXPECT * 4
    assert not gr[20:].any()


def test_nv_group_flags_use_the_tensor_scale():
    """An amax on a midpoint under s_g = 1 is not flagged under s_g = 0.7 (and the reverse)."""
    rows = group_rows([6.0 * 1.0625, 6.0 * 0.7 * 1.0625], 16)
    gr = o.flags(nv_res(rows, np.ones((2, 1)), 0.7))[1][:, 0]
    assert list(gr) == [False, True]


def test_mbs_macro_flags():
    """m8 = ceil(256 f) steps where 256 f is an integer: A_M = 6 (1 + t / 256)."""
    ts = [43.0, 43.0 + 2.0e-3, 43.0 - 2.0e-3, 43.0 + 3.0e-3, 43.0 - 3.0e-3, 43.5, 200.25]
    rows = np.zeros((len(ts), 128))
    rows[:, 5] = [6.0 * (1 + t / 256.0) for t in ts]
    res = {"y64": rows, "block": 1}
    d = o.mbs_macro_distance(res)[:, 0]
    assert list(d <= 1e-5) == [True, True, True, False, False, False, False]
    # and through F: every group of a flagged macro block is flagged
    r8 = o.rotate_quantize_mbs(np.zeros((len(ts), 128), np.uint16), 32, 1, o.SCALE_FLOOR_OCP)
    r8["y64"] = rows
    r8["macro"] = o.mbs_macro_byte(np.max(np.abs(rows), axis=1, keepdims=True).astype(np.float32))
    gr = o.flags(r8)[1]
    assert list(gr.all(axis=1)) == [True, True, True, False, False, False, False]


# ---- the comparison (oracle.parity.compare)

def _res_b2(pairs):
    """b = 2 rotations of bf16 pairs: y = ((x0 + x1), (x0 - x1)) / sqrt 2."""
    import test_oracle_pins as pins
    x = np.zeros((len(pairs), 32), np.float32)
    for i, (a, b) in enumerate(pairs):
        x[i, 0], x[i, 1] = a, b
        x[i, 2] = 4.0                      # the group's amax: 4 / sqrt 2 -> floor e = 0
    return o.rotate_quantize(pins.bf16(x), o.MXFP4, 32, 2, o.SCALE_FLOOR_OCP)


def test_compare_forgives_a_zero_sign_only_near_zero():
    # row 0: x0 = x1 -> y1 = 0 exactly; row 1: y1 = -(2^-7) / sqrt 2, which rounds to a zero
    # magnitude but is 0.4 % of the block norm, far outside the rotated-value tolerance
    res = _res_b2([(1.0, 1.0), (1.0, 1.0 + 2.0 ** -7)])
    q = o.unpack_nibbles(res["codes"])
    assert (q[0, 1] & 7) == 0 and (q[1, 1] & 7) == 0 and q[1, 1] == 0x8
    flipped = q.copy()
    flipped[0, 1] ^= 0x8
    rep = parity.compare(res, o.pack_nibbles(flipped), res["scales"])
    assert rep.ok() and rep.zero_sign_forgiven == 1 and rep.mismatch_elements == 0
    flipped = q.copy()
    flipped[1, 1] ^= 0x8                    # +0 where y is clearly negative
    rep = parity.compare(res, o.pack_nibbles(flipped), res["scales"])
    assert rep.unflagged_code_mismatch == 1 and not rep.ok(count_bound=False)


def test_compare_judges_codes_in_an_agreeing_group_on_their_own():
    """A flagged group does not forgive an unflagged code when both sides chose the same scale."""
    rows = group_rows([1.0 * (1 + NEAR)])           # floor: group flagged
    rows[0, 2] = 0.6                                 # an element far from any midpoint
    x_res = mx_res(rows, [[2.0 ** -2]])
    x_res["codes"] = o.pack_nibbles(o.e2m1_encode((rows / 2.0 ** -2).astype(np.float32)))
    x_res["scales"] = np.array([[125]], np.uint8)
    q = o.unpack_nibbles(x_res["codes"])
    bad = q.copy()
    bad[0, 2] ^= 0x1
    rep = parity.compare(x_res, o.pack_nibbles(bad), x_res["scales"])
    assert rep.flagged_groups == 1 and rep.unflagged_code_mismatch == 1
    # with the scale byte also different, the whole flagged group is forgiven
    rep = parity.compare(x_res, o.pack_nibbles(bad), x_res["scales"] + 1)
    assert rep.unflagged_code_mismatch == 0 and rep.unflagged_scale_mismatch == 0


def test_compare_counts_and_histogram():
    rows = np.stack([element_row([0.25 * (1 + 3e-9), 0.25 * (1 + 3e-6), 1.0])])
    res = mx_res(rows, [[1.0]])
    res["codes"] = o.pack_nibbles(o.e2m1_encode(rows.astype(np.float32)))
    res["scales"] = np.array([[127]], np.uint8)
    q = o.unpack_nibbles(res["codes"])
    bad = q.copy()
    bad[0, 0] ^= 0x1
    bad[0, 1] ^= 0x1
    rep = parity.compare(res, o.pack_nibbles(bad), res["scales"], label="probe")
    assert rep.code_mismatch == 2 and rep.unflagged_code_mismatch == 0
    assert rep.hist_elements == (0, 1, 0, 0, 1, 0)
    assert "probe" in rep.line()
    bad[0, 2] ^= 0x1
    rep = parity.compare(res, o.pack_nibbles(bad), res["scales"])
    assert rep.hist_elements[-1] == 1 and rep.unflagged_code_mismatch == 1
