"""Plant plausible mistakes in the CPU oracle and check that its pins catch each one.

Each mutation replaces one oracle function with a subtly wrong variant (a transposed or
permuted operand, a dropped normalisation, a wrong tie direction, an off-by-one exponent,
a swapped nibble order ...).  The pins in test_oracle_pins.py must then fail."""

import math

import numpy as np
import pytest

import oracle as o
import oracle.fp4q_oracle as core
import test_oracle_pins as pins


def patch(monkeypatch, name, fn):
    monkeypatch.setattr(core, name, fn)
    monkeypatch.setattr(o, name, fn, raising=False)


def fails(fn, *args):
    try:
        fn(*args)
    except AssertionError:
        return True
    return False


_orig_H = core.sylvester_hadamard
_orig_rotate = core.rotate
_orig_e2m1 = core.e2m1_encode
_orig_mx = core.mx_scale_exponent
_orig_e4m3 = core.e4m3_encode
_orig_pack = core.pack_nibbles


def h_columns_swapped(b):
    H = _orig_H(b).copy()
    if b >= 2:
        H[:, [b - 2, b - 1]] = H[:, [b - 1, b - 2]]
    return H


def h_wrong_sign(b):
    H = _orig_H(b).copy()
    if b >= 4:
        H[1, 1] = -H[1, 1]
    return H


def rotate_unnormalised(x_bits, b):
    return _orig_rotate(x_bits, b) * math.sqrt(b)


def rotate_along_rows(x_bits, b):
    """Rotates across M instead of along K when the shape allows it."""
    x = np.asarray(x_bits)
    if x.shape[0] % b == 0 and x.shape[0] >= b:
        return _orig_rotate(np.ascontiguousarray(x.T), b).T
    return _orig_rotate(np.roll(x, 1, axis=1), b)


def e2m1_ties_away(v):
    """Ties round away from zero instead of to the even code."""
    v = np.asarray(v, np.float32)
    c = _orig_e2m1(v)
    a = np.abs(v.astype(np.float64))
    for mid, up in ((0.25, 1), (0.75, 2), (1.25, 3), (1.75, 4), (2.5, 5), (3.5, 6), (5.0, 7)):
        c = np.where(a == mid, (c & 8) | up, c)
    return c.astype(np.uint8)


def e2m1_no_sign(v):
    return (_orig_e2m1(v) & 7).astype(np.uint8)


def mx_floor_off_by_one(A32, rule):
    e = _orig_mx(A32, rule)
    if rule == o.SCALE_FLOOR_OCP:
        e = np.where(np.asarray(A32) > 0, np.clip(e + 1, -127, 127), e)
    return e


def mx_ceil_wrong_threshold(A32, rule):
    """ceil rule that bumps at m >= 1.5 instead of m > 1.5."""
    e = _orig_mx(A32, rule)
    if rule == o.SCALE_CEIL_NOCLIP:
        A = np.asarray(A32, np.float64)
        m = np.frexp(A)[0] * 2
        e = np.where((A > 0) & (m == 1.5), e + 1, e)
    return e


def e4m3_ties_up(s):
    s32 = np.asarray(s, np.float32)
    c = _orig_e4m3(s32)
    T = o.e4m3_table()
    mids = (T[1:] + T[:-1]) / 2
    a = s32.astype(np.float64)
    hit = np.isin(a, mids)
    idx = np.searchsorted(mids, a)
    return np.where(hit, np.minimum(idx + 1, 126), c).astype(np.uint8)


def pack_swapped(codes):
    c = np.asarray(codes, np.uint8)
    return (c[..., 1::2] | (c[..., 0::2] << 4)).astype(np.uint8)


MUTATIONS = [
    ("sylvester_hadamard", h_columns_swapped,
     [(pins.test_sylvester_closed_form, 32), (pins.test_rotation_matches_fast_butterfly, 32)]),
    ("sylvester_hadamard", h_wrong_sign,
     [(pins.test_sylvester_closed_form, 16), (pins.test_rotation_of_basis_vectors_gives_rows, 16)]),
    ("rotate", rotate_unnormalised,
     [(pins.test_rotation_norm_inverse_and_gemm_identity, 32), (pins.test_rotation_matches_fast_butterfly, 16)]),
    ("rotate", rotate_along_rows,
     [(pins.test_rotation_matches_fast_butterfly, 16), (pins.test_rotation_of_basis_vectors_gives_rows, 32)]),
    ("e2m1_encode", e2m1_ties_away,
     [(pins.test_e2m1_dense_sweep_against_ml_dtypes_cast,), (pins.test_mx_worked_groups,)]),
    ("e2m1_encode", e2m1_no_sign,
     [(pins.test_e2m1_dense_sweep_against_ml_dtypes_cast,), (pins.test_mx_worked_groups,)]),
    ("mx_scale_exponent", mx_floor_off_by_one,
     [(pins.test_mx_exponent_brute_force, o.SCALE_FLOOR_OCP), (pins.test_mx_worked_groups,)]),
    ("mx_scale_exponent", mx_ceil_wrong_threshold,
     [(pins.test_mx_exponent_brute_force, o.SCALE_CEIL_NOCLIP), (pins.test_mx_worked_groups,)]),
    ("e4m3_encode", e4m3_ties_up,
     [(pins.test_e4m3_encode_against_torch_cast,)]),
    ("pack_nibbles", pack_swapped,
     [(pins.test_pack_nibbles_order,), (pins.test_mx_worked_groups,)]),
]


@pytest.mark.parametrize("name,fn,catchers", MUTATIONS, ids=[m[1].__name__ for m in MUTATIONS])
def test_pins_catch_planted_mistake(monkeypatch, name, fn, catchers):
    patch(monkeypatch, name, fn)
    for catcher in catchers:
        assert fails(catcher[0], *catcher[1:]), f"{catcher[0].__name__} missed {fn.__name__}"


def test_nv_divisor_mistake_is_caught(monkeypatch):
    """s_b computed with A / (448 s_g) instead of A / (6 s_g)."""
    orig = core.rotate_quantize

    def wrong(x_bits, fmt, group, block, rule, tensor_scale=None):
        if fmt == o.NVFP4 and tensor_scale is not None:
            tensor_scale = np.float32(tensor_scale) * np.float32(448.0 / 6.0)
        return orig(x_bits, fmt, group, block, rule, tensor_scale)

    patch(monkeypatch, "rotate_quantize", wrong)
    assert fails(pins.test_nv_worked_groups)


# ---- quantization-error energies (pins in test_oracle_qsnr.py)

import test_oracle_qsnr as qpins  # noqa: E402


def _quant_error_variant(kind):
    def qe(x_bits, fmt, group, block, rule, tensor_scale=None, chunk_rows=512):
        x_bits = np.asarray(x_bits, np.uint16)
        M, K = x_bits.shape
        if fmt == o.NVFP4 and tensor_scale is None:
            tensor_scale = o.nv_tensor_scale(o.rotated_amax(x_bits, block))
        res = o.rotate_quantize(x_bits, fmt, group, block, rule, tensor_scale)
        y = res["y64"]
        q = o.e2m1_decode(o.unpack_nibbles(res["codes"])).reshape(M, K // group, group)
        S = res["S64"]
        if kind == "no_tensor_scale" and fmt == o.NVFP4:
            S = S / np.float64(tensor_scale)
        yhat = (q * S[..., None]).reshape(M, K)
        ref = o.bf16_to_f64(x_bits) if kind == "mixed_domain" else y
        err = ref - yhat
        noise = float(np.sum(np.abs(err))) if kind == "abs_error" else float(np.sum(err * err))
        signal = float(np.sum(y * y)) * (block if kind == "unnormalised_signal" else 1)
        qsnr = math.inf if noise == 0 else 10 * math.log10(signal / noise) if signal > 0 else -math.inf
        return {"signal": signal, "noise": noise, "qsnr_db": qsnr, "mse": noise / max(M * K, 1),
                "tensor_scale": tensor_scale}
    qe.__name__ = "quant_error_" + kind
    return qe


QE_MUTATIONS = [
    ("abs_error", [qpins.test_hand_worked_mx_group, qpins.test_hand_worked_nv_group]),
    ("mixed_domain", [qpins.test_energies_match_the_unrotated_domain]),
    ("no_tensor_scale", [qpins.test_energies_match_the_unrotated_domain]),
    ("unnormalised_signal", [qpins.test_energies_match_the_unrotated_domain]),
]


@pytest.mark.parametrize("kind,catchers", QE_MUTATIONS, ids=[m[0] for m in QE_MUTATIONS])
def test_qsnr_pins_catch_planted_mistake(monkeypatch, kind, catchers):
    patch(monkeypatch, "quant_error", _quant_error_variant(kind))
    for catcher in catchers:
        assert fails(catcher), f"{catcher.__name__} missed quant_error_{kind}"


def test_qsnr_variant_without_mistake_passes(monkeypatch):
    """The mutation harness itself: the variant with no planted mistake passes every pin."""
    patch(monkeypatch, "quant_error", _quant_error_variant("none"))
    for pin in (qpins.test_energies_match_the_unrotated_domain, qpins.test_hand_worked_mx_group,
                qpins.test_hand_worked_nv_group):
        pin()


# ---- randomised rotation (pins in test_oracle_signs.py)

import test_oracle_signs as spins  # noqa: E402

_orig_sign_vector = core.sign_vector


def rotate_signs_after(x_bits, b, signs=None):
    """Applies the signs to the rotated values instead of the channels."""
    y = _orig_rotate(x_bits, b)
    return y if signs is None else y * np.asarray(signs, np.float64)[None, :]


def rotate_signs_ignored(x_bits, b, signs=None):
    return _orig_rotate(x_bits, b)


def sign_vector_msb_first(mask_words, K):
    w = np.asarray(mask_words, np.uint32)
    k = np.arange(K)
    bit = (w[k // 32] >> (31 - k % 32).astype(np.uint32)) & np.uint32(1)
    return np.where(bit == 1, -1.0, 1.0)


SIGN_MUTATIONS = [
    ("rotate", rotate_signs_after, [spins.test_rotated_basis_vectors]),
    ("rotate", rotate_signs_ignored, [spins.test_rotated_basis_vectors, spins.test_signs_reach_the_codes_and_the_error]),
    ("sign_vector", sign_vector_msb_first, [spins.test_sign_mask_bit_layout]),
]


@pytest.mark.parametrize("name,fn,catchers", SIGN_MUTATIONS, ids=[m[1].__name__ for m in SIGN_MUTATIONS])
def test_sign_pins_catch_planted_mistake(monkeypatch, name, fn, catchers):
    patch(monkeypatch, name, fn)
    for catcher in catchers:
        assert fails(catcher), f"{catcher.__name__} missed {fn.__name__}"


# ---- MBS-Static (pins in test_oracle_mbs.py)

import test_oracle_mbs as mpins  # noqa: E402

_orig_macro_byte = core.mbs_macro_byte
_orig_rq_mbs = core.rotate_quantize_mbs


def macro_byte_nearest(A_M32):
    """Rounds the mantissa to nearest instead of up."""
    r = (np.asarray(A_M32, np.float32) / np.float32(6.0)).astype(np.float32)
    m, _ = np.frexp(r.astype(np.float64))
    f = np.where(r > 0, 2.0 * m - 1.0, 0.0)
    return (np.rint(f * 256.0).astype(np.int64) % 256).astype(np.uint8)


def macro_byte_amax_not_divided(A_M32):
    """Takes the mantissa of A_M instead of A_M / 6."""
    return _orig_macro_byte(np.asarray(A_M32, np.float32) * np.float32(6.0))


def rq_mbs_macro_64(x_bits, group, block, rule, signs=None):
    """Macro blocks of 64 elements: quantizes each half of a 128-element block on its own."""
    x = np.asarray(x_bits, np.uint16)
    M, K = x.shape
    if K % 128 == 0 and block <= 64:
        halves = x.reshape(M, K // 64, 64)
        pad = np.concatenate([halves, np.zeros_like(halves)], axis=2).reshape(M * K // 64, 128)
        r = _orig_rq_mbs(pad, group, block, rule, signs=None)
        q = o.unpack_nibbles(r["codes"]).reshape(M, K // 64, 128)[:, :, :64].reshape(M, K)
        r["codes"] = o.pack_nibbles(q)
        r["scales"] = r["scales"].reshape(M, K // 64, 4)[:, :, :2].reshape(M, K // 32)
        r["macro"] = r["macro"].reshape(M, K // 64)[:, ::2]
        return r
    return _orig_rq_mbs(x_bits, group, block, rule, signs)


MBS_MUTATIONS = [
    ("mbs_macro_byte", macro_byte_nearest, [mpins.test_macro_byte_brute_force,
                                            mpins.test_block_maximum_takes_the_top_code_under_the_ceil_rule]),
    ("mbs_macro_byte", macro_byte_amax_not_divided, [mpins.test_hand_worked_macro_block,
                                                     mpins.test_macro_byte_brute_force]),
    ("rotate_quantize_mbs", rq_mbs_macro_64, [mpins.test_hand_worked_macro_block]),
]


@pytest.mark.parametrize("name,fn,catchers", MBS_MUTATIONS, ids=[m[1].__name__ for m in MBS_MUTATIONS])
def test_mbs_pins_catch_planted_mistake(monkeypatch, name, fn, catchers):
    patch(monkeypatch, name, fn)
    for catcher in catchers:
        assert fails(catcher), f"{catcher.__name__} missed {fn.__name__}"


# ---- FP4 GEMM (pins in test_oracle_gemm.py)

import test_oracle_gemm as gpins  # noqa: E402

_orig_gemm = core.gemm_fp4


def gemm_no_tensor_scale(a_codes, a_scales, b_codes, b_scales, fmt, a_tensor_scale=None, b_tensor_scale=None):
    return _orig_gemm(a_codes, a_scales, b_codes, b_scales, fmt, 1.0, 1.0)


def gemm_scale_off_by_one(a_codes, a_scales, b_codes, b_scales, fmt, a_tensor_scale=None, b_tensor_scale=None):
    """Reads the E8M0 byte as 2^(byte - 126)."""
    if fmt == o.MXFP4:
        return 4.0 * _orig_gemm(a_codes, a_scales, b_codes, b_scales, fmt)
    return _orig_gemm(a_codes, a_scales, b_codes, b_scales, fmt, a_tensor_scale, b_tensor_scale)


def gemm_b_not_transposed(a_codes, a_scales, b_codes, b_scales, fmt, a_tensor_scale=None, b_tensor_scale=None):
    D = _orig_gemm(a_codes, a_scales, b_codes, b_scales, fmt, a_tensor_scale, b_tensor_scale)
    return D.T if D.shape[0] == D.shape[1] else D[:, ::-1]


GEMM_MUTATIONS = [
    (gemm_no_tensor_scale, [gpins.test_hand_worked_nv_dot_product]),
    (gemm_scale_off_by_one, [gpins.test_hand_worked_mx_dot_product]),
    (gemm_b_not_transposed, [lambda: gpins.test_gemm_equals_dequantize_then_product(o.MXFP4, 32, 32, 0)]),
]


@pytest.mark.parametrize("fn,catchers", GEMM_MUTATIONS, ids=[m[0].__name__ for m in GEMM_MUTATIONS])
def test_gemm_pins_catch_planted_mistake(monkeypatch, fn, catchers):
    patch(monkeypatch, "gemm_fp4", fn)
    for catcher in catchers:
        assert fails(catcher), f"pin missed {fn.__name__}"


# ---- the flagged set F of the parity rule (pins in test_oracle_flags.py)

import test_oracle_flags as fpins  # noqa: E402

_orig_bd = core.boundary_distance
_orig_dsp = core._dist_scaled_power
_orig_mmd = core.mbs_macro_distance


def bd_widened(res):
    """A window three times too wide (3e-5 instead of 1e-5)."""
    el, gr = _orig_bd(res)
    return el / 3.0, gr / 3.0


def dsp_shifted(A, base):
    """Group boundaries shifted by 1e-5 relative (the window centred off the boundary)."""
    return _orig_dsp(np.asarray(A, np.float64) / (1.0 + 1e-5), base)


def dsp_base_ignored(A, base):
    """Every rule measured against powers of two (the floor rule's boundary)."""
    return _orig_dsp(A, 1.0)


def bd_nv_values_not_midpoints(res):
    """NV: distance to the E4M3 values instead of the midpoints between them."""
    el, gr = _orig_bd(res)
    if res["fmt"] != o.NVFP4:
        return el, gr
    y64 = res["y64"]
    M, K = y64.shape
    A = np.abs(y64.reshape(M, K // 16, 16)).max(axis=2)
    s_b = A / (6.0 * np.float64(res["tensor_scale"]))
    T = core.e4m3_table()[1:]
    d = np.min(np.abs(s_b[..., None] - T) / T, axis=-1)
    return el, d


def bd_nv_tensor_scale_ignored(res):
    if res["fmt"] != o.NVFP4:
        return _orig_bd(res)
    return _orig_bd(dict(res, tensor_scale=np.float32(1.0)))


def bd_elements_not_divided(res):
    """Element distances of y itself, not of y / S."""
    return _orig_bd(dict(res, S64=np.ones_like(res["S64"])))[0], _orig_bd(res)[1]


def mmd_unscaled(res):
    """The macro distance in units of 256 f (the window 256 times too wide)."""
    return _orig_mmd(res) * 256.0 / 65536.0


FLAG_MUTATIONS = [
    ("boundary_distance", bd_widened,
     [(fpins.test_element_flags_at_every_midpoint, 1.0), (fpins.test_group_flags_floor, 0)]),
    ("_dist_scaled_power", dsp_shifted,
     [(fpins.test_group_flags_floor, 3), (fpins.test_group_flags_ceil, -1), (fpins.test_group_flags_oas, 0)]),
    ("_dist_scaled_power", dsp_base_ignored,
     [(fpins.test_group_flags_ceil, 0), (fpins.test_group_flags_oas, 3)]),
    ("boundary_distance", bd_nv_values_not_midpoints,
     [(fpins.test_nv_group_flags_at_e4m3_midpoints, 1.0)]),
    ("boundary_distance", bd_nv_tensor_scale_ignored,
     [(fpins.test_nv_group_flags_at_e4m3_midpoints, 0.5), (fpins.test_nv_group_flags_use_the_tensor_scale,)]),
    ("boundary_distance", bd_elements_not_divided,
     [(fpins.test_element_flags_at_every_midpoint, 0.125), (fpins.test_element_flags_use_the_group_divisor,)]),
    ("mbs_macro_distance", mmd_unscaled,
     [(fpins.test_mbs_macro_flags,)]),
]


@pytest.mark.parametrize("name,fn,catchers", FLAG_MUTATIONS, ids=[m[1].__name__ for m in FLAG_MUTATIONS])
def test_flag_pins_catch_planted_mistake(monkeypatch, name, fn, catchers):
    patch(monkeypatch, name, fn)
    for catcher in catchers:
        assert fails(catcher[0], *catcher[1:]), f"{catcher[0].__name__} missed {fn.__name__}"


@pytest.mark.parametrize("shift", ["dropped", "shifted"])
def test_flag_pins_catch_wrong_midpoints(monkeypatch, shift):
    """A midpoint left out (5.0), or every element window centred 1e-5 off its midpoint."""
    mids = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5) if shift == "dropped" else \
        tuple(m * (1 + 1e-5) for m in core.E2M1_MIDPOINTS)
    monkeypatch.setattr(core, "E2M1_MIDPOINTS", mids)
    assert fails(fpins.test_element_flags_at_every_midpoint, 1.0)


def test_flag_pins_catch_a_zero_sign_forgiven_everywhere(monkeypatch):
    """The sign of a zero code forgiven whatever the exact rotated value is."""
    from oracle import parity
    monkeypatch.setattr(parity, "small_zero", lambda res, tol=1e-5: np.ones(res["y64"].shape, bool))
    assert fails(fpins.test_compare_forgives_a_zero_sign_only_near_zero)


def test_flag_pins_catch_group_flags_forgiving_agreeing_groups(monkeypatch):
    """An element mismatch forgiven by its group's flag although both sides chose the same scale."""
    from oracle import parity
    orig = parity.compare

    def lax(res, codes_gpu, scales_gpu, tol=1e-5, label="", macro_gpu=None):
        r = orig(res, codes_gpu, scales_gpu, tol, label, macro_gpu)
        _, gr = core.flags(res, tol)
        qo, qg = core.unpack_nibbles(res["codes"]), core.unpack_nibbles(np.asarray(codes_gpu, np.uint8))
        in_flagged = ((qo != qg) & np.repeat(gr, res["group"], axis=1)).sum()
        r.unflagged_code_mismatch = max(0, r.unflagged_code_mismatch - int(in_flagged))
        return r

    monkeypatch.setattr(parity, "compare", lax)
    assert fails(fpins.test_compare_judges_codes_in_an_agreeing_group_on_their_own)
