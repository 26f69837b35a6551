"""Pins of the oracle's MBS-Static quantizer (CPU only).

Source: "Unveiling the Potential of Quantization with MXFP4: Strategies for Quantization
Error Reduction", Technische samenvatting, Methodologie 2 (Macro Block Scaling: a macro
block of 128 elements gets one extra scale factor with 8 mantissa bits; MBS-Static takes it
directly from the macro block's maximum; the values are scaled by it before the standard
MXFP4 quantization).  The reading pinned here: s_M is the mantissa of A_M / 6 rounded up to
8 fraction bits, so that the macro block's maximum lands on the top E2M1 value.

Each pin checks the oracle against something other than its own formula: a hand-worked
macro block, the reduction to plain MXFP4 when the maximum is already 6 * 2^k, a brute-force
search for the byte, the property that the maximum always takes the top code under the
ceil rule, the unrotated-domain invariant of the error, and the gain the page claims."""

import math

import numpy as np
import pytest

import oracle as o
from microscaling_fp4_quantization_b200 import workloads as W

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def bf16(a):
    return W.f32_to_bf16_bits(np.asarray(a, np.float32))


def test_hand_worked_macro_block():
    """7 then 127 x 0.3125, no rotation, floor rule.  fp32(7/6) = 1.1666666 = 2^0 (1 + f),
    256 f = 42.67 -> m8 = 43, s_M = 299/256.  Group 0: 7 / s_M = 5.993 -> e = 0, code 6.0
    (yhat 6 * 299/256 = 7.0078125); 0.3125 / s_M = 0.2676 -> 0.5 (yhat 0.583984375).
    Groups 1-3: maximum 0.2676 -> e = -4, 0.2676 * 16 = 4.28 -> 4 (yhat 4/16 * 299/256)."""
    x = bf16([[7.0] + [0.3125] * 127])
    r = o.rotate_quantize_mbs(x, 32, 1, o.SCALE_FLOOR_OCP)
    assert r["macro"].tolist() == [[43]]
    assert r["scales"].tolist() == [[127, 123, 123, 123]]
    q = o.unpack_nibbles(r["codes"])[0]
    assert q[0] == 7 and np.all(q[1:32] == 1) and np.all(q[32:] == 6)
    xh = o.dequantize_mbs(r["codes"], r["scales"], r["macro"], 32, 1)[0]
    sM = 299 / 256
    assert xh[0] == 6 * sM and xh[1] == 0.5 * sM and xh[40] == 0.25 * sM
    qe = o.quant_error(x, o.MXFP4_MBS, 32, 1, o.SCALE_FLOOR_OCP)
    noise = (7 - 6 * sM) ** 2 + 31 * (0.3125 - 0.5 * sM) ** 2 + 96 * (0.3125 - 0.25 * sM) ** 2
    assert qe["noise"] == pytest.approx(noise, rel=1e-15)
    assert qe["signal"] == 49 + 127 * 0.3125 ** 2


def test_reduces_to_mxfp4_when_the_maximum_is_six_times_a_power_of_two():
    rng = np.random.default_rng(4)
    M, K = 16, 512
    x = rng.standard_normal((M, K))
    mb = np.abs(x.reshape(M, K // 128, 128)).max(axis=2)
    top = 6 * np.exp2(np.ceil(np.log2(mb / 6)) + 1)       # above every element of its block
    xr = x.reshape(M, K // 128, 128)
    xr[:, :, 5] = top * np.sign(xr[:, :, 5] + 0.5)
    xb = bf16(xr.reshape(M, K))
    for rule in (o.SCALE_FLOOR_OCP, o.SCALE_CEIL_NOCLIP, o.SCALE_OAS):
        r = o.rotate_quantize_mbs(xb, 32, 1, rule)
        p = o.rotate_quantize(xb, o.MXFP4, 32, 1, rule)
        assert np.all(r["macro"] == 0)
        assert np.array_equal(r["codes"], p["codes"]) and np.array_equal(r["scales"], p["scales"])


def test_macro_byte_brute_force():
    """m8 is the smallest m in 0..256 with 1 + m/256 >= the mantissa of fp32(A/6); 256 -> 0."""
    rng = np.random.default_rng(8)
    A = np.concatenate([np.exp(rng.uniform(-60, 60, 4000)), np.array([6.0, 12.0, 7.0, 6.0 * 255 / 256, 0.0,
                                                                       6.0 * (1 + 255.5 / 256)])]).astype(np.float32)
    got = o.mbs_macro_byte(A)
    for a, g in zip(A, got):
        r = float(np.float32(a) / np.float32(6.0))
        if r == 0:
            assert g == 0
            continue
        mant = r / 2.0 ** math.floor(math.log2(r))
        m = next(m for m in range(257) if 1 + m / 256 >= mant)
        assert g == m % 256, (a, g, m)


def test_block_maximum_takes_the_top_code_under_the_ceil_rule():
    """A_M / s_M <= 6 * 2^E and above 6 * 2^E (1 - 2^-8): the ceil rule never bumps the
    exponent of the maximum's group, so the maximum's code magnitude is 7 (6.0)."""
    rng = np.random.default_rng(9)
    M, K = 64, 1024
    xb = bf16(rng.laplace(size=(M, K)) * np.exp(rng.normal(0, 2, (M, 1))))
    for b in (1, 32):
        r = o.rotate_quantize_mbs(xb, 32, b, o.SCALE_CEIL_NOCLIP)
        q = o.unpack_nibbles(r["codes"]).reshape(M, K // 128, 128)
        y = np.abs(r["y32"]).reshape(M, K // 128, 128)
        idx = np.argmax(y, axis=2)
        top = np.take_along_axis(q, idx[..., None], axis=2)[..., 0] & 7
        assert np.all(top == 7), b


def test_dequantized_values_are_exact():
    rng = np.random.default_rng(10)
    xb = bf16(rng.standard_normal((8, 256)))
    r = o.rotate_quantize_mbs(xb, 32, 32, o.SCALE_OAS)
    xh = o.dequantize_mbs(r["codes"], r["scales"], r["macro"], 32, 32).astype(np.float64)
    q = o.e2m1_decode(o.unpack_nibbles(r["codes"])).reshape(8, 8, 32)
    assert np.array_equal(xh, (q * r["S64"][..., None]).reshape(8, 256))


def test_error_energies_match_the_unrotated_domain():
    rng = np.random.default_rng(11)
    xb = bf16(rng.laplace(size=(300, 512)))
    x = o.bf16_to_f64(xb)
    for b in (32, 128):
        qe = o.quant_error(xb, o.MXFP4_MBS, 32, b, o.SCALE_FLOOR_OCP, chunk_rows=128)
        r = o.rotate_quantize_mbs(xb, 32, b, o.SCALE_FLOOR_OCP)
        xh = o.dequantize_mbs(r["codes"], r["scales"], r["macro"], 32, b, unrotate_back=True)
        assert qe["signal"] == pytest.approx(float(np.sum(x * x)), rel=1e-12)
        assert qe["noise"] == pytest.approx(float(np.sum((x - xh) ** 2)), rel=1e-9)


def test_mbs_improves_on_mxfp4_on_laplace_rows():
    xb = W.f32_to_bf16_bits(np.random.default_rng(7).laplace(size=(128, 4096)).astype(np.float32))
    for b in (1, 32):
        for rule in (o.SCALE_FLOOR_OCP, o.SCALE_CEIL_NOCLIP, o.SCALE_OAS):
            plain = o.quant_error(xb, o.MXFP4, 32, b, rule)["qsnr_db"]
            mbs = o.quant_error(xb, o.MXFP4_MBS, 32, b, rule)["qsnr_db"]
            assert mbs > plain + 0.2, (b, rule, mbs, plain)
