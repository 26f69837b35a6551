"""Pins of the oracle's quantization-error energies and QSNR (CPU only).

Sources: "Bridging the Gap Between Promise and Performance for Microscaling FP4
Quantization", Technische Zusammenfassung, 2. Methodik, "Theoretische Analyse der Fehler"
(quantization MSE; on Laplace-like data a block rotation improves MXFP4 and worsens NVFP4
under round-to-nearest); "Unveiling the Potential of Quantization with MXFP4",
Technische samenvatting, Methodologie 1 (Overflow-Aware Scaling gains about 0.5 dB QSNR
over the rule that maps the block maximum into (3, 6]).

Each pin checks the oracle against something other than its own formula: an invariant of
the orthonormal rotation (the energies in the unrotated domain, through the inverse
rotation), data exactly on the quantization grid, hand-worked groups, and the trends the
pages state."""

import math

import numpy as np
import pytest

import oracle as o
from microscaling_fp4_quantization_b200 import workloads as W

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def bf16(a) -> np.ndarray:
    return W.f32_to_bf16_bits(np.asarray(a, np.float32))


def laplace_rows(M=128, K=4096, seed=7):
    return bf16(np.random.default_rng(seed).laplace(size=(M, K)))


def test_energies_match_the_unrotated_domain():
    """H_b / sqrt(b) is orthonormal: sum x^2 = sum y^2, and the error of the dequantized
    values rotated back equals the error in the rotated domain.  700 rows with 512-row chunks
    leaves a ragged last chunk."""
    rng = np.random.default_rng(3)
    xb = bf16(rng.standard_normal((700, 256)) * np.exp(rng.standard_normal((700, 1))))
    x = o.bf16_to_f64(xb)
    for fmt, g, b, rule in ((o.MXFP4, 32, 32, o.SCALE_FLOOR_OCP), (o.MXFP4, 32, 128, o.SCALE_CEIL_NOCLIP),
                            (o.NVFP4, 16, 16, o.SCALE_NV_DYNAMIC), (o.NVFP4, 16, 64, o.SCALE_NV_DYNAMIC)):
        qe = o.quant_error(xb, fmt, g, b, rule)
        ts = qe["tensor_scale"]
        res = o.rotate_quantize(xb, fmt, g, b, rule, ts)
        xhat = o.dequantize(res["codes"], res["scales"], fmt, g, b, ts, unrotate_back=True)
        noise_x = float(np.sum((x - xhat) ** 2))
        assert qe["signal"] == pytest.approx(float(np.sum(x * x)), rel=1e-12)
        # dequantize rounds q * S to fp32: 2^-24 relative per element
        assert qe["noise"] == pytest.approx(noise_x, rel=1e-6), (fmt, b)
        assert qe["mse"] == pytest.approx(noise_x / x.size, rel=1e-6)


def test_values_on_the_grid_have_no_error():
    """MX floor, no rotation: a group whose maximum is 6 * 2^k and whose values are E2M1
    magnitudes times 2^k quantizes exactly."""
    rng = np.random.default_rng(5)
    mags = np.array(o.E2M1_MAGNITUDES)
    M, K = 8, 256
    vals = rng.choice(mags, size=(M, K)) * rng.choice([-1.0, 1.0], size=(M, K))
    vals[:, ::32] = 6.0
    vals *= np.exp2(rng.integers(-20, 20, size=(M, K // 32))).repeat(32, axis=1)
    qe = o.quant_error(bf16(vals), o.MXFP4, 32, 1, o.SCALE_FLOOR_OCP)
    assert qe["noise"] == 0.0 and qe["qsnr_db"] == math.inf
    assert qe["signal"] == pytest.approx(float(np.sum(vals ** 2)), rel=1e-15)


def test_zero_tensor():
    qe = o.quant_error(np.zeros((4, 64), np.uint16), o.NVFP4, 16, 16, o.SCALE_NV_DYNAMIC)
    assert qe["signal"] == 0.0 and qe["noise"] == 0.0 and qe["qsnr_db"] == math.inf


def test_hand_worked_mx_group():
    """One 32-element group, no rotation: 7 then 31 x 0.3125.
    floor: X = 1; 7 -> 6 (error 1), 0.3125 -> 0.5 (error 0.1875).
    ceil:  X = 2; 3.5 is a tie -> 4, so 7 -> 8 (error 1); 0.15625 -> 0 (error 0.3125).
    OAS:   mantissa 1.75 is not above 1.75, so the floor scale: as floor."""
    row = np.array([[7.0] + [0.3125] * 31])
    xb = bf16(row)
    signal = 49.0 + 31 * 0.3125 ** 2
    for rule, noise in ((o.SCALE_FLOOR_OCP, 1.0 + 31 * 0.1875 ** 2), (o.SCALE_CEIL_NOCLIP, 1.0 + 31 * 0.3125 ** 2),
                        (o.SCALE_OAS, 1.0 + 31 * 0.1875 ** 2)):
        qe = o.quant_error(xb, o.MXFP4, 32, 1, rule)
        assert qe["signal"] == signal
        assert qe["noise"] == noise, rule
        assert qe["qsnr_db"] == pytest.approx(10 * math.log10(signal / noise), rel=1e-14)


def test_hand_worked_nv_group():
    """One 16-element group, no rotation, s_g = 1: 5 then 15 x 1.
    s_b = 5/6 -> E4M3 0.8125; 5 / 0.8125 = 6.15 -> 6 (yhat 4.875, error 0.125);
    1 / 0.8125 = 1.23 -> 1 (yhat 0.8125, error 0.1875)."""
    xb = bf16(np.array([[5.0] + [1.0] * 15]))
    qe = o.quant_error(xb, o.NVFP4, 16, 1, o.SCALE_NV_STATIC, tensor_scale=np.float32(1.0))
    assert qe["signal"] == 40.0
    assert qe["noise"] == 0.125 ** 2 + 15 * 0.1875 ** 2


def test_rotation_helps_mxfp4_on_laplace_rows():
    xb = laplace_rows()
    base = o.quant_error(xb, o.MXFP4, 32, 1, o.SCALE_FLOOR_OCP)["qsnr_db"]
    for b in (32, 128):
        rot = o.quant_error(xb, o.MXFP4, 32, b, o.SCALE_FLOOR_OCP)["qsnr_db"]
        assert rot > base + 0.3, (b, rot, base)


def test_rotation_hurts_nvfp4_rtn_on_laplace_rows():
    xb = laplace_rows()
    base = o.quant_error(xb, o.NVFP4, 16, 1, o.SCALE_NV_DYNAMIC)["qsnr_db"]
    rot = o.quant_error(xb, o.NVFP4, 16, 16, o.SCALE_NV_DYNAMIC)["qsnr_db"]
    assert rot < base - 0.1, (rot, base)


def test_oas_gain_over_the_ceil_rule():
    """About 0.5 dB by the page; on Laplace rows without rotation it lands in (0.3, 0.8)."""
    xb = laplace_rows()
    ceil = o.quant_error(xb, o.MXFP4, 32, 1, o.SCALE_CEIL_NOCLIP)["qsnr_db"]
    oas = o.quant_error(xb, o.MXFP4, 32, 1, o.SCALE_OAS)["qsnr_db"]
    assert 0.3 < oas - ceil < 0.8, (oas, ceil)
