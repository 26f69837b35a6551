"""Pins of the oracle's block-scaled FP4 GEMM (CPU only).

Source: "Bridging the Gap Between Promise and Performance for Microscaling FP4
Quantization", Technische Zusammenfassung, 2. Methodik (GPU-Kernel-Unterstützung: FP4
matrix multiplication of the quantized operands) and the English abstract (the rotation is
fused into the weights, so the product of the rotated operands is the layer's product).

The pins check the oracle's GEMM by other routes: hand-worked dot products with known codes
and scales, the oracle's own dequantize (a separate decode) followed by a plain product,
and the rotation identity against X W^T."""

import numpy as np
import pytest

import oracle as o
from microscaling_fp4_quantization_b200 import workloads as W


def pack(codes):
    return o.pack_nibbles(np.asarray(codes, np.uint8))


def test_hand_worked_mx_dot_product():
    """A: 64 codes 0x2 (1.0), scales 2^0 and 2^1; B: 64 codes 0x4 (2.0), scales 2^-1 and 2^0,
    except element 1 of B is 0xC (-2.0).  D = 31 * 1*2*0.5 - 1*2*0.5 + 32 * 2*2*1 = 158."""
    a = pack([[2] * 64])
    b_codes = [4] * 64
    b_codes[1] = 12
    b = pack([b_codes])
    D = o.gemm_fp4(a, np.array([[127, 128]], np.uint8), b, np.array([[126, 127]], np.uint8), o.MXFP4)
    assert D.shape == (1, 1) and D[0, 0] == 158.0


def test_hand_worked_nv_dot_product():
    """A: 16 codes 0x3 (1.5), E4M3 scale 0x38 (1.0), s_g = 0.5; B: 16 codes 0x7 (6.0), E4M3
    scale 0x40 (2.0), s_g = 4.  D = 16 * 1.5*6 * 1*2 * 0.5*4 = 576; element 0 of A set to 0x1
    (0.5) instead: D = 576 - (1.5 - 0.5)*6*2*2 = 552."""
    a = [3] * 16
    a[0] = 1
    D = o.gemm_fp4(pack([a]), np.array([[0x38]], np.uint8), pack([[7] * 16]), np.array([[0x40]], np.uint8),
                   o.NVFP4, np.float32(0.5), np.float32(4.0))
    assert D[0, 0] == 552.0


@pytest.mark.parametrize("fmt,g,b,rule", [(o.MXFP4, 32, 32, o.SCALE_FLOOR_OCP), (o.NVFP4, 16, 16, o.SCALE_NV_DYNAMIC)])
def test_gemm_equals_dequantize_then_product(fmt, g, b, rule):
    rng = np.random.default_rng(3)
    X = W.f32_to_bf16_bits(rng.standard_normal((24, 256)).astype(np.float32))
    Wt = W.synthetic_weights(40, 256, seed=4)
    rx = o.rotate_quantize(X, fmt, g, b, rule)
    rw = o.rotate_quantize(Wt, fmt, g, b, rule)
    D = o.gemm_fp4(rx["codes"], rx["scales"], rw["codes"], rw["scales"], fmt, rx["tensor_scale"], rw["tensor_scale"])
    assert D.shape == (24, 40)
    xh = o.dequantize(rx["codes"], rx["scales"], fmt, g, b, rx["tensor_scale"]).astype(np.float64)
    wh = o.dequantize(rw["codes"], rw["scales"], fmt, g, b, rw["tensor_scale"]).astype(np.float64)
    ref = xh @ wh.T
    if fmt == o.MXFP4:
        assert np.array_equal(D, ref)     # every dequantized value is exact in fp32
    else:
        assert np.allclose(D, ref, rtol=1e-6, atol=1e-6 * np.abs(ref).max())


def test_rotated_product_approximates_the_layer():
    """With the same signed rotation on both operands, the product of the dequantized rotated
    operands equals that of the operands rotated back, and approximates X W^T."""
    rng = np.random.default_rng(5)
    K = 512
    s = o.sign_vector(W.random_sign_mask(K, 2), K)
    X = W.f32_to_bf16_bits(rng.standard_normal((32, K)).astype(np.float32))
    Wt = W.synthetic_weights(48, K, seed=6)
    rx = o.rotate_quantize(X, o.MXFP4, 32, 128, o.SCALE_OAS, signs=s)
    rw = o.rotate_quantize(Wt, o.MXFP4, 32, 128, o.SCALE_OAS, signs=s)
    D = o.gemm_fp4(rx["codes"], rx["scales"], rw["codes"], rw["scales"], o.MXFP4)
    xb = o.dequantize(rx["codes"], rx["scales"], o.MXFP4, 32, 128, unrotate_back=True, signs=s)
    wb = o.dequantize(rw["codes"], rw["scales"], o.MXFP4, 32, 128, unrotate_back=True, signs=s)
    assert np.allclose(D, xb @ wb.T, rtol=1e-9, atol=1e-9 * np.abs(D).max())
    ref = o.bf16_to_f64(X) @ o.bf16_to_f64(Wt).T
    rel = np.linalg.norm(D - ref) / np.linalg.norm(ref)
    assert 0.01 < rel < 0.25, rel
