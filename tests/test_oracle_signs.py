"""Pins of the oracle's randomised (per-channel sign) Hadamard rotation, CPU only.

Source: "Bridging the Gap Between Promise and Performance for Microscaling FP4
Quantization", Technische Zusammenfassung, 2. Methodik (block-wise Hadamard transforms of
weights and activations, "wie in QuIP/QuaRot") and the English abstract (rotation fused
into the weights, fast online computation for the activations).  The rotation with signs
is Q = diag(s) (I kron H_b / sqrt(b)); the weights absorb the same Q, so the GEMM of the
rotated operands equals the original one.

The pins check the oracle against the definition by other routes: the bit layout on a
hand-written mask, rotated basis vectors (a sign applied after the block rotation, or on
the wrong channel, changes them), the GEMM identity with the same signs on both sides, and
the inverse."""

import math

import numpy as np

import oracle as o
from microscaling_fp4_quantization_b200 import workloads as W


def bf16(a):
    return W.f32_to_bf16_bits(np.asarray(a, np.float32))


def test_sign_mask_bit_layout():
    s = o.sign_vector(np.array([0x00000001, 0x80000000, 0x00000005], np.uint32), 70)
    neg = np.flatnonzero(s < 0).tolist()
    assert neg == [0, 63, 64, 66]
    assert np.all(np.abs(s) == 1.0)


def test_all_positive_signs_change_nothing():
    x = bf16(np.random.default_rng(1).standard_normal((5, 256)))
    for b in (1, 16, 128):
        assert np.array_equal(o.rotate(x, b, np.ones(256)), o.rotate(x, b))


def test_rotated_basis_vectors():
    """e_k rotates to s_k H_b[k mod b, :] / sqrt(b) inside block k // b, zero elsewhere."""
    K, b = 64, 16
    s = o.sign_vector(W.random_sign_mask(K, 9), K)
    H = o.sylvester_hadamard(b)
    for k in (0, 5, 17, 63):
        e = np.zeros((1, K))
        e[0, k] = 1.0
        y = o.rotate(bf16(e), b, s)[0]
        want = np.zeros(K)
        blk = k // b
        want[blk * b:(blk + 1) * b] = s[k] * H[k % b] / math.sqrt(b)
        assert np.array_equal(y, want), k


def test_gemm_identity_and_inverse_with_signs():
    rng = np.random.default_rng(2)
    K = 512
    s = o.sign_vector(W.random_sign_mask(K, 4), K)
    X = bf16(rng.standard_normal((6, K)))
    Wt = W.synthetic_weights(5, K, 3)
    for b in (2, 32, 128):
        XQ, WQ = o.rotate(X, b, s), o.rotate(Wt, b, s)
        ref = o.bf16_to_f64(X) @ o.bf16_to_f64(Wt).T
        assert np.allclose(XQ @ WQ.T, ref, rtol=0, atol=1e-12 * np.abs(ref).max())
        assert np.allclose(o.unrotate(XQ, b, s), o.bf16_to_f64(X), rtol=0, atol=1e-12)
        # a different sign vector on the weights breaks the identity
        s2 = o.sign_vector(W.random_sign_mask(K, 5), K)
        assert not np.allclose(XQ @ o.rotate(Wt, b, s2).T, ref, atol=1e-3 * np.abs(ref).max())


def test_signs_reach_the_codes_and_the_error():
    """The quantizer and the error pass see the signed rotation: codes differ from the
    unsigned ones, and the energies stay those of the unrotated domain."""
    rng = np.random.default_rng(6)
    K = 256
    s = o.sign_vector(W.random_sign_mask(K, 8), K)
    x = bf16(rng.laplace(size=(64, K)))
    a = o.rotate_quantize(x, o.MXFP4, 32, 32, o.SCALE_FLOOR_OCP)
    b = o.rotate_quantize(x, o.MXFP4, 32, 32, o.SCALE_FLOOR_OCP, signs=s)
    assert not np.array_equal(a["codes"], b["codes"])
    qe = o.quant_error(x, o.MXFP4, 32, 32, o.SCALE_FLOOR_OCP, signs=s)
    xhat = o.dequantize(b["codes"], b["scales"], o.MXFP4, 32, 32, unrotate_back=True, signs=s)
    xx = o.bf16_to_f64(x)
    assert math.isclose(qe["signal"], float(np.sum(xx * xx)), rel_tol=1e-12)
    assert math.isclose(qe["noise"], float(np.sum((xx - xhat) ** 2)), rel_tol=1e-6)
