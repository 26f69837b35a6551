"""GPU parity of the block-scaled FP4 GEMM (tcgen05 kind::mxf4 / kind::mxf4nvf4) with the
CPU oracle: D = alpha A_hat B_hat^T from the quantizer's own codes and scales.

Tolerance, from the arithmetic: every product q_a s_a q_b s_b is exact in fp32 (2 + 8 or
2 + 4 significand bits per factor), so the only roundings are the fp32 accumulation of K
products (in K/64 MMA steps of 64-term sums) and the final bf16 rounding.  For an fp32
accumulator that rounds (or truncates) each step, |error| <= (K/64 + 6) * 2^-23 * sum |a b|;
the bf16 result adds 2^-9 |D| (round to nearest even); the test allows twice both terms."""

import numpy as np
import pytest
import torch

import oracle as o
from microscaling_fp4_quantization_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F(cuda_device):
    from microscaling_fp4_quantization_b200 import fp4q
    return fp4q


FORMATS = [(o.MXFP4, 32, 32, o.SCALE_FLOOR_OCP), (o.NVFP4, 16, 16, o.SCALE_NV_DYNAMIC)]


def quantize_on_gpu(F, x_bits, fmt, g, b, rule):
    plan = F.fp4q_plan_create(fmt, g, b, rule)
    R, K = x_bits.shape
    xd = torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).cuda().view(torch.bfloat16)
    codes = torch.empty((R, K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((R, K // g), dtype=torch.uint8, device="cuda")
    ts = torch.empty(1, dtype=torch.float32, device="cuda")
    F.fp4q_rotate_quantize(plan, xd, R, K, codes, scales, ts if fmt == o.NVFP4 else None)
    return codes, scales, ts


def run_gemm(F, fmt, qa, qb, M, N, K):
    d = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    F.fp4q_gemm(fmt, qa[0], qa[1], qa[2] if fmt == o.NVFP4 else None, qb[0], qb[1], qb[2] if fmt == o.NVFP4 else None,
                M, N, K, d)
    torch.cuda.synchronize()
    assert F.fp4q_device_status() == F.FP4Q_OK
    return d.float().cpu().numpy().astype(np.float64)


def exact_operand(codes, scales, fmt):
    g = 32 if fmt == o.MXFP4 else 16
    q = o.e2m1_decode(o.unpack_nibbles(codes))
    R, K = q.shape
    S = np.ldexp(1.0, scales.astype(np.int64) - 127) if fmt == o.MXFP4 else o.e4m3_decode(scales)
    return (q.reshape(R, K // g, g) * S.reshape(R, K // g)[..., None]).reshape(R, K)


def check(D, qa, qb, fmt, K, rows=None, label=""):
    ac, as_ = qa[0].cpu().numpy(), qa[1].cpu().numpy()
    bc, bs = qb[0].cpu().numpy(), qb[1].cpu().numpy()
    if rows is not None:
        ac, as_, D = ac[rows], as_[rows], D[rows]
    ta = float(qa[2].item()) if fmt == o.NVFP4 else None
    tb = float(qb[2].item()) if fmt == o.NVFP4 else None
    ref = o.gemm_fp4(ac, as_, bc, bs, fmt, ta, tb)
    mag = np.abs(exact_operand(ac, as_, fmt)) @ np.abs(exact_operand(bc, bs, fmt)).T
    if fmt == o.NVFP4:
        mag = mag * (float(np.float32(ta)) * float(np.float32(tb)))
    bound = 2 * (2.0 ** -9 * np.abs(ref) + (K / 64 + 6) * 2.0 ** -23 * mag)
    err = np.abs(D - ref)
    worst = float(np.max(err / np.maximum(bound, 1e-300)))
    assert np.all(err <= bound), (label, worst, float(err.max()))
    return worst


@pytest.mark.parametrize("fmt,g,b,rule", FORMATS, ids=["mxfp4", "nvfp4"])
@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (1, 256, 512), (200, 512, 1024), (1000, 768, 2048),
                                   (300, 32, 256), (257, 512, 512), (384, 288, 768), (129, 1024, 256)])
def test_gemm_matches_oracle(F, fmt, g, b, rule, M, N, K):
    """Ragged shapes: a last M tile of one row (257, 129) or of a few rows (200, 300, 1000), and
    a last N tile of 32 columns (N = 288)."""
    rng = np.random.default_rng(M + N + K)
    X = W.f32_to_bf16_bits((rng.standard_normal((M, K)) * np.exp(rng.normal(0, 1, (M, 1)))).astype(np.float32))
    Wt = W.synthetic_weights(N, K, seed=N + K)
    qa = quantize_on_gpu(F, X, fmt, g, b, rule)
    qb = quantize_on_gpu(F, Wt, fmt, g, b, rule)
    D = run_gemm(F, fmt, qa, qb, M, N, K)
    check(D, qa, qb, fmt, K, label=f"{M}x{N}x{K}")
    # deterministic
    assert np.array_equal(D, run_gemm(F, fmt, qa, qb, M, N, K))


@pytest.mark.parametrize("fmt,g,b,rule", FORMATS, ids=["mxfp4", "nvfp4"])
def test_gemm_at_layer_size_on_sampled_rows(F, fmt, g, b, rule):
    """4096 x 4096 x 4096 (many tiles per CTA, 16 K-stages): the oracle on 48 sampled rows."""
    M = N = K = 4096
    X = W.NV_4K.generate()
    Wt = W.synthetic_weights(N, K, seed=9)
    qa = quantize_on_gpu(F, X, fmt, g, b, rule)
    qb = quantize_on_gpu(F, Wt, fmt, g, b, rule)
    D = run_gemm(F, fmt, qa, qb, M, N, K)
    rows = np.sort(np.random.default_rng(1).choice(M, 48, replace=False))
    check(D, qa, qb, fmt, K, rows=rows, label="4096^3")


def test_gemm_of_rotated_operands_approximates_the_layer(F):
    """The same signed rotation on activations and weights: the FP4 GEMM approximates X W^T."""
    M, N, K = 256, 512, 2048
    rng = np.random.default_rng(4)
    X = W.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    Wt = W.synthetic_weights(N, K, seed=5)
    mask = torch.from_numpy(W.random_sign_mask(K, 3).view(np.int32)).cuda()
    outs = []
    for A in (X, Wt):
        plan = F.fp4q_plan_create(o.MXFP4, 32, 128, o.SCALE_OAS)
        F.fp4q_plan_set_signs(plan, mask, K)
        R = A.shape[0]
        xd = torch.from_numpy(np.ascontiguousarray(A).view(np.int16)).cuda().view(torch.bfloat16)
        c = torch.empty((R, K // 2), dtype=torch.uint8, device="cuda")
        s = torch.empty((R, K // 32), dtype=torch.uint8, device="cuda")
        F.fp4q_rotate_quantize(plan, xd, R, K, c, s, None)
        outs.append((c, s, None))
    D = run_gemm(F, o.MXFP4, outs[0], outs[1], M, N, K)
    ref = o.bf16_to_f64(X) @ o.bf16_to_f64(Wt).T
    rel = np.linalg.norm(D - ref) / np.linalg.norm(ref)
    assert rel < 0.2, rel
