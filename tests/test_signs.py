"""GPU parity of the randomised rotation (per-channel random signs, plan-level) with the
CPU oracle, and the weight-side path it serves: the same signs on activations and weights,
round-to-nearest FP4 weights, and the GEMM identity of the rotated operands.

Source: "Bridging the Gap Between Promise and Performance for Microscaling FP4
Quantization", Technische Zusammenfassung, 2. Methodik (block-wise Hadamard transforms
of weights and activations, "wie in QuIP/QuaRot") and the English abstract (rotation
fused into the weights, fast online computation of the activations)."""

import numpy as np
import pytest
import torch

import oracle as o
from microscaling_fp4_quantization_b200 import workloads as W
from oracle.parity import assert_parity, rotated_value_error
from test_parity_small import COMBOS, combo_id, make_input

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F(cuda_device):
    from microscaling_fp4_quantization_b200 import fp4q
    return fp4q


def signed_plan(F, combo, K, seed):
    fmt, g, b, rule = combo
    plan = F.fp4q_plan_create(fmt, g, b, rule)
    mask = W.random_sign_mask(K, seed)
    md = torch.from_numpy(mask.view(np.int32)).cuda()
    F.fp4q_plan_set_signs(plan, md, K)
    return plan, o.sign_vector(mask, K)


SIGN_CASES = ([(c, 1) for c in COMBOS] + [(c, 2) for c in COMBOS if c[2] >= 16 and c[2] >= c[1]])


@pytest.mark.parametrize("combo,kernel", SIGN_CASES,
                         ids=[combo_id(c) + ("-tc" if k == 2 else "-bf") for c, k in SIGN_CASES])
def test_signed_rotate_quantize_matches_oracle(F, combo, kernel):
    """kernel 1: the butterfly kernel (signs applied as it loads); 2: the tensor-core kernel
    (signs flipped in the landed shared-memory stage before the product)."""
    import gpu_util as gu
    fmt, g, b, rule = combo
    unit = max(g, b)
    for i, (M, K) in enumerate([(3, 2 * unit), (37, 6 * unit), (130, 4096 // unit * unit), (200, 1536),
                                (1100, 4096)]):
        plan, s = signed_plan(F, combo, K, seed=500 + i)
        F.fp4q_plan_set_kernel(plan, kernel)
        x = make_input(M, K, seed=9000 + 100 * b + 10 * rule + i, adversarial=M >= 8)
        s_g = o.nv_tensor_scale(o.rotated_amax(x, b, signs=s)) if rule == o.SCALE_NV_STATIC else None
        res = o.rotate_quantize(x, fmt, g, b, rule, tensor_scale=s_g, signs=s)
        out = gu.run_rotate_quantize(F, plan, x, tensor_scale=s_g, dump=True)
        adversarial = M >= 8
        assert_parity(res, out["codes"], out["scales"], f"{combo_id(combo)} {M}x{K} signed",
                      count_bound=not adversarial)
        assert rotated_value_error(out["y"], res) <= 1e-5, (M, K)
        if rule == o.SCALE_NV_DYNAMIC:
            assert abs(float(out["tensor_scale"]) - float(res["tensor_scale"])) <= 2.5e-7 * float(res["tensor_scale"])


@pytest.mark.parametrize("b,kernel", [(1, 1), (16, 1), (128, 1), (16, 2), (32, 2), (128, 2)],
                         ids=["b1-bf", "b16-bf", "b128-bf", "b16-tc", "b32-tc", "b128-tc"])
def test_signed_amax_and_quant_error(F, b, kernel):
    """The signed amax (butterfly-only pass) and the signed error pass on either kernel."""
    import gpu_util as gu
    from test_quant_error import assert_energies, run_qe
    M, K = 300, 1024
    x = make_input(M, K, seed=40 + b, adversarial=False)
    plan, s = signed_plan(F, (o.NVFP4, 16, b, o.SCALE_NV_STATIC), K, seed=7)
    F.fp4q_plan_set_kernel(plan, kernel)
    ours = gu.run_amax(F, plan, x)
    ref = o.nv_tensor_scale(o.rotated_amax(x, b, signs=s))
    assert abs(float(ours) - float(ref)) <= 2.5e-7 * float(ref)
    assert ref != o.nv_tensor_scale(o.rotated_amax(x, b)) or b == 1
    qe_ref = o.quant_error(x, o.NVFP4, 16, b, o.SCALE_NV_STATIC, tensor_scale=ref, signs=s)
    assert_energies(run_qe(F, plan, x, tensor_scale=ref), qe_ref, f"b{b} signed")
    if b >= 32 or kernel == 1:
        mplan, ms = signed_plan(F, (o.MXFP4, 32, b, o.SCALE_OAS), K, seed=8)
        F.fp4q_plan_set_kernel(mplan, kernel)
        assert_energies(run_qe(F, mplan, x), o.quant_error(x, o.MXFP4, 32, b, o.SCALE_OAS, signs=ms),
                        f"mx b{b} signed")


@pytest.mark.parametrize("b", [2, 32, 128])
def test_signed_dequantize_rotates_back(F, b):
    import gpu_util as gu
    M, K = 64, 512
    x = make_input(M, K, seed=3 + b, adversarial=False)
    plan, s = signed_plan(F, (o.MXFP4, 32, b, o.SCALE_FLOOR_OCP), K, seed=11)
    out = gu.run_rotate_quantize(F, plan, x)
    back = gu.run_dequantize(F, plan, out["codes"], out["scales"], None, unrotate=True)
    ref = o.dequantize(out["codes"], out["scales"], o.MXFP4, 32, b, unrotate_back=True, signs=s)
    scale = np.abs(ref).max()
    assert np.max(np.abs(back - ref)) <= 1e-6 * scale


def test_weight_path_gemm_identity(F):
    """Weights rotated and quantized with the same signs as the activations: the GEMM of the
    rotated dequantized operands equals the GEMM of the operands rotated back (Q is
    orthogonal), and it approximates X W^T with the quantization error that the error pass
    reports for each side."""
    import gpu_util as gu
    K, M, N = 2048, 256, 192
    b = 128
    X = W.NV_4K.with_rows(M).generate()[:, :K].copy()
    Wt = W.synthetic_weights(N, K, seed=2)
    mask = W.random_sign_mask(K, 21)
    md = torch.from_numpy(mask.view(np.int32)).cuda()
    plan = F.fp4q_plan_create(o.MXFP4, 32, b, o.SCALE_OAS)
    F.fp4q_plan_set_signs(plan, md, K)
    xq = gu.run_rotate_quantize(F, plan, X)
    wq = gu.run_rotate_quantize(F, plan, Wt)
    Xr = gu.run_dequantize(F, plan, xq["codes"], xq["scales"], None, unrotate=False).astype(np.float64)
    Wr = gu.run_dequantize(F, plan, wq["codes"], wq["scales"], None, unrotate=False).astype(np.float64)
    Xb = gu.run_dequantize(F, plan, xq["codes"], xq["scales"], None, unrotate=True).astype(np.float64)
    Wb = gu.run_dequantize(F, plan, wq["codes"], wq["scales"], None, unrotate=True).astype(np.float64)
    G_rot = Xr @ Wr.T
    G_back = Xb @ Wb.T
    assert np.max(np.abs(G_rot - G_back)) <= 1e-5 * np.abs(G_rot).max()
    ref = o.bf16_to_f64(X) @ o.bf16_to_f64(Wt).T
    rel = np.linalg.norm(G_rot - ref) / np.linalg.norm(ref)
    assert rel < 0.2, rel
    # the codes are those of the oracle with the same signs
    s = o.sign_vector(mask, K)
    for A, q in ((X, xq), (Wt, wq)):
        res = o.rotate_quantize(A, o.MXFP4, 32, b, o.SCALE_OAS, signs=s)
        assert_parity(res, q["codes"], q["scales"], "weight path")


@pytest.mark.parametrize("combo,kernel", [((o.MXFP4, 32, 32, o.SCALE_OAS), 1), ((o.MXFP4, 32, 32, o.SCALE_OAS), 2),
                                          ((o.NVFP4, 16, 16, o.SCALE_NV_STATIC), 1),
                                          ((o.NVFP4, 16, 128, o.SCALE_NV_STATIC), 2)],
                         ids=["mx-b32-bf", "mx-b32-tc", "nv-b16-bf", "nv-b128-tc"])
def test_signed_rows_longer_than_the_staged_mask(F, combo, kernel):
    """K = 135168: the mask (4224 words, 16.5 KB) is larger than either kernel stages in shared
    memory, so both read it where the caller keeps it."""
    import gpu_util as gu
    fmt, g, b, rule = combo
    M, K = 3, 135168
    plan, s = signed_plan(F, combo, K, seed=77)
    F.fp4q_plan_set_kernel(plan, kernel)
    x = make_input(M, K, seed=4242 + b, adversarial=False)
    s_g = o.nv_tensor_scale(o.rotated_amax(x, b, signs=s)) if rule == o.SCALE_NV_STATIC else None
    res = o.rotate_quantize(x, fmt, g, b, rule, tensor_scale=s_g, signs=s)
    out = gu.run_rotate_quantize(F, plan, x, tensor_scale=s_g)
    assert_parity(res, out["codes"], out["scales"], f"{combo_id(combo)} K={K} signed")


SIGN_SOURCE_CASES = [((o.NVFP4, 16, 16, o.SCALE_NV_STATIC), 4096), ((o.NVFP4, 16, 16, o.SCALE_NV_STATIC), 32768),
                     ((o.NVFP4, 16, 64, o.SCALE_NV_DYNAMIC), 32768), ((o.MXFP4, 32, 32, o.SCALE_CEIL_NOCLIP), 4096),
                     ((o.MXFP4, 32, 32, o.SCALE_CEIL_NOCLIP), 32768), ((o.MXFP4, 32, 128, o.SCALE_FLOOR_OCP), 8192),
                     ((o.MXFP4, 32, 128, o.SCALE_FLOOR_OCP), 32768), ((o.NVFP4, 16, 128, o.SCALE_NV_STATIC), 14336),
                     ((o.NVFP4, 16, 128, o.SCALE_NV_STATIC), 32768)]


@pytest.mark.parametrize("combo,K", SIGN_SOURCE_CASES,
                         ids=[f"{combo_id(c)}-K{K}" for c, K in SIGN_SOURCE_CASES])
def test_tensor_core_sign_sources(F, combo, K):
    """The tensor-core kernel reads the signs from one of three shared-memory sources, chosen
    by K: the expanded table (one CTA per SM, 4 K bytes up to 64 KB: NVFP4 b <= 64, K <= 16384),
    the word table (two CTAs per SM, while it fits beside them: K = 4096 at b = 32, K = 8192 and
    14336 at b = 128) and the mask's bytes (K = 32768 in every configuration).  Each against the
    oracle, on every row kind."""
    import gpu_util as gu
    fmt, g, b, rule = combo
    M = 40
    plan, s = signed_plan(F, combo, K, seed=90 + b)
    F.fp4q_plan_set_kernel(plan, F.FP4Q_KERNEL_TENSOR_CORE)
    x = make_input(M, K, seed=4545 + b + K, adversarial=True)
    s_g = o.nv_tensor_scale(o.rotated_amax(x, b, signs=s)) if rule == o.SCALE_NV_STATIC else None
    res = o.rotate_quantize(x, fmt, g, b, rule, tensor_scale=s_g, signs=s)
    out = gu.run_rotate_quantize(F, plan, x, tensor_scale=s_g, dump=True)
    assert_parity(res, out["codes"], out["scales"], f"{combo_id(combo)} {M}x{K} signed, tensor core",
                  count_bound=False)
    assert rotated_value_error(out["y"], res) <= 1e-5, (M, K)


def every_byte_mask(K):
    """Mask words whose 8-channel chunks take every byte value 0 .. 255 in turn (K a multiple
    of 32): every pattern each kernel's sign expansion can meet."""
    n = K // 8
    return np.tile(np.arange(256, dtype=np.uint8), n // 256 + 1)[:n].view(np.uint32).copy()


EVERY_BYTE_CASES = [((o.NVFP4, 16, 16, o.SCALE_NV_STATIC), 4096, 2), ((o.NVFP4, 16, 16, o.SCALE_NV_STATIC), 32768, 2),
                    ((o.MXFP4, 32, 32, o.SCALE_FLOOR_OCP), 4096, 2), ((o.MXFP4, 32, 128, o.SCALE_FLOOR_OCP), 8192, 2),
                    ((o.MXFP4, 32, 128, o.SCALE_FLOOR_OCP), 32768, 2), ((o.NVFP4, 16, 16, o.SCALE_NV_STATIC), 4096, 1),
                    ((o.MXFP4, 32, 128, o.SCALE_FLOOR_OCP), 8192, 1)]


@pytest.mark.parametrize("combo,K,kernel", EVERY_BYTE_CASES,
                         ids=[f"{combo_id(c)}-K{K}-{'tc' if k == 2 else 'bf'}" for c, K, k in EVERY_BYTE_CASES])
def test_every_mask_byte(F, combo, K, kernel):
    """All 256 values of a chunk's eight sign bits, through each sign source of the tensor-core
    kernel (expanded table, word table, mask bytes) and through the butterfly kernel."""
    import gpu_util as gu
    fmt, g, b, rule = combo
    M = 16
    mask = every_byte_mask(K)
    plan = F.fp4q_plan_create(fmt, g, b, rule)
    F.fp4q_plan_set_signs(plan, torch.from_numpy(mask.view(np.int32)).cuda(), K)
    F.fp4q_plan_set_kernel(plan, kernel)
    s = o.sign_vector(mask, K)
    x = make_input(M, K, seed=4646 + b + K, adversarial=False)
    s_g = o.nv_tensor_scale(o.rotated_amax(x, b, signs=s)) if rule == o.SCALE_NV_STATIC else None
    res = o.rotate_quantize(x, fmt, g, b, rule, tensor_scale=s_g, signs=s)
    out = gu.run_rotate_quantize(F, plan, x, tensor_scale=s_g, dump=True)
    assert_parity(res, out["codes"], out["scales"], f"{combo_id(combo)} {M}x{K} every mask byte, kernel {kernel}")
    assert rotated_value_error(out["y"], res) <= 1e-5, (M, K)


@pytest.mark.parametrize("b,kernel", [(16, 1), (128, 1), (16, 2), (128, 2)],
                         ids=["b16-bf", "b128-bf", "b16-tc", "b128-tc"])
def test_unstaged_mask_on_every_signed_path(F, b, kernel):
    """K = 135168 (a 16.5 KB mask, read in place by every kernel): the NV amax pass (fp4q_amax
    and a DYNAMIC plan), the error pass and dequantize with rotate-back all switch between a
    staged and an in-place mask by the same rule as rotate + quantize."""
    import gpu_util as gu
    from test_quant_error import assert_energies, run_qe
    M, K = 3, 135168
    x = make_input(M, K, seed=4343 + b, adversarial=False)
    plan, s = signed_plan(F, (o.NVFP4, 16, b, o.SCALE_NV_DYNAMIC), K, seed=78)
    F.fp4q_plan_set_kernel(plan, kernel)
    ref_sg = o.nv_tensor_scale(o.rotated_amax(x, b, signs=s))
    res = o.rotate_quantize(x, o.NVFP4, 16, b, o.SCALE_NV_DYNAMIC, signs=s)
    out = gu.run_rotate_quantize(F, plan, x)
    assert abs(float(out["tensor_scale"]) - float(ref_sg)) <= 2.5e-7 * float(ref_sg)
    assert_parity(res, out["codes"], out["scales"], f"nv-b{b} K={K} signed dynamic kernel {kernel}")
    assert abs(float(gu.run_amax(F, plan, x)) - float(ref_sg)) <= 2.5e-7 * float(ref_sg)
    assert_energies(run_qe(F, plan, x), o.quant_error(x, o.NVFP4, 16, b, o.SCALE_NV_DYNAMIC, signs=s),
                    f"nv-b{b} K={K} signed error pass")
    back = gu.run_dequantize(F, plan, out["codes"], out["scales"], out["tensor_scale"], unrotate=True)
    ref_back = o.dequantize(out["codes"], out["scales"], o.NVFP4, 16, b, tensor_scale=out["tensor_scale"],
                            unrotate_back=True, signs=s)
    assert np.max(np.abs(back - ref_back)) <= 1e-6 * np.abs(ref_back).max()
    mx, smx = signed_plan(F, (o.MXFP4, 32, b, o.SCALE_OAS), K, seed=79)
    if b >= 32 or kernel == 1:
        F.fp4q_plan_set_kernel(mx, kernel)
        assert_energies(run_qe(F, mx, x), o.quant_error(x, o.MXFP4, 32, b, o.SCALE_OAS, signs=smx),
                        f"mx-b{b} K={K} signed error pass")
