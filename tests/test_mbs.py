"""GPU parity of MBS-Static (MXFP4 under 128-element macro-block scales with 8 mantissa bits)
with the CPU oracle, through the C ABI.

Source: "Unveiling the Potential of Quantization with MXFP4: Strategies for Quantization
Error Reduction", Technische samenvatting, Methodologie 2 (Macro Block Scaling, MBS-Static).
Codes, group scales and macro bytes must match bit for bit outside the flagged set (which,
for MBS, also flags every group of a macro block whose exact 256 f lies within 1e-5 of an
integer); the dequantized values are exact in fp32."""

import numpy as np
import pytest
import torch

import oracle as o
from microscaling_fp4_quantization_b200 import workloads as W
from oracle.parity import assert_parity
from test_parity_small import make_input

pytestmark = pytest.mark.gpu

BLOCKS = [1, 2, 4, 8, 16, 32, 64, 128]
RULES = [o.SCALE_FLOOR_OCP, o.SCALE_CEIL_NOCLIP, o.SCALE_OAS]


@pytest.fixture(scope="module")
def F(cuda_device):
    from microscaling_fp4_quantization_b200 import fp4q
    return fp4q


def check_macro(res, out, label):
    """Macro bytes match except on macro blocks whose exact 256 f is within 1e-5 (times 256)
    of an integer (compare() also judges them, given the bytes; this names them alone)."""
    flagged_macro = o.mbs_macro_distance(res) <= 1e-5
    bad = (res["macro"] != out["macro"]) & ~flagged_macro
    assert not bad.any(), (label, int(bad.sum()))


# (block, kernel): the butterfly for every block, the tensor-core kernel where blocks hold whole groups
CASES = [(b, 1) for b in BLOCKS] + [(b, 2) for b in BLOCKS if b >= 32]


@pytest.mark.parametrize("b,kernel", CASES, ids=[f"b{b}-{'tc' if k == 2 else 'bf'}" for b, k in CASES])
@pytest.mark.parametrize("rule", RULES, ids=[W.RULE_NAMES[r] for r in RULES])
def test_mbs_matches_oracle(F, b, kernel, rule):
    import gpu_util as gu
    plan = F.fp4q_plan_create(o.MXFP4_MBS, 32, b, rule)
    F.fp4q_plan_set_kernel(plan, kernel)
    for i, (M, K) in enumerate([(1, 128), (3, 256), (37, 768), (130, 4096), (300, 1536)]):
        x = make_input(M, K, seed=3000 + 10 * b + rule + 100 * i, adversarial=M >= 8)
        res = o.rotate_quantize_mbs(x, 32, b, rule)
        out = gu.run_rotate_quantize_mbs(F, plan, x)
        label = f"mbs b{b} {W.RULE_NAMES[rule]} {M}x{K}"
        assert_parity(res, out["codes"], out["scales"], label, count_bound=M < 8, macro_gpu=out["macro"])
        check_macro(res, out, label)
        if M >= 8:
            real = slice(8, M)
            res_r = {k: (v[real] if isinstance(v, np.ndarray) and v.ndim == 2 and v.shape[0] == M else v)
                     for k, v in res.items()}
            assert_parity(res_r, out["codes"][real], out["scales"][real], label + " rows 8+",
                          macro_gpu=out["macro"][real])


@pytest.mark.parametrize("b,kernel", [(1, 1), (32, 1), (128, 1), (32, 2), (64, 2), (128, 2)],
                         ids=["b1-bf", "b32-bf", "b128-bf", "b32-tc", "b64-tc", "b128-tc"])
def test_mbs_dequantize_and_error(F, b, kernel):
    import gpu_util as gu
    from test_quant_error import assert_energies, run_qe
    M, K = 256, 2048
    x = make_input(M, K, seed=77 + b, adversarial=False)
    plan = F.fp4q_plan_create(o.MXFP4_MBS, 32, b, o.SCALE_OAS)
    F.fp4q_plan_set_kernel(plan, kernel)
    out = gu.run_rotate_quantize_mbs(F, plan, x)
    flat = gu.run_dequantize_mbs(F, plan, out["codes"], out["scales"], out["macro"], unrotate=False)
    ref = o.dequantize_mbs(out["codes"], out["scales"], out["macro"], 32, b)
    assert np.array_equal(flat, ref)
    back = gu.run_dequantize_mbs(F, plan, out["codes"], out["scales"], out["macro"], unrotate=True)
    ref_b = o.dequantize_mbs(out["codes"], out["scales"], out["macro"], 32, b, unrotate_back=True)
    assert np.max(np.abs(back - ref_b)) <= 1e-6 * np.abs(ref_b).max()
    assert_energies(run_qe(F, plan, x), o.quant_error(x, o.MXFP4_MBS, 32, b, o.SCALE_OAS), f"mbs b{b}")


@pytest.mark.parametrize("b,kernel", [(32, 1), (32, 2), (128, 2)], ids=["b32-bf", "b32-tc", "b128-tc"])
def test_mbs_with_signs(F, b, kernel):
    import gpu_util as gu
    M, K = 100, 1024
    x = make_input(M, K, seed=5, adversarial=False)
    plan = F.fp4q_plan_create(o.MXFP4_MBS, 32, b, o.SCALE_FLOOR_OCP)
    F.fp4q_plan_set_kernel(plan, kernel)
    mask = W.random_sign_mask(K, 31)
    md = torch.from_numpy(mask.view(np.int32)).cuda()
    F.fp4q_plan_set_signs(plan, md, K)
    out = gu.run_rotate_quantize_mbs(F, plan, x)
    res = o.rotate_quantize_mbs(x, 32, b, o.SCALE_FLOOR_OCP, signs=o.sign_vector(mask, K))
    assert_parity(res, out["codes"], out["scales"], "mbs signed", macro_gpu=out["macro"])
    check_macro(res, out, "mbs signed")


def test_mbs_beats_mxfp4_on_the_gpu(F):
    """The page's claim, on Laplace rows: MBS-Static improves QSNR over plain MXFP4."""
    from test_quant_error import run_qe
    x = W.f32_to_bf16_bits(np.random.default_rng(21).laplace(size=(1024, 4096)).astype(np.float32))
    for b in (1, 32):
        for rule in RULES:
            plain = run_qe(F, F.fp4q_plan_create(o.MXFP4, 32, b, rule), x)[2]
            mbs = run_qe(F, F.fp4q_plan_create(o.MXFP4_MBS, 32, b, rule), x)[2]
            assert mbs > plain + 0.2, (b, rule, mbs, plain)


def test_mbs_plan_routes(F):
    """fp4q_rotate_quantize refuses an MBS plan; the MBS entry refuses other plans."""
    import gpu_util as gu
    plan = F.fp4q_plan_create(o.MXFP4_MBS, 32, 32, o.SCALE_FLOOR_OCP)
    x = gu.to_device_bf16(make_input(4, 256, seed=1, adversarial=False))
    c = torch.empty(512, dtype=torch.uint8, device="cuda")
    with pytest.raises(F.Fp4qError) as e:
        F.fp4q_rotate_quantize(plan, x, 4, 256, c, c, None)
    assert e.value.status == F.FP4Q_ERR_UNSUPPORTED
    mx = F.fp4q_plan_create(o.MXFP4, 32, 32, o.SCALE_FLOOR_OCP)
    with pytest.raises(F.Fp4qError) as e:
        F.fp4q_rotate_quantize_mbs(mx, x, 4, 256, c, c, c)
    assert e.value.status == F.FP4Q_ERR_UNSUPPORTED
