"""GPU parity of fp4q_quant_error (signal and error energies of rotate + quantize, and the
QSNR) with the CPU oracle, through the C ABI.

Tolerances, from the arithmetic of the kernel:
  * signal: each y^2 is (v X)^2 with v = fl(y / X) (2^-24 relative) and y itself fp32
    (2^-24 from the exact value); per-group sums of at most 16 terms per fp32 lane
    (16 * 2^-24 at worst), fp64 beyond that: under 2e-6 relative.
  * error: e = (v - q) X against the exact y - q X differs by at most about 2^-23 |y|;
    relative to the error energy that is 2^-23 * sum|e||y| / sum e^2, with |y| / |e| of
    order 10 at these QSNRs (about 1e-6), plus the fp32 group sums: 1e-5 relative.  Codes
    that differ from the oracle's only do so at flagged near-ties (within 1e-5 of a
    midpoint, where both roundings give nearly the same |e|), so they do not count.
  * QSNR: 10 / ln 10 times the sum of both relative errors: 1e-4 dB.
"""

import math

import numpy as np
import pytest
import torch

import oracle as o
from microscaling_fp4_quantization_b200 import workloads as W
from test_parity_small import COMBOS, combo_id, make_input

pytestmark = pytest.mark.gpu

SIG_RTOL = 2e-6
ERR_RTOL = 1e-5
QSNR_ATOL_DB = 1e-4


@pytest.fixture(scope="module")
def F(cuda_device):
    from microscaling_fp4_quantization_b200 import fp4q
    return fp4q


def run_qe(F, plan, x_bits=None, tensor_scale=None, x_dev=None):
    import gpu_util as gu
    xd = x_dev if x_dev is not None else gu.to_device_bf16(x_bits)
    M, K = xd.shape
    out = gu.Guarded(24)
    ts = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    if tensor_scale is not None:
        ts.fill_(float(tensor_scale))
    F.fp4q_quant_error(plan, xd, M, K, ts if plan.fmt == F.FP4Q_NVFP4 else None, out.view)
    torch.cuda.synchronize()
    assert F.fp4q_device_status() == F.FP4Q_OK
    out.check("quant_error out")
    s, e, q = (float(v) for v in out.numpy().view(np.float64))
    return s, e, q, np.float32(ts.item())


BUTTERFLY, TENSOR_CORE = 1, 2


def tc_capable(fmt, g, b):
    """The tensor-core kernel serves MXFP4 / NVFP4 plans whose blocks hold whole groups."""
    return fmt in (o.MXFP4, o.NVFP4) and b >= 16 and b >= g


def kernel_cases(combos):
    return [(c, BUTTERFLY) for c in combos] + [(c, TENSOR_CORE) for c in combos if tc_capable(c[0], c[1], c[2])]


def kernel_id(case):
    c, k = case
    return combo_id(c) + ("-tc" if k == TENSOR_CORE else "-bf")


def static_scale(x, fmt, b, rule):
    if fmt == o.NVFP4 and rule == o.SCALE_NV_STATIC:
        return o.nv_tensor_scale(o.rotated_amax(x, b))
    return None


def assert_energies(ours, ref, label):
    s, e, q = ours[:3]
    assert s == pytest.approx(ref["signal"], rel=SIG_RTOL, abs=1e-300), label
    assert e == pytest.approx(ref["noise"], rel=ERR_RTOL, abs=1e-300), label
    if math.isinf(ref["qsnr_db"]):
        assert q == ref["qsnr_db"], label
    else:
        assert abs(q - ref["qsnr_db"]) <= QSNR_ATOL_DB, (label, q, ref["qsnr_db"])


QE_CASES = kernel_cases(COMBOS)


@pytest.mark.parametrize("case", QE_CASES, ids=[kernel_id(c) for c in QE_CASES])
def test_quant_error_matches_oracle(F, case):
    combo, kernel = case
    fmt, g, b, rule = combo
    plan = F.fp4q_plan_create(fmt, g, b, rule)
    F.fp4q_plan_set_kernel(plan, kernel)
    unit = max(g, b)
    for i, (M, K) in enumerate([(1, unit), (37, 6 * unit), (130, 4096 // unit * unit), (1000, 1536)]):
        x = make_input(M, K, seed=7000 + 100 * b + 10 * rule + i, adversarial=M >= 8)
        s_g = static_scale(x, fmt, b, rule)
        ref = o.quant_error(x, fmt, g, b, rule, tensor_scale=s_g)
        ours = run_qe(F, plan, x, tensor_scale=s_g)
        assert_energies(ours, ref, f"{combo_id(combo)} {M}x{K}")
        if fmt == o.NVFP4 and rule == o.SCALE_NV_DYNAMIC:
            assert abs(float(ours[3]) - float(ref["tensor_scale"])) <= 2.5e-7 * float(ref["tensor_scale"])


STORE_CASES = kernel_cases([(o.MXFP4, 32, 32, o.SCALE_FLOOR_OCP), (o.MXFP4, 32, 128, o.SCALE_OAS),
                            (o.NVFP4, 16, 16, o.SCALE_NV_STATIC), (o.NVFP4, 16, 2, o.SCALE_NV_DYNAMIC),
                            (o.NVFP4, 16, 64, o.SCALE_NV_DYNAMIC)])


@pytest.mark.parametrize("case", STORE_CASES, ids=[kernel_id(c) for c in STORE_CASES])
def test_quant_error_measures_the_codes_rotate_quantize_stores(F, case):
    """The error pass decides exactly as the quantize kernel of the same plan: its error
    energy is the one of that kernel's stored codes, dequantized on the GPU, against its
    dumped fp32 y (butterfly and tensor-core kernels alike)."""
    import gpu_util as gu
    combo, kernel = case
    fmt, g, b, rule = combo
    plan = F.fp4q_plan_create(fmt, g, b, rule)
    F.fp4q_plan_set_kernel(plan, kernel)
    x = make_input(512, 2048, seed=11 + b, adversarial=False)
    s_g = static_scale(x, fmt, b, rule)
    rq = gu.run_rotate_quantize(F, plan, x, tensor_scale=s_g, dump=True)
    yhat = gu.run_dequantize(F, plan, rq["codes"], rq["scales"], rq["tensor_scale"], unrotate=False)
    y = rq["y"].astype(np.float64)
    noise = float(np.sum((y - yhat.astype(np.float64)) ** 2))
    signal = float(np.sum(y * y))
    s, e, _, _ = run_qe(F, plan, x, tensor_scale=s_g)
    assert s == pytest.approx(signal, rel=SIG_RTOL)
    assert e == pytest.approx(noise, rel=ERR_RTOL)


@pytest.mark.parametrize("kernel", [BUTTERFLY, TENSOR_CORE], ids=["bf", "tc"])
def test_quant_error_is_deterministic_and_additive_over_rows(F, kernel):
    """Two calls give the same bits; the energies of row blocks add up to the whole
    tensor's (a grid of many waves against one of a few CTAs)."""
    w = W.NV_4K
    x = w.generate()
    plan = F.fp4q_plan_create(w.fmt, w.group, w.block, o.SCALE_NV_STATIC)
    F.fp4q_plan_set_kernel(plan, kernel)
    import gpu_util as gu
    xd = gu.to_device_bf16(x)
    ts = o.nv_tensor_scale(o.rotated_amax(x, w.block))
    a = run_qe(F, plan, x_dev=xd, tensor_scale=ts)
    b = run_qe(F, plan, x_dev=xd, tensor_scale=ts)
    assert a[:3] == b[:3]
    parts = [run_qe(F, plan, x_dev=xd[r:r + 512], tensor_scale=ts) for r in range(0, w.M, 512)]
    assert sum(p[0] for p in parts) == pytest.approx(a[0], rel=1e-12)
    assert sum(p[1] for p in parts) == pytest.approx(a[1], rel=1e-12)
    # the oracle on two of the blocks
    for r in (0, 2048):
        ref = o.quant_error(x[r:r + 512], w.fmt, w.group, w.block, o.SCALE_NV_STATIC, tensor_scale=ts)
        assert_energies(parts[r // 512], ref, f"rows {r}..")


WORKLOAD_NAMES = [W.SMALL_MX.name, W.MX_8K_FLOOR.name, W.MX_8K_CEIL.name, W.PREFILL_NV.name,
                  W.PREFILL_MX.name] + [w.name for w in W.DECODE]
WORKLOAD_CASES = [(n, BUTTERFLY) for n in WORKLOAD_NAMES] + [
    (n, TENSOR_CORE) for n in WORKLOAD_NAMES
    if tc_capable(W.BY_NAME[n].fmt, W.BY_NAME[n].group, W.BY_NAME[n].block)]


@pytest.mark.parametrize("name,kernel", WORKLOAD_CASES,
                         ids=[n + ("-tc" if k == TENSOR_CORE else "-bf") for n, k in WORKLOAD_CASES])
def test_quant_error_on_workloads(F, name, kernel):
    """Full-size workloads: the GPU over the whole tensor equals the sum of the GPU over row
    blocks, and the oracle agrees with the GPU on sampled blocks."""
    import gpu_util as gu
    w = W.BY_NAME[name]
    x = w.generate()
    rule = w.rule
    plan = F.fp4q_plan_create(w.fmt, w.group, w.block, rule)
    F.fp4q_plan_set_kernel(plan, kernel)
    xd = gu.to_device_bf16(x)
    ts = None
    if w.fmt == o.NVFP4:
        ts = gu.run_amax(F, plan, None, x_dev=xd)
        rule_o = o.SCALE_NV_STATIC if rule == o.SCALE_NV_STATIC else rule
    whole = run_qe(F, plan, x_dev=xd, tensor_scale=ts)
    step = max(1, min(w.M, (1 << 22) // w.K))
    blocks = list(range(0, w.M, step))
    parts = [run_qe(F, plan, x_dev=xd[r:r + step], tensor_scale=ts) for r in blocks]
    assert sum(p[0] for p in parts) == pytest.approx(whole[0], rel=1e-12)
    assert sum(p[1] for p in parts) == pytest.approx(whole[1], rel=1e-12)
    sample = sorted({blocks[0], blocks[len(blocks) // 2], blocks[-1]})
    for r in sample:
        rows = x[r:r + min(step, 256)]
        ref = o.quant_error(rows, w.fmt, w.group, w.block, o.SCALE_NV_STATIC if w.fmt == o.NVFP4 else rule,
                            tensor_scale=ts)
        ours = run_qe(F, plan, x_dev=xd[r:r + rows.shape[0]], tensor_scale=ts)
        assert_energies(ours, ref, f"{name} rows {r}..")


def laplace(M=1024, K=4096, seed=21):
    return W.f32_to_bf16_bits(np.random.default_rng(seed).laplace(size=(M, K)).astype(np.float32))


def qsnr(F, x, fmt, g, b, rule):
    plan = F.fp4q_plan_create(fmt, g, b, rule)
    return run_qe(F, plan, x)[2]


def test_pages_trends_on_the_gpu(F):
    """On Laplace rows: a block rotation improves MXFP4 and worsens NVFP4 under
    round-to-nearest; OAS gains about 0.5 dB over the ceil rule."""
    x = laplace()
    mx1 = qsnr(F, x, o.MXFP4, 32, 1, o.SCALE_FLOOR_OCP)
    mx32 = qsnr(F, x, o.MXFP4, 32, 32, o.SCALE_FLOOR_OCP)
    nv1 = qsnr(F, x, o.NVFP4, 16, 1, o.SCALE_NV_DYNAMIC)
    nv16 = qsnr(F, x, o.NVFP4, 16, 16, o.SCALE_NV_DYNAMIC)
    ceil = qsnr(F, x, o.MXFP4, 32, 1, o.SCALE_CEIL_NOCLIP)
    oas = qsnr(F, x, o.MXFP4, 32, 1, o.SCALE_OAS)
    assert mx32 > mx1 + 0.3, (mx32, mx1)
    assert nv16 < nv1 - 0.1, (nv16, nv1)
    assert 0.3 < oas - ceil < 0.8, (oas, ceil)


def test_quant_error_of_empty_input(F):
    import gpu_util as gu
    plan = F.fp4q_plan_create(o.MXFP4, 32, 32, o.SCALE_FLOOR_OCP)
    out = gu.Guarded(24)
    F.fp4q_quant_error(plan, 0, 0, 4096, None, out.view)
    torch.cuda.synchronize()
    out.check("out")
    s, e, q = out.numpy().view(np.float64)
    assert s == 0.0 and e == 0.0 and q == math.inf
