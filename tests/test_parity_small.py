"""GPU parity on small shapes: every format / block / rule the library offers, against
the CPU oracle, through the C ABI.  Shapes span several units per lane, several warps and
ragged tails; inputs include adversarial rows."""

import numpy as np
import pytest

import oracle as o
from microscaling_fp4_quantization_b200 import workloads as W
from oracle.parity import assert_parity, rotated_value_error

pytestmark = pytest.mark.gpu

BLOCKS = [1, 2, 4, 8, 16, 32, 64, 128]
COMBOS = ([(o.MXFP4, 32, b, r) for b in BLOCKS for r in (o.SCALE_FLOOR_OCP, o.SCALE_CEIL_NOCLIP, o.SCALE_OAS)]
          + [(o.NVFP4, 16, b, r) for b in BLOCKS for r in (o.SCALE_NV_STATIC, o.SCALE_NV_DYNAMIC)])


def combo_id(c):
    fmt, g, b, r = c
    return f"{'mx' if fmt == o.MXFP4 else 'nv'}-b{b}-{W.RULE_NAMES[r]}"


def make_input(M, K, seed, adversarial=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K)).astype(np.float32)
    x *= np.exp(rng.normal(0, 1.5, (M, 1))).astype(np.float32)
    cols = rng.choice(K, max(1, K // 200), replace=False)
    x[:, cols] *= 50
    if adversarial and M >= 8:
        x[0] = 0.0                                        # all-zero row
        x[1] = 0.0
        x[1, K // 3] = -7.5                               # one spike
        x[2] = np.ldexp(1.0, rng.integers(-20, 20, K)).astype(np.float32) * rng.choice([-1, 1], K)
        x[3] = -0.0                                       # negative zeros
        x[4] *= 1e-30                                     # tiny row (zero NV block scales)
        x[5] = rng.choice([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, -0.25, -5.0], K)   # midpoints at X = 1
        x[6] *= 1e4
    return W.f32_to_bf16_bits(x)


def shapes_for(unit):
    return [(1, unit), (3, 2 * unit), (37, 6 * unit), (130, 4096 // unit * unit), (1000, 1536)]


@pytest.fixture(scope="module")
def F(cuda_device):
    from microscaling_fp4_quantization_b200 import fp4q
    return fp4q


def mma_capable(combo):
    fmt, g, b, rule = combo
    return b >= 16 and b >= g


KERNEL_CASES = ([(c, 1) for c in COMBOS] + [(c, 2) for c in COMBOS if mma_capable(c)])


@pytest.mark.parametrize("combo,kernel", KERNEL_CASES,
                         ids=[combo_id(c) + ("-tc" if k == 2 else "-bf") for c, k in KERNEL_CASES])
def test_rotate_quantize_matches_oracle(F, combo, kernel):
    """kernel 1: the butterfly kernel; 2: the tensor-core kernel."""
    import gpu_util as gu
    fmt, g, b, rule = combo
    plan = F.fp4q_plan_create(fmt, g, b, rule)
    F.fp4q_plan_set_kernel(plan, kernel)
    unit = max(g, b)
    for i, (M, K) in enumerate(shapes_for(unit)):
        x = make_input(M, K, seed=100 * b + 10 * rule + i)
        adversarial = M >= 8
        if fmt == o.NVFP4 and rule == o.SCALE_NV_STATIC:
            s_g = o.nv_tensor_scale(o.rotated_amax(x, b))
            res = o.rotate_quantize(x, fmt, g, b, rule, tensor_scale=s_g)
            out = gu.run_rotate_quantize(F, plan, x, tensor_scale=s_g, dump=True)
        else:
            res = o.rotate_quantize(x, fmt, g, b, rule)
            out = gu.run_rotate_quantize(F, plan, x, dump=True)
        if fmt == o.NVFP4 and rule == o.SCALE_NV_DYNAMIC:
            rel = abs(float(out["tensor_scale"]) - float(res["tensor_scale"])) / float(res["tensor_scale"])
            assert rel <= 2.5e-7, (M, K, out["tensor_scale"], res["tensor_scale"])
        # rows built on ties (midpoints, powers of two) make near-ties dense: there only the
        # "every mismatch is flagged" part of the rule applies; realistic rows get the count bound too
        assert_parity(res, out["codes"], out["scales"], f"{combo_id(combo)} {M}x{K}", count_bound=not adversarial)
        if adversarial:
            real = slice(8, M)
            res_r = {k: (v[real] if isinstance(v, np.ndarray) and v.ndim == 2 and v.shape[0] == M else v)
                     for k, v in res.items()}
            assert_parity(res_r, out["codes"][real], out["scales"][real], f"{combo_id(combo)} {M}x{K} rows 8+")
        assert rotated_value_error(out["y"], res) <= 1e-5, (M, K)
        # the non-dumping kernel gives the same bytes as the dumping one
        plain = gu.run_rotate_quantize(F, plan, x, tensor_scale=out["tensor_scale"] if fmt == o.NVFP4 and
                                       rule == o.SCALE_NV_STATIC else None)
        assert np.array_equal(plain["codes"], out["codes"]) and np.array_equal(plain["scales"], out["scales"])


@pytest.mark.parametrize("rule", [o.SCALE_FLOOR_OCP, o.SCALE_CEIL_NOCLIP, o.SCALE_OAS])
def test_mx_ties_and_golden_groups_exact(F, rule):
    """Block 1: every hand-worked group and every exact midpoint is reproduced bit for bit."""
    import gpu_util as gu
    import test_oracle_pins as pins
    rows = [r for r in pins.load_rows("mx_worked_groups.txt") if pins.RULES[r[0]] == rule]
    x = np.zeros((len(rows), 32), np.float32)
    for i, r in enumerate(rows):
        x[i, 0], x[i, 1] = float(r[1]), float(r[2])
    xb = pins.bf16(x)
    plan = F.fp4q_plan_create(o.MXFP4, 32, 1, rule)
    out = gu.run_rotate_quantize(F, plan, xb)
    q = o.unpack_nibbles(out["codes"])
    for i, r in enumerate(rows):
        assert out["scales"][i, 0] == int(r[3]), r
        assert (q[i, 0], q[i, 1]) == (int(r[4]), int(r[5])), r


def test_nv_golden_groups_exact(F):
    import gpu_util as gu
    import test_oracle_pins as pins
    rows = pins.load_rows("nv_worked_groups.txt")
    plan = F.fp4q_plan_create(o.NVFP4, 16, 1, o.SCALE_NV_STATIC)
    for r in rows:
        x = np.zeros((1, 16), np.float32)
        x[0, 0], x[0, 1] = float(r[1]), float(r[2])
        out = gu.run_rotate_quantize(F, plan, pins.bf16(x), tensor_scale=float(r[0]))
        q = o.unpack_nibbles(out["codes"])
        assert out["scales"][0, 0] == int(r[3]), r
        assert (q[0, 0], q[0, 1]) == (int(r[4]), int(r[5])), r


@pytest.mark.parametrize("b", [16, 128])
def test_amax_entry_point(F, b):
    import gpu_util as gu
    plan = F.fp4q_plan_create(o.NVFP4, 16, b, o.SCALE_NV_STATIC)
    for M, K in [(1, 128), (300, 1024), (2048, 4096)]:
        x = make_input(M, K, seed=M + b)
        ours = gu.run_amax(F, plan, x)
        ref = o.nv_tensor_scale(o.rotated_amax(x, b))
        assert abs(float(ours) - float(ref)) <= 2.5e-7 * float(ref), (M, K, ours, ref)
    assert gu.run_amax(F, plan, np.zeros((4, 128), np.uint16)) == np.float32(1.0)


def exact_sum_input(M, K, seed):
    """Rows of small integers times a power of two per row: every block sum of up to 128 of
    them is an integer below 2^14 times that power of two, exact in fp32, so the kernel's
    butterfly sums equal the exact sums and its rotated values RN(s / sqrt(b)) equal the
    oracle's fp64 product rounded once."""
    rng = np.random.default_rng(seed)
    x = rng.integers(-64, 65, (M, K)).astype(np.float32)
    x *= np.ldexp(1.0, rng.integers(-30, 30, (M, 1))).astype(np.float32)
    return W.f32_to_bf16_bits(x)


@pytest.mark.parametrize("b", BLOCKS)
def test_amax_equals_the_definition_on_exact_sums(F, b):
    """s_g = fp32(A_t / 2688) with A_t the largest fp32 rotated value: bit for bit, for every
    block size (1 / sqrt(b) irrational for b = 2, 8, 32, 128), through fp4q_amax and through a
    DYNAMIC plan's own amax pass, on both kernels (each runs the amax pass on the kernel its
    plan names; AUTO on the tensor core from 2^22 elements on, b >= 16)."""
    import gpu_util as gu
    kernels = (0, 1, 2) if b >= 16 else (0, 1)
    for i, (M, K) in enumerate([(1, 128), (300, 1024), (2048, 4096)]):
        x = exact_sum_input(M, K, seed=31 * b + i)
        ref = o.nv_tensor_scale(o.rotated_amax(x, b))
        for kernel in kernels:
            plan = F.fp4q_plan_create(o.NVFP4, 16, b, o.SCALE_NV_STATIC)
            F.fp4q_plan_set_kernel(plan, kernel)
            assert gu.run_amax(F, plan, x) == ref, (b, M, K, kernel)
        res = o.rotate_quantize(x, o.NVFP4, 16, b, o.SCALE_NV_DYNAMIC)
        for kernel in (1, 2) if b >= 16 else (1,):
            dyn = F.fp4q_plan_create(o.NVFP4, 16, b, o.SCALE_NV_DYNAMIC)
            F.fp4q_plan_set_kernel(dyn, kernel)
            out = gu.run_rotate_quantize(F, dyn, x)
            assert out["tensor_scale"] == ref, (b, M, K, kernel)
            assert_parity(res, out["codes"], out["scales"], f"nv-b{b} exact sums {M}x{K} dynamic kernel {kernel}")


def test_empty_input_is_a_no_op(F):
    import torch
    plan = F.fp4q_plan_create(o.MXFP4, 32, 32, o.SCALE_FLOOR_OCP)
    F.fp4q_rotate_quantize(plan, 0, 0, 4096, 0, 0, None)
    F.fp4q_rotate_quantize(plan, 0, 16, 0, 0, 0, None)
    torch.cuda.synchronize()
    assert F.fp4q_device_status() == F.FP4Q_OK


@pytest.mark.parametrize("kernel", [0, 1, 2])
def test_amax_of_an_empty_tensor_is_one(F, kernel):
    """s_g of an empty X is 1 (the all-zero rule), whichever kernel the plan names."""
    import torch
    plan = F.fp4q_plan_create(o.NVFP4, 16, 16, o.SCALE_NV_STATIC)
    F.fp4q_plan_set_kernel(plan, kernel)
    ts = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    F.fp4q_amax(plan, 0, 0, 4096, ts)
    torch.cuda.synchronize()
    assert F.fp4q_device_status() == F.FP4Q_OK
    assert ts.item() == 1.0
