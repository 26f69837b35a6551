"""GPU parity at the five workloads' full sizes, in the launch configuration the bench
times (the non-dumping kernel the plan picks, and the other kernel too).  The oracle checks
every row of every workload: the large ones are cut into row chunks that a pool of host
processes runs (parity_pool).  The rotated values are checked through the dumping kernel on
a sample of rows (first, last and random), which the oracle recomputes."""

import numpy as np
import pytest

import oracle as o
from microscaling_fp4_quantization_b200 import workloads as W
from oracle.parity import assert_parity, record, rotated_value_error

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F(cuda_device):
    from microscaling_fp4_quantization_b200 import fp4q
    return fp4q


@pytest.fixture(scope="module")
def pool():
    import parity_pool
    with parity_pool.oracle_pool() as p:
        yield p


def sample_rows(M, n=192, seed=0):
    if M <= n:
        return np.arange(M)
    rng = np.random.default_rng(seed)
    mid = rng.choice(np.arange(32, M - 32), n - 64, replace=False)
    return np.unique(np.concatenate([np.arange(32), mid, np.arange(M - 32, M)]))


KERNELS = {1: "butterfly", 2: "tensor_core"}


def oracle_tensor_scale(x, block, pool=None):
    if pool is None:
        return o.nv_tensor_scale(o.rotated_amax(x, block))
    import parity_pool
    return o.nv_tensor_scale(parity_pool.rotated_amax(pool, x, block))


def check_workload(F, w, rows=None, x=None, pool=None):
    """Both kernels (butterfly and tensor core) against the oracle on the same input, with
    the rotated values dumped (on ``rows`` only, when given)."""
    import gpu_util as gu
    x = w.generate() if x is None else x
    ts = None
    if w.fmt == o.NVFP4:
        ts = oracle_tensor_scale(x, w.block, pool)
        # the library's own amax pass agrees with the oracle's (to the fp32 rounding of the
        # butterfly sums; equality where those are exact is tested in test_parity_small)
        nv_plan = F.fp4q_plan_create(o.NVFP4, 16, w.block, o.SCALE_NV_STATIC)
        ours = gu.run_amax(F, nv_plan, x)
        assert abs(float(ours) - float(ts)) <= 2.5e-7 * float(ts), (ours, ts)
    xs = x if rows is None else x[rows]
    res = o.rotate_quantize(xs, w.fmt, w.group, w.block, w.rule, tensor_scale=ts)
    reps = {}
    for kernel in (F.FP4Q_KERNEL_BUTTERFLY, F.FP4Q_KERNEL_TENSOR_CORE):
        plan = F.fp4q_plan_create(w.fmt, w.group, w.block, w.rule)
        F.fp4q_plan_set_kernel(plan, kernel)
        out = gu.run_rotate_quantize(F, plan, x, tensor_scale=ts, dump=True, rows=rows)
        what = "all rows" if rows is None else f"{len(rows)} sampled rows, dumping kernel"
        reps[kernel] = assert_parity(res, out["codes"], out["scales"],
                                     f"workload {w.name} {KERNELS[kernel]} ({what})")
        err = rotated_value_error(out["y"], res)
        assert err <= 1e-5, (w.name, kernel, err)
        del out
    return reps, x


def check_workload_all_rows(F, pool, w, x, extra_dynamic=False):
    """Every row, in the bench's launch configuration: the non-dumping kernel on the whole
    tensor (each kernel), against the oracle run chunk by chunk in the pool.  With
    ``extra_dynamic`` (NVFP4), also the DYNAMIC plan, which quantizes with the library's own
    per-tensor scale from its amax pass."""
    import gpu_util as gu
    import parity_pool
    ts = oracle_tensor_scale(x, w.block, pool) if w.fmt == o.NVFP4 else None
    xd = gu.to_device_bf16(x)
    outs, labels = [], []
    for kernel in (F.FP4Q_KERNEL_BUTTERFLY, F.FP4Q_KERNEL_TENSOR_CORE):
        plan = F.fp4q_plan_create(w.fmt, w.group, w.block, w.rule)
        F.fp4q_plan_set_kernel(plan, kernel)
        out = gu.run_rotate_quantize(F, plan, None, tensor_scale=ts, x_dev=xd)
        outs.append((out["codes"], out["scales"]))
        labels.append(f"workload {w.name} {KERNELS[kernel]} (all {w.M} rows)")
    if extra_dynamic:
        plan = F.fp4q_plan_create(o.NVFP4, 16, w.block, o.SCALE_NV_DYNAMIC)
        out = gu.run_rotate_quantize(F, plan, None, x_dev=xd)
        # the library's s_g: the correctly rounded quotient of its rotated amax, which equals the
        # oracle's wherever the fp32 butterfly sum of the largest element is exact, and is within
        # one ulp of it otherwise (every decision that this can move is inside the flagged set)
        assert abs(float(out["tensor_scale"]) - float(ts)) <= np.spacing(np.float32(ts)), (out["tensor_scale"], ts)
        outs.append((out["codes"], out["scales"]))
        labels.append(f"workload {w.name} DYNAMIC, library's own s_g (all {w.M} rows)")
    del xd
    reps = parity_pool.compare_all_rows(pool, x, outs, labels, w.fmt, w.group, w.block, w.rule, tensor_scale=ts)
    for rep in reps:
        record(rep)
    return reps


def test_small_mx(F):
    check_workload(F, W.SMALL_MX)


def test_nv_4k(F):
    check_workload(F, W.NV_4K)


@pytest.mark.parametrize("m", [1, 4, 16])
def test_decode_rows(F, m):
    check_workload(F, W.DECODE[[1, 4, 16].index(m)])


def test_mx_8k_floor_and_ceil(F, pool):
    rows = sample_rows(W.MX_8K_FLOOR.M, seed=2)
    _, x = check_workload(F, W.MX_8K_FLOOR, rows=rows)
    check_workload(F, W.MX_8K_CEIL, rows=rows, x=x)
    check_workload_all_rows(F, pool, W.MX_8K_FLOOR, x)
    check_workload_all_rows(F, pool, W.MX_8K_CEIL, x)


def test_prefill_nv_and_mx(F, pool):
    rows = sample_rows(W.PREFILL_NV.M, n=160, seed=4)
    _, x = check_workload(F, W.PREFILL_NV, rows=rows, pool=pool)
    check_workload(F, W.PREFILL_MX, rows=rows, x=x)
    check_workload_all_rows(F, pool, W.PREFILL_NV, x, extra_dynamic=True)
    check_workload_all_rows(F, pool, W.PREFILL_MX, x)
