"""GPU parity at the five workloads' full sizes, in the launch configuration the bench
times.  The CUDA path runs on the whole tensor; the oracle checks every row of the small
workloads and a sample of rows (first, last and random) of the large ones."""

import numpy as np
import pytest

import oracle as o
from microscaling_fp4_quantization_b200 import workloads as W
from parity import assert_parity, rotated_value_error

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F(cuda_device):
    from microscaling_fp4_quantization_b200 import fp4q
    return fp4q


def sample_rows(M, n=192, seed=0):
    if M <= n:
        return np.arange(M)
    rng = np.random.default_rng(seed)
    mid = rng.choice(np.arange(32, M - 32), n - 64, replace=False)
    return np.unique(np.concatenate([np.arange(32), mid, np.arange(M - 32, M)]))


def check_workload(F, w, rows=None, x=None):
    """Both kernels (butterfly and tensor core) against the oracle on the same input."""
    import gpu_util as gu
    x = w.generate() if x is None else x
    ts = None
    if w.fmt == o.NVFP4:
        ts = o.nv_tensor_scale(o.rotated_amax(x, w.block))
        # the library's own amax pass agrees with the oracle's
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
        reps[kernel] = assert_parity(res, out["codes"], out["scales"], f"{w.name} kernel {kernel}")
        err = rotated_value_error(out["y"], res)
        assert err <= 1e-5, (w.name, kernel, err)
        del out
    return reps, x


def test_small_mx(F):
    check_workload(F, W.SMALL_MX)


def test_nv_4k(F):
    check_workload(F, W.NV_4K)


@pytest.mark.parametrize("m", [1, 4, 16])
def test_decode_rows(F, m):
    check_workload(F, W.DECODE[[1, 4, 16].index(m)])


def test_mx_8k_floor_and_ceil(F):
    rows = sample_rows(W.MX_8K_FLOOR.M, seed=2)
    _, x = check_workload(F, W.MX_8K_FLOOR, rows=rows)
    check_workload(F, W.MX_8K_CEIL, rows=rows, x=x)


def test_prefill_nv_and_mx(F):
    rows = sample_rows(W.PREFILL_NV.M, n=160, seed=4)
    _, x = check_workload(F, W.PREFILL_NV, rows=rows)
    check_workload(F, W.PREFILL_MX, rows=rows, x=x)
