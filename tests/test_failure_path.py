"""The failure path of the bounded waits, exercised without a GPU fault: a kernel whose wait
nothing satisfies gives up after its time limit, the status word reports FP4Q_ERR_TIMEOUT once
(reading clears it), and the CUDA context stays usable for the next correct call."""

import numpy as np
import pytest

import oracle as o
from oracle.parity import assert_parity
from test_parity_small import make_input

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F(cuda_device):
    from microscaling_fp4_quantization_b200 import fp4q
    return fp4q


def test_bounded_wait_reports_timeout_and_context_survives(F):
    import time

    import gpu_util as gu
    import torch
    assert F.fp4q_device_status() == F.FP4Q_OK
    t0 = time.perf_counter()
    F.fp4q_selftest_wait_timeout()
    assert F.fp4q_device_status() == F.FP4Q_ERR_TIMEOUT   # synchronizes: the wait gave up
    elapsed = time.perf_counter() - t0
    assert 0.5 < elapsed < 30.0, elapsed
    assert F.fp4q_device_status() == F.FP4Q_OK            # read once, then clear
    # the context still runs the library correctly
    plan = F.fp4q_plan_create(o.MXFP4, 32, 32, o.SCALE_FLOOR_OCP)
    x = make_input(64, 1024, seed=3, adversarial=False)
    res = o.rotate_quantize(x, o.MXFP4, 32, 32, o.SCALE_FLOOR_OCP)
    out = gu.run_rotate_quantize(F, plan, x)
    assert_parity(res, out["codes"], out["scales"], "after the self-test")
    torch.cuda.synchronize()
