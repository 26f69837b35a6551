"""The no-allocation NVFP4 dynamic-scale entry point, checked against the planned one.

Some callers cannot allocate device memory (the library runs inside a framework or a
serving runtime whose allocator owns all device memory, or in a service that must not
allocate after start-up), so they cannot create the dynamic-scale plan, which allocates its
partial-maximum array.  fp4q_rotate_quantize_nvfp4_dynamic_noalloc keeps that array in a
fixed buffer inside the library instead.  This test calls it twice in a row through the C
ABI, on different inputs, and requires the same codes, scales and tensor scale as
fp4q_rotate_quantize with an FP4Q_SCALE_NV_DYNAMIC plan on the same (butterfly) kernel —
exact equality, inside the parity tolerance the other tests use.  This file is collected
last on purpose."""

import numpy as np
import pytest
import torch

from microscaling_fp4_quantization_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("b", [16, 128])
def test_noalloc_matches_planned_entry_point(cuda_device, b):
    from microscaling_fp4_quantization_b200 import fp4q as F
    plan = F.fp4q_plan_create(F.FP4Q_NVFP4, 16, b, F.FP4Q_SCALE_NV_DYNAMIC)
    F.fp4q_plan_set_kernel(plan, F.FP4Q_KERNEL_BUTTERFLY)
    shapes = [(512, 4096), (37, 6 * max(b, 32))]
    for call, (M, K) in enumerate(shapes):             # two calls in a row, different inputs
        w = W.Workload(f"noalloc_{call}", M, K, 40 + call, "normal", max(1, K // 200), 50.0,
                       row_lognormal_sigma=1.0, fmt=W.NVFP4, group=16, block=b, rule=W.SCALE_NV_DYNAMIC)
        x = torch.from_numpy(w.generate().view(np.int16)).to(cuda_device).view(torch.bfloat16)
        c_ref = torch.empty((M, K // 2), dtype=torch.uint8, device=cuda_device)
        s_ref = torch.empty((M, K // 16), dtype=torch.uint8, device=cuda_device)
        t_ref = torch.empty(1, dtype=torch.float32, device=cuda_device)
        F.fp4q_rotate_quantize(plan, x, M, K, c_ref, s_ref, t_ref)
        c_na = torch.full((M, K // 2), 0xEE, dtype=torch.uint8, device=cuda_device)
        s_na = torch.full((M, K // 16), 0xEE, dtype=torch.uint8, device=cuda_device)
        t_na = torch.full((1,), -1.0, dtype=torch.float32, device=cuda_device)
        F.fp4q_rotate_quantize_nvfp4_dynamic_noalloc(x, M, K, b, c_na, s_na, t_na)
        torch.cuda.synchronize()
        assert F.fp4q_device_status() == F.FP4Q_OK
        assert t_na.item() == t_ref.item()
        assert torch.equal(c_na, c_ref) and torch.equal(s_na, s_ref), (b, M, K)


def test_noalloc_rejects_bad_arguments(cuda_device):
    from microscaling_fp4_quantization_b200 import fp4q as F
    call = lambda *a: F.raw_call("fp4q_rotate_quantize_nvfp4_dynamic_noalloc", *a)
    A = 1 << 20
    assert call(A, 4, 100, 16, A, A, A, None) == F.FP4Q_ERR_SHAPE
    assert call(A, 4, 128, 3, A, A, A, None) == F.FP4Q_ERR_UNSUPPORTED
    assert call(A, 4, 128, 16, A, A, None, None) == F.FP4Q_ERR_ARG
    assert call(A + 8, 4, 128, 16, A, A, A, None) == F.FP4Q_ERR_ALIGN
