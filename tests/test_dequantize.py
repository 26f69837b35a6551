"""GPU parity of fp4q_dequantize against the oracle: bit-exact without the inverse
rotation; within 1e-5 of the block norm with it."""

import numpy as np
import pytest

import oracle as o
from test_parity_small import make_input

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F(cuda_device):
    from microscaling_fp4_quantization_b200 import fp4q
    return fp4q


@pytest.mark.parametrize("fmt,g,b,rule", [(o.MXFP4, 32, 32, o.SCALE_FLOOR_OCP), (o.MXFP4, 32, 128, o.SCALE_CEIL_NOCLIP),
                                          (o.MXFP4, 32, 1, o.SCALE_OAS), (o.NVFP4, 16, 16, o.SCALE_NV_STATIC),
                                          (o.NVFP4, 16, 128, o.SCALE_NV_STATIC), (o.NVFP4, 16, 1, o.SCALE_NV_STATIC)])
def test_dequantize(F, fmt, g, b, rule):
    import gpu_util as gu
    x = make_input(77, 1024, seed=b + fmt)
    ts = o.nv_tensor_scale(o.rotated_amax(x, b)) if fmt == o.NVFP4 else None
    res = o.rotate_quantize(x, fmt, g, b, rule, tensor_scale=ts)
    plan = F.fp4q_plan_create(fmt, g, b, rule)
    d0 = gu.run_dequantize(F, plan, res["codes"], res["scales"], ts, unrotate=False)
    ref0 = o.dequantize(res["codes"], res["scales"], fmt, g, b, ts)
    assert np.array_equal(d0.view(np.uint32) & 0x7FFFFFFF, ref0.view(np.uint32) & 0x7FFFFFFF)
    d1 = gu.run_dequantize(F, plan, res["codes"], res["scales"], ts, unrotate=True)
    ref1 = o.dequantize(res["codes"], res["scales"], fmt, g, b, ts, unrotate_back=True)
    nb = np.linalg.norm(ref1.reshape(77, 1024 // b, b), axis=2)
    err = np.abs(d1 - ref1).reshape(77, 1024 // b, b)
    assert np.all(err <= 1e-5 * nb[..., None] + 1e-30)
