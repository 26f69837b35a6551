"""Child process of test_contexts.py (run on its own, never imported by pytest).

Drives the library under two CUDA contexts on device 0 — the primary context and a second
one made through the driver API — with every buffer allocated through the driver API in the
context that uses it.  Prints one JSON object with what it saw; the parent test judges it.
No torch: the library's own runtime picks up whichever context is current."""

import ctypes
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from microscaling_fp4_quantization_b200 import fp4q as F  # noqa: E402
from microscaling_fp4_quantization_b200 import workloads as W  # noqa: E402

cu = ctypes.CDLL("libcuda.so.1")
_u64 = ctypes.c_uint64


def ck(r, what):
    if r != 0:
        raise RuntimeError(f"{what}: CUresult {r}")


class Buf:
    """Device memory of the context current at construction."""

    def __init__(self, nbytes, host=None):
        self.n = nbytes
        self.ptr = _u64()
        ck(cu.cuMemAlloc_v2(ctypes.byref(self.ptr), _u64(nbytes)), "cuMemAlloc")
        if host is not None:
            ck(cu.cuMemcpyHtoD_v2(self.ptr, host.ctypes.data_as(ctypes.c_void_p), _u64(nbytes)), "cuMemcpyHtoD")

    def get(self, dtype):
        out = np.empty(self.n // np.dtype(dtype).itemsize, dtype)
        ck(cu.cuMemcpyDtoH_v2(out.ctypes.data_as(ctypes.c_void_p), self.ptr, _u64(self.n)), "cuMemcpyDtoH")
        return out

    def free(self):
        ck(cu.cuMemFree_v2(self.ptr), "cuMemFree")


def run(x, M, K, b, plan=None):
    """codes, scales and s_g of one NVFP4 DYNAMIC rotate + quantize in the current context:
    through the plan when given, else through the no-allocation entry point."""
    xb = Buf(x.nbytes, x)
    codes, scales, ts = Buf(M * K // 2), Buf(M * K // 16), Buf(4)
    if plan is None:
        st = F.raw_call("fp4q_rotate_quantize_nvfp4_dynamic_noalloc", xb.ptr.value, M, K, b, codes.ptr.value,
                        scales.ptr.value, ts.ptr.value, 0)
    else:
        st = F.raw_call("fp4q_rotate_quantize", plan.handle, xb.ptr.value, M, K, codes.ptr.value, scales.ptr.value,
                        ts.ptr.value, 0)
    assert st == F.FP4Q_OK, st
    ck(cu.cuCtxSynchronize(), "cuCtxSynchronize")
    assert F.fp4q_device_status() == F.FP4Q_OK
    out = (codes.get(np.uint8), scales.get(np.uint8), ts.get(np.float32))
    for bb in (xb, codes, scales, ts):
        bb.free()
    return out


def same(a, b):
    return all(np.array_equal(p, q) for p, q in zip(a, b))


def refused_first(plan, K):
    """Each plan call with an invalid row count M = -1: FP4Q_ERR_ARG means the context check
    came first; FP4Q_ERR_SHAPE means it passed (nothing is launched either way)."""
    return {
        "rotate_quantize": F.raw_call("fp4q_rotate_quantize", plan.handle, 0, -1, K, 0, 0, 0, 0),
        "amax": F.raw_call("fp4q_amax", plan.handle, 0, -1, K, 0, 0),
        "quant_error": F.raw_call("fp4q_quant_error", plan.handle, 0, -1, K, 0, 0, 0),
        "dequantize": F.raw_call("fp4q_dequantize", plan.handle, 0, 0, 0, -1, K, 0, 0, 0),
    }


def main():
    b = int(sys.argv[1]) if len(sys.argv) > 1 else 128
    M, K = 512, 4096
    w = W.Workload("contexts", M, K, 41, "normal", 20, 50.0, row_lognormal_sigma=1.0, fmt=W.NVFP4, group=16,
                   block=b, rule=W.SCALE_NV_DYNAMIC)
    x = np.ascontiguousarray(w.generate())
    ck(cu.cuInit(0), "cuInit")
    dev = ctypes.c_int()
    ck(cu.cuDeviceGet(ctypes.byref(dev), 0), "cuDeviceGet")
    primary = ctypes.c_void_p()
    ck(cu.cuDevicePrimaryCtxRetain(ctypes.byref(primary), dev), "cuDevicePrimaryCtxRetain")
    ck(cu.cuCtxPushCurrent_v2(primary), "cuCtxPushCurrent")
    seen = {}

    plan = F.fp4q_plan_create(F.FP4Q_NVFP4, 16, b, F.FP4Q_SCALE_NV_DYNAMIC)
    F.fp4q_plan_set_kernel(plan, F.FP4Q_KERNEL_BUTTERFLY)
    ref = run(x, M, K, b, plan)
    seen["noalloc_primary_first"] = same(run(x, M, K, b), ref)
    seen["checks_in_primary"] = refused_first(plan, K)

    ctx2 = ctypes.c_void_p()
    ck(cu.cuCtxCreate_v2(ctypes.byref(ctx2), 0, dev), "cuCtxCreate")      # now current
    seen["noalloc_second_context"] = same(run(x, M, K, b), ref)
    seen["checks_in_second_context"] = refused_first(plan, K)
    plan2 = F.fp4q_plan_create(F.FP4Q_NVFP4, 16, b, F.FP4Q_SCALE_NV_DYNAMIC)
    F.fp4q_plan_set_kernel(plan2, F.FP4Q_KERNEL_BUTTERFLY)
    seen["plan_made_in_second_context"] = same(run(x, M, K, b, plan2), ref)
    F.fp4q_plan_destroy(plan2)
    ck(cu.cuCtxDestroy_v2(ctx2), "cuCtxDestroy")                        # the primary is current again

    seen["noalloc_primary_after"] = same(run(x, M, K, b), ref)
    seen["planned_primary_after"] = same(run(x, M, K, b, plan), ref)
    F.fp4q_plan_destroy(plan)
    ck(cu.cuCtxPopCurrent_v2(ctypes.byref(ctypes.c_void_p())), "cuCtxPopCurrent")
    ck(cu.cuDevicePrimaryCtxRelease_v2(dev), "cuDevicePrimaryCtxRelease")
    print(json.dumps(seen), flush=True)


if __name__ == "__main__":
    main()
