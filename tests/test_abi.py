"""The C ABI library, without a GPU: it loads, it exports every function include/*.h
declares, and argument errors come back as status codes before any CUDA call."""

import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def F():
    from microscaling_fp4_quantization_b200 import build
    build.build()
    from microscaling_fp4_quantization_b200 import fp4q
    return fp4q


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b(fp4q_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_every_declared_symbol_is_exported(F):
    names = declared_functions()
    assert "fp4q_rotate_quantize" in names and "fp4q_plan_create" in names
    lib = ctypes.CDLL(F.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) <= set(F.EXPORTED) | {n for n in names if hasattr(lib, n)}


def test_version_and_strings(F):
    assert F.fp4q_version() >= 100
    for s in range(7):
        assert F.fp4q_status_string(s)


def test_plan_validation_without_gpu(F):
    for args in [(0, 16, 32, 0), (1, 32, 16, 3), (0, 32, 3, 0), (0, 32, 256, 0), (0, 32, 32, 3), (1, 16, 16, 0),
                 (3, 32, 32, 0), (0, 32, 0, 0), (2, 16, 32, 0), (2, 32, 32, 3)]:
        with pytest.raises(F.Fp4qError) as e:
            F.fp4q_plan_create(*args)
        assert e.value.status == F.FP4Q_ERR_UNSUPPORTED, args
    assert F.raw_call("fp4q_plan_create", None, 0, 32, 32, 0) == F.FP4Q_ERR_ARG
    # MX plans need a device only for the error pass's scratch, so they can be made on a CPU-only machine
    p = F.fp4q_plan_create(F.FP4Q_MXFP4, 32, 32, F.FP4Q_SCALE_FLOOR_OCP)
    F.fp4q_plan_destroy(p)
    assert F.raw_call("fp4q_plan_destroy", None) == F.FP4Q_OK


def test_kernel_selection_without_gpu(F):
    p = F.fp4q_plan_create(F.FP4Q_MXFP4, 32, 1, F.FP4Q_SCALE_FLOOR_OCP)
    assert F.raw_call("fp4q_plan_set_kernel", p.handle, F.FP4Q_KERNEL_TENSOR_CORE) == F.FP4Q_ERR_UNSUPPORTED
    assert F.raw_call("fp4q_plan_set_kernel", p.handle, 7) == F.FP4Q_ERR_ARG
    assert F.raw_call("fp4q_plan_set_kernel", None, 0) == F.FP4Q_ERR_ARG
    q = F.fp4q_plan_create(F.FP4Q_MXFP4, 32, 128, F.FP4Q_SCALE_CEIL_NOCLIP)
    for k in (F.FP4Q_KERNEL_TENSOR_CORE, F.FP4Q_KERNEL_BUTTERFLY, F.FP4Q_KERNEL_AUTO):
        F.fp4q_plan_set_kernel(q, k)


def test_sign_validation_without_gpu(F):
    p = F.fp4q_plan_create(F.FP4Q_MXFP4, 32, 128, F.FP4Q_SCALE_FLOOR_OCP)
    ss = lambda *a: F.raw_call("fp4q_plan_set_signs", *a)
    A = 1 << 20
    assert ss(None, A, 128) == F.FP4Q_ERR_ARG
    assert ss(p.handle, A, 100) == F.FP4Q_ERR_SHAPE            # not a multiple of max(g, b)
    assert ss(p.handle, A, 0) == F.FP4Q_ERR_SHAPE
    assert ss(p.handle, A, 1 << 35) == F.FP4Q_ERR_SHAPE
    assert ss(p.handle, A + 2, 128) == F.FP4Q_ERR_ALIGN
    assert ss(p.handle, A, 256) == F.FP4Q_OK
    rq = lambda *a: F.raw_call("fp4q_rotate_quantize", *a)
    assert rq(p.handle, A, 4, 128, A, A, None, None) == F.FP4Q_ERR_SHAPE      # K differs from the signs'
    F.fp4q_plan_set_kernel(p, F.FP4Q_KERNEL_TENSOR_CORE)       # signs work on both kernels
    assert ss(p.handle, None, 0) == F.FP4Q_OK                   # cleared
    assert ss(p.handle, A, 256) == F.FP4Q_OK
    F.fp4q_plan_destroy(p)


def test_mbs_validation_without_gpu(F):
    p = F.fp4q_plan_create(F.FP4Q_MXFP4_MBS, 32, 32, F.FP4Q_SCALE_OAS)
    A = 1 << 20
    mq = lambda *a: F.raw_call("fp4q_rotate_quantize_mbs", *a)
    assert mq(p.handle, A, 4, 96, A, A, A, None) == F.FP4Q_ERR_SHAPE          # K % 128 (the macro block)
    assert mq(p.handle, A, 4, 256, A, A, None, None) == F.FP4Q_ERR_ARG        # no macro output
    assert mq(p.handle, A + 8, 4, 256, A, A, A, None) == F.FP4Q_ERR_ALIGN
    assert mq(p.handle, A, 0, 256, None, None, None, None) == F.FP4Q_OK       # empty call
    rq = lambda *a: F.raw_call("fp4q_rotate_quantize", *a)
    assert rq(p.handle, A, 4, 256, A, A, None, None) == F.FP4Q_ERR_UNSUPPORTED
    dq = lambda *a: F.raw_call("fp4q_dequantize", *a)
    assert dq(p.handle, A, A, None, 4, 256, 0, A, None) == F.FP4Q_ERR_UNSUPPORTED
    dm = lambda *a: F.raw_call("fp4q_dequantize_mbs", *a)
    assert dm(p.handle, A, A, None, 4, 256, 0, A, None) == F.FP4Q_ERR_ARG
    # the tensor-core kernel takes MBS plans whose blocks hold whole groups (b >= 32)
    assert F.raw_call("fp4q_plan_set_kernel", p.handle, F.FP4Q_KERNEL_TENSOR_CORE) == F.FP4Q_OK
    p16 = F.fp4q_plan_create(F.FP4Q_MXFP4_MBS, 32, 16, F.FP4Q_SCALE_OAS)
    assert F.raw_call("fp4q_plan_set_kernel", p16.handle, F.FP4Q_KERNEL_TENSOR_CORE) == F.FP4Q_ERR_UNSUPPORTED
    F.fp4q_plan_destroy(p16)
    mx = F.fp4q_plan_create(F.FP4Q_MXFP4, 32, 32, F.FP4Q_SCALE_OAS)
    assert mq(mx.handle, A, 4, 256, A, A, A, None) == F.FP4Q_ERR_UNSUPPORTED
    assert dm(mx.handle, A, A, A, 4, 256, 0, A, None) == F.FP4Q_ERR_UNSUPPORTED
    F.fp4q_plan_destroy(p)


def test_gemm_validation_without_gpu(F):
    gm = lambda *a: F.raw_call("fp4q_gemm", *a)
    A = 1 << 20
    assert gm(5, A, A, None, A, A, None, 128, 256, 256, A, None) == F.FP4Q_ERR_UNSUPPORTED
    assert gm(F.FP4Q_MXFP4, A, A, None, A, A, None, 128, 250, 256, A, None) == F.FP4Q_ERR_SHAPE   # N % 32
    assert gm(F.FP4Q_MXFP4, A, A, None, A, A, None, 128, 256, 300, A, None) == F.FP4Q_ERR_SHAPE   # K % 256
    assert gm(F.FP4Q_MXFP4, A, A, None, A, A, None, 128, 256, 0, A, None) == F.FP4Q_ERR_SHAPE     # empty K
    assert gm(F.FP4Q_MXFP4, A, A, None, A, A, None, 0, 256, 256, None, None) == F.FP4Q_OK         # empty M
    assert gm(F.FP4Q_MXFP4, None, A, None, A, A, None, 128, 256, 256, A, None) == F.FP4Q_ERR_ARG
    assert gm(F.FP4Q_NVFP4, A, A, None, A, A, A, 128, 256, 256, A, None) == F.FP4Q_ERR_ARG       # tensor scale
    assert gm(F.FP4Q_MXFP4, A + 8, A, None, A, A, None, 128, 256, 256, A, None) == F.FP4Q_ERR_ALIGN
    assert gm(F.FP4Q_MXFP4, A, A, None, A, A, None, 128, 256, 256, A + 2, None) == F.FP4Q_ERR_ALIGN


def test_call_validation_without_gpu(F):
    p = F.fp4q_plan_create(F.FP4Q_MXFP4, 32, 128, F.FP4Q_SCALE_FLOOR_OCP)
    rq = lambda *a: F.raw_call("fp4q_rotate_quantize", *a)
    A = 1 << 20            # an aligned fake address: never dereferenced, validation fails first
    assert rq(None, A, 4, 128, A, A, None, None) == F.FP4Q_ERR_ARG
    assert rq(p.handle, A, 4, 96, A, A, None, None) == F.FP4Q_ERR_SHAPE        # K % 128
    assert rq(p.handle, A, -1, 128, A, A, None, None) == F.FP4Q_ERR_SHAPE
    assert rq(p.handle, A, 1 << 34, 1 << 7, A, A, None, None) == F.FP4Q_ERR_SHAPE   # > 2^40 elements
    assert rq(p.handle, None, 4, 128, A, A, None, None) == F.FP4Q_ERR_ARG
    assert rq(p.handle, A, 4, 128, None, A, None, None) == F.FP4Q_ERR_ARG
    assert rq(p.handle, A + 8, 4, 128, A, A, None, None) == F.FP4Q_ERR_ALIGN
    assert rq(p.handle, A, 4, 128, A + 4, A, None, None) == F.FP4Q_ERR_ALIGN
    assert rq(p.handle, A, 4, 128, A, A + 2, None, None) == F.FP4Q_ERR_ALIGN
    assert rq(p.handle, A, 0, 128, None, None, None, None) == F.FP4Q_OK          # empty call
    dq = lambda *a: F.raw_call("fp4q_dequantize", *a)
    assert dq(p.handle, A, A, None, 4, 100, 0, A, None) == F.FP4Q_ERR_SHAPE
    assert dq(p.handle, A, None, None, 4, 128, 0, A, None) == F.FP4Q_ERR_ARG
    assert dq(p.handle, A, A, None, 4, 128, 0, A + 4, None) == F.FP4Q_ERR_ALIGN
    am = lambda *a: F.raw_call("fp4q_amax", *a)
    assert am(p.handle, A, 4, 128, A, None) == F.FP4Q_ERR_UNSUPPORTED            # MX plan
    qe = lambda *a: F.raw_call("fp4q_quant_error", *a)
    assert qe(None, A, 4, 128, None, A, None) == F.FP4Q_ERR_ARG
    assert qe(p.handle, A, 4, 96, None, A, None) == F.FP4Q_ERR_SHAPE
    assert qe(p.handle, A, 4, 128, None, None, None) == F.FP4Q_ERR_ARG           # no output
    assert qe(p.handle, None, 4, 128, None, A, None) == F.FP4Q_ERR_ARG
    assert qe(p.handle, A + 8, 4, 128, None, A, None) == F.FP4Q_ERR_ALIGN
    assert qe(p.handle, A, 4, 128, None, A + 4, None) == F.FP4Q_ERR_ALIGN         # out: 8 bytes
    # an MX plan made without a CUDA device holds no scratch for the error pass (with a
    # device the call would get past validation, so it is not made with the fake address)
    from conftest import gpu_available
    if not gpu_available():
        assert qe(p.handle, A, 4, 128, None, A, None) == F.FP4Q_ERR_UNSUPPORTED
    F.fp4q_plan_destroy(p)


def test_product_path_does_not_reference_the_oracle():
    pkg = os.path.join(ROOT, "microscaling_fp4_quantization_b200")
    for path in glob.glob(os.path.join(pkg, "**", "*"), recursive=True):
        if os.path.isfile(path) and path.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
            text = open(path, encoding="utf-8").read()
            assert "import oracle" not in text and "from oracle" not in text, path
