"""bench.py's host logic that needs no GPU: the kernel name each line reports for AUTO, which
restates the library's rule (include/fp4q.h, fp4q_kernel): the tensor core for b >= 16,
b >= g and M*K >= 2^22, except MXFP4 plans with channel signs at b = 128 from 3 * 2^26
elements on."""

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from microscaling_fp4_quantization_b200 import workloads as W  # noqa: E402


@pytest.mark.parametrize("w,signed,name", [
    (W.NV_4K, False, "tensor_core"),
    (W.NV_4K, True, "tensor_core"),
    (W.MX_8K_FLOOR, False, "tensor_core"),
    (W.MX_8K_FLOOR, True, "tensor_core"),                  # 2^26 elements: below 3 * 2^26
    (W.MX_8K_FLOOR.with_rows(24576), True, "butterfly"),   # exactly 3 * 2^26
    (W.PREFILL_MX, True, "butterfly"),
    (W.PREFILL_NV, True, "tensor_core"),                   # the exception is MXFP4's only
    (W.MX_8K_FLOOR.with_rows(511), False, "butterfly"),    # below 2^22 elements
    (W.MX_8K_FLOOR.with_rows(512), False, "tensor_core"),  # exactly 2^22
])
def test_auto_kernel_name(w, signed, name):
    assert bench.kernel_name(w, "auto", signed=signed) == name


def test_a_requested_kernel_is_reported_as_requested():
    for k in ("butterfly", "tensor_core"):
        assert bench.kernel_name(W.NV_4K, k) == k
        assert bench.kernel_name(W.PREFILL_MX, k, signed=True) == k


def test_decode_rows_take_the_butterfly():
    for w in W.DECODE:
        assert bench.kernel_name(w, "auto") == "butterfly"
