"""Python binding of the fp4q C ABI (include/fp4q.h), through ctypes.

The functions carry the C names and do argument marshalling only: every step of the
rotate + quantize path runs in the library's CUDA kernels.  PyTorch tensors are used as
device allocations and streams.  Importing this module loads lib/libfp4q.so and raises
ImportError when it is missing; there is no fallback.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libfp4q.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"fp4q native library not built: {LIB_PATH} (run python -m "
                      "microscaling_fp4_quantization_b200.build)")

_lib = ctypes.CDLL(LIB_PATH)

FP4Q_OK, FP4Q_ERR_ARG, FP4Q_ERR_SHAPE, FP4Q_ERR_ALIGN, FP4Q_ERR_UNSUPPORTED, FP4Q_ERR_CUDA, FP4Q_ERR_TIMEOUT = range(7)
FP4Q_MXFP4, FP4Q_NVFP4, FP4Q_MXFP4_MBS = 0, 1, 2
FP4Q_KERNEL_AUTO, FP4Q_KERNEL_BUTTERFLY, FP4Q_KERNEL_TENSOR_CORE = 0, 1, 2
(FP4Q_SCALE_FLOOR_OCP, FP4Q_SCALE_CEIL_NOCLIP, FP4Q_SCALE_OAS,
 FP4Q_SCALE_NV_STATIC, FP4Q_SCALE_NV_DYNAMIC) = range(5)

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_int = ctypes.c_int

_SIGS = {
    "fp4q_plan_create": (_int, [ctypes.POINTER(_vp), _int, _int, _int, _int]),
    "fp4q_plan_destroy": (_int, [_vp]),
    "fp4q_plan_set_kernel": (_int, [_vp, _int]),
    "fp4q_plan_set_signs": (_int, [_vp, _vp, _i64]),
    "fp4q_rotate_quantize": (_int, [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp]),
    "fp4q_rotate_quantize_dump": (_int, [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _vp]),
    "fp4q_amax": (_int, [_vp, _vp, _i64, _i64, _vp, _vp]),
    "fp4q_dequantize": (_int, [_vp, _vp, _vp, _vp, _i64, _i64, _int, _vp, _vp]),
    "fp4q_rotate_quantize_nvfp4_dynamic_noalloc": (_int, [_vp, _i64, _i64, _int, _vp, _vp, _vp, _vp]),
    "fp4q_quant_error": (_int, [_vp, _vp, _i64, _i64, _vp, _vp, _vp]),
    "fp4q_rotate_quantize_mbs": (_int, [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp]),
    "fp4q_dequantize_mbs": (_int, [_vp, _vp, _vp, _vp, _i64, _i64, _int, _vp, _vp]),
    "fp4q_gemm": (_int, [_int, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp]),
    "fp4q_device_status": (_int, []),
    "fp4q_selftest_wait_timeout": (_int, [_vp]),
    "fp4q_status_string": (ctypes.c_char_p, [_int]),
    "fp4q_last_cuda_error": (ctypes.c_char_p, []),
    "fp4q_version": (_int, []),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args

EXPORTED = tuple(_SIGS)


class Fp4qError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = _lib.fp4q_status_string(status).decode()
        if status == FP4Q_ERR_CUDA:
            msg += ": " + _lib.fp4q_last_cuda_error().decode()
        super().__init__(f"{where}: {msg} (status {status})")
        self.status = status


def _check(status: int, where: str) -> None:
    if status != FP4Q_OK:
        raise Fp4qError(status, where)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


class Plan:
    """An fp4q plan handle (format, group, Hadamard block, scale rule)."""

    def __init__(self, handle: int, fmt: int, group: int, block: int, rule: int):
        self.handle = handle
        self.fmt, self.group, self.block, self.rule = fmt, group, block, rule
        self.kernel = FP4Q_KERNEL_AUTO

    def __del__(self):
        h, self.handle = getattr(self, "handle", None), None
        if h:
            try:
                _lib.fp4q_plan_destroy(h)
            except Exception:
                pass

    @property
    def unit(self) -> int:
        return max(self.group, self.block)


# ---------------------------------------------------------------- the C names

def fp4q_plan_create(fmt: int, group: int, hadamard_block: int, scale_rule: int) -> Plan:
    h = _vp()
    _check(_lib.fp4q_plan_create(ctypes.byref(h), fmt, group, hadamard_block, scale_rule), "fp4q_plan_create")
    return Plan(h.value, fmt, group, hadamard_block, scale_rule)


def fp4q_plan_set_kernel(plan: Plan, kernel: int) -> None:
    _check(_lib.fp4q_plan_set_kernel(plan.handle, kernel), "fp4q_plan_set_kernel")
    plan.kernel = kernel


def fp4q_plan_set_signs(plan: Plan, signs, K: int) -> None:
    """signs: device uint32 tensor [ceil(K/32)] (bit k negates channel k) or None to clear.
    The plan keeps a reference to the tensor so that it stays alive."""
    _check(_lib.fp4q_plan_set_signs(plan.handle, _ptr(signs), K), "fp4q_plan_set_signs")
    plan.signs = signs


def fp4q_plan_destroy(plan: Plan) -> None:
    h, plan.handle = plan.handle, None
    _check(_lib.fp4q_plan_destroy(h), "fp4q_plan_destroy")


def fp4q_rotate_quantize(plan: Plan, x, M: int, K: int, codes_out, scales_out, tensor_scale=None,
                         stream=None) -> None:
    _check(_lib.fp4q_rotate_quantize(plan.handle, _ptr(x), M, K, _ptr(codes_out), _ptr(scales_out),
                                     _ptr(tensor_scale), _stream(stream)), "fp4q_rotate_quantize")


def fp4q_rotate_quantize_dump(plan: Plan, x, M: int, K: int, codes_out, scales_out, tensor_scale, y_out,
                              stream=None) -> None:
    _check(_lib.fp4q_rotate_quantize_dump(plan.handle, _ptr(x), M, K, _ptr(codes_out), _ptr(scales_out),
                                          _ptr(tensor_scale), _ptr(y_out), _stream(stream)),
           "fp4q_rotate_quantize_dump")


def fp4q_amax(plan: Plan, x, M: int, K: int, tensor_scale_out, stream=None) -> None:
    _check(_lib.fp4q_amax(plan.handle, _ptr(x), M, K, _ptr(tensor_scale_out), _stream(stream)), "fp4q_amax")


def fp4q_dequantize(plan: Plan, codes, scales, tensor_scale, M: int, K: int, unrotate: bool, out_f32,
                    stream=None) -> None:
    _check(_lib.fp4q_dequantize(plan.handle, _ptr(codes), _ptr(scales), _ptr(tensor_scale), M, K,
                                int(bool(unrotate)), _ptr(out_f32), _stream(stream)), "fp4q_dequantize")


def fp4q_rotate_quantize_nvfp4_dynamic_noalloc(x, M: int, K: int, hadamard_block: int, codes_out, scales_out,
                                                tensor_scale_out, stream=None) -> None:
    """NVFP4 dynamic-scale rotate + quantize without any device allocation (its scratch is a
    fixed array inside the library); for callers that cannot allocate device memory."""
    _check(_lib.fp4q_rotate_quantize_nvfp4_dynamic_noalloc(_ptr(x), M, K, hadamard_block, _ptr(codes_out),
                                                           _ptr(scales_out), _ptr(tensor_scale_out),
                                                           _stream(stream)),
           "fp4q_rotate_quantize_nvfp4_dynamic_noalloc")


def fp4q_quant_error(plan: Plan, x, M: int, K: int, tensor_scale, out_f64, stream=None) -> None:
    """out_f64: device float64 [3] <- {signal energy, error energy, QSNR dB}."""
    _check(_lib.fp4q_quant_error(plan.handle, _ptr(x), M, K, _ptr(tensor_scale), _ptr(out_f64), _stream(stream)),
           "fp4q_quant_error")


def fp4q_rotate_quantize_mbs(plan: Plan, x, M: int, K: int, codes_out, scales_out, macro_out, stream=None) -> None:
    _check(_lib.fp4q_rotate_quantize_mbs(plan.handle, _ptr(x), M, K, _ptr(codes_out), _ptr(scales_out),
                                         _ptr(macro_out), _stream(stream)), "fp4q_rotate_quantize_mbs")


def fp4q_dequantize_mbs(plan: Plan, codes, scales, macro, M: int, K: int, unrotate: bool, out_f32,
                        stream=None) -> None:
    _check(_lib.fp4q_dequantize_mbs(plan.handle, _ptr(codes), _ptr(scales), _ptr(macro), M, K, int(bool(unrotate)),
                                    _ptr(out_f32), _stream(stream)), "fp4q_dequantize_mbs")


def fp4q_gemm(fmt: int, a_codes, a_scales, a_tensor_scale, b_codes, b_scales, b_tensor_scale, M: int, N: int,
              K: int, d_bf16, stream=None) -> None:
    """D [M, N] bf16 = alpha * A B^T from the quantizer's codes and scales of A [M, K] and B [N, K]."""
    _check(_lib.fp4q_gemm(fmt, _ptr(a_codes), _ptr(a_scales), _ptr(a_tensor_scale), _ptr(b_codes), _ptr(b_scales),
                          _ptr(b_tensor_scale), M, N, K, _ptr(d_bf16), _stream(stream)), "fp4q_gemm")


def fp4q_device_status() -> int:
    return _lib.fp4q_device_status()


def fp4q_selftest_wait_timeout(stream=None) -> None:
    """One warp whose bounded wait runs out: the next fp4q_device_status is FP4Q_ERR_TIMEOUT."""
    _check(_lib.fp4q_selftest_wait_timeout(_stream(stream)), "fp4q_selftest_wait_timeout")


def fp4q_status_string(status: int) -> str:
    return _lib.fp4q_status_string(status).decode()


def fp4q_version() -> int:
    return _lib.fp4q_version()


def raw_call(name: str, *args) -> int:
    """Call a C entry point with raw arguments and return its status (for tests of the
    host-side argument checks)."""
    return getattr(_lib, name)(*args)


# ---------------------------------------------------------------- tensor conveniences

def empty_outputs(plan: Plan, M: int, K: int, device="cuda"):
    """Allocate codes (uint8 [M, K/2]), scales (uint8 [M, K/g]) and the fp32 tensor scale."""
    import torch
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device=device)
    scales = torch.empty((M, K // plan.group), dtype=torch.uint8, device=device)
    ts = torch.empty((1,), dtype=torch.float32, device=device)
    return codes, scales, ts


def rotate_quantize(plan: Plan, x, tensor_scale=None, stream=None) -> Tuple[object, object, object]:
    """x: bf16 CUDA tensor [M, K] -> (codes, scales, tensor_scale)."""
    import torch
    if x.dtype != torch.bfloat16 or not x.is_cuda or x.dim() != 2 or not x.is_contiguous():
        raise ValueError("x must be a contiguous 2-D bf16 CUDA tensor")
    M, K = x.shape
    codes, scales, ts = empty_outputs(plan, M, K, x.device)
    if tensor_scale is not None:
        ts = tensor_scale
    fp4q_rotate_quantize(plan, x, M, K, codes, scales, ts if plan.fmt == FP4Q_NVFP4 else None, stream)
    return codes, scales, ts


def quant_error(plan: Plan, x, tensor_scale=None, stream=None):
    """x: bf16 CUDA tensor [M, K] -> (signal, error, qsnr_db) as Python floats (synchronises)."""
    import torch
    if x.dtype != torch.bfloat16 or not x.is_cuda or x.dim() != 2 or not x.is_contiguous():
        raise ValueError("x must be a contiguous 2-D bf16 CUDA tensor")
    M, K = x.shape
    out = torch.empty(3, dtype=torch.float64, device=x.device)
    ts = tensor_scale
    if plan.fmt == FP4Q_NVFP4 and ts is None:
        ts = torch.empty(1, dtype=torch.float32, device=x.device)
    fp4q_quant_error(plan, x, M, K, ts, out, stream)
    s, e, q = out.tolist()
    return s, e, q
