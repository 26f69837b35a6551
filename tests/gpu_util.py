"""Helpers for the GPU tests: run the CUDA path through the C ABI on numpy inputs, with
canary guard bands around every output buffer."""

from __future__ import annotations

import numpy as np
import torch

GUARD = 512            # bytes of canary before and after each output (keeps 256-byte alignment)
CANARY = 0xA5


class Guarded:
    """A device byte buffer with canary bands; .view is the usable middle part."""

    def __init__(self, nbytes: int, device="cuda"):
        self.nbytes = nbytes
        self.raw = torch.full((nbytes + 2 * GUARD,), CANARY, dtype=torch.uint8, device=device)
        self.view = self.raw[GUARD:GUARD + nbytes]

    def check(self, what: str) -> None:
        head = self.raw[:GUARD].cpu().numpy()
        tail = self.raw[GUARD + self.nbytes:].cpu().numpy()
        assert np.all(head == CANARY), f"{what}: write before the buffer"
        assert np.all(tail == CANARY), f"{what}: write past the buffer"

    def numpy(self) -> np.ndarray:
        return self.view.cpu().numpy()


def to_device_bf16(x_bits: np.ndarray, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).to(device)
    return t.view(torch.bfloat16)


def run_rotate_quantize(F, plan, x_bits: np.ndarray, tensor_scale=None, dump=False, x_dev=None, rows=None):
    """Returns dict(codes (M, K/2), scales (M, K/g), tensor_scale, y (when dump)); with
    `rows`, only those rows are copied back."""
    M, K = x_bits.shape if x_bits is not None else x_dev.shape
    xd = x_dev if x_dev is not None else to_device_bf16(x_bits)
    codes = Guarded(M * K // 2)
    scales = Guarded(M * K // plan.group)
    ts = torch.empty(1, dtype=torch.float32, device="cuda")
    if tensor_scale is not None:
        ts.fill_(float(tensor_scale))
    y = Guarded(M * K * 4) if dump else None
    tsp = ts if plan.fmt == F.FP4Q_NVFP4 else None
    if dump:
        F.fp4q_rotate_quantize_dump(plan, xd, M, K, codes.view, scales.view, tsp, y.view)
    else:
        F.fp4q_rotate_quantize(plan, xd, M, K, codes.view, scales.view, tsp)
    torch.cuda.synchronize()
    assert F.fp4q_device_status() == F.FP4Q_OK
    codes.check("codes")
    scales.check("scales")
    sel = (lambda t: t) if rows is None else (lambda t: t[torch.as_tensor(rows, device=t.device)])
    out = {
        "codes": sel(codes.view.view(M, K // 2)).cpu().numpy(),
        "scales": sel(scales.view.view(M, K // plan.group)).cpu().numpy(),
        "tensor_scale": np.float32(ts.item()),
    }
    if dump:
        y.check("y")
        out["y"] = sel(y.view.view(torch.float32).view(M, K)).cpu().numpy()
    return out


def run_amax(F, plan, x_bits: np.ndarray, x_dev=None) -> np.float32:
    M, K = x_bits.shape if x_bits is not None else x_dev.shape
    xd = x_dev if x_dev is not None else to_device_bf16(x_bits)
    ts = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    F.fp4q_amax(plan, xd, M, K, ts)
    torch.cuda.synchronize()
    assert F.fp4q_device_status() == F.FP4Q_OK
    return np.float32(ts.item())


def run_dequantize(F, plan, codes: np.ndarray, scales: np.ndarray, tensor_scale, unrotate: bool):
    M = codes.shape[0]
    K = codes.shape[1] * 2
    cd = torch.from_numpy(np.ascontiguousarray(codes)).cuda()
    sd = torch.from_numpy(np.ascontiguousarray(scales)).cuda()
    ts = torch.tensor([float(tensor_scale) if tensor_scale is not None else 1.0], dtype=torch.float32, device="cuda")
    out = Guarded(M * K * 4)
    F.fp4q_dequantize(plan, cd, sd, ts, M, K, unrotate, out.view)
    torch.cuda.synchronize()
    out.check("dequantize out")
    return out.numpy().view(np.float32).reshape(M, K)


def run_rotate_quantize_mbs(F, plan, x_bits: np.ndarray):
    """MBS-Static rotate + quantize: dict(codes (M, K/2), scales (M, K/32), macro (M, K/128))."""
    M, K = x_bits.shape
    xd = to_device_bf16(x_bits)
    codes = Guarded(M * K // 2)
    scales = Guarded(M * K // 32)
    macro = Guarded(M * K // 128)
    F.fp4q_rotate_quantize_mbs(plan, xd, M, K, codes.view, scales.view, macro.view)
    torch.cuda.synchronize()
    assert F.fp4q_device_status() == F.FP4Q_OK
    for g, n in ((codes, "codes"), (scales, "scales"), (macro, "macro")):
        g.check(n)
    return {"codes": codes.numpy().reshape(M, K // 2), "scales": scales.numpy().reshape(M, K // 32),
            "macro": macro.numpy().reshape(M, K // 128)}


def run_dequantize_mbs(F, plan, codes: np.ndarray, scales: np.ndarray, macro: np.ndarray, unrotate: bool):
    M = codes.shape[0]
    K = codes.shape[1] * 2
    cd = torch.from_numpy(np.ascontiguousarray(codes)).cuda()
    sd = torch.from_numpy(np.ascontiguousarray(scales)).cuda()
    md = torch.from_numpy(np.ascontiguousarray(macro)).cuda()
    out = Guarded(M * K * 4)
    F.fp4q_dequantize_mbs(plan, cd, sd, md, M, K, unrotate, out.view)
    torch.cuda.synchronize()
    out.check("dequantize_mbs out")
    return out.numpy().view(np.float32).reshape(M, K)
