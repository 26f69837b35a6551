"""CPU oracle for block-Hadamard rotation + microscaling FP4 quantization.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this module.  The library (``include/fp4q.h``,
``microscaling_fp4_quantization_b200``) never calls it, and it shares no code with the
CUDA path: it is a plain, slow restatement of what the path computes, in fp64 where the
arithmetic is real-valued and in fp32 where an fp32 value decides an integer code.

Sources (page title and section):
  [BG]  "Bridging the Gap Between Promise and Performance for Microscaling FP4
        Quantization" (gist.science/de/paper/2509.23202): Technische Zusammenfassung,
        1. Problemstellung (MXFP4 = 32-element blocks, NVFP4 = 16-element blocks, one
        shared scale per block); 2. Methodik (block-wise Hadamard transforms of weights
        and activations, "wie in QuIP/QuaRot"); GPU-Kernel-Unterstützung (QuTLASS: the
        activation rotation fused into the online quantization kernel).
  [BG-en] the same paper's English abstract (chatpaper.ai, page "Preenchendo a Lacuna ...",
        section "English"): block-wise Hadamard transforms, rotation fused into the
        weights, fast online computation for the activations.
  [BG-es] the same paper (gist.science/es/paper/2509.23202): Resumen técnico, 2.A
        (E8M0 dead-zone; NVFP4 uses E4M3 shared scales), 2.B.2 (NVFP4 optimises group
        and tensor scales).
  [UP]  "Unveiling the Potential of Quantization with MXFP4: Strategies for
        Quantization Error Reduction" (gist.science/nl/paper/2603.08713): Technische
        samenvatting, Probleemstelling (MXFP4 blocks of 32 with an E8M0 scale = 8
        exponent bits, 0 mantissa bits, i.e. powers of two; NVFP4 blocks of 16 with an
        E4M3 scale) and Methodologie 1 (Overflow-Aware Scaling: the standard rule maps
        the block maximum into (3, 6]; maxima in [3, 3.5] are pushed to [6, 7]).
  [TQ]  "TORQ: Two-Level Orthogonal Rotation for MXFP4 Quantization"
        (gist.science/de/paper/2605.19561): Technische Zusammenfassung, 1.
        Problemstellung (the geometrically progressive e2m1 codebook).

Readings where the pages are silent:
  * Hadamard: Sylvester construction, natural order, orthonormal 1/sqrt(b), applied to
    every contiguous b-block of a row (the GEMM reduction axis).  By default no random
    signs; an optional per-channel sign vector s (QuaRot-style randomised Hadamard, "wie in
    QuIP/QuaRot", [BG] 2. Methodik) is applied to the channels before the block rotation,
    the same s on the activations online and in the weights offline.
  * E2M1: magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}; round to nearest, ties to the even
    code; saturate at 6; the sign bit is the sign of the rotated value.
  * MX scale X = 2^e, stored as the E8M0 byte e + 127, e clamped to [-127, 127]:
      floor (OCP)      e = floor(log2 A) - 2          (2 = exponent of the top E2M1 value)
      ceil (no clip)   e = ceil(log2(A / 6))          (maps A into (3, 6], nothing clips)
      OAS              ceil rule, then e -= 1 when A / 2^e lies in [3, 3.5]
    A = 0 gives e = -127 (byte 0) and all-zero codes.
  * NV scale: per-tensor fp32 s_g (from the rotated tensor's amax: s_g = A_t / (6*448),
    1 when A_t = 0); block scale s_b = E4M3_RNE_satfinite(A / fp32(6 * s_g)); element
    divisor S = fp32(E4M3(s_b) * s_g); a zero block scale gives all-zero codes.
  * Packing: element 2j in the low nibble of byte j, 2j+1 in the high nibble; codes and
    scales row-major.
  * Precision: the rotation is exact up to one rounding (fp64 product of bf16 values with
    +-1), then rounded once to fp32; every decision (amax, scale byte, element code)
    is taken on fp32 values, as the kernel takes it; the fp32 divisions are IEEE.
"""

from __future__ import annotations

import math

import numpy as np

MXFP4 = 0
NVFP4 = 1
MXFP4_MBS = 2          # MXFP4 under an MBS-Static macro-block scale ([UP] Methodologie 2)
MBS_MACRO = 128        # elements per macro block

SCALE_FLOOR_OCP = 0
SCALE_CEIL_NOCLIP = 1
SCALE_OAS = 2
SCALE_NV_STATIC = 3
SCALE_NV_DYNAMIC = 4

# E2M1 (TQ 1.): code k in 0..7 has magnitude E2M1_MAGNITUDES[k]; bit 3 is the sign.
E2M1_MAGNITUDES = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)
E2M1_MAX = 6.0
# E4M3 finite range (UP, Probleemstelling: 4 exponent bits, 3 mantissa bits).
E4M3_MAX = 448.0
NV_TENSOR_DIVISOR = 6.0 * 448.0  # 2688: E2M1 max times E4M3 max

_CHUNK = 1 << 16


# ----------------------------------------------------------------------------------
# Rotation ([BG] 2. Methodik; [BG-en]: block-wise Hadamard transforms)
# ----------------------------------------------------------------------------------

def sylvester_hadamard(b: int) -> np.ndarray:
    """H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]] (integer matrix, natural order)."""
    if b < 1 or (b & (b - 1)) != 0:
        raise ValueError(f"Hadamard block must be a power of two, got {b}")
    H = np.ones((1, 1), dtype=np.int64)
    while H.shape[0] < b:
        H = np.block([[H, H], [H, -H]])
    return H


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float64 (exact)."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def sign_vector(mask_words: np.ndarray, K: int) -> np.ndarray:
    """Per-channel signs from a bit mask: channel k is negated when bit (k mod 32) of word
    k // 32 is set.  Returns float64 +-1 of length K."""
    w = np.asarray(mask_words, np.uint32)
    if w.size * 32 < K:
        raise ValueError("the sign mask holds fewer than K bits")
    k = np.arange(K)
    bit = (w[k // 32] >> (k % 32).astype(np.uint32)) & np.uint32(1)
    return np.where(bit == 1, -1.0, 1.0)


def rotate(x_bits: np.ndarray, b: int, signs=None) -> np.ndarray:
    """y[r, kb*b + j] = (1/sqrt(b)) * sum_l s[kb*b + l] x[r, kb*b + l] H_b[l, j], in float64.

    An explicit matrix product with the Sylvester matrix (not a fast transform).  ``signs``
    (length K, +-1, or None for all +1) is the random diagonal of a QuaRot-style
    randomised Hadamard transform, applied to the channels before the block rotation, so
    that the rotation is Q = diag(s) (I kron H_b / sqrt(b))."""
    x = bf16_to_f64(x_bits)
    M, K = x.shape
    if K % b:
        raise ValueError("K must be a multiple of the Hadamard block")
    if signs is not None:
        x = x * np.asarray(signs, np.float64)[None, :]
    H = sylvester_hadamard(b).astype(np.float64)
    y = (x.reshape(M * (K // b), b) @ H) / math.sqrt(b)
    return y.reshape(M, K)


def unrotate(y: np.ndarray, b: int, signs=None) -> np.ndarray:
    """Inverse rotation.  H_b / sqrt(b) is symmetric and orthogonal, so it is its own
    inverse: the same product again, then the signs again (Q^-1 = Q^T)."""
    M, K = y.shape
    H = sylvester_hadamard(b).astype(np.float64)
    x = ((np.asarray(y, np.float64).reshape(M * (K // b), b) @ H) / math.sqrt(b)).reshape(M, K)
    if signs is not None:
        x = x * np.asarray(signs, np.float64)[None, :]
    return x


# ----------------------------------------------------------------------------------
# Element code: E2M1 by brute-force nearest search (TQ 1.; ties to even)
# ----------------------------------------------------------------------------------

def e2m1_encode(v: np.ndarray) -> np.ndarray:
    """fp32 values (already divided by the block scale) -> 4-bit codes (uint8).

    Nearest of the 8 magnitudes; on an exact tie the even code wins; |v| > 6 lands on 6
    (the nearest magnitude) which is saturation; bit 3 is the sign bit of v (so -0.0 and
    negative values that round to zero keep it)."""
    v = np.asarray(v, dtype=np.float32)
    flat = v.reshape(-1)
    out = np.empty(flat.shape, np.uint8)
    G = np.array(E2M1_MAGNITUDES, dtype=np.float64)
    even = (np.arange(8) % 2) == 0
    for s in range(0, flat.size, _CHUNK):
        # saturation first: above 6 the nearest magnitude is 6 (and fp64 distances from
        # huge values would all round to the same number)
        a = np.minimum(np.abs(flat[s:s + _CHUNK].astype(np.float64)), E2M1_MAX)
        d = np.abs(a[:, None] - G[None, :])
        cand = d == d.min(axis=1, keepdims=True)
        cand_even = cand & even[None, :]
        k = np.where(cand_even.any(axis=1), cand_even.argmax(axis=1), cand.argmax(axis=1))
        sign = np.signbit(flat[s:s + _CHUNK])
        out[s:s + _CHUNK] = (k | (sign.astype(np.int64) << 3)).astype(np.uint8)
    return out.reshape(v.shape)


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    """4-bit codes -> float64 values."""
    c = np.asarray(codes, dtype=np.uint8)
    mag = np.array(E2M1_MAGNITUDES, dtype=np.float64)[c & 7]
    return np.where((c & 8) != 0, -mag, mag)


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """(..., K) 4-bit codes -> (..., K/2) bytes: element 2j low nibble, 2j+1 high."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


# ----------------------------------------------------------------------------------
# MX block scale: E8M0 power of two ([UP] Probleemstelling and Methodologie 1)
# ----------------------------------------------------------------------------------

def floor_log2(A: np.ndarray) -> np.ndarray:
    """floor(log2 A) for A > 0, exactly (frexp: A = f * 2^p with f in [0.5, 1))."""
    _, p = np.frexp(np.asarray(A, np.float64))
    return p.astype(np.int64) - 1


def mx_scale_exponent(A32: np.ndarray, rule: int) -> np.ndarray:
    """Group amax (fp32) -> E8M0 exponent e (int64), clamped to [-127, 127]."""
    A = np.asarray(A32, np.float32).astype(np.float64)
    e = np.full(A.shape, -127, np.int64)
    pos = A > 0
    Ap = A[pos]
    if rule == SCALE_FLOOR_OCP:
        ep = floor_log2(Ap) - 2
    elif rule in (SCALE_CEIL_NOCLIP, SCALE_OAS):
        # ceil(log2(A/6)) = the smallest integer e with A <= 6 * 2^e.  Starting three
        # below floor(log2 A) is below that integer; step up until the bound holds.
        ep = floor_log2(Ap) - 3
        for _ in range(6):
            ep = ep + (Ap > np.ldexp(6.0, ep)).astype(np.int64)
        if rule == SCALE_OAS:
            alpha = Ap / np.ldexp(1.0, ep)       # normalised block maximum, in (3, 6]
            ep = ep - ((alpha >= 3.0) & (alpha <= 3.5)).astype(np.int64)
    else:
        raise ValueError(f"not an MX scale rule: {rule}")
    e[pos] = ep
    return np.clip(e, -127, 127)


# ----------------------------------------------------------------------------------
# NV block scale: E4M3 under an fp32 tensor scale ([BG] 1.; [BG-es] 2.A, 2.B.2)
# ----------------------------------------------------------------------------------

def e4m3_table() -> np.ndarray:
    """Values of the 127 non-negative finite E4M3 codes 0x00..0x7E (0x7F is NaN)."""
    c = np.arange(127)
    ex, m = c >> 3, c & 7
    return np.where(ex == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.ldexp(1.0, ex - 7))


def e4m3_encode(s: np.ndarray) -> np.ndarray:
    """Non-negative fp32 -> E4M3 code by brute-force nearest search over all finite
    codes, ties to the even code; values past 448 land on 448 (satfinite)."""
    s = np.asarray(s, dtype=np.float32)
    flat = s.reshape(-1).astype(np.float64)
    if np.any(flat < 0):
        raise ValueError("block scales are non-negative")
    T = e4m3_table()
    even = (np.arange(127) % 2) == 0
    out = np.empty(flat.shape, np.uint8)
    for i in range(0, flat.size, _CHUNK // 4):
        a = np.minimum(flat[i:i + _CHUNK // 4], E4M3_MAX)   # satfinite
        d = np.abs(a[:, None] - T[None, :])
        cand = d == d.min(axis=1, keepdims=True)
        cand_even = cand & even[None, :]
        out[i:i + _CHUNK // 4] = np.where(cand_even.any(axis=1), cand_even.argmax(axis=1),
                                          cand.argmax(axis=1)).astype(np.uint8)
    return out.reshape(s.shape)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    return e4m3_table()[np.asarray(codes, np.int64)]


def nv_tensor_scale(A_tensor: float) -> np.float32:
    """s_g = fp32(A_t / 2688), with s_g = 1 for an all-zero tensor."""
    A = np.float32(A_tensor)
    if A == 0:
        return np.float32(1.0)
    return np.float32(A / np.float32(NV_TENSOR_DIVISOR))


# ----------------------------------------------------------------------------------
# The whole path
# ----------------------------------------------------------------------------------

def check_plan(fmt: int, group: int, block: int, rule: int) -> None:
    if fmt in (MXFP4, MXFP4_MBS):
        if group != 32 or rule not in (SCALE_FLOOR_OCP, SCALE_CEIL_NOCLIP, SCALE_OAS):
            raise ValueError("MXFP4 uses groups of 32 and an MX scale rule")
    elif fmt == NVFP4:
        if group != 16 or rule not in (SCALE_NV_STATIC, SCALE_NV_DYNAMIC):
            raise ValueError("NVFP4 uses groups of 16 and an NV scale rule")
    else:
        raise ValueError("format")
    sylvester_hadamard(block)


def rotated_amax(x_bits: np.ndarray, block: int, chunk_rows: int = 512, signs=None) -> np.float32:
    """max |y| over the whole tensor, taken on the fp32 rotated values (row chunks keep the
    fp64 intermediate small)."""
    m = np.float32(0)
    for r in range(0, x_bits.shape[0], chunk_rows):
        y32 = rotate(x_bits[r:r + chunk_rows], block, signs).astype(np.float32)
        if y32.size:
            m = max(m, np.float32(np.max(np.abs(y32))))
    return np.float32(m)


def rotate_quantize(x_bits: np.ndarray, fmt: int, group: int, block: int, rule: int,
                    tensor_scale=None, signs=None) -> dict:
    """Rotate then quantize X (M x K bf16 bit patterns).

    For NVFP4 ``tensor_scale`` is the fp32 s_g (the static rule needs it; the dynamic
    rule computes it here from the rotated amax when it is None).

    Returns codes (M, K/2) uint8, scales (M, K/group) uint8, the fp64 and fp32 rotated
    values, the fp32 group amax, the exact per-group divisor and s_g."""
    check_plan(fmt, group, block, rule)
    x_bits = np.asarray(x_bits, np.uint16)
    M, K = x_bits.shape
    if K % group or K % block:
        raise ValueError("K must be a multiple of the group and of the block")
    y64 = rotate(x_bits, block, signs)
    y32 = y64.astype(np.float32)                     # one rounding to fp32
    yg = y32.reshape(M, K // group, group)
    A32 = np.max(np.abs(yg), axis=2) if K else np.zeros((M, 0), np.float32)

    if fmt == MXFP4:
        e = mx_scale_exponent(A32, rule)
        scales = (e + 127).astype(np.uint8)
        S64 = np.ldexp(1.0, e)                       # 2^e, exact
        v = (yg.astype(np.float64) / S64[..., None]).astype(np.float32)   # exact: power of two
        q = e2m1_encode(v)
        s_g = None
    else:
        if tensor_scale is None:
            if rule != SCALE_NV_DYNAMIC:
                raise ValueError("the static NV rule needs the tensor scale")
            s_g = nv_tensor_scale(np.max(A32) if A32.size else 0.0)
        else:
            s_g = np.float32(tensor_scale)
        den = np.float32(np.float32(6.0) * s_g)
        s_b = (A32 / den).astype(np.float32)         # fp32 IEEE division
        scales = e4m3_encode(s_b)
        S32 = (e4m3_decode(scales).astype(np.float32) * s_g).astype(np.float32)   # fp32 product
        S64 = e4m3_decode(scales) * np.float64(s_g)
        zero = S32 == 0
        S_safe = np.where(zero, np.float32(1.0), S32)
        v = (yg / S_safe[..., None]).astype(np.float32)   # fp32 IEEE division
        q = e2m1_encode(v)
        q[np.broadcast_to(zero[..., None], q.shape)] = 0
    codes = pack_nibbles(q.reshape(M, K))
    return {
        "codes": codes,
        "scales": scales.reshape(M, K // group),
        "y64": y64,
        "y32": y32,
        "amax32": A32,
        "S64": S64,
        "tensor_scale": s_g,
        "fmt": fmt, "group": group, "block": block, "rule": rule,
    }


# ----------------------------------------------------------------------------------
# MBS-Static ([UP] Technische samenvatting, Methodologie 2, "Macro Block Scaling"): every
# macro block of 128 elements gets one extra scale factor with 8 mantissa bits, computed
# directly from the macro block's maximum; the values are divided by it before the
# standard MXFP4 quantization of their 32-element groups.
# ----------------------------------------------------------------------------------

def mbs_macro_byte(A_M32: np.ndarray) -> np.ndarray:
    """Macro-scale byte m8 from the fp32 macro-block maximum A_M.

    With fp32(A_M / 6) = 2^E (1 + f), f in [0, 1): m8 = ceil(256 f) mod 256 and the macro
    scale is s_M = 1 + m8 / 256.  s_M is the mantissa of A_M / 6 rounded up to 8 bits, so
    A_M / s_M <= 6 * 2^E: the block maximum lands on (or just under) the top E2M1 value
    under its power-of-two group scale and never above it.  ceil(256 f) = 256 means
    s_M = 2, which is s_M = 1 with every group exponent one higher: byte 0.  A_M = 0 gives
    byte 0."""
    r = (np.asarray(A_M32, np.float32) / np.float32(6.0)).astype(np.float32)   # fp32 IEEE division
    m, _ = np.frexp(r.astype(np.float64))                                       # r = m 2^E', m in [0.5, 1)
    f = np.where(r > 0, 2.0 * m - 1.0, 0.0)                                     # exact
    return (np.ceil(f * 256.0).astype(np.int64) % 256).astype(np.uint8)


def mbs_macro_scale(m8: np.ndarray) -> np.ndarray:
    """s_M = 1 + m8 / 256 (exact in fp32)."""
    return (1.0 + np.asarray(m8, np.float64) / 256.0).astype(np.float32)


def rotate_quantize_mbs(x_bits: np.ndarray, group: int, block: int, rule: int, signs=None) -> dict:
    """Rotate, then MXFP4 (groups of 32, E8M0 by ``rule``) under MBS-Static macro scales.

    y' = fp32(y32 / s_M) (IEEE division) for the 128 elements of each macro block; the
    group amax, the E8M0 exponent e and the E2M1 codes are taken on y' exactly as for
    MXFP4.  The dequantized value is q * 2^e * s_M.  Returns the keys of
    ``rotate_quantize`` plus ``macro`` (M, K/128) uint8 and ``yp32``."""
    check_plan(MXFP4_MBS, group, block, rule)
    x_bits = np.asarray(x_bits, np.uint16)
    M, K = x_bits.shape
    if K % MBS_MACRO or K % block:
        raise ValueError("K must be a multiple of the macro block (128) and of the Hadamard block")
    y64 = rotate(x_bits, block, signs)
    y32 = y64.astype(np.float32)
    ym = y32.reshape(M, K // MBS_MACRO, MBS_MACRO)
    AM = np.max(np.abs(ym), axis=2) if K else np.zeros((M, 0), np.float32)
    m8 = mbs_macro_byte(AM)
    sM = mbs_macro_scale(m8)
    yp = (ym / sM[..., None]).astype(np.float32).reshape(M, K)      # fp32 IEEE division
    yg = yp.reshape(M, K // group, group)
    A32 = np.max(np.abs(yg), axis=2) if K else np.zeros((M, 0), np.float32)
    e = mx_scale_exponent(A32, rule)
    v = (yg.astype(np.float64) / np.ldexp(1.0, e)[..., None]).astype(np.float32)   # exact: power of two
    q = e2m1_encode(v)
    sM_g = np.repeat(sM.astype(np.float64), MBS_MACRO // group, axis=1)
    return {
        "codes": pack_nibbles(q.reshape(M, K)),
        "scales": (e + 127).astype(np.uint8).reshape(M, K // group),
        "macro": m8.reshape(M, K // MBS_MACRO),
        "y64": y64, "y32": y32, "yp32": yp,
        "amax32": A32,
        "S64": np.ldexp(1.0, e) * sM_g,
        "tensor_scale": None,
        "fmt": MXFP4_MBS, "group": group, "block": block, "rule": rule,
    }


def dequantize_mbs(codes: np.ndarray, scales: np.ndarray, macro: np.ndarray, group: int, block: int,
                   unrotate_back: bool = False, signs=None) -> np.ndarray:
    """q * 2^(byte - 127) * s_M (exact in fp32: 2 + 9 significant bits), optionally rotated back."""
    q = e2m1_decode(unpack_nibbles(codes))
    M, K = q.shape
    S = np.ldexp(1.0, np.asarray(scales, np.int64).reshape(M, K // group) - 127)
    sM = np.repeat(mbs_macro_scale(np.asarray(macro, np.uint8).reshape(M, K // MBS_MACRO)).astype(np.float64),
                   MBS_MACRO // group, axis=1)
    x = (q.reshape(M, K // group, group) * (S * sM)[..., None]).astype(np.float32).reshape(M, K)
    if unrotate_back:
        return unrotate(x.astype(np.float64), block, signs)
    return x


def dequantize(codes: np.ndarray, scales: np.ndarray, fmt: int, group: int, block: int,
               tensor_scale=None, unrotate_back: bool = False, signs=None) -> np.ndarray:
    """codes x block scale (x tensor scale), optionally rotated back.

    MX: x = q * 2^(byte - 127), exact.  NV: x = fp32(q * fp32(E4M3(byte) * s_g)).
    Returns fp32 values when not rotating back, else the fp64 inverse rotation of them."""
    q = e2m1_decode(unpack_nibbles(codes))
    M, K = q.shape
    sc = np.asarray(scales, np.uint8).reshape(M, K // group)
    if fmt == MXFP4:
        S = np.ldexp(1.0, sc.astype(np.int64) - 127)
        x = (q.reshape(M, K // group, group) * S[..., None]).astype(np.float32)
    else:
        s_g = np.float32(tensor_scale)
        S32 = (e4m3_decode(sc).astype(np.float32) * s_g).astype(np.float32)
        x = (q.reshape(M, K // group, group).astype(np.float32) * S32[..., None]).astype(np.float32)
    x = x.reshape(M, K)
    if unrotate_back:
        return unrotate(x.astype(np.float64), block, signs)
    return x


# ----------------------------------------------------------------------------------
# Near-boundary flags for the parity rule
# ----------------------------------------------------------------------------------

E2M1_MIDPOINTS = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)


def _dist_scaled_power(A: np.ndarray, base: float) -> np.ndarray:
    """Relative distance |A - base*2^k| / (base*2^k) to the nearest point base*2^k (A > 0);
    +inf where A = 0 (no boundary near zero)."""
    A = np.asarray(A, np.float64)
    out = np.full(A.shape, np.inf)
    pos = A > 0
    k = np.round(np.log2(A[pos] / base))
    ref = base * np.exp2(k)
    out[pos] = np.abs(A[pos] - ref) / ref
    return out


def boundary_distance(res: dict):
    """How far each decision of the oracle's result lies from a place where it flips.

    Element: the relative distance of the exact |y| / S to the nearest E2M1 rounding midpoint
    (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5: the codes change only there; above 6 everything
    saturates to 6, so 6 is no boundary).  Group: the relative distance of its exact amax to
    the nearest boundary of the scale rule, where the scale byte steps:
      floor (OCP)  2^k            (floor(log2 A) steps)
      ceil         1.5 * 2^k      (ceil(log2(A / 6)) steps at 6 * 2^j = 1.5 * 2^(j+2))
      OAS          1.5 * 2^k and 1.75 * 2^k (the ceil rule's boundary, and the top of the
                   [3, 3.5] window it pushes down)
      NV           the nearest midpoint between two E4M3 values of s_b = A / (6 s_g)
    and, for MBS, also the distance of the macro block's exact 256 f to an integer (where
    the ceil of m8 steps), divided by 256, for every group of the block.  The group rule of
    MBS sees A / s_M.  Distances are +inf where there is no boundary (a zero amax).

    Returns (element distances (M, K), group distances (M, K/group)), float64."""
    y64 = res["y64"]
    M, K = y64.shape
    g = res["group"]
    yg = np.abs(y64.reshape(M, K // g, g))
    A64 = yg.max(axis=2) if K else np.zeros((M, 0))
    S = res["S64"]
    with np.errstate(divide="ignore", invalid="ignore"):
        a = np.where(S[..., None] > 0, yg / np.where(S > 0, S, 1.0)[..., None], 0.0)
    el = np.full(a.shape, np.inf)
    for mp in E2M1_MIDPOINTS:
        el = np.minimum(el, np.abs(a - mp) / mp)
    # a zero scale (all-zero group, or a zero NV block scale) makes every code 0: no element
    # boundary there
    el = np.where((S > 0)[..., None], el, np.inf)
    rule = res["rule"]
    if res["fmt"] in (MXFP4, MXFP4_MBS):
        if res["fmt"] == MXFP4_MBS:
            sM = np.repeat(mbs_macro_scale(res["macro"]).astype(np.float64), MBS_MACRO // g, axis=1)
            A64 = A64 / sM
            dm = mbs_macro_distance(res)
        base = {SCALE_FLOOR_OCP: 1.0, SCALE_CEIL_NOCLIP: 1.5, SCALE_OAS: 1.75}[rule]
        gr = _dist_scaled_power(A64, base)
        if rule == SCALE_OAS:
            gr = np.minimum(gr, _dist_scaled_power(A64, 1.5))
        if res["fmt"] == MXFP4_MBS:
            gr = np.minimum(gr, np.repeat(dm, MBS_MACRO // g, axis=1))
    else:
        s_b = A64 / (6.0 * np.float64(res["tensor_scale"]))
        T = e4m3_table()
        mids = (T[1:] + T[:-1]) / 2.0
        idx = np.clip(np.searchsorted(mids, s_b), 1, len(mids) - 1)
        gr = np.minimum(np.abs(s_b - mids[idx - 1]) / mids[idx - 1], np.abs(s_b - mids[idx]) / mids[idx])
    return el.reshape(M, K), gr


def mbs_macro_distance(res: dict) -> np.ndarray:
    """MBS: for every macro block, the distance of its exact 256 f (A_M / 6 = 2^E (1 + f)) to
    the nearest integer, divided by 256 — where m8 = ceil(256 f) steps.  +inf for a zero
    block.  Shape (M, K/128)."""
    y64 = res["y64"]
    M, K = y64.shape
    ym = np.abs(y64.reshape(M, K // MBS_MACRO, MBS_MACRO))
    r = ym.max(axis=2) / 6.0 if K else np.zeros((M, 0))
    mm, _ = np.frexp(r)
    t = np.where(r > 0, (2.0 * mm - 1.0) * 256.0, 0.0)
    return np.where(r > 0, np.abs(t - np.round(t)) / 256.0, np.inf)


def flags(res: dict, tol: float = 1e-5):
    """The flagged set F of the parity rule: elements and groups whose exact value lies
    within ``tol`` (relative) of a place where the code changes (``boundary_distance``).

    Returns (element_flags (M, K) bool, group_flags (M, K/group) bool)."""
    el, gr = boundary_distance(res)
    return el <= tol, gr <= tol


# ----------------------------------------------------------------------------------
# Quantization error ([BG] Technische Zusammenfassung, 2. Methodik, "Theoretische Analyse
# der Fehler": the mean squared quantization error; [UP] Methodologie 1: the gain of OAS
# is stated in QSNR, the quantization signal-to-noise ratio, in dB)
# ----------------------------------------------------------------------------------

def quant_error(x_bits: np.ndarray, fmt: int, group: int, block: int, rule: int,
                tensor_scale=None, chunk_rows: int = 512, signs=None) -> dict:
    """Signal and error energy of rotate + quantize on X, and the QSNR.

    signal = sum of y^2 and noise = sum of (y - yhat)^2 over all elements, where y are the
    exact rotated values (fp64) and yhat the dequantized codes, exact in fp64: q * 2^e for
    MXFP4, q * E4M3(s_b) * s_g for NVFP4.  qsnr_db = 10 log10(signal / noise), +inf when
    noise is 0.  The rotation is orthonormal, so these are also the energies in the
    unrotated domain.  The sums are additive over rows: row chunks are summed in order.

    NVFP4 takes ``tensor_scale`` like ``rotate_quantize``; the dynamic rule computes it
    from the whole tensor's rotated amax when it is None."""
    check_plan(fmt, group, block, rule)
    x_bits = np.asarray(x_bits, np.uint16)
    M, K = x_bits.shape
    if fmt == NVFP4 and tensor_scale is None:
        if rule != SCALE_NV_DYNAMIC:
            raise ValueError("the static NV rule needs the tensor scale")
        tensor_scale = nv_tensor_scale(rotated_amax(x_bits, block, signs=signs))
    signal = 0.0
    noise = 0.0
    for r in range(0, M, chunk_rows):
        if fmt == MXFP4_MBS:
            res = rotate_quantize_mbs(x_bits[r:r + chunk_rows], group, block, rule, signs)
        else:
            res = rotate_quantize(x_bits[r:r + chunk_rows], fmt, group, block, rule, tensor_scale, signs)
        y = res["y64"]
        m = y.shape[0]
        q = e2m1_decode(unpack_nibbles(res["codes"])).reshape(m, K // group, group)
        yhat = (q * res["S64"][..., None]).reshape(m, K)
        signal += float(np.sum(y * y))
        noise += float(np.sum((y - yhat) ** 2))
    qsnr = math.inf if noise == 0.0 else 10.0 * math.log10(signal / noise) if signal > 0 else -math.inf
    return {"signal": signal, "noise": noise, "qsnr_db": qsnr,
            "mse": noise / (M * K) if M * K else 0.0, "tensor_scale": tensor_scale}


# ----------------------------------------------------------------------------------
# The FP4 GEMM that consumes the codes ([BG] Technische Zusammenfassung, 2. Methodik,
# GPU-Kernel-Unterstützung: block-scaled FP4 matrix multiplication of the rotated, quantized
# activations and weights; [BG-en]: the weights absorb the rotation, so the product of the
# rotated operands is the layer's product)
# ----------------------------------------------------------------------------------

def gemm_fp4(a_codes: np.ndarray, a_scales: np.ndarray, b_codes: np.ndarray, b_scales: np.ndarray, fmt: int,
             a_tensor_scale=None, b_tensor_scale=None) -> np.ndarray:
    """D = A_hat B_hat^T in fp64, with A_hat (M x K) and B_hat (N x K) the exact dequantized
    operands: q * 2^(byte - 127) for MXFP4, q * E4M3(byte) * s_g for NVFP4 (the product of the
    two tensor scales is applied once to the result, which is the same number)."""
    group = 32 if fmt == MXFP4 else 16

    def exact(codes, scales):
        q = e2m1_decode(unpack_nibbles(codes))
        R, K = q.shape
        sc = np.asarray(scales, np.uint8).reshape(R, K // group)
        S = np.ldexp(1.0, sc.astype(np.int64) - 127) if fmt == MXFP4 else e4m3_decode(sc)
        return (q.reshape(R, K // group, group) * S[..., None]).reshape(R, K)

    D = exact(a_codes, a_scales) @ exact(b_codes, b_scales).T
    if fmt == NVFP4:
        D = D * (float(np.float32(a_tensor_scale)) * float(np.float32(b_tensor_scale)))
    return D
