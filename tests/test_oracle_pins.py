"""Pins of the CPU oracle against facts that do not come from the oracle itself:
closed forms, invariants, an independent algorithm (the fast Walsh-Hadamard butterfly),
independent library casts (ml_dtypes, torch), brute-force searches and hand-worked
groups under tests/golden/.  CPU only."""

import math
import os

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle as o

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RULES = {"floor": o.SCALE_FLOOR_OCP, "ceil": o.SCALE_CEIL_NOCLIP, "oas": o.SCALE_OAS}


def bf16(a):
    a = np.asarray(a, np.float32)
    return torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def fwht_reference(x: np.ndarray) -> np.ndarray:
    """Textbook in-place fast Walsh-Hadamard butterfly on the last axis (unnormalised)."""
    y = np.array(x, np.float64, copy=True)
    n = y.shape[-1]
    h = 1
    while h < n:
        for i in range(0, n, 2 * h):
            a = y[..., i:i + h].copy()
            b = y[..., i + h:i + 2 * h].copy()
            y[..., i:i + h] = a + b
            y[..., i + h:i + 2 * h] = a - b
        h *= 2
    return y


# ---------------------------------------------------------------- Hadamard / rotation

@pytest.mark.parametrize("b", [1, 2, 4, 8, 16, 32, 64, 128])
def test_sylvester_closed_form(b):
    H = o.sylvester_hadamard(b)
    i = np.arange(b)
    closed = np.array([[(-1) ** bin(r & c).count("1") for c in i] for r in i])
    assert np.array_equal(H, closed)
    assert np.array_equal(H @ H.T, b * np.eye(b, dtype=np.int64))


@pytest.mark.parametrize("b", [16, 32, 128])
def test_rotation_matches_fast_butterfly(b):
    rng = np.random.default_rng(11)
    x = bf16(rng.standard_normal((3, 4 * b)).astype(np.float32) * 3)
    y = o.rotate(x, b)
    xf = o.bf16_to_f64(x).reshape(3, 4, b)
    ref = (fwht_reference(xf) / math.sqrt(b)).reshape(3, 4 * b)
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-12 * np.abs(ref).max())


@pytest.mark.parametrize("b", [16, 32, 128])
def test_rotation_of_basis_vectors_gives_rows(b):
    H = o.sylvester_hadamard(b)
    for i in (0, 1, b // 2 - 1, b - 1):
        e = np.zeros((1, b), np.float32)
        e[0, i] = 1.0
        y = o.rotate(bf16(e), b)
        np.testing.assert_allclose(y[0], H[i] / math.sqrt(b), rtol=0, atol=1e-15)
    ones = bf16(np.ones((1, b), np.float32))
    y = o.rotate(ones, b)
    assert abs(y[0, 0] - math.sqrt(b)) < 1e-12 and np.all(np.abs(y[0, 1:]) < 1e-12)


@pytest.mark.parametrize("b", [16, 32, 128])
def test_rotation_norm_inverse_and_gemm_identity(b):
    rng = np.random.default_rng(5)
    K = 4 * b
    x = bf16(rng.standard_normal((6, K)).astype(np.float32))
    xf = o.bf16_to_f64(x)
    y = o.rotate(x, b)
    nx = np.linalg.norm(xf.reshape(6, 4, b), axis=2)
    ny = np.linalg.norm(y.reshape(6, 4, b), axis=2)
    np.testing.assert_allclose(ny, nx, rtol=1e-12)
    np.testing.assert_allclose(o.unrotate(y, b), xf, rtol=0, atol=1e-12)
    w = bf16(rng.standard_normal((5, K)).astype(np.float32))
    yw = o.rotate(w, b)
    np.testing.assert_allclose(y @ yw.T, xf @ o.bf16_to_f64(w).T, rtol=1e-10, atol=1e-10)


def test_block_one_is_identity():
    rng = np.random.default_rng(1)
    x = bf16(rng.standard_normal((2, 64)).astype(np.float32))
    assert np.array_equal(o.rotate(x, 1), o.bf16_to_f64(x))


# ---------------------------------------------------------------- E2M1

def test_e2m1_dense_sweep_against_ml_dtypes_cast():
    v = np.linspace(-8.0, 8.0, 400001, dtype=np.float32)
    extra = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 7.0, 1e30, -1e30, 0.0, -0.0,
                      np.nextafter(np.float32(0.25), np.float32(1)),
                      np.nextafter(np.float32(0.25), np.float32(0))], np.float32)
    v = np.concatenate([v, extra, -extra])
    ours = o.e2m1_encode(v)
    lib = v.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    assert np.array_equal(ours, lib)


def test_e2m1_interval_characterisation():
    """Round-to-nearest-even on the grid written as intervals with closed tie ends."""
    edges = [(0.0, 0.25, True, 0), (0.25, 0.75, False, 1), (0.75, 1.25, True, 2), (1.25, 1.75, False, 3),
             (1.75, 2.5, True, 4), (2.5, 3.5, False, 5), (3.5, 5.0, True, 6)]
    rng = np.random.default_rng(3)
    a = np.concatenate([rng.uniform(0, 8, 200000), [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]]).astype(np.float32)
    af = a.astype(np.float64)
    exp = np.full(a.shape, 7)
    for lo, hi, closed, k in edges:
        m = ((af >= lo) & (af <= hi)) if closed else ((af > lo) & (af < hi))
        exp = np.where(m & (exp == 7), k, exp)
    assert np.array_equal(o.e2m1_encode(a), exp.astype(np.uint8))


def test_pack_nibbles_order():
    assert o.pack_nibbles(np.array([1, 2, 3, 4, 0xF, 0], np.uint8)).tolist() == [0x21, 0x43, 0x0F]
    assert np.array_equal(o.unpack_nibbles(np.array([0x21, 0x43], np.uint8)), [1, 2, 3, 4])


# ---------------------------------------------------------------- E4M3

def test_e4m3_table_against_torch_float8():
    t = torch.arange(127, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    assert np.array_equal(o.e4m3_table(), t)


def test_e4m3_encode_against_torch_cast():
    rng = np.random.default_rng(7)
    s = np.concatenate([np.exp2(rng.uniform(-14, 8.8, 100000)), o.e4m3_table(),
                        (o.e4m3_table()[1:] + o.e4m3_table()[:-1]) / 2, [0.0, 2.0 ** -10, 448.0, 455.0]])
    s = s.astype(np.float32)
    s = s[s <= 456]
    ours = o.e4m3_encode(s)
    ref = torch.from_numpy(s).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)
    assert o.e4m3_encode(np.array([500.0, 1e30], np.float32)).tolist() == [0x7E, 0x7E]


# ---------------------------------------------------------------- MX scale rules

def brute_force_exponent(A: float, rule: int) -> int:
    """Search e over a wide integer range directly from the rule's definition."""
    if A == 0:
        return -127
    es = np.arange(-200, 200)
    if rule == o.SCALE_FLOOR_OCP:           # largest e with 2^(e+2) <= A
        e = int(es[np.ldexp(1.0, es + 2) <= A].max())
    else:                                    # smallest e with A / 2^e <= 6
        e = int(es[A / np.ldexp(1.0, es) <= 6.0].min())
        if rule == o.SCALE_OAS and 3.0 <= A / 2.0 ** e <= 3.5:
            e -= 1
    return max(-127, min(127, e))


@pytest.mark.parametrize("rule", [o.SCALE_FLOOR_OCP, o.SCALE_CEIL_NOCLIP, o.SCALE_OAS])
def test_mx_exponent_brute_force(rule):
    rng = np.random.default_rng(2 + rule)
    A = np.concatenate([np.exp2(rng.uniform(-140, 120, 3000)),
                        np.exp2(np.arange(-130, 120)), 1.5 * np.exp2(np.arange(-60, 60)),
                        1.75 * np.exp2(np.arange(-60, 60)), [0.0]]).astype(np.float32)
    ours = o.mx_scale_exponent(A, rule)
    ref = np.array([brute_force_exponent(float(a), rule) for a in A])
    assert np.array_equal(ours, ref)


def test_mx_rule_invariants():
    rng = np.random.default_rng(9)
    A = np.exp2(rng.uniform(-30, 30, 50000)).astype(np.float32)
    af = A.astype(np.float64)
    n_floor = af / np.exp2(o.mx_scale_exponent(A, o.SCALE_FLOOR_OCP))
    n_ceil = af / np.exp2(o.mx_scale_exponent(A, o.SCALE_CEIL_NOCLIP))
    n_oas = af / np.exp2(o.mx_scale_exponent(A, o.SCALE_OAS))
    assert np.all((n_floor >= 4) & (n_floor < 8))
    assert np.all((n_ceil > 3) & (n_ceil <= 6))          # nothing ever clips
    assert np.all(((n_oas > 3.5) & (n_oas <= 6)) | ((n_oas > 6) & (n_oas <= 7)))
    m = np.frexp(af)[0] * 2                               # mantissa in [1, 2)
    differ = o.mx_scale_exponent(A, o.SCALE_FLOOR_OCP) != o.mx_scale_exponent(A, o.SCALE_CEIL_NOCLIP)
    assert np.array_equal(differ, m > 1.5)


# ---------------------------------------------------------------- whole-path worked groups

def load_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def test_mx_worked_groups():
    rows = load_rows("mx_worked_groups.txt")
    assert len(rows) >= 40
    for r in rows:
        rule = RULES[r[0]]
        amax, probe = float(r[1]), float(r[2])
        byte, ca, cp = int(r[3]), int(r[4]), int(r[5])
        da, dp = float(r[6]), float(r[7])
        g = np.zeros((1, 32), np.float32)
        g[0, 0], g[0, 1] = amax, probe
        x = bf16(g)
        assert np.array_equal(o.bf16_to_f64(x)[0, :2], [amax, probe]), r
        res = o.rotate_quantize(x, o.MXFP4, 32, 1, rule)
        q = o.unpack_nibbles(res["codes"])[0]
        assert res["scales"][0, 0] == byte, r
        assert (q[0], q[1]) == (ca, cp), r
        assert np.all(q[2:] == 0), r
        deq = o.dequantize(res["codes"], res["scales"], o.MXFP4, 32, 1)[0]
        assert (deq[0], deq[1]) == (np.float32(da), np.float32(dp)), r


def test_nv_worked_groups():
    rows = load_rows("nv_worked_groups.txt")
    assert len(rows) >= 9
    for r in rows:
        s_g, amax, probe = float(r[0]), float(r[1]), float(r[2])
        byte, ca, cp = int(r[3]), int(r[4]), int(r[5])
        da, dp = float(r[6]), float(r[7])
        g = np.zeros((1, 16), np.float32)
        g[0, 0], g[0, 1] = amax, probe
        x = bf16(g)
        assert np.array_equal(o.bf16_to_f64(x)[0, :2], [amax, probe]), r
        res = o.rotate_quantize(x, o.NVFP4, 16, 1, o.SCALE_NV_STATIC, tensor_scale=s_g)
        q = o.unpack_nibbles(res["codes"])[0]
        assert res["scales"][0, 0] == byte, r
        assert (q[0], q[1]) == (ca, cp), r
        assert np.all(q[2:] == 0), r
        deq = o.dequantize(res["codes"], res["scales"], o.NVFP4, 16, 1, tensor_scale=s_g)[0]
        assert (deq[0], deq[1]) == (np.float32(da), np.float32(dp)), r


def test_nv_tensor_scale_definition():
    x = np.zeros((2, 16), np.float32)
    x[1, 3] = -2688.0
    res = o.rotate_quantize(bf16(x), o.NVFP4, 16, 1, o.SCALE_NV_DYNAMIC)
    assert res["tensor_scale"] == np.float32(1.0)
    res0 = o.rotate_quantize(bf16(np.zeros((1, 16), np.float32)), o.NVFP4, 16, 1, o.SCALE_NV_DYNAMIC)
    assert res0["tensor_scale"] == np.float32(1.0)
    assert np.all(res0["codes"] == 0) and np.all(res0["scales"] == 0)
    # the amax is taken after the rotation: one spike of 1 in a 16-block becomes 16 values of 1/4
    e = np.zeros((1, 16), np.float32)
    e[0, 5] = 1.0
    r = o.rotate_quantize(bf16(e), o.NVFP4, 16, 16, o.SCALE_NV_DYNAMIC)
    assert r["tensor_scale"] == np.float32(np.float32(0.25) / np.float32(2688.0))


# ---------------------------------------------------------------- brute-force optimality

@pytest.mark.parametrize("fmt,g,rule", [(o.MXFP4, 32, o.SCALE_FLOOR_OCP), (o.MXFP4, 32, o.SCALE_CEIL_NOCLIP),
                                        (o.NVFP4, 16, o.SCALE_NV_DYNAMIC)])
def test_codes_are_nearest_under_the_chosen_scale(fmt, g, rule):
    """Given the block scale, every element code is the nearest of all 16 codes to y/S
    (ties to even); checked by trying every code."""
    rng = np.random.default_rng(21)
    x = bf16((rng.standard_normal((4, 256)) * np.exp(rng.standard_normal((4, 1)))).astype(np.float32))
    res = o.rotate_quantize(x, fmt, g, 32, rule)
    q = o.unpack_nibbles(res["codes"]).reshape(4, 256 // g, g)
    S = res["S64"]
    v = res["y32"].reshape(4, 256 // g, g).astype(np.float64) / S[..., None]
    allv = o.e2m1_decode(np.arange(16, dtype=np.uint8))
    d = np.abs(v[..., None] - allv)                   # distance to each of 16 codes
    best = d.min(axis=-1)
    chosen = np.take_along_axis(d, q[..., None].astype(np.int64), axis=-1)[..., 0]
    assert np.all(chosen <= best * (1 + 1e-6) + 1e-300)
    assert np.all((q & 8 != 0) == np.signbit(v))


def test_quantization_is_idempotent_on_its_own_grid():
    rng = np.random.default_rng(4)
    x = bf16(rng.standard_normal((8, 128)).astype(np.float32) * 4)
    # an NV tensor scale that is a power of two keeps every grid value representable in bf16
    for fmt, g, rule, ts in [(o.MXFP4, 32, o.SCALE_FLOOR_OCP, None), (o.MXFP4, 32, o.SCALE_CEIL_NOCLIP, None),
                             (o.MXFP4, 32, o.SCALE_OAS, None), (o.NVFP4, 16, o.SCALE_NV_STATIC, 2.0 ** -7)]:
        r1 = o.rotate_quantize(x, fmt, g, 1, rule, tensor_scale=ts)
        d1 = o.dequantize(r1["codes"], r1["scales"], fmt, g, 1, r1["tensor_scale"])
        x2 = bf16(d1)
        assert np.array_equal(o.bf16_to_f64(x2), d1.astype(np.float64))   # grid values fit bf16
        r2 = o.rotate_quantize(x2, fmt, g, 1, rule, tensor_scale=r1["tensor_scale"])
        d2 = o.dequantize(r2["codes"], r2["scales"], fmt, g, 1, r2["tensor_scale"])
        assert np.array_equal(d1, d2), (fmt, rule)


def test_block_one_reduces_to_absmax_rtn():
    """With no rotation and a group maximum that is an exact power of two, the floor rule
    puts it at E2M1 4 and every element is rounded on the grid X*{0,.5,...,6}."""
    rng = np.random.default_rng(8)
    x = rng.uniform(-1, 1, (16, 32)).astype(np.float32)
    x[:, 0] = np.float32(1.0)
    xb = bf16(x)
    res = o.rotate_quantize(xb, o.MXFP4, 32, 1, o.SCALE_FLOOR_OCP)
    assert np.all(res["scales"] == 125)                       # X = 1/4
    deq = o.dequantize(res["codes"], res["scales"], o.MXFP4, 32, 1)
    xf = o.bf16_to_f64(xb)
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6]) * 0.25
    nearest = grid[np.argmin(np.abs(np.abs(xf)[..., None] - grid), axis=-1)]
    ok = np.isclose(np.abs(deq), nearest) | np.isclose(np.abs(np.abs(xf) - np.abs(deq)),
                                                        np.abs(np.abs(xf) - nearest))
    assert np.all(ok)
