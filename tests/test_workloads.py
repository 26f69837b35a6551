"""The seeded input generators: determinism, the bf16 cast, the recipe's structure."""

import dataclasses

import numpy as np
import torch

from microscaling_fp4_quantization_b200 import workloads as W


def test_bf16_cast_matches_torch():
    rng = np.random.default_rng(0)
    a = np.concatenate([rng.standard_normal(200000) * np.exp(rng.uniform(-30, 30, 200000)),
                        [0.0, -0.0, 1.0, 1.00390625, 1.0 + 2 ** -9, 1.0 + 3 * 2 ** -9, 3e38, -3e38]]).astype(np.float32)
    ours = W.f32_to_bf16_bits(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(W.bf16_bits_to_f32(ours), torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).float().numpy())


def test_generation_is_deterministic_and_chunk_invariant():
    w = dataclasses.replace(W.NV_4K, M=40, K=256, n_outlier=3)
    a = w.generate()
    b = w.generate()
    assert np.array_equal(a, b)
    chunks = np.concatenate(list(w.row_chunks(chunk_rows=7)))
    assert np.array_equal(a, chunks)
    w2 = dataclasses.replace(w, seed=w.seed + 1)
    assert not np.array_equal(a, w2.generate())


def test_outlier_columns_are_scaled():
    w = dataclasses.replace(W.NV_4K, M=512)
    x = W.bf16_bits_to_f32(w.generate())
    cols = w.outlier_columns()
    assert len(cols) == 20 and len(set(cols.tolist())) == 20
    std = x.std(axis=0)
    others = np.setdiff1d(np.arange(w.K), cols)
    assert np.all(std[cols] > 30) and np.all(std[others] < 2)


def test_recipe_table():
    assert W.SMALL_MX.M == 128 and W.SMALL_MX.K == 4096 and W.SMALL_MX.n_outlier == 8
    assert W.NV_4K.n_outlier == 20 and W.PREFILL_NV.n_outlier == 72
    assert (W.MX_8K_FLOOR.block, W.MX_8K_CEIL.rule) == (128, W.SCALE_CEIL_NOCLIP)
    assert [d.M for d in W.DECODE] == [1, 4, 16]
    assert W.PREFILL_NV.bytes_per_call() == 32768 * 14336 * 2 + 32768 * 14336 // 2 + 32768 * 14336 // 16 + 4
    assert W.SMALL_MX.bytes_per_call() == 1048576 + 262144 + 16384


def test_lognormal_rows_and_student_t_body():
    w = dataclasses.replace(W.PREFILL_NV, M=256, K=1024, n_outlier=5)
    x = W.bf16_bits_to_f32(w.generate())
    rs = np.median(np.abs(x), axis=1)
    assert rs.max() / rs.min() > 20          # per-row magnitude spread of a log-normal(0, 1)
    t = dataclasses.replace(W.MX_8K_FLOOR, M=64, K=1024)
    xt = W.bf16_bits_to_f32(t.generate()).astype(np.float64)
    kurt = ((xt - xt.mean()) ** 4).mean() / xt.var() ** 2
    assert kurt > 6                          # heavy tails of Student-t(3)
