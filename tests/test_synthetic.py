"""Host checks of the seeded input generator (formats and recipe)."""

import numpy as np
import pytest
import torch

from lm_head_cross_flash_b200 import synthetic as S
from oracle import flash_cce as O


def test_bf16_rounding_matches_torch():
    g = np.random.default_rng(0)
    x = np.concatenate([g.standard_normal(10000).astype(np.float32) * 10,
                        np.array([1.00390625, 1.01171875, -3.0e-39, 65504.0], np.float32)])
    mine = S.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mine, ref)
    assert np.array_equal(S.bf16_bits_to_f32(mine),
                           torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_q4_roundtrip_error_bounded_by_half_step():
    g = np.random.default_rng(1)
    w = (g.standard_normal((37, 256)) / 16).astype(np.float32)
    packed, sc, bi = S.quantize_affine_q4(w)
    deq = O.dequant_affine_q4(packed, sc, bi)
    step = np.repeat(O.bf16_bits_to_f64(sc), 64, axis=1)
    # q is the nearest level to w given the rounded scale/bias, unless clipped
    # by the bf16 rounding of the range ends, which moves it by < 1 step.
    assert np.all(np.abs(deq - w) <= 1.01 * step)
    assert np.mean(np.abs(deq - w) <= 0.5 * step + 1e-7) > 0.97


def test_workload_recipe_small():
    wl = S.make_custom(1, M_split=(5, 6, 7), D=64, V=300)
    assert wl.M == 18 and wl.labels[0] == -1
    assert wl.H.dtype == np.float32 and wl.H_bits is not None
    assert np.array_equal(S.bf16_bits_to_f32(wl.H_bits), wl.H)
    assert np.all((wl.labels[1:] >= 0) & (wl.labels[1:] < 300))
    again = S.make_custom(1, M_split=(5, 6, 7), D=64, V=300, threads=1)
    assert np.array_equal(again.H, wl.H) and np.array_equal(again.W, wl.W)
    q = S.make_custom(4, M_split=(4, 4, 4), D=128, V=100)
    assert q.W is None and q.q_packed.shape == (100, 16) and q.q_scales.shape == (100, 2)


def test_sample_rows_cover_segments():
    wl = S.make_custom(2, M_split=(40, 30, 30), D=64, V=1000)
    r = S.sample_rows(wl, n_uniform=10)
    assert r[0] == 0 and 40 in r and 69 in r and 70 in r and 99 in r
    assert np.all(np.diff(r) > 0)


def test_q8_roundtrip_error_bounded_by_half_step():
    g = np.random.default_rng(2)
    w = (g.standard_normal((23, 128)) / 16).astype(np.float32)
    packed, sc, bi = S.quantize_affine_q8(w)
    deq = O.dequant_affine_q8(packed, sc, bi)
    step = np.repeat(O.bf16_bits_to_f64(sc), 64, axis=1)
    assert np.all(np.abs(deq - w) <= 1.01 * step)
    assert np.mean(np.abs(deq - w) <= 0.5 * step + 1e-7) > 0.97
