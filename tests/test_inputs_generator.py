"""Pins for the seeded input generator shared by the oracle and the GPU tests.

Nothing here is method arithmetic: these check that the counter-based draws
follow their published definitions, so that both sides get well-defined,
reproducible inputs.
"""
import math
import os

import numpy as np
import pytest
import torch

import kin_inputs as ki

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.txt")


def _kat_rows():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            v = [int(x, 16) for x in line.split()]
            rows.append((v[0:4], v[4:6], v[6:10]))
    return rows


@pytest.mark.parametrize("ctr,key,expect", _kat_rows())
def test_philox_known_answers(ctr, key, expect):
    assert list(ki.philox4x32_10(ctr, key)) == expect


def test_log_matches_libm():
    us = np.concatenate([np.linspace(1e-10, 1.0 - 1e-12, 2001), [2.0 ** -33, 0.5, 0.70710678, 0.9999999]])
    for u in us:
        assert abs(ki.log_d(u) - math.log(u)) <= 4.5e-16 * max(1.0, abs(math.log(u)))  # 2 ulp


def test_sincos_matches_libm():
    for t in np.linspace(0.0, 1.0 - 1e-9, 4001):
        s, c = ki.sincos_turns(t)
        assert abs(s - math.sin(2 * math.pi * t)) < 9e-16  # libm side also rounds 2*pi*t
        assert abs(c - math.cos(2 * math.pi * t)) < 9e-16
        assert abs(s * s + c * c - 1.0) < 1e-15


def test_normal_moments():
    n = 1 << 17
    z = np.concatenate([ki.normal4(7, ki.TID_K, i, 3) for i in range(n // 4)])
    assert abs(z.mean()) < 5.0 / math.sqrt(n)
    assert abs(z.var() - 1.0) < 5.0 * math.sqrt(2.0 / n)
    # fourth moment of N(0,1) is 3
    assert abs((z ** 4).mean() - 3.0) < 0.1
    # Box-Muller pairs are uncorrelated
    assert abs(np.corrcoef(z[0::2], z[1::2])[0, 1]) < 5.0 / math.sqrt(n / 2)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(100000).astype(np.float32),
        (rng.standard_normal(1000) * 1e30).astype(np.float32),
        np.array([0.0, -0.0, np.inf, -np.inf, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 65504.0], np.float32),
    ])
    mine = ki.bf16_from_f32(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mine, ref)
    nan = ki.bf16_from_f32(np.array([np.nan], np.float32))
    assert nan[0] == ki.BF16_NAN
    # widening back is exact
    back = ki.bf16_to_f32(mine)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_seq_lens_range_and_spread():
    lens = ki.seq_lens(2, 4096, 8192, 32768)
    assert lens.min() >= 8192 and lens.max() <= 32768
    assert abs(lens.mean() - (8192 + 32768) / 2) < 0.05 * 24576
    assert np.all(ki.seq_lens(1, 8, 32768, 32768) == 32768)


def test_heavy_flag_counts():
    lens = np.array([4096, 4000, 17, 16], np.int32)
    hh = ki.heavy_flags(0, 4, 3, 256, 16, lens)
    for b, L in enumerate(lens):
        nb = -(-int(L) // 16)
        m = (nb * 10 + 100) // 200  # round(nb / 20), half up
        for h in range(3):
            assert hh[b, h, :nb].sum() == m
            assert hh[b, h, nb:].sum() == 0
    # different pairs choose different blocks
    assert not np.array_equal(hh[0, 0], hh[0, 1])


def test_kv_rows_match_cache_and_poison():
    w = ki.Workload("t", 2, 2, 4, 128, 16, 40, 70, 4, 9, Lcap=80)
    lens, _, hh = ki.case_meta(w)
    kc = ki.kv_cache_host(w.seed, True, w.B, w.Hkv, w.cap, w.D, w.bs, lens, hh, True)
    vc = ki.kv_cache_host(w.seed, False, w.B, w.Hkv, w.cap, w.D, w.bs, lens, hh, False)
    for b in range(w.B):
        for h in range(w.Hkv):
            L = int(lens[b])
            k, v = ki.pair_rows(w, hh, b, h, L)
            assert np.array_equal(kc[b, h, :L], k)
            assert np.array_equal(vc[b, h, :L], v)
            assert np.all(kc[b, h, L:] == ki.BF16_NAN)
            assert np.all(vc[b, h, L:] == 0)
            # a slice regenerated from the middle equals the same rows
            mid = ki.kv_rows(w.seed, True, b * w.Hkv + h, 5, 21, w.D, w.bs, hh[b, h])
            assert np.array_equal(mid, k[5:21])


def test_heavy_bias_applied_only_to_chosen_blocks():
    w = ki.Workload("t", 1, 1, 1, 128, 16, 320, 320, 4, 3)
    lens, _, hh = ki.case_meta(w)
    hh_none = np.zeros_like(hh)
    k_bias = ki.kv_rows(w.seed, True, 0, 0, 320, 128, 16, hh[0, 0])
    k_plain = ki.kv_rows(w.seed, True, 0, 0, 320, 128, 16, hh_none[0, 0])
    blk_diff = (k_bias != k_plain).reshape(20, 16 * 128).any(axis=1)
    assert np.array_equal(blk_diff, hh[0, 0, :20].astype(bool))
    beta = np.concatenate([ki.normal4(w.seed, ki.TID_BETA, d4, 0) for d4 in range(32)]) * 2.0
    i = int(np.argmax(hh[0, 0]))
    delta = ki.bf16_to_f32(k_bias[i * 16:(i + 1) * 16]).astype(np.float64) - \
        ki.bf16_to_f32(k_plain[i * 16:(i + 1) * 16]).astype(np.float64)
    # each row moved by beta up to the two bf16 roundings
    assert np.allclose(delta.mean(axis=0), beta, atol=0.05 * (1 + np.abs(beta)).max())
