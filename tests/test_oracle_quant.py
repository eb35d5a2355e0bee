"""Pins for the oracle's INT8 quantiser and sum-pools (CPU only).

Each test checks the oracle against something it does not compute itself:
hand-derived ties, exact-rational rounding, brute-force integer sums and
invariants that any correct symmetric amax/127 quantiser satisfies.
"""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16_values(shape, seed, scale=1.0):
    x = np.random.default_rng(seed).standard_normal(shape).astype(np.float32) * scale
    return torch.from_numpy(x).to(torch.bfloat16).float().numpy()


def test_golden_ties_round_half_even():
    rows = []
    for line in open(os.path.join(GOLDEN, "quant_ties.txt")):
        if line.startswith("#") or not line.strip():
            continue
        x, q = (t.strip() for t in line.split("|"))
        rows.append((float(x), int(q)))
    blk = np.zeros((64, 4), np.float32)
    for n, (x, _) in enumerate(rows):
        blk[n // 4, n % 4] = x
    q8, s = oracle.quantize_blocks(blk, 64)
    assert s[0] == np.float32(0.125)
    for n, (_, q) in enumerate(rows):
        assert q8[n // 4, n % 4] == q, (rows[n], q8[n // 4, n % 4])


def _nearest_f32(fr: Fraction) -> np.float32:
    """The float32 nearest to an exact rational (ties to even), by search."""
    f = np.float32(float(fr))
    best = f
    for c in (np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))):
        if abs(Fraction(float(c)) - fr) < abs(Fraction(float(best)) - fr):
            best = c
    return best


def test_scale_is_correctly_rounded_amax_over_127():
    x = _bf16_values((640, 32), 3, scale=3.0)
    _, s = oracle.quantize_blocks(x, 64)
    for b in range(10):
        amax = Fraction(float(np.abs(x[64 * b:64 * b + 64]).max()))
        assert s[b] == _nearest_f32(amax / 127)


def test_bounds_amax_and_reconstruction():
    x = _bf16_values((1000, 64), 4, scale=2.5)
    for rows in (64, 128):
        q8, s = oracle.quantize_blocks(x, rows)
        assert q8.dtype == np.int8
        assert np.abs(q8.astype(int)).max() <= 127
        assert (q8 != -128).all()
        for b, (r0, r1) in enumerate(oracle.block_rows(1000, rows)):
            blk, qb = x[r0:r1], q8[r0:r1].astype(np.float64)
            am = np.abs(blk).max()
            hit = np.abs(blk) == am
            assert (np.abs(qb[hit]) == 127).all()
            assert (np.sign(qb[hit]) == np.sign(blk[hit])).all()
            # fl32(x/s) may sit half an ulp (2^-18 below 128) from x/s before rounding
            err = np.abs(blk - qb * float(s[b]))
            assert err.max() <= float(s[b]) * (0.5 + 2.0 ** -17)


def test_zero_block_and_block_independence():
    x = _bf16_values((256, 16), 5)
    x[64:128] = 0.0
    q8, s = oracle.quantize_blocks(x, 64)
    assert s[1] == 0 and (q8[64:128] == 0).all()
    y = x.copy()
    y[128:192] *= 4.0                       # exact in fp32: a power of two
    q8y, sy = oracle.quantize_blocks(y, 64)
    assert sy[2] == 4 * s[2]
    assert (q8y == q8).all()
    assert (np.delete(sy, 2) == np.delete(s, 2)).all()


def test_sign_symmetry():
    x = _bf16_values((320, 16), 6)
    q1, s1 = oracle.quantize_blocks(x, 64)
    q2, s2 = oracle.quantize_blocks(-x, 64)
    assert (s1 == s2).all() and (q2 == -q1).all()


def test_tail_block_uses_only_valid_rows():
    x = _bf16_values((200, 8), 7)
    q8, s = oracle.quantize_blocks(x, 128)
    assert len(s) == 2
    amax = Fraction(float(np.abs(x[128:200]).max()))
    assert s[1] == _nearest_f32(amax / 127)


def test_pools_equal_bruteforce_integer_sums():
    x = _bf16_values((1000, 16), 8)
    q8, _ = oracle.quantize_blocks(x, 128)
    k8, _ = oracle.quantize_blocks(x[::-1].copy(), 64)
    PQ = oracle.q_pools(q8)
    PK = oracle.k_half_pools(k8)
    assert PQ.shape == (8, 16) and PK.shape == (16, 2, 16)
    for i in (0, 7):
        rows = range(128 * i, min(1000, 128 * i + 128))
        for c in (0, 5, 15):
            assert PQ[i, c] == sum(int(q8[r, c]) for r in rows)
    # tail K block: 1000 = 15*64 + 40 -> halves [960, 992) and [992, 1000)
    for c in (0, 9):
        assert PK[15, 0, c] == sum(int(k8[t, c]) for t in range(960, 992))
        assert PK[15, 1, c] == sum(int(k8[t, c]) for t in range(992, 1000))


def test_tail_half_can_be_empty():
    x = _bf16_values((1304, 8), 9)          # 1304 = 20*64 + 24
    k8, _ = oracle.quantize_blocks(x, 64)
    PK = oracle.k_half_pools(k8)
    assert PK.shape[0] == 21
    assert (PK[20, 1] == 0).all()
    assert (PK[20, 0] == k8[1280:1304].astype(np.int64).sum(0)).all()


def test_dequantised_v_within_half_a_step_and_exact_on_grid():
    # INT8 V reuses the K quantiser; its dequantised value x8*s is within half a
    # quantisation step of the input (plus the fp32 rounding of x/s), and exact
    # for inputs that already sit on the grid
    rng = np.random.default_rng(12)
    v = (rng.standard_normal((1000, 64)) * rng.uniform(0.1, 3, (1000, 1))).astype(np.float32)
    v8, sv = oracle.quantize_blocks(v, oracle.quant.K_ROWS)
    deq = oracle.dequantize_blocks(v8, sv, oracle.quant.K_ROWS)
    for b, (t0, t1) in enumerate(oracle.block_rows(1000, 64)):
        err = np.abs(deq[t0:t1] - v[t0:t1].astype(np.float64))
        assert (err <= sv[b] * (0.5 + 2.0 ** -17) + 1e-30).all()
    # values n*s with |n| <= 127 come back exactly (n = 127 sets amax)
    s = np.float32(0.03125)
    n = rng.integers(-127, 128, (64, 32)).astype(np.float32)
    n[0, 0] = 127
    x8, sx = oracle.quantize_blocks(n * s, 64)
    assert np.array_equal(oracle.dequantize_blocks(x8, sx, 64), (n * s).astype(np.float64))
