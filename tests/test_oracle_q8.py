"""Pins for the oracle's Q8 sync-buffer quantiser (CPU only).

The distributed-llama task list (issue #29, buildLlama2Arch) names the
Quantize*/Dequantize* steps; the format (int8, blocks of 32, one fp32 scale,
half-away rounding) is the reading documented in the oracle. These tests pin
the oracle to hand-worked blocks and to properties any correct quantiser of
that format has.
"""
import os

import numpy as np
import pytest

from oracle import q8_dequantize, q8_quantize

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "q8_blocks.txt")


def _golden_blocks():
    blocks, cur = [], {}
    for ln in open(GOLDEN):
        if ln.startswith("#") or not ln.strip():
            continue
        k, v = ln.split(":", 1)
        cur[k] = v.split()
        if k == "d":
            blocks.append(cur)
            cur = {}
    out = []
    for b in blocks:
        x = np.zeros(32, np.float32)
        x[: len(b["x"])] = [float(v) for v in b["x"]]
        q = np.zeros(32, np.int8)
        q[: len(b["q"])] = [int(v) for v in b["q"]]
        out.append((x, q, np.float32(float(b["d"][0]))))
    return out


@pytest.mark.parametrize("idx", range(len(_golden_blocks())))
def test_golden_blocks(idx):
    x, q_exp, d_exp = _golden_blocks()[idx]
    q, d = q8_quantize(x)
    assert d.shape == (1,)
    assert d[0] == d_exp
    np.testing.assert_array_equal(q, q_exp)
    np.testing.assert_array_equal(q8_dequantize(q, d), q_exp.astype(np.float32) * d_exp)


def test_golden_blocks_concatenated_rows():
    blocks = _golden_blocks()
    x = np.concatenate([b[0] for b in blocks]).reshape(1, -1)
    q, d = q8_quantize(x)
    np.testing.assert_array_equal(q.ravel(), np.concatenate([b[1] for b in blocks]))
    np.testing.assert_array_equal(d.ravel(), np.array([b[2] for b in blocks], np.float32))


def test_invariants_random():
    rng = np.random.default_rng(7)
    x = (rng.standard_normal((64, 4096)) * rng.uniform(1e-3, 1e3, (64, 1))).astype(np.float32)
    q, d = q8_quantize(x)
    assert q.dtype == np.int8 and d.dtype == np.float32 and d.shape == (64, 128)
    assert np.all(np.abs(q.astype(np.int32)) <= 127)
    blk = x.reshape(-1, 32)
    qb = q.reshape(-1, 32).astype(np.int32)
    # the largest-magnitude element maps to +-127 with the sign of x
    am = np.argmax(np.abs(blk), axis=1)
    sel = qb[np.arange(len(am)), am]
    np.testing.assert_array_equal(np.abs(sel), 127)
    np.testing.assert_array_equal(np.sign(sel), np.sign(blk[np.arange(len(am)), am]))
    # reconstruction error at most half a step (plus float32 rounding of x/d and q*d)
    xr = q8_dequantize(q, d).reshape(-1, 32).astype(np.float64)
    db = d.reshape(-1).astype(np.float64)[:, None]
    err = np.abs(xr - blk.astype(np.float64))
    assert np.all(err <= db * (0.5 + 1e-5) + np.abs(blk) * 2e-7)
    # codes are monotone in x within a block
    order = np.argsort(blk, axis=1, kind="stable")
    qs = np.take_along_axis(qb, order, axis=1)
    assert np.all(np.diff(qs, axis=1) >= 0)


def test_zero_and_signed_zero_block():
    x = np.zeros((2, 32), np.float32)
    x[1] = -0.0
    q, d = q8_quantize(x)
    assert np.all(q == 0) and np.all(d == 0)
    assert np.all(q8_dequantize(q, d) == 0)


def test_denormal_blocks():
    # amax so small that amax/127 underflows to zero -> zero block
    x = np.zeros(32, np.float32)
    x[3] = np.float32(1e-44)
    q, d = q8_quantize(x)
    assert d[0] == 0 and np.all(q == 0)
    # denormal scale: codes stay in range and the max element still maps to 127
    x = np.zeros(32, np.float32)
    x[0] = np.float32(1e-40)
    x[1] = np.float32(-5e-41)
    q, d = q8_quantize(x)
    assert d[0] > 0 and d[0] < np.finfo(np.float32).tiny
    assert q[0] == 127 and -66 <= q[1] <= -61


def test_ties_go_away_from_zero():
    # d = 1 (amax 127); x/d = k + 0.5 exactly for every k
    x = np.zeros(32, np.float32)
    x[0] = 127
    ks = np.arange(-15, 16)
    x[1:] = (ks + 0.5).astype(np.float32)
    q, _ = q8_quantize(x)
    exp = np.where(ks + 0.5 > 0, ks + 1, ks)
    np.testing.assert_array_equal(q[1:], exp)


def test_just_below_half_rounds_down():
    # 0.49999997 (largest float32 below 0.5) must round to 0; a float32 floor(v+0.5)
    # would round it up.
    x = np.zeros(32, np.float32)
    x[0] = 127
    x[1] = np.nextafter(np.float32(0.5), np.float32(0))
    x[2] = np.nextafter(np.float32(1.5), np.float32(0))
    q, _ = q8_quantize(x)
    assert q[1] == 0 and q[2] == 1
