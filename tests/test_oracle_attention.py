"""Pins for the oracle's RoPE, attention, RMSNorm and activations (CPU only).

The distributed-llama task list names RMSNorm, RoPE and multi-head attention
(llamaRmsAttNorm, llamaMultiheadAtt) without formulas; the tt-metal Llama-2
thread contrasts GQA and MHA. The oracle states textbook definitions; these
tests pin them to library routines (torch CPU, float64), to closed forms and
to brute force.
"""
import cmath
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import attention_decode, relu, rmsnorm, rope, silu, swiglu


def _rand(seed, shape, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


# ------------------------------------------------------------------ RMSNorm

def test_rmsnorm_vs_torch():
    x = _rand(1, (5, 96), 3.0)
    g = _rand(2, (96,))
    ref = F.rms_norm(torch.from_numpy(x), (96,), weight=torch.from_numpy(g), eps=1e-5).numpy()
    np.testing.assert_allclose(rmsnorm(x, g, 1e-5), ref, rtol=1e-13, atol=1e-13)


def test_rmsnorm_constant_row_closed_form():
    c, eps = 0.37, 1e-5
    x = np.full((1, 64), c)
    g = np.linspace(0.5, 2.0, 64)
    np.testing.assert_allclose(rmsnorm(x, g, eps)[0], g * c / math.sqrt(c * c + eps), rtol=1e-14)


def test_rmsnorm_scale_invariance():
    x = _rand(3, (2, 128))
    g = np.ones(128)
    np.testing.assert_allclose(rmsnorm(x * 1000.0, g, 0.0), rmsnorm(x, g, 0.0), rtol=1e-12)
    y = rmsnorm(x, g, 0.0)
    np.testing.assert_allclose(np.mean(y * y, axis=1), 1.0, rtol=1e-12)


# ------------------------------------------------------------------ activations

def test_silu_vs_torch_and_limits():
    z = np.linspace(-30, 30, 601)
    np.testing.assert_allclose(silu(z), F.silu(torch.from_numpy(z)).numpy(), rtol=1e-13, atol=1e-300)
    assert silu(np.array([0.0]))[0] == 0.0
    assert abs(silu(np.array([50.0]))[0] - 50.0) < 1e-15 * 50
    np.testing.assert_allclose(swiglu(z, np.full_like(z, 2.0)), 2.0 * silu(z), rtol=1e-15)
    np.testing.assert_array_equal(relu(np.array([-1.0, 0.0, 2.5])), [0.0, 0.0, 2.5])


# ------------------------------------------------------------------ RoPE

def test_rope_vs_complex_rotation():
    hd, H, theta = 16, 3, 10000.0
    v = _rand(4, (2, H * hd))
    pos = np.array([0, 37])
    out = rope(v, pos, H, hd, theta)
    for b in range(2):
        for h in range(H):
            for i in range(hd // 2):
                z = complex(v[b, h * hd + 2 * i], v[b, h * hd + 2 * i + 1])
                w = z * cmath.exp(1j * pos[b] * theta ** (-2 * i / hd))
                assert abs(out[b, h * hd + 2 * i] - w.real) < 1e-12
                assert abs(out[b, h * hd + 2 * i + 1] - w.imag) < 1e-12


def test_rope_identity_norm_and_relative_position():
    hd, H = 32, 2
    q = _rand(5, (1, H * hd))
    k = _rand(6, (1, H * hd))
    np.testing.assert_allclose(rope(q, np.array([0]), H, hd, 1e4), q, rtol=0, atol=0)
    r = rope(q, np.array([1234]), H, hd, 1e4)
    pn = lambda a: np.hypot(a[0, 0::2], a[0, 1::2])  # noqa: E731
    np.testing.assert_allclose(pn(r), pn(q), rtol=1e-13)
    dots = []
    for m, n in ((5, 2), (103, 100), (4003, 4000)):
        qm = rope(q, np.array([m]), H, hd, 1e4)
        kn = rope(k, np.array([n]), H, hd, 1e4)
        dots.append(float(qm[0, :hd] @ kn[0, :hd]))
    np.testing.assert_allclose(dots, dots[0], rtol=1e-9)
    # the first pair turns by exactly pos radians
    r1 = rope(np.array([[1.0, 0.0] + [0.0] * (hd - 2)]), np.array([3]), 1, hd, 1e4)
    assert abs(r1[0, 0] - math.cos(3)) < 1e-15 and abs(r1[0, 1] - math.sin(3)) < 1e-15


# ------------------------------------------------------------------ attention

def _sdpa_ref(q, kc, vc, pos, H, Hkv, hd):
    B = q.shape[0]
    out = np.zeros((B, H * hd))
    for b in range(B):
        P = pos[b] + 1
        qt = torch.from_numpy(q[b].reshape(1, H, 1, hd))
        kt = torch.from_numpy(kc[b, :, :P]).repeat_interleave(H // Hkv, dim=0).unsqueeze(0)
        vt = torch.from_numpy(vc[b, :, :P]).repeat_interleave(H // Hkv, dim=0).unsqueeze(0)
        o = F.scaled_dot_product_attention(qt, kt, vt)
        out[b] = o.reshape(-1).numpy()
    return out


@pytest.mark.parametrize("H,Hkv", [(4, 4), (8, 2), (8, 1)])
def test_attention_vs_torch_sdpa(H, Hkv):
    hd, T, B = 16, 40, 3
    q = _rand(7, (B, H * hd))
    kc, vc = _rand(8, (B, Hkv, T, hd)), _rand(9, (B, Hkv, T, hd))
    pos = np.array([0, 17, 39])
    got = attention_decode(q, kc, vc, pos, range(H), H, Hkv, hd)
    np.testing.assert_allclose(got, _sdpa_ref(q, kc, vc, pos, H, Hkv, hd), rtol=1e-12, atol=1e-12)
    # a head subset returns exactly those heads' columns
    sub = attention_decode(q, kc, vc, pos, range(2, 4), H, Hkv, hd)
    np.testing.assert_allclose(sub, got[:, 2 * hd:4 * hd], rtol=0, atol=0)


def test_attention_brute_force_loops():
    H, Hkv, hd, T = 4, 2, 8, 5
    q = _rand(10, (1, H * hd))
    kc, vc = _rand(11, (1, Hkv, T, hd)), _rand(12, (1, Hkv, T, hd))
    pos = np.array([4])
    got = attention_decode(q, kc, vc, pos, range(H), H, Hkv, hd)
    for h in range(H):
        kv = h // (H // Hkv)
        s = [sum(q[0, h * hd + d] * kc[0, kv, t, d] for d in range(hd)) / math.sqrt(hd)
             for t in range(5)]
        m = max(s)
        e = [math.exp(v - m) for v in s]
        tot = sum(e)
        for d in range(hd):
            o = sum(e[t] / tot * vc[0, kv, t, d] for t in range(5))
            assert abs(got[0, h * hd + d] - o) < 1e-12


def test_attention_special_cases():
    H, hd, T = 2, 8, 6
    q = _rand(13, (1, H * hd), 5.0)
    kc, vc = _rand(14, (1, H, T, hd)), _rand(15, (1, H, T, hd))
    # one position: output is v_0
    out = attention_decode(q, kc, vc, np.array([0]), range(H), H, H, hd)
    np.testing.assert_allclose(out[0].reshape(H, hd), vc[0, :, 0], rtol=1e-15)
    # all keys equal: uniform weights, output is the mean of V over 0..pos
    kc2 = np.repeat(kc[:, :, :1], T, axis=2)
    out = attention_decode(q, kc2, vc, np.array([T - 1]), range(H), H, H, hd)
    np.testing.assert_allclose(out[0].reshape(H, hd), vc[0].mean(axis=1), rtol=1e-13)
    # positions beyond pos are ignored
    vc3 = vc.copy()
    vc3[:, :, 3:] = 1e6
    a = attention_decode(q, kc, vc, np.array([2]), range(H), H, H, hd)
    b = attention_decode(q, kc, vc3, np.array([2]), range(H), H, H, hd)
    np.testing.assert_array_equal(a, b)
