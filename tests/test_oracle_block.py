"""Pins for the oracle's decoder block and full decode step (CPU only).

A tiny block is restated here with plain Python loops and ``math`` (no NumPy
matrix products, no oracle helpers except the separately pinned Q8 codec) and
compared with ``oracle.block_forward``; the slice count must not change the
result (the tensor-parallelism glossary's column-then-row split plus
all-reduce is exact), and the 2D FFN grid must agree with 1D.
"""
import math

import numpy as np
import pytest

import synth
from oracle import bf16_to_f64, block_forward, model_forward, q8_dequantize, q8_quantize

TINY = synth.BlockShape(dim=64, n_heads=4, n_kv_heads=2, head_dim=16, ffn_dim=128, vocab=96,
                        max_seq=8, batch=2, n_slices=2, sync_quant=False, pos=5,
                        w_std=0.2, kv_std=1.0)


def _bf(bits):
    return [float(v) for v in bf16_to_f64(bits).ravel()]


def _mat(bits, rows, cols):
    flat = _bf(bits)
    return [flat[r * cols:(r + 1) * cols] for r in range(rows)]


def _bf16_round(v):
    b = np.array([v], np.float32).view(np.uint32)[0]
    b = (int(b) + 0x7FFF + ((int(b) >> 16) & 1)) >> 16
    return float(np.array([b << 16], np.uint32).view(np.float32)[0])


def _q8_roundtrip(vec):
    q, d = q8_quantize(np.array(vec, np.float32).reshape(1, -1))
    return [float(v) for v in q8_dequantize(q, d).ravel()]


def _loop_block(inp, quant):
    s = inp.shape
    D, H, Hkv, hd, Fd = s.dim, s.n_heads, s.n_kv_heads, s.head_dim, s.ffn_dim
    g = H // Hkv
    wq, wk, wv = _mat(inp.wq, H * hd, D), _mat(inp.wk, Hkv * hd, D), _mat(inp.wv, Hkv * hd, D)
    wo = _mat(inp.wo, D, H * hd)
    w1, w3, w2 = _mat(inp.w1, Fd, D), _mat(inp.w3, Fd, D), _mat(inp.w2, D, Fd)
    outs = []
    for b in range(inp.x.shape[0]):
        x = [float(v) for v in inp.x[b]]
        p = int(inp.pos[b])

        def norm(v):
            r = math.sqrt(sum(t * t for t in v) / len(v) + s.norm_eps)
            out = [t / r for t in v]
            return _q8_roundtrip(out) if quant else out

        xn = norm(x)
        q = [sum(wq[r][c] * xn[c] for c in range(D)) for r in range(H * hd)]
        k = [sum(wk[r][c] * xn[c] for c in range(D)) for r in range(Hkv * hd)]
        v = [sum(wv[r][c] * xn[c] for c in range(D)) for r in range(Hkv * hd)]

        def rot(vec, nh):
            out = list(vec)
            for h in range(nh):
                for i in range(hd // 2):
                    ang = p * s.rope_theta ** (-2.0 * i / hd)
                    a0, a1 = vec[h * hd + 2 * i], vec[h * hd + 2 * i + 1]
                    out[h * hd + 2 * i] = a0 * math.cos(ang) - a1 * math.sin(ang)
                    out[h * hd + 2 * i + 1] = a0 * math.sin(ang) + a1 * math.cos(ang)
            return out

        q, k = rot(q, H), rot(k, Hkv)
        kc = bf16_to_f64(inp.k_cache[b]).tolist()
        vc = bf16_to_f64(inp.v_cache[b]).tolist()
        for j in range(Hkv):
            kc[j][p] = [_bf16_round(t) for t in k[j * hd:(j + 1) * hd]]
            vc[j][p] = [_bf16_round(t) for t in v[j * hd:(j + 1) * hd]]
        att = []
        for h in range(H):
            kv = h // g
            sc = [sum(q[h * hd + d] * kc[kv][t][d] for d in range(hd)) / math.sqrt(hd)
                  for t in range(p + 1)]
            m = max(sc)
            e = [math.exp(t - m) for t in sc]
            z = sum(e)
            att += [sum(e[t] / z * vc[kv][t][d] for t in range(p + 1)) for d in range(hd)]
        n = s.n_slices
        x1 = list(x)
        part_cols = H * hd // n
        for sl in range(n):
            cols = range(sl * part_cols, (sl + 1) * part_cols)
            part = [sum(wo[r][c] * att[c] for c in cols) for r in range(D)]
            if quant:
                part = _q8_roundtrip(part)
            x1 = [a + c for a, c in zip(x1, part)]
        xn2 = norm(x1)
        x2 = list(x1)
        fcols = Fd // n
        for sl in range(n):
            hh = []
            for f in range(sl * fcols, (sl + 1) * fcols):
                a = sum(w1[f][c] * xn2[c] for c in range(D))
                c3 = sum(w3[f][c] * xn2[c] for c in range(D))
                hh.append(a / (1 + math.exp(-a)) * c3)
            part = [sum(w2[r][sl * fcols + j] * hh[j] for j in range(fcols)) for r in range(D)]
            if quant:
                part = _q8_roundtrip(part)
            x2 = [a + c for a, c in zip(x2, part)]
        outs.append(x2)
    return np.array(outs)


@pytest.mark.parametrize("quant", [False, True])
def test_tiny_block_brute_force(quant):
    inp = synth.block_inputs(77, TINY)
    got, k_new, v_new = block_forward(inp, n_slices=2, sync_quant=quant)
    ref = _loop_block(inp, quant)
    tol = 1e-10
    assert np.max(np.abs(got - ref)) <= tol
    assert k_new.shape == (2, 2, 16) and v_new.dtype == np.uint16


def test_slice_count_invariance_and_2d():
    inp = synth.block_inputs(78, TINY)
    ref, k1, v1 = block_forward(inp, n_slices=1, sync_quant=False)
    scale = np.max(np.abs(ref))
    for n in (2,):
        y, k, v = block_forward(inp, n_slices=n, sync_quant=False)
        assert np.max(np.abs(y - ref)) <= 1e-12 * scale
        np.testing.assert_array_equal(k, k1)
        np.testing.assert_array_equal(v, v1)
    y2d, _, _ = block_forward(inp, n_slices=2, sync_quant=False, partition=2, grid=(2, 1))
    assert np.max(np.abs(y2d - ref)) <= 1e-12 * scale
    y2d, _, _ = block_forward(inp, n_slices=2, sync_quant=False, partition=2, grid=(1, 2))
    assert np.max(np.abs(y2d - ref)) <= 1e-12 * scale


def test_mha_shape_and_quant_changes_little():
    mha = synth.BlockShape(dim=64, n_heads=4, n_kv_heads=4, head_dim=16, ffn_dim=128, vocab=96,
                           max_seq=8, batch=1, n_slices=4, sync_quant=True, pos=7, w_std=0.2)
    inp = synth.block_inputs(79, mha)
    yq, _, _ = block_forward(inp, n_slices=4, sync_quant=True)
    y, _, _ = block_forward(inp, n_slices=4, sync_quant=False)
    rel = np.max(np.abs(yq - y)) / np.max(np.abs(y))
    assert 0 < rel < 2e-2
    np.testing.assert_allclose(_loop_block(inp, False), y, rtol=0, atol=1e-10)


def test_model_forward_logits_concat():
    s = TINY
    seed = 80
    emb = synth.normal_bf16(seed, "embed", (s.vocab, s.dim), 0.5)
    wcls = synth.normal_bf16(seed, "wcls", (s.vocab, s.dim), 0.2)
    toks = synth.uniform_ids(seed, "tokens", 2, s.vocab)
    g = np.ones(s.dim)
    logits = model_forward(toks, emb, [lambda x: x], g, wcls, n_slices=4, sync_quant=False,
                           eps=1e-5)
    xe = bf16_to_f64(emb)[toks]
    xn = xe / np.sqrt(np.mean(xe * xe, axis=1, keepdims=True) + 1e-5)
    W = bf16_to_f64(wcls)
    for b in range(2):
        for vtok in (0, 17, 95):
            ref = sum(W[vtok, c] * xn[b, c] for c in range(s.dim))
            assert abs(logits[b, vtok] - ref) < 1e-10


def test_synth_is_deterministic_and_subrange_consistent():
    a = synth.normal_bf16(5, "t", (1000,), 0.02)
    b = synth.normal_bf16(5, "t", (1000,), 0.02)
    np.testing.assert_array_equal(a, b)
    c = synth.normal_bf16(5, "t", (300,), 0.02, start=500)
    np.testing.assert_array_equal(a[500:800], c)
    f = synth.normal_f32(5, "u", (200000,))
    assert abs(f.mean()) < 0.01 and abs(f.std() - 1) < 0.01
    ids = synth.uniform_ids(5, "ids", 10000, 32000)
    assert ids.min() >= 0 and ids.max() < 32000
