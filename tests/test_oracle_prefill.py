"""Pins of the oracle's multi-token step: rows that share a sequence (a prefill chunk).

Pope et al. demo 2 contrasts decode (a few hundred tokens per step) with prefill
(many tokens per step); the pages define no prefill computation of their own. The
reading taken: a chunk of consecutive tokens of one sequence computes exactly what
decoding them one at a time does. These tests hold ``block_forward(seq=...)`` to
that, and its attention to the textbook masked-softmax form of causal attention,
written independently as one matrix product with a mask.
"""
import math

import numpy as np
import pytest

import oracle
import synth

SMALL = synth.BlockShape(dim=64, n_heads=4, n_kv_heads=2, head_dim=16, ffn_dim=128, vocab=0,
                         max_seq=24, batch=1, n_slices=2, sync_quant=False, pos=5, w_std=0.1)


def _one_row(inp, b, k_cache, v_cache, seq_b):
    """Row b as a one-row decode step of its own sequence's cache."""
    import dataclasses

    return dataclasses.replace(inp, x=inp.x[b:b + 1], pos=inp.pos[b:b + 1],
                               k_cache=k_cache[seq_b:seq_b + 1], v_cache=v_cache[seq_b:seq_b + 1],
                               extra={})


def _sequential(inp, n, quant, seq):
    """Decode the rows one at a time in position order, each writing its k/v row
    into its sequence's cache before the next row runs."""
    kc, vc = inp.k_cache.copy(), inp.v_cache.copy()
    B = inp.x.shape[0]
    out = np.zeros((B, inp.shape.dim))
    rows = np.zeros((2, B, inp.shape.n_kv_heads, inp.shape.head_dim), dtype=np.uint16)
    for b in sorted(range(B), key=lambda r: inp.pos[r]):
        y, k, v = oracle.block_forward(_one_row(inp, b, kc, vc, seq[b]), n, quant)
        out[b], rows[0, b], rows[1, b] = y[0], k[0], v[0]
        kc[seq[b], :, inp.pos[b]] = k[0]
        vc[seq[b], :, inp.pos[b]] = v[0]
    return out, rows


@pytest.mark.parametrize("quant", [False, True])
@pytest.mark.parametrize("n", [1, 2])
def test_chunk_equals_token_by_token_decode(n, quant):
    pos = np.arange(5, 11)  # six tokens after a prefix of five
    inp = synth.chunk_inputs(31, SMALL, pos, np.zeros(6, dtype=np.int32))
    y, k, v = oracle.block_forward(inp, n, quant, seq=inp.extra["seq"])
    y_seq, rows = _sequential(inp, n, quant, inp.extra["seq"])
    assert np.max(np.abs(y - y_seq)) <= 1e-12 * np.max(np.abs(y_seq))
    np.testing.assert_array_equal(k, rows[0])
    np.testing.assert_array_equal(v, rows[1])


def test_mixed_sequences_equal_token_by_token_decode():
    """Decode rows of two sequences and a prefill run of a third in one step."""
    s = synth.BlockShape(**{**SMALL.__dict__, "max_seq": 16})
    seq = np.array([2, 0, 2, 1, 2, 0], dtype=np.int32)
    pos = np.array([5, 9, 6, 5, 7, 5], dtype=np.int32)
    inp = synth.chunk_inputs(32, s, pos, seq)
    y, _, _ = oracle.block_forward(inp, 2, True, seq=seq)
    y_seq, _ = _sequential(inp, 2, True, seq)
    assert np.max(np.abs(y - y_seq)) <= 1e-12 * np.max(np.abs(y_seq))


def test_chunk_attention_is_masked_softmax():
    """Causal attention of a chunk: S = Q K^T / sqrt(d) over every cached position,
    positions after each row's own masked to -inf, softmax by rows, times V."""
    rng = np.random.default_rng(5)
    H, Hkv, hd, T, p0, L = 4, 2, 16, 20, 7, 9
    q = rng.standard_normal((L, H * hd))
    kc = rng.standard_normal((1, Hkv, T, hd))
    vc = rng.standard_normal((1, Hkv, T, hd))
    pos = p0 + np.arange(L)
    got = oracle.attention_decode(q, kc, vc, pos, range(H), H, Hkv, hd, seq=np.zeros(L, int))
    for h in range(H):
        K, V = kc[0, h // (H // Hkv)], vc[0, h // (H // Hkv)]
        S = q[:, h * hd:(h + 1) * hd] @ K.T / math.sqrt(hd)            # [L, T]
        mask = np.arange(T)[None, :] > pos[:, None]                      # after the row's position
        S = np.where(mask, -np.inf, S)
        P = np.exp(S - S.max(axis=1, keepdims=True))
        P /= P.sum(axis=1, keepdims=True)
        want = P @ V
        assert np.max(np.abs(got[:, h * hd:(h + 1) * hd] - want)) <= 1e-13 * np.max(np.abs(want))
    # the first row sees p0 + 1 positions only: moving any later cache row changes nothing
    kc2 = kc.copy()
    kc2[0, :, p0 + 1:] += 1.0
    got2 = oracle.attention_decode(q, kc2, vc, pos, range(H), H, Hkv, hd, seq=np.zeros(L, int))
    np.testing.assert_array_equal(got2[0], got[0])
    assert not np.array_equal(got2[1], got[1])


def test_default_sequence_map_is_the_row():
    inp = synth.block_inputs(33, synth.BlockShape(**{**SMALL.__dict__, "batch": 3}))
    a = oracle.block_forward(inp, 2, True)
    b = oracle.block_forward(inp, 2, True, seq=np.arange(3))
    for u, w in zip(a, b):
        np.testing.assert_array_equal(u, w)
