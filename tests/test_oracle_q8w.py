"""Pins of the oracle's int8-weight block (``q8_weights``, ``block_forward(weights_q8=True)``).

The new arithmetic in that form is the slice product of Q8 weights with Q8
activations. The oracle computes it as a float64 matmul of dequantised values;
the GPU as integer dot products per 32-value block scaled by ``d_w * d_x``. The
identity between the two is pinned here with exact rational arithmetic (Python
integers and fractions), independently of NumPy. The Q8 codec itself is pinned
by tests/test_oracle_q8.py, the rest of the block by tests/test_oracle_block.py.
"""
from fractions import Fraction

import numpy as np

import oracle
import synth


def _exact_q8_dot(qw, dw, qx, dx):
    """sum over blocks of d_w d_x sum_i q_w,i q_x,i, exactly (float32 scales as fractions)."""
    total = Fraction(0)
    for blk in range(qw.size // 32):
        s = sum(int(a) * int(b) for a, b in zip(qw[32 * blk:32 * blk + 32], qx[32 * blk:32 * blk + 32]))
        total += Fraction(float(dw[blk])) * Fraction(float(dx[blk])) * s
    return total


def test_q8_weight_product_is_the_integer_block_dot():
    rng = np.random.default_rng(5)
    K, rows = 256, 6
    w_bits = synth.f32_to_bf16_bits((rng.standard_normal((rows, K)) * 0.02).astype(np.float32))
    x = (rng.standard_normal((2, K)) * 3).astype(np.float32)
    qw, dw = oracle.q8_weights(w_bits)
    qx, dx = oracle.q8_quantize(x)
    wq = qw.astype(np.float64) * np.repeat(dw.astype(np.float64), 32, axis=-1)
    got = oracle.q8_exact(x) @ wq.T
    for b in range(2):
        for r in range(rows):
            exact = _exact_q8_dot(qw[r], dw[r], qx[b], dx[b])
            assert abs(float(exact) - got[b, r]) <= 1e-12 * max(1.0, abs(float(exact)))


def test_q8_weights_rows_and_error_bound():
    """Each row is quantised on its own, in blocks of 32 along the input dimension:
    every element is within half a step of its block's scale, and the max-|w|
    element of each block is recovered exactly (code +-127)."""
    rng = np.random.default_rng(9)
    w = (rng.standard_normal((4, 96)) * 0.05).astype(np.float32)
    w_bits = synth.f32_to_bf16_bits(w)
    wf = oracle.bf16_to_f64(w_bits).astype(np.float32)
    q, d = oracle.q8_weights(w_bits)
    assert q.shape == (4, 96) and d.shape == (4, 3)
    back = q.astype(np.float64) * np.repeat(d.astype(np.float64), 32, axis=-1)
    for r in range(4):
        for blk in range(3):
            seg = wf[r, 32 * blk:32 * blk + 32].astype(np.float64)
            err = np.abs(seg - back[r, 32 * blk:32 * blk + 32])
            # half a step, plus the float32 rounding of x / d (|x / d| <= 127)
            assert np.all(err <= float(d[r, blk]) * (0.5 + 127 * 2.0 ** -24))
            k = int(np.argmax(np.abs(seg)))
            assert abs(int(q[r, 32 * blk + k])) == 127


def test_q8_weight_block_close_to_bf16_block():
    """The int8-weight block moves the block's update x_out - x by about the Q8
    rounding of the weights (1/254 of a block maximum per weight): more than
    float32 rounding, less than a few per cent."""
    s = synth.BlockShape(dim=256, n_heads=2, n_kv_heads=2, head_dim=128, ffn_dim=512, vocab=0,
                         max_seq=40, batch=2, n_slices=2, sync_quant=True, pos=39, w_std=0.05)
    inp = synth.block_inputs(31, s)
    ref, _, _ = oracle.block_forward(inp, 2, True)
    q8w, _, _ = oracle.block_forward(inp, 2, True, weights_q8=True)
    dx_ref = ref - inp.x
    dx_q = q8w - inp.x
    rel = np.max(np.abs(dx_q - dx_ref)) / np.max(np.abs(dx_ref))
    assert 1e-4 < rel < 5e-2, rel  # changed, by about the weights' Q8 rounding
