"""Pins for the oracle's partitioned FFN (CPU only).

The aiterms.tw "Tensor Parallelism" glossary ("how it works": Linear1 split by
columns, ReLU local, Linear2 split by rows, one all-reduce) fixes that the
partitioned FFN equals the unpartitioned one; the Pope et al. lecture script
(demo1_1d_vs_2d) fixes that 1D and 2D weight-stationary partitions of the same
weights compute the same layer. The unpartitioned reference here is a plain
triple loop or one matrix product of the whole matrices.
"""
import numpy as np
import pytest

from oracle import ffn_forward, grid_2d, q8_quantize, relu, silu


def _rand(seed, shape, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _loop_ffn(X, W1, W2, act, W3=None):
    B, E = X.shape
    F = W1.shape[0]
    H = [[0.0] * F for _ in range(B)]
    for b in range(B):
        for f in range(F):
            a = sum(X[b, e] * W1[f, e] for e in range(E))
            if act == "relu":
                H[b][f] = a if a > 0 else 0.0
            else:
                c = sum(X[b, e] * W3[f, e] for e in range(E))
                H[b][f] = a / (1.0 + np.exp(-a)) * c
    Y = np.zeros((B, E))
    for b in range(B):
        for e in range(E):
            Y[b, e] = sum(H[b][f] * W2[e, f] for f in range(F))
    return Y


@pytest.mark.parametrize("act", ["relu", "swiglu"])
def test_brute_force_tiny(act):
    X, W1, W2 = _rand(1, (3, 8)), _rand(2, (16, 8)), _rand(3, (8, 16))
    W3 = _rand(4, (16, 8)) if act == "swiglu" else None
    ref = _loop_ffn(X, W1, W2, act, W3)
    for n in (1, 2, 4, 8):
        y = ffn_forward(X, W1, W2, act=act, W3=W3, partition=1, n_slices=n)
        np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)
    for grid in ((2, 2), (2, 4), (4, 2), (8, 1), (1, 8)):
        y = ffn_forward(X, W1, W2, act=act, W3=W3, partition=2, n_slices=grid[0] * grid[1],
                        grid=grid)
        np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("act", ["relu", "swiglu"])
def test_split_equals_unsharded(act):
    B, E, F = 8, 64, 512
    X, W1, W2 = _rand(5, (B, E)), _rand(6, (F, E), 0.1), _rand(7, (E, F), 0.1)
    W3 = _rand(8, (F, E), 0.1) if act == "swiglu" else None
    a = X @ W1.T
    H = relu(a) if act == "relu" else silu(a) * (X @ W3.T)
    full = H @ W2.T
    scale = np.max(np.abs(full))
    for n in (1, 2, 4, 8, 64):
        y = ffn_forward(X, W1, W2, act=act, W3=W3, partition=1, n_slices=n)
        assert np.max(np.abs(y - full)) <= 1e-12 * scale
    y2d = ffn_forward(X, W1, W2, act=act, W3=W3, partition=2, n_slices=64, grid=(8, 8))
    y1d = ffn_forward(X, W1, W2, act=act, W3=W3, partition=1, n_slices=64)
    assert np.max(np.abs(y2d - full)) <= 1e-12 * scale
    assert np.max(np.abs(y2d - y1d)) <= 1e-12 * scale


def test_ggml_example_shape_relu_first_stage_only():
    # ggmlR ggml_pp_dp_forward example: z = W x per stage, ReLU after stage 1 only.
    K = 64
    X = _rand(9, (8, K))
    W1, W2 = _rand(10, (K, K)), _rand(11, (K, K))
    y = ffn_forward(X, W1, W2, act="relu", partition=1, n_slices=2)
    np.testing.assert_allclose(y, _loop_ffn(X, W1, W2, "relu"), rtol=1e-12, atol=1e-10)


def test_partial_signs_matter():
    # a dropped or sign-flipped slice would change the result by far more than rounding
    X, W1, W2 = _rand(12, (4, 32)), _rand(13, (64, 32)), _rand(14, (32, 64))
    full = relu(X @ W1.T) @ W2.T
    y = ffn_forward(X, W1, W2, act="relu", partition=1, n_slices=4)
    np.testing.assert_allclose(y, full, rtol=1e-12, atol=1e-12)
    first = relu(X @ W1[:16].T) @ W2[:, :16].T
    assert np.max(np.abs(y - first)) > 1e-3


def test_quantised_partials_within_bound():
    B, E, F, n = 4, 64, 256, 4
    X, W1, W2 = _rand(15, (B, E)), _rand(16, (F, E), 0.2), _rand(17, (E, F), 0.2)
    exact = ffn_forward(X, W1, W2, act="relu", partition=1, n_slices=n)
    yq = ffn_forward(X, W1, W2, act="relu", partition=1, n_slices=n, quant=True)
    # bound: each partial loses at most d/2 per element (plus float32 rounding)
    bound = np.zeros((B, E))
    for s in range(n):
        fs = slice(s * F // n, (s + 1) * F // n)
        P = relu(X @ W1[fs].T) @ W2[:, fs].T
        _, d = q8_quantize(P.astype(np.float32))
        bound += np.repeat(d.astype(np.float64), 32, axis=-1) * 0.5 + np.abs(P) * 1e-6
    assert np.all(np.abs(yq - exact) <= bound)
    assert np.max(np.abs(yq - exact)) > 0


def test_grid_2d_default():
    assert grid_2d(64) == (8, 8)
    assert grid_2d(4) == (2, 2)
    assert grid_2d(8) == (2, 4)
    assert grid_2d(1) == (1, 1)


@pytest.mark.parametrize("act", ["relu", "swiglu"])
def test_chunked_unsharded_matches_ffn_forward(act):
    import synth
    from oracle import bf16_to_f64, ffn_unsharded_chunked

    s = synth.FfnShape(batch=3, E=64, F=320, dtype="bf16", act=act, n_slices=1, w_std=0.1)
    inp = synth.ffn_inputs(21, s)
    X = bf16_to_f64(inp["X"])
    W3 = inp.get("W3")
    ref = ffn_forward(X, bf16_to_f64(inp["W1"]), bf16_to_f64(inp["W2"]), act=act,
                      W3=bf16_to_f64(W3) if W3 is not None else None)
    got = ffn_unsharded_chunked(X, inp["W1"], inp["W2"], act=act, W3_bits=W3, chunk=96)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)
