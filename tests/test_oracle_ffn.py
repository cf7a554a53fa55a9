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


# ---------------------------------------------------------------------------
# 2D partition with Q8 sync buffers (Pope et al. demo1's 2D weight-stationary
# layout with the distributed-llama Quantize/Dequantize around every exchange)
# ---------------------------------------------------------------------------

def _q8_trip(P):
    """The sync round trip of one partial (q8_quantize / q8_dequantize are pinned in
    test_oracle_q8.py): float32, codes per 32 values along the last axis, back."""
    from oracle import q8_dequantize

    q, d = q8_quantize(np.asarray(P, dtype=np.float32))
    return q8_dequantize(q, d).astype(np.float64)


def _loop_ffn_2d_q8(X, W1, W2, gx, gy, act, W3=None):
    """Plain loops over the gx x gy grid: every stage-1 partial (one per (x, y) cell,
    summed over x) and every stage-2 partial (one per cell, summed over y) crosses
    its own quantised sync."""
    B, E = X.shape
    F = W1.shape[0]
    ex, fy = E // gx, F // gy
    H = np.zeros((B, F))
    for y in range(gy):
        a = np.zeros((B, fy))
        c = np.zeros((B, fy))
        for x in range(gx):
            p1 = np.zeros((B, fy))
            p3 = np.zeros((B, fy))
            for b in range(B):
                for f in range(fy):
                    p1[b, f] = sum(X[b, x * ex + e] * W1[y * fy + f, x * ex + e] for e in range(ex))
                    if W3 is not None:
                        p3[b, f] = sum(X[b, x * ex + e] * W3[y * fy + f, x * ex + e]
                                       for e in range(ex))
            a = a + _q8_trip(p1)
            if W3 is not None:
                c = c + _q8_trip(p3)
        for b in range(B):
            for f in range(fy):
                z = a[b, f]
                H[b, y * fy + f] = max(z, 0.0) if act == "relu" else z / (1.0 + np.exp(-z)) * c[b, f]
    Y = np.zeros((B, E))
    for x in range(gx):
        acc = np.zeros((B, ex))
        for y in range(gy):
            p2 = np.zeros((B, ex))
            for b in range(B):
                for e in range(ex):
                    p2[b, e] = sum(H[b, y * fy + f] * W2[x * ex + e, y * fy + f] for f in range(fy))
            acc = acc + _q8_trip(p2)
        Y[:, x * ex:(x + 1) * ex] = acc
    return Y


@pytest.mark.parametrize("act", ["relu", "swiglu"])
@pytest.mark.parametrize("grid", [(2, 2), (2, 1), (1, 2)])
def test_quantised_2d_loop_restatement(act, grid):
    gx, gy = grid
    B, E, F = 2, 64, 128
    X, W1, W2 = _rand(31, (B, E)), _rand(32, (F, E), 0.2), _rand(33, (E, F), 0.2)
    W3 = _rand(34, (F, E), 0.2) if act == "swiglu" else None
    ref = _loop_ffn_2d_q8(X, W1, W2, gx, gy, act, W3)
    y = ffn_forward(X, W1, W2, act=act, W3=W3, partition=2, n_slices=gx * gy, grid=grid,
                    quant=True)
    scale = np.max(np.abs(ref))
    assert np.max(np.abs(y - ref)) <= 1e-12 * scale


def test_quantised_2d_quantises_every_cell():
    """The same grid quantising once after each sum over x (stage 1) or y (stage 2),
    instead of every cell's partial, gives a different layer: the loop restatement
    above tells the two apart."""
    B, E, F, gx, gy = 2, 64, 128, 2, 2
    X, W1, W2 = _rand(35, (B, E)), _rand(36, (F, E), 0.2), _rand(37, (E, F), 0.2)
    ex, fy = E // gx, F // gy
    H = np.zeros((B, F))
    for y in range(gy):
        fs = slice(y * fy, (y + 1) * fy)
        H[:, fs] = relu(_q8_trip(X @ W1[fs].T))
    Y = np.zeros((B, E))
    for x in range(gx):
        es = slice(x * ex, (x + 1) * ex)
        Y[:, es] = _q8_trip(H @ W2[es].T)
    y = ffn_forward(X, W1, W2, act="relu", partition=2, n_slices=4, grid=(gx, gy), quant=True)
    assert np.max(np.abs(y - Y)) > 1e-6 * np.max(np.abs(Y))
    np.testing.assert_allclose(y, _loop_ffn_2d_q8(X, W1, W2, gx, gy, "relu"), rtol=0,
                               atol=1e-12 * np.max(np.abs(y)))


@pytest.mark.parametrize("grid", [(2, 2), (4, 2), (2, 4)])
def test_quantised_2d_within_bound(grid):
    """Every quantised sync moves a value by at most half its block's scale d (plus
    float32 rounding). Stage 1: |A_q - A| <= sum_x d_xy / 2; ReLU is 1-Lipschitz, so
    H moves by no more; stage 2 carries that through |W2| and adds each cell's own
    d / 2, whose block scale is at most (block max of |P2| + its carried error) / 127."""
    gx, gy = grid
    B, E, F = 4, 128, 256
    X, W1, W2 = _rand(38, (B, E)), _rand(39, (F, E), 0.15), _rand(40, (E, F), 0.15)
    ex, fy = E // gx, F // gy
    exact = ffn_forward(X, W1, W2, act="relu", partition=2, n_slices=gx * gy, grid=grid)
    yq = ffn_forward(X, W1, W2, act="relu", partition=2, n_slices=gx * gy, grid=grid, quant=True)
    rnd = 2.0 ** -23
    eA = np.zeros((B, F))
    H = np.zeros((B, F))
    for y in range(gy):
        fs = slice(y * fy, (y + 1) * fy)
        A = np.zeros((B, fy))
        for x in range(gx):
            P = X[:, x * ex:(x + 1) * ex] @ W1[fs, x * ex:(x + 1) * ex].T
            _, d = q8_quantize(P.astype(np.float32))
            dd = np.repeat(d.astype(np.float64), 32, axis=-1)
            eA[:, fs] += dd * 0.5 + rnd * (np.abs(P) + dd)
            A += P
        H[:, fs] = relu(A)
    bound = np.zeros((B, E))
    for x in range(gx):
        es = slice(x * ex, (x + 1) * ex)
        for y in range(gy):
            fs = slice(y * fy, (y + 1) * fy)
            P2 = H[:, fs] @ W2[es, fs].T
            e2 = eA[:, fs] @ np.abs(W2[es, fs]).T
            hi = np.abs(P2) + e2
            dmax = hi.reshape(B, -1, 32).max(axis=-1) / 127.0 * (1 + 4 * rnd)
            dd = np.repeat(dmax, 32, axis=-1)
            bound[:, es] += e2 + dd * 0.5 + rnd * (hi + dd)
    diff = np.abs(yq - exact)
    assert np.all(diff <= bound)
    assert np.max(diff) > 0
