"""Partitioned FFN on the GPU through the C ABI versus the float64 oracle.

float32 (the ggmlR-shaped two-stage ReLU FFN, 1e-5) on CUDA cores; bf16 on the
tcgen05 tensor-core contraction (2e-2), in 1D and 2D partitions, with every
slice's partial formed on its own and summed in slice order (faithful merge:
in the GEMM's epilogue, or through partial planes for the 2D SwiGLU first
stage) or accumulated in the contraction (fused merge), ReLU and SwiGLU, with
and without Q8 sync of the partials; bit-exact on integer-valued inputs.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth.device import bf16_tensor, f32_tensor
from tests.metrics import BF16_TOL, report

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tpb(cuda_ok):
    import tensor_llama_transformer_b200 as t

    return t


def run_ffn(tpb, s: synth.FfnShape, inputs, partition, merge, quant=False):
    up = f32_tensor if s.dtype == "f32" else bf16_tensor
    X, W1, W2 = up(inputs["X"]), up(inputs["W1"]), up(inputs["W2"])
    W3 = up(inputs["W3"]) if "W3" in inputs else None
    B = inputs["X"].shape[0]
    gx, gy = (s.grid_x, s.grid_y) if partition == 2 else (1, 1)
    desc = tpb.tp_ffn_desc(B, s.E, s.F, tpb.TP_F32 if s.dtype == "f32" else tpb.TP_BF16,
                           tpb.TP_ACT_RELU if s.act == "relu" else tpb.TP_ACT_SWIGLU, partition,
                           s.n_slices, gx, gy, int(quant), merge)
    nbytes = tpb.tp_ffn_workspace_bytes(desc)
    ws = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device="cuda")
    Y = torch.full((B, s.E), float("nan"), dtype=torch.float32, device="cuda")
    tpb.tp_ffn_forward(desc, X, W1, W3, W2, Y, ws, nbytes)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0, "a bounded wait in a kernel gave up"
    return Y.cpu().numpy().astype(np.float64)


def _ref(s, inputs, partition, quant):
    cv = (lambda a: a.astype(np.float64)) if s.dtype == "f32" else oracle.bf16_to_f64
    X, W1, W2 = cv(inputs["X"]), cv(inputs["W1"]), cv(inputs["W2"])
    W3 = cv(inputs["W3"]) if "W3" in inputs else None
    return oracle.ffn_forward(X, W1, W2, act=s.act, W3=W3, partition=partition,
                              n_slices=s.n_slices, grid=(s.grid_x, s.grid_y), quant=quant)


@pytest.mark.parametrize("partition", [1, 2])
@pytest.mark.parametrize("quant", [False, True])
def test_c1_fp32(tpb, partition, quant):
    s = synth.C1 if partition == 1 else synth.FfnShape(**{**synth.C1.__dict__, "grid_x": 1,
                                                          "grid_y": 2, "partition": 2})
    inputs = synth.ffn_inputs(synth.CONFIG_SEED["C1"], s)
    y = run_ffn(tpb, s, inputs, partition, tpb.TP_MERGE_FAITHFUL, quant)
    ref = _ref(s, inputs, partition, quant)
    r, p = report(f"C1 fp32 part{partition} q{int(quant)}", y, ref)
    # quantised partials: the float32 and float64 partials can straddle a code
    # boundary, so the quantised case is held to the quantisation step instead
    assert r <= (1e-5 if not quant else 1e-2)
    if not quant:
        unsharded = np.maximum(inputs["X"].astype(np.float64) @ inputs["W1"].T.astype(np.float64), 0) \
            @ inputs["W2"].T.astype(np.float64)
        assert np.max(np.abs(y - unsharded)) / np.max(np.abs(unsharded)) <= 1e-5


SMALL_BF16 = synth.FfnShape(batch=200, E=512, F=1024, dtype="bf16", act="relu", n_slices=4,
                            grid_x=2, grid_y=2, x_std=1.0, w_std=0.05)


@pytest.mark.parametrize("act", ["relu", "swiglu"])
@pytest.mark.parametrize("partition,merge,quant", [
    (1, 0, False), (1, 1, False), (2, 0, False), (1, 0, True), (2, 0, True)])
def test_bf16_small(tpb, act, partition, merge, quant):
    s = synth.FfnShape(**{**SMALL_BF16.__dict__, "act": act})
    inputs = synth.ffn_inputs(5151, s)
    y = run_ffn(tpb, s, inputs, partition, merge, quant)
    ref = _ref(s, inputs, partition, quant)
    r, p = report(f"bf16 {act} part{partition} merge{merge} q{int(quant)}", y, ref)
    assert r <= BF16_TOL
    assert p > 0.9999


@pytest.mark.parametrize("M", [1, 127, 128, 129, 384])
def test_bf16_m_tails(tpb, M):
    s = synth.FfnShape(batch=M, E=256, F=768, dtype="bf16", act="relu", n_slices=3,
                       x_std=1.0, w_std=0.06)
    inputs = synth.ffn_inputs(6161 + M, s)
    for merge in (0, 1):
        y = run_ffn(tpb, s, inputs, 1, merge)
        r, _ = report(f"bf16 M={M} merge{merge}", y, _ref(s, inputs, 1, False))
        assert r <= BF16_TOL


def _int_bf16(a):
    """bf16 bits of small integers (exact: they need at most 8 significant bits)."""
    a = np.asarray(a, dtype=np.float32)
    assert np.all(np.abs(a) <= 256)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


@pytest.mark.parametrize("partition,quant", [(1, False), (1, True), (2, False)])
def test_bf16_faithful_bit_exact_on_integers(tpb, partition, quant):
    """Integer-valued X, W1, W2 make every partial an exact integer in float32, so the
    faithful form's output is fixed bit for bit: the float32 sum, in slice order, of
    each slice's partial after the sync (oracle.sync_buffer: the Q8 round trip when
    quantising). The quantised 1D case checks the order and the per-partial rounding:
    a sum in another order, or a Q8 round trip of the sum instead of each partial,
    changes low bits. B = 130 and E = 320, F = 480 leave partial M and N tiles."""
    rng = np.random.default_rng(2024 + partition + 10 * quant)
    B, E, F = 130, 320, 480
    n, (gx, gy) = 3, (2, 3)
    X = rng.integers(-1, 2, (B, E)).astype(np.float64)
    W1 = rng.integers(-1, 2, (F, E)).astype(np.float64)
    W2 = rng.integers(-1, 2, (E, F)).astype(np.float64)
    H = np.maximum(X @ W1.T, 0.0)
    assert H.max() <= 256  # every hidden value an exact bf16
    Y32 = np.zeros((B, E), dtype=np.float32)
    if partition == 1:
        for s in range(n):
            fs = oracle.slice_range(F, n, s)
            P = H[:, fs] @ W2[:, fs].T
            Y32 = (Y32 + oracle.sync_buffer(P, quant).astype(np.float32)).astype(np.float32)
    else:  # integer partials without quantisation: every sum exact
        Y32 = (H @ W2.T).astype(np.float32)
        assert np.all(np.abs(H @ W2.T) < 2 ** 24)
    desc = tpb.tp_ffn_desc(B, E, F, tpb.TP_BF16, tpb.TP_ACT_RELU, partition, n, gx, gy, int(quant),
                           tpb.TP_MERGE_FAITHFUL)
    nbytes = tpb.tp_ffn_workspace_bytes(desc)
    ws = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device="cuda")
    Y = torch.full((B, E), float("nan"), dtype=torch.float32, device="cuda")
    tpb.tp_ffn_forward(desc, bf16_tensor(_int_bf16(X)), bf16_tensor(_int_bf16(W1)), None,
                       bf16_tensor(_int_bf16(W2)), Y, ws, nbytes)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    got = Y.cpu().numpy()
    bad = np.argwhere(got.view(np.uint32) != Y32.view(np.uint32))
    assert bad.size == 0, f"{len(bad)} values differ, first at {bad[0]}: {got[tuple(bad[0])]!r} " \
                          f"vs {Y32[tuple(bad[0])]!r}"
    if quant:  # the quantised sum must differ from the exact one somewhere (the test has teeth)
        assert np.any(Y32 != (H @ W2.T).astype(np.float32))
    print(f"[parity] faithful FFN part{partition} q{int(quant)} on integers: bit-exact")


@pytest.mark.parametrize("partition", [1, 2])
def test_bf16_faithful_n_tails(tpb, partition):
    """Feature and model dims that leave partial 128-column tiles (E 320, F 480) in
    both stages, with Q8, SwiGLU and ReLU, against the oracle."""
    for act in ("relu", "swiglu"):
        s = synth.FfnShape(batch=130, E=320, F=480, dtype="bf16", act=act, n_slices=3, grid_x=2,
                           grid_y=3, x_std=1.0, w_std=0.06)
        inputs = synth.ffn_inputs(7272 + partition, s)
        for quant in (False, True):
            y = run_ffn(tpb, s, inputs, partition, tpb.TP_MERGE_FAITHFUL, quant)
            r, p = report(f"bf16 {act} part{partition} q{int(quant)} E320 F480", y,
                          _ref(s, inputs, partition, quant))
            assert r <= BF16_TOL and p > 0.9999


@pytest.fixture(scope="module")
def c5_weights(cuda_ok):
    """PaLM-shaped FFN weights (E 18432, F 73728), generated once for the C5 cases."""
    s = synth.C5
    seed = synth.CONFIG_SEED["C5"]
    W1 = synth.normal_bf16(seed, "W1", (s.F, s.E), s.w_std)
    W2 = synth.normal_bf16(seed, "W2", (s.E, s.F), s.w_std)
    return W1, W2, bf16_tensor(W1), bf16_tensor(W2)


@pytest.mark.slow
@pytest.mark.parametrize("B,forms", [(512, ("fused", "1d", "2d")), (2048, ("fused", "2d")),
                                     (8192, ("fused",))])
def test_c5_full_size_sampled_rows(tpb, c5_weights, B, forms):
    """Full PaLM FFN on the GPU; the oracle checks 8 token rows spread over the M tiles."""
    W1, W2, W1d, W2d = c5_weights
    s = synth.FfnShape(**{**synth.C5.__dict__, "batch": B})
    seed = synth.CONFIG_SEED["C5"]
    X = synth.normal_bf16(seed, f"X{B}", (B, s.E), s.x_std)
    Xd = bf16_tensor(X)
    rows = np.unique(np.array([0, 1, 127, 128, B // 3, B // 2, B - 2, B - 1]))
    ref = oracle.ffn_unsharded_chunked(oracle.bf16_to_f64(X[rows]), W1, W2, chunk=2048)
    for form in forms:
        part, merge = {"fused": (1, 1), "1d": (1, 0), "2d": (2, 0)}[form]
        gx, gy = (8, 8) if part == 2 else (1, 1)
        desc = tpb.tp_ffn_desc(B, s.E, s.F, tpb.TP_BF16, tpb.TP_ACT_RELU, part, 64, gx, gy, 0, merge)
        nb = tpb.tp_ffn_workspace_bytes(desc)
        ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
        Y = torch.full((B, s.E), float("nan"), dtype=torch.float32, device="cuda")
        tpb.tp_ffn_forward(desc, Xd, W1d, None, W2d, Y, ws, nb)
        torch.cuda.synchronize()
        assert int(ws[:4].view(torch.int32).item()) == 0
        y = Y[torch.from_numpy(rows).cuda()].cpu().numpy().astype(np.float64)
        r, p = report(f"C5 B={B} {form}", y, ref)
        assert r <= BF16_TOL and p > 0.9999
        assert torch.isfinite(Y).all()
        del ws, Y
        torch.cuda.empty_cache()
