"""Rows that share a cache sequence (tp_block_forward_seq) on the GPU versus the oracle.

A prefill chunk is several consecutive tokens of one sequence in one step (Pope
et al. demo 2's prefill regime); a mixed step holds decode rows of some
sequences and a chunk of another. Every row's k/v are written before any row's
attention, so each row attends causally. Checked against
``oracle.block_forward(seq=...)`` (itself pinned to token-by-token decode and to
the masked-softmax form of causal attention), on the weight-streaming path
(up to 5 rows) and the tensor-core path (6 or more), at the 7B block's shapes for
a 64-token chunk, and through the model entry point; prompts longer than the
handle's max_batch run as successive passes inside one call.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth.device import DeviceBlock, bf16_tensor, f32_tensor, i32_tensor, to_bits
from tests.metrics import BF16_TOL, assert_q8_codes_exact, report
from tests.test_gpu_block import TIGHT, TIGHT_Q8, _dims

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tpb(cuda_ok):
    import tensor_llama_transformer_b200 as t

    return t


def run_seq(tpb, inp, n, quant, max_batch=None):
    s = inp.shape
    B = inp.x.shape[0]
    mb = max_batch or B
    dev = DeviceBlock(inp, max_batch=mb)
    dims = _dims(tpb, s, mb)
    nbytes = tpb.tp_block_workspace_bytes(dims, n, 1, quant)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    h = tpb.tp_block_create(dims, n, 1, quant, tpb.make_weights(*dev.weights()), ws, nbytes)
    try:
        tpb.tp_block_forward_seq(h, dev.x, dev.k_cache, dev.v_cache, dev.pos, dev.seq,
                                 dev.k_cache.shape[0], B)
        torch.cuda.synchronize()
        off, _ = tpb.tp_block_buffer(h, 7)
        err = int(ws[off:off + 4].view(torch.int32).item())
        norm = {}
        for key, which, dt in (("xn", tpb.BUF_XN, torch.float32), ("xq", tpb.BUF_XQ, torch.int8),
                               ("xd", tpb.BUF_XD, torch.float32)):
            o, size = tpb.tp_block_buffer(h, which)
            norm[key] = ws[o:o + size].view(dt).cpu().numpy()
    finally:
        tpb.tp_block_destroy(h)
    seq, pos = inp.extra["seq"], inp.pos
    kb, vb = to_bits(dev.k_cache), to_bits(dev.v_cache)
    k_rows = np.stack([kb[seq[b], :, pos[b], :] for b in range(B)])
    v_rows = np.stack([vb[seq[b], :, pos[b], :] for b in range(B)])
    return dev.x.cpu().numpy().astype(np.float64), k_rows, v_rows, err, norm


def check_seq(tpb, inp, n, quant, tight, name):
    tr = {}
    ref, k_ref, v_ref = oracle.block_forward(inp, n, bool(quant), seq=inp.extra["seq"], trace=tr)
    y, k_rows, v_rows, err, norm = run_seq(tpb, inp, n, quant)
    assert err == 0, "a bounded wait in a kernel gave up"
    r_out, p_out = report(f"{name} out", y, ref)
    r_dx, _ = report(f"{name} out-x", y - inp.x, ref - inp.x)
    r_k, _ = report(f"{name} k@pos", oracle.bf16_to_f64(k_rows), oracle.bf16_to_f64(k_ref))
    r_v, _ = report(f"{name} v@pos", oracle.bf16_to_f64(v_rows), oracle.bf16_to_f64(v_ref))
    for r in (r_out, r_dx, r_k, r_v):
        assert r <= BF16_TOL
    assert max(r_out, r_dx) <= tight, "regression against the expected error level"
    assert p_out > 0.9999
    # the FFN RMSNorm (+Q8) of every row: float32 output against the oracle's, codes
    # bit-exact against the oracle's Q8 of the kernel's own float32 rows
    B, D = inp.x.shape
    xn_ref = oracle.rmsnorm(tr["x1"], inp.ffn_norm, inp.shape.norm_eps)
    r_xn, _ = report(f"{name} xnorm(ffn)", norm["xn"][:B * D].reshape(B, D), xn_ref)
    assert r_xn <= tight
    if quant:
        assert_q8_codes_exact(norm["xn"], norm["xq"], norm["xd"], B, D, f"{name} xnorm(ffn)")
    return y


MHA = synth.BlockShape(dim=256, n_heads=4, n_kv_heads=4, head_dim=128, ffn_dim=512, vocab=0,
                       max_seq=300, batch=1, n_slices=2, sync_quant=False, pos=100, w_std=0.05)
GQA = synth.BlockShape(dim=512, n_heads=8, n_kv_heads=2, head_dim=128, ffn_dim=1024, vocab=0,
                       max_seq=200, batch=1, n_slices=2, sync_quant=False, pos=63, w_std=0.04)


@pytest.mark.parametrize("quant", [0, 1])
@pytest.mark.parametrize("shape,p0,L", [
    (MHA, 100, 4),    # weight-streaming path, chunk inside a tile
    (GQA, 62, 5),     # crosses the 64-position tile boundary
    (MHA, 0, 16),     # a prompt's first chunk: no cached prefix
    (GQA, 63, 37),    # tensor-core path, ragged length
    (MHA, 200, 64),   # the largest chunk (max_batch)
])
def test_prefill_chunk(tpb, shape, p0, L, quant):
    s = synth.BlockShape(**{**shape.__dict__, "pos": p0})  # cached prefix: positions < p0
    inp = synth.chunk_inputs(8181, s, p0 + np.arange(L), np.zeros(L, dtype=np.int32))
    tight = (TIGHT_Q8 if quant else TIGHT) if L <= 5 else 1e-2
    check_seq(tpb, inp, shape.n_slices, quant, tight, f"prefill d{s.dim} p0 {p0} L{L} q{quant}")


@pytest.mark.parametrize("quant", [0, 1])
@pytest.mark.parametrize("seq,pos", [
    ([2, 0, 2, 1, 2], [100, 150, 101, 7, 102]),                       # 5 rows: ring path
    ([1, 1, 1, 0, 3, 1, 2, 1], [60, 61, 62, 299, 0, 63, 140, 64]),   # 8 rows: tensor cores
])
def test_mixed_decode_and_prefill(tpb, seq, pos, quant):
    s = synth.BlockShape(**{**MHA.__dict__, "pos": 60})
    inp = synth.chunk_inputs(8282, s, pos, seq)
    tight = (TIGHT_Q8 if quant else TIGHT) if len(pos) <= 5 else 1e-2
    check_seq(tpb, inp, 2, quant, tight, f"mixed B{len(pos)} q{quant}")


@pytest.mark.parametrize("quant", [0, 1])
def test_prompt_longer_than_max_batch(tpb, quant):
    """37 tokens of one sequence through a block built for 16 rows: passes of 16, 16 and 5
    rows (tensor-core path, then the weight-streaming path), each attending to the cache
    rows the earlier passes wrote."""
    s = synth.BlockShape(**{**GQA.__dict__, "pos": 40})
    L, mb = 37, 16
    inp = synth.chunk_inputs(8585, s, 40 + np.arange(L), np.zeros(L, dtype=np.int32))
    ref, k_ref, v_ref = oracle.block_forward(inp, 2, bool(quant), seq=inp.extra["seq"])
    y, k_rows, v_rows, err, _ = run_seq(tpb, inp, 2, quant, max_batch=mb)
    assert err == 0, "a bounded wait in a kernel gave up"
    name = f"prompt L{L} in passes of {mb} q{quant}"
    r_out, p_out = report(f"{name} out", y, ref)
    r_dx, _ = report(f"{name} out-x", y - inp.x, ref - inp.x)
    r_k, _ = report(f"{name} k@pos", oracle.bf16_to_f64(k_rows), oracle.bf16_to_f64(k_ref))
    r_v, _ = report(f"{name} v@pos", oracle.bf16_to_f64(v_rows), oracle.bf16_to_f64(v_ref))
    for r in (r_out, r_dx, r_k, r_v):
        assert r <= BF16_TOL
    assert max(r_out, r_dx) <= 1e-2 and p_out > 0.9999


def test_prefill_chunk_equals_token_by_token(tpb):
    """The GPU's chunk against the GPU decoding the same tokens one per call."""
    s = synth.BlockShape(**{**GQA.__dict__, "pos": 30})
    L = 8
    inp = synth.chunk_inputs(8383, s, 30 + np.arange(L), np.zeros(L, dtype=np.int32))
    y_chunk = run_seq(tpb, inp, 2, 1)[0]
    dev = DeviceBlock(inp, max_batch=L)
    dims = _dims(tpb, s, L)
    nbytes = tpb.tp_block_workspace_bytes(dims, 2, 1, 1)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    h = tpb.tp_block_create(dims, 2, 1, 1, tpb.make_weights(*dev.weights()), ws, nbytes)
    try:
        for t in range(L):
            tpb.tp_block_forward_seq(h, dev.x[t:t + 1], dev.k_cache, dev.v_cache, dev.pos[t:t + 1],
                                     dev.seq[t:t + 1], dev.k_cache.shape[0], 1)
        torch.cuda.synchronize()
    finally:
        tpb.tp_block_destroy(h)
    y_tok = dev.x.cpu().numpy().astype(np.float64)
    r, _ = report("chunk vs token by token", y_chunk - inp.x, y_tok - inp.x)
    assert r <= 1e-2  # tensor-core chunk (bf16 operand pairs) vs weight-streaming rows


def test_prefill_chunk_c2_shapes(tpb):
    """A 64-token chunk of the 7B block (n = 4, Q8 sync) after a 960-token prefix."""
    s = synth.BlockShape(**{**synth.C2.__dict__, "pos": 960})
    inp = synth.chunk_inputs(synth.CONFIG_SEED["C2"], s, 960 + np.arange(64),
                             np.zeros(64, dtype=np.int32))
    check_seq(tpb, inp, s.n_slices, 1, 1e-2, "prefill C2 L64")


@pytest.mark.parametrize("mb", [12, 5])
def test_model_prefill_chunk(tpb, mb):
    """tp_model_forward_seq: a 12-token chunk through 2 layers, embedding to logits; with
    max_batch 5 the call runs as passes of 5, 5 and 2 rows through every layer."""
    s = synth.BlockShape(dim=512, n_heads=4, n_kv_heads=2, head_dim=128, ffn_dim=1024, vocab=1000,
                         max_seq=100, batch=1, n_slices=2, sync_quant=False, pos=40, w_std=0.05)
    L, n_layers, seed = 12, 2, 8484
    pos = 40 + np.arange(L, dtype=np.int32)
    seq = np.zeros(L, dtype=np.int32)
    emb = synth.normal_bf16(seed, "embed", (s.vocab, s.dim), s.w_std)
    wcls = synth.normal_bf16(seed, "wcls", (s.vocab, s.dim), s.w_std)
    toks = synth.uniform_ids(seed, "tokens", L, s.vocab)
    kc = torch.zeros((n_layers, 1, s.n_kv_heads, s.max_seq, s.head_dim), dtype=torch.bfloat16,
                     device="cuda")
    vc = torch.zeros_like(kc)
    keep, weights = [], []

    def make_layer(layer):
        def step(x):
            inp = synth.chunk_inputs(seed, s, pos, seq, layer=layer)
            kc[layer] = bf16_tensor(inp.k_cache)
            vc[layer] = bf16_tensor(inp.v_cache)
            dev = [f32_tensor(inp.attn_norm)] + \
                [bf16_tensor(getattr(inp, k)) for k in ("wq", "wk", "wv", "wo")] + \
                [f32_tensor(inp.ffn_norm)] + [bf16_tensor(getattr(inp, k)) for k in ("w1", "w3", "w2")]
            keep.append(dev)
            weights.append(tpb.make_weights(*dev))
            inp.x = x
            return oracle.block_forward(inp, s.n_slices, False, seq=seq)[0]
        return step

    ref = oracle.model_forward(toks, emb, [make_layer(i) for i in range(n_layers)], np.ones(s.dim),
                               wcls, s.n_slices, False, s.norm_eps)
    dims = tpb.make_dims(s.dim, s.n_heads, s.n_kv_heads, s.head_dim, s.ffn_dim, s.vocab, mb,
                         s.max_seq, s.norm_eps, s.rope_theta)
    nbytes = tpb.tp_model_workspace_bytes(dims, n_layers, s.n_slices, 1, 0)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    # the handle borrows these pointers: keep the tensors alive until it is destroyed
    emb_d, wcls_d = bf16_tensor(emb), bf16_tensor(wcls)
    fn = torch.ones(s.dim, dtype=torch.float32, device="cuda")
    h = tpb.tp_model_create(dims, n_layers, s.n_slices, 1, 0, weights, emb_d, fn, wcls_d, ws, nbytes)
    logits = torch.empty((L, s.vocab), dtype=torch.float32, device="cuda")
    try:
        tpb.tp_model_forward_seq(h, i32_tensor(toks), kc, vc, i32_tensor(pos), i32_tensor(seq), 1, L,
                                 logits)
        torch.cuda.synchronize()
    finally:
        tpb.tp_model_destroy(h)
    got = logits.cpu().numpy().astype(np.float64)
    r, p = report("model prefill chunk", got, ref)
    assert r <= BF16_TOL and p > 0.9999
    assert np.array_equal(np.argmax(got, axis=1), np.argmax(ref, axis=1))
