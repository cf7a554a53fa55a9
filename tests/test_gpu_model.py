"""Full decode step on the GPU (embedding, every block, final norm, logits) vs the oracle.

distributed-llama task list: the layer loop (llamaNextBlock) followed by
llamaRmsFinal/RmsFinalNorm and the vocab-split llamaLogits whose merge is a
concatenation. Each layer has its own weights and KV cache.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth.device import bf16_tensor, f32_tensor, i32_tensor
from tests.metrics import BF16_TOL, report

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tpb(cuda_ok):
    import tensor_llama_transformer_b200 as t

    return t


def run_model(tpb, s: synth.BlockShape, seed: int, pos, quant: int, n_layers: int,
              sample_rows=None, persistent=None):
    """Builds the model layer by layer on the GPU while the oracle runs the same layers.

    With ``sample_rows`` the GPU runs every batch row but the oracle only the
    sampled ones (rows are independent); the other rows' caches are filled on
    the device with seeded random values. Returns (gpu logits of the oracle's
    rows, oracle logits)."""
    B = len(pos)
    rows = list(range(B)) if sample_rows is None else list(sample_rows)
    emb = synth.normal_bf16(seed, "embed", (s.vocab, s.dim), s.w_std)
    wcls = synth.normal_bf16(seed, "wcls", (s.vocab, s.dim), s.w_std)
    toks = synth.uniform_ids(seed, "tokens", B, s.vocab)
    cache_shape = (n_layers, B, s.n_kv_heads, s.max_seq, s.head_dim)
    kc = torch.empty(cache_shape, dtype=torch.bfloat16, device="cuda")
    vc = torch.empty(cache_shape, dtype=torch.bfloat16, device="cuda")
    if sample_rows is not None:
        g = torch.Generator(device="cuda")
        g.manual_seed(seed)
        for layer in range(n_layers):
            kc[layer].normal_(generator=g)
            vc[layer].normal_(generator=g)
    keep, weights = [], []
    sub = synth.BlockShape(**{**s.__dict__, "batch": len(rows)})

    def make_layer(layer):
        def step(x):
            ones = np.ones(s.dim, dtype=np.float32)
            inp = synth.BlockInputs(
                shape=sub, x=np.zeros((len(rows), s.dim), np.float32), attn_norm=ones,
                ffn_norm=ones.copy(),
                k_cache=np.stack([synth.kv_row(seed, s, "k", b, layer) for b in rows]),
                v_cache=np.stack([synth.kv_row(seed, s, "v", b, layer) for b in rows]),
                pos=np.array([pos[b] for b in rows], dtype=np.int32),
                **synth.block_weights(seed, s, layer))
            for i, b in enumerate(rows):
                kc[layer, b] = bf16_tensor(inp.k_cache[i])
                vc[layer, b] = bf16_tensor(inp.v_cache[i])
            dev = [f32_tensor(inp.attn_norm)] + \
                [bf16_tensor(getattr(inp, k)) for k in ("wq", "wk", "wv", "wo")] + \
                [f32_tensor(inp.ffn_norm)] + [bf16_tensor(getattr(inp, k)) for k in ("w1", "w3", "w2")]
            keep.append(dev)
            weights.append(tpb.make_weights(*dev))
            inp.x = x
            y, _, _ = oracle.block_forward(inp, s.n_slices, bool(quant))
            return y
        return step

    ref = oracle.model_forward(toks[rows], emb, [make_layer(i) for i in range(n_layers)],
                               np.ones(s.dim), wcls, s.n_slices, bool(quant), s.norm_eps)

    dims = tpb.make_dims(s.dim, s.n_heads, s.n_kv_heads, s.head_dim, s.ffn_dim, s.vocab, B,
                         s.max_seq, s.norm_eps, s.rope_theta)
    nbytes = tpb.tp_model_workspace_bytes(dims, n_layers, s.n_slices, 1, quant)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    emb_d, wcls_d = bf16_tensor(emb), bf16_tensor(wcls)
    fn = torch.ones(s.dim, dtype=torch.float32, device="cuda")
    h = tpb.tp_model_create(dims, n_layers, s.n_slices, 1, quant, weights, emb_d, fn, wcls_d, ws,
                            nbytes)
    logits = torch.empty((B, s.vocab), dtype=torch.float32, device="cuda")
    try:
        if persistent is not None:
            tpb.tp_model_set_persistent(h, persistent)
        tpb.tp_model_forward(h, i32_tensor(toks), kc, vc, i32_tensor(np.array(pos)), B, logits)
        torch.cuda.synchronize()
    finally:
        tpb.tp_model_destroy(h)
    return logits.cpu().numpy().astype(np.float64)[rows], ref


SMALL = synth.BlockShape(dim=512, n_heads=4, n_kv_heads=2, head_dim=128, ffn_dim=1024, vocab=1000,
                         max_seq=100, batch=2, n_slices=2, sync_quant=False, pos=99, w_std=0.05)


@pytest.mark.parametrize("quant", [0, 1])
def test_model_small(tpb, quant):
    got, ref = run_model(tpb, SMALL, 3131, [99, 37], quant, n_layers=3)
    r, p = report(f"model small q{quant}", got, ref)
    assert r <= BF16_TOL and p > 0.9999
    assert np.array_equal(np.argmax(got, axis=1), np.argmax(ref, axis=1))


@pytest.mark.slow
def test_model_c3_full_size_batch1(tpb):
    """Llama-2-7B shapes, 32 layers, context 4096 (decode at position 4095), n = 8 slices."""
    s = synth.C3
    got, ref = run_model(tpb, s, synth.CONFIG_SEED["C3"], [s.pos], 0, n_layers=s.n_layers)
    r, p = report("model C3 32 layers", got, ref)
    assert r <= BF16_TOL and p > 0.9999


@pytest.mark.slow
def test_model_c3_full_size_batch16_sampled(tpb):
    """32 layers, context 4096, batch 16 on the GPU; the oracle checks rows 0 and 11."""
    s = synth.BlockShape(**{**synth.C3.__dict__, "batch": 16})
    pos = [s.pos] * 16
    got, ref = run_model(tpb, s, synth.CONFIG_SEED["C3"], pos, 0, n_layers=s.n_layers,
                         sample_rows=[0, 11])
    r, p = report("model C3 32 layers batch 16 (rows 0, 11)", got, ref)
    assert r <= BF16_TOL and p > 0.9999
