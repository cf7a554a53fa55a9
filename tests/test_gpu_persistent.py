"""The persistent block kernel (batch 1-2, one launch per block) versus the oracle.

The same decoder-block forward as tests/test_gpu_block.py (distributed-llama
issue #29 task list, per-slice partials merged in slice order with the optional
Q8 sync), run as one cooperative kernel whose phases are separated by grid
barriers. Besides parity on ragged and degenerate contexts, these tests check
what only this kernel has: its counters return to zero so a handle can run
again, and the phase trace is written in order.
"""
import numpy as np
import pytest
import torch

import synth
from synth.device import DeviceBlock
from tests.metrics import BF16_TOL, report
from tests.test_gpu_block import TIGHT, TIGHT_Q8, _dims, check_block
from tests.test_gpu_model import SMALL as SMALL_MODEL
from tests.test_gpu_model import run_model

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tpb(cuda_ok):
    import tensor_llama_transformer_b200 as t

    return t


MHA = synth.BlockShape(dim=256, n_heads=2, n_kv_heads=2, head_dim=128, ffn_dim=512, vocab=0,
                       max_seq=300, batch=2, n_slices=2, sync_quant=False, pos=299, w_std=0.05)
GQA4 = synth.BlockShape(dim=512, n_heads=8, n_kv_heads=2, head_dim=128, ffn_dim=1024, vocab=0,
                        max_seq=260, batch=2, n_slices=2, sync_quant=False, pos=259, w_std=0.04)
GQA8 = synth.BlockShape(dim=1024, n_heads=8, n_kv_heads=1, head_dim=128, ffn_dim=2048, vocab=0,
                        max_seq=129, batch=1, n_slices=1, sync_quant=False, pos=128, w_std=0.03)
N8 = synth.BlockShape(dim=1024, n_heads=8, n_kv_heads=8, head_dim=128, ffn_dim=2048, vocab=0,
                      max_seq=700, batch=2, n_slices=8, sync_quant=False, pos=699, w_std=0.03)


@pytest.mark.parametrize("quant", [0, 1])
@pytest.mark.parametrize("shape,pos", [
    (MHA, [299]),            # batch 1: 5 tiles of 64, the last one ragged
    (MHA, [130, 0]),         # batch 2: 3 tiles, and a context of one position
    (GQA4, [259, 127]),      # GQA group of 4
    (GQA8, [128]),           # GQA group of 8, one slice
    (N8, [699, 64]),         # 8 slices; a context ending exactly on a tile boundary + 1
])
def test_persistent_small(tpb, shape, pos, quant):
    s = synth.BlockShape(**{**shape.__dict__, "batch": len(pos)})
    inp = synth.block_inputs(5151, s)
    inp.pos[:] = pos
    check_block(tpb, inp, s.n_slices, quant, tight=TIGHT_Q8 if quant else TIGHT,
                name=f"persistent d{s.dim} H{s.n_heads}/{s.n_kv_heads} n{s.n_slices} B{len(pos)} q{quant}",
                persistent=1)


def test_persistent_c2_full_size(tpb):
    """The bench's block (Llama-2-7B shapes, n=4, Q8 sync, KV 1024, batch 1)."""
    inp = synth.block_inputs(synth.CONFIG_SEED["C2"], synth.C2)
    check_block(tpb, inp, synth.C2.n_slices, 1, tight=TIGHT_Q8, name="persistent C2", persistent=1)


def test_persistent_runs_again(tpb):
    """Two forwards on one handle from the same state give the same bits: the grid
    barrier and split counters are back at zero after each launch."""
    s = synth.BlockShape(**{**N8.__dict__, "batch": 2})
    inp = synth.block_inputs(77, s)
    dev = DeviceBlock(inp, max_batch=2)
    dims = _dims(tpb, s, 2)
    nbytes = tpb.tp_block_workspace_bytes(dims, s.n_slices, 1, 1)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    h = tpb.tp_block_create(dims, s.n_slices, 1, 1, tpb.make_weights(*dev.weights()), ws, nbytes)
    x0, k0, v0 = dev.x.clone(), dev.k_cache.clone(), dev.v_cache.clone()
    outs = []
    try:
        tpb.tp_block_set_persistent(h, 1)
        for _ in range(3):
            dev.x.copy_(x0)
            dev.k_cache.copy_(k0)
            dev.v_cache.copy_(v0)
            tpb.tp_block_forward(h, dev.x, dev.k_cache, dev.v_cache, dev.pos, 2)
            torch.cuda.synchronize()
            outs.append(dev.x.clone())
        off, _ = tpb.tp_block_buffer(h, 7)
        words = ws[off:off + 16].view(torch.int32).cpu().numpy()
    finally:
        tpb.tp_block_destroy(h)
    assert words[0] == 0, "a bounded wait gave up"
    assert words[2] == 0 and words[3] == 0, "grid barrier counters not reset"
    for o in outs[1:]:
        assert torch.equal(o, outs[0])


def test_persistent_trace(tpb):
    """Phase stamps are written by every CTA and are ordered within each CTA."""
    s = synth.BlockShape(**{**MHA.__dict__, "batch": 1})
    inp = synth.block_inputs(12, s)
    dev = DeviceBlock(inp, max_batch=1)
    dims = _dims(tpb, s, 1)
    nbytes = tpb.tp_block_workspace_bytes(dims, s.n_slices, 1, 0)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    h = tpb.tp_block_create(dims, s.n_slices, 1, 0, tpb.make_weights(*dev.weights()), ws, nbytes)
    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    tr = torch.zeros(nsm * tpb.TP_BLOCK_TRACE_SLOTS, dtype=torch.int64, device="cuda")
    try:
        tpb.tp_block_set_persistent(h, 1)
        tpb.tp_block_set_trace(h, tr, tr.numel() * 8)
        tpb.tp_block_forward(h, dev.x, dev.k_cache, dev.v_cache, dev.pos, 1)
        torch.cuda.synchronize()
    finally:
        tpb.tp_block_destroy(h)
    t = tr.view(nsm, -1).cpu().numpy()
    used = t[:, 0] != 0
    assert used.sum() >= 1
    order = [0, 1, 2, 3, 4, 5, 6, 13, 14, 7, 8, 9, 10, 11]  # start, phases and barriers in order
    for row in t[used]:
        seq = row[order]
        assert np.all(np.diff(seq) >= 0), seq


@pytest.mark.parametrize("quant", [0, 1])
def test_persistent_model_small(tpb, quant):
    got, ref = run_model(tpb, SMALL_MODEL, 3131, [99, 37], quant, n_layers=3, persistent=1)
    r, p = report(f"persistent model small q{quant}", got, ref)
    assert r <= BF16_TOL and p > 0.9999
    assert np.array_equal(np.argmax(got, axis=1), np.argmax(ref, axis=1))


@pytest.mark.slow
def test_persistent_model_c3_full_size_batch1(tpb):
    """Llama-2-7B shapes, 32 layers, context 4096, n = 8, one persistent launch per layer."""
    s = synth.C3
    got, ref = run_model(tpb, s, synth.CONFIG_SEED["C3"], [s.pos], 0, n_layers=s.n_layers,
                         persistent=1)
    r, p = report("persistent model C3 32 layers", got, ref)
    assert r <= BF16_TOL and p > 0.9999
