"""tp_block_forward_noalloc: the block step for callers that cannot allocate.

Some callers cannot give this library a device workspace: for example a plugin
inside a host runtime that owns all device memory through its own pool, or a
serving loop that may not call cudaMalloc once it runs. For them the library
offers one entry point that takes its scratch from a fixed 16 MiB array
compiled into the library instead of a caller-allocated workspace.

This file checks, through the C ABI, that this entry point gives the same
block output (and the same k/v rows written to the caches) as
tp_block_create + tp_block_forward on identical inputs, for two calls in a
row, and that a configuration too large for the array is refused. It is named
so that pytest collects it last; it needs no state from other test files.
"""
import numpy as np
import pytest
import torch

import synth
from synth.device import DeviceBlock
from tests.metrics import BF16_TOL, report

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tpb(cuda_ok):
    import tensor_llama_transformer_b200 as t

    return t


def _dims(tpb, s):
    return tpb.make_dims(s.dim, s.n_heads, s.n_kv_heads, s.head_dim, s.ffn_dim, max(s.vocab, 2),
                         s.batch, s.max_seq, s.norm_eps, s.rope_theta)


CASES = [
    (synth.BlockShape(dim=512, n_heads=8, n_kv_heads=2, head_dim=128, ffn_dim=1024, vocab=0,
                      max_seq=260, batch=2, n_slices=2, sync_quant=True, pos=258, w_std=0.04),
     1, [200, 100]),
    (synth.C2, 1, [1000]),
]


@pytest.mark.parametrize("shape,partition,pos", CASES, ids=["small_gqa_q8", "c2_7b_block"])
def test_noalloc_matches_workspace_entry_point(tpb, shape, partition, pos):
    inp = synth.block_inputs(9090, shape)
    inp.pos[:] = pos
    quant = int(shape.sync_quant)
    dims = _dims(tpb, shape)
    B = shape.batch

    # reference path: caller-allocated workspace
    ref = DeviceBlock(inp)
    nbytes = tpb.tp_block_workspace_bytes(dims, shape.n_slices, partition, quant)
    assert nbytes <= tpb.TP_NOALLOC_SCRATCH_BYTES
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    h = tpb.tp_block_create(dims, shape.n_slices, partition, quant,
                            tpb.make_weights(*ref.weights()), ws, nbytes)
    # path under test: no workspace argument
    dev = DeviceBlock(inp)
    w = tpb.make_weights(*dev.weights())
    try:
        for call in range(2):  # two steps in a row: the array keeps the first call's contents
            tpb.tp_block_forward(h, ref.x, ref.k_cache, ref.v_cache, ref.pos, B)
            tpb.tp_block_forward_noalloc(dims, shape.n_slices, partition, quant, w, dev.x,
                                         dev.k_cache, dev.v_cache, dev.pos, B)
            torch.cuda.synchronize()
            r, _ = report(f"noalloc call {call}", dev.x.cpu().numpy(), ref.x.cpu().numpy())
            assert r <= BF16_TOL
            for b in range(B):
                p = int(ref.pos[b].item())
                for cache_ref, cache_dev in ((ref.k_cache, dev.k_cache), (ref.v_cache, dev.v_cache)):
                    a = cache_dev[b, :, p].float().cpu().numpy()
                    e = cache_ref[b, :, p].float().cpu().numpy()
                    assert np.max(np.abs(a - e)) <= BF16_TOL * max(np.max(np.abs(e)), 1e-30)
            ref.pos += 1
            dev.pos += 1
    finally:
        tpb.tp_block_destroy(h)


def test_noalloc_refuses_oversized_workspace(tpb):
    s = synth.C4  # 70B shapes at batch 32: the workspace is far above 16 MiB
    dims = _dims(tpb, s)
    assert tpb.tp_block_workspace_bytes(dims, s.n_slices, 1, 0) > tpb.TP_NOALLOC_SCRATCH_BYTES
    dummy = torch.zeros(64, dtype=torch.float32, device="cuda")
    w = tpb.make_weights(*([dummy] * 9))
    with pytest.raises(tpb.TpError) as e:
        tpb.tp_block_forward_noalloc(dims, s.n_slices, 1, 0, w, dummy, dummy, dummy, dummy, 1)
    assert e.value.status == tpb.TP_ESCRATCH
