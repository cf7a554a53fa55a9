"""tp_block_forward_noalloc: the block step for callers that cannot allocate.

Some callers cannot give this library a device workspace: for example a plugin
inside a host runtime that owns all device memory through its own pool, or a
serving loop that may not call cudaMalloc once it runs. For them the library
offers one entry point that takes its scratch from a fixed 16 MiB array
compiled into the library instead of a caller-allocated workspace.

This file checks, through the C ABI, that this entry point gives bit for bit the
block output and the k/v rows written to the caches that tp_block_create +
tp_block_forward give on identical inputs (both run the same kernels, whose
results do not depend on where the scratch lives), for two calls in a row, on
the weight-streaming kernels, on the tensor-core path (batch 8) and, in a child
process started with TP_PERSISTENT=1, on the persistent block kernel, whose grid
barrier counters live in the shared array; that the kernels' error word, read
back through tp_block_noalloc_error, stays 0; and that a configuration too large
for the array is refused. It is named so that pytest collects it last; it needs
no state from other test files.
"""
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402
from synth.device import DeviceBlock  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tpb(cuda_ok):
    import tensor_llama_transformer_b200 as t

    return t


def _dims(tpb, s):
    return tpb.make_dims(s.dim, s.n_heads, s.n_kv_heads, s.head_dim, s.ffn_dim, max(s.vocab, 2),
                         s.batch, s.max_seq, s.norm_eps, s.rope_theta)


SMALL_GQA_Q8 = synth.BlockShape(dim=512, n_heads=8, n_kv_heads=2, head_dim=128, ffn_dim=1024,
                                vocab=0, max_seq=260, batch=2, n_slices=2, sync_quant=True,
                                pos=258, w_std=0.04)
BATCHED_GQA_Q8 = synth.BlockShape(dim=512, n_heads=8, n_kv_heads=2, head_dim=128, ffn_dim=1024,
                                  vocab=0, max_seq=200, batch=8, n_slices=2, sync_quant=True,
                                  pos=198, w_std=0.04)
CASES = [
    (SMALL_GQA_Q8, 1, [200, 100]),
    (synth.C2, 1, [1000]),
    (BATCHED_GQA_Q8, 1, [198, 3, 64, 120, 0, 77, 150, 31]),  # batch >= 6: tcgen05 products
]


def compare_two_calls(tpb, shape, partition, pos):
    """Runs both entry points twice on the same inputs; asserts identical bits."""
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
    err_off, _ = tpb.tp_block_buffer(h, 7)
    # path under test: no workspace argument
    dev = DeviceBlock(inp)
    w = tpb.make_weights(*dev.weights())
    try:
        for call in range(2):  # two steps in a row: the array keeps the first call's contents
            tpb.tp_block_forward(h, ref.x, ref.k_cache, ref.v_cache, ref.pos, B)
            tpb.tp_block_forward_noalloc(dims, shape.n_slices, partition, quant, w, dev.x,
                                         dev.k_cache, dev.v_cache, dev.pos, B)
            assert tpb.tp_block_noalloc_error() == 0, "a bounded wait in a kernel gave up"
            assert int(ws[err_off:err_off + 4].view(torch.int32).item()) == 0
            assert torch.equal(dev.x, ref.x), f"call {call}: block output differs"
            for b in range(B):
                p = int(ref.pos[b].item())
                assert torch.equal(dev.k_cache[b, :, p], ref.k_cache[b, :, p]), f"call {call}: k row"
                assert torch.equal(dev.v_cache[b, :, p], ref.v_cache[b, :, p]), f"call {call}: v row"
            print(f"[parity] noalloc call {call}: output and cache rows bit-identical")
            ref.pos += 1
            dev.pos += 1
    finally:
        tpb.tp_block_destroy(h)


@pytest.mark.parametrize("shape,partition,pos", CASES, ids=["small_gqa_q8", "c2_7b_block",
                                                             "batched_gqa_q8"])
def test_noalloc_matches_workspace_entry_point(tpb, shape, partition, pos):
    compare_two_calls(tpb, shape, partition, pos)


def test_noalloc_persistent_kernel(cuda_ok):
    """With TP_PERSISTENT=1 (read when the library loads, hence a child process)
    batch 1-2 runs as the one persistent kernel on both paths."""
    env = dict(os.environ, TP_PERSISTENT="1")
    r = subprocess.run([sys.executable, os.path.abspath(__file__), "persistent"], env=env,
                       capture_output=True, text=True, timeout=600)
    print(r.stdout[-2000:], r.stderr[-2000:])
    assert r.returncode == 0 and "persistent ok" in r.stdout


def test_noalloc_refuses_oversized_workspace(tpb):
    s = synth.C4  # 70B shapes at batch 32: the workspace is far above 16 MiB
    dims = _dims(tpb, s)
    assert tpb.tp_block_workspace_bytes(dims, s.n_slices, 1, 0) > tpb.TP_NOALLOC_SCRATCH_BYTES
    dummy = torch.zeros(64, dtype=torch.float32, device="cuda")
    w = tpb.make_weights(*([dummy] * 9))
    with pytest.raises(tpb.TpError) as e:
        tpb.tp_block_forward_noalloc(dims, s.n_slices, 1, 0, w, dummy, dummy, dummy, dummy, 1)
    assert e.value.status == tpb.TP_ESCRATCH


if __name__ == "__main__" and sys.argv[1:] == ["persistent"]:
    import tensor_llama_transformer_b200 as lib

    torch.cuda.set_device(0)
    compare_two_calls(lib, SMALL_GQA_Q8, 1, [200, 100])
    compare_two_calls(lib, synth.C2, 1, [1000])
    print("persistent ok")
