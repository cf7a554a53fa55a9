"""Decoder block with int8 weights (tp_block_create_q8w) on the GPU versus the oracle.

Pope et al. demo4: small-batch decode is bound by the weight bytes, and int8
weights cut them. Each matrix is quantised on the GPU with tp_quantize_q8 (its
codes and scales are first checked bit for bit against the oracle's q8_weights),
the block runs its slice products as integer dot products per 32-value block,
and the result is compared with oracle.block_forward(weights_q8=True).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth.device import DeviceBlock, to_bits
from tests.metrics import BF16_TOL, report
from tests.test_gpu_block import _dims

# Expected error level. Besides float32 accumulation, either side may put a value
# that lies within rounding of a Q8 code boundary on the neighbouring code; one
# step is 1/127 (7.9e-3) of its block's maximum, and this form quantises four
# activations per block (both normalised inputs, the attention output, the SwiGLU
# output) plus the two partials. A flipped input code of a slice product moves
# every output of that product by about |w| d_x (~1e-3 of the output scale), so
# the error is spread, not sparse; shapes where no code flips agree to ~1e-7.
TIGHT_Q8W = 1e-2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tpb(cuda_ok):
    import tensor_llama_transformer_b200 as t

    return t


def _quantize(tpb, w_bf16: torch.Tensor):
    """(codes int8, scales float32) of a bf16 [out, in] matrix, by tp_quantize_q8."""
    f = w_bf16.float().contiguous()
    q = torch.empty(f.shape, dtype=torch.int8, device="cuda")
    d = torch.empty((f.shape[0], f.shape[1] // 32), dtype=torch.float32, device="cuda")
    tpb.tp_quantize_q8(f, q, d, f.numel())
    return q, d


def run_block_q8w(tpb, inp, n, check_codes=False):
    s = inp.shape
    B = inp.x.shape[0]
    dev = DeviceBlock(inp, max_batch=B)
    (attn_norm, wq, wk, wv, wo, ffn_norm, w1, w3, w2) = dev.weights()
    qd = {k: _quantize(tpb, t) for k, t in (("wq", wq), ("wk", wk), ("wv", wv), ("wo", wo),
                                            ("w1", w1), ("w3", w3), ("w2", w2))}
    if check_codes:
        for k, (q, d) in qd.items():
            q_ref, d_ref = oracle.q8_weights(getattr(inp, k))
            np.testing.assert_array_equal(q.cpu().numpy(), q_ref)
            np.testing.assert_array_equal(d.cpu().numpy().view(np.uint32), d_ref.view(np.uint32))
    dims = _dims(tpb, s, B)
    nbytes = tpb.tp_block_workspace_bytes(dims, n, 1, 1)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    w = tpb.make_weights_q8(attn_norm, *qd["wq"], *qd["wk"], *qd["wv"], *qd["wo"], ffn_norm,
                            *qd["w1"], *qd["w3"], *qd["w2"])
    h = tpb.tp_block_create_q8w(dims, n, 1, 1, w, ws, nbytes)
    try:
        tpb.tp_block_forward(h, dev.x, dev.k_cache, dev.v_cache, dev.pos, B)
        torch.cuda.synchronize()
        bufs = {}
        for name, which in (("att", tpb.BUF_ATT), ("q", tpb.BUF_Q), ("h", tpb.BUF_H)):
            off, size = tpb.tp_block_buffer(h, which)
            bufs[name] = ws[off:off + size].view(torch.float32).cpu().numpy()
        err = int(ws[tpb.tp_block_buffer(h, 7)[0]:][:4].view(torch.int32).item())
    finally:
        tpb.tp_block_destroy(h)
    kb, vb = to_bits(dev.k_cache), to_bits(dev.v_cache)
    k_rows = np.stack([kb[b, :, inp.pos[b], :] for b in range(B)])
    v_rows = np.stack([vb[b, :, inp.pos[b], :] for b in range(B)])
    return dev.x.cpu().numpy().astype(np.float64), k_rows, v_rows, bufs, err


def check_q8w(tpb, inp, n, name, check_codes=False):
    s = inp.shape
    B = inp.x.shape[0]
    tr = {}
    ref, k_ref, v_ref = oracle.block_forward(inp, n, True, trace=tr, weights_q8=True)
    y, k_rows, v_rows, bufs, err = run_block_q8w(tpb, inp, n, check_codes)
    assert err == 0
    QD = s.n_heads * s.head_dim
    r_q, _ = report(f"{name} q", bufs["q"][:B * QD].reshape(B, QD), tr["q"])
    r_att, _ = report(f"{name} att", bufs["att"][:B * QD].reshape(B, QD), tr["att"])
    r_k, _ = report(f"{name} k@pos", oracle.bf16_to_f64(k_rows), oracle.bf16_to_f64(k_ref))
    r_out, p_out = report(f"{name} out", y, ref)
    r_dx, _ = report(f"{name} out-x", y - inp.x, ref - inp.x)
    for r in (r_q, r_att, r_k, r_out, r_dx):
        assert r <= BF16_TOL
    assert max(r_q, r_att, r_out, r_dx) <= TIGHT_Q8W, "regression against the expected error level"
    assert p_out > 0.9999


MHA = synth.BlockShape(dim=256, n_heads=2, n_kv_heads=2, head_dim=128, ffn_dim=512, vocab=0,
                       max_seq=300, batch=3, n_slices=2, sync_quant=True, pos=299, w_std=0.05)
GQA = synth.BlockShape(dim=512, n_heads=8, n_kv_heads=2, head_dim=128, ffn_dim=1024, vocab=0,
                       max_seq=260, batch=2, n_slices=2, sync_quant=True, pos=259, w_std=0.04)
ODD_W2 = synth.BlockShape(dim=256, n_heads=2, n_kv_heads=2, head_dim=128, ffn_dim=192, vocab=0,
                          max_seq=70, batch=1, n_slices=2, sync_quant=True, pos=69, w_std=0.05)
GQA8 = synth.BlockShape(dim=1024, n_heads=8, n_kv_heads=1, head_dim=128, ffn_dim=2048, vocab=0,
                        max_seq=129, batch=5, n_slices=1, sync_quant=True, pos=128, w_std=0.03)


@pytest.mark.parametrize("shape,n,pos", [
    (MHA, 2, [299, 130, 0]),              # batch 3: two launches per product (2 + 1 rows)
    (GQA, 2, [259, 127]),
    (ODD_W2, 2, [69]),                    # W2 segments of 96: scale runs off 16-byte boundaries
    (GQA8, 1, [128, 1, 64, 127, 5]),
])
def test_q8w_small(tpb, shape, n, pos):
    inp = synth.block_inputs(6161, shape)
    inp.pos[:] = pos
    check_q8w(tpb, inp, n, f"q8w d{shape.dim} H{shape.n_heads}/{shape.n_kv_heads} n{n} B{len(pos)}",
              check_codes=True)


def test_q8w_c2_full_size(tpb):
    """The C2 block (Llama-2-7B shapes, n = 4, KV 1024, batch 1) with int8 weights;
    W2's segments of 2752 columns have scale runs of 86 floats."""
    inp = synth.block_inputs(synth.CONFIG_SEED["C2"], synth.C2)
    check_q8w(tpb, inp, synth.C2.n_slices, "q8w C2")


@pytest.mark.parametrize("shape,n,pos", [
    (GQA, 2, [259, 127, 0, 64, 63, 200]),              # batch 6: three launches of 2 rows
    (MHA, 2, [299, 130, 0, 1, 2, 64, 65, 250, 128]),   # batch 9: four of 2 and one of 1
])
def test_q8w_batched(tpb, shape, n, pos):
    """Batches from 6 rows on, where bf16 handles take the tensor cores: int8 weights stay on
    the weight-streaming kernels, 2 rows per launch."""
    s = synth.BlockShape(**{**shape.__dict__, "batch": len(pos)})
    inp = synth.block_inputs(6262, s)
    inp.pos[:] = pos
    check_q8w(tpb, inp, n, f"q8w d{s.dim} n{n} B{len(pos)}", check_codes=True)
