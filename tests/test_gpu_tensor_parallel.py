"""The block with its slices spread over ranks (tp_block_rank_step) on the GPU.

Each rank holds n/world of the n slices (distributed-llama issue #29's nodes):
its weights (``tensor_parallel.rank_weights``), its kv heads' caches, and a
replicated residual. Phase 0 leaves its W_O partials in its send buffer, phase 1
merges the gathered buffer and leaves its W2 partials, phase 2 merges again.

Here every GPU call runs on one GPU, so the ranks of a step run one after another
on it and the all-gather between phases is a device copy of the send buffers, in
rank order, into every rank's receive buffer; no kernel waits on another. The
ranks must end with the same residual bit for bit, equal to the oracle's block
and to the single-process block within the error levels of tests/test_gpu_block.py.
A second test runs one rank with a real NCCL process group (world size 1, the
all-gather through ``torch.distributed``): it must give exactly the bits of
tp_block_forward.
"""
import datetime
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import synth
from synth.device import DeviceBlock, to_bits
from tensor_llama_transformer_b200 import tensor_parallel as tp
from tests.metrics import BF16_TOL, assert_q8_codes_exact, report
from tests.test_gpu_block import SMALL_TC_GQA, SMALL_TC_MHA, TIGHT, TIGHT_Q8, _dims, run_block

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tpb(cuda_ok):
    import tensor_llama_transformer_b200 as t

    return t


def run_ranks(tpb, inp, n, quant, world):
    """One decode step of the block over `world` ranks emulated on this GPU.
    Returns (x of every rank, k/v rows at pos assembled over ranks [B, Hkv, hd],
    error words)."""
    s = inp.shape
    B = inp.x.shape[0]
    dev = DeviceBlock(inp, max_batch=B)
    dims = _dims(tpb, s, B)
    full = dict(zip(tp.WEIGHT_ORDER, dev.weights()))
    ranks = []
    try:
        for r in range(world):
            kvh = tp.rank_kv_heads(s.n_kv_heads, r, world)
            w = tp.rank_weights(full, s.n_heads, s.n_kv_heads, s.head_dim, r, world)
            ranks.append(dict(rb=tp.RankBlock(dims, n, quant, r, world, w), x=dev.x.clone(),
                              kc=dev.k_cache[:, kvh].contiguous(), vc=dev.v_cache[:, kvh].contiguous()))
        for phase in (tp.TP_RANK_ATT, tp.TP_RANK_FFN, tp.TP_RANK_OUT):
            if phase != tp.TP_RANK_ATT:  # the all-gather: send buffers in rank order
                gathered = torch.cat([rk["rb"].buffers(B)[0] for rk in ranks])
                for rk in ranks:
                    rk["rb"].buffers(B)[1].copy_(gathered)
            for rk in ranks:
                rk["rb"].step(phase, rk["x"], rk["kc"], rk["vc"], dev.pos, B)
            if phase == tp.TP_RANK_ATT:  # the attention RMSNorm (+Q8) each rank's prologue wrote
                torch.cuda.synchronize()
                for rk in ranks:
                    norm = {}
                    for key, which, dt in (("xn", tpb.BUF_XN, torch.float32),
                                           ("xq", tpb.BUF_XQ, torch.int8),
                                           ("xd", tpb.BUF_XD, torch.float32)):
                        off, size = tpb.tp_block_buffer(rk["rb"].h, which)
                        norm[key] = rk["rb"].ws[off:off + size].view(dt).cpu().numpy()
                    rk["att_norm"] = norm
        torch.cuda.synchronize()
        errs = []
        for rk in ranks:
            off, _ = tpb.tp_block_buffer(rk["rb"].h, 7)
            errs.append(int(rk["rb"].ws[off:off + 4].view(torch.int32).item()))
        xs = [rk["x"].cpu().numpy().astype(np.float64) for rk in ranks]
        norms = [rk["att_norm"] for rk in ranks]
        kb = np.concatenate([to_bits(rk["kc"]) for rk in ranks], axis=1)
        vb = np.concatenate([to_bits(rk["vc"]) for rk in ranks], axis=1)
    finally:
        for rk in ranks:
            rk["rb"].close()
    k_rows = np.stack([kb[b, :, inp.pos[b], :] for b in range(B)])
    v_rows = np.stack([vb[b, :, inp.pos[b], :] for b in range(B)])
    return xs, k_rows, v_rows, errs, norms


def check_ranks(tpb, inp, n, quant, world, tight, name):
    xs, k_rows, v_rows, errs, norms = run_ranks(tpb, inp, n, quant, world)
    assert errs == [0] * world, "a bounded wait in a kernel gave up"
    for x in xs[1:]:
        assert np.array_equal(x, xs[0]), "ranks ended with different residuals"
    ref, k_ref, v_ref = oracle.block_forward(inp, n, bool(quant))
    r_out, p_out = report(f"{name} out", xs[0], ref)
    r_dx, _ = report(f"{name} out-x", xs[0] - inp.x, ref - inp.x)
    r_k, _ = report(f"{name} k@pos", oracle.bf16_to_f64(k_rows), oracle.bf16_to_f64(k_ref))
    r_v, _ = report(f"{name} v@pos", oracle.bf16_to_f64(v_rows), oracle.bf16_to_f64(v_ref))
    for r in (r_out, r_dx, r_k, r_v):
        assert r <= BF16_TOL
    assert max(r_out, r_dx) <= tight, "regression against the expected error level"
    assert p_out > 0.9999
    whole = run_block(tpb, inp, n, quant)[0]
    r_w, _ = report(f"{name} vs whole block", xs[0] - inp.x, whole - inp.x)
    assert r_w <= tight
    # the attention RMSNorm of phase 0 on every rank: float32 output against the
    # oracle's, and with the Q8 sync its codes bit-exact from that same float32 row
    s = inp.shape
    B, D = inp.x.shape
    xn_ref = oracle.rmsnorm(inp.x, inp.attn_norm, s.norm_eps)
    for r, nm in enumerate(norms):
        r_xn, _ = report(f"{name} rank {r} xnorm(att)", nm["xn"][:B * D].reshape(B, D), xn_ref)
        assert r_xn <= 1e-5
        if quant:
            assert_q8_codes_exact(nm["xn"], nm["xq"], nm["xd"], B, D, f"{name} rank {r} xnorm(att)")


MHA4 = synth.BlockShape(dim=256, n_heads=4, n_kv_heads=4, head_dim=128, ffn_dim=512, vocab=0,
                        max_seq=300, batch=2, n_slices=4, sync_quant=False, pos=299, w_std=0.05)
GQA = synth.BlockShape(dim=512, n_heads=8, n_kv_heads=2, head_dim=128, ffn_dim=1024, vocab=0,
                       max_seq=260, batch=3, n_slices=2, sync_quant=False, pos=259, w_std=0.04)


@pytest.mark.parametrize("quant", [0, 1])
@pytest.mark.parametrize("shape,n,world,pos", [
    (MHA4, 4, 2, [299, 0]),        # two slices per rank; a one-position context
    (MHA4, 4, 4, [130, 64]),       # one slice per rank
    (GQA, 2, 2, [259, 127, 3]),    # GQA group of 4, one kv head per rank
])
def test_ranks_weight_streaming_path(tpb, shape, n, world, pos, quant):
    inp = synth.block_inputs(6262, shape)
    inp.pos[:] = pos
    check_ranks(tpb, inp, n, quant, world, TIGHT_Q8 if quant else TIGHT,
                f"ranks d{shape.dim} n{n} w{world} q{quant}")


@pytest.mark.parametrize("quant", [0, 1])
@pytest.mark.parametrize("shape,n,world", [(SMALL_TC_GQA, 2, 2), (SMALL_TC_MHA, 8, 4)])
def test_ranks_tensor_core_path(tpb, shape, n, world, quant):
    """Batches of 6 or more: the slice products on the tcgen05 GEMM, W2 split into
    contraction parts that the pack sums before the sync format."""
    inp = synth.block_inputs(6363, shape)
    B = shape.batch
    inp.pos[:] = [(shape.pos * (i + 1)) // B for i in range(B)]
    check_ranks(tpb, inp, n, quant, world, 1e-2, f"ranks tc B{B} n{n} w{world} q{quant}")


def test_ranks_c2_full_size(tpb):
    """The 7B block (n = 4, Q8 sync, KV 1024, batch 1) over 4 ranks, one slice each."""
    inp = synth.block_inputs(synth.CONFIG_SEED["C2"], synth.C2)
    check_ranks(tpb, inp, synth.C2.n_slices, 1, 4, TIGHT_Q8, "ranks C2")


def test_rank_phase_order_enforced(tpb):
    s = MHA4
    inp = synth.block_inputs(1, s)
    dev = DeviceBlock(inp)
    dims = _dims(tpb, s, s.batch)
    w = tp.rank_weights(dict(zip(tp.WEIGHT_ORDER, dev.weights())), s.n_heads, s.n_kv_heads,
                        s.head_dim, 0, 2)
    kc, vc = dev.k_cache[:, :2].contiguous(), dev.v_cache[:, :2].contiguous()
    rb = tp.RankBlock(dims, 4, 1, 0, 2, w)
    try:
        with pytest.raises(tpb.TpError) as e:  # phase 1 before phase 0
            rb.step(tp.TP_RANK_FFN, dev.x, kc, vc, dev.pos, 2)
        assert e.value.status == tpb.TP_EINVAL
        with pytest.raises(tpb.TpError) as e:  # the whole-block entry point
            tpb.tp_block_forward(rb.h, dev.x, kc, vc, dev.pos, 2)
        assert e.value.status == tpb.TP_EINVAL
        rb.step(tp.TP_RANK_ATT, dev.x, kc, vc, dev.pos, 2)
        with pytest.raises(tpb.TpError) as e:  # batch changed within the step
            rb.step(tp.TP_RANK_FFN, dev.x, kc, vc, dev.pos, 1)
        assert e.value.status == tpb.TP_EINVAL
        assert tpb.tp_block_rank_sync_bytes(rb.h, 2) == 2 * (2 * 256 + 2 * 8 * 4)
        torch.cuda.synchronize()
    finally:
        rb.close()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _nccl_world1(port, shape_kw, pos, quant, out):
    import torch.distributed as dist

    import tensor_llama_transformer_b200 as tpb

    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        s = synth.BlockShape(**shape_kw)
        inp = synth.block_inputs(7373, s)
        inp.pos[:] = pos
        B = len(pos)
        dev = DeviceBlock(inp, max_batch=B)
        dims = _dims(tpb, s, B)
        k0, v0, x0 = dev.k_cache.clone(), dev.v_cache.clone(), dev.x.clone()
        nbytes = tpb.tp_block_workspace_bytes(dims, s.n_slices, 1, quant)
        ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
        h = tpb.tp_block_create(dims, s.n_slices, 1, quant, tpb.make_weights(*dev.weights()), ws,
                                nbytes)
        tpb.tp_block_forward(h, dev.x, dev.k_cache, dev.v_cache, dev.pos, B)
        tpb.tp_block_destroy(h)
        rb = tp.RankBlock(dims, s.n_slices, quant, 0, 1, dict(zip(tp.WEIGHT_ORDER, dev.weights())))
        xr, kr, vr = x0.clone(), k0.clone(), v0.clone()
        rb.forward(xr, kr, vr, dev.pos, B)
        torch.cuda.synchronize()
        rb.close()
        out.put((bool(torch.equal(xr, dev.x)), bool(torch.equal(kr, dev.k_cache)),
                 bool(torch.equal(vr, dev.v_cache)), float((xr - dev.x).abs().max())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("shape,pos,quant", [
    (MHA4, [299, 17], 1),
    (MHA4, [40, 299], 0),
    (SMALL_TC_GQA, [199, 3, 50, 100, 150, 9, 70, 199], 1),
])
def test_rank_nccl_world1_matches_block(cuda_ok, shape, pos, quant):
    """One rank holding every slice, its exchanges through an NCCL all-gather:
    the same launches and the same merge as tp_block_forward, so the same bits."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_nccl_world1, args=(_free_port(), shape.__dict__, pos, quant, q))
    p.start()
    res = q.get(timeout=240)
    p.join(60)
    assert p.exitcode == 0
    assert res[:3] == (True, True, True), res
