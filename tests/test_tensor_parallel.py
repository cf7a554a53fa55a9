"""The block with its slices spread over ranks: host logic, two gloo ranks on CPU.

distributed-llama issue #29's nodes each compute their slices' partials; the
SyncAtt / SyncFfn2 transfers carry them, quantised when the sync is, to be
dequantised and merged. ``tensor_parallel`` gives each rank its weights
(``rank_weights``), its kv heads, and the phase / exchange order (``run_step``
with ``all_gather_exchange``). Here each rank's phases are computed on the CPU
from the oracle's steps on the rank's own weights and kv heads, its partials are
written in the library's sync format (float32 [B, dim], or int8 codes [B, dim]
then float32 scales [B, dim/32] per slice), the exchanges are real gloo
all-gathers, and every rank merges the gathered slices in slice order. The result
must equal the oracle's whole block: that checks the weight and head split, the
gathered layout (rank order = slice order) and the phase order. The CUDA kernels
of the same steps are checked on the GPU in test_gpu_tensor_parallel.py.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from tensor_llama_transformer_b200 import tensor_parallel as tp

SEED = 2929
SHAPE = dict(dim=256, n_heads=4, n_kv_heads=4, head_dim=128, ffn_dim=512, vocab=0, max_seq=40,
             batch=2, n_slices=4, sync_quant=False, pos=39, w_std=0.05)
GQA = dict(SHAPE, n_heads=8, n_kv_heads=4, dim=512, ffn_dim=1024)
POS = [39, 6]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_worker(rank, world, port, shape_kw, quant, out):
    import datetime

    import torch
    import torch.distributed as dist

    import oracle
    import synth

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    s = synth.BlockShape(**shape_kw)
    inp = synth.block_inputs(SEED, s)
    inp.pos[:] = POS
    n, H, Hkv, hd, D, F = s.n_slices, s.n_heads, s.n_kv_heads, s.head_dim, s.dim, s.ffn_dim
    B = inp.x.shape[0]
    pos = inp.pos
    full = {k: torch.from_numpy(getattr(inp, k).view(np.int16)) for k in
            ("wq", "wk", "wv", "wo", "w1", "w3", "w2")}
    full["attn_norm"] = torch.from_numpy(inp.attn_norm)
    full["ffn_norm"] = torch.from_numpy(inp.ffn_norm)
    local = tp.rank_weights(full, H, Hkv, hd, rank, world)
    w = {k: oracle.bf16_to_f64(local[k].numpy().view(np.uint16))
         for k in ("wq", "wk", "wv", "wo", "w1", "w3", "w2")}
    kvh = tp.rank_kv_heads(Hkv, rank, world)
    c = len(tp.rank_slices(n, rank, world))
    Hl, Hkvl, Fl = H // world, Hkv // world, F // world
    kc = oracle.bf16_to_f64(inp.k_cache[:, kvh])
    vc = oracle.bf16_to_f64(inp.v_cache[:, kvh])
    x = inp.x.astype(np.float64)
    chunk = B * D + B * (D // 32) * 4 if quant else B * D * 4
    send = torch.zeros(c * chunk, dtype=torch.uint8)
    recv = torch.zeros(world * c * chunk, dtype=torch.uint8)
    state = {}

    def pack(parts):
        buf = b""
        for p in parts:
            p32 = np.asarray(p, dtype=np.float32)
            if quant:
                q, d = oracle.q8_quantize(p32)
                buf += q.astype(np.int8).tobytes() + d.astype(np.float32).tobytes()
            else:
                buf += p32.tobytes()
        send.copy_(torch.frombuffer(bytearray(buf), dtype=torch.uint8))

    def merge(xv):
        raw = recv.numpy().tobytes()
        acc = np.zeros_like(xv)
        for j in range(n):  # every slice of every rank, in slice order
            b = raw[j * chunk:(j + 1) * chunk]
            if quant:
                q = np.frombuffer(b[:B * D], np.int8).reshape(B, D)
                d = np.frombuffer(b[B * D:], np.float32).reshape(B, D // 32)
                p = oracle.q8_dequantize(q, d)
            else:
                p = np.frombuffer(b, np.float32).reshape(B, D)
            acc = acc + p.astype(np.float64)
        return xv + acc

    def step(phase):
        if phase == tp.TP_RANK_ATT:
            xin = oracle.sync_buffer(oracle.rmsnorm(x, inp.attn_norm, s.norm_eps), quant)
            q = oracle.rope(xin @ w["wq"].T, pos, Hl, hd, s.rope_theta)
            k = oracle.rope(xin @ w["wk"].T, pos, Hkvl, hd, s.rope_theta)
            v = xin @ w["wv"].T
            rows = np.zeros((2, B, Hkvl, hd), dtype=np.uint16)
            for b in range(B):
                for j in range(Hkvl):
                    rows[0, b, j] = oracle.round_to_bf16(k[b, j * hd:(j + 1) * hd])
                    rows[1, b, j] = oracle.round_to_bf16(v[b, j * hd:(j + 1) * hd])
                    kc[b, j, pos[b]] = oracle.bf16_to_f64(rows[0, b, j])
                    vc[b, j, pos[b]] = oracle.bf16_to_f64(rows[1, b, j])
            state["kv_rows"] = rows
            att = oracle.attention_decode(q, kc, vc, pos, range(Hl), Hl, Hkvl, hd)
            cols = [oracle.slice_range(Hl * hd, c, j) for j in range(c)]
            pack([att[:, cs] @ w["wo"][:, cs].T for cs in cols])
        elif phase == tp.TP_RANK_FFN:
            state["x1"] = merge(x)
            xin2 = oracle.sync_buffer(oracle.rmsnorm(state["x1"], inp.ffn_norm, s.norm_eps), quant)
            h = oracle.swiglu(xin2 @ w["w1"].T, xin2 @ w["w3"].T)
            fs = [oracle.slice_range(Fl, c, j) for j in range(c)]
            pack([h[:, f] @ w["w2"][:, f].T for f in fs])
        else:
            state["x2"] = merge(state["x1"])
            state["bytes"] = (send.numpy().copy(), recv.numpy().copy())

    tp.run_step(step, tp.all_gather_exchange(), send, recv)
    out.put((rank, state["x2"], state["kv_rows"], state["bytes"]))
    dist.destroy_process_group()


def _run(world, shape_kw, quant):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_worker, args=(r, world, port, shape_kw, quant, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=120) for _ in range(world)), key=lambda t: t[0])
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    return res


@pytest.mark.parametrize("shape_kw,world", [(SHAPE, 2), (GQA, 2), (SHAPE, 4)],
                         ids=["mha-2", "gqa2-2", "mha-4"])
@pytest.mark.parametrize("quant", [0, 1])
def test_ranks_equal_the_whole_block(shape_kw, world, quant):
    import oracle
    import synth

    s = synth.BlockShape(**dict(shape_kw, sync_quant=bool(quant)))
    inp = synth.block_inputs(SEED, s)
    inp.pos[:] = POS
    ref, k_ref, v_ref = oracle.block_forward(inp, s.n_slices, bool(quant))
    res = _run(world, shape_kw, quant)
    # every rank ends with the same residual (the same bytes merged the same way)
    for r in res[1:]:
        assert np.array_equal(r[1], res[0][1])
    err = np.max(np.abs(res[0][1] - ref)) / np.max(np.abs(ref))
    assert err < 1e-6, err  # float32 transfer of the partials vs the oracle's float64
    # the gathered buffer is the ranks' send buffers in rank order (= slice order)
    sends = np.concatenate([r[3][0] for r in res])
    for r in res:
        np.testing.assert_array_equal(r[3][1], sends)
    # each rank wrote the k / v rows of its own kv heads
    Hkvl = s.n_kv_heads // world
    for r, _, rows, _ in res:
        heads = slice(r * Hkvl, (r + 1) * Hkvl)
        np.testing.assert_array_equal(rows[0], k_ref[:, heads])
        np.testing.assert_array_equal(rows[1], v_ref[:, heads])


def test_rank_split_helpers():
    import torch

    assert list(tp.rank_slices(8, 1, 4)) == [2, 3]
    assert tp.rank_kv_heads(8, 3, 4) == slice(6, 8)
    with pytest.raises(ValueError):
        tp.rank_slices(6, 0, 4)
    H, Hkv, hd, D, F = 4, 2, 2, 6, 8
    w = {"attn_norm": torch.arange(D), "ffn_norm": torch.arange(D),
         "wq": torch.arange(H * hd * D).reshape(H * hd, D),
         "wk": torch.arange(Hkv * hd * D).reshape(Hkv * hd, D),
         "wv": -torch.arange(Hkv * hd * D).reshape(Hkv * hd, D),
         "wo": torch.arange(D * H * hd).reshape(D, H * hd),
         "w1": torch.arange(F * D).reshape(F, D), "w3": -torch.arange(F * D).reshape(F, D),
         "w2": torch.arange(D * F).reshape(D, F)}
    parts = [tp.rank_weights(w, H, Hkv, hd, r, 2) for r in range(2)]
    # column-split matrices: rank r's rows; row-split matrices: rank r's columns
    for k in ("wq", "wk", "wv", "w1", "w3"):
        assert torch.equal(torch.cat([p[k] for p in parts], 0), w[k])
    for k in ("wo", "w2"):
        assert torch.equal(torch.cat([p[k] for p in parts], 1), w[k])
        assert all(p[k].is_contiguous() for p in parts)
    assert parts[1]["wq"].shape == (H // 2 * hd, D) and parts[1]["wo"].shape == (D, H // 2 * hd)


def _failing_worker(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=5))
    send = torch.zeros(16, dtype=torch.uint8)
    recv = torch.zeros(16 * world, dtype=torch.uint8)

    def step(phase):
        if rank == 1 and phase == tp.TP_RANK_ATT:
            raise RuntimeError("rank 1 failed in phase 0")

    try:
        tp.run_step(step, tp.all_gather_exchange(), send, recv)
        out.put((rank, "completed"))
    except Exception as e:  # reported to the parent, which checks that nobody hangs
        out.put((rank, f"{type(e).__name__}: {str(e)[:80]}"))


def test_failed_rank_ends_the_others_step_with_an_error():
    """A rank that fails before its first exchange never joins the all-gather: the
    other rank's exchange ends with an error (process-group timeout or closed
    connection) instead of waiting for ever. Host-side failure only."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_failing_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(60)
        assert p.exitcode is not None
    assert res[1].startswith("RuntimeError: rank 1 failed")
    assert res[0] != "completed", res[0]
