#!/usr/bin/env python
"""Benchmark: decode step of a tensor-parallel Llama-2-7B-shaped block on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one decode step of one decoder block (dim 4096, 32 heads x 128,
SwiGLU 11008, KV cache 1024, batch 1) partitioned into n = 4 slices with int8
(Q8) sync buffers, i.e. every step on the hot path: RMSNorm+Q8, q/k/v slice
products with RoPE and cache write, split-context attention, W_O partials,
merge, RMSNorm+Q8, W1/W3+SwiGLU, W2 partials, merge. Inputs are seeded
synthetic tensors of those shapes; the 404.75 MB of weights per step are
larger than L2, so no flush is needed between steps.

Rank 0 prints one JSON line. With N > 1 (torchrun) every rank runs its own
replica on its own GPU (the path does not shard across GPUs), the time is the
max over ranks and the value is the sum of all ranks' tokens.

Also measured (same run, N=1 fields): the PaLM-shaped FFN (E 18432, F 73728,
B 512) through tp_ffn_forward in its fused, 1D-64 and 2D-8x8 forms, as TFLOP/s.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode tokens/s & HBM GB/s per TP-sliced block; FFN TFLOP/s at B=512 (1 B200)"
# the workload of the headline (both arms print this same dict)
CONFIG = {"workload": "C2: Llama-2-7B-shaped decoder block decode, dim 4096, 32x128 heads, "
                      "SwiGLU 11008, KV 1024, batch 1, n=4 slices, Q8 sync buffers",
          "batch": 1, "n_slices": 4, "sync_quant": True, "kv_len": 1024}
STAGES = ["norm_qkv_rope", "attention", "wo_partials", "merge", "norm_w13_swiglu", "w2_partials",
          "merge2"]


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[1])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--graph-steps", type=int, default=100, help="steps captured per CUDA graph")
    ap.add_argument("--e2e-steps", type=int, default=1000)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-seconds", type=float, default=150.0)
    ap.add_argument("--no-ffn", action="store_true", help="skip the PaLM FFN measurement")
    ap.add_argument("--ffn-iters", type=int, default=5)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the C4 block and C3 model measurements")
    ap.add_argument("--extras", default=None,
                    help="comma list of the extra workloads to time (default: all of them): "
                         "c2_block_persistent, c2_block_int8_weights, c2_prefill_chunk64, c4_block, "
                         "c4_block_mqa, "
                         "c3_model_b1, c3_model_b16")
    ap.add_argument("--profile", choices=["c4", "c3b1", "c2p", "c2q8w", "c2prefill", "ffn"],
                    default=None,
                    help="only run a few eager steps of one extra workload (for profiler launch "
                         "lists: c4 block, c3 model at batch 1, c2 block on the persistent kernel, "
                         "c2 block with int8 weights, c2 prefill chunk, or the fused PaLM-shaped "
                         "FFN at B 512 with F cut to --profile-ffn-f)")
    ap.add_argument("--profile-ffn-form", choices=["fused", "faithful", "faithful_q8"],
                    default="fused",
                    help="--profile ffn: the merge form (faithful: 1D over F / 1152 slices, so every "
                         "slice has the 1152-wide contraction of the full-size 1D-64 form)")
    ap.add_argument("--profile-ffn-f", type=int, default=18432,
                    help="intermediate size of the --profile ffn case (PaLM: 73728)")
    ap.add_argument("--profile-steps", type=int, default=3)
    ap.add_argument("--rank-exchange", action="store_true",
                    help="also time the C2 block spread over the ranks (one slice group per GPU, "
                         "NCCL all-gather of the sync buffers); on by default when N > 1, and with "
                         "N = 1 it runs a one-rank NCCL group")
    return ap.parse_args(argv)


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled while the GPU works.

    Read-only NVML queries from a thread of this process (every 10 ms), so that a
    short timed region still gets samples; nvidia-smi --query-gpu as the fallback
    when the NVML bindings cannot load. Nothing here changes a GPU setting."""

    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        import threading

        self.rows = []  # (sm_mhz, sm_max_mhz, reasons)
        self.proc = None
        self.thread = None
        self.stop_flag = threading.Event()
        self.source = None
        try:
            import pynvml
            import torch

            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
            h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            bits = (pynvml.nvmlClocksEventReasonHwSlowdown,
                    pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                    pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                    pynvml.nvmlClocksEventReasonSwPowerCap)
            smax = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)

            def poll():
                while not self.stop_flag.is_set():
                    try:
                        sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                        r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.rows.append((float(sm), float(smax),
                                          [n for n, b in zip(self.NAMES, bits) if r & b]))
                    except Exception:
                        pass
                    self.stop_flag.wait(0.01)

            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            self.source = "nvml"
            return
        except Exception:
            self.thread = None
        self._start_smi(device_index)

    def _start_smi(self, device_index: int):
        try:
            import torch

            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        except Exception:
            sel = None
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "100"]
        if sel:
            cmd += ["-i", sel]
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(cmd, stdout=self.out, stderr=subprocess.DEVNULL)
            self.source = "nvidia-smi"
        except Exception:
            self.proc = None

    def count(self) -> int:
        return len(self.rows)

    def stop(self):
        if self.thread is not None:
            self.stop_flag.set()
            self.thread.join(timeout=5)
        elif self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.out.close()
            for ln in open(self.path):
                r = [p.strip() for p in ln.split(",")]
                if len(r) >= 9 and r[1].replace(".", "").isdigit():
                    self.rows.append((float(r[1]), float(r[2]) if r[2].replace(".", "").isdigit()
                                      else None,
                                      [self.NAMES[i] for i in range(4) if r[5 + i].lower() == "active"]))
            os.unlink(self.path)
        if not self.rows:
            return None
        sm = [r[0] for r in self.rows]
        smax = [r[1] for r in self.rows if r[1]]
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted({n for r in self.rows for n in r[2]}),
                "samples": len(self.rows), "source": self.source}


def dist_setup():
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def allreduce_max(v: float, world: int) -> float:
    """Max of a per-rank value over all ranks (device tensor under NCCL, host under gloo)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


# DRAM bytes (read + write) of one launch of the W1/W3 slice GEMV in the C2 block,
# the mean over the 10 graph-replayed launches of an ncu capture of the step (180.460339 MB
# read + 0.252544 MB written): the weights once, plus the activations and the SwiGLU output.
W13_DRAM_BYTES = 180460339 + 252544


def block_bytes(s):
    qd, kd = s.n_heads * s.head_dim, s.n_kv_heads * s.head_dim
    weights = (qd * s.dim + 2 * kd * s.dim + s.dim * qd + 3 * s.ffn_dim * s.dim) * 2
    kv = 2 * s.batch * s.n_kv_heads * (s.pos + 1) * s.head_dim * 2
    return weights, kv


# ---------------------------------------------------------------------------
# CPU oracle (baseline / reference arm)
# ---------------------------------------------------------------------------

def time_oracle(inp, s, seconds: float, max_steps: int | None = None, warmup: int = 1):
    """Oracle steps/s on the host; returns (tokens/s, timed steps, seconds, cores, warm-up
    steps done). Up to `warmup` untimed steps (at least one: the first call pages the
    code in), stopping early once they have taken `seconds`."""
    import oracle

    cores = len(os.sched_getaffinity(0))
    w, t0 = 0, time.perf_counter()
    while w < max(1, warmup):
        oracle.block_forward(inp, s.n_slices, s.sync_quant)
        w += 1
        if time.perf_counter() - t0 >= seconds:
            break
    n, t0 = 0, time.perf_counter()
    while True:
        oracle.block_forward(inp, s.n_slices, s.sync_quant)
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds or (max_steps is not None and n >= max_steps):
            break
    return n * s.batch / el, n, el, cores, w


def run_reference(args):
    """The oracle (float64 NumPy on the host cores) on the same workload."""
    import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    s = synth.C2
    inp = synth.block_inputs(synth.CONFIG_SEED["C2"], s)
    tps, n, el, cores, warm = time_oracle(inp, s, args.ref_seconds, max_steps=args.steps,
                                          warmup=args.warmup)
    w, kv = block_bytes(s)
    sample = (f"{n} of {args.steps} requested steps of the C2 block (batch 1) through the float64 "
              f"oracle after {warm} untimed, each phase bounded to {args.ref_seconds:.0f} s")
    line = {
        "impl": "reference", "metric": METRIC, "value": tps, "unit": "tokens/s", "n_gpus": world,
        "steps": n, "warmup": warm, "ms_per_step": el / n * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(CONFIG),
        "cpu_baseline": {"value": tps, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": tps, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "hbm_gbs_equiv": (w + kv) * tps / 1e9,
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def make_events(torch, n):
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for e in evs:  # force creation so that the raw handle exists
        e.record()
    torch.cuda.synchronize()
    return evs


def gemv_timeline(torch, tpb, h, fwd, local):
    """Per-CTA timeline of the four slice GEMVs of a block step (%globaltimer stamps)
    in one replay of two captured steps, relative to the first q/k/v CTA's start of
    the first: per GEMV and mark, [min, median, max] over CTAs in us, and how many
    CTAs started more than 2 us after the GEMV's first."""
    nsm = torch.cuda.get_device_properties(local).multi_processor_count
    tr = torch.zeros(nsm * tpb.TP_BLOCK_TRACE_SLOTS, dtype=torch.int64, device="cuda")
    tpb.tp_block_set_trace(h, tr, tr.numel() * 8)
    g_tr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_tr):
        for _ in range(2):
            fwd()
    tpb.tp_block_set_trace(h, None, 0)
    g_tr.replay()
    torch.cuda.synchronize()
    del g_tr
    t = tr.view(nsm, -1).cpu().numpy().astype("float64")
    timeline = {}
    base = t[t[:, 0] > 0, 0].min()
    marks = ("start", "prev_done", "norm", "staged", "first_stage", "consumed", "end")
    merge_marks = ("start", "prev_done", "end")
    for name, c0, mk in (("qkv", 0, marks), ("wo", 7, marks), ("merge_wo", 28, merge_marks),
                         ("w13", 14, marks), ("w2", 21, marks), ("merge_w2", 31, merge_marks)):
        cols = t[:, c0:c0 + len(mk)]
        cols = cols[cols[:, 0] > 0]
        if not len(cols):
            continue
        timeline[name] = {m: [round(float(f((cols[:, k] - base) / 1e3)), 2)
                              for f in (min, statistics.median, max)]
                          for k, m in enumerate(mk)}
        st = (cols[:, 0] - cols[:, 0].min()) / 1e3
        timeline[name]["late_ctas"] = int((st > 2.0).sum())
    return timeline


def bench_block(args, world, rank, local):
    import torch

    import synth
    import tensor_llama_transformer_b200 as tpb
    from synth.device import DeviceBlock

    s = synth.C2
    B = s.batch
    inp = synth.block_inputs(synth.CONFIG_SEED["C2"], s)
    dev = DeviceBlock(inp)
    dims = tpb.make_dims(s.dim, s.n_heads, s.n_kv_heads, s.head_dim, s.ffn_dim, s.vocab, B,
                         s.max_seq, s.norm_eps, s.rope_theta)
    nbytes = tpb.tp_block_workspace_bytes(dims, s.n_slices, tpb.TP_PART_1D, 1)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    h = tpb.tp_block_create(dims, s.n_slices, tpb.TP_PART_1D, 1, tpb.make_weights(*dev.weights()),
                            ws, nbytes)
    x0 = dev.x.clone()

    def fwd():
        tpb.tp_block_forward(h, dev.x, dev.k_cache, dev.v_cache, dev.pos, B)

    # eager warm-up (module load, attribute setup), then capture
    for _ in range(3):
        fwd()
    torch.cuda.synchronize()
    K = max(1, args.steps)
    S = max(1, min(args.graph_steps, K))
    R = (K + S - 1) // S
    K = R * S
    nstage = len(STAGES) + 1
    # timed graph: S steps back to back, no extra nodes between kernels (so that
    # programmatic dependent launches overlap each kernel with its predecessor)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(S):
            fwd()
    # stage graph: the same S steps with a timing event before every stage; event
    # nodes serialise the stages, so these per-stage times are upper bounds
    evs = [make_events(torch, nstage) for _ in range(S)]
    arrs = [(ctypes.c_void_p * nstage)(*[e.cuda_event for e in ev]) for ev in evs]
    g_ev = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_ev):
        for i in range(S):
            tpb.tp_block_set_events(h, arrs[i], nstage)
            fwd()
    tpb.tp_block_set_events(h, None, 0)

    stream = torch.cuda.current_stream()
    for _ in range(max(1, (args.warmup + S - 1) // S)):
        g.replay()
    dev.x.copy_(x0)
    torch.cuda.synchronize()
    barrier(world)
    clocks = ClockSampler(local)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier(world)
    start.record(stream)
    for _ in range(R):
        g.replay()
    end.record(stream)
    end.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    ms = start.elapsed_time(end)
    # a timed region of a few ms gives the sampler few or no samples: keep the same
    # graph running (untimed) until it holds at least 20, at most 2 s more
    t_extra, extra_replays = time.perf_counter(), 0
    while clocks.count() < 20 and time.perf_counter() - t_extra < 2.0:
        g.replay()
        extra_replays += 1
        if extra_replays % 20 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()
    clk = clocks.stop()
    if clk is not None:
        clk["window"] = (f"the timed region ({ms:.1f} ms) and {extra_replays} more untimed replays "
                         f"of the same graph right after it")
    ms_max = allreduce_max(ms, world)
    # per-stage device time: one replay of the stage graph right after the timed region
    g_ev.replay()
    torch.cuda.synchronize()
    stage_ms = [0.0] * len(STAGES)
    for ev in evs:
        for i in range(len(STAGES)):
            stage_ms[i] += ev[i].elapsed_time(ev[i + 1]) / S
    stage_ms_max = [allreduce_max(v, world) for v in stage_ms]
    del g, g_ev

    timeline = gemv_timeline(torch, tpb, h, fwd, local)

    # end to end through the public API: host buffers, copies inside the timed region. A
    # step's inputs (x, then pos) sit in one pinned host buffer and one device buffer, as a
    # serving loop would pack them: one copy in, the forward on views of that buffer, and
    # the new x copied back.
    xbytes, pbytes = B * s.dim * 4, B * 4
    inh = torch.empty(xbytes + ((pbytes + 15) // 16) * 16, dtype=torch.uint8).pin_memory()
    inh[:xbytes].view(torch.float32).copy_(x0.cpu().reshape(-1))
    inh[xbytes:xbytes + pbytes].view(torch.int32).copy_(torch.from_numpy(inp.pos.copy()))
    ind = torch.empty(inh.numel(), dtype=torch.uint8, device="cuda")
    x_in = ind[:xbytes].view(torch.float32).view(B, s.dim)
    pos_in = ind[xbytes:xbytes + pbytes].view(torch.int32)
    outh = torch.empty((B, s.dim), dtype=torch.float32).pin_memory()

    def step_e2e():
        ind.copy_(inh, non_blocking=True)
        tpb.tp_block_forward(h, x_in, dev.k_cache, dev.v_cache, pos_in, B)
        outh.copy_(x_in, non_blocking=True)

    E = max(1, args.e2e_steps)
    for _ in range(3):
        step_e2e()
        stream.synchronize()
    barrier(world)
    t0 = time.perf_counter()
    for _ in range(E):
        step_e2e()
        stream.synchronize()
    e2e_eager_s = allreduce_max(time.perf_counter() - t0, world)
    # the same step as a serving loop runs it: one CUDA graph per step holding the copy of
    # the step's inputs from the pinned host buffer, the block forward (the same entry
    # point, captured) and the copy of the result back to pinned host memory; the host
    # waits for each step's result before the next replay
    g_e2e = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_e2e):
        step_e2e()
    for _ in range(3):
        g_e2e.replay()
        stream.synchronize()
    barrier(world)
    t0 = time.perf_counter()
    for _ in range(E):
        g_e2e.replay()
        torch.cuda.current_stream().synchronize()
    e2e_s = allreduce_max(time.perf_counter() - t0, world)
    del g_e2e
    tpb.tp_block_destroy(h)

    wbytes, kvbytes = block_bytes(s)
    step_s = ms_max / 1e3 / K
    hbm, bf16_tf, bf16_sus, peak_kind = peaks()
    w13_bytes = 2 * s.ffn_dim * s.dim * 2 + B * s.dim * (1 + 4 / 32) + B * s.ffn_dim * 4
    w13_s = stage_ms_max[STAGES.index("norm_w13_swiglu")] / 1e3
    # batch 1 (weight-streaming path): q/k/v GEMV, attention splits, W_O GEMV (which also
    # combines the splits), merge, W1/W3 GEMV, W2 GEMV, merge
    launches_per_step = 7
    res = {
        "tokens_per_s": world * B * K / (ms_max / 1e3), "ms_per_step": ms_max / K, "K": K,
        "block_gbs": (wbytes + kvbytes) / step_s / 1e9, "stage_us": {
            n: v * 1e3 for n, v in zip(STAGES, stage_ms_max)},
        "roofline": {"bound": "hbm", "achieved": w13_bytes / w13_s / 1e9, "peak": hbm,
                     "unit": "GB/s", "frac": w13_bytes / w13_s / 1e9 / hbm,
                     "traffic": W13_DRAM_BYTES,
                     "traffic_source": "dram__bytes_read.sum + dram__bytes_write.sum per "
                                       "launch (mean of 10 graph-replayed launches), ncu "
                                       "capture of this kernel in this workload",
                     "kernel": "k_gemv<1, EPI_SWIGLU, false, 1> (RMSNorm+Q8, W1/W3, SwiGLU)",
                     "algorithmic_bytes": w13_bytes, "peak_kind": peak_kind},
        "e2e": {"value": world * B * E / e2e_s, "unit": "tokens/s",
                "h2d_bytes_per_step": inh.numel(), "d2h_bytes_per_step": outh.numel() * 4,
                "how": "per step one CUDA graph replay: one copy of x and pos (packed in one "
                       "pinned buffer) to the device, tp_block_forward, copy of x back to "
                       "pinned host memory; host waits for every step's result",
                "eager_value": world * B * E / e2e_eager_s,
                "eager_how": "the same copies and tp_block_forward called from Python every step"},
        "gpu_launches": launches_per_step * K, "clocks": clk, "inp": inp,
        "gemv_timeline_us": timeline,
        "stage_sum_us": sum(stage_ms_max) * 1e3,
        "block_roofline_frac": (wbytes + kvbytes) / step_s / 1e9 / hbm,
    }
    return res


def bench_rank_block(args, world, rank, local):
    """The C2 block (Llama-2-7B shapes, Q8 sync, KV 1024, batch 1) with its slices
    spread over the ranks, one GPU each (tp_block_rank_step: three phases per step
    and two NCCL all-gathers of the sync buffers between them, every rank merging
    all slices in slice order). n = 4 slices, or one per rank when world > 4.
    Each rank's weights are its slices, drawn from its own seeded generator (a
    timing workload: parity of this path is tests/test_gpu_tensor_parallel.py)."""
    import torch
    import torch.distributed as dist

    import synth
    import tensor_llama_transformer_b200 as tpb
    from tensor_llama_transformer_b200 import tensor_parallel as tp

    s = synth.C2
    n = s.n_slices if s.n_slices % world == 0 else world
    B, D, F, H, Hkv, hd = s.batch, s.dim, s.ffn_dim, s.n_heads, s.n_kv_heads, s.head_dim
    if H % n or Hkv % n or n % world:
        return {"error": f"C2 does not split into {n} slices over {world} ranks"}
    gen = torch.Generator(device="cuda")
    gen.manual_seed(2000 + rank)
    Hr, Hkvr, Fr = H // world, Hkv // world, F // world
    w = {"attn_norm": torch.ones(D, device="cuda"), "ffn_norm": torch.ones(D, device="cuda")}
    for k, shp in (("wq", (Hr * hd, D)), ("wk", (Hkvr * hd, D)), ("wv", (Hkvr * hd, D)),
                   ("wo", (D, Hr * hd)), ("w1", (Fr, D)), ("w3", (Fr, D)), ("w2", (D, Fr))):
        w[k] = _randn_bf16(torch, gen, shp, s.w_std)
    kc = _randn_bf16(torch, gen, (B, Hkvr, s.max_seq, hd), 1.0)
    vc = _randn_bf16(torch, gen, (B, Hkvr, s.max_seq, hd), 1.0)
    gx = torch.Generator(device="cuda")
    gx.manual_seed(2999)  # the residual is replicated: the same values on every rank
    x = torch.randn((B, D), generator=gx, device="cuda")
    pos = torch.full((B,), s.pos, dtype=torch.int32, device="cuda")
    dims = tpb.make_dims(D, H, Hkv, hd, F, s.vocab, B, s.max_seq, s.norm_eps, s.rope_theta)
    rb = tp.RankBlock(dims, n, 1, rank, world, w)
    sync_bytes = tpb.tp_block_rank_sync_bytes(rb.h, B)

    def step():
        rb.forward(x, kc, vc, pos, B)

    for _ in range(5):
        step()
    torch.cuda.synchronize()
    dist.barrier()
    mode, g = "eager", None
    try:  # NCCL collectives inside a CUDA graph (the communicator exists after the warm-up)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(10):
                step()
        g.replay()
        torch.cuda.synchronize()
        mode = "graph"
    except Exception:
        g = None
        torch.cuda.synchronize()
    dist.barrier()
    reps = max(1, min(args.steps, 2000) // 10)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    dist.barrier()
    a.record()
    for _ in range(reps):
        if g is not None:
            g.replay()
        else:
            for _ in range(10):
                step()
    b.record()
    b.synchronize()
    torch.cuda.synchronize()
    dist.barrier()
    ms = allreduce_max(a.elapsed_time(b), world) / (10 * reps)
    err_off, _ = tpb.tp_block_buffer(rb.h, 7)
    err = int(rb.ws[err_off:err_off + 4].view(torch.int32).item())
    del g  # a graph holding NCCL calls goes before the process group
    rb.close()
    return {"world": world, "n_slices": n, "us_per_step": ms * 1e3, "tokens_per_s": B / (ms / 1e3),
            "mode": mode, "steps": 10 * reps, "pipeline_error": err,
            "exchange": "two NCCL all-gathers per step of every rank's Q8 sync buffers "
                        f"({sync_bytes} bytes per rank each)",
            "workload": "C2 block, batch 1, KV 1024, Q8 sync, slices spread over the ranks"}


def _randn_bf16(torch, gen, shape, std):
    out = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    flat = out.view(-1)
    step = 1 << 26
    for o in range(0, flat.numel(), step):
        n = min(step, flat.numel() - o)
        flat[o:o + n] = (torch.randn(n, generator=gen, device="cuda") * std).to(torch.bfloat16)
    return out


def _time_graph(torch, fn, steps_per_graph, replays, warm=2):
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(steps_per_graph):
            fn()
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(replays):
        g.replay()
    b.record()
    b.synchronize()
    ms = a.elapsed_time(b) / (steps_per_graph * replays)
    del g
    return ms


def bench_c4(args, kv_heads=None):
    """70B-shape GQA block (dim 8192, 64/8 heads, F 28672), batch 32, context 4096, n = 8;
    with kv_heads = 1 the multi-query form of the same block as one slice (64 query heads
    on one kv head: every group of 8 query heads streams the kv head's tiles; Pope et al.
    demo 3)."""
    import dataclasses

    import torch

    import synth
    import tensor_llama_transformer_b200 as tpb

    # one kv head cannot be split over slices by heads: the multi-query block is one slice
    s = synth.C4 if kv_heads is None else dataclasses.replace(synth.C4, n_kv_heads=kv_heads,
                                                              n_slices=1)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(1003)
    B, D, F, H, Hkv, hd = s.batch, s.dim, s.ffn_dim, s.n_heads, s.n_kv_heads, s.head_dim
    w = [torch.ones(D, device="cuda"), _randn_bf16(torch, gen, (H * hd, D), s.w_std),
         _randn_bf16(torch, gen, (Hkv * hd, D), s.w_std), _randn_bf16(torch, gen, (Hkv * hd, D), s.w_std),
         _randn_bf16(torch, gen, (D, H * hd), s.w_std), torch.ones(D, device="cuda"),
         _randn_bf16(torch, gen, (F, D), s.w_std), _randn_bf16(torch, gen, (F, D), s.w_std),
         _randn_bf16(torch, gen, (D, F), s.w_std)]
    kc = _randn_bf16(torch, gen, (B, Hkv, s.max_seq, hd), 1.0)
    vc = _randn_bf16(torch, gen, (B, Hkv, s.max_seq, hd), 1.0)
    x = torch.randn((B, D), generator=gen, device="cuda")
    pos = torch.full((B,), s.pos, dtype=torch.int32, device="cuda")
    dims = tpb.make_dims(D, H, Hkv, hd, F, s.vocab, B, s.max_seq, s.norm_eps, s.rope_theta)
    nb = tpb.tp_block_workspace_bytes(dims, s.n_slices, 1, 0)
    ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    h = tpb.tp_block_create(dims, s.n_slices, 1, 0, tpb.make_weights(*w), ws, nb)
    if args.profile == "c4":
        for _ in range(args.profile_steps):
            tpb.tp_block_forward(h, x, kc, vc, pos, B)
        torch.cuda.synchronize()
        tpb.tp_block_destroy(h)
        return {"profile": "c4", "steps": args.profile_steps}
    ms = _time_graph(torch, lambda: tpb.tp_block_forward(h, x, kc, vc, pos, B), 10, 5)
    tpb.tp_block_destroy(h)
    wb, kvb = block_bytes(s)
    hbm, _, _, kind = peaks()
    gbs = (wb + kvb) / (ms / 1e3) / 1e9
    return {"us_per_step": ms * 1e3, "tokens_per_s": B / (ms / 1e3), "hbm_gbs": gbs,
            "frac": gbs / hbm, "bytes_per_step": wb + kvb,
            "workload": f"C4{'' if kv_heads is None else ' multi-query'}: 70B-shape block, dim 8192, "
                        f"{s.n_heads}/{s.n_kv_heads} heads, SwiGLU 28672, batch 32, context 4096, "
                        f"n={s.n_slices}, float32 sync buffers"}


def bench_c2_prefill(args):
    """A 64-token prefill chunk of one sequence through the C2 block (Llama-2-7B
    shapes, n = 4, Q8 sync) after a 960-token prefix: tp_block_forward_seq, the
    slice products on the tensor cores with the 64 tokens as the GEMMs' N."""
    import torch

    import synth
    import tensor_llama_transformer_b200 as tpb

    s = synth.C2
    L, p0 = 64, 960
    gen = torch.Generator(device="cuda")
    gen.manual_seed(1011)
    D, F, H, Hkv, hd = s.dim, s.ffn_dim, s.n_heads, s.n_kv_heads, s.head_dim
    w = [torch.ones(D, device="cuda"), _randn_bf16(torch, gen, (H * hd, D), s.w_std),
         _randn_bf16(torch, gen, (Hkv * hd, D), s.w_std), _randn_bf16(torch, gen, (Hkv * hd, D), s.w_std),
         _randn_bf16(torch, gen, (D, H * hd), s.w_std), torch.ones(D, device="cuda"),
         _randn_bf16(torch, gen, (F, D), s.w_std), _randn_bf16(torch, gen, (F, D), s.w_std),
         _randn_bf16(torch, gen, (D, F), s.w_std)]
    kc = _randn_bf16(torch, gen, (1, Hkv, s.max_seq, hd), 1.0)
    vc = _randn_bf16(torch, gen, (1, Hkv, s.max_seq, hd), 1.0)
    x = torch.randn((L, D), generator=gen, device="cuda")
    pos = torch.arange(p0, p0 + L, dtype=torch.int32, device="cuda")
    seq = torch.zeros(L, dtype=torch.int32, device="cuda")
    dims = tpb.make_dims(D, H, Hkv, hd, F, s.vocab, L, s.max_seq, s.norm_eps, s.rope_theta)
    nb = tpb.tp_block_workspace_bytes(dims, s.n_slices, 1, 1)
    ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    h = tpb.tp_block_create(dims, s.n_slices, 1, 1, tpb.make_weights(*w), ws, nb)
    if args.profile == "c2prefill":
        for _ in range(args.profile_steps):
            tpb.tp_block_forward_seq(h, x, kc, vc, pos, seq, 1, L)
        torch.cuda.synchronize()
        tpb.tp_block_destroy(h)
        return {"profile": "c2prefill", "steps": args.profile_steps}
    ms = _time_graph(torch, lambda: tpb.tp_block_forward_seq(h, x, kc, vc, pos, seq, 1, L), 10, 5)
    tpb.tp_block_destroy(h)
    wb, _ = block_bytes(s)
    kvb = 2 * Hkv * (p0 + L) * hd * 2  # the sequence's cache, read once from HBM
    hbm, _, _, kind = peaks()
    gbs = (wb + kvb) / (ms / 1e3) / 1e9
    return {"us_per_chunk": ms * 1e3, "tokens_per_s": L / (ms / 1e3), "hbm_gbs": gbs,
            "frac": gbs / hbm, "bytes_per_chunk": wb + kvb,
            "workload": "C2 block (Llama-2-7B shapes, n=4, Q8 sync), one sequence: a 64-token "
                        "prefill chunk at positions 960..1023"}


def bench_c2_persistent(args):
    """The C2 block (Llama-2-7B shapes, n = 4, Q8 sync, KV 1024, batch 1) as one persistent
    kernel per step (tp_block_set_persistent), for comparison with the headline's
    kernel-per-step graph."""
    import torch

    import synth
    import tensor_llama_transformer_b200 as tpb

    s = synth.C2
    gen = torch.Generator(device="cuda")
    gen.manual_seed(1001)
    B, D, F, H, Hkv, hd = s.batch, s.dim, s.ffn_dim, s.n_heads, s.n_kv_heads, s.head_dim
    w = [torch.ones(D, device="cuda"), _randn_bf16(torch, gen, (H * hd, D), s.w_std),
         _randn_bf16(torch, gen, (Hkv * hd, D), s.w_std), _randn_bf16(torch, gen, (Hkv * hd, D), s.w_std),
         _randn_bf16(torch, gen, (D, H * hd), s.w_std), torch.ones(D, device="cuda"),
         _randn_bf16(torch, gen, (F, D), s.w_std), _randn_bf16(torch, gen, (F, D), s.w_std),
         _randn_bf16(torch, gen, (D, F), s.w_std)]
    kc = _randn_bf16(torch, gen, (B, Hkv, s.max_seq, hd), 1.0)
    vc = _randn_bf16(torch, gen, (B, Hkv, s.max_seq, hd), 1.0)
    x = torch.randn((B, D), generator=gen, device="cuda")
    pos = torch.full((B,), s.pos, dtype=torch.int32, device="cuda")
    dims = tpb.make_dims(D, H, Hkv, hd, F, s.vocab, B, s.max_seq, s.norm_eps, s.rope_theta)
    nb = tpb.tp_block_workspace_bytes(dims, s.n_slices, 1, 1)
    ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    h = tpb.tp_block_create(dims, s.n_slices, 1, 1, tpb.make_weights(*w), ws, nb)
    tpb.tp_block_set_persistent(h, 1)
    if args.profile == "c2p":
        for _ in range(args.profile_steps):
            tpb.tp_block_forward(h, x, kc, vc, pos, B)
        torch.cuda.synchronize()
        tpb.tp_block_destroy(h)
        return {"profile": "c2p", "steps": args.profile_steps}
    ms = _time_graph(torch, lambda: tpb.tp_block_forward(h, x, kc, vc, pos, B), 100, 20)
    err = int(ws[tpb.tp_block_buffer(h, 7)[0]:][:4].view(torch.int32).item())
    # one traced step: per-phase durations (median over CTAs, from kernel start)
    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    tr = torch.zeros(nsm * tpb.TP_BLOCK_TRACE_SLOTS, dtype=torch.int64, device="cuda")
    tpb.tp_block_set_trace(h, tr, tr.numel() * 8)
    tpb.tp_block_forward(h, x, kc, vc, pos, B)
    torch.cuda.synchronize()
    tpb.tp_block_set_trace(h, None, 0)
    tpb.tp_block_destroy(h)
    t = tr.view(nsm, -1).cpu().numpy().astype("float64")
    t = t[t[:, 0] > 0]
    base = t[:, 0].min()
    marks = {"qkv_end": 1, "barrier1": 2, "attention_end": 3, "barrier2": 4, "wo_end": 5,
             "barrier3": 6, "merge_barrier": 13, "w13_staged": 14, "w13_end": 7, "barrier5": 8,
             "w2_end": 9, "barrier6": 10, "final_merge_end": 11}
    phase_us = {k: round(float(statistics.median((t[:, i] - base) / 1e3)), 2) for k, i in marks.items()}
    phase_us["kernel_end_max"] = round(float(((t[:, 11] - base) / 1e3).max()), 2)
    wb, kvb = block_bytes(s)
    hbm, _, _, kind = peaks()
    gbs = (wb + kvb) / (ms / 1e3) / 1e9
    return {"us_per_step": ms * 1e3, "tokens_per_s": B / (ms / 1e3), "hbm_gbs": gbs,
            "frac": gbs / hbm, "pipeline_error": err, "phase_end_us_median": phase_us,
            "workload": "C2 block as one persistent kernel per step (same shapes as the headline)"}


def bench_c2_q8w(args):
    """The C2 block with int8 weights (tp_block_create_q8w): Q8 codes and scales for every
    matrix, Q8 activations, integer block dot products; same shapes and batch 1."""
    import torch

    import synth
    import tensor_llama_transformer_b200 as tpb

    s = synth.C2
    gen = torch.Generator(device="cuda")
    gen.manual_seed(1001)
    B, D, F, H, Hkv, hd = s.batch, s.dim, s.ffn_dim, s.n_heads, s.n_kv_heads, s.head_dim
    mats = {k: _randn_bf16(torch, gen, shp, s.w_std) for k, shp in
            (("wq", (H * hd, D)), ("wk", (Hkv * hd, D)), ("wv", (Hkv * hd, D)), ("wo", (D, H * hd)),
             ("w1", (F, D)), ("w3", (F, D)), ("w2", (D, F)))}
    qd = {}
    for k, t in mats.items():
        f = t.float()
        q = torch.empty(f.shape, dtype=torch.int8, device="cuda")
        d = torch.empty((f.shape[0], f.shape[1] // 32), dtype=torch.float32, device="cuda")
        tpb.tp_quantize_q8(f, q, d, f.numel())
        qd[k] = (q, d)
        del f
    del mats
    ones = torch.ones(D, device="cuda")
    kc = _randn_bf16(torch, gen, (B, Hkv, s.max_seq, hd), 1.0)
    vc = _randn_bf16(torch, gen, (B, Hkv, s.max_seq, hd), 1.0)
    x = torch.randn((B, D), generator=gen, device="cuda")
    pos = torch.full((B,), s.pos, dtype=torch.int32, device="cuda")
    dims = tpb.make_dims(D, H, Hkv, hd, F, s.vocab, B, s.max_seq, s.norm_eps, s.rope_theta)
    nb = tpb.tp_block_workspace_bytes(dims, s.n_slices, 1, 1)
    ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    w = tpb.make_weights_q8(ones, *qd["wq"], *qd["wk"], *qd["wv"], *qd["wo"], ones, *qd["w1"],
                            *qd["w3"], *qd["w2"])
    h = tpb.tp_block_create_q8w(dims, s.n_slices, 1, 1, w, ws, nb)
    if args.profile == "c2q8w":
        for _ in range(args.profile_steps):
            tpb.tp_block_forward(h, x, kc, vc, pos, B)
        torch.cuda.synchronize()
        tpb.tp_block_destroy(h)
        return {"profile": "c2q8w", "steps": args.profile_steps}
    fwd = lambda: tpb.tp_block_forward(h, x, kc, vc, pos, B)  # noqa: E731
    ms = _time_graph(torch, fwd, 100, 20)
    timeline = gemv_timeline(torch, tpb, h, fwd, torch.cuda.current_device())
    err = int(ws[tpb.tp_block_buffer(h, 7)[0]:][:4].view(torch.int32).item())
    tpb.tp_block_destroy(h)
    wb_bf16, kvb = block_bytes(s)
    wb = wb_bf16 // 2 + wb_bf16 // 2 // 32 * 4  # int8 codes + a float32 scale per 32
    hbm, _, _, kind = peaks()
    gbs = (wb + kvb) / (ms / 1e3) / 1e9
    return {"us_per_step": ms * 1e3, "tokens_per_s": B / (ms / 1e3), "hbm_gbs": gbs,
            "frac": gbs / hbm, "bytes_per_step": wb + kvb, "pipeline_error": err,
            "gemv_timeline_us": timeline,
            "workload": "C2 block with int8 weights (Q8 codes + float32 scales per 32) and Q8 "
                        "activations, batch 1, n=4"}


def bench_c3(args, B):
    """Full 32-layer Llama-2-7B-shaped decode step (embedding -> logits), context 4096, n = 8."""
    import torch

    import synth
    import tensor_llama_transformer_b200 as tpb

    s = synth.C3
    gen = torch.Generator(device="cuda")
    gen.manual_seed(1002)
    D, F, H, Hkv, hd, L, V = s.dim, s.ffn_dim, s.n_heads, s.n_kv_heads, s.head_dim, s.n_layers, s.vocab
    ones = torch.ones(D, device="cuda")
    layers, keep = [], []
    for _ in range(L):
        t = [_randn_bf16(torch, gen, shp, s.w_std) for shp in
             ((H * hd, D), (Hkv * hd, D), (Hkv * hd, D), (D, H * hd), (F, D), (F, D), (D, F))]
        keep.append(t)
        layers.append(tpb.make_weights(ones, t[0], t[1], t[2], t[3], ones, t[4], t[5], t[6]))
    emb = _randn_bf16(torch, gen, (V, D), s.w_std)
    wcls = _randn_bf16(torch, gen, (V, D), s.w_std)
    kc = _randn_bf16(torch, gen, (L, B, Hkv, s.max_seq, hd), 1.0)
    vc = _randn_bf16(torch, gen, (L, B, Hkv, s.max_seq, hd), 1.0)
    toks = torch.randint(0, V, (B,), generator=gen, device="cuda", dtype=torch.int32)
    pos = torch.full((B,), s.pos, dtype=torch.int32, device="cuda")
    logits = torch.empty((B, V), dtype=torch.float32, device="cuda")
    dims = tpb.make_dims(D, H, Hkv, hd, F, V, B, s.max_seq, s.norm_eps, s.rope_theta)
    nb = tpb.tp_model_workspace_bytes(dims, L, s.n_slices, 1, 0)
    ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    m = tpb.tp_model_create(dims, L, s.n_slices, 1, 0, layers, emb, ones, wcls, ws, nb)
    if args.profile == "c3b1":
        for _ in range(args.profile_steps):
            tpb.tp_model_forward(m, toks, kc, vc, pos, B, logits)
        torch.cuda.synchronize()
        tpb.tp_model_destroy(m)
        return {"profile": "c3b1", "steps": args.profile_steps}
    ms = _time_graph(torch, lambda: tpb.tp_model_forward(m, toks, kc, vc, pos, B, logits), 3, 5)
    tpb.tp_model_destroy(m)
    wb = L * block_bytes(s)[0] + V * D * 2  # every layer's weights + the classifier
    kvb = L * 2 * B * Hkv * (s.pos + 1) * hd * 2
    hbm, _, _, kind = peaks()
    gbs = (wb + kvb) / (ms / 1e3) / 1e9
    return {"ms_per_step": ms, "tokens_per_s": B / (ms / 1e3), "hbm_gbs": gbs, "frac": gbs / hbm,
            "bytes_per_step": wb + kvb,
            "workload": f"C3: 32-layer Llama-2-7B-shaped decode, vocab 32000, context 4096, n=8, "
                        f"batch {B}"}


def bench_ffn(args):
    """PaLM FFN (E 18432, F 73728, B 512, ReLU) through tp_ffn_forward; TFLOP/s per form."""
    import torch

    import tensor_llama_transformer_b200 as tpb

    B, E, F = 512, 18432, 73728
    gen = torch.Generator(device="cuda")
    gen.manual_seed(1004)

    def randn_bf16(shape, std):
        out = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
        rows = max(1, (1 << 26) // shape[1])
        for r0 in range(0, shape[0], rows):
            r1 = min(shape[0], r0 + rows)
            out[r0:r1] = (torch.randn((r1 - r0, shape[1]), generator=gen, device="cuda") * std).to(
                torch.bfloat16)
        return out

    X = randn_bf16((B, E), 1.0)
    W1 = randn_bf16((F, E), 0.01)
    W2 = randn_bf16((E, F), 0.01)
    Y = torch.empty((B, E), dtype=torch.float32, device="cuda")
    flops = 2.0 * B * 2 * E * F
    out = {}
    _, bf16_tf, _, peak_kind = peaks()
    # faithful: every slice's partial formed on its own and summed in slice order (in
    # the GEMM epilogue), _q8 with the Q8 round trip of every partial
    forms = [("fused", tpb.TP_PART_1D, 64, 1, 1, tpb.TP_MERGE_FUSED, 0),
             ("1d64_faithful", tpb.TP_PART_1D, 64, 1, 1, tpb.TP_MERGE_FAITHFUL, 0),
             ("1d64_faithful_q8", tpb.TP_PART_1D, 64, 1, 1, tpb.TP_MERGE_FAITHFUL, 1),
             ("2d8x8_faithful", tpb.TP_PART_2D, 64, 8, 8, tpb.TP_MERGE_FAITHFUL, 0),
             ("2d8x8_faithful_q8", tpb.TP_PART_2D, 64, 8, 8, tpb.TP_MERGE_FAITHFUL, 1)]
    for name, part, n, gx, gy, merge, quant in forms:
        desc = tpb.tp_ffn_desc(B, E, F, tpb.TP_BF16, tpb.TP_ACT_RELU, part, n, gx, gy, quant, merge)
        nb = tpb.tp_ffn_workspace_bytes(desc)
        ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
        for _ in range(2):
            tpb.tp_ffn_forward(desc, X, W1, None, W2, Y, ws, nb)
        torch.cuda.synchronize()
        t = []
        for _ in range(max(1, args.ffn_iters)):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            tpb.tp_ffn_forward(desc, X, W1, None, W2, Y, ws, nb)
            b.record()
            b.synchronize()
            t.append(a.elapsed_time(b))
        err = int(ws[:4].view(torch.int32).item())
        ms = statistics.median(t)
        out[name] = {"ms": ms, "tflops": flops / (ms / 1e3) / 1e12,
                     "frac": flops / (ms / 1e3) / 1e12 / bf16_tf, "pipeline_error": err}
        del ws
        torch.cuda.empty_cache()
    out["peak_tflops"] = bf16_tf
    out["peak_kind"] = peak_kind
    out["config"] = "E=18432 F=73728 B=512 ReLU, bf16 weights/activations, fp32 accumulate"
    return out


def profile_ffn(args):
    """A few forwards of the PaLM-shaped FFN (B 512, E 18432, ReLU, 1D) with F cut to
    --profile-ffn-f, so that a full-section capture of one tcgen05 GEMM launch holds a
    few GB on the device (F 18432: 1.36 GB of weights). --profile-ffn-form: fused (64
    slices), or faithful / faithful_q8 over F / 1152 slices (16 at F 18432), the slice
    width of the full-size 1D-64 form, so the segment-sum GEMM does the same work per
    segment as at full size."""
    import torch

    import tensor_llama_transformer_b200 as tpb

    B, E, F = 512, 18432, args.profile_ffn_f
    gen = torch.Generator(device="cuda")
    gen.manual_seed(1004)
    X = _randn_bf16(torch, gen, (B, E), 1.0)
    W1 = _randn_bf16(torch, gen, (F, E), 0.01)
    W2 = _randn_bf16(torch, gen, (E, F), 0.01)
    Y = torch.empty((B, E), dtype=torch.float32, device="cuda")
    form = args.profile_ffn_form
    n = 64 if form == "fused" else max(1, F // 1152)
    merge = tpb.TP_MERGE_FUSED if form == "fused" else tpb.TP_MERGE_FAITHFUL
    desc = tpb.tp_ffn_desc(B, E, F, tpb.TP_BF16, tpb.TP_ACT_RELU, tpb.TP_PART_1D, n, 1, 1,
                           int(form == "faithful_q8"), merge)
    nb = tpb.tp_ffn_workspace_bytes(desc)
    ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    for _ in range(args.profile_steps):
        tpb.tp_ffn_forward(desc, X, W1, None, W2, Y, ws, nb)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    tpb.tp_ffn_forward(desc, X, W1, None, W2, Y, ws, nb)
    b.record()
    b.synchronize()
    ms = a.elapsed_time(b)
    flops = 2.0 * B * 2 * E * F
    return {"profile": "ffn", "form": form, "n_slices": n, "steps": args.profile_steps + 1, "B": B,
            "E": E, "F": F,
            "last_forward_ms": ms, "tflops": flops / (ms / 1e3) / 1e12,
            "pipeline_error": int(ws[:4].view(torch.int32).item())}


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    import torch

    if not torch.cuda.is_available():
        print(json.dumps({"metric": METRIC, "error": "no CUDA device"}))
        return 1
    if args.profile:
        fn = {"c4": bench_c4, "c3b1": lambda a: bench_c3(a, 1), "c2p": bench_c2_persistent,
              "c2q8w": bench_c2_q8w, "c2prefill": bench_c2_prefill, "ffn": profile_ffn}
        print(json.dumps(fn[args.profile](args)))
        return 0
    world, rank, local = dist_setup()
    res = bench_block(args, world, rank, local)
    multi_rank = None
    if world > 1 or args.rank_exchange:
        own_group = False
        try:
            import torch.distributed as dist

            if not dist.is_initialized():  # one rank: a one-rank NCCL group
                import datetime
                import socket

                sk = socket.socket()
                sk.bind(("127.0.0.1", 0))
                port = sk.getsockname()[1]
                sk.close()
                dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                                        world_size=1, timeout=datetime.timedelta(seconds=120),
                                        device_id=torch.device("cuda", local))
                own_group = True
            multi_rank = bench_rank_block(args, world, rank, local)
        except Exception as e:  # reported, not fatal: the headline does not depend on it
            multi_rank = {"error": str(e)[:200]}
        if own_group:
            dist.destroy_process_group()
        torch.cuda.empty_cache()
    ffn = None if args.no_ffn else bench_ffn(args)
    extra = None
    if not args.no_extra:
        import torch

        runs = [("c2_block_persistent", bench_c2_persistent), ("c2_block_int8_weights", bench_c2_q8w),
                ("c2_prefill_chunk64", bench_c2_prefill), ("c4_block", bench_c4),
                ("c4_block_mqa", lambda a: bench_c4(a, kv_heads=1)),
                ("c3_model_b1", lambda a: bench_c3(a, 1)), ("c3_model_b16", lambda a: bench_c3(a, 16))]
        want = set(args.extras.split(",")) if args.extras else None
        extra = {}
        for name, fn in runs:
            if want is not None and name not in want:
                continue
            try:
                extra[name] = fn(args)
            except Exception as e:  # reported, not fatal: the headline does not depend on it
                extra[name] = {"error": str(e)[:200]}
            torch.cuda.empty_cache()
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import synth

        tps, n, el, cores, _ = time_oracle(res["inp"], synth.C2, args.cpu_seconds)
        cpu = {"value": tps, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"{n} full C2 block decode steps (batch 1) in {el:.1f} s"}
    if rank == 0:
        line = {
            "metric": METRIC, "value": res["tokens_per_s"], "unit": "tokens/s", "n_gpus": world,
            "steps": res["K"], "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "dtype_detail": "bf16 weights, fp32 activations and accumulation, int8 Q8 sync buffers",
            "data": "synthetic",
            "config": dict(CONFIG),
            "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2 (404.75 MB of weights per step), no flush",
            "hbm_gbs": res["block_gbs"], "block_roofline_frac": res["block_roofline_frac"],
            "stage_us": res["stage_us"], "stage_sum_us": res["stage_sum_us"],
            "gemv_timeline_us": res["gemv_timeline_us"],
            "gemv_timeline_note": "one replay of a captured step: per slice GEMV, [min, median, "
                                  "max] over CTAs (us from the first q/k/v CTA's start) of its "
                                  "start, previous kernel complete, RMSNorm scale known, "
                                  "activations staged, first weight stage arrived, last stage "
                                  "consumed, end",
            "stage_note": "per-stage CUDA-event times from a replay of the same steps with an event "
                          "before every stage (serialised, so upper bounds); value and ms_per_step "
                          "come from the event-free graph; each merge stage is one k_merge "
                          "launch (the slices' partials into the residual)",
            "pdl": os.environ.get("TP_PDL", "1") != "0",
            "roofline": res["roofline"], "cpu_baseline": cpu,
            "e2e": res["e2e"], "gpu_launches": res["gpu_launches"], "clocks": res["clocks"],
            "ffn_b512": ffn,
            "multi_rank": multi_rank,
            "extra": extra,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
