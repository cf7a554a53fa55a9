"""Analytical partitioning cost model after Pope et al., "Efficiently Scaling Transformer
Inference" (CS349E lecture 4 script ``03_pope_partitioning.py``).

Bandwidth-only estimates for choosing how to split a transformer across chips:
the FFN's communication under 1D and 2D weight-stationary layouts and under the
weight-gathered layout used for prefill (demo 2), the
per-chip weight-read and compute times that communication competes with, the
longest context a KV-cache budget holds under the ways of splitting multi-query
attention, and a roofline lower bound on decode latency. Times follow the
script's convention: the papers' "elements / bandwidth" multiplied by the bytes
per element (bf16 = 2). Host-side arithmetic only; nothing here runs on the GPU.

Defaults are the TPU v4 figures the script takes from the paper (275 TFLOP/s
bf16, 32 GiB and 1200 GB/s HBM, 270 GB/s interconnect) and the PaLM 540B shape
(118 layers, E 18432, F 73728, 64 heads of 128, or one shared KV head of 256
under multi-query attention). ``Chip`` can describe any part, e.g. a B200 from
measured peaks.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

BF16 = 2


@dataclass(frozen=True)
class Chip:
    peak_flops: float  # dense bf16 FLOP/s
    mem_bw: float      # HBM bytes/s
    mem_cap: float     # HBM bytes
    link_bw: float     # inter-chip bytes/s per chip


TPU_V4 = Chip(peak_flops=275e12, mem_bw=1.2e12, mem_cap=32 * 2 ** 30, link_bw=270e9)


@dataclass(frozen=True)
class Model:
    layers: int
    E: int
    F: int
    heads: int
    d_head_mha: int
    d_head_mqa: int
    params: float


PALM_540B = Model(layers=118, E=18432, F=73728, heads=64, d_head_mha=128, d_head_mqa=256,
                  params=540e9)


def ffn_comm_1d(tokens: int, E: int, link_bw: float, dtype_bytes: int = BF16) -> float:
    """1D weight-stationary FFN (split along F only): every chip all-gathers and
    reduce-scatters a whole [tokens, E] activation per layer, 2 * tokens * E
    elements over its link, whatever the number of chips."""
    return 2.0 * tokens * E * dtype_bytes / link_bw


def ffn_comm_2d(tokens: int, E: int, F: int, n_chips: int, link_bw: float,
                dtype_bytes: int = BF16) -> float:
    """2D weight-stationary FFN (split along E and F, roughly square blocks per
    chip): activations are gathered along one mesh axis only, so the traffic falls
    as 1 / sqrt(n). Reading taken: 4 * tokens * sqrt(E * F / n) elements per
    layer, which for the paper's F = 4 E models is 8 * tokens * E / sqrt(n) and
    equals the 1D traffic at n = 16 (sqrt(n) = 4)."""
    return 4.0 * tokens * math.sqrt(E * F / n_chips) * dtype_bytes / link_bw


def ffn_comm_gathered(tokens: int, E: int, F: int, n_chips: int, link_bw: float,
                      dtype_bytes: int = BF16) -> tuple[float, float]:
    """Weight-gathered FFN (Pope et al., the prefill layout of demo 2): the weights
    are all-gathered over N of the n chips and the activations exchanged over the
    rest, 2 * tokens * E / N + 2 * N * E * F / n elements per layer, least at
    N = sqrt(tokens * n / F). Reading taken: this form, which the page does not
    print but whose statements it meets -- traffic growing as sqrt(tokens), equal
    to the 2D weight-stationary traffic at tokens = F / 4, and the optimal N the
    page states. Returns (seconds, N at the optimum, not rounded)."""
    N = math.sqrt(tokens * n_chips / F)
    elems = 2.0 * tokens * E / N + 2.0 * N * E * F / n_chips
    return elems * dtype_bytes / link_bw, N


def ffn_layout(tokens: int, E: int, F: int, n_chips: int, link_bw: float) -> str:
    """'gathered' when moving weights is cheaper than moving activations
    (prefill-sized token counts), else 'stationary' (2D weight-stationary)."""
    t_g, _ = ffn_comm_gathered(tokens, E, F, n_chips, link_bw)
    return "gathered" if t_g < ffn_comm_2d(tokens, E, F, n_chips, link_bw) else "stationary"


def ffn_weight_read(E: int, F: int, layers: int, n_chips: int, mem_bw: float,
                    dtype_bytes: int = BF16) -> float:
    """Per-chip time to read its share of the FFN weights (two E x F matrices)."""
    return 2.0 * E * F * dtype_bytes * layers / n_chips / mem_bw


def ffn_compute(tokens: int, E: int, F: int, layers: int, n_chips: int,
                peak_flops: float) -> float:
    """Per-chip FFN compute time: 2 FLOPs per multiply-add, two E x F matrices."""
    return 2.0 * tokens * 2 * E * F * layers / n_chips / peak_flops


def kv_bytes_per_token(m: Model, multi_query: bool, dtype_bytes: int = BF16) -> float:
    """K and V of one token over all layers: every head's under multi-head
    attention, the one shared head's under multi-query attention."""
    if multi_query:
        return 2.0 * m.layers * m.d_head_mqa * dtype_bytes
    return 2.0 * m.layers * m.heads * m.d_head_mha * dtype_bytes


def max_context(m: Model, chip: Chip, n_chips: int, batch: int, layout: str,
                kv_fraction: float = 0.30) -> int:
    """Longest context whose KV cache fits in `kv_fraction` of all chips' memory.
    layout: 'mha' (multi-head, split by heads: no copies), 'mqa_heads' (multi-query
    split by heads: the one KV head is copied to every chip), 'mqa_batch'
    (multi-query split by batch: one copy)."""
    budget = n_chips * chip.mem_cap * kv_fraction
    if layout == "mha":
        per, copies = kv_bytes_per_token(m, False), 1
    elif layout == "mqa_heads":
        per, copies = kv_bytes_per_token(m, True), n_chips
    elif layout == "mqa_batch":
        per, copies = kv_bytes_per_token(m, True), 1
    else:
        raise ValueError(layout)
    return int(budget / (batch * per * copies))


@dataclass(frozen=True)
class DecodeBound:
    weights: float   # s, reading every chip's share of the weights
    kv: float        # s, reading the KV cache
    compute: float   # s
    comm: float      # s, 2D weight-stationary FFN traffic (bandwidth term only)
    bound: float     # s, max(weights + kv, compute) + comm


def decode_bound(m: Model, chip: Chip, n_chips: int, batch: int, context: int,
                 weight_bytes: float) -> DecodeBound:
    """Roofline lower bound on one decode step of a multi-query model split 2D
    weight-stationary over `n_chips`: memory time (weights + KV) against compute,
    plus the FFN communication. Launch latencies, imperfect overlap and small
    operations are not in it, which is why measured steps take 2-4 times this."""
    t_w = m.params * weight_bytes / (n_chips * chip.mem_bw)
    t_kv = batch * context * kv_bytes_per_token(m, True) / n_chips / chip.mem_bw
    t_fl = 2.0 * m.params * batch / (n_chips * chip.peak_flops)
    t_comm = ffn_comm_2d(batch, m.E, m.F, n_chips, chip.link_bw) * m.layers
    return DecodeBound(t_w, t_kv, t_fl, t_comm, max(t_w + t_kv, t_fl) + t_comm)


def cost_chip_ms_per_token(n_chips: int, step_seconds: float, batch: int) -> float:
    """Serving cost: chips x milliseconds per step / tokens per step."""
    return n_chips * step_seconds * 1e3 / batch
