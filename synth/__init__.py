"""Seeded synthetic inputs shared by the CPU oracle and the CUDA path.

This module only *generates numbers*: it holds none of the decoder-block
arithmetic. Every tensor is a pure function of (config seed, tensor name,
element index), so any sub-range of a tensor (one batch row of a KV cache,
one layer of a 32-layer model) can be regenerated on its own, bit for bit the
same; the tensors are made here, on the host, and copied to the device.

Generator (counter based):
  * SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
    generators", OOPSLA 2014): ``mix(z)`` is its output finaliser, and element
    ``i`` of a stream with key ``k`` is ``mix(k + (i + 1) * 0x9E3779B97F4A7C15)``
    computed modulo 2**64.
  * The stream key of a tensor is ``mix(seed * GAMMA ^ crc32(name))``.
  * A standard-normal sample is ``NORMAL_TABLE[h >> 48]``: a 65,536-entry
    inverse-CDF table, ``Phi^-1((j + 0.5) / 65536)`` rounded to float32. The
    samples are therefore normal quantiles, truncated at about +/-4.32 sigma.
  * ``N(0, sigma)`` in float32 is ``float32(table[j] * float32(sigma))`` (one
    IEEE round-to-nearest multiply); in bf16 it is that value rounded to
    bf16 with round-to-nearest-even.
  * Token ids uniform in ``[0, V)`` are ``((h >> 32) * V) >> 32``.

Only integer operations and one correctly rounded float multiply are used, so
the device fill reproduces these bytes exactly.
"""
from __future__ import annotations

import os
import zlib
from dataclasses import dataclass, field

import numpy as np

GAMMA = 0x9E3779B97F4A7C15
M64 = (1 << 64) - 1
_C1 = np.uint64(0xBF58476D1CE4E5B9)
_C2 = np.uint64(0x94D049BB133111EB)


def _mix_int(z: int) -> int:
    z &= M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
    return z ^ (z >> 31)


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _C1
    z = (z ^ (z >> np.uint64(27))) * _C2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, name: str) -> int:
    """64-bit key of the stream that tensor ``name`` of config ``seed`` draws from."""
    return _mix_int(((seed * GAMMA) & M64) ^ zlib.crc32(name.encode()))


def raw64(key: int, start: int, count: int) -> np.ndarray:
    """Elements ``start .. start+count-1`` of stream ``key`` as uint64."""
    i = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(key) + i * np.uint64(GAMMA)
        return _mix(z)


def _build_normal_table() -> np.ndarray:
    from scipy.special import ndtri

    j = np.arange(65536, dtype=np.float64)
    return ndtri((j + 0.5) / 65536.0).astype(np.float32)


NORMAL_TABLE = _build_normal_table()


# ---------------------------------------------------------------------------
# bf16 storage helpers (bf16 is stored as its uint16 bit pattern on the host)
# ---------------------------------------------------------------------------

def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (round to nearest, ties to even); returns uint16 bits."""
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ---------------------------------------------------------------------------
# generators
# ---------------------------------------------------------------------------

_CHUNK = 1 << 22


def _parallel_fill(out: np.ndarray, fill, n: int):
    """Run ``fill(offset, count)`` over chunks of ``out`` on a thread pool."""
    spans = [(o, min(_CHUNK, n - o)) for o in range(0, n, _CHUNK)]
    if len(spans) <= 1:
        for o, c in spans:
            fill(o, c)
        return out
    import concurrent.futures as cf

    workers = min(len(spans), max(1, len(os.sched_getaffinity(0))))
    with cf.ThreadPoolExecutor(max_workers=workers) as ex:
        list(ex.map(lambda oc: fill(*oc), spans))
    return out


def normal_f32(seed: int, name: str, shape, std: float = 1.0, start: int = 0) -> np.ndarray:
    """float32 samples of N(0, std) for tensor ``name``; element 0 is stream index ``start``."""
    n = int(np.prod(shape))
    key = stream_key(seed, name)
    out = np.empty(n, dtype=np.float32)
    s = np.float32(std)

    def fill(o, c):
        h = raw64(key, start + o, c)
        out[o:o + c] = NORMAL_TABLE[(h >> np.uint64(48)).astype(np.int64)] * s

    _parallel_fill(out, fill, n)
    return out.reshape(shape)


def normal_bf16(seed: int, name: str, shape, std: float = 1.0, start: int = 0) -> np.ndarray:
    """bf16 bit patterns (uint16) of N(0, std) samples for tensor ``name``."""
    n = int(np.prod(shape))
    key = stream_key(seed, name)
    out = np.empty(n, dtype=np.uint16)
    s = np.float32(std)

    def fill(o, c):
        h = raw64(key, start + o, c)
        out[o:o + c] = f32_to_bf16_bits(NORMAL_TABLE[(h >> np.uint64(48)).astype(np.int64)] * s)

    _parallel_fill(out, fill, n)
    return out.reshape(shape)


def uniform_ids(seed: int, name: str, count: int, high: int) -> np.ndarray:
    """int32 ids uniform in [0, high)."""
    h = raw64(stream_key(seed, name), 0, count)
    return (((h >> np.uint64(32)) * np.uint64(high)) >> np.uint64(32)).astype(np.int32)


# ---------------------------------------------------------------------------
# workload shapes (sizes only; the arithmetic lives elsewhere)
# ---------------------------------------------------------------------------

@dataclass(frozen=True)
class BlockShape:
    """Shape of one Llama-style decoder block and its decode step."""

    dim: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    ffn_dim: int
    vocab: int
    max_seq: int
    batch: int
    n_slices: int
    sync_quant: bool
    pos: int
    n_layers: int = 1
    norm_eps: float = 1e-5
    rope_theta: float = 1e4
    w_std: float = 0.02
    kv_std: float = 1.0
    partition: int = 1  # 1 = 1D, 2 = 2D (FFN only)


@dataclass(frozen=True)
class FfnShape:
    """Shape of a two-matrix (or SwiGLU) feed-forward layer partitioned n ways."""

    batch: int
    E: int
    F: int
    dtype: str  # "f32" | "bf16"
    act: str  # "relu" | "swiglu"
    n_slices: int
    grid_x: int = 1
    grid_y: int = 1
    partition: int = 1
    x_std: float = 1.0
    w_std: float = 1.0
    sync_quant: bool = False


SEED_BASE = 1000

# The five workloads. C1 follows the ggmlR two-stage ReLU FFN example widened to a
# 256-wide intermediate; C2..C4 are Llama-2 7B/70B shapes; C5 is the PaLM 540B FFN.
C1 = FfnShape(batch=8, E=64, F=256, dtype="f32", act="relu", n_slices=2,
              x_std=1.0 / 8.0, w_std=1.0 / 8.0)
C2 = BlockShape(dim=4096, n_heads=32, n_kv_heads=32, head_dim=128, ffn_dim=11008, vocab=32000,
                max_seq=1024, batch=1, n_slices=4, sync_quant=True, pos=1023)
C3 = BlockShape(dim=4096, n_heads=32, n_kv_heads=32, head_dim=128, ffn_dim=11008, vocab=32000,
                max_seq=4096, batch=1, n_slices=8, sync_quant=False, pos=4095, n_layers=32)
C4 = BlockShape(dim=8192, n_heads=64, n_kv_heads=8, head_dim=128, ffn_dim=28672, vocab=32000,
                max_seq=4096, batch=32, n_slices=8, sync_quant=False, pos=4095)
C5 = FfnShape(batch=512, E=18432, F=73728, dtype="bf16", act="relu", n_slices=64,
              grid_x=8, grid_y=8, x_std=1.0, w_std=0.01)

CONFIG_SEED = {"C1": SEED_BASE + 0, "C2": SEED_BASE + 1, "C3": SEED_BASE + 2,
               "C4": SEED_BASE + 3, "C5": SEED_BASE + 4}


# ---------------------------------------------------------------------------
# block inputs
# ---------------------------------------------------------------------------

@dataclass
class BlockInputs:
    """Host copies of one decoder block's inputs. bf16 tensors are uint16 bits."""

    shape: BlockShape
    x: np.ndarray                      # [B, dim] float32
    attn_norm: np.ndarray              # [dim] float32
    ffn_norm: np.ndarray               # [dim] float32
    wq: np.ndarray                     # [H*hd, dim] bf16
    wk: np.ndarray                     # [Hkv*hd, dim] bf16
    wv: np.ndarray                     # [Hkv*hd, dim] bf16
    wo: np.ndarray                     # [dim, H*hd] bf16
    w1: np.ndarray                     # [F, dim] bf16
    w3: np.ndarray                     # [F, dim] bf16
    w2: np.ndarray                     # [dim, F] bf16
    k_cache: np.ndarray                # [B, Hkv, max_seq, hd] bf16
    v_cache: np.ndarray
    pos: np.ndarray                    # [B] int32
    extra: dict = field(default_factory=dict)


def block_weight_names(layer: int = 0):
    p = f"L{layer}."
    return {k: p + k for k in ("wq", "wk", "wv", "wo", "w1", "w3", "w2")}


def block_weights(seed: int, s: BlockShape, layer: int = 0) -> dict:
    names = block_weight_names(layer)
    qd, kd = s.n_heads * s.head_dim, s.n_kv_heads * s.head_dim
    shapes = {"wq": (qd, s.dim), "wk": (kd, s.dim), "wv": (kd, s.dim), "wo": (s.dim, qd),
              "w1": (s.ffn_dim, s.dim), "w3": (s.ffn_dim, s.dim), "w2": (s.dim, s.ffn_dim)}
    return {k: normal_bf16(seed, names[k], shapes[k], s.w_std) for k in shapes}


def kv_row(seed: int, s: BlockShape, which: str, b: int, layer: int = 0) -> np.ndarray:
    """Cache of batch row ``b``: [Hkv, max_seq, hd] bf16, positions < pos filled, rest zero."""
    hk, T, hd = s.n_kv_heads, s.max_seq, s.head_dim
    row = normal_bf16(seed, f"L{layer}.{which}cache.b{b}", (hk, T, hd), s.kv_std)
    row[:, s.pos:, :] = 0
    return row


def block_inputs(seed: int, s: BlockShape, layer: int = 0, batch: int | None = None) -> BlockInputs:
    B = s.batch if batch is None else batch
    w = block_weights(seed, s, layer)
    k = np.stack([kv_row(seed, s, "k", b, layer) for b in range(B)])
    v = np.stack([kv_row(seed, s, "v", b, layer) for b in range(B)])
    ones = np.ones(s.dim, dtype=np.float32)
    return BlockInputs(
        shape=s, x=normal_f32(seed, f"L{layer}.x", (B, s.dim)), attn_norm=ones.copy(),
        ffn_norm=ones.copy(), k_cache=k, v_cache=v,
        pos=np.full(B, s.pos, dtype=np.int32), **w)


def chunk_inputs(seed: int, s: BlockShape, pos, seq, n_seq: int | None = None,
                 layer: int = 0) -> BlockInputs:
    """Rows of one or more sequences in one step (a prefill chunk, or decode rows of
    several sequences mixed with one): row b is a token of sequence ``seq[b]`` at
    position ``pos[b]``. The caches hold ``n_seq`` sequences (default max(seq) + 1),
    each with positions < ``s.pos`` filled; ``extra["seq"]`` holds ``seq``."""
    seq = np.asarray(seq, dtype=np.int32)
    pos = np.asarray(pos, dtype=np.int32)
    S = int(seq.max()) + 1 if n_seq is None else n_seq
    w = block_weights(seed, s, layer)
    k = np.stack([kv_row(seed, s, "k", q, layer) for q in range(S)])
    v = np.stack([kv_row(seed, s, "v", q, layer) for q in range(S)])
    ones = np.ones(s.dim, dtype=np.float32)
    return BlockInputs(
        shape=s, x=normal_f32(seed, f"L{layer}.chunk.x", (len(pos), s.dim)), attn_norm=ones.copy(),
        ffn_norm=ones.copy(), k_cache=k, v_cache=v, pos=pos.copy(), extra={"seq": seq.copy()}, **w)


def ffn_inputs(seed: int, s: FfnShape, rows: np.ndarray | None = None) -> dict:
    """X, W1, W2 (and W3 for SwiGLU). ``rows`` restricts X to those token rows."""
    gen = normal_f32 if s.dtype == "f32" else normal_bf16
    out = {}
    if rows is None:
        out["X"] = gen(seed, "X", (s.batch, s.E), s.x_std)
    else:
        out["X"] = np.stack([gen(seed, "X", (s.E,), s.x_std, start=int(r) * s.E) for r in rows])
    out["W1"] = gen(seed, "W1", (s.F, s.E), s.w_std)
    out["W2"] = gen(seed, "W2", (s.E, s.F), s.w_std)
    if s.act == "swiglu":
        out["W3"] = gen(seed, "W3", (s.F, s.E), s.w_std)
    return out
