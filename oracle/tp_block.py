"""Float64 CPU oracle of the tensor-parallel Llama decoder block — TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline
and reference legs) may import this module. It is a plain restatement of the
method for checking the CUDA path; nothing in the product calls it.

Sources (pages on the subject, cited by title and part):
  [DL]   distributed-llama issue #29, "[Feature Suggest] Tensor Parallellism for
         Accelerating LLM": the ``buildLlama2Arch`` task list (root node order
         RmsAttNorm, QuantizeRmsAtt, SyncRmsAtt, Qkv, MultiheadAtt, AttOutput,
         QuantizeAtt, SyncAtt, DequantizeAtt, MergeAtt, RmfFfn/RmfFfnNorm,
         QuantizeRmfFfn, SyncRmfFfn, Ffn, Ffn2, QuantizeFfn2, SyncFfn2,
         DequantizeFfn2, MergeFfn2, NextBlock, then RmsFinal, Logits, MergeLogits).
  [TP]   aiterms.tw "Tensor Parallelism" glossary, section "how it works": the FFN
         ``Linear2(ReLU(Linear1(x)))`` with the input replicated, Linear1 split by
         columns, ReLU applied locally, Linear2 split by rows, one all-reduce; and
         the "core concept" list (column split, row split, 2D split).
  [POPE] CS349E lecture 4 script ``03_pope_partitioning.py`` (Pope et al.,
         "Efficiently Scaling Transformer Inference"), ``demo1_1d_vs_2d``: 1D
         splits only F, 2D weight-stationary splits both E and F.
  [GG]   ggmlR ``ggml_pp_dp_forward`` reference page, "Examples": a two-stage
         ``z = W x`` FFN with ReLU after the first stage only.
  [TT]   tt-metal issue "Llama-2 (meta) TT implementation": GQA vs MHA, and tests
         asserting Pearson correlation against a plain golden model.

Where the pages name a step without defining it (RMSNorm, RoPE, attention,
SwiGLU, the quantisation format), the oracle writes out the textbook
definition; each such reading is stated at the function. Every function here
is pinned by ``tests/test_oracle_*.py`` against closed forms, invariants,
library routines or brute force — except where a docstring says
"parity unpinned".

Conventions: weights are stored ``[out, in]`` (PyTorch ``Linear``), so
``y = x @ W.T``. A column split of the math matrix ``W.T`` is a contiguous row
range of the storage; a row split is a contiguous column range. Activations
are ``[B, features]``.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "bf16_to_f64", "round_to_bf16", "rmsnorm", "q8_quantize", "q8_dequantize", "sync_buffer",
    "rope", "attention_decode", "silu", "swiglu", "relu", "block_forward", "ffn_forward",
    "model_forward", "grid_2d", "slice_range", "ffn_unsharded_chunked", "q8_weights", "q8_exact",
]


# ---------------------------------------------------------------------------
# storage helpers
# ---------------------------------------------------------------------------

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact upcast of bf16 bit patterns (uint16) to float64."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16 (via float32, ties to even); returns uint16 bits.

    Used only where the layout stores bf16: the KV cache rows written at ``pos``.
    """
    f = np.asarray(a, dtype=np.float32)
    b = f.view(np.uint32)
    r = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def slice_range(total: int, n: int, s: int) -> slice:
    """Contiguous range owned by slice ``s`` of ``n`` equal slices of ``total`` ([TP] core concept)."""
    assert total % n == 0, (total, n)
    w = total // n
    return slice(s * w, (s + 1) * w)


# ---------------------------------------------------------------------------
# elementwise and normalisation
# ---------------------------------------------------------------------------

def rmsnorm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm of each row: ``x * g / sqrt(mean(x^2) + eps)``.

    [DL] llamaRmsAttNorm / llamaRmfFfnNorm / llamaRmsFinalNorm name the step; the
    pages give no formula, so this is the textbook RMSNorm (Zhang & Sennrich
    2019) with the gain applied after normalising.
    """
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(g, dtype=np.float64)


def silu(z: np.ndarray) -> np.ndarray:
    """``z / (1 + exp(-z))``, the SiLU of the SwiGLU named by [DL] llamaFfn."""
    z = np.asarray(z, dtype=np.float64)
    return z / (1.0 + np.exp(-z))


def swiglu(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """SwiGLU gate: ``silu(a) * b`` with ``a = x W1^T`` and ``b = x W3^T`` ([DL] llamaFfn)."""
    return silu(a) * np.asarray(b, dtype=np.float64)


def relu(z: np.ndarray) -> np.ndarray:
    """ReLU of the [TP] FFN and of the first [GG] stage."""
    return np.maximum(np.asarray(z, dtype=np.float64), 0.0)


# ---------------------------------------------------------------------------
# Q8 block quantisation of the sync buffers
# ---------------------------------------------------------------------------

Q8_BLOCK = 32


def q8_quantize(x: np.ndarray):
    """Symmetric int8 quantisation in blocks of 32 consecutive values.

    [DL] names llamaQuantizeRmsAtt / QuantizeAtt / QuantizeRmfFfn / QuantizeFfn2
    without a format. Reading taken (int8 blocks of 32 + one fp32 scale), all in
    IEEE float32 with round-to-nearest:
        amax = max |x_i| over the block
        d    = fp32(amax / 127)
        d == 0  ->  q_i = 0
        else    ->  v_i = fp32(x_i / d);  q_i = clamp(round_half_away(v_i), -127, 127)
    The rounding is done in float64 as ``sign(v) * floor(|v| + 0.5)``, exact for
    any float32 ``v``. Inputs must be finite. Returns ``(q int8 [..., n],
    d float32 [..., n/32])``.
    """
    x = np.asarray(x, dtype=np.float32)
    shp = x.shape
    assert shp[-1] % Q8_BLOCK == 0, shp
    blk = x.reshape(-1, Q8_BLOCK)
    amax = np.max(np.abs(blk), axis=1)
    d = (amax / np.float32(127.0)).astype(np.float32)
    safe = np.where(d == 0, np.float32(1.0), d).astype(np.float32)
    v = (blk / safe[:, None]).astype(np.float32).astype(np.float64)
    r = np.sign(v) * np.floor(np.abs(v) + 0.5)
    q = np.clip(r, -127, 127)
    q[d == 0] = 0
    return q.astype(np.int8).reshape(shp), d.reshape(shp[:-1] + (shp[-1] // Q8_BLOCK,))


def q8_dequantize(q: np.ndarray, d: np.ndarray) -> np.ndarray:
    """``x'_i = fp32(q_i * d_block)`` ([DL] llamaDequantizeAtt / DequantizeFfn2)."""
    q = np.asarray(q, dtype=np.int8)
    d = np.asarray(d, dtype=np.float32)
    rep = np.repeat(d, Q8_BLOCK, axis=-1)
    return (q.astype(np.float32) * rep).astype(np.float32)


def sync_buffer(v: np.ndarray, quant: bool) -> np.ndarray:
    """What the receiver of a [DL] Sync* transfer sees.

    Without quantisation the value crosses unchanged. With it the sender stores
    the value in float32, quantises it (Quantize* task) and the receiver
    dequantises it (Dequantize* task, or directly on use for the broadcast
    ``xnorm``).
    """
    if not quant:
        return np.asarray(v, dtype=np.float64)
    q, d = q8_quantize(np.asarray(v, dtype=np.float32))
    return q8_dequantize(q, d).astype(np.float64)


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------

def rope(v: np.ndarray, pos: np.ndarray, n_heads: int, head_dim: int, theta: float) -> np.ndarray:
    """Rotary position encoding of every head at each row's position.

    [DL] llamaMultiheadAtt "add RoPE encoding" names the step only. Reading:
    pairs (2i, 2i+1) of each head rotate by ``pos * theta^(-2i/head_dim)``:
        out[2i]   = v[2i] cos(phi) - v[2i+1] sin(phi)
        out[2i+1] = v[2i] sin(phi) + v[2i+1] cos(phi)
    ``v`` is ``[B, n_heads*head_dim]``; ``pos`` is ``[B]``.
    """
    v = np.asarray(v, dtype=np.float64)
    B = v.shape[0]
    out = np.empty_like(v)
    for b in range(B):
        for h in range(n_heads):
            base = h * head_dim
            for i in range(head_dim // 2):
                freq = theta ** (-2.0 * i / head_dim)
                phi = float(pos[b]) * freq
                c, s = math.cos(phi), math.sin(phi)
                a0, a1 = v[b, base + 2 * i], v[b, base + 2 * i + 1]
                out[b, base + 2 * i] = a0 * c - a1 * s
                out[b, base + 2 * i + 1] = a0 * s + a1 * c
    return out


def attention_decode(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray, pos: np.ndarray,
                     heads: range, n_heads: int, n_kv_heads: int, head_dim: int,
                     seq=None) -> np.ndarray:
    """Causal softmax attention of one token per row over cache positions ``0..pos``.

    [DL] llamaMultiheadAtt: each slice computes "a part of multi-head attention
    locally" for its heads; [TT] distinguishes GQA from MHA. For query head h
    the key/value head is ``h // (n_heads // n_kv_heads)``.
        s_t = q_h . k_t / sqrt(head_dim),  p = softmax(s),  o_h = sum_t p_t v_t
    ``q`` is ``[B, n_heads*head_dim]`` (already rotated); caches are float64
    ``[S, n_kv_heads, T, head_dim]`` and row b reads sequence ``seq[b]`` (default
    b). Rows of one sequence at consecutive positions are a prefill chunk: each
    row attends to its own position and the ones before it, i.e. causal
    attention. Returns ``[B, len(heads)*head_dim]``.
    """
    group = n_heads // n_kv_heads
    B = q.shape[0]
    out = np.zeros((B, len(heads) * head_dim), dtype=np.float64)
    for b in range(B):
        P = int(pos[b]) + 1
        sq = b if seq is None else int(seq[b])
        for j, h in enumerate(heads):
            kv = h // group
            qh = q[b, h * head_dim:(h + 1) * head_dim]
            K = k_cache[sq, kv, :P, :]
            V = v_cache[sq, kv, :P, :]
            s = K @ qh / math.sqrt(head_dim)
            s = s - np.max(s)
            p = np.exp(s)
            p /= np.sum(p)
            out[b, j * head_dim:(j + 1) * head_dim] = p @ V
    return out


# ---------------------------------------------------------------------------
# 2D slice grid
# ---------------------------------------------------------------------------

def grid_2d(n: int):
    """Default 2D grid for ``n`` slices: ``gx`` = largest divisor of n with gx*gx <= n
    splits E (the model dim), ``gy = n // gx`` splits F. 64 -> 8 x 8, 4 -> 2 x 2, 8 -> 2 x 4."""
    gx = max(d for d in range(1, n + 1) if n % d == 0 and d * d <= n)
    return gx, n // gx


# ---------------------------------------------------------------------------
# feed-forward, 1D and 2D
# ---------------------------------------------------------------------------

def _act_of(act, a, b):
    return relu(a) if act == "relu" else swiglu(a, b)


def ffn_forward(X, W1, W2, act: str = "relu", W3=None, partition: int = 1, n_slices: int = 1,
                grid=None, quant: bool = False, residual=None) -> np.ndarray:
    """Tensor-parallel FFN ``Y = act(X W1^T [, X W3^T]) W2^T`` summed over slices.

    1D ([TP] how-it-works; [POPE] demo1 "1D"): slice s owns F-range F_s, i.e.
    rows F_s of W1/W3 (column split of Linear1) and columns F_s of W2 (row split
    of Linear2). Each slice computes ``H_s = act(X W1_s^T)`` locally with no
    communication and the partial ``P_s = H_s W2_s^T``; the all-reduce is the
    sum of the partials in slice order 0..n-1.

    2D ([TP] core concept "2D split"; [POPE] demo1 "2D"): slices form a grid
    gx x gy; x splits E into E_x, y splits F into F_y. Stage 1 sums over x:
    ``A[:, F_y] = sum_x X[:, E_x] W1[F_y, E_x]^T`` (and likewise for W3), then
    ``H = act(A)``; stage 2 sums over y: ``Y[:, E_x] = sum_y H[:, F_y] W2[E_x, F_y]^T``.

    Partials are passed through ``sync_buffer`` (Q8 when ``quant``). Inputs are
    float64 arrays; ``residual`` (if given) is added after the merge.
    """
    X = np.asarray(X, dtype=np.float64)
    B, E = X.shape
    F = W1.shape[0]
    if partition == 1:
        n = n_slices
        Y = np.zeros((B, E))
        for s in range(n):
            fs = slice_range(F, n, s)
            a = X @ W1[fs, :].T
            b = X @ W3[fs, :].T if W3 is not None else None
            H = _act_of(act, a, b)
            P = H @ W2[:, fs].T
            Y = Y + sync_buffer(P, quant)
    else:
        gx, gy = grid if grid is not None else grid_2d(n_slices)
        H = np.zeros((B, F))
        for y in range(gy):
            fy = slice_range(F, gy, y)
            a = np.zeros((B, fy.stop - fy.start))
            b = np.zeros_like(a) if W3 is not None else None
            for x in range(gx):
                ex = slice_range(E, gx, x)
                a = a + sync_buffer(X[:, ex] @ W1[fy, ex].T, quant)
                if W3 is not None:
                    b = b + sync_buffer(X[:, ex] @ W3[fy, ex].T, quant)
            H[:, fy] = _act_of(act, a, b)
        Y = np.zeros((B, E))
        for x in range(gx):
            ex = slice_range(E, gx, x)
            acc = np.zeros((B, ex.stop - ex.start))
            for y in range(gy):
                fy = slice_range(F, gy, y)
                acc = acc + sync_buffer(H[:, fy] @ W2[ex, fy].T, quant)
            Y[:, ex] = acc
    if residual is not None:
        Y = np.asarray(residual, dtype=np.float64) + Y
    return Y


# ---------------------------------------------------------------------------
# decoder block
# ---------------------------------------------------------------------------

def q8_exact(v: np.ndarray) -> np.ndarray:
    """The Q8 round trip of ``v`` with the dequantised values kept exact in float64
    (``q * d``, 7 + 24 bits): the value an integer block dot product uses."""
    q, d = q8_quantize(np.asarray(v, dtype=np.float32))
    return q.astype(np.float64) * np.repeat(d.astype(np.float64), Q8_BLOCK, axis=-1)


def q8_weights(w_bits: np.ndarray):
    """Int8 weights: each row of a bf16 weight matrix ``[out, in]`` in the Q8 block
    format along ``in`` (``q8_quantize`` of the row's float32 values).

    [POPE] demo4 ("int8 weights" for PaLM decode, which is bound by weight bytes)
    gives no format; the reading taken is the one the [DL] task list already uses
    for its sync buffers: 32 consecutive values share one float32 scale
    ``d = amax / 127``. Returns ``(codes int8 [out, in], scales float32 [out, in/32])``.
    """
    return q8_quantize(bf16_to_f64(w_bits).astype(np.float32))


def block_forward(inp, n_slices: int, sync_quant: bool, partition: int = 1, grid=None,
                  trace: dict | None = None, weights_q8: bool = False, seq=None):
    """One decode step of one decoder block, partitioned into ``n_slices`` slices.

    Follows the [DL] root-node task order for one layer:
      a1 RmsAttNorm + QuantizeRmsAtt, SyncRmsAtt: ``xin = sync(rmsnorm(x))``
      a3 Qkv: slice s computes its q/k/v heads (column split of Wq/Wk/Wv)
      a4 MultiheadAtt: RoPE on q and k at ``pos``, k/v stored to the bf16 cache
         at ``pos``, attention over ``0..pos`` for the slice's heads
      a5 AttOutput + QuantizeAtt: partial ``p_s = att_s Wo[:, cols_s]^T`` (row split)
      a6 SyncAtt, DequantizeAtt, MergeAtt: ``x1 = x + sum_s sync(p_s)``
      a7 RmfFfn/RmfFfnNorm + QuantizeRmfFfn, SyncRmfFfn: ``xin2 = sync(rmsnorm(x1))``
      a8 Ffn: ``h_s = silu(xin2 W1_s^T) * (xin2 W3_s^T)``
      a9 Ffn2 + QuantizeFfn2: ``p_s = h_s W2[:, F_s]^T``
      a10 SyncFfn2, DequantizeFfn2, MergeFfn2: ``x2 = x1 + sum_s sync(p_s)``
    With ``partition == 2`` the FFN follows ``ffn_forward``'s 2D grid; attention
    stays split by heads. Slice s owns q heads ``[s H/n, (s+1) H/n)`` and kv heads
    ``[s Hkv/n, (s+1) Hkv/n)``.

    ``trace`` (optional dict) receives the intermediates ``xin``, ``q`` (rotated),
    ``att`` (all heads), ``x1``, ``xin2`` and, for 1D, ``h``; recording them does
    not change the arithmetic.

    ``weights_q8`` (1D partition, with ``sync_quant``): int8 weights with Q8
    activations, the form in which every slice product is an integer dot product
    per 32-value block scaled by ``d_w * d_x``, i.e. exactly
    ``sum_i (q_w,i d_w)(q_x,i d_x)``. Every weight matrix enters as its Q8 codes
    times scales (``q8_weights``, exact in float64) and every slice product's
    input as ``q8_exact`` of it: the normalised inputs, each slice's attention
    output before W_O and its SwiGLU output before W2. The partials cross the
    sync as with ``sync_quant``.

    ``seq`` (optional, ``[B]``): the cache sequence of each row (default row b
    uses sequence b). Several rows of one sequence at distinct positions form a
    prefill chunk (Pope et al. demo 2's prefill, many tokens per step): every
    row's k/v are written to the cache before any row's attention, so row b
    attends to positions ``0..pos[b]`` of its sequence, including the rows of
    this step below it. Reading taken (the pages define no prefill step): a
    prefill chunk computes exactly what decoding its tokens one at a time does.

    ``inp`` is a ``synth.BlockInputs``. Returns ``(x_out float64 [B, dim],
    k_row uint16 [B, Hkv, hd], v_row uint16 [B, Hkv, hd])``: the new block
    output and the bf16 k/v rows written at ``pos`` (the caches are not modified).
    """
    s_ = inp.shape
    H, Hkv, hd, dim = s_.n_heads, s_.n_kv_heads, s_.head_dim, s_.dim
    n = n_slices
    assert H % n == 0 and Hkv % n == 0
    x = np.asarray(inp.x, dtype=np.float64)
    B = x.shape[0]
    pos = np.asarray(inp.pos)
    sq = np.arange(B) if seq is None else np.asarray(seq)
    if weights_q8:
        assert partition == 1 and sync_quant

        def wload(bits):
            q, d = q8_weights(bits)
            return q.astype(np.float64) * np.repeat(d.astype(np.float64), Q8_BLOCK, axis=-1)

        def act(v):
            return q8_exact(v)
    else:
        wload = bf16_to_f64

        def act(v):
            return sync_buffer(v, sync_quant)
    wq, wk, wv = wload(inp.wq), wload(inp.wk), wload(inp.wv)
    wo = wload(inp.wo)

    # a1-a2
    xin = act(rmsnorm(x, inp.attn_norm, s_.norm_eps))

    # a3-a4, per slice
    kc = bf16_to_f64(inp.k_cache)
    vc = bf16_to_f64(inp.v_cache)
    k_new = np.zeros((B, Hkv, hd), dtype=np.uint16)
    v_new = np.zeros((B, Hkv, hd), dtype=np.uint16)
    q_all = np.zeros((B, H * hd))
    for s in range(n):
        qs = slice_range(H * hd, n, s)
        ks = slice_range(Hkv * hd, n, s)
        q_all[:, qs] = xin @ wq[qs, :].T
        k_s = xin @ wk[ks, :].T
        v_s = xin @ wv[ks, :].T
        kv0 = s * (Hkv // n)
        k_rot = rope(k_s, pos, Hkv // n, hd, s_.rope_theta)
        for b in range(B):
            for j in range(Hkv // n):
                kr = round_to_bf16(k_rot[b, j * hd:(j + 1) * hd])
                vr = round_to_bf16(v_s[b, j * hd:(j + 1) * hd])
                k_new[b, kv0 + j] = kr
                v_new[b, kv0 + j] = vr
                kc[sq[b], kv0 + j, pos[b], :] = bf16_to_f64(kr)
                vc[sq[b], kv0 + j, pos[b], :] = bf16_to_f64(vr)
    q_rot = rope(q_all, pos, H, hd, s_.rope_theta)

    # a4-a6
    x1 = x.copy()
    att_all = np.zeros((B, H * hd))
    for s in range(n):
        heads = range(s * (H // n), (s + 1) * (H // n))
        att_s = attention_decode(q_rot, kc, vc, pos, heads, H, Hkv, hd, seq=sq)
        cols = slice_range(H * hd, n, s)
        att_all[:, cols] = att_s
        if weights_q8:
            att_s = q8_exact(att_s)
        p_s = att_s @ wo[:, cols].T
        x1 = x1 + sync_buffer(p_s, sync_quant)

    # a7-a10
    xin2 = act(rmsnorm(x1, inp.ffn_norm, s_.norm_eps))
    w1, w3, w2 = wload(inp.w1), wload(inp.w3), wload(inp.w2)
    if trace is not None:
        trace.update(xin=xin, q=q_rot, att=att_all, x1=x1, xin2=xin2)
        if partition == 1:
            trace["h"] = swiglu(xin2 @ w1.T, xin2 @ w3.T)
    if weights_q8:  # 1D FFN whose W2 inputs are Q8 too
        hq = q8_exact(swiglu(xin2 @ w1.T, xin2 @ w3.T))
        F = w1.shape[0]
        x2 = x1.copy()
        for s in range(n):
            fs = slice_range(F, n, s)
            x2 = x2 + sync_buffer(hq[:, fs] @ w2[:, fs].T, True)
        return x2, k_new, v_new
    x2 = ffn_forward(xin2, w1, w2, act="swiglu", W3=w3, partition=partition, n_slices=n,
                     grid=grid, quant=sync_quant, residual=x1)
    return x2, k_new, v_new


def model_forward(tokens, embed, layers, final_norm, wcls, n_slices: int, sync_quant: bool,
                  eps: float):
    """Full decode step: embedding gather, every block in order, final norm, logits.

    [DL]: the layer loop ends with llamaNextBlock; then llamaRmsFinal /
    llamaRmsFinalNorm, llamaLogits (vocab split by columns) and MergeLogits,
    which for a column split is a concatenation of the slices' logits. The
    embedding lookup is not a task on that list; it is the plain row gather.
    ``layers`` is a list of callables ``x -> x`` (one decoder block each).
    Logits are not quantised (the quantisation flag covers the block's sync
    buffers). Returns float64 ``[B, vocab]``.
    """
    x = bf16_to_f64(embed[np.asarray(tokens)]) if embed.dtype == np.uint16 else embed[tokens]
    for layer in layers:
        x = layer(x)
    xn = rmsnorm(x, final_norm, eps)
    W = bf16_to_f64(wcls)
    V = W.shape[0]
    parts = [xn @ W[slice_range(V, n_slices, s), :].T for s in range(n_slices)]
    return np.concatenate(parts, axis=1)


def ffn_unsharded_chunked(X, W1_bits, W2_bits, act: str = "relu", W3_bits=None,
                          chunk: int = 4096) -> np.ndarray:
    """``act(X W1^T [, X W3^T]) W2^T`` for a few rows of X, memory-bounded.

    The same unpartitioned FFN as ``ffn_forward`` with one slice ([TP] how it
    works: the partitioned layer must equal it), for weights too large to hold
    in float64 at once (the PaLM 540B shapes): the F dimension is walked in
    ``chunk``-wide pieces, each piece's bf16 weights upcast exactly to float64,
    and the contributions summed in order. ``X`` is float64 ``[rows, E]``.
    """
    X = np.asarray(X, dtype=np.float64)
    F = W1_bits.shape[0]
    Y = np.zeros((X.shape[0], W2_bits.shape[0]))
    for f0 in range(0, F, chunk):
        fs = slice(f0, min(F, f0 + chunk))
        a = X @ bf16_to_f64(W1_bits[fs]).T
        if act == "relu":
            H = relu(a)
        else:
            H = swiglu(a, X @ bf16_to_f64(W3_bits[fs]).T)
        Y = Y + H @ bf16_to_f64(W2_bits[:, fs]).T
    return Y
