"""Python binding of ``libtp_block.so`` (the C ABI in ``include/tp_block.h``).

Argument marshalling only: every step of the decoder block runs in the CUDA
kernels of the shared library. Functions keep the C names; tensor arguments
may be ``torch.Tensor`` (their ``data_ptr()`` is passed) or plain integer
addresses. A non-zero status raises ``TpError``. Importing fails loudly when
the library has not been built (``python tensor_llama_transformer_b200/build.py``).
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libtp_block.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python tensor_llama_transformer_b200/build.py` "
        "(there is no fallback implementation)")
_lib = C.CDLL(LIB_PATH)

TP_OK, TP_EINVAL, TP_EWORKSPACE, TP_EARCH, TP_ECUDA, TP_ENOTSUP, TP_EALIGN, TP_ESCRATCH = range(8)
TP_NOALLOC_SCRATCH_BYTES = 16 << 20
TP_PART_1D, TP_PART_2D = 1, 2
TP_ACT_RELU, TP_ACT_SWIGLU = 0, 1
TP_F32, TP_BF16 = 0, 1
TP_MERGE_FAITHFUL, TP_MERGE_FUSED = 0, 1
BUF_XQ, BUF_XD, BUF_XN, BUF_Q, BUF_ATT, BUF_PART, BUF_H = range(7)
TP_RANK_ATT, TP_RANK_FFN, TP_RANK_OUT = 0, 1, 2
TP_BUF_SEND, TP_BUF_RECV = 18, 19


class TpError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {tp_status_string(status)} ({status})")


class tp_dims(C.Structure):
    _fields_ = [(n, C.c_int32) for n in ("dim", "n_heads", "n_kv_heads", "head_dim", "ffn_dim",
                                         "vocab", "max_batch", "max_seq")] + \
               [("norm_eps", C.c_float), ("rope_theta", C.c_float)]


class tp_block_weights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w1",
                                          "w3", "w2")]


class tp_block_weights_q8(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("attn_norm", "wq", "wq_d", "wk", "wk_d", "wv", "wv_d", "wo",
                                          "wo_d", "ffn_norm", "w1", "w1_d", "w3", "w3_d", "w2",
                                          "w2_d")]


class tp_ffn_desc(C.Structure):
    _fields_ = [(n, C.c_int32) for n in ("batch", "E", "F", "dtype", "act", "partition", "n_slices",
                                         "grid_x", "grid_y", "sync_quant", "merge")]


_P = C.c_void_p
_SZ = C.POINTER(C.c_size_t)
_sig = {
    "tp_status_string": (C.c_char_p, [C.c_int]),
    "tp_version": (C.c_char_p, []),
    "tp_block_workspace_bytes": (C.c_int, [C.POINTER(tp_dims), C.c_int, C.c_int, C.c_int, _SZ]),
    "tp_block_create": (C.c_int, [C.POINTER(tp_dims), C.c_int, C.c_int, C.c_int,
                                  C.POINTER(tp_block_weights), _P, C.c_size_t, C.POINTER(_P)]),
    "tp_block_create_q8w": (C.c_int, [C.POINTER(tp_dims), C.c_int, C.c_int, C.c_int,
                                      C.POINTER(tp_block_weights_q8), _P, C.c_size_t,
                                      C.POINTER(_P)]),
    "tp_block_forward": (C.c_int, [_P, _P, _P, _P, _P, C.c_int, _P]),
    "tp_block_forward_seq": (C.c_int, [_P, _P, _P, _P, _P, _P, C.c_int, C.c_int, _P]),
    "tp_model_forward_seq": (C.c_int, [_P, _P, _P, _P, _P, _P, C.c_int, C.c_int, _P, _P]),
    "tp_block_rank_workspace_bytes": (C.c_int, [C.POINTER(tp_dims), C.c_int, C.c_int, C.c_int,
                                                C.c_int, _SZ]),
    "tp_block_create_rank": (C.c_int, [C.POINTER(tp_dims), C.c_int, C.c_int, C.c_int, C.c_int,
                                       C.POINTER(tp_block_weights), _P, C.c_size_t,
                                       C.POINTER(_P)]),
    "tp_block_rank_sync_bytes": (C.c_int, [_P, C.c_int, _SZ]),
    "tp_block_rank_step": (C.c_int, [_P, C.c_int, _P, _P, _P, _P, C.c_int, _P]),
    "tp_block_buffer": (C.c_int, [_P, C.c_int, _SZ, _SZ]),
    "tp_block_destroy": (None, [_P]),
    "tp_block_set_events": (C.c_int, [_P, _P, C.c_int]),
    "tp_block_set_trace": (C.c_int, [_P, _P, C.c_size_t]),
    "tp_block_set_persistent": (C.c_int, [_P, C.c_int]),
    "tp_model_set_persistent": (C.c_int, [_P, C.c_int]),
    "tp_ffn_workspace_bytes": (C.c_int, [C.POINTER(tp_ffn_desc), _SZ]),
    "tp_ffn_forward": (C.c_int, [C.POINTER(tp_ffn_desc), _P, _P, _P, _P, _P, _P, C.c_size_t, _P]),
    "tp_model_workspace_bytes": (C.c_int, [C.POINTER(tp_dims), C.c_int, C.c_int, C.c_int, C.c_int,
                                           _SZ]),
    "tp_model_create": (C.c_int, [C.POINTER(tp_dims), C.c_int, C.c_int, C.c_int, C.c_int,
                                  C.POINTER(tp_block_weights), _P, _P, _P, _P, C.c_size_t,
                                  C.POINTER(_P)]),
    "tp_model_forward": (C.c_int, [_P, _P, _P, _P, _P, C.c_int, _P, _P]),
    "tp_model_destroy": (None, [_P]),
    "tp_quantize_q8": (C.c_int, [_P, _P, _P, C.c_int64, _P]),
    "tp_dequantize_q8": (C.c_int, [_P, _P, _P, C.c_int64, _P]),
    "tp_block_forward_noalloc": (C.c_int, [C.POINTER(tp_dims), C.c_int, C.c_int, C.c_int,
                                           C.POINTER(tp_block_weights), _P, _P, _P, _P, C.c_int,
                                           _P]),
    "tp_block_noalloc_error": (C.c_int, [C.POINTER(C.c_int), _P]),
}
for _name, (_res, _args) in _sig.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args

EXPORTED = tuple(_sig)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(s):
    if s is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(rc: int, where: str):
    if rc != TP_OK:
        raise TpError(rc, where)


def tp_status_string(status: int) -> str:
    return _lib.tp_status_string(status).decode()


def tp_version() -> str:
    return _lib.tp_version().decode()


def make_dims(dim, n_heads, n_kv_heads, head_dim, ffn_dim, vocab, max_batch, max_seq,
              norm_eps=1e-5, rope_theta=1e4) -> tp_dims:
    return tp_dims(dim, n_heads, n_kv_heads, head_dim, ffn_dim, vocab, max_batch, max_seq,
                   norm_eps, rope_theta)


def make_weights(attn_norm, wq, wk, wv, wo, ffn_norm, w1, w3, w2) -> tp_block_weights:
    return tp_block_weights(*[_ptr(t) for t in (attn_norm, wq, wk, wv, wo, ffn_norm, w1, w3, w2)])


def tp_block_workspace_bytes(dims: tp_dims, n_slices: int, partition: int, sync_quant: int) -> int:
    out = C.c_size_t()
    _check(_lib.tp_block_workspace_bytes(C.byref(dims), n_slices, partition, int(sync_quant),
                                         C.byref(out)), "tp_block_workspace_bytes")
    return out.value


def tp_block_create(dims, n_slices, partition, sync_quant, weights, workspace, ws_bytes) -> int:
    h = C.c_void_p()
    _check(_lib.tp_block_create(C.byref(dims), n_slices, partition, int(sync_quant),
                                C.byref(weights), _ptr(workspace), ws_bytes, C.byref(h)),
           "tp_block_create")
    return h.value


def make_weights_q8(attn_norm, wq, wq_d, wk, wk_d, wv, wv_d, wo, wo_d, ffn_norm, w1, w1_d, w3,
                    w3_d, w2, w2_d) -> tp_block_weights_q8:
    """Int8 weights: each matrix as Q8 codes (int8) and float32 scales [out, in/32]."""
    return tp_block_weights_q8(*[_ptr(t) for t in (attn_norm, wq, wq_d, wk, wk_d, wv, wv_d, wo, wo_d,
                                                   ffn_norm, w1, w1_d, w3, w3_d, w2, w2_d)])


def tp_block_create_q8w(dims, n_slices, partition, sync_quant, weights, workspace, ws_bytes) -> int:
    h = C.c_void_p()
    _check(_lib.tp_block_create_q8w(C.byref(dims), n_slices, partition, int(sync_quant),
                                    C.byref(weights), _ptr(workspace), ws_bytes, C.byref(h)),
           "tp_block_create_q8w")
    return h.value


def tp_block_forward(handle, x, k_cache, v_cache, pos, batch, stream=None):
    _check(_lib.tp_block_forward(handle, _ptr(x), _ptr(k_cache), _ptr(v_cache), _ptr(pos), batch,
                                 _stream(stream)), "tp_block_forward")


def tp_block_forward_seq(handle, x, k_cache, v_cache, pos, seq, n_seq, batch, stream=None):
    """Rows mapped to cache sequences (seq [batch] int32): prefill chunks, mixed batches."""
    _check(_lib.tp_block_forward_seq(handle, _ptr(x), _ptr(k_cache), _ptr(v_cache), _ptr(pos),
                                     _ptr(seq), n_seq, batch, _stream(stream)),
           "tp_block_forward_seq")


def tp_model_forward_seq(handle, tokens, k_cache, v_cache, pos, seq, n_seq, batch, logits,
                         stream=None):
    _check(_lib.tp_model_forward_seq(handle, _ptr(tokens), _ptr(k_cache), _ptr(v_cache), _ptr(pos),
                                     _ptr(seq), n_seq, batch, _ptr(logits), _stream(stream)),
           "tp_model_forward_seq")


def tp_block_rank_workspace_bytes(dims, n_slices, sync_quant, rank, world) -> int:
    out = C.c_size_t()
    _check(_lib.tp_block_rank_workspace_bytes(C.byref(dims), n_slices, int(sync_quant), rank, world,
                                              C.byref(out)), "tp_block_rank_workspace_bytes")
    return out.value


def tp_block_create_rank(dims, n_slices, sync_quant, rank, world, weights, workspace,
                         ws_bytes) -> int:
    """Handle for rank `rank` of `world` holding slices [rank n/world, (rank+1) n/world);
    `weights` are that rank's slices (``tensor_parallel.rank_weights``)."""
    h = C.c_void_p()
    _check(_lib.tp_block_create_rank(C.byref(dims), n_slices, int(sync_quant), rank, world,
                                     C.byref(weights), _ptr(workspace), ws_bytes, C.byref(h)),
           "tp_block_create_rank")
    return h.value


def tp_block_rank_sync_bytes(handle, batch) -> int:
    out = C.c_size_t()
    _check(_lib.tp_block_rank_sync_bytes(handle, batch, C.byref(out)), "tp_block_rank_sync_bytes")
    return out.value


def tp_block_rank_step(handle, phase, x, k_cache, v_cache, pos, batch, stream=None):
    _check(_lib.tp_block_rank_step(handle, phase, _ptr(x), _ptr(k_cache), _ptr(v_cache), _ptr(pos),
                                   batch, _stream(stream)), "tp_block_rank_step")


def tp_block_buffer(handle, which):
    off, size = C.c_size_t(), C.c_size_t()
    _check(_lib.tp_block_buffer(handle, which, C.byref(off), C.byref(size)), "tp_block_buffer")
    return off.value, size.value


def tp_block_destroy(handle):
    _lib.tp_block_destroy(handle)


TP_BLOCK_STAGES = 7  # stages of one block step (include/tp_block.h)
TP_BLOCK_STAGE_EVENTS = TP_BLOCK_STAGES + 1  # events tp_block_set_events takes: one per stage, one after


def tp_block_set_events(handle, events, n):
    """events: a ctypes array of n cudaEvent_t handles (kept alive by the caller) or None."""
    _check(_lib.tp_block_set_events(handle, events, n), "tp_block_set_events")


def tp_block_set_persistent(handle, enable):
    """1: run this handle's batch 1-2 forwards as the one persistent kernel; 0: never."""
    _check(_lib.tp_block_set_persistent(handle, int(enable)), "tp_block_set_persistent")


def tp_model_set_persistent(handle, enable):
    """tp_block_set_persistent for every layer of a model handle."""
    _check(_lib.tp_model_set_persistent(handle, int(enable)), "tp_model_set_persistent")


def tp_block_set_trace(handle, buf, nbytes):
    """buf: device buffer (tensor or pointer) of nbytes for the persistent kernel's
    per-CTA phase timestamps (TP_BLOCK_TRACE_SLOTS uint64 per CTA), or None."""
    _check(_lib.tp_block_set_trace(handle, _ptr(buf), nbytes), "tp_block_set_trace")


TP_BLOCK_TRACE_SLOTS = 40


def tp_ffn_workspace_bytes(desc: tp_ffn_desc) -> int:
    out = C.c_size_t()
    _check(_lib.tp_ffn_workspace_bytes(C.byref(desc), C.byref(out)), "tp_ffn_workspace_bytes")
    return out.value


def tp_ffn_forward(desc, X, W1, W3, W2, Y, workspace, ws_bytes, stream=None):
    _check(_lib.tp_ffn_forward(C.byref(desc), _ptr(X), _ptr(W1), _ptr(W3), _ptr(W2), _ptr(Y),
                               _ptr(workspace), ws_bytes, _stream(stream)), "tp_ffn_forward")


def tp_model_workspace_bytes(dims, n_layers, n_slices, partition, sync_quant) -> int:
    out = C.c_size_t()
    _check(_lib.tp_model_workspace_bytes(C.byref(dims), n_layers, n_slices, partition,
                                         int(sync_quant), C.byref(out)), "tp_model_workspace_bytes")
    return out.value


def tp_model_create(dims, n_layers, n_slices, partition, sync_quant, layer_weights, embed,
                    final_norm, wcls, workspace, ws_bytes) -> int:
    arr = (tp_block_weights * n_layers)(*layer_weights)
    h = C.c_void_p()
    _check(_lib.tp_model_create(C.byref(dims), n_layers, n_slices, partition, int(sync_quant), arr,
                                _ptr(embed), _ptr(final_norm), _ptr(wcls), _ptr(workspace),
                                ws_bytes, C.byref(h)), "tp_model_create")
    return h.value


def tp_model_forward(handle, tokens, k_cache, v_cache, pos, batch, logits, stream=None):
    _check(_lib.tp_model_forward(handle, _ptr(tokens), _ptr(k_cache), _ptr(v_cache), _ptr(pos),
                                 batch, _ptr(logits), _stream(stream)), "tp_model_forward")


def tp_model_destroy(handle):
    _lib.tp_model_destroy(handle)


def tp_quantize_q8(x, q, d, n, stream=None):
    _check(_lib.tp_quantize_q8(_ptr(x), _ptr(q), _ptr(d), n, _stream(stream)), "tp_quantize_q8")


def tp_dequantize_q8(q, d, x, n, stream=None):
    _check(_lib.tp_dequantize_q8(_ptr(q), _ptr(d), _ptr(x), n, _stream(stream)),
           "tp_dequantize_q8")


def tp_block_forward_noalloc(dims, n_slices, partition, sync_quant, weights, x, k_cache, v_cache,
                             pos, batch, stream=None):
    """Block decode step on the library's fixed scratch array (no workspace argument)."""
    _check(_lib.tp_block_forward_noalloc(C.byref(dims), n_slices, partition, int(sync_quant),
                                         C.byref(weights), _ptr(x), _ptr(k_cache), _ptr(v_cache),
                                         _ptr(pos), batch, _stream(stream)),
           "tp_block_forward_noalloc")


def tp_block_noalloc_error(stream=None) -> int:
    """The kernels' error word of the last tp_block_forward_noalloc on this device
    (copied on `stream`; this call then synchronises the device; 0 = no wait gave up)."""
    import torch

    out = C.c_int(-1)
    _check(_lib.tp_block_noalloc_error(C.byref(out), _stream(stream)), "tp_block_noalloc_error")
    torch.cuda.synchronize()
    return out.value
