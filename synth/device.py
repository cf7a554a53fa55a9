"""Copy generated host inputs into torch CUDA tensors (no arithmetic)."""
from __future__ import annotations

import numpy as np
import torch


def bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 bf16 bit patterns -> torch.bfloat16 tensor on ``device``."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).to(device)


def f32_tensor(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def i32_tensor(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)


def to_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 CUDA/CPU tensor -> uint16 bit patterns on the host."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


class DeviceBlock:
    """Device copies of one ``synth.BlockInputs`` (weights, caches, x, pos)."""

    def __init__(self, inp, max_batch=None, device="cuda"):
        s = inp.shape
        B = inp.x.shape[0]
        mb = max_batch or B
        self.x = f32_tensor(inp.x, device)
        self.attn_norm = f32_tensor(inp.attn_norm, device)
        self.ffn_norm = f32_tensor(inp.ffn_norm, device)
        for k in ("wq", "wk", "wv", "wo", "w1", "w3", "w2"):
            setattr(self, k, bf16_tensor(getattr(inp, k), device))
        S = inp.k_cache.shape[0]  # cache sequences (one per row unless rows share them)
        shape = (max(mb, S), s.n_kv_heads, s.max_seq, s.head_dim)
        self.k_cache = torch.zeros(shape, dtype=torch.bfloat16, device=device)
        self.v_cache = torch.zeros(shape, dtype=torch.bfloat16, device=device)
        self.k_cache[:S] = bf16_tensor(inp.k_cache, device)
        self.v_cache[:S] = bf16_tensor(inp.v_cache, device)
        self.pos = i32_tensor(inp.pos, device)
        seq = inp.extra.get("seq") if getattr(inp, "extra", None) else None
        self.seq = i32_tensor(seq, device) if seq is not None else None

    def weights(self):
        return (self.attn_norm, self.wq, self.wk, self.wv, self.wo, self.ffn_norm, self.w1,
                self.w3, self.w2)
