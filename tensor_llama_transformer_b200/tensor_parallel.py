"""The decoder block with its slices spread over processes, one GPU each.

In distributed-llama issue #29's task list every node computes the partials of
its slices, and the SyncAtt / SyncFfn2 transfers carry them (quantised when the
sync is) to be dequantised and merged; the aiterms.tw "Tensor Parallelism"
glossary's FFN ("how it works") replicates the input, keeps the column-split
products local and sums the row-split products across devices. Here each rank
runs its slices through the library (``tp_block_rank_step``, three phases per
decode step) and each transfer is an all-gather of the ranks' sync buffers over
``torch.distributed`` (NCCL between GPUs). Every rank then merges all n slices in
slice order, so the replicated residual stays bit-identical across ranks and
equals what one process holding every slice computes from the same partials.

Host-side plumbing only: which rows and columns of each weight a rank holds, the
order of phases and exchanges, and the buffers the exchanges move.
"""
from __future__ import annotations

from typing import Callable

WEIGHT_ORDER = ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w1", "w3", "w2")
TP_RANK_ATT, TP_RANK_FFN, TP_RANK_OUT = 0, 1, 2


def _part(total: int, rank: int, world: int) -> slice:
    if total % world:
        raise ValueError(f"{total} does not split over {world} ranks")
    return slice(rank * total // world, (rank + 1) * total // world)


def rank_slices(n_slices: int, rank: int, world: int) -> range:
    """The slices rank `rank` of `world` holds: a contiguous run of n/world."""
    s = _part(n_slices, rank, world)
    return range(s.start, s.stop)


def rank_kv_heads(n_kv_heads: int, rank: int, world: int) -> slice:
    """The kv heads of the rank's slices (its KV cache holds these only)."""
    return _part(n_kv_heads, rank, world)


def rank_weights(w: dict, n_heads: int, n_kv_heads: int, head_dim: int, rank: int,
                 world: int) -> dict:
    """This rank's parameters, contiguous, from the whole block's ``w`` (tensors in
    the [out, in] layout, keys ``WEIGHT_ORDER``): the rows of its query and kv heads
    of wq / wk / wv (column split), the columns of its heads of wo (row split), its
    rows of w1 / w3 and columns of w2; the norm gains whole."""
    q = _part(n_heads, rank, world)
    kv = _part(n_kv_heads, rank, world)
    qr = slice(q.start * head_dim, q.stop * head_dim)
    kr = slice(kv.start * head_dim, kv.stop * head_dim)
    f = _part(w["w1"].shape[0], rank, world)
    return {
        "attn_norm": w["attn_norm"],
        "wq": w["wq"][qr].contiguous(),
        "wk": w["wk"][kr].contiguous(),
        "wv": w["wv"][kr].contiguous(),
        "wo": w["wo"][:, qr].contiguous(),
        "ffn_norm": w["ffn_norm"],
        "w1": w["w1"][f].contiguous(),
        "w3": w["w3"][f].contiguous(),
        "w2": w["w2"][:, f].contiguous(),
    }


def all_gather_exchange(group=None) -> Callable:
    """The transfer between phases: every rank's send bytes, in rank order, into
    every rank's receive buffer."""
    import torch.distributed as dist

    def exchange(send, recv):
        dist.all_gather_into_tensor(recv, send, group=group)

    return exchange


def run_step(step: Callable[[int], None], exchange: Callable, send, recv) -> None:
    """One decode step of a rank: phase 0, exchange, phase 1, exchange, phase 2.
    Every rank makes the same two collective calls in the same order."""
    step(TP_RANK_ATT)
    exchange(send, recv)
    step(TP_RANK_FFN)
    exchange(send, recv)
    step(TP_RANK_OUT)


class RankBlock:
    """One rank's handle: its slices' weights (``rank_weights``), a workspace it
    owns, and the exchange between phases (``all_gather_exchange`` by default)."""

    def __init__(self, dims, n_slices: int, sync_quant: int, rank: int, world: int, weights: dict,
                 exchange: Callable | None = None, device=None):
        import torch

        import tensor_llama_transformer_b200 as lib

        self.lib = lib
        self.rank, self.world = rank, world
        self.exchange = exchange or all_gather_exchange()
        nbytes = lib.tp_block_rank_workspace_bytes(dims, n_slices, sync_quant, rank, world)
        self.ws = torch.zeros(nbytes, dtype=torch.uint8, device=device or "cuda")
        self.weights = weights  # kept alive: the handle borrows the pointers
        self.h = lib.tp_block_create_rank(dims, n_slices, sync_quant, rank, world,
                                          lib.make_weights(*[weights[k] for k in WEIGHT_ORDER]),
                                          self.ws, nbytes)
        self.send_off, _ = lib.tp_block_buffer(self.h, lib.TP_BUF_SEND)
        self.recv_off, _ = lib.tp_block_buffer(self.h, lib.TP_BUF_RECV)

    def buffers(self, batch: int):
        """(send, recv) views of the workspace for `batch` rows."""
        n = self.lib.tp_block_rank_sync_bytes(self.h, batch)
        return (self.ws[self.send_off:self.send_off + n],
                self.ws[self.recv_off:self.recv_off + self.world * n])

    def step(self, phase: int, x, k_cache, v_cache, pos, batch: int, stream=None) -> None:
        self.lib.tp_block_rank_step(self.h, phase, x, k_cache, v_cache, pos, batch, stream)

    def forward(self, x, k_cache, v_cache, pos, batch: int, stream=None) -> None:
        send, recv = self.buffers(batch)
        run_step(lambda ph: self.step(ph, x, k_cache, v_cache, pos, batch, stream), self.exchange,
                 send, recv)

    def close(self) -> None:
        if self.h:
            self.lib.tp_block_destroy(self.h)
            self.h = None

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()
