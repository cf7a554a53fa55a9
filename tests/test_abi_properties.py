"""Host-side properties of the C ABI's sizing and validation over random shapes (CPU only).

The workspace functions must accept exactly the shapes the header documents
(dim % 128, head_dim 128, the query-per-kv-head groups, H % n, Hkv % n,
ffn_dim % 32n, 1 <= max_batch <= 64) and reject the rest with TP_EINVAL or
TP_ENOTSUP before any CUDA call; an accepted size is 256-byte aligned, holds at
least the buffers the header names, and grows with max_batch and max_seq. A rank's
share of a block needs less than the whole block once the heads are split.
"""
import pytest
from hypothesis import given, settings
from hypothesis import strategies as st


@pytest.fixture(scope="module")
def tpb():
    import tensor_llama_transformer_b200 as t

    return t


def _documented_ok(dim, H, Hkv, hd, F, mb, n):
    if n < 1 or dim <= 0 or dim % 128 or hd != 128 or Hkv <= 0 or H <= 0 or H % Hkv:
        return False
    G = H // Hkv
    if not (G in (1, 2, 4) or (G % 8 == 0 and G <= 64)):
        return False
    return H % n == 0 and Hkv % n == 0 and F > 0 and F % (32 * n) == 0 and 1 <= mb <= 64


shapes = st.tuples(
    st.sampled_from([128, 256, 384, 4096, 4000, 8192]),   # dim
    st.sampled_from([1, 2, 4, 8, 16, 32, 64, 6]),         # n_heads
    st.sampled_from([1, 2, 4, 8, 3]),                     # n_kv_heads
    st.sampled_from([128, 64]),                           # head_dim
    st.sampled_from([256, 512, 11008, 1000, 28672]),      # ffn_dim
    st.integers(min_value=0, max_value=70),               # max_batch
    st.sampled_from([1, 64, 1000, 4096]),                 # max_seq
    st.sampled_from([1, 2, 3, 4, 8]),                     # n_slices
    st.sampled_from([0, 1]),                              # sync_quant
)


@settings(max_examples=300, deadline=None)
@given(shapes)
def test_workspace_accepts_exactly_the_documented_shapes(tpb, shape):
    dim, H, Hkv, hd, F, mb, T, n, q = shape
    d = tpb.make_dims(dim, H, Hkv, hd, F, 32000, mb, T)
    ok = _documented_ok(dim, H, Hkv, hd, F, mb, n)
    if not ok:
        with pytest.raises(tpb.TpError) as e:
            tpb.tp_block_workspace_bytes(d, n, tpb.TP_PART_1D, q)
        assert e.value.status in (tpb.TP_EINVAL, tpb.TP_ENOTSUP)
        return
    ws = tpb.tp_block_workspace_bytes(d, n, tpb.TP_PART_1D, q)
    assert ws % 256 == 0
    QD = H * hd
    # at least: q and attention output, the partial planes, the SwiGLU output, xnorm
    assert ws >= mb * (2 * QD * 4 + n * dim * 4 + F * 4 + dim * 4)
    bigger = tpb.make_dims(dim, H, Hkv, hd, F, 32000, mb, T + 64)
    assert tpb.tp_block_workspace_bytes(bigger, n, tpb.TP_PART_1D, q) >= ws
    if mb < 64:
        more = tpb.make_dims(dim, H, Hkv, hd, F, 32000, mb + 1, T)
        assert tpb.tp_block_workspace_bytes(more, n, tpb.TP_PART_1D, q) > ws


@settings(max_examples=200, deadline=None)
@given(shapes, st.sampled_from([1, 2, 4, 8]))
def test_rank_workspace_consistent_with_the_whole_block(tpb, shape, world):
    dim, H, Hkv, hd, F, mb, T, n, q = shape
    d = tpb.make_dims(dim, H, Hkv, hd, F, 32000, mb, T)
    ok = _documented_ok(dim, H, Hkv, hd, F, mb, n) and n % world == 0
    if not ok:
        with pytest.raises(tpb.TpError):
            tpb.tp_block_rank_workspace_bytes(d, n, q, 0, world)
        return
    sizes = {tpb.tp_block_rank_workspace_bytes(d, n, q, r, world) for r in range(world)}
    assert len(sizes) == 1  # every rank holds an equal share
    ws = sizes.pop()
    assert ws % 256 == 0
    chunk = mb * dim + mb * (dim // 32) * 4 if q else mb * dim * 4
    assert ws >= n * chunk  # the receive buffer holds every slice
    if world > 1 and mb >= 6:
        assert ws < tpb.tp_block_workspace_bytes(d, n, tpb.TP_PART_1D, q) + n * chunk * 2
