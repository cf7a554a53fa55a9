"""The C ABI library loads and exports every function include/tp_block.h declares (CPU only).

Only calls that need no GPU are made here: status strings, workspace sizing
and argument validation that rejects inputs before any CUDA call.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tp_block.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(tp_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def tpb():
    import tensor_llama_transformer_b200 as t

    return t


def test_every_declared_symbol_is_exported(tpb):
    names = _declared()
    assert "tp_block_forward" in names and "tp_ffn_forward" in names and len(names) >= 15
    lib = ctypes.CDLL(tpb.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    assert set(names) <= set(tpb.EXPORTED)


def test_status_strings_and_version(tpb):
    assert tpb.tp_status_string(0) == "ok"
    assert "workspace" in tpb.tp_status_string(tpb.TP_EWORKSPACE)
    assert tpb.tp_status_string(99) == "unknown status"
    assert "sm_100a" in tpb.tp_version()


def _dims(tpb, **kw):
    base = dict(dim=4096, n_heads=32, n_kv_heads=32, head_dim=128, ffn_dim=11008, vocab=32000,
                max_batch=1, max_seq=1024)
    base.update(kw)
    return tpb.make_dims(**base)


def test_workspace_sizes(tpb):
    d = _dims(tpb)
    w1 = tpb.tp_block_workspace_bytes(d, 4, tpb.TP_PART_1D, 1)
    w2 = tpb.tp_block_workspace_bytes(d, 4, tpb.TP_PART_2D, 1)
    assert 0 < w1 < w2  # the 2D stage-1 partials need room
    assert w1 % 256 == 0
    d16 = _dims(tpb, max_batch=16)
    assert tpb.tp_block_workspace_bytes(d16, 4, tpb.TP_PART_1D, 1) > w1
    m = tpb.tp_model_workspace_bytes(d, 32, 8, tpb.TP_PART_1D, 0)
    assert m > tpb.tp_block_workspace_bytes(d, 8, tpb.TP_PART_1D, 0)


@pytest.mark.parametrize("kw,n", [
    (dict(dim=4000), 4),              # dim not a multiple of 128
    (dict(head_dim=64), 4),           # head_dim other than 128 -> not supported
    (dict(n_heads=30), 4),            # heads do not divide
    (dict(n_kv_heads=8), 16),         # kv heads fewer than slices
    (dict(ffn_dim=11000), 4),         # F % (32 n) != 0
    (dict(max_batch=0), 4),
    (dict(max_batch=65), 4),
    (dict(), 0),
])
def test_invalid_dims_rejected(tpb, kw, n):
    d = _dims(tpb, **kw)
    with pytest.raises(tpb.TpError) as e:
        tpb.tp_block_workspace_bytes(d, n, tpb.TP_PART_1D, 0)
    assert e.value.status in (tpb.TP_EINVAL, tpb.TP_ENOTSUP)


def test_create_rejects_missing_workspace_before_cuda(tpb):
    d = _dims(tpb)
    w = tpb.make_weights(*([16] * 9))  # aligned fake addresses; never dereferenced
    with pytest.raises(tpb.TpError) as e:
        tpb.tp_block_create(d, 4, tpb.TP_PART_1D, 1, w, None, 0)
    assert e.value.status == tpb.TP_EWORKSPACE
    w_bad = tpb.make_weights(*([16] * 8 + [18]))
    with pytest.raises(tpb.TpError) as e:
        tpb.tp_block_create(d, 4, tpb.TP_PART_1D, 1, w_bad, 256, 1 << 40)
    assert e.value.status == tpb.TP_EALIGN


def test_ffn_plan_validation(tpb):
    desc = tpb.tp_ffn_desc(512, 18432, 73728, tpb.TP_BF16, tpb.TP_ACT_RELU, tpb.TP_PART_1D, 64, 1, 1,
                           0, tpb.TP_MERGE_FAITHFUL)
    h_bytes = 512 * 73728 * 2  # the hidden activations H, bf16
    # bf16 faithful: the partials are summed in the GEMM epilogue, no planes
    ws1d = tpb.tp_ffn_workspace_bytes(desc)
    assert h_bytes <= ws1d < h_bytes + 4096
    desc2 = tpb.tp_ffn_desc(512, 18432, 73728, tpb.TP_BF16, tpb.TP_ACT_RELU, tpb.TP_PART_2D, 64, 8,
                            8, 0, tpb.TP_MERGE_FAITHFUL)
    assert tpb.tp_ffn_workspace_bytes(desc2) == ws1d
    # ... except the 2D SwiGLU first stage: two products per hidden value, one plane
    # per E-slice each
    sw2 = tpb.tp_ffn_desc(512, 18432, 73728, tpb.TP_BF16, tpb.TP_ACT_SWIGLU, tpb.TP_PART_2D, 64, 8,
                          8, 0, tpb.TP_MERGE_FAITHFUL)
    assert tpb.tp_ffn_workspace_bytes(sw2) >= h_bytes + 2 * 8 * 512 * 73728 * 4
    # float32: every stage's partials materialised (64 planes of the row split)
    f32 = tpb.tp_ffn_desc(64, 256, 4096, tpb.TP_F32, tpb.TP_ACT_RELU, tpb.TP_PART_1D, 64, 1, 1, 0,
                          tpb.TP_MERGE_FAITHFUL)
    assert tpb.tp_ffn_workspace_bytes(f32) >= 64 * 64 * 256 * 4 + 64 * 4096 * 4 * 2
    fused = tpb.tp_ffn_desc(512, 18432, 73728, tpb.TP_BF16, tpb.TP_ACT_RELU, tpb.TP_PART_1D, 64, 1,
                            1, 0, tpb.TP_MERGE_FUSED)
    assert tpb.tp_ffn_workspace_bytes(fused) < h_bytes + 4096
    bad = tpb.tp_ffn_desc(8, 64, 250, tpb.TP_F32, tpb.TP_ACT_RELU, tpb.TP_PART_1D, 2, 1, 1, 0, 0)
    with pytest.raises(tpb.TpError):
        tpb.tp_ffn_workspace_bytes(bad)
    fused_f32 = tpb.tp_ffn_desc(8, 64, 256, tpb.TP_F32, tpb.TP_ACT_RELU, tpb.TP_PART_1D, 2, 1, 1, 0,
                                tpb.TP_MERGE_FUSED)
    with pytest.raises(tpb.TpError) as e:
        tpb.tp_ffn_workspace_bytes(fused_f32)
    assert e.value.status == tpb.TP_ENOTSUP


def test_quantize_rejects_bad_sizes(tpb):
    with pytest.raises(tpb.TpError) as e:
        tpb.tp_quantize_q8(16, 16, 16, 33, stream=0)
    assert e.value.status == tpb.TP_EINVAL
    tpb.tp_quantize_q8(16, 16, 16, 0, stream=0)  # empty input: nothing to do


def test_rank_block_sizes_and_validation(tpb):
    """A block spread over ranks: each rank's workspace covers its share of the
    heads and ffn rows plus the send / receive buffers; bad rank layouts are
    rejected before any CUDA call."""
    d = _dims(tpb)
    whole = tpb.tp_block_workspace_bytes(d, 8, tpb.TP_PART_1D, 1)
    sizes = [tpb.tp_block_rank_workspace_bytes(d, 8, 1, r, 4) for r in range(4)]
    assert len(set(sizes)) == 1 and 0 < sizes[0] < whole and sizes[0] % 256 == 0
    assert tpb.tp_block_rank_workspace_bytes(d, 8, 0, 0, 4) > sizes[0]  # float32 sync buffers
    for n, rank, world in ((8, 4, 4), (8, -1, 4), (8, 0, 0), (6, 0, 4), (4, 0, 8)):
        with pytest.raises(tpb.TpError) as e:
            tpb.tp_block_rank_workspace_bytes(d, n, 1, rank, world)
        assert e.value.status == tpb.TP_EINVAL
    w = tpb.make_weights(*([16] * 9))
    with pytest.raises(tpb.TpError) as e:
        tpb.tp_block_create_rank(d, 8, 1, 0, 4, w, None, 0)
    assert e.value.status == tpb.TP_EWORKSPACE
    with pytest.raises(tpb.TpError) as e:
        tpb.tp_block_rank_step(None, 0, 16, 16, 16, 16, 1, stream=0)
    assert e.value.status == tpb.TP_EINVAL
    with pytest.raises(tpb.TpError) as e:
        tpb.tp_block_rank_sync_bytes(None, 1)
    assert e.value.status == tpb.TP_EINVAL


def test_sequence_map_entry_points_validate(tpb):
    """Rows mapped to cache sequences: NULL handles and sequence maps are refused."""
    for call in (lambda: tpb.tp_block_forward_seq(None, 16, 16, 16, 16, 16, 1, 1, stream=0),
                 lambda: tpb.tp_model_forward_seq(None, 16, 16, 16, 16, 16, 1, 1, 16, stream=0)):
        with pytest.raises(tpb.TpError) as e:
            call()
        assert e.value.status == tpb.TP_EINVAL
