"""Q8 sync-buffer codec on the GPU: codes and scales bit-exact with the oracle.

The oracle's quantiser (pinned by tests/test_oracle_q8.py) and the CUDA codec
get identical float32 inputs; every code and scale must match bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.test_oracle_q8 import _golden_blocks

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tpb(cuda_ok):
    import tensor_llama_transformer_b200 as t

    return t


def _gpu_q8(tpb, x: np.ndarray):
    n = x.size
    xt = torch.from_numpy(np.ascontiguousarray(x, np.float32).ravel()).cuda()
    q = torch.empty(n, dtype=torch.int8, device="cuda")
    d = torch.empty(n // 32, dtype=torch.float32, device="cuda")
    tpb.tp_quantize_q8(xt, q, d, n)
    back = torch.empty(n, dtype=torch.float32, device="cuda")
    tpb.tp_dequantize_q8(q, d, back, n)
    torch.cuda.synchronize()
    return q.cpu().numpy(), d.cpu().numpy(), back.cpu().numpy()


def _edge_cases():
    rng = np.random.default_rng(11)
    blocks = [b[0] for b in _golden_blocks()]
    z = np.zeros(32, np.float32)
    blocks.append(z.copy())                                   # all zero
    nz = z.copy(); nz[:] = -0.0; blocks.append(nz)            # all -0
    t = np.zeros(32, np.float32); t[0] = 127; t[1:] = np.arange(-15, 16) + 0.5
    blocks.append(t)                                          # ties at .5
    h = np.zeros(32, np.float32); h[0] = 127
    h[1] = np.nextafter(np.float32(0.5), np.float32(0)); h[2] = np.nextafter(np.float32(1.5), np.float32(0))
    blocks.append(h)                                          # just below .5
    dn = np.zeros(32, np.float32); dn[0] = np.float32(1e-40); dn[5] = np.float32(-3e-41)
    blocks.append(dn)                                         # denormal scale
    tiny = np.zeros(32, np.float32); tiny[7] = np.float32(1e-44)
    blocks.append(tiny)                                       # scale underflows to 0
    for pos in (0, 13, 31):                                   # amax at several positions
        b = rng.standard_normal(32).astype(np.float32)
        b[pos] = 50.0 * (1 if pos % 2 else -1)
        blocks.append(b)
    big = (rng.standard_normal(32) * 3e37).astype(np.float32)
    blocks.append(big)                                        # near the float32 range
    return np.concatenate(blocks)


def _near_ties(rng, nblocks=20_000):
    """Blocks whose quotients x/d sit within a few ulp of k + 1/2 (and exactly on
    it), where the rounded code depends on the last bit of the quotient."""
    amax = rng.uniform(1e-3, 1e3, nblocks).astype(np.float32)
    d = (amax / np.float32(127)).astype(np.float32)
    k = rng.integers(-127, 127, (nblocks, 31)).astype(np.float32)
    off = rng.choice(np.array([-2e-4, -5e-5, -4.2e-5, -3e-5, -1e-5, -1e-6, 0.0, 1e-6, 1e-5,
                              3e-5, 4.2e-5, 5e-5, 2e-4], np.float32), (nblocks, 31))
    vals = ((k + np.float32(0.5) + off) * d[:, None]).astype(np.float32)
    vals = np.clip(vals, -amax[:, None], amax[:, None])
    return np.concatenate([amax[:, None], vals], axis=1).astype(np.float32).ravel()


@pytest.mark.parametrize("kind", ["edge", "random", "ragged_large", "near_ties"])
def test_q8_bit_exact(tpb, kind):
    rng = np.random.default_rng(3)
    if kind == "edge":
        x = _edge_cases()
    elif kind == "near_ties":
        x = _near_ties(rng)
    elif kind == "random":
        x = (rng.standard_normal(4096 * 37) * rng.uniform(1e-6, 1e4, 4096 * 37)).astype(np.float32)
    else:  # not a multiple of the grid stride or of a warp's 1024 values
        x = rng.standard_normal(32 * 100_003).astype(np.float32) * 7
    q, d, back = _gpu_q8(tpb, x)
    q_ref, d_ref = oracle.q8_quantize(x.reshape(1, -1))
    np.testing.assert_array_equal(d.view(np.uint32), d_ref.ravel().view(np.uint32))
    np.testing.assert_array_equal(q, q_ref.ravel())
    np.testing.assert_array_equal(back.view(np.uint32),
                                  oracle.q8_dequantize(q_ref, d_ref).ravel().view(np.uint32))


def test_q8_empty_is_noop(tpb):
    x = torch.empty(0, device="cuda")
    tpb.tp_quantize_q8(x, x, x, 0)
    tpb.tp_dequantize_q8(x, x, x, 0)
