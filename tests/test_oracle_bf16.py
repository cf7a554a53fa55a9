"""Pin of the oracle's bf16 rounding (CPU only).

The KV-cache layout stores bf16, so the k and v rows a decode step writes at
``pos`` are rounded from float32 to bf16 (round to nearest, ties to even).
``oracle.round_to_bf16`` is checked here against an implementation that shares
nothing with it: PyTorch's float32 -> bfloat16 conversion, on the inputs where
a rounding rule shows itself -- exact ties with both parities of the kept last
bit, the neighbours one float32 ulp either side of a tie, subnormals, signed
zeros, the largest finite values (which round up to infinity) and values spread
over every exponent. A truncating, ties-away or ties-odd rounding fails here.
"""
import numpy as np
import torch

import oracle


def _torch_bf16_bits(f32: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(f32, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _from_bits(u32) -> np.ndarray:
    return np.asarray(u32, dtype=np.uint32).view(np.float32)


def _edge_patterns() -> np.ndarray:
    hi = np.array([0x0000, 0x0001, 0x0002, 0x0003, 0x007F, 0x0080, 0x3F80, 0x3F81, 0x4049,
                   0x7F7E, 0x7F7F, 0x1234, 0x00FF], dtype=np.uint32)
    lo = np.array([0x0000, 0x0001, 0x7FFE, 0x7FFF, 0x8000, 0x8001, 0xFFFE, 0xFFFF],
                  dtype=np.uint32)
    pats = (hi[:, None] << np.uint32(16)) | lo[None, :]
    pats = pats.ravel()
    return np.concatenate([pats, pats | np.uint32(0x80000000)])


def test_round_to_bf16_matches_torch_on_edges():
    f = _from_bits(_edge_patterns())
    assert np.all(np.isfinite(f))
    got = oracle.round_to_bf16(f.astype(np.float64))
    np.testing.assert_array_equal(got, _torch_bf16_bits(f))


def test_round_to_bf16_ties_go_to_even():
    # kept part even (bit 16 clear) -> a tie rounds down; odd -> up
    even_tie = _from_bits([0x3F808000])  # 1.0 + half a bf16 ulp
    odd_tie = _from_bits([0x3F818000])
    assert oracle.round_to_bf16(even_tie.astype(np.float64))[0] == 0x3F80
    assert oracle.round_to_bf16(odd_tie.astype(np.float64))[0] == 0x3F82
    # one float32 ulp either side of a tie: never a tie, nearest wins
    assert oracle.round_to_bf16(_from_bits([0x3F807FFF]).astype(np.float64))[0] == 0x3F80
    assert oracle.round_to_bf16(_from_bits([0x3F808001]).astype(np.float64))[0] == 0x3F81


def test_round_to_bf16_subnormals_zero_and_overflow():
    sub = _from_bits(np.arange(1, 1 << 16, 97, dtype=np.uint32))  # float32 subnormals
    np.testing.assert_array_equal(oracle.round_to_bf16(sub.astype(np.float64)),
                                  _torch_bf16_bits(sub))
    z = np.array([0.0, -0.0])
    np.testing.assert_array_equal(oracle.round_to_bf16(z), np.array([0x0000, 0x8000], np.uint16))
    big = _from_bits([0x7F7FFFFF, 0xFF7FFFFF, 0x7F7F7FFF])
    np.testing.assert_array_equal(oracle.round_to_bf16(big.astype(np.float64)),
                                  np.array([0x7F80, 0xFF80, 0x7F7F], np.uint16))


def test_round_to_bf16_random_bit_patterns():
    rng = np.random.default_rng(20261203)
    u = rng.integers(0, 1 << 32, size=200_000, dtype=np.uint64).astype(np.uint32)
    f = _from_bits(u)
    f = f[np.isfinite(f)]
    np.testing.assert_array_equal(oracle.round_to_bf16(f.astype(np.float64)), _torch_bf16_bits(f))


def test_round_to_bf16_goes_through_float32():
    # float64 input: rounded to float32 first (the kernels compute the row in float32).
    # 1 + 2^-8 + 2^-30 is a tie once in float32 (ties to even: 1.0), though the float64
    # value lies above the tie (a direct float64 rounding would give 1 + 2^-7).
    x = np.array([1.0 + 2.0 ** -8 + 2.0 ** -30, -3.0 - 2.0 ** -9 + 2.0 ** -45, 1e-42, 7.1e37])
    f = x.astype(np.float32)
    got = oracle.round_to_bf16(x)
    np.testing.assert_array_equal(got, _torch_bf16_bits(f))
    assert got[0] == 0x3F80
