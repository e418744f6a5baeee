"""The exactness claims the kernels rest on, checked on the CPU with numpy/torch emulations
of the bit constructions (no GPU): each is a fact of the floating-point formats that a
kernel comment or a tolerance derivation states.

- the two-term bf16 split of W' (both routers): |W' - hi - lo| <= 2^-16 |W'|;
- int8 codes to fp16 by exponent bias (converter warps, weight-streaming kernel): the
  fp16 number with the bits of 1024 and the byte q + 128 in its low mantissa bits, minus
  1152, is q exactly;
- E2M1 codes to fp16 by bit placement (weight-streaming kernel): the three magnitude bits
  as the low exponent bits and the top mantissa bit give the E2M1 value times 2^-14, and
  times any E4M3 block scale the product is still exact in fp16.
"""
import numpy as np
import torch


def _bf16(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float32).numpy()


def test_two_term_bf16_split_residual():
    rng = np.random.default_rng(5)
    v = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * 0.02,
        (rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000)).astype(np.float32),
        np.array([1.0, -1.0, 1.0 + 2.0 ** -9, 3.0e38, 1.0e-30], dtype=np.float32),
    ])
    v = v[np.isfinite(v)]
    hi = _bf16(v)
    lo = _bf16(v - hi)  # the residual of a rounding to a coarser format is exact in fp32
    d = v.astype(np.float64) - hi.astype(np.float64) - lo.astype(np.float64)
    assert np.all(np.abs(d) <= 2.0 ** -16 * np.abs(v.astype(np.float64)))
    # and the bound is not loose by more than a factor of two somewhere
    rel = np.abs(d[v != 0]) / np.abs(v[v != 0].astype(np.float64))
    assert rel.max() > 2.0 ** -18


def test_int8_to_fp16_exponent_bias_is_exact():
    q = np.arange(-127, 128, dtype=np.int32)
    biased = (q + 128).astype(np.uint16)               # the byte q + 128
    bits = (np.uint16(0x6400) | biased).astype(np.uint16)  # 1024's exponent, byte in the mantissa
    h = bits.view(np.float16).astype(np.float32)
    assert np.array_equal(h, 1024.0 + q + 128)
    # fp16 subtraction of 1152 (both exact integers below 2048): q, exactly
    r = (h.astype(np.float16) - np.float16(1152)).astype(np.float32)
    assert np.array_equal(r, q.astype(np.float32))


E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _e4m3_values():
    codes = torch.arange(0, 0x7F, dtype=torch.uint8)  # positive finite codes (0x7F is NaN)
    return codes.view(torch.float8_e4m3fn).to(torch.float32).numpy()


def test_e2m1_bit_placement_and_block_scale_exact():
    # magnitude m (3 bits) -> fp16 bits m << 9 (exponent bits 10..14 get m >> 1, the top
    # mantissa bit m & 1): the E2M1 value times 2^-14, subnormals included
    m = np.arange(8, dtype=np.uint16)
    placed = (m << 9).astype(np.uint16).view(np.float16).astype(np.float64)
    assert np.array_equal(placed, E2M1 * 2.0 ** -14)
    # the sign bit: code bit 3 moved to fp16 bit 15
    neg = ((m << 9) | 0x8000).astype(np.uint16).view(np.float16).astype(np.float64)
    assert np.array_equal(neg, -E2M1 * 2.0 ** -14)
    # the move itself: a 4-bit code at bits 9..12 (sign at 12), masked with 0x1E00, plus
    # 7 x (the isolated bit 12) carries the sign to bit 15 and leaves the magnitude alone
    for code in range(16):
        x = (code << 9) & 0x1E00
        y = (x + 7 * (x & 0x1000)) & 0xFFFF
        want = ((code & 7) << 9) | (0x8000 if code & 8 else 0)
        assert y == want, code
    # times every E4M3 block scale (fp16 multiply): the exact product survives
    b = _e4m3_values().astype(np.float16)
    assert np.array_equal(b.astype(np.float64), _e4m3_values().astype(np.float64))
    prod = (placed.astype(np.float16)[:, None] * b[None, :]).astype(np.float64)
    exact = (E2M1 * 2.0 ** -14)[:, None] * _e4m3_values().astype(np.float64)[None, :]
    assert np.array_equal(prod, exact)
