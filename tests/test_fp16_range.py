"""The FP8 decode's fp16 operand contract, checked with IEEE fp16 on the host.

The FP8 instance of the decode kernel expands each cached E4M3 code to fp16
and multiplies it by the token's power-of-two scale as an fp16 pair. The
claim behind that: for scales 2^k with k in [-15, 7] every product is exact
on the fp16 grid (so the kernel sees exactly the dequantized value the
oracle uses); below 2^-15 only the smallest codes round (absolute error below
2^-25); above 2^7 the largest codes overflow, which the kernel reports as
MLA_DEV_RANGE. The same holds for the query's bf16 latent values in fp16's
normal range. numpy's float16 is IEEE binary16 with round-to-nearest-even,
like the hardware's conversion and multiply.
"""

import numpy as np

from oracle import mla_oracle as O


def _finite_codes():
    codes = np.arange(256, dtype=np.uint8)
    vals = O.e4m3_value(codes)
    keep = np.isfinite(vals)
    return codes[keep], vals[keep]


def test_every_code_times_an_in_range_scale_is_exact_in_fp16():
    _, vals = _finite_codes()
    for k in range(-15, 8):
        s = np.float16(2.0 ** k)
        got = (vals.astype(np.float16) * s).astype(np.float64)
        assert np.array_equal(got, vals * 2.0 ** k), k


def test_below_the_range_only_tiny_values_round():
    _, vals = _finite_codes()
    for k in range(-24, -15):
        got = (vals.astype(np.float16) * np.float16(2.0 ** k)).astype(np.float64)
        err = np.abs(got - vals * 2.0 ** k)
        assert err.max() <= 2.0 ** -25, k


def test_above_the_range_the_largest_codes_overflow():
    _, vals = _finite_codes()
    with np.errstate(over="ignore"):
        got = vals.astype(np.float16) * np.float16(2.0 ** 8)
    assert np.isinf(got).any()


def test_bf16_values_in_the_fp16_normal_range_convert_exactly():
    rng = np.random.default_rng(3)
    x = rng.standard_normal(200000) * np.exp2(rng.integers(-13, 15, 200000))
    bits = O.round_to_bf16(x)
    b = O.bf16_to_f64(bits)
    b = b[(np.abs(b) >= 2.0 ** -14) & (np.abs(b) < 65504)]
    assert np.array_equal(b.astype(np.float16).astype(np.float64), b)
