"""The arithmetic the tensor-core fp32 path (GQA_F32_TC) rests on, checked on the CPU
with numpy's IEEE float16 (no GPU, no library code).

After the per-head power-of-two scaling, an operand x' has |x'| < 2^15 and is held as
hi = fp16(x'), lo = fp16(x' - hi).  The bounds used in the kernel's error budget:
  * |x' - hi - lo| <= 2^-22 |x'| while lo stays a normal fp16 number, and an absolute
    2^-25 (half of fp16's subnormal spacing) below that;
  * hi_a hi_b + hi_a lo_b + lo_a hi_b (the three MMAs) is within about 3 * 2^-22 of
    x'_a x'_b relative to |x'_a x'_b|;
  * a two-term bf16 split (8 significant bits per term) would be off by up to 2^-16,
    the reason the kernel splits into fp16 rather than bf16.
"""

import numpy as np


def _split16(x):
    hi = x.astype(np.float16).astype(np.float64)
    lo = (x - hi).astype(np.float16).astype(np.float64)
    return hi, lo


def _bf16(x):
    """Round-to-nearest-even to bfloat16 (top 16 bits of the float32 pattern)."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return b.astype(np.uint32).view(np.float32).astype(np.float64)


def _scaled_operands(n, seed):
    """fp32 values with |x'| in [2^-6, 2^15): the range of a scaled N(0,1) head that
    still carries weight in a dot product (the scale puts the head's maximum in
    [2^14, 2^15))."""
    rng = np.random.default_rng(seed)
    mag = 2.0 ** rng.uniform(-6, 15, n)
    return (mag * rng.choice([-1.0, 1.0], n)).astype(np.float32).astype(np.float64)


def test_two_term_fp16_split_holds_22_bits():
    x = _scaled_operands(200_000, 1)
    hi, lo = _split16(x)
    normal_lo = np.abs(x) >= 2.0 ** -3  # lo ~ 2^-11 x' stays >= 2^-14 (fp16 normal)
    rel = np.abs(x - hi - lo) / np.abs(x)
    assert float(rel[normal_lo].max()) <= 2.0 ** -22
    assert float(np.abs(x - hi - lo)[~normal_lo].max()) <= 2.0 ** -25


def test_three_products_bound():
    a = _scaled_operands(200_000, 2)
    b = _scaled_operands(200_000, 3)
    keep = (np.abs(a) >= 2.0 ** -3) & (np.abs(b) >= 2.0 ** -3)
    a, b = a[keep], b[keep]
    ah, al = _split16(a)
    bh, bl = _split16(b)
    approx = ah * bh + ah * bl + al * bh  # each product exact in fp64 (11 x 11 bits)
    rel = np.abs(approx - a * b) / np.abs(a * b)
    assert float(rel.max()) <= 3 * 2.0 ** -22
    # the dropped term is what the bound is made of: adding it back leaves only the
    # two split remainders
    full = approx + al * bl
    assert float((np.abs(full - a * b) / np.abs(a * b)).max()) <= 2 * 2.0 ** -22 + 2.0 ** -40


def test_bf16_two_terms_would_not_reach_fp32_accuracy():
    x = _scaled_operands(200_000, 4) / 2.0 ** 10
    hi = _bf16(x)
    lo = _bf16(x - hi)
    rel = np.abs(x - hi - lo) / np.abs(x)
    assert float(rel.max()) > 2.0 ** -20          # far above fp16's 2^-22
    assert float(rel.max()) <= 2.0 ** -16


def test_probability_bias_lowers_the_error_floor():
    # P = 2^(s - m + 6) <= 2^14 < 65504 (lazy-max threshold 8).  The split of P is exact
    # to 2^-22 relative while lo is a normal fp16 number (P' >= 2^-3); below that its
    # error is at most 2^-25 absolute (half of fp16's subnormal spacing).  A row's
    # largest term is >= 2^6 after the bias, so every probability is held to 2^-31 of
    # it -- 2^6 better than unbiased probabilities in (0, 1].
    p = 2.0 ** np.linspace(-40, 8, 8001)
    ps = (p * 2.0 ** 6).astype(np.float32).astype(np.float64)
    assert float(ps.max()) <= 2.0 ** 14 < 65504
    hi, lo = _split16(ps)
    err = np.abs(ps - hi - lo)
    big = ps >= 2.0 ** -3
    assert float((err[big] / ps[big]).max()) <= 2.0 ** -22
    assert float(err[~big].max()) <= 2.0 ** -25
    assert float(err[~big].max()) / 2.0 ** 6 <= 2.0 ** -31
