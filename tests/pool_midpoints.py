"""Hand-built key caches whose 32-key window means sit on, or a hair beside, a bf16 rounding midpoint.

The semantic kernel is the window mean rounded once to bf16 ("Tsinghua & ModelBest: MiniCPM4 technical
details", "Model architecture: InfLLM v2", item 1; the rounding point is this library's reading).  Every
planted column below mixes a large key (32), a mid-sized one and a tiny one (2^-30).  The exact sum of the
window is a bf16 midpoint plus or minus 2^-30; an fp32 sum drops the tiny key (fp32 spacing at 32 is 2^-18),
lands exactly on the midpoint and then rounds to even, the wrong way.  A correctly rounded mean does not.

All other keys are 0, so each column's window means are worked out by hand below; the expected bf16 bit
patterns are literals, not the output of any implementation:
  1.0 = 0x3f80, 1 + 2^-7 = 0x3f81, 1 + 2^-6 = 0x3f82, -(1 + 2^-7) = 0xbf81, 2^-35 = 0x2e00.
Windows are [16 j, 16 j + 32); a 96-key cache has windows j = 0..4.
"""
import numpy as np

from trainable_block_sparse_v2_b200.workloads import f32_to_bf16_bits

L = 96
TINY = 2.0 ** -30

# (head, dim, {key position: value}, {window j: expected bf16 bits}); windows not listed are 0
COLUMNS = [
    # window 0: (32 + 1/8 + 2^-30) / 32 = 1 + 2^-8 + 2^-35, just above the midpoint of 1 and 1 + 2^-7
    (0, 1, {2: 32.0, 7: 0.125, 11: TINY}, {0: 0x3F81}),
    # window 0 holds 32 and 1/8 only: exactly the midpoint 1 + 2^-8, ties to the even 1.0;
    # window 1 holds all three, split over its two 16-key halves: above the midpoint, 1 + 2^-7;
    # window 2 holds only the tiny key: 2^-30 / 32 = 2^-35, exact
    (1, 2, {20: 32.0, 21: 0.125, 40: TINY}, {0: 0x3F80, 1: 0x3F81, 2: 0x2E00}),
    # the negative of the first column
    (0, 5, {3: -32.0, 4: -0.125, 6: -TINY}, {0: 0xBF81}),
    # windows 2 and 3: (32 + 3/8 - 2^-30) / 32 = 1 + 3 * 2^-8 - 2^-35, just below the midpoint of
    # 1 + 2^-7 (odd) and 1 + 2^-6 (even): rounds down to 1 + 2^-7 (an fp32 sum ties up to 1 + 2^-6)
    (1, 7, {50: 32.0, 55: 0.375, 60: -TINY}, {2: 0x3F81, 3: 0x3F81}),
    # windows 3 and 4: exactly that midpoint, ties to the even 1 + 2^-6
    (0, 9, {70: 32.0, 71: 0.375}, {3: 0x3F82, 4: 0x3F82}),
]


def midpoint_case(d: int):
    """Returns (K [1, 96, 2, d] bf16 bits, expected kern [1, 2, 5, d] bf16 bits)."""
    K = np.zeros((1, L, 2, d), np.float32)
    want = np.zeros((1, 2, 5, d), np.uint16)
    for h, c, keys, wins in COLUMNS:
        for pos, v in keys.items():
            K[0, pos, h, c] = v
        for j, bits in wins.items():
            want[0, h, j, c] = bits
    Kb = f32_to_bf16_bits(K)
    # every planted value is a bf16 value, so the cast is exact
    assert np.array_equal((Kb.astype(np.uint32) << 16).view(np.float32), K)
    return Kb, want


def rne_bf16_of_exact_mean(values) -> int:
    """The exact rational mean of some bf16 values, rounded once to bf16 (nearest, ties to even), by hand
    with Python fractions: independent of both the oracle and the library."""
    from fractions import Fraction
    q = sum(Fraction(float(v)) for v in values) / len(values)
    if q == 0:
        return 0
    sign = 0x8000 if q < 0 else 0
    q = abs(q)
    e = q.numerator.bit_length() - q.denominator.bit_length()
    if Fraction(2) ** e > q:
        e -= 1
    m = q / Fraction(2) ** (e - 7)  # significand scaled to [128, 256)
    fl = m.numerator // m.denominator
    rest = m - fl
    if rest > Fraction(1, 2) or (rest == Fraction(1, 2) and fl % 2):
        fl += 1
    if fl == 256:
        fl, e = 128, e + 1
    assert -126 <= e <= 127, "normal range only"
    return sign | ((e + 127) << 7) | (fl - 128)
