"""The arithmetic the quantized decode kernels use to widen codes on chip, checked exhaustively on the CPU.

FP8 (decode_fp8.cuh, e4m3_pairs_to_bf16x2): a code shifted left by 4, with its sign moved from bit 11 to bit 15
by adding 15 times that bit, read as a bf16 and multiplied by 2^120, is the E4M3 value. NVFP4 (e2m1_pair_to_bf16x2):
a code's exponent and mantissa bits moved to bits 8..6 and its sign to bit 15, read as a bf16, is 2^-126 times the
E2M1 value; multiplied by (block scale x 2^63) it must be the weight times 2^-63, a normal bf16 that the multiply
does not round. Checked here for every code and every block scale, against torch's own float8 decode and the
E2M1 table of the format."""

import numpy as np
import torch

E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _bf16(bits16: int) -> float:
    return float(np.array([bits16 << 16], dtype=np.uint32).view(np.float32)[0])


def _bf16_exact(v: float) -> bool:
    """v is a bf16 value: 8 significant bits and within bf16's exponent range (normal or zero)."""
    if v == 0.0:
        return True
    m, e = np.frexp(abs(v))  # v = m 2^e, m in [0.5, 1)
    return float(m * 256.0).is_integer() and -125 <= e <= 128


def test_e4m3_widening_is_exact():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            continue  # NaN codes: the fold never writes them
        t = (c << 4) & 0xFFFF
        f = ((t & 0x0800) * 15 + t) & 0xFFFF
        val = _bf16(f) * 2.0 ** 120
        assert val == ref[c] and np.signbit(val) == np.signbit(ref[c]), c


def test_e2m1_widening_times_block_scale_is_exact():
    scales = torch.from_numpy(np.arange(256, dtype=np.uint8)).view(torch.float8_e4m3fn).float().numpy()
    for c in range(16):
        bits = ((c & 7) << 6) | ((c & 8) << 12)
        want = (-1.0 if c & 8 else 1.0) * E2M1_TABLE[c & 7]
        assert _bf16(bits) * 2.0 ** 126 == want, c
        for s in range(0x7F):  # the non-negative E4M3 scales the fold writes (0 included)
            scale63 = float(scales[s]) * 2.0 ** 63
            assert _bf16_exact(scale63), s
            prod = _bf16(bits) * scale63        # exact in fp64: at most 6 significant bits
            assert _bf16_exact(prod), (c, s)    # so the bf16 multiply returns it unrounded
            assert prod == want * float(scales[s]) * 2.0 ** -63


def _e2m1_by_midpoints(t: np.ndarray) -> np.ndarray:
    """The fold kernel's E2M1 rounding (fp8.cuh, e2m1_rn_satfinite): the count of midpoints a magnitude passes,
    strict where the lower neighbour has the even code, inclusive where the upper one has, and the sign bit."""
    a = np.abs(t)
    m = ((a > 0.25).astype(np.uint8) + (a >= 0.75) + (a > 1.25) + (a >= 1.75) + (a > 2.5) + (a >= 3.5) + (a > 5.0))
    return (m | np.where(np.signbit(t), 8, 0)).astype(np.uint8)


def test_e2m1_rounding_by_midpoints_matches_the_oracle():
    """Every midpoint between neighbouring E2M1 magnitudes, its float32 neighbours on both sides, both signs, and
    random values: the comparison form and the oracle's round-to-nearest-even agree code for code."""
    from oracle import flashnorm_oracle as O

    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=np.float32)
    around = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(10)),
                             np.array(E2M1_TABLE, dtype=np.float32), np.array([6.5, 100.0, 3e38], dtype=np.float32)])
    rng = np.random.default_rng(3)
    vals = np.concatenate([around, -around, rng.uniform(-8, 8, 20000).astype(np.float32), np.float32([0.0, -0.0])])
    assert np.array_equal(_e2m1_by_midpoints(vals), O.f64_to_e2m1(vals.astype(np.float64)))
