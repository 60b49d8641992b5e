"""IEEE identities the dequantising dot products rely on (CPU, numpy float32).

The single-token kernel reads a code masked in place at bit offset s of a 32-bit word
as a float32 and multiplies it by an activation stored pre-scaled by 2^(P - s), where
the exponent P = 100 - e is chosen per chunk of activations from the largest exponent
e of the chunk (e clamped to [-26, 78]).  These tests check, for every code and every
position of 4- and 2-bit words:
  - the masked bit pattern read as float32 is exactly code * 2^(s - 149) (a subnormal,
    or the first normal binade when bit 23 is set);
  - the pre-scale factor 2^(P - s) and the rescale 2^(149 - P) are plain powers of two
    built from their exponents, for every exponent the clamp admits;
  - code * (x * 2^(P - s)) equals code * x * 2^(P - 149) exactly, for activations from
    2^-100 to 2^100 in magnitude (bf16 x, and fp32 h), so the per-chunk sum needs one
    rescale by 2^(149 - P);
  - the positions whose code would cross bit 24 are read from the word shifted right by
    8 without picking up bits of the neighbouring word.
"""
import numpy as np
import pytest

import oracle

PRE_EXP = 100
MIN_EXP, MAX_EXP = -26, 78


def chunk_pre(max_abs):
    """The kernel's pre-scale exponent for a chunk whose largest |activation| is max_abs."""
    bits = int(np.array([max_abs], dtype=np.float32).view(np.uint32)[0]) & 0x7FFFFFFF
    e = (bits >> 23) - 127
    return PRE_EXP - min(max(e, MIN_EXP), MAX_EXP)


def shift_pos(bits, p):
    """Bit offset at which position p of a word is masked (after the 8-bit shift when
    the code would end above bit 24)."""
    return bits * p - 8 if bits * p + bits > 24 else bits * p


def as_f32(pattern):
    return np.array([pattern], dtype=np.uint32).view(np.float32)[0]


@pytest.mark.parametrize("bits", [4, 2])
def test_masked_code_reads_as_scaled_subnormal(bits):
    for p in range(32 // bits):
        s = shift_pos(bits, p)
        assert 0 <= s and s + bits <= 24
        for c in range(1 << bits):
            v = float(as_f32(c << s))
            assert v == c * 2.0 ** (s - 149), (bits, p, c)


@pytest.mark.parametrize("bits", [4, 2])
def test_prescale_and_rescale_are_powers_of_two(bits):
    for e in range(MIN_EXP, MAX_EXP + 1):
        pre = PRE_EXP - e
        assert float(as_f32((127 + 149 - pre) << 23)) == 2.0 ** (149 - pre)
        for p in range(32 // bits):
            s = shift_pos(bits, p)
            assert 1 <= 127 + pre - s <= 254
            assert float(as_f32((127 + pre - s) << 23)) == 2.0 ** (pre - s)


@pytest.mark.parametrize("bits", [4, 2])
@pytest.mark.parametrize("magnitude", [1e-20, 2.0 ** -30, 1.0, 2.0 ** 20, 2.0 ** 46, 2.0 ** 64])
def test_products_with_prescaled_activations_are_exact(bits, magnitude):
    """A chunk of bf16 activations spread over about +-13 binades around `magnitude`
    (and an fp32 chunk of the same spread, as h is), its largest exponent inside the
    clamp: pre-scaled values are finite and exact; every product with a masked code is
    exact for bf16 activations and the correctly rounded fp32 product (no underflow)
    for fp32 ones."""
    rng = np.random.default_rng(0)
    z = rng.standard_normal(64) * np.exp(rng.standard_normal(64) * 3)
    for exact, x in ((True, oracle.bf16_to_f64(oracle.f64_to_bf16_bits(z * magnitude))),
                     (False, (z * magnitude).astype(np.float32).astype(np.float64))):
        pre = chunk_pre(np.max(np.abs(x)))
        for p in range(32 // bits):
            s = shift_pos(bits, p)
            xs = (x * 2.0 ** (pre - s)).astype(np.float32)
            assert np.all(np.isfinite(xs))
            assert np.array_equal(xs.astype(np.float64), x * 2.0 ** (pre - s))  # scaling is exact
            for c in range(1 << bits):
                prod = (as_f32(c << s) * xs).astype(np.float64)   # float32 multiply
                want = c * x * 2.0 ** (pre - 149)
                if not exact:
                    want = want.astype(np.float32).astype(np.float64)
                assert np.array_equal(prod, want), (bits, p, c)


@pytest.mark.parametrize("bits", [4, 2])
def test_prescaled_values_stay_finite_outside_the_clamp(bits):
    """Chunks whose largest exponent lies outside the clamp: up to |x| < 2^105 the
    pre-scaled values are finite, and products of the chunk's largest entries are
    still exact; tiny chunks (down to 2^-100) never overflow either."""
    for mx in (2.0 ** 79, 2.0 ** 90, 2.0 ** 104.9, 2.0 ** -27, 2.0 ** -60, 2.0 ** -100):
        x = np.array([mx, mx / 3.0, -mx / 7.0, mx / 1024.0])
        x = oracle.bf16_to_f64(oracle.f64_to_bf16_bits(x))
        pre = chunk_pre(np.max(np.abs(x)))
        for p in range(32 // bits):
            s = shift_pos(bits, p)
            xs = (x * 2.0 ** (pre - s)).astype(np.float32)
            assert np.all(np.isfinite(xs)), (mx, p)
            c = (1 << bits) - 1
            prod = (as_f32(c << s) * xs[:1]).astype(np.float64)
            if mx >= 2.0 ** -50:
                assert np.array_equal(prod, c * x[:1] * 2.0 ** (pre - 149)), (mx, p)


@pytest.mark.parametrize("bits", [4, 2])
def test_shifted_pair_does_not_mix_words(bits):
    """Two words viewed as one 64-bit value (w_a low, w_b high), shifted right by 8: the
    masks of the high positions select only w_a's (resp. w_b's) own bits."""
    rng = np.random.default_rng(1)
    for _ in range(200):
        wa, wb = (int(v) for v in rng.integers(0, 2 ** 32, size=2, dtype=np.uint64))
        pair = (wb << 32) | wa
        shifted = pair >> 8
        for p in range(32 // bits):
            if bits * p + bits <= 24:
                continue
            s = shift_pos(bits, p)
            m32 = ((1 << bits) - 1) << s
            mask = (m32 << 32) | m32
            got = shifted & mask
            code_a = (wa >> (bits * p)) & ((1 << bits) - 1)
            code_b = (wb >> (bits * p)) & ((1 << bits) - 1)
            assert got == ((code_b << s) << 32) | (code_a << s), (bits, p)


# ------------------------------------------------------------- batched path --
# The grouped (tensor-core) matvecs enter a code c as the bf16 value 1 + c/2^b' (b' = 4
# for 4-bit codes, 2 for 2-bit), built by one rotate and one mask-and-or from the code
# word, and fold each 64-column group's accumulator D = sum (1 + c/2^b') x with the
# group's scale and bias.

def rotr(w, n):
    n &= 31
    return ((w >> n) | (w << (32 - n))) & 0xFFFFFFFF if n else w


def bf16_value(bits16):
    return float(np.array([bits16 << 16], dtype=np.uint32).view(np.float32)[0])


def test_rotate_builds_bf16_pairs_of_4bit_codes():
    rng = np.random.default_rng(2)
    for w in [0, 0xFFFFFFFF, 0x76543210, 0xFEDCBA98] + [int(v) for v in rng.integers(0, 2 ** 32, 50, dtype=np.uint64)]:
        for q in range(4):
            r = (rotr(w, 4 * q - 3) & 0x00780078) | 0x3F803F80
            lo, hi = (w >> (4 * q)) & 15, (w >> (4 * (q + 4))) & 15
            assert bf16_value(r & 0xFFFF) == 1 + lo / 16 and bf16_value(r >> 16) == 1 + hi / 16


def test_rotate_builds_bf16_pairs_of_2bit_codes():
    rng = np.random.default_rng(3)
    for w in [0, 0xFFFFFFFF, 0xE4E4E4E4] + [int(v) for v in rng.integers(0, 2 ** 32, 50, dtype=np.uint64)]:
        for q in range(4):
            for h in range(2):
                r = (rotr(w, 2 * q + 8 * h - 5) & 0x00600060) | 0x3F803F80
                k = q + 4 * h
                lo, hi = (w >> (2 * k)) & 3, (w >> (2 * (k + 8))) & 3
                assert bf16_value(r & 0xFFFF) == 1 + lo / 4 and bf16_value(r >> 16) == 1 + hi / 4


@pytest.mark.parametrize("bits", [4, 2])
def test_group_fold_identity_is_exact(bits):
    """sum_c (s c + b) x_c = (2^b' s) D + (b - 2^b' s) X, in exact rational arithmetic."""
    from fractions import Fraction
    rng = np.random.default_rng(4)
    for _ in range(20):
        c = rng.integers(0, 1 << bits, 64)
        x = oracle.bf16_to_f64(oracle.f64_to_bf16_bits(rng.standard_normal(64)))
        s = float(oracle.bf16_to_f64(oracle.f64_to_bf16_bits(np.array([abs(rng.standard_normal()) * 0.02])))[0])
        b = float(oracle.bf16_to_f64(oracle.f64_to_bf16_bits(
            np.array([-(2 ** bits / 2) * s + rng.standard_normal() * 1e-3])))[0])
        F = [Fraction(float(v)) for v in x]
        lhs = sum((Fraction(s) * int(ci) + Fraction(b)) * xi for ci, xi in zip(c, F))
        D = sum((1 + Fraction(int(ci), 2 ** bits)) * xi for ci, xi in zip(c, F))
        X = sum(F)
        assert lhs == Fraction(2 ** bits) * Fraction(s) * D + (Fraction(b) - Fraction(2 ** bits) * Fraction(s)) * X


@pytest.mark.parametrize("bits", [4, 2])
def test_fold_coefficients_exact_in_fp32_for_the_workload(bits):
    """b - 2^b' s is exact in float32 for the workload's (scale, bias) values."""
    import fmoe_synth as synth
    p = synth.gen_expert(0, 0, 3, 512, 128, bits)
    for sb in (p.gate_sb, p.up_sb, p.down_sb):
        s = oracle.bf16_to_f64((sb & 0xFFFF).astype(np.uint16))
        b = oracle.bf16_to_f64((sb >> 16).astype(np.uint16))
        f32 = (b.astype(np.float32) - (s * 2 ** bits).astype(np.float32)).astype(np.float64)
        assert np.array_equal(f32, b - s * 2 ** bits)


# The tcgen05 form of the same product: a converter thread turns a group's code words
# into 32 TMEM words (4-bit word m -> columns 4m + j, j = 0..3, pair (code j, code j+4);
# 2-bit word m -> columns 8m + j, j = 0..7, pair (code j, code j+8)); the MMA reads a
# TMEM column as K positions 2c (low half) and 2c + 1 (high half).  The activation
# tiles put column col of a row at K position kpos(col); every code must meet its own
# activation.
def _kpos(bits, c):
    if bits == 4:
        return (c & ~7) + 2 * (c & 3) + ((c >> 2) & 1)
    return (c & ~15) + 2 * (c & 7) + ((c >> 3) & 1)


@pytest.mark.parametrize("bits", [4, 2])
def test_tcgen05_k_order_pairs_every_code_with_its_activation(bits):
    rng = np.random.default_rng(40 + bits)
    per = 32 // bits
    assert sorted(_kpos(bits, c) for c in range(64)) == list(range(64))  # a permutation of the group
    for _ in range(20):
        words = [int(v) for v in rng.integers(0, 2 ** 32, 64 // per, dtype=np.uint64)]
        x = rng.standard_normal(64)
        cols = {}  # TMEM column -> 32-bit word
        for m, w in enumerate(words):
            if bits == 4:
                for j in range(4):
                    cols[4 * m + j] = (rotr(w, 4 * j - 3) & 0x00780078) | 0x3F803F80
            else:
                for j in range(8):
                    cols[8 * m + j] = (rotr(w, 2 * j - 5) & 0x00600060) | 0x3F803F80
        assert sorted(cols) == list(range(32))
        a = np.zeros(64)
        for c, r in cols.items():
            a[2 * c], a[2 * c + 1] = bf16_value(r & 0xFFFF), bf16_value(r >> 16)
        b = np.zeros(64)
        for col in range(64):
            b[_kpos(bits, col)] = x[col]
        codes = [(words[col // per] >> (bits * (col % per))) & ((1 << bits) - 1) for col in range(64)]
        want = sum((1 + codes[col] / 2 ** bits) * x[col] for col in range(64))
        assert abs(float(a @ b) - want) <= 1e-12 * (1 + np.abs(x).sum())
