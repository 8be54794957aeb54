"""Exhaustive CPU checks of the number-format facts that the tensor-core operands rely on.

The kernels never round a weight: the decode kernel feeds the int4 codes to the tensor core
as fp16 subnormals (the code bits masked in place) against fp16 activations, and the prefill
kernel feeds each weight as two exact fp16 parts s (q & 14) and s (q & 1) formed by one fp16
FMA.  These facts are properties of the IEEE half and bfloat16 formats, checked here over
every bf16 value (numpy's float16 conversion rounds to nearest even, like __float2half_rn).
"""
import numpy as np

ALL_BF16 = np.arange(1 << 16, dtype=np.uint32)


def bf16_values():
    v = (ALL_BF16 << 16).view(np.float32)
    return v[np.isfinite(v)].astype(np.float64)


def f16(x):
    with np.errstate(over="ignore"):
        return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


def test_masked_code_nibbles_are_exact_fp16_subnormals():
    # a nibble q at bits 0-3 of a half reads as q 2^-24, at bits 4-7 as q 2^-20
    q = np.arange(16, dtype=np.uint16)
    assert np.array_equal(q.view(np.float16).astype(np.float64), q * 2.0 ** -24)
    assert np.array_equal((q << 4).view(np.float16).astype(np.float64), q * 2.0 ** -20)
    # the odd element of a nibble pair, held as v / 16, makes the same product scale
    v = bf16_values()
    v = v[(np.abs(v) >= 2.0 ** -13) & (np.abs(v) < 65520.0)]
    for qq in (1, 7, 15):
        even = np.float32(qq * 2.0 ** -24) * f16(v).astype(np.float32)
        odd = np.float32(qq * 2.0 ** -20) * f16(v / 16).astype(np.float32)
        assert np.array_equal(even.astype(np.float64), qq * v * 2.0 ** -24)
        assert np.array_equal(odd.astype(np.float64), qq * v * 2.0 ** -24)


def test_activation_operand_range_and_error_bound():
    v = bf16_values()
    inside = (np.abs(v) >= 2.0 ** -13) & (np.abs(v) < 65520.0)
    # exact over the stated range, for even (v) and odd (v / 16) elements
    assert np.array_equal(f16(v[inside]), v[inside])
    assert np.array_equal(f16(v[inside] / 16) * 16, v[inside])
    # below it the error stays under 2^-20 absolute
    tiny = np.abs(v) < 2.0 ** -13
    assert np.max(np.abs(f16(v[tiny]) - v[tiny])) <= 2.0 ** -25
    assert np.max(np.abs(f16(v[tiny] / 16) * 16 - v[tiny])) <= 2.0 ** -20
    # at and beyond 65520 the even operand overflows (the kernels latch a range error there)
    big = np.abs(v) >= 65520.0
    assert big.any() and np.all(np.isinf(f16(v[big])))
    assert np.all(np.isfinite(f16(v[np.abs(v) < 65520.0])))


def test_prefill_two_part_weights_are_exact():
    # every bf16 scale with 2^-13 <= |s| < 64, every code q: one fp16 FMA (exact product
    # and sum, one rounding: the float64 value rounded once) on the masked code bits with
    # an fp16 1024 exponent gives s (q & 14) and s (q & 1) exactly
    v = bf16_values()
    s = v[(np.abs(v) >= 2.0 ** -13) & (np.abs(v) < 64.0)]
    s16, c16 = f16(s / 16), f16(-64 * s)
    assert np.array_equal(s16, s / 16) and np.array_equal(c16, -64 * s)
    assert np.array_equal(f16(s), s)
    s2, c2 = f16(s), f16(-1024 * s)
    assert np.array_equal(c2, -1024 * s)
    for q in range(16):
        # odd nibble (bits 4-7): 1024 + 16 (q & 14) and 1024 + 16 (q & 1) with s / 16, -64 s
        assert np.array_equal(f16((1024.0 + 16 * (q & 14)) * s16 + c16), s * (q & 14)), q
        assert np.array_equal(f16((1024.0 + 16 * (q & 1)) * s16 + c16), s * (q & 1)), q
        # even nibble (bits 0-3): 1024 + (q & 14) and 1024 + (q & 1) with s, -1024 s
        assert np.array_equal(f16((1024.0 + (q & 14)) * s2 + c2), s * (q & 14)), q
        assert np.array_equal(f16((1024.0 + (q & 1)) * s2 + c2), s * (q & 1)), q
    # the parts are exact fp16 numbers
    for q in range(16):
        assert np.array_equal(f16(s * (q & 14)), s * (q & 14))
        assert np.array_equal(f16(s * (q & 1)), s * (q & 1))
