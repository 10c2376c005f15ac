"""The integer form of the E4M3 -> bf16 expansion used by the quantised cache and the FP8
weights (csrc/e4m3_bf16.cuh), checked on the host for every code and every exponent the
kernels accept: a code's bits placed into a bf16 as (s << 15) | ((c & 0x7F) << 4), then one
bf16 multiply by 2^(120 + e) (e <= 7) or two, by 2^120 and then 2^e (e > 7), each rounded to
nearest, give the bf16 nearest to 2^e times the code's value (the oracle's E4M3 decode,
OCP FP8 E4M3), which is that value exactly while it is a normal bf16 number.

The bf16 multiply is emulated as the exact product (float64: every factor here is a power of
two times at most four significant bits) rounded to nearest-even bf16, which is how the
hardware's round-to-nearest multiply is defined."""

import numpy as np
import torch

import oracle

CODES = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)  # NaN codes


def _bf16_round(x: np.ndarray) -> np.ndarray:
    """Nearest-even bf16 of float64 values exactly representable in float32."""
    f32 = torch.from_numpy(x.astype(np.float32))
    assert np.array_equal(f32.double().numpy(), x), "product not exact in float32"
    return f32.to(torch.bfloat16).double().numpy()


def _bits_to_bf16(bits: np.ndarray) -> np.ndarray:
    return torch.from_numpy((bits.astype(np.int32) << 16).astype(np.int32)).view(torch.float32).double().numpy()


def _integer_form(codes: np.ndarray, e: int) -> np.ndarray:
    c = codes.astype(np.uint32)
    placed = _bits_to_bf16(((c & 0x80) << 8) | ((c & 0x7F) << 4))
    if e <= 7:
        return _bf16_round(placed * 2.0 ** (120 + e))
    return _bf16_round(_bf16_round(placed * 2.0 ** 120) * 2.0 ** e)


def test_placed_bits_are_the_code_value_times_two_to_the_minus_120():
    c = CODES.astype(np.uint32)
    placed = _bits_to_bf16(((c & 0x80) << 8) | ((c & 0x7F) << 4))
    assert np.array_equal(placed * 2.0 ** 120, oracle.e4m3_decode(CODES))


def test_integer_form_equals_the_rounded_scaled_code_for_every_exponent():
    ref_codes = oracle.e4m3_decode(CODES)
    for e in range(-126, 21):   # the kernels clamp e to [-126, 127]; 8..20 take two multiplies
        got = _integer_form(CODES, e)
        want = _bf16_round(ref_codes * 2.0 ** e)
        assert np.array_equal(got, want), e
        normal = np.abs(want) >= 2.0 ** -126
        assert np.array_equal(got[normal], (ref_codes * 2.0 ** e)[normal]), e   # exact there


def test_signed_zero_and_the_extremes():
    assert _integer_form(np.array([0x00], np.uint8), -3)[0] == 0.0
    neg0 = _integer_form(np.array([0x80], np.uint8), -3)[0]
    assert neg0 == 0.0 and np.signbit(neg0)
    assert _integer_form(np.array([0x7E], np.uint8), 0)[0] == 448.0          # largest code
    assert _integer_form(np.array([0x01], np.uint8), 0)[0] == 2.0 ** -9       # smallest subnormal
    assert _integer_form(np.array([0x01], np.uint8), 20)[0] == 2.0 ** 11
