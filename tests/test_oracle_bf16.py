"""Pins for the oracle's bf16 rounding (round to nearest, ties to even)."""
import numpy as np
import torch

from oracle import hier_local_attn as O


def torch_bf16_bits(x32: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def test_every_bf16_value_round_trips():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    x = O.bf16_to_f64(bits)
    back = O.f64_to_bf16(x)
    finite = ~np.isnan(x)
    np.testing.assert_array_equal(back[finite], bits[finite])
    assert np.all((back[~finite] & 0x7FFF) == 0x7FC0)


def test_matches_library_rounding_on_fp32_values():
    """For fp32 inputs fp64->bf16 and torch's fp32->bf16 (RNE) must agree."""
    rng = np.random.default_rng(1)
    u = rng.integers(0, 1 << 32, size=2_000_000, dtype=np.uint64).astype(np.uint32)
    x32 = u.view(np.float32)
    x32 = x32[np.isfinite(x32)]
    np.testing.assert_array_equal(O.f64_to_bf16(x32.astype(np.float64)), torch_bf16_bits(x32))


def test_ties_go_to_even_and_subnormals():
    bits = np.arange(0, 0x7F7F, dtype=np.uint16)  # positive finite, excluding the max
    lo = O.bf16_to_f64(bits)
    hi = O.bf16_to_f64(bits + 1)
    mid = (lo + hi) / 2  # exact in fp64
    r = O.f64_to_bf16(mid)
    even = np.where(bits % 2 == 0, bits, bits + 1)
    np.testing.assert_array_equal(r, even)
    np.testing.assert_array_equal(O.f64_to_bf16(-mid), even | 0x8000)


def test_single_rounding_from_fp64():
    """A value a hair above a bf16 midpoint rounds up even when rounding it
    to fp32 first would have produced the exact midpoint (double rounding)."""
    bits = np.arange(0x3F80, 0x3FFF, 2, dtype=np.uint16)  # even patterns in [1, 2)
    lo = O.bf16_to_f64(bits)
    hi = O.bf16_to_f64(bits + 1)
    mid = (lo + hi) / 2
    above = mid + 2.0 ** -40
    below = mid - 2.0 ** -40
    np.testing.assert_array_equal(O.f64_to_bf16(above), bits + 1)
    np.testing.assert_array_equal(O.f64_to_bf16(below), bits)
    # fp32 rounding of `above` lands on the midpoint, where RNE picks `bits`.
    np.testing.assert_array_equal(torch_bf16_bits(above.astype(np.float32)), bits)


def test_overflow_and_zero():
    big = O.bf16_to_f64(np.array([0x7F7F], np.uint16))[0]  # largest finite bf16
    ulp = 2.0 ** (127 - 7)
    assert O.f64_to_bf16(np.array([big + ulp / 2]))[0] == 0x7F80  # tie -> even = inf
    assert O.f64_to_bf16(np.array([big + ulp / 4]))[0] == 0x7F7F
    assert O.f64_to_bf16(np.array([1e300]))[0] == 0x7F80
    assert O.f64_to_bf16(np.array([0.0]))[0] == 0
    assert O.f64_to_bf16(np.array([-0.0]))[0] == 0x8000
    assert O.f64_to_bf16(np.array([2.0 ** -134]))[0] == 0  # half the smallest subnormal: tie -> 0
    assert O.f64_to_bf16(np.array([2.0 ** -134 * 1.5]))[0] == 1


def test_half_ulp_bound_of_the_parity_checks():
    """parity.half_ulp_bf16 is the most that rounding to bf16 moves a value:
    torch's (single) rounding of 200k random fp32 values from many binades
    stays within it, and values exactly halfway between two bf16 neighbours
    reach it."""
    from parity import half_ulp_bf16
    rng = np.random.default_rng(3)
    x32 = (rng.standard_normal(200_000) * np.exp2(rng.integers(-20, 20, 200_000)))
    x32 = x32.astype(np.float32)
    x = x32.astype(np.float64)
    r = torch.from_numpy(x32).to(torch.bfloat16).double().numpy()
    assert (np.abs(r - x) <= half_ulp_bf16(x)).all()
    # midpoints between consecutive bf16 values in [1, 2): ulp 2^-7
    k = np.arange(128)
    mid = 1.0 + (k + 0.5) * 2.0 ** -7
    rm = torch.from_numpy(mid.astype(np.float32)).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(np.abs(rm - mid), half_ulp_bf16(mid))
