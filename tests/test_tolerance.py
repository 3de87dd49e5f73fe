"""The O tolerance of the GPU parity tests, on CPU: max-abs 2e-2 and rel-RMS
5e-3 against the fp64 oracle, with half a bf16 ulp more (and a warning) only
where |O_ref| >= 8, and the bf16-P spread bound (with a warning) only where
a test passes the oracle's spread and that bound is the larger."""
import numpy as np
import pytest

from parity import bf16_half_ulp, check_o


def test_bf16_half_ulp():
    assert bf16_half_ulp(np.array([1.0]))[0] == 2.0 ** -8
    assert bf16_half_ulp(np.array([8.0]))[0] == 2.0 ** -5
    assert bf16_half_ulp(np.array([-9.5]))[0] == 2.0 ** -5
    assert bf16_half_ulp(np.array([0.75]))[0] == 2.0 ** -9


def test_check_o_bars():
    rng = np.random.default_rng(0)
    ref = rng.standard_normal(4096)
    assert not check_o(ref + 1e-3, ref)["half_ulp_fallback"]
    with pytest.raises(AssertionError, match="beyond their bound"):
        check_o(ref + np.where(np.arange(4096) == 7, 0.021, 0.0), ref)
    ref3 = np.clip(ref, -3.0, 3.0)
    with pytest.raises(AssertionError, match="rel-RMS"):
        check_o(ref3 * 1.006, ref3)  # every element within 0.018, rel-RMS 6e-3


def test_check_o_large_values_fallback_is_flagged():
    ref = np.concatenate([np.full(100, 0.5), [9.0, -12.0]])
    got = ref.copy()
    got[-2:] += [0.03, -0.04]  # within 2e-2 + 2^-5 = 0.05125, beyond 2e-2
    with pytest.warns(UserWarning, match="half a bf16 ulp"):
        assert check_o(got, ref)["half_ulp_fallback"]
    got[-1] = ref[-1] - 0.06
    with pytest.raises(AssertionError, match="beyond their bound"):
        check_o(got, ref)


def test_check_o_spread_bound_is_flagged():
    # |O| in [4, 8): half an ulp is 2^-6; with spread E = 6 the bf16-P bound
    # is 2^-8 * 6 + 2^-6 + 1e-3 = 0.0402 (the outlier channels of ViT-L)
    ref = np.concatenate([np.full(1000, 0.3), [5.0]])
    spread = np.concatenate([np.full(1000, 0.5), [6.0]])
    got = ref.copy()
    got[-1] += 0.03
    with pytest.raises(AssertionError, match="beyond their bound"):
        check_o(got, ref)  # without the spread: the plain 2e-2 bar
    with pytest.warns(UserWarning, match="spread bound"):
        assert check_o(got, ref, spread=spread)["half_ulp_fallback"]
    got[-1] = ref[-1] + 0.041
    with pytest.raises(AssertionError, match="beyond their bound"):
        check_o(got, ref, spread=spread)
    # small spreads never loosen the 2e-2 bar
    got = ref.copy()
    got[3] += 0.021
    with pytest.raises(AssertionError, match="beyond their bound"):
        check_o(got, ref, spread=spread)
