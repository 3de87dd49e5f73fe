"""The O tolerance of the GPU parity tests, on CPU: max-abs 2e-2 and rel-RMS
5e-3 against the fp64 oracle, with half a bf16 ulp more (and a warning) only
where |O_ref| >= 8."""
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
    with pytest.raises(AssertionError, match="max-abs"):
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
    with pytest.raises(AssertionError, match="large-"):
        check_o(got, ref)
