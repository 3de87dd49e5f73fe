"""The CPU oracle against its pins (no GPU)."""
import pytest

from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_pin(orc, pin):
    pin(orc)


def test_oracle_rejects_mismatched_inputs(orc):
    # V and the bias must be bf16 bit patterns of the right shape: the C code
    # reads them by the sizes of Q, so a short or float array is refused.
    import numpy as np

    q = np.zeros((1, 2, 5, 8), dtype=np.float32)
    v = np.zeros((1, 2, 5, 8), dtype=np.uint16)
    bias = np.zeros((2, 5, 5), dtype=np.uint16)
    orc.forward(q, q, bias, v, 1.0)
    with pytest.raises(TypeError, match="bf16 bit patterns"):
        orc.forward(q, q, bias, v.astype(np.float32), 1.0)
    with pytest.raises(ValueError, match="bias has shape"):
        orc.forward(q, q, bias[:1], v, 1.0)
    with pytest.raises(ValueError, match="v has shape"):
        orc.forward_rows(q, q, None, v[:, :1], 1.0, [0, 1])
    with pytest.raises(ValueError, match="differ"):
        orc.scores_rows(q, q[:, :1], [0])
    with pytest.raises(TypeError, match="bf16 bit patterns"):
        orc.probs_rows(q, q, bias.astype(np.float32), 1.0, [0])
