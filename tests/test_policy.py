"""The per-layer code-width policy (host logic only)."""
import pytest

from bit_error_compensated_echo_b200.policy import LayerPolicy


def test_llama_first_half_promoted():
    pol = LayerPolicy(32, 2, 0.5)
    s = pol.schedule()
    assert len(s) == 64 and s[:32] == [8] * 32 and s[32:] == [4] * 32
    assert pol.bits_for_layer(15) == 8 and pol.bits_for_layer(16) == 4
    assert pol.bits_for_site(64) == 8           # the next step starts over


def test_fractions_and_errors():
    assert LayerPolicy(28, 2, 0.0).schedule() == [4] * 56
    assert LayerPolicy(28, 2, 1.0).schedule() == [8] * 56
    assert LayerPolicy(3, 1, 0.5).schedule() == [8, 8, 4]   # round(1.5) = 2
    with pytest.raises(ValueError):
        LayerPolicy(0)
    with pytest.raises(ValueError):
        LayerPolicy(4, 2, 1.5)
    with pytest.raises(ValueError):
        LayerPolicy(4, 2, 0.5, high=6)
    with pytest.raises(IndexError):
        LayerPolicy(4).bits_for_layer(4)
