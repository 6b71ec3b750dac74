"""The oracle's sparse attention against closed forms and the dense-attention
special case (torch's scaled_dot_product_attention in float64)."""
import pytest

from tests import attn_pins


@pytest.mark.parametrize("pin", attn_pins.ALL, ids=lambda f: f.__name__)
def test_attention_pin(pin):
    assert pin() is None
