"""Host-side checks of the MXFP8 grouped-GEMM module's options (no GPU).

backward_override and wgrad_with_hp (ao "[moe training] Add
backward_override to the MXFP8 grouped GEMM", Design notes and Known
follow-ups): the page leaves the interaction of the two open. Reading taken:
"high_precision" subsumes wgrad_with_hp (the flag changes nothing), and the
pair ("dequantized", wgrad_with_hp) is rejected, since the two would take dw
from different operands (the bf16 activations against the forward's codes).
"""
import pytest


def test_override_names_and_wgrad_with_hp_combinations():
    from mxfp8_block_scaled_cast_b200 import mx
    with pytest.raises(ValueError):
        mx.MXFP8GroupedMM(backward_override="fp32")
    with pytest.raises(ValueError):
        mx.MXFP8GroupedMM(backward_override="dequantized", wgrad_with_hp=True)
    assert mx.MXFP8GroupedMM(wgrad_with_hp=True).wgrad_with_hp
    assert mx.MXFP8GroupedMM(backward_override="quantized", wgrad_with_hp=True).wgrad_with_hp
    hp = mx.MXFP8GroupedMM(backward_override="high_precision", wgrad_with_hp=True)
    assert hp.backward_override == "high_precision" and not hp.wgrad_with_hp
    assert not mx.MXFP8GroupedMM().wgrad_with_hp


def test_backward_before_forward_is_an_error():
    import torch
    from mxfp8_block_scaled_cast_b200 import mx
    op = mx.MXFP8GroupedMM(wgrad_with_hp=True)
    with pytest.raises(RuntimeError):
        op.backward(torch.zeros(4, 4, dtype=torch.bfloat16))


def test_saved_state_round_trips_through_save_for_backward_layout():
    """The grouped layer's autograd entry hands the layer's saved state to
    save_for_backward as a flat list of tensors plus a layout; the layout puts
    every tensor (repeated ones too), tuple and plain value back in place, for
    the shape of each backward arm's state."""
    import torch
    from mxfp8_block_scaled_cast_b200.mx import _flatten_saved, _unflatten_saved
    t = [torch.zeros(i + 1) for i in range(5)]
    states = [
        ((t[0], t[1], 256, 384), t[2], t[3], t[4], 1536),      # MXFP8: x's codes, scales, M, K; w; offs; m_cap
        (t[0], t[1], t[2]),                                    # high_precision: x, w, offs
        (t[0], t[1], t[2], t[3], t[4], 1000, 1536),            # dequantized
        (t[0], t[2], t[3], t[4], None),                        # repeated slots and a None
    ]
    for state in states:
        flat = []
        layout = _flatten_saved(state, flat)
        assert all(isinstance(x, torch.Tensor) for x in flat)
        back = _unflatten_saved(layout, tuple(flat))

        def same(a, b):
            if isinstance(a, torch.Tensor):
                return a is b
            if isinstance(a, tuple):
                return isinstance(b, tuple) and len(a) == len(b) and all(same(x, y) for x, y in zip(a, b))
            return a == b
        assert same(state, back)
