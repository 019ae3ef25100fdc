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
