"""Failure detection without a GPU fault: a pipeline wait that nothing will
complete gives up after its time limit, the host reads MX_ERR_TIMEOUT from
the sticky flag, and the context keeps working."""
import numpy as np
import pytest
import torch

from oracle import mx_oracle as O
from mxfp8_block_scaled_cast_b200 import synthetic as S

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_the_context_survives():
    from mxfp8_block_scaled_cast_b200 import mx
    mx.lib()
    mx.mx_device_error()                               # start clean
    status = mx.lib().mx_selftest_wait_timeout(mx._stream())
    assert status == 0
    with pytest.raises(mx.MXError) as e:
        mx.mx_device_error()
    assert e.value.status == 5                         # MX_ERR_TIMEOUT
    mx.mx_device_error()                               # the flag was cleared
    xb = S.normal_bf16((64, 64), seed=3)
    q, s = mx.cast_dim0(xb.cuda())                     # the context still works
    eq, _ = O.cast_dim0(S.bf16_bits(xb))
    assert np.array_equal(q.cpu().numpy(), eq)
    mx.mx_device_error()
