"""Failure detection on the GPU without faulting it: a bounded wait that nothing
satisfies gives up after its limit, records SAGE_ERR_TIMEOUT in the device status word,
and the context stays usable for the next call."""
import pytest
import torch

import quantized_attention_03_b200 as sage
from quantized_attention_03_b200 import inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    assert sage.sage_get_device_status() == sage.SAGE_OK
    sage.sage_debug_wait_timeout(20_000_000)            # 20 ms, nothing ever arrives
    assert sage.sage_get_device_status() == sage.SAGE_ERR_TIMEOUT
    assert sage.sage_get_device_status() == sage.SAGE_OK  # read clears the word
    w = inputs.Workload("after-timeout", 5, 1, 2, 300, 64, False, 1.0)
    q, k, v = (t.cuda() for t in inputs.make_dense(w))
    out = sage.sageattn(q, k, v)
    assert sage.sage_get_device_status() == sage.SAGE_OK
    assert torch.isfinite(out.float()).all()


def test_timeout_argument_is_checked():
    with pytest.raises(sage.SageError):
        sage.sage_debug_wait_timeout(5_000_000_000)     # over the 1 s cap
