"""Failure detection on the GPU without a fault: every wait in the library's
kernels is bounded; when one gives up it records a device error word that the
host reads. Here a kernel waits on a barrier nobody arrives on (a short
limit), the error surfaces as QLORA_ERR_DEVICE, and the context keeps
working afterwards."""
import pytest
import torch

import bit_nf4_quantized_03_b200 as q
from bit_nf4_quantized_03_b200 import synth
from tests.gpu_util import ensure_built

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_error_and_context_survives():
    ensure_built()
    q.qlora_check_device_error()                       # clean start
    q.qlora_selftest_wait_timeout(100)
    with pytest.raises(q.QloraError) as e:
        q.qlora_check_device_error()
    assert e.value.status == 5
    q.qlora_check_device_error()                       # the word was cleared
    W = synth.weight(256, 256)
    qw = q.QuantizedWeight(256, 256, q.QLORA_SCALE_DQ_FP8)
    q.qlora_nf4_quantize(W.cuda(), qw)                 # the context still works
    q.qlora_check_device_error()
    assert torch.count_nonzero(qw.codes).item() > 0


def test_selftest_rejects_bad_limits():
    ensure_built()
    assert q.lib().qlora_selftest_wait_timeout(0, None) == 1
    assert q.lib().qlora_selftest_wait_timeout(5000, None) == 1
