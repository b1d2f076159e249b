"""The allocation-free quantize entry point against the allocating one.

Some callers cannot give the library a device workspace: a plugin that its
host framework hands only input and output pointers (the framework owns all
device memory), or a latency-critical path that must not call cudaMalloc.
qlora_nf4_quantize_noalloc serves them from a fixed scratch array inside the
library. These tests call it through the C ABI and require the same bytes as
qlora_nf4_quantize, on two calls in a row (the second call reuses the scratch
the first one left behind).

The file name sorts last, so pytest collects it after every other test file: a
run that stops at the first failure (-x) has then already run the rest of the
suite when one of these fails. The tests themselves depend on no order; they
pass alone in a fresh process as well.
"""
import ctypes

import numpy as np
import pytest
import torch

import bit_nf4_quantized_03_b200 as q
from bit_nf4_quantized_03_b200 import synth
from tests.gpu_util import assert_weight_bitexact, ensure_built, gpu_weight_dict

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mode", [q.QLORA_SCALE_DQ_FP8, q.QLORA_SCALE_BF16])
def test_noalloc_quantize_matches_allocating_entry_point(mode):
    ensure_built()
    for shape in ((4096, 4096), (300, 257), (8192, 1024)):
        W = synth.weight(*shape, outlier_frac=0.001).cuda()
        ref = q.QuantizedWeight(*shape, mode)
        q.qlora_nf4_quantize(W, ref)
        torch.cuda.synchronize()
        want = gpu_weight_dict(ref)
        for _ in range(2):
            got = q.QuantizedWeight(*shape, mode)
            q.qlora_nf4_quantize_noalloc(W, got)
            q.qlora_check_device_error()
            assert_weight_bitexact(gpu_weight_dict(got), want)


def test_noalloc_rejects_requests_beyond_the_scratch_limit():
    ensure_built()
    L = q.lib()
    buf = torch.zeros(1 << 12, dtype=torch.uint8, device="cuda")   # never touched: rejected on the host
    p = buf.data_ptr()
    w = q.NF4Weight(16384, 16384 + 64, 64, 256, q.QLORA_SCALE_DQ_FP8, 0, p, None, p, p, p)
    assert L.qlora_nf4_quantize_noalloc(p, ctypes.byref(w), None) == 2
    torch.cuda.synchronize()
    assert torch.count_nonzero(buf).item() == 0
