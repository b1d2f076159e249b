"""Adapter merge on the GPU against the oracle:
W_merged = W' + (alpha/r) B A ("QLoRA: Quantized Low-Rank Adaptation",
Price 2: deployment friction; "QLoRA Explained", Step 5).

Bound per element, derived from the arithmetic the kernel performs: the r
products of bf16 values are exact in fp32, their tensor-core sum carries at
most r roundings (taken with a factor 2 for the accumulator's alignment),
the fused multiply-add onto w' rounds once, and the BF16 output rounds once
more (half a BF16 ulp of the exact value).
"""
import numpy as np
import pytest
import torch

import bit_nf4_quantized_03_b200 as q
from bit_nf4_quantized_03_b200 import synth
from oracle import nf4_oracle as o
from tests.gpu_util import ensure_built, gpu_quantize, gpu_weight_dict, assert_weight_bitexact

pytestmark = pytest.mark.gpu
U32 = 2.0 ** -24


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


def _half_ulp_bf16(x):
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126)))
    return 0.5 * np.exp2(e - 7)


def check_merge(got, Wd, A, B, alpha, bf16_out):
    r = A.shape[0]
    s = alpha / r
    A64, B64 = o._f64(A), o._f64(B)
    exact = o.lora_merge(Wd, A, B, alpha)
    prod_abs = s * (np.abs(B64) @ np.abs(A64))
    allow = 2 * r * U32 * prod_abs + 2 * U32 * np.abs(exact)
    if bf16_out:
        allow = allow + _half_ulp_bf16(exact)
    got = o._f64(got)
    assert got.shape == exact.shape
    assert np.all(np.isfinite(got))
    bad = np.abs(got - exact) > allow
    assert not bad.any(), f"{int(bad.sum())} elements over the bound; worst {float(np.max(np.abs(got - exact) / allow)):.3f}x"
    if bf16_out:
        rn = o.bf16_to_f32(o.bf16_bits(exact.astype(np.float32))).astype(np.float64)
        # exact.astype(float32) may itself round; compare only where that step is exact enough to decide
        frac = float(np.mean(got != rn))
        assert frac < 1e-3, frac


def _case(n, k, r, mode, layer=0, zero_b=False):
    W = synth.weight(n, k, layer=layer)
    qw = gpu_quantize(W, mode)
    Wd = o.dequantize_f64(o.quantize(W.numpy(), mode), (n, k))
    A, B = synth.lora_pair(r, k, n, layer=layer)
    if zero_b:
        B = torch.zeros_like(B)
    return qw, Wd, A, B


def _merge(qw, A, B, r, alpha, dtype):
    dt = torch.float32 if dtype == q.QLORA_DTYPE_FP32 else torch.bfloat16
    out = torch.full((qw.n, qw.k), float("nan"), dtype=dt, device="cuda")
    q.qlora_lora_merge(qw, A.cuda(), B.cuda(), r, 16.0, out, dtype)
    q.qlora_check_device_error()
    return out


@pytest.mark.parametrize("mode", [q.QLORA_SCALE_BF16, q.QLORA_SCALE_DQ_FP8])
@pytest.mark.parametrize("dtype", [q.QLORA_DTYPE_BF16, q.QLORA_DTYPE_FP32])
@pytest.mark.parametrize("n,k,r", [(128, 256, 8), (300, 576, 16), (1000, 1088, 128), (520, 4096, 32), (4096, 4096, 64)])
def test_merge_matches_oracle(n, k, r, mode, dtype):
    qw, Wd, A, B = _case(n, k, r, mode, layer=1)
    out = _merge(qw, A, B, r, 16.0, dtype)
    check_merge(out.float().cpu(), Wd, A, B, 16.0, dtype == q.QLORA_DTYPE_BF16)


@pytest.mark.parametrize("mode", [q.QLORA_SCALE_BF16, q.QLORA_SCALE_DQ_FP8])
def test_merge_with_zero_adapter_is_the_dequantized_weight(mode):
    # a freshly initialised adapter (B = 0) merges to exactly the dequantized BF16 weight
    n, k, r = 384, 1024, 64
    qw, _, A, B = _case(n, k, r, mode, layer=2, zero_b=True)
    out = _merge(qw, A, B, r, 16.0, q.QLORA_DTYPE_BF16)
    deq = torch.empty(n, k, dtype=torch.bfloat16, device="cuda")
    q.qlora_nf4_dequantize(qw, deq)
    ref = o.dequantize(o.quantize(synth.weight(n, k, layer=2).numpy(), mode))     # bf16 bit patterns
    got = out.view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1)
    assert np.array_equal(got, ref[: n * k])
    assert torch.equal(out.view(torch.int16), deq.view(torch.int16))


def test_merge_then_quantize_again():
    # fine-tune -> merge -> quantize again for deployment: the fp32 merge feeds qlora_nf4_quantize,
    # whose output must be bit-exact against the oracle's quantization of the same fp32 values
    n, k, r = 512, 2048, 64
    qw, Wd, A, B = _case(n, k, r, q.QLORA_SCALE_DQ_FP8, layer=3)
    merged = _merge(qw, A, B, r, 16.0, q.QLORA_DTYPE_FP32)
    check_merge(merged.cpu(), Wd, A, B, 16.0, False)
    q2 = q.QuantizedWeight(n, k, q.QLORA_SCALE_DQ_FP8)
    q.qlora_nf4_quantize(merged, q2)
    q.qlora_check_device_error()
    ref = o.quantize(merged.cpu().numpy(), o.MODE_DQ_FP8)
    assert_weight_bitexact(gpu_weight_dict(q2), ref)


@pytest.mark.slow
def test_merge_65b_q_proj_full():
    n = k = 8192
    r = 64
    qw, Wd, A, B = _case(n, k, r, q.QLORA_SCALE_DQ_FP8, layer=4)
    out = _merge(qw, A, B, r, 16.0, q.QLORA_DTYPE_BF16)
    check_merge(out.float().cpu(), Wd, A, B, 16.0, True)


def test_merge_repeatable():
    n, k, r = 640, 1536, 64
    qw, _, A, B = _case(n, k, r, q.QLORA_SCALE_DQ_FP8, layer=5)
    a = _merge(qw, A, B, r, 16.0, q.QLORA_DTYPE_BF16)
    b = _merge(qw, A, B, r, 16.0, q.QLORA_DTYPE_BF16)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
