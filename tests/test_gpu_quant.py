"""GPU parity of quantize / double-quant / dequantize: bit-exact against the
oracle on the same seeded inputs (codes, bf16 scales, E4M3 scales, the fp32
second-level scales and mean, and every dequantized bf16 weight)."""
import numpy as np
import pytest
import torch

import bit_nf4_quantized_03_b200 as q
from bit_nf4_quantized_03_b200 import synth
from oracle import nf4_oracle as o
from tests.gpu_util import assert_weight_bitexact, ensure_built, gpu_quantize, gpu_weight_dict, u16, _first_diff

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


def _roundtrip(W: torch.Tensor, mode: int):
    ref = o.quantize(W.numpy(), mode)
    qw = gpu_quantize(W, mode)
    assert_weight_bitexact(gpu_weight_dict(qw), ref)
    out = torch.empty(W.shape, dtype=torch.bfloat16, device="cuda")
    q.qlora_nf4_dequantize(qw, out)
    q.qlora_check_device_error()
    got = u16(out).reshape(-1)
    want = o.dequantize(ref)
    assert np.array_equal(got, want), _first_diff(got, want)
    return qw


@pytest.mark.parametrize("mode", [q.QLORA_SCALE_BF16, q.QLORA_SCALE_DQ_FP8])
@pytest.mark.parametrize("shape", [(256, 256), (37, 45), (1, 1), (1, 64), (3, 1000), (64, 4160), (300, 257)])
def test_quantize_dequantize_bitexact_small(shape, mode):
    W = synth.weight(*shape, outlier_frac=0.01)
    _roundtrip(W, mode)


@pytest.mark.parametrize("mode", [q.QLORA_SCALE_BF16, q.QLORA_SCALE_DQ_FP8])
def test_quantize_roundtrip_4096_with_outliers(mode):
    # 4096 x 4096 fp32 ~ N(0, 0.02), 0.1% outliers at 10 sigma
    W = synth.weight(4096, 4096, outlier_frac=0.001)
    _roundtrip(W, mode)


@pytest.mark.parametrize("mode", [q.QLORA_SCALE_BF16, q.QLORA_SCALE_DQ_FP8])
def test_edge_blocks(mode):
    rng = np.random.default_rng(21)
    W = rng.normal(0, 0.02, (16, 1024)).astype(np.float32)
    W[0, :64] = 0.0                                  # all-zero block
    W[1, :64] = 1e-40                                # subnormal absmax
    W[1, 64:128] = -3e-39
    mid = o.nf4_midpoints()
    W[2, :64] = np.resize(mid, 64)                   # values exactly on the thresholds ...
    W[2, 0] = 1.0                                    # ... of a block whose absmax is 1 (x == w)
    W[3, 64:128] = -np.resize(mid, 64)
    W[3, 64] = -1.0
    W[4, :] = 0.05                                   # constant row
    W[5, :64] = np.resize(o.nf4_levels(), 64) * np.float32(0.25)   # on the grid
    _roundtrip(torch.from_numpy(W), mode)


def test_double_quant_constant_absmax():
    W = np.tile(np.float32([0.5] + [0.25] * 63), (8, 64))
    qw = _roundtrip(torch.from_numpy(W.reshape(8, -1)), q.QLORA_SCALE_DQ_FP8)
    assert float(qw.dq_mean.cpu()[0]) == 0.5
    assert torch.all(qw.scale_fp8 == 0)


def test_codes_identical_across_modes():
    W = synth.weight(512, 512, outlier_frac=0.001)
    a = gpu_quantize(W, q.QLORA_SCALE_BF16)
    b = gpu_quantize(W, q.QLORA_SCALE_DQ_FP8)
    assert torch.equal(a.codes, b.codes)


def test_quantize_deterministic():
    W = synth.weight(1024, 2048, outlier_frac=0.001)
    a = gpu_quantize(W, q.QLORA_SCALE_DQ_FP8)
    b = gpu_quantize(W, q.QLORA_SCALE_DQ_FP8)
    for x, y in ((a.codes, b.codes), (a.scale_fp8, b.scale_fp8), (a.dq_scale, b.dq_scale), (a.dq_mean, b.dq_mean)):
        assert torch.equal(x, y)


@pytest.mark.slow
def test_double_quant_65b_gate_shape_full():
    # 22016 x 8192: 2.8M blocks -> three passes of the fixed-order mean reduction
    n, k = 22016, 8192
    W = synth.weight(n, k)
    qw = gpu_quantize(W, q.QLORA_SCALE_DQ_FP8)
    w_np = W.numpy().reshape(-1)
    absmax = o.block_absmax(w_np)
    qv, s2, mu = o.double_quantize(absmax)
    assert np.float32(qw.dq_mean.cpu().numpy()[0]).view(np.uint32) == np.float32(mu).view(np.uint32)
    assert np.array_equal(qw.dq_scale.cpu().numpy().view(np.uint32), s2.view(np.uint32))
    assert np.array_equal(qw.scale_fp8.cpu().numpy(), qv)
    # codes: sampled rows (each row is 128 whole blocks)
    rows = synth.sample_rows(n, 64).numpy()
    codes = qw.codes.cpu().numpy().reshape(n, k // 2)
    for r_ in rows:
        want = o.pack_nibbles(o.nf4_codes(W[r_].numpy()))
        assert np.array_equal(codes[r_], want)
