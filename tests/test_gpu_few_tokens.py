"""GPU parity of the forward pass at 1 to 16 tokens, the regime where the layer
streams its 4-bit weight once (the single-CTA fused GEMM with its reduction
split over the SMs, and U = X A^T on CUDA cores), against the fp64 oracle.
The shapes cover its edges: K not a multiple of 256, n % 16 == 8, K = 64 (one
block per row), reductions split several ways with a short last split, token
counts from 1 to 16, both scale modes, fp32 and bf16 outputs, U saved or not,
outlier blocks and alpha != 16. Same bounds as the other layer tests."""
import numpy as np
import pytest
import torch

import bit_nf4_quantized_03_b200 as q
from bit_nf4_quantized_03_b200 import synth
from oracle import nf4_oracle as o
from tests.gpu_util import Layer, check_close, ensure_built

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


def _fwd_check(L: Layer, y_dtype=q.QLORA_DTYPE_FP32, save_u=True):
    Y, U = L.fwd(y_dtype, save_u=save_u)
    Y_ref, U_ref = o.linear_forward(L.oracle_weight(), L.X, L.A, L.B, L.alpha)
    check_close(Y.float().cpu(), Y_ref, "Y", bf16_out=(y_dtype == q.QLORA_DTYPE_BF16))
    if save_u:
        check_close(U.cpu(), U_ref, "U")
    return Y


@pytest.mark.parametrize("m,n,k,r", [
    (16, 264, 832, 32),      # K = 13 blocks (not a multiple of 256), n % 16 == 8
    (5, 512, 4608, 16),      # 72 K blocks split over the SMs
    (16, 2048, 22016, 64),   # 344 K blocks: the 65B down_proj reduction length
    (16, 8, 64, 8),          # one 8-row feature group, one K block
    (1, 1024, 1024, 128),    # one token, rank 128
    (12, 776, 1344, 64),     # 776 rows (not a multiple of 128), 21 K blocks
    (16, 4096, 4096, 64),    # 7B q_proj shape at 16 tokens
])
def test_few_token_shapes(m, n, k, r):
    _fwd_check(Layer(m, n, k, r))


@pytest.mark.parametrize("m", [3, 16])
def test_few_tokens_bf16_scales_bf16_output_no_u(m):
    L = Layer(m, 1032, 1536, 32, mode=q.QLORA_SCALE_BF16, layer=2)
    _fwd_check(L, y_dtype=q.QLORA_DTYPE_BF16, save_u=False)


def test_few_tokens_with_outliers_and_alpha():
    # outlier blocks give large block scales; alpha != 16 checks the low-rank scale
    L = Layer(16, 640, 2304, 16, alpha=32.0, outlier_frac=0.01, layer=3)
    _fwd_check(L)


def test_few_tokens_deterministic_and_backward_consistent():
    # the fixed-order reductions make repeated calls bit-identical; the backward pass
    # then consumes the forward's saved U
    L = Layer(16, 1024, 3072, 64, layer=4)
    Y1 = _fwd_check(L)
    Y2, U = L.fwd()
    assert torch.equal(Y1, Y2)
    dX, dA, dB = L.bwd(U)
    dX_ref, dA_ref, dB_ref = o.linear_backward(L.oracle_weight(), L.X, L.dY, L.A, L.B, L.alpha)
    check_close(dX.cpu(), dX_ref, "dX")
    check_close(dA.cpu(), dA_ref, "dA")
    check_close(dB.cpu(), dB_ref, "dB")


def test_few_tokens_match_dequantized_weight_product():
    # same result as multiplying by the library's own dequantized BF16 weight in fp64
    # (the GEMM's in-kernel expansion against the bit-exact dequantize kernel)
    L = Layer(16, 512, 1024, 8, layer=5)
    Wq = torch.empty(L.n, L.k, dtype=torch.bfloat16, device="cuda")
    q.qlora_nf4_dequantize(L.qw, Wq)
    Wd = Wq.float().double().cpu().numpy()
    assert np.array_equal(Wd, L.oracle_weight())          # dequantize is bit-exact
    Y, _ = L.fwd()
    Y_ref, _ = o.linear_forward(Wd, L.X, L.A, L.B, L.alpha)
    check_close(Y.cpu(), Y_ref, "Y")
