"""LoRA dropout on the GPU against the oracle ("QLoRA Explained", Step 3:
lora_dropout = 0.05): the Philox4x32-10 keep mask bit for bit, then the
forward and backward of the dropped layer within the layer tolerances."""
import numpy as np
import pytest
import torch

import bit_nf4_quantized_03_b200 as q
from bit_nf4_quantized_03_b200 import synth
from oracle import nf4_oracle as o
from tests.gpu_util import check_close, ensure_built, gpu_quantize

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


class DropLayer:
    def __init__(self, m, n, k, r, p, seed, offset, mode=q.QLORA_SCALE_DQ_FP8, layer=0):
        self.m, self.n, self.k, self.r, self.p = m, n, k, r, p
        W = synth.weight(n, k, layer=layer)
        self.qw = gpu_quantize(W, mode)
        self.Wd = o.dequantize_f64(o.quantize(W.numpy(), mode), (n, k))
        self.X = synth.activations(m, k, layer=layer)
        self.dY = synth.grad_output(m, n, layer=layer)
        self.A, self.B = synth.lora_pair(r, k, n, layer=layer)
        self.Xd, self.dYd, self.Ad, self.Bd = (t.cuda() for t in (self.X, self.dY, self.A, self.B))
        self.mask = torch.zeros(m * k // 8, dtype=torch.uint8, device="cuda")
        self.drop = q.Dropout(p, seed, offset, self.mask)
        self.ws = torch.empty(q.qlora_linear_workspace_bytes_ex(m, n, k, r, self.drop), dtype=torch.uint8,
                              device="cuda")
        self.ref_mask = o.dropout_mask(m, k, p, seed, offset)

    def fwd(self, y_dtype=q.QLORA_DTYPE_FP32):
        dt = torch.float32 if y_dtype == q.QLORA_DTYPE_FP32 else torch.bfloat16
        Y = torch.empty(self.m, self.n, dtype=dt, device="cuda")
        U = torch.empty(self.m, self.r, dtype=torch.float32, device="cuda")
        q.qlora_linear_fwd_ex(self.qw, self.Xd, self.Ad, self.Bd, self.r, 16.0, Y, y_dtype, U, self.drop, self.ws)
        q.qlora_check_device_error()
        return Y, U

    def bwd(self, U=None, flags=0, dX=None, dA=None, dB=None):
        dX = torch.zeros(self.m, self.k, dtype=torch.float32, device="cuda") if dX is None else dX
        dA = torch.zeros(self.r, self.k, dtype=torch.float32, device="cuda") if dA is None else dA
        dB = torch.zeros(self.n, self.r, dtype=torch.float32, device="cuda") if dB is None else dB
        q.qlora_linear_bwd_ex(self.qw, self.Xd, self.dYd, self.Ad, self.Bd, self.r, 16.0, U, dX,
                              q.QLORA_DTYPE_FP32, dA, dB, flags, self.drop, self.ws)
        q.qlora_check_device_error()
        return dX, dA, dB


@pytest.mark.parametrize("m,k,p,seed,offset", [(128, 256, 0.05, 1, 0), (200, 320, 0.3, 77, 5),
                                               (16, 8192, 0.05, 2 ** 40 + 3, 2 ** 33 + 9), (1024, 4096, 0.5, 9, 1)])
def test_mask_bitexact(m, k, p, seed, offset):
    L = DropLayer(m, 256, k, 8, p, seed, offset)
    L.fwd()
    got = L.mask.cpu().numpy()
    want = o.pack_mask_bits(L.ref_mask)
    assert np.array_equal(got, want), f"{int(np.sum(got != want))} mask bytes differ"


@pytest.mark.parametrize("mode", [q.QLORA_SCALE_BF16, q.QLORA_SCALE_DQ_FP8])
@pytest.mark.parametrize("m,n,k,r", [(128, 256, 256, 8), (200, 264, 320, 16), (256, 512, 512, 64),
                                     (130, 512, 384, 128), (16, 1024, 2048, 64), (1, 256, 256, 64)])
def test_dropout_fwd_bwd(m, n, k, r, mode):
    L = DropLayer(m, n, k, r, 0.05, seed=1234, offset=m, mode=mode, layer=1)
    Y, U = L.fwd()
    Y_r, U_r = o.linear_forward_dropout(L.Wd, L.X, L.A, L.B, 16.0, L.ref_mask, L.p)
    check_close(Y.cpu(), Y_r, "Y")
    check_close(U.cpu(), U_r, "U")
    dX, dA, dB = L.bwd(U)
    dX_r, dA_r, dB_r = o.linear_backward_dropout(L.Wd, L.X, L.dY, L.A, L.B, 16.0, L.ref_mask, L.p)
    check_close(dX.cpu(), dX_r, "dX")
    check_close(dA.cpu(), dA_r, "dA")
    check_close(dB.cpu(), dB_r, "dB")


def test_dropout_bwd_recomputes_u_and_accumulates():
    L = DropLayer(192, 384, 512, 32, 0.1, seed=5, offset=3, layer=2)
    L.fwd()
    dX, dA, dB = L.bwd(None)                    # U recomputed from the saved mask
    dX_r, dA_r, dB_r = o.linear_backward_dropout(L.Wd, L.X, L.dY, L.A, L.B, 16.0, L.ref_mask, L.p)
    check_close(dB.cpu(), dB_r, "dB recomputed U")
    dX2, dA2, dB2 = L.bwd(None, flags=q.QLORA_BWD_ACCUMULATE_GRADS | q.QLORA_BWD_ACCUMULATE_DX,
                          dX=dX.clone(), dA=dA.clone(), dB=dB.clone())
    check_close(dX2.cpu(), 2 * dX_r, "2 dX")
    check_close(dA2.cpu(), 2 * dA_r, "2 dA")
    check_close(dB2.cpu(), 2 * dB_r, "2 dB")


def test_dropout_zero_rate_is_the_plain_call():
    L = DropLayer(256, 512, 512, 64, 0.0, seed=1, offset=0, layer=3)
    Y, U = L.fwd(q.QLORA_DTYPE_BF16)
    Y2 = torch.empty_like(Y)
    U2 = torch.empty_like(U)
    q.qlora_linear_fwd(L.qw, L.Xd, L.Ad, L.Bd, L.r, 16.0, Y2, q.QLORA_DTYPE_BF16, U2, L.ws)
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16)) and torch.equal(U, U2)


def test_dropout_deterministic_and_offset_changes_mask():
    L = DropLayer(256, 256, 1024, 16, 0.05, seed=99, offset=0, layer=4)
    Y1, _ = L.fwd()
    m1 = L.mask.clone()
    Y2, _ = L.fwd()
    assert torch.equal(Y1, Y2) and torch.equal(m1, L.mask)
    L.drop.offset = 1
    L.fwd()
    assert not torch.equal(m1, L.mask)
    assert np.array_equal(L.mask.cpu().numpy(), o.pack_mask_bits(o.dropout_mask(256, 1024, 0.05, 99, 1)))


@pytest.mark.slow
def test_dropout_65b_q_proj_8192_tokens_sampled():
    m = n = k = 8192
    L = DropLayer(m, n, k, 64, 0.05, seed=2024, offset=11, layer=5)
    Y, U = L.fwd(q.QLORA_DTYPE_BF16)
    assert np.array_equal(L.mask.cpu().numpy(), o.pack_mask_bits(L.ref_mask))
    rows = synth.sample_rows(m, 64).numpy()
    Y_r, U_r = o.linear_forward_dropout(L.Wd, L.X, L.A, L.B, 16.0, L.ref_mask, L.p, rows=rows)
    check_close(Y.float().cpu().numpy()[rows], Y_r, "Y", bf16_out=True)
    check_close(U.cpu().numpy()[rows], U_r, "U")
    dX = torch.empty(m, k, dtype=torch.bfloat16, device="cuda")
    dA = torch.empty(64, k, dtype=torch.float32, device="cuda")
    dB = torch.empty(n, 64, dtype=torch.float32, device="cuda")
    q.qlora_linear_bwd_ex(L.qw, L.Xd, L.dYd, L.Ad, L.Bd, 64, 16.0, U, dX, q.QLORA_DTYPE_BF16, dA, dB, 0, L.drop, L.ws)
    q.qlora_check_device_error()
    dX_r, dA_r, dB_r = o.linear_backward_dropout(L.Wd, L.X, L.dY, L.A, L.B, 16.0, L.ref_mask, L.p, dx_rows=rows)
    check_close(dX.float().cpu().numpy()[rows], dX_r, "dX", bf16_out=True)
    check_close(dA.cpu(), dA_r, "dA")
    check_close(dB.cpu(), dB_r, "dB")
