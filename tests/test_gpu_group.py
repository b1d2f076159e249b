"""Grouped backward of layers that share an input (q/k/v of attention, gate/up of
an MLP) against the fp64 oracle: dX is the sum of every layer's dX term, formed by
one weight GEMM over the layers' reductions in turn (CTA-pair kernel, above 128
tokens) or by the layers one after the other (at most 128 tokens); each layer's
dA, dB are its own. Same bounds as the single-layer tests (relative Frobenius
<= 2e-3, max |error| <= 1e-2 x RMS, bf16 outputs widened by half an ulp)."""
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


class Member:
    """One layer of a group: weight [n, k], adapters, dY, and its oracle weight."""

    def __init__(self, m, n, k, r, mode, layer, with_oracle=True):
        self.n = n
        W = synth.weight(n, k, layer=layer)
        self.qw = gpu_quantize(W, mode)
        self.Wd = o.dequantize_f64(o.quantize(W.numpy(), mode), (n, k)) if with_oracle else None
        self.A, self.B = synth.lora_pair(r, k, n, layer=layer)
        self.dY = synth.grad_output(m, n, layer=layer)
        self.Ad, self.Bd, self.dYd = self.A.cuda(), self.B.cuda(), self.dY.cuda()


def _run_group(mem, X, r, alpha, dx_dtype, flags=0, dX=None, grads=None, u_saved=True, rows=None):
    m, k = X.shape
    Xd = X.cuda()
    dt = torch.float32 if dx_dtype == q.QLORA_DTYPE_FP32 else torch.bfloat16
    if dX is None:
        dX = torch.empty(m, k, dtype=dt, device="cuda")
    if grads is None:
        grads = [(torch.empty(r, k, device="cuda"), torch.empty(mb.n, r, device="cuda")) for mb in mem]
    Us = None
    if u_saved:
        # U_l from the layer's own forward (U_l = X A_l^T, fp32)
        Us = []
        for mb in mem:
            U = torch.empty(m, r, dtype=torch.float32, device="cuda")
            Y = torch.empty(m, mb.n, dtype=torch.bfloat16, device="cuda")
            ws = torch.empty(q.qlora_linear_workspace_bytes(m, mb.n, k, r), dtype=torch.uint8, device="cuda")
            q.qlora_linear_fwd(mb.qw, Xd, mb.Ad, mb.Bd, r, alpha, Y, q.QLORA_DTYPE_BF16, U, ws)
            Us.append(U)
        Us[-1] = None if len(mem) > 1 else Us[-1]      # the last layer recomputes its U
    ws = torch.empty(q.qlora_linear_group_workspace_bytes(m, [mb.n for mb in mem], k, r), dtype=torch.uint8,
                     device="cuda")
    q.qlora_linear_bwd_group([mb.qw for mb in mem], Xd, [mb.dYd for mb in mem], [mb.Ad for mb in mem],
                             [mb.Bd for mb in mem], r, alpha, Us, dX, dx_dtype, [g[0] for g in grads],
                             [g[1] for g in grads], flags, ws)
    q.qlora_check_device_error()
    return dX, grads


def _oracle(mem, X, alpha, rows=None):
    dX = 0.0
    out = []
    for mb in mem:
        dXl, dA, dB = o.linear_backward(mb.Wd, X, mb.dY, mb.A, mb.B, alpha, dx_rows=rows)
        dX = dX + dXl
        out.append((dA, dB))
    return dX, out


@pytest.mark.parametrize("m,ns,k,r,modes,dx_dtype", [
    # three layers, ragged tokens and output widths, CTA-pair kernel with 256-token units
    (300, (256, 392, 128), 320, 16, (q.QLORA_SCALE_DQ_FP8,) * 3, q.QLORA_DTYPE_FP32),
    # two layers with different scale formats, 512-token units, bf16 dX
    (1100, (576, 704), 512, 64, (q.QLORA_SCALE_BF16, q.QLORA_SCALE_DQ_FP8), q.QLORA_DTYPE_BF16),
    # at most 128 tokens: the layers one after the other
    (96, (256, 320, 192), 384, 32, (q.QLORA_SCALE_DQ_FP8,) * 3, q.QLORA_DTYPE_FP32),
    # rank 128 (two extension steps per layer)
    (260, (384, 256), 256, 128, (q.QLORA_SCALE_DQ_FP8,) * 2, q.QLORA_DTYPE_FP32),
])
def test_group_backward_matches_the_sum_of_layers(m, ns, k, r, modes, dx_dtype):
    alpha = 16.0
    mem = [Member(m, n, k, r, mode, layer=50 + i) for i, (n, mode) in enumerate(zip(ns, modes))]
    X = synth.activations(m, k, layer=49)
    dX, grads = _run_group(mem, X, r, alpha, dx_dtype)
    dX_ref, g_ref = _oracle(mem, X, alpha)
    check_close(dX.float().cpu(), dX_ref, "dX", bf16_out=(dx_dtype == q.QLORA_DTYPE_BF16))
    for i, ((dA, dB), (dA_r, dB_r)) in enumerate(zip(grads, g_ref)):
        check_close(dA.cpu(), dA_r, f"dA[{i}]")
        check_close(dB.cpu(), dB_r, f"dB[{i}]")


def test_group_backward_accumulates():
    m, ns, k, r, alpha = 520, (448, 256, 320), 448, 32, 32.0
    mem = [Member(m, n, k, r, q.QLORA_SCALE_DQ_FP8, layer=60 + i) for i, n in enumerate(ns)]
    X = synth.activations(m, k, layer=59)
    gen = torch.Generator().manual_seed(7)
    dX0 = torch.randn(m, k, generator=gen)
    g0 = [(torch.randn(r, k, generator=gen) * 1e-2, torch.randn(n, r, generator=gen) * 1e-2) for n in ns]
    grads = [(a.cuda(), b.cuda()) for a, b in g0]
    dX, grads = _run_group(mem, X, r, alpha, q.QLORA_DTYPE_FP32,
                           q.QLORA_BWD_ACCUMULATE_DX | q.QLORA_BWD_ACCUMULATE_GRADS, dX=dX0.cuda(), grads=grads)
    dX_ref, g_ref = _oracle(mem, X, alpha)
    check_close(dX.cpu(), dX_ref + dX0.double().numpy(), "dX+")
    for i, ((dA, dB), (dA_r, dB_r), (a0, b0)) in enumerate(zip(grads, g_ref, g0)):
        check_close(dA.cpu(), dA_r + a0.double().numpy(), f"dA+[{i}]")
        check_close(dB.cpu(), dB_r + b0.double().numpy(), f"dB+[{i}]")


def test_group_rejects_mismatched_inputs():
    m, r = 256, 16
    a = Member(m, 256, 256, r, q.QLORA_SCALE_DQ_FP8, layer=70, with_oracle=False)
    b = Member(m, 256, 320, r, q.QLORA_SCALE_DQ_FP8, layer=71, with_oracle=False)   # other k
    X = synth.activations(m, 256, layer=72).cuda()
    dX = torch.empty(m, 256, device="cuda")
    g = [(torch.empty(r, 256, device="cuda"), torch.empty(256, r, device="cuda")) for _ in range(2)]
    ws = torch.empty(1 << 24, dtype=torch.uint8, device="cuda")
    with pytest.raises(q.QloraError) as e:
        q.qlora_linear_bwd_group([a.qw, b.qw], X, [a.dYd, b.dYd], [a.Ad, b.Ad], [a.Bd, b.Bd], r, 16.0, None, dX,
                                 q.QLORA_DTYPE_FP32, [x[0] for x in g], [x[1] for x in g], 0, ws)
    assert e.value.status == q.QLORA_ERR_INVALID
    with pytest.raises(q.QloraError) as e:      # four layers: more than a group holds
        q.qlora_linear_bwd_group([a.qw] * 4, X, [a.dYd] * 4, [a.Ad] * 4, [a.Bd] * 4, r, 16.0, None, dX,
                                 q.QLORA_DTYPE_FP32, [g[0][0]] * 4, [g[0][1]] * 4, 0, ws)
    assert e.value.status == q.QLORA_ERR_INVALID
    assert q.qlora_linear_group_workspace_bytes(m, [256] * 4, 256, r) == 0


@pytest.mark.slow
def test_65b_attention_qkv_group_8192_tokens_sampled():
    # q/k/v 8192 x 8192 sharing X, 8192 tokens, r = 64, bf16 dX as the step computes it;
    # dX on seeded sampled token rows, every dA, dB in full
    M, H, r, alpha = 8192, 8192, 64, 16.0
    mem = [Member(M, H, H, r, q.QLORA_SCALE_DQ_FP8, layer=80 + i) for i in range(3)]
    X = synth.activations(M, H, layer=79)
    dX, grads = _run_group(mem, X, r, alpha, q.QLORA_DTYPE_BF16)
    rows = synth.sample_rows(M, 64).numpy()
    dX_ref, g_ref = _oracle(mem, X, alpha, rows=rows)
    check_close(dX.float().cpu().numpy()[rows], dX_ref, "dX", bf16_out=True)
    for i, ((dA, dB), (dA_r, dB_r)) in enumerate(zip(grads, g_ref)):
        check_close(dA.cpu(), dA_r, f"dA[{i}]")
        check_close(dB.cpu(), dB_r, f"dB[{i}]")
