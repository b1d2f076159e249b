"""Parity at the full workload sizes, in the launch configuration bench.py
times (bf16 activations, double-quantized NF4 weights, r = 64, alpha = 16).

Outputs the oracle cannot afford in full are compared on seeded sampled
token rows (every row of Y and dX depends only on its own token); the
adapter gradients dA, dB, which sum over all tokens, are compared in full.
"""
import numpy as np
import pytest
import torch

import bit_nf4_quantized_03_b200 as q
from bit_nf4_quantized_03_b200 import synth
from oracle import nf4_oracle as o
from tests.gpu_util import check_close, ensure_built, gpu_quantize

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
R, ALPHA = 64, 16.0


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


def _bf16_round(x):
    return o.bf16_to_f32(o.bf16_bits(np.asarray(x, dtype=np.float32))).astype(np.float64)


class Lin:
    def __init__(self, n, k, layer):
        self.n, self.k = n, k
        W = synth.weight(n, k, layer=layer)
        self.qw = gpu_quantize(W, q.QLORA_SCALE_DQ_FP8)
        self.Wd = o.dequantize_f64(o.quantize(W.numpy(), o.MODE_DQ_FP8), (n, k))
        self.A, self.B = synth.lora_pair(R, k, n, layer=layer)
        self.Ad, self.Bd = self.A.cuda(), self.B.cuda()

    def fwd(self, X, Y, U, ws):
        q.qlora_linear_fwd(self.qw, X, self.Ad, self.Bd, R, ALPHA, Y, q.QLORA_DTYPE_BF16, U, ws)

    def bwd(self, X, dY, U, dX, dA, dB, flags, ws):
        q.qlora_linear_bwd(self.qw, X, dY, self.Ad, self.Bd, R, ALPHA, U, dX, q.QLORA_DTYPE_BF16, dA, dB, flags, ws)


def test_7b_mlp_silu_chain_fwd_bwd():
    # gate/up 11008 x 4096, down 4096 x 11008, 4096 tokens, SiLU-gated between
    M, H, I = 4096, 4096, 11008
    gate, up, down = Lin(I, H, 0), Lin(I, H, 1), Lin(H, I, 2)
    X = synth.activations(M, H, layer=10)
    dY = synth.grad_output(M, H, layer=11)
    Xd, dYd = X.cuda(), dY.cuda()
    ws = torch.empty(max(q.qlora_linear_workspace_bytes(M, I, H, R), q.qlora_linear_workspace_bytes(M, H, I, R)),
                     dtype=torch.uint8, device="cuda")
    bf, f32 = torch.bfloat16, torch.float32
    g, u, h = (torch.empty(M, I, dtype=bf, device="cuda") for _ in range(3))
    y = torch.empty(M, H, dtype=bf, device="cuda")
    Ug, Uu, Ud = (torch.empty(M, R, dtype=f32, device="cuda") for _ in range(3))
    gate.fwd(Xd, g, Ug, ws)
    up.fwd(Xd, u, Uu, ws)
    q.qlora_silu_gate_fwd(g, u, h)
    down.fwd(h, y, Ud, ws)
    dh, dg, du = (torch.empty(M, I, dtype=bf, device="cuda") for _ in range(3))
    dX = torch.empty(M, H, dtype=bf, device="cuda")
    grads = {nm: (torch.empty(R, lin.k, dtype=f32, device="cuda"), torch.empty(lin.n, R, dtype=f32, device="cuda"))
             for nm, lin in (("gate", gate), ("up", up), ("down", down))}
    down.bwd(h, dYd, Ud, dh, *grads["down"], 0, ws)
    q.qlora_silu_gate_bwd(dh, g, u, dg, du)
    gate.bwd(Xd, dg, Ug, dX, *grads["gate"], 0, ws)
    up.bwd(Xd, du, Uu, dX, *grads["up"], q.QLORA_BWD_ACCUMULATE_DX, ws)
    q.qlora_check_device_error()

    # oracle chain in fp64, rounded to bf16 where the ABI stores bf16 tensors
    Xf, dYf = o._f64(X), o._f64(dY)
    g_r, _ = o.linear_forward(gate.Wd, Xf, gate.A, gate.B, ALPHA)
    u_r, _ = o.linear_forward(up.Wd, Xf, up.A, up.B, ALPHA)
    g_b, u_b = _bf16_round(g_r), _bf16_round(u_r)
    h_b = _bf16_round(o.silu_gate_forward(g_b, u_b))
    rows = synth.sample_rows(M, 64).numpy()
    y_r, _ = o.linear_forward(down.Wd, h_b, down.A, down.B, ALPHA, rows=rows)
    check_close(y.float().cpu().numpy()[rows], y_r, "y", bf16_out=True)
    dh_r, dA_d, dB_d = o.linear_backward(down.Wd, h_b, dYf, down.A, down.B, ALPHA)
    check_close(grads["down"][0].cpu(), dA_d, "dA down")
    check_close(grads["down"][1].cpu(), dB_d, "dB down")
    dh_b = _bf16_round(dh_r)
    dg_r, du_r = o.silu_gate_backward(dh_b, g_b, u_b)
    dg_b, du_b = _bf16_round(dg_r), _bf16_round(du_r)
    dXg, dA_g, dB_g = o.linear_backward(gate.Wd, Xf, dg_b, gate.A, gate.B, ALPHA, dx_rows=rows)
    dXu, dA_u, dB_u = o.linear_backward(up.Wd, Xf, du_b, up.A, up.B, ALPHA, dx_rows=rows)
    check_close(dX.float().cpu().numpy()[rows], dXg + dXu, "dX", bf16_out=True)
    check_close(grads["gate"][0].cpu(), dA_g, "dA gate")
    check_close(grads["gate"][1].cpu(), dB_g, "dB gate")
    check_close(grads["up"][0].cpu(), dA_u, "dA up")
    check_close(grads["up"][1].cpu(), dB_u, "dB up")


@pytest.mark.parametrize("name,n,k", [("q_proj", 8192, 8192), ("gate_proj", 22016, 8192), ("down_proj", 8192, 22016)])
def test_65b_linear_fwd_bwd_8192_tokens_sampled(name, n, k):
    M = 8192
    lin = Lin(n, k, 3)
    X = synth.activations(M, k, layer=20)
    dY = synth.grad_output(M, n, layer=21)
    Xd, dYd = X.cuda(), dY.cuda()
    ws = torch.empty(q.qlora_linear_workspace_bytes(M, n, k, R), dtype=torch.uint8, device="cuda")
    Y = torch.empty(M, n, dtype=torch.bfloat16, device="cuda")
    U = torch.empty(M, R, dtype=torch.float32, device="cuda")
    dX = torch.empty(M, k, dtype=torch.bfloat16, device="cuda")
    dA = torch.empty(R, k, dtype=torch.float32, device="cuda")
    dB = torch.empty(n, R, dtype=torch.float32, device="cuda")
    lin.fwd(Xd, Y, U, ws)
    lin.bwd(Xd, dYd, U, dX, dA, dB, 0, ws)
    q.qlora_check_device_error()
    rows = synth.sample_rows(M, 64).numpy()
    Y_r, U_r = o.linear_forward(lin.Wd, X, lin.A, lin.B, ALPHA, rows=rows)
    check_close(Y.float().cpu().numpy()[rows], Y_r, "Y", bf16_out=True)
    check_close(U.cpu().numpy()[rows], U_r, "U")
    dX_r, dA_r, dB_r = o.linear_backward(lin.Wd, X, dY, lin.A, lin.B, ALPHA, dx_rows=rows)
    check_close(dX.float().cpu().numpy()[rows], dX_r, "dX", bf16_out=True)
    check_close(dA.cpu(), dA_r, "dA")
    check_close(dB.cpu(), dB_r, "dB")


@pytest.mark.parametrize("name,n,k", [("q_proj", 8192, 8192), ("gate_proj", 22016, 8192), ("down_proj", 8192, 22016)])
def test_65b_linear_fwd_16_tokens_full(name, n, k):
    M = 16
    lin = Lin(n, k, 4)
    X = synth.activations(M, k, layer=30)
    ws = torch.empty(q.qlora_linear_workspace_bytes(M, n, k, R), dtype=torch.uint8, device="cuda")
    Y = torch.empty(M, n, dtype=torch.bfloat16, device="cuda")
    U = torch.empty(M, R, dtype=torch.float32, device="cuda")
    q.qlora_linear_fwd(lin.qw, X.cuda(), lin.Ad, lin.Bd, R, ALPHA, Y, q.QLORA_DTYPE_BF16, U, ws)
    q.qlora_check_device_error()
    Y_r, U_r = o.linear_forward(lin.Wd, X, lin.A, lin.B, ALPHA)
    check_close(Y.float().cpu(), Y_r, "Y", bf16_out=True)
    check_close(U.cpu(), U_r, "U")
