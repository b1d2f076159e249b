"""GPU parity of the fused QLoRA linear layer (forward and backward) against
the fp64 oracle on the same seeded inputs: relative Frobenius error <= 2e-3
and max |error| <= 1e-2 x RMS of the reference, per output (Y, U, dX, dA, dB).
fp32 outputs are checked at exactly those bounds; bf16 outputs with each
element's bound widened by half a bf16 ulp of the reference."""
import threading

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


def _full_check(L: Layer, y_dtype=q.QLORA_DTYPE_FP32, dx_dtype=q.QLORA_DTYPE_FP32, save_u=True):
    Wd = L.oracle_weight()
    Y, U = L.fwd(y_dtype, save_u=save_u)
    Y_ref, U_ref = o.linear_forward(Wd, L.X, L.A, L.B, L.alpha)
    check_close(Y.float().cpu(), Y_ref, "Y", bf16_out=(y_dtype == q.QLORA_DTYPE_BF16))
    if save_u:
        check_close(U.cpu(), U_ref, "U")
    dX, dA, dB = L.bwd(U if save_u else None, dx_dtype)
    dX_ref, dA_ref, dB_ref = o.linear_backward(Wd, L.X, L.dY, L.A, L.B, L.alpha)
    check_close(dX.float().cpu(), dX_ref, "dX", bf16_out=(dx_dtype == q.QLORA_DTYPE_BF16))
    check_close(dA.cpu(), dA_ref, "dA")
    check_close(dB.cpu(), dB_ref, "dB")


def test_single_linear_256_r8():
    # 128 tokens, W 256 x 256, r = 8, alpha = 16, double-quant weights
    _full_check(Layer(128, 256, 256, 8))


@pytest.mark.parametrize("m,n,k,r", [
    (200, 264, 320, 16),     # ragged M, N (not a multiple of 64 or 256) and K (not a multiple of 256)
    (256, 512, 512, 32),
    (384, 768, 1024, 64),
    (130, 512, 384, 128),
    (1, 256, 256, 64),       # single token
    (16, 1024, 2048, 64),    # small-M split-K path
    (40, 512, 832, 32),      # 17-64 tokens: the wider small-M U kernel; K slices of 104, padded rank rows
    (8, 256, 512, 8),        # rank 8 padded to 64 in the forward's K extension
    (72, 4096, 1024, 16),
])
def test_linear_shapes_and_ranks(m, n, k, r):
    _full_check(Layer(m, n, k, r))


def test_linear_bf16_scales_and_bf16_outputs():
    L = Layer(256, 512, 768, 64, mode=q.QLORA_SCALE_BF16)
    _full_check(L, y_dtype=q.QLORA_DTYPE_BF16, dx_dtype=q.QLORA_DTYPE_BF16)


def test_backward_recomputes_u_when_not_saved():
    _full_check(Layer(192, 320, 448, 32), save_u=False)


def test_accumulate_flags():
    L = Layer(160, 384, 512, 16)
    Wd = L.oracle_weight()
    dX_ref, dA_ref, dB_ref = o.linear_backward(Wd, L.X, L.dY, L.A, L.B, L.alpha)
    g = torch.Generator().manual_seed(99)
    dX0 = torch.randn(L.m, L.k, generator=g)
    dA0 = torch.randn(L.r, L.k, generator=g) * 1e-2
    dB0 = torch.randn(L.n, L.r, generator=g) * 1e-2
    dX, dA, dB = dX0.cuda(), dA0.cuda(), dB0.cuda()
    L.bwd(None, q.QLORA_DTYPE_FP32, q.QLORA_BWD_ACCUMULATE_GRADS | q.QLORA_BWD_ACCUMULATE_DX, dX, dA, dB)
    check_close(dX.cpu(), dX_ref + dX0.double().numpy(), "dX+")
    check_close(dA.cpu(), dA_ref + dA0.double().numpy(), "dA+")
    check_close(dB.cpu(), dB_ref + dB0.double().numpy(), "dB+")


@pytest.mark.parametrize("dx_dtype", [q.QLORA_DTYPE_FP32, q.QLORA_DTYPE_BF16])
def test_accumulate_dx_many_tokens(dx_dtype):
    # on the CTA-pair path an accumulating dX goes through fp32 partials and the reduce pass while a
    # plain one is written by the GEMM: both against the oracle, on ragged token and feature counts
    L = Layer(2312, 520, 1088, 16)
    Wd = L.oracle_weight()
    dX_ref, _, _ = o.linear_backward(Wd, L.X, L.dY, L.A, L.B, L.alpha)
    g = torch.Generator().manual_seed(7)
    dX0 = torch.randn(L.m, L.k, generator=g)
    if dx_dtype == q.QLORA_DTYPE_BF16:
        dX0 = dX0.to(torch.bfloat16).float()
        dX = dX0.to(torch.bfloat16).cuda()
    else:
        dX = dX0.clone().cuda()
    L.bwd(None, dx_dtype, q.QLORA_BWD_ACCUMULATE_DX, dX)
    check_close(dX.float().cpu(), dX_ref + dX0.double().numpy(), "dX+", bf16_out=(dx_dtype == q.QLORA_DTYPE_BF16))
    dXp, _, _ = L.bwd(None, dx_dtype)
    check_close(dXp.float().cpu(), dX_ref, "dX", bf16_out=(dx_dtype == q.QLORA_DTYPE_BF16))


def test_backward_without_dx():
    L = Layer(128, 256, 256, 8)
    Wd = L.oracle_weight()
    _, dA, dB = L.bwd(None, with_dx=False)
    _, dA_ref, dB_ref = o.linear_backward(Wd, L.X, L.dY, L.A, L.B, L.alpha)
    check_close(dA.cpu(), dA_ref, "dA")
    check_close(dB.cpu(), dB_ref, "dB")


def test_repeat_calls_identical():
    L = Layer(256, 512, 512, 64)
    Y1, _ = L.fwd()
    Y2, _ = L.fwd()
    assert torch.equal(Y1, Y2)
    _, dA1, dB1 = L.bwd()
    _, dA2, dB2 = L.bwd()
    assert torch.equal(dA1, dA2) and torch.equal(dB1, dB2)


def test_7b_q_proj_full():
    # 7B-shape q_proj: X 2048 x 4096 (batch 4 x seq 512), W 4096 x 4096, r = 64, alpha = 16
    _full_check(Layer(2048, 4096, 4096, 64))


def test_backward_beside_dx_accumulating_grads():
    # 512 tokens, W 256 x 2048: the CTA-pair dX GEMM (one split) takes 16 of 148 SMs, and dB and dA
    # run beside it on the library's internal stream; accumulated into nonzero gradients
    L = Layer(512, 256, 2048, 64)
    Wd = L.oracle_weight()
    _, U = L.fwd()
    dX_ref, dA_ref, dB_ref = o.linear_backward(Wd, L.X, L.dY, L.A, L.B, L.alpha)
    dX, dA1, dB1 = L.bwd(U)
    check_close(dX.cpu(), dX_ref, "dX")
    check_close(dA1.cpu(), dA_ref, "dA")
    check_close(dB1.cpu(), dB_ref, "dB")
    g = torch.Generator().manual_seed(5)
    dA0 = torch.randn(L.r, L.k, generator=g) * 1e-2
    dB0 = torch.randn(L.n, L.r, generator=g) * 1e-2
    dA, dB = dA0.cuda(), dB0.cuda()
    L.bwd(U, q.QLORA_DTYPE_FP32, q.QLORA_BWD_ACCUMULATE_GRADS, None, dA, dB)
    check_close(dA.cpu(), dA_ref + dA0.double().numpy(), "dA+")
    check_close(dB.cpu(), dB_ref + dB0.double().numpy(), "dB+")


def _capture_bwd(L: Layer, U, outs):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=torch.cuda.Stream()):
        q.qlora_linear_bwd(L.qw, L.Xd, L.dYd, L.Ad, L.Bd, L.r, L.alpha, U, outs[0], q.QLORA_DTYPE_FP32,
                           outs[1], outs[2], 0, L.ws)
    return g


@pytest.mark.parametrize("shape", [(512, 256, 2048, 64), (2048, 4096, 4096, 64)])
def test_backward_side_stream_same_bits_and_graph_replay(shape):
    # With idle SMs beside the dX GEMM the backward forks dB and dA onto an internal stream and joins
    # them back; a thread's first call under stream capture has no such stream yet and keeps all on
    # the caller's stream. Eager, captured with the fork, and captured without it: the same bits.
    L = Layer(*shape)
    _, U = L.fwd()

    def outs():
        return tuple(torch.full(s, float("nan"), device="cuda") for s in ((L.m, L.k), (L.r, L.k), (L.n, L.r)))

    eager = L.bwd(U)
    forked = outs()
    g_fork = _capture_bwd(L, U, forked)
    single = outs()
    box = {}

    def in_thread():
        try:
            box["g"] = _capture_bwd(L, U, single)
        except BaseException as e:      # reported by the assertion below
            box["err"] = e

    t = threading.Thread(target=in_thread)
    t.start()
    t.join()
    assert "g" in box, box.get("err")
    g_fork.replay()
    box["g"].replay()
    torch.cuda.synchronize()
    q.qlora_check_device_error()
    for name, a, b, c in zip(("dX", "dA", "dB"), eager, forked, single):
        assert torch.equal(a, b), name + ": graph with the fork differs from the eager call"
        assert torch.equal(a, c), name + ": one-stream graph differs from the eager call"


def test_silu_gate_glue():
    g = synth.activations(333, 129, seed=31)
    u = synth.activations(333, 129, seed=32)
    dh = synth.activations(333, 129, seed=33)
    gd, ud, dhd = g.cuda(), u.cuda(), dh.cuda()
    h = torch.empty_like(gd)
    dg = torch.empty_like(gd)
    du = torch.empty_like(gd)
    q.qlora_silu_gate_fwd(gd, ud, h)
    q.qlora_silu_gate_bwd(dhd, gd, ud, dg, du)
    check_close(h.float().cpu(), o.silu_gate_forward(g, u), "h", bf16_out=True)
    dg_ref, du_ref = o.silu_gate_backward(dh, g, u)
    check_close(dg.float().cpu(), dg_ref, "dg", bf16_out=True)
    check_close(du.float().cpu(), du_ref, "du", bf16_out=True)
