"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
on seeded inputs and compare with the oracle on the same inputs."""
from __future__ import annotations

import math

import numpy as np
import torch

import bit_nf4_quantized_03_b200 as q
from bit_nf4_quantized_03_b200 import synth
from oracle import nf4_oracle as o

REL_FROB = 2e-3        # relative Frobenius error bound
MAX_ABS_RMS = 1e-2     # max |error| / RMS(reference)


def ensure_built():
    from bit_nf4_quantized_03_b200 import build
    build.build(bounds_check=q.BOUNDS_CHECK)
    q.lib()


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def gpu_quantize(W_cpu: torch.Tensor, mode: int) -> q.QuantizedWeight:
    n, k = W_cpu.shape
    qw = q.QuantizedWeight(n, k, mode)
    q.qlora_nf4_quantize(W_cpu.cuda(), qw)
    q.qlora_check_device_error()
    return qw


def gpu_weight_dict(qw: q.QuantizedWeight) -> dict:
    d = {"codes": qw.codes.cpu().numpy(), "n_elem": qw.n * qw.k, "mode": qw.mode}
    if qw.mode == q.QLORA_SCALE_BF16:
        d["scale_bf16"] = qw.scale_bf16.cpu().numpy().view(np.uint16)
    else:
        d["scale_fp8"] = qw.scale_fp8.cpu().numpy()
        d["dq_scale"] = qw.dq_scale.cpu().numpy()
        d["dq_mean"] = np.float32(qw.dq_mean.cpu().numpy()[0])
    return d


def assert_weight_bitexact(got: dict, ref: dict):
    assert np.array_equal(got["codes"], ref["codes"]), _first_diff(got["codes"], ref["codes"])
    if ref["mode"] == o.MODE_BF16:
        assert np.array_equal(got["scale_bf16"], ref["scale_bf16"]), _first_diff(got["scale_bf16"], ref["scale_bf16"])
    else:
        assert np.float32(got["dq_mean"]).view(np.uint32) == np.float32(ref["dq_mean"]).view(np.uint32), \
            (got["dq_mean"], ref["dq_mean"])
        assert np.array_equal(got["dq_scale"].view(np.uint32), ref["dq_scale"].view(np.uint32)), \
            _first_diff(got["dq_scale"], ref["dq_scale"])
        assert np.array_equal(got["scale_fp8"], ref["scale_fp8"]), _first_diff(got["scale_fp8"], ref["scale_fp8"])


def _first_diff(a, b):
    a, b = np.asarray(a), np.asarray(b)
    if a.shape != b.shape:
        return f"shape {a.shape} vs {b.shape}"
    idx = np.nonzero(a.reshape(-1) != b.reshape(-1))[0]
    return f"{idx.size} mismatches, first at {idx[:5].tolist()}: got {a.reshape(-1)[idx[:5]]} want {b.reshape(-1)[idx[:5]]}"


def check_close(got, ref, name: str, bf16_out: bool = False):
    """Relative Frobenius <= 2e-3 and max-abs <= 1e-2 * RMS(ref); for bf16
    outputs each element's bound is widened by half a bf16 ulp of the
    reference, and the Frobenius bound by the reference's own bf16 rounding."""
    got = o._f64(got)
    ref = o._f64(ref)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), name
    diff = got - ref
    ref_norm = math.sqrt(float(np.sum(ref * ref)))
    rms = math.sqrt(float(np.mean(ref * ref)))
    frob_allow = REL_FROB * ref_norm
    elem_allow = np.full(ref.shape, MAX_ABS_RMS * rms)
    if bf16_out:
        rounded = o.bf16_to_f32(o.bf16_bits(ref.astype(np.float32))).astype(np.float64)
        frob_allow += math.sqrt(float(np.sum((rounded - ref) ** 2)))
        e = np.floor(np.log2(np.maximum(np.abs(ref), 1e-300)))
        elem_allow = elem_allow + 0.5 * np.exp2(e - 7)
    frob = math.sqrt(float(np.sum(diff * diff)))
    assert frob <= frob_allow, f"{name}: rel frob {frob / max(ref_norm, 1e-300):.3e} > allowed {frob_allow / max(ref_norm, 1e-300):.3e}"
    bad = np.abs(diff) > elem_allow
    assert not bad.any(), f"{name}: {int(bad.sum())} elements over the max-abs bound; worst {float(np.max(np.abs(diff) / elem_allow)):.3f}x"
    return frob / max(ref_norm, 1e-300), float(np.max(np.abs(diff))) / max(rms, 1e-300)


class Layer:
    """Seeded inputs of one linear layer on the host and on the device."""

    def __init__(self, m, n, k, r, alpha=16.0, mode=q.QLORA_SCALE_DQ_FP8, layer=0, outlier_frac=0.0):
        self.m, self.n, self.k, self.r, self.alpha, self.mode = m, n, k, r, alpha, mode
        self.W = synth.weight(n, k, outlier_frac=outlier_frac, layer=layer)
        self.X = synth.activations(m, k, layer=layer)
        self.A, self.B = synth.lora_pair(r, k, n, layer=layer)
        self.dY = synth.grad_output(m, n, layer=layer)
        self.qw = gpu_quantize(self.W, mode)
        self.Xd, self.Ad, self.Bd, self.dYd = (t.cuda() for t in (self.X, self.A, self.B, self.dY))
        self.ws = torch.empty(q.qlora_linear_workspace_bytes(m, n, k, r), dtype=torch.uint8, device="cuda")
        self._ref_w = None

    def oracle_weight(self):
        if self._ref_w is None:
            ref = o.quantize(self.W.numpy(), self.mode)
            self._ref_w = o.dequantize_f64(ref, (self.n, self.k))
        return self._ref_w

    def fwd(self, y_dtype=q.QLORA_DTYPE_FP32, save_u=True):
        dt = torch.float32 if y_dtype == q.QLORA_DTYPE_FP32 else torch.bfloat16
        Y = torch.empty(self.m, self.n, dtype=dt, device="cuda")
        U = torch.empty(self.m, self.r, dtype=torch.float32, device="cuda") if save_u else None
        q.qlora_linear_fwd(self.qw, self.Xd, self.Ad, self.Bd, self.r, self.alpha, Y, y_dtype, U, self.ws)
        q.qlora_check_device_error()
        return Y, U

    def bwd(self, U=None, dx_dtype=q.QLORA_DTYPE_FP32, flags=0, dX=None, dA=None, dB=None, with_dx=True):
        dt = torch.float32 if dx_dtype == q.QLORA_DTYPE_FP32 else torch.bfloat16
        if with_dx and dX is None:
            dX = torch.empty(self.m, self.k, dtype=dt, device="cuda")
        dA = torch.empty(self.r, self.k, dtype=torch.float32, device="cuda") if dA is None else dA
        dB = torch.empty(self.n, self.r, dtype=torch.float32, device="cuda") if dB is None else dB
        q.qlora_linear_bwd(self.qw, self.Xd, self.dYd, self.Ad, self.Bd, self.r, self.alpha, U,
                           dX if with_dx else None, dx_dtype, dA, dB, flags, self.ws)
        q.qlora_check_device_error()
        return dX, dA, dB
