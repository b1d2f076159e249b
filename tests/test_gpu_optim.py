"""Paged AdamW (32-bit) for the adapters against the oracle.

Bound: each fp32 step rounds the decayed parameter (about 2^-24 |p|) and the
update lr/(1-b1^t) m/(sqrt(v)/sqrt(1-b2^t) + eps), a short chain of roundings
(a few 2^-24 of the update, at most lr/(1-b1^t) in size). Over T steps the
parameter error stays below T (4 * 2^-24 |p| + 16 * 2^-24 lr_t) with lr_t the
largest bias-corrected step. m carries a few roundings of the size of the
terms it sums (the recurrence on |g|); v, a sum of squares, of its own size.
"""
import ctypes

import numpy as np
import pytest
import torch

import bit_nf4_quantized_03_b200 as q
from oracle import nf4_oracle as o
from tests.gpu_util import ensure_built

pytestmark = pytest.mark.gpu
U = 2.0 ** -24


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


def _run_oracle(p0, grads, lr, wd, beta1=0.9, beta2=0.999, eps=1e-8):
    # the hyperparameters cross the C ABI as fp32: the oracle uses the same values
    f = lambda x: float(np.float32(x))
    lr, wd, beta1, beta2, eps = f(lr), f(wd), f(beta1), f(beta2), f(eps)
    p, m, v = p0.astype(np.float64), np.zeros(p0.size), np.zeros(p0.size)
    for t, g in enumerate(grads, start=1):
        p, m, v = o.adamw_step(p, g.astype(np.float64), m, v, step=t, lr=lr, beta1=beta1, beta2=beta2, eps=eps,
                               weight_decay=wd)
    return p, m, v


def _magnitude(grads, beta1=0.9):
    """The first-moment recurrence run on |g|: the size of the terms m sums, which
    bounds its rounding error even where signed gradients cancel."""
    mag = np.zeros(grads[0].size)
    for g in grads:
        mag = beta1 * mag + (1 - beta1) * np.abs(g.astype(np.float64))
    return mag


def _check(p_got, m_got, v_got, p_ref, m_ref, v_ref, T, lr, grads, beta1=0.9):
    lr_t = lr / (1 - beta1)
    bound_p = T * (4 * U * np.abs(p_ref) + 16 * U * lr_t) + 1e-30
    assert np.all(np.abs(p_got - p_ref) <= bound_p), float(np.max(np.abs(p_got - p_ref) / bound_p))
    bound_m = T * 4 * U * _magnitude(grads, beta1) + 1e-38
    assert np.all(np.abs(m_got - m_ref) <= bound_m), float(np.max(np.abs(m_got - m_ref) / bound_m))
    bound_v = T * 8 * U * np.abs(v_ref) + 1e-38
    assert np.all(np.abs(v_got - v_ref) <= bound_v), float(np.max(np.abs(v_got - v_ref) / bound_v))


@pytest.mark.parametrize("count", [1, 3, 10007, 1 << 20])
def test_adamw_device_arrays(count):
    rng = np.random.default_rng(count)
    T, lr, wd = 6, 2e-4, 0.01
    p0 = rng.normal(0, 0.02, count).astype(np.float32)
    grads = [rng.normal(0, 1e-2, count).astype(np.float32) for _ in range(T)]
    p = torch.from_numpy(p0.copy()).cuda()
    m = torch.zeros(count, device="cuda")
    v = torch.zeros(count, device="cuda")
    pb = torch.empty(count, dtype=torch.bfloat16, device="cuda")
    for t, g in enumerate(grads, start=1):
        q.qlora_adamw_step(p, torch.from_numpy(g).cuda(), m, v, pb, count, q.AdamWConfig(lr, t, weight_decay=wd))
    q.qlora_check_device_error()
    p_ref, m_ref, v_ref = _run_oracle(p0, grads, lr, wd)
    p_got = p.cpu().numpy()
    _check(p_got.astype(np.float64), m.cpu().numpy().astype(np.float64), v.cpu().numpy().astype(np.float64),
           p_ref, m_ref, v_ref, T, lr, grads)
    # the bf16 working copy is the round-to-nearest-even of the fp32 master
    assert np.array_equal(pb.view(torch.int16).cpu().numpy().view(np.uint16), o.bf16_bits(p_got))


def test_adamw_grad_scale_and_no_copy():
    count = 4096
    rng = np.random.default_rng(5)
    p0 = rng.normal(0, 0.02, count).astype(np.float32)
    g = rng.normal(0, 1e-2, count).astype(np.float32)
    p = torch.from_numpy(p0.copy()).cuda()
    m = torch.zeros(count, device="cuda")
    v = torch.zeros(count, device="cuda")
    q.qlora_adamw_step(p, torch.from_numpy(2 * g).cuda(), m, v, None, count, q.AdamWConfig(1e-3, 1, grad_scale=0.5))
    p_ref, m_ref, v_ref = _run_oracle(p0, [g], 1e-3, 0.0)
    _check(p.cpu().numpy().astype(np.float64), m.cpu().numpy().astype(np.float64),
           v.cpu().numpy().astype(np.float64), p_ref, m_ref, v_ref, 1, 1e-3, [g])


def _host_view(addr, count):
    return np.ctypeslib.as_array((ctypes.c_float * count).from_address(addr))


def test_paged_states_resident_and_evicted():
    # masters and moments in paged (managed) memory: initialised from the host, prefetched to the device for
    # the step, evicted to host RAM and stepped again (the driver migrates on access), read back on the host
    count = 300_001
    rng = np.random.default_rng(9)
    T, lr, wd = 4, 2e-4, 0.05
    p0 = rng.normal(0, 0.02, count).astype(np.float32)
    grads = [rng.normal(0, 1e-2, count).astype(np.float32) for _ in range(T)]
    nbytes = count * 4
    addrs = [q.qlora_paged_alloc(nbytes) for _ in range(3)]
    try:
        hp, hm, hv = (_host_view(a, count) for a in addrs)
        hp[:] = p0
        hm[:] = 0
        hv[:] = 0
        for t, g in enumerate(grads, start=1):
            for a in addrs:
                q.qlora_paged_prefetch(a, nbytes, to_host=(t == 3))      # step 3 runs on evicted pages
            q.qlora_adamw_step(addrs[0], torch.from_numpy(g).cuda(), addrs[1], addrs[2], None, count,
                               q.AdamWConfig(lr, t, weight_decay=wd))
        for a in addrs:
            q.qlora_paged_prefetch(a, nbytes, to_host=True)
        torch.cuda.synchronize()
        q.qlora_check_device_error()
        p_ref, m_ref, v_ref = _run_oracle(p0, grads, lr, wd)
        _check(hp.astype(np.float64), hm.astype(np.float64), hv.astype(np.float64), p_ref, m_ref, v_ref, T, lr,
               grads)
    finally:
        torch.cuda.synchronize()
        for a in addrs:
            q.qlora_paged_free(a)
