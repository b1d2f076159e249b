"""Pins for the CPU oracle: each test ties it to something other than itself.

Pins used: the one-block worked example and storage arithmetic printed on the
pages (golden files), closed forms, invariants of the level construction,
an independent inverse normal CDF (bisection on math.erfc), brute-force
nearest-level and nearest-E4M3 searches, torch's own bf16/fp8 casts, exact
round trips for weights that sit on the level grid, pure-Python loops for the
layer on tiny shapes, and finite differences for the gradients.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import nf4_oracle as o

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _kv(name):
    out = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        k, *v = line.split()
        out[k] = v
    return out


# ---------------------------------------------------------------- levels ----
def _phi_inv_bisect(p: float) -> float:
    """Inverse standard-normal CDF by bisection on erfc (independent of scipy)."""
    lo, hi = -40.0, 40.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if 0.5 * math.erfc(-mid / math.sqrt(2.0)) < p:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def test_levels_invariants():
    L = o.nf4_levels()
    assert L.dtype == np.float32 and L.shape == (16,)
    assert np.all(np.diff(L) > 0), "16 strictly increasing levels"
    assert L[7] == 0.0 and not np.signbit(L[7]), "exact zero"
    assert L[0] == -1.0 and L[15] == 1.0, "normalised to [-1, 1] at both ends"
    assert np.sum(L > 0) == 8 and np.sum(L < 0) == 7


def test_levels_are_normal_quantiles_independent_inverse():
    # positive side: 8 quantiles on the 9-point grid from delta to 1/2;
    # negative side: 7 quantiles on the 8-point grid, mirrored.
    d = o.NF4_DELTA
    pos = [_phi_inv_bisect(d + (0.5 - d) * i / 8.0) for i in range(8)]
    neg = [-_phi_inv_bisect(d + (0.5 - d) * i / 7.0) for i in range(7)]
    ref = np.array(sorted(pos + [0.0] + neg))
    ref = ref / ref.max()
    np.testing.assert_allclose(o.nf4_levels_f64(), ref, rtol=0, atol=1e-12)
    assert np.array_equal(o.nf4_levels(), ref.astype(np.float32))
    # the outermost positive and negative levels are the same quantile
    assert pos[0] == pytest.approx(-neg[0], rel=1e-14)


def test_levels_quantile_roundtrip_through_cdf():
    # Phi(L_j * Phi^-1(delta)) must land back on the probability grid.
    d = o.NF4_DELTA
    qmax = _phi_inv_bisect(d)
    L = o.nf4_levels_f64()
    cdf = [0.5 * math.erfc(-(x * qmax) / math.sqrt(2.0)) for x in L]
    want = sorted([d + (0.5 - d) * i / 8.0 for i in range(8)] + [0.5] +
                  [1.0 - (d + (0.5 - d) * i / 7.0) for i in range(7)])
    np.testing.assert_allclose(cdf, want, rtol=0, atol=1e-12)


# ------------------------------------------------ nearest level (midpoints) --
def _brute_nearest(x):
    L = o.nf4_levels().astype(np.float64)
    x = np.asarray(x, dtype=np.float64)
    d = np.abs(x[:, None] - L[None, :])
    return np.argmin(d, axis=1)          # first minimum = lower level on a tie


def test_midpoint_rule_equals_bruteforce_nearest_on_all_bf16_in_range():
    bits = np.arange(65536, dtype=np.uint16)
    x = o.bf16_to_f32(bits)
    x = x[np.isfinite(x) & (np.abs(x) <= 1.0)]
    got = o.nf4_code_of(x)
    want = _brute_nearest(x)
    L = o.nf4_levels().astype(np.float64)
    exact_mid = 0.5 * (L[:-1] + L[1:])
    m32 = o.nf4_midpoints().astype(np.float64)
    bad = np.nonzero(got != want)[0]
    for i in bad:   # only values between fp32(m_i) and the exact midpoint may differ
        xi = float(x[i])
        assert any(min(a, b) <= xi <= max(a, b) for a, b in zip(m32, exact_mid)), xi


def test_midpoint_rule_random_and_near_thresholds():
    rng = np.random.default_rng(11)
    x = rng.uniform(-1, 1, 200000).astype(np.float32)
    m = o.nf4_midpoints()
    near = np.concatenate([np.nextafter(m, np.float32(2)), np.nextafter(m, np.float32(-2)),
                           np.nextafter(np.nextafter(m, np.float32(2)), np.float32(2))])
    xs = np.concatenate([x, near, o.nf4_levels()])
    got = o.nf4_code_of(xs)
    want = _brute_nearest(xs)
    L = o.nf4_levels().astype(np.float64)
    exact_mid = 0.5 * (L[:-1] + L[1:])
    for i in np.nonzero(got != want)[0]:
        xi = float(xs[i])
        assert any(min(a, b) <= xi <= max(a, b) for a, b in zip(m.astype(np.float64), exact_mid))
    # each level maps to its own code; a value exactly on a midpoint goes down
    assert np.array_equal(o.nf4_code_of(o.nf4_levels()), np.arange(16))
    assert np.array_equal(o.nf4_code_of(m), np.arange(15))


# ------------------------------------------------------------ worked example -
def test_worked_example_block():
    g = _kv("worked_example_block.txt")
    w = np.array([float(v) for v in g["weights"]], dtype=np.float32)
    assert len(w) == 8
    qw = o.quantize(w, o.MODE_BF16)
    # largest magnitude is the block scale, kept in BF16
    assert qw["absmax"][0] == np.float32(float(g["absmax"][0]))
    assert o.bf16_to_f32(qw["scale_bf16"])[0] == 1.0
    assert qw["scale_bf16"].nbytes == int(g["scale_bytes_bf16"][0])
    # 16 bytes in BF16 vs 4 bytes of NF4 codes
    assert w.astype(np.float32).size * 2 == int(g["bf16_bytes"][0])
    assert qw["codes"].nbytes == int(g["nf4_bytes"][0])
    codes = o.unpack_nibbles(qw["codes"], 8)
    # each weight snapped to the nearest of the 16 levels
    assert np.array_equal(codes, _brute_nearest(w))
    deq = o.bf16_to_f32(o.dequantize(qw))
    assert deq[4] == 1.0 and codes[4] == 15, "the 1.00 element is reproduced exactly"
    gap = np.max(np.diff(o.nf4_levels().astype(np.float64)))
    assert np.all(np.abs(deq - w) <= gap / 2 + 2 ** -8)


# ---------------------------------------------------------- storage pins -----
def test_four_x_shrink_and_65b_storage():
    g = _kv("storage_closed_forms.txt")
    n, k = 512, 1024
    w = np.random.default_rng(0).normal(0, 0.02, (n, k)).astype(np.float32)
    qw = o.quantize(w, o.MODE_BF16)
    bf16_bytes = 2 * n * k
    assert bf16_bytes / qw["codes"].nbytes == float(g["shrink_factor"][0])
    per_param = qw["codes"].nbytes / (n * k)
    per_param_scaled = (qw["codes"].nbytes + qw["scale_bf16"].nbytes) / (n * k)
    P = float(g["params_65b"][0])
    assert P * 2 == float(g["bf16_bytes_65b"][0])
    assert P * per_param == float(g["nf4_bytes_65b"][0])
    assert abs(P * per_param_scaled - float(g["nf4_with_scales_bytes_65b_about"][0])) < 0.05 * 35e9


def test_double_quant_saving_closed_form():
    g = _kv("storage_closed_forms.txt")
    n_elem = 1 << 22
    w = np.random.default_rng(1).normal(0, 0.02, n_elem).astype(np.float32)
    qd = o.quantize(w, o.MODE_DQ_FP8)
    nblk = qd["scale_fp8"].size
    fp32_first_level_bits = 32 * nblk
    dq_bits = 8 * qd["scale_fp8"].nbytes + 8 * qd["dq_scale"].nbytes + 32   # + fp32 mean
    saving = (fp32_first_level_bits - dq_bits) / n_elem
    want = float(g["dq_saving_bits_per_param"][0])
    assert abs(saving - want) <= 32.0 / n_elem + 1e-15
    assert abs(want * float(g["params_65b"][0]) / 8 - float(g["dq_saving_bytes_65b_about"][0])) < 0.1e9


# ---------------------------------------------------------- bf16 / e4m3 ------
def test_bf16_rounding_matches_torch_cast():
    rng = np.random.default_rng(2)
    x = np.concatenate([rng.normal(0, 1, 100000), rng.normal(0, 1e-30, 1000),
                        rng.normal(0, 1e30, 1000)]).astype(np.float32)
    # exact ties: low 16 bits == 0x8000
    ties = (rng.integers(0, 2 ** 31, 2000, dtype=np.uint32) & 0xFFFF0000) | 0x8000
    x = np.concatenate([x, ties.view(np.float32)])
    x = x[np.isfinite(x)]
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(o.bf16_bits(x), want)


def test_e4m3_spec_values():
    for line in open(os.path.join(GOLDEN, "e4m3_spec_values.txt")):
        if line.startswith("#") or not line.strip():
            continue
        v, c = line.split()
        v, c = float(v), int(c, 16)
        assert o.e4m3_decode(np.array([c], np.uint8))[0] == np.float32(v)
        assert o.e4m3_encode(np.array([v], np.float32))[0] == c
    assert np.isnan(o.e4m3_decode(np.array([0x7F, 0xFF], np.uint8))).all()


def _e4m3_brute(v):
    vals = o.e4m3_decode(np.arange(127, dtype=np.uint8)).astype(np.float64)
    out = []
    for x in np.asarray(v, dtype=np.float32):
        a = abs(float(x))
        if a >= 448.0:
            c = 126
        else:
            d = np.abs(vals - a)
            best = np.nonzero(d == d.min())[0]
            c = int(best[0]) if len(best) == 1 else int([b for b in best if b % 2 == 0][0])
        if np.signbit(x):
            c |= 0x80
        out.append(c)
    return np.array(out, dtype=np.uint8)


def test_e4m3_encode_bruteforce():
    rng = np.random.default_rng(3)
    mags = np.exp2(rng.uniform(-14, 9.5, 4000))
    sgn = np.where(rng.random(4000) < 0.5, -1.0, 1.0)
    v = (mags * sgn).astype(np.float32)
    vals = o.e4m3_decode(np.arange(127, dtype=np.uint8)).astype(np.float64)
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)     # exact in fp32
    edge = np.concatenate([mids, np.nextafter(mids, np.float32(0)),
                           np.nextafter(mids, np.float32(1e9)), -mids,
                           np.float32([0.0, -0.0, 1e-20, -1e-20, 500.0, -1e9])])
    v = np.concatenate([v, edge]).astype(np.float32)
    assert np.array_equal(o.e4m3_encode(v), _e4m3_brute(v))


def test_e4m3_encode_matches_torch_cast_in_range():
    rng = np.random.default_rng(4)
    v = (rng.normal(0, 1, 50000) * np.exp2(rng.uniform(-12, 8, 50000))).astype(np.float32)
    v = v[np.abs(v) < 464.0]
    want = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(o.e4m3_encode(v), want)


# ---------------------------------------------------------- double quant -----
def test_dq_sum_order_against_fsum():
    rng = np.random.default_rng(5)
    a = np.abs(rng.normal(0, 0.05, 300001)).astype(np.float32)
    s = o.dq_absmax_sum(a)
    assert s == pytest.approx(math.fsum(a.astype(np.float64)), rel=1e-13)
    ints = rng.integers(0, 1000, 70000).astype(np.float32)     # every partial sum exact
    assert o.dq_absmax_sum(ints) == float(ints.astype(np.int64).sum())


def test_dq_reconstruction_bound_and_constant_case():
    rng = np.random.default_rng(6)
    w = rng.normal(0, 0.02, 256 * 64 * 9 + 64 * 17 + 5).astype(np.float32)
    w[rng.choice(w.size, 40, replace=False)] = 0.2
    qd = o.quantize(w, o.MODE_DQ_FP8)
    a = qd["absmax"].astype(np.float64)
    c = o.block_scales(qd).astype(np.float64)
    mu = float(qd["dq_mean"])
    assert mu == pytest.approx(a.mean(), rel=1e-6)
    s2 = np.repeat(qd["dq_scale"].astype(np.float64), 256)[: a.size]
    d = a - mu
    # E4M3 keeps 3 mantissa bits: half an ulp is <= |v| / 16 (normal) or 2^-10 (subnormal)
    bound = np.maximum(np.abs(d) / 16.0, s2 * 2.0 ** -10) + 4 * np.spacing(np.float32(np.abs(a).max()))
    assert np.all(np.abs(c - a) <= bound)
    # the block holding max|d| reconstructs through q = +-448
    q = qd["scale_fp8"]
    for j in range(qd["dq_scale"].size):
        blk = q[j * 256:(j + 1) * 256]
        assert np.any((blk & 0x7F) == 0x7E)
    # all-equal absmax: zero deviations, s2 = 1, q = 0, scales reproduce exactly
    flat = np.tile(np.float32([0.5] + [0.25] * 63), 300)
    qc = o.quantize(flat, o.MODE_DQ_FP8)
    assert np.all(qc["scale_fp8"] == 0) and np.all(qc["dq_scale"] == 1.0)
    assert qc["dq_mean"] == np.float32(0.5)
    assert np.all(o.block_scales(qc) == np.float32(0.5))


# ----------------------------------------------------- grid round trips ------
@pytest.mark.parametrize("mode", [o.MODE_BF16, o.MODE_DQ_FP8])
def test_weights_on_the_grid_roundtrip_exactly(mode):
    rng = np.random.default_rng(7)
    L = o.nf4_levels()
    nblk = 256 * 3
    codes = rng.integers(0, 16, (nblk, 64)).astype(np.uint8)
    codes[:, 0] = 15                               # absmax = scale exactly
    scale = np.float32(0.5) if mode == o.MODE_DQ_FP8 else np.exp2(rng.integers(-8, 2, nblk)).astype(np.float32)
    w = (L[codes] * (scale if np.ndim(scale) == 0 else scale[:, None])).astype(np.float32)
    qw = o.quantize(w.reshape(-1), mode)
    assert np.array_equal(o.unpack_nibbles(qw["codes"], w.size), codes.reshape(-1))
    deq = o.bf16_to_f32(o.dequantize(qw))
    assert np.array_equal(deq, o.bf16_to_f32(o.bf16_bits(w.reshape(-1))))


def test_packing_nibble_order_and_tails():
    codes = np.array([1, 2, 3, 4, 15, 0, 9], dtype=np.uint8)
    packed = o.pack_nibbles(codes)
    assert packed.tolist() == [0x21, 0x43, 0x0F, 0x09]
    assert np.array_equal(o.unpack_nibbles(packed, 7), codes)


def test_partial_and_zero_blocks():
    rng = np.random.default_rng(8)
    w = rng.normal(0, 0.02, 64 * 3 + 10).astype(np.float32)
    w[64:128] = 0.0
    qw = o.quantize(w, o.MODE_BF16)
    assert qw["absmax"].size == 4
    assert qw["absmax"][3] == np.abs(w[192:]).max()
    codes = o.unpack_nibbles(qw["codes"], w.size)
    assert np.all(codes[64:128] == 7) and qw["absmax"][1] == 0.0
    deq = o.bf16_to_f32(o.dequantize(qw))
    assert np.all(deq[64:128] == 0.0)
    assert qw["codes"].size == (w.size + 1) // 2


# ---------------------------------------------------------- the layer --------
def _loops_forward(Wd, X, A, B, alpha):
    M, K = X.shape
    N, r = B.shape
    s = alpha / r
    Y = np.zeros((M, N))
    for i in range(M):
        u = [sum(X[i, k] * A[j, k] for k in range(K)) for j in range(r)]
        for n in range(N):
            Y[i, n] = sum(X[i, k] * Wd[n, k] for k in range(K)) + s * sum(u[j] * B[n, j] for j in range(r))
    return Y


def _tiny_layer(seed=9, M=4, N=6, K=64, r=2):
    rng = np.random.default_rng(seed)
    w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    Wd = o.dequantize_f64(o.quantize(w, o.MODE_DQ_FP8), (N, K))
    X = rng.normal(0, 1, (M, K))
    A = rng.normal(0, 1.0 / r, (r, K))
    B = rng.normal(0, 0.01, (N, r))
    dY = rng.normal(0, 1, (M, N))
    return Wd, X, A, B, dY


def test_forward_against_python_loops():
    Wd, X, A, B, _ = _tiny_layer()
    Y, U = o.linear_forward(Wd, X, A, B, alpha=16.0)
    np.testing.assert_allclose(Y, _loops_forward(Wd, X, A, B, 16.0), rtol=1e-12, atol=1e-12)
    Yr, _ = o.linear_forward(Wd, X, A, B, alpha=16.0, rows=[1, 3])
    np.testing.assert_allclose(Yr, Y[[1, 3]], rtol=0, atol=1e-13)


def test_backward_against_finite_differences():
    Wd, X, A, B, dY = _tiny_layer(M=3, N=5, K=64, r=2)
    alpha = 16.0

    def loss(X_, A_, B_):
        Y, _ = o.linear_forward(Wd, X_, A_, B_, alpha)
        return float(np.sum(Y * dY))

    dX, dA, dB = o.linear_backward(Wd, X, dY, A, B, alpha)
    h = 1e-4
    for name, T, G in (("X", X, dX), ("A", A, dA), ("B", B, dB)):
        num = np.zeros_like(T)
        for idx in np.ndindex(T.shape):
            Tp, Tm = T.copy(), T.copy()
            Tp[idx] += h
            Tm[idx] -= h
            if name == "X":
                num[idx] = (loss(Tp, A, B) - loss(Tm, A, B)) / (2 * h)
            elif name == "A":
                num[idx] = (loss(X, Tp, B) - loss(X, Tm, B)) / (2 * h)
            else:
                num[idx] = (loss(X, A, Tp) - loss(X, A, Tm)) / (2 * h)
        np.testing.assert_allclose(G, num, rtol=1e-6, atol=1e-8, err_msg=name)
    dXr, _, _ = o.linear_backward(Wd, X, dY, A, B, alpha, dx_rows=[0, 2])
    np.testing.assert_allclose(dXr, dX[[0, 2]], rtol=0, atol=1e-13)


def test_layer_special_cases():
    Wd, X, A, B, dY = _tiny_layer(M=5, N=7, K=128, r=4)
    Y, _ = o.linear_forward(Wd, X, A, np.zeros_like(B), alpha=16.0)
    np.testing.assert_allclose(Y, X @ Wd.T, rtol=1e-13, atol=1e-13)          # no adapter: plain linear
    _, dA, dB = o.linear_backward(Wd, X, dY, np.zeros_like(A), B, alpha=16.0)
    assert np.all(dB == 0)                                                    # U = 0 -> dB = 0
    Y0, _ = o.linear_forward(np.zeros_like(Wd), X, A, B, alpha=16.0)
    np.testing.assert_allclose(Y0, (16.0 / 4) * X @ A.T @ B.T, rtol=1e-12)   # base of zeros


def test_silu_gate_against_finite_differences():
    rng = np.random.default_rng(10)
    g, u, dh = rng.normal(0, 2, 50), rng.normal(0, 1, 50), rng.normal(0, 1, 50)
    h = o.silu_gate_forward(g, u)
    np.testing.assert_allclose(h, g / (1 + np.exp(-g)) * u, rtol=1e-14)
    dg, du = o.silu_gate_backward(dh, g, u)
    eps = 1e-6
    num_g = (o.silu_gate_forward(g + eps, u) - o.silu_gate_forward(g - eps, u)) / (2 * eps) * dh
    num_u = (o.silu_gate_forward(g, u + eps) - o.silu_gate_forward(g, u - eps)) / (2 * eps) * dh
    np.testing.assert_allclose(dg, num_g, rtol=1e-6, atol=1e-9)
    np.testing.assert_allclose(du, num_u, rtol=1e-6, atol=1e-9)


def test_lora_merge_against_python_loops_and_the_layer():
    # W_merged = W' + (alpha/r) B A ("Price 2: deployment friction": merge onto a dequantized copy)
    Wd, X, A, B, _ = _tiny_layer(M=6, N=5, K=64, r=3)
    alpha = 16.0
    Wm = o.lora_merge(Wd, A, B, alpha)
    s = alpha / 3
    for i in range(5):
        for j in range(64):
            acc = float(Wd[i, j])
            for t in range(3):
                acc += s * float(B[i, t]) * float(A[t, j])
            assert abs(Wm[i, j] - acc) <= 1e-15 * (1 + abs(acc)), (i, j)
    # the merged weight reproduces the adapted layer's output
    Y, _ = o.linear_forward(Wd, X, A, B, alpha)
    np.testing.assert_allclose(X @ Wm.T, Y, rtol=1e-12, atol=1e-13)
    # a freshly initialised adapter (B = 0) leaves the dequantized weight unchanged
    assert np.array_equal(o.lora_merge(Wd, A, np.zeros_like(B), alpha), Wd)
    # the update has rank at most r
    sv = np.linalg.svd(Wm - Wd, compute_uv=False)
    assert np.all(sv[3:] <= 1e-12 * sv[0])


# ---------------------------------------------------------------- LoRA dropout
def test_philox_known_answer_vectors():
    # the generator's authors' published vectors pin the whole bit stream: a swapped
    # word, a wrong multiplier or a missing key bump changes every output word
    rows = []
    for line in open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            rows.append([int(t, 16) for t in line.split()])
    assert len(rows) == 3
    for v in rows:
        ctr, key, want = v[0:4], v[4:6], v[6:10]
        got = o.philox4x32_10(*ctr, *key)
        assert [int(g) for g in got] == want, [hex(int(g)) for g in got]
    # vectorised over many counters: every lane equals the scalar call
    c0 = np.array([rows[0][0], rows[1][0], rows[2][0]], dtype=np.uint64)
    cs = [np.array([r[i] for r in rows], dtype=np.uint64) for i in range(1, 6)]
    got = o.philox4x32_10(c0, *cs)
    for j, r in enumerate(rows):
        assert [int(g[j]) for g in got] == r[6:10]


def test_dropout_keep_rate_and_uniformity():
    # reading 10: 16-bit values uniform on [0, 65536); kept iff >= round(p * 65536)
    n = 1 << 22
    r = o.dropout_random16(n, seed=20231, offset=5)
    assert r.min() >= 0 and r.max() <= 0xFFFF
    hist = np.bincount((r >> 8).astype(np.int64), minlength=256)
    expect = n / 256.0
    chi2 = float(np.sum((hist - expect) ** 2 / expect))
    assert chi2 < 255 + 6 * np.sqrt(2 * 255), chi2            # 255 dof, ~6 sigma
    for lane in range(8):                                       # every 16-bit lane of the 4 words is used alike
        mu = r[lane::8].mean()
        assert abs(mu - 32767.5) < 6 * 18918.0 / np.sqrt(n / 8), (lane, mu)
    p = 0.05
    keep = (r >= o.dropout_threshold(p)).mean()
    q = o.dropout_threshold(p) / 65536.0
    assert abs(keep - (1 - q)) < 6 * np.sqrt(q * (1 - q) / n), keep
    assert o.dropout_threshold(p) == 3277 and abs(o.dropout_keep_scale(p) - 65536 / 62259) < 1e-15


def test_dropout_streams_are_independent():
    m, k, p = 512, 1024, 0.05
    a = o.dropout_mask(m, k, p, seed=1, offset=0)
    for other in (o.dropout_mask(m, k, p, seed=2, offset=0), o.dropout_mask(m, k, p, seed=1, offset=1)):
        diff = np.mean(a != other)
        q = o.dropout_threshold(p) / 65536.0
        assert abs(diff - 2 * q * (1 - q)) < 0.01, diff           # independent masks disagree at rate 2q(1-q)
    # neighbouring elements (same Philox call, and across calls) are uncorrelated
    x = a.reshape(-1).astype(np.float64)
    for lag in (1, 2, 7, 8, 9):
        c = np.corrcoef(x[:-lag], x[lag:])[0, 1]
        assert abs(c) < 0.01, (lag, c)
    assert np.array_equal(a, o.dropout_mask(m, k, p, seed=1, offset=0))   # deterministic in (seed, offset)


def test_dropout_zero_rate_is_the_plain_layer():
    Wd, X, A, B, dY = _tiny_layer(M=5, N=6, K=128, r=4)
    mask = o.dropout_mask(5, 128, 0.0, seed=3, offset=0)
    assert mask.all() and o.dropout_keep_scale(0.0) == 1.0
    Y, U = o.linear_forward(Wd, X, A, B, 16.0)
    Yd, Ud = o.linear_forward_dropout(Wd, X, A, B, 16.0, mask, 0.0)
    assert np.array_equal(Y, Yd) and np.array_equal(U, Ud)
    g = o.linear_backward(Wd, X, dY, A, B, 16.0)
    gd = o.linear_backward_dropout(Wd, X, dY, A, B, 16.0, mask, 0.0)
    for a, b in zip(g, gd):
        np.testing.assert_allclose(a, b, rtol=1e-14, atol=1e-15)


def test_dropout_layer_against_loops_and_finite_differences():
    Wd, X, A, B, dY = _tiny_layer(M=4, N=6, K=64, r=2)
    p = 0.3
    mask = o.dropout_mask(4, 64, p, seed=11, offset=2)
    assert 0 < mask.mean() < 1
    c = 65536.0 / (65536.0 - round(p * 65536))
    Y, _ = o.linear_forward_dropout(Wd, X, A, B, 16.0, mask, p)
    s = 16.0 / 2
    for i in range(4):                                            # Python loops over the definition
        for j in range(6):
            base = sum(float(X[i, t]) * float(Wd[j, t]) for t in range(64))
            low = 0.0
            for q in range(2):
                u = c * sum(float(X[i, t]) * float(mask[i, t]) * float(A[q, t]) for t in range(64))
                low += u * float(B[j, q])
            assert abs(Y[i, j] - (base + s * low)) < 1e-12 * (1 + abs(Y[i, j]))

    def loss(Xv, Av, Bv):
        return float(np.sum(o.linear_forward_dropout(Wd, Xv, Av, Bv, 16.0, mask, p)[0] * dY))

    dX, dA, dB = o.linear_backward_dropout(Wd, X, dY, A, B, 16.0, mask, p)
    h = 1e-4
    for name, T, G in (("X", X, dX), ("A", A, dA), ("B", B, dB)):
        num = np.zeros_like(T)
        for idx in np.ndindex(T.shape):
            Tp, Tm = T.copy(), T.copy()
            Tp[idx] += h
            Tm[idx] -= h
            args_p = {"X": (Tp, A, B), "A": (X, Tp, B), "B": (X, A, Tp)}[name]
            args_m = {"X": (Tm, A, B), "A": (X, Tm, B), "B": (X, A, Tm)}[name]
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        np.testing.assert_allclose(G, num, rtol=1e-6, atol=1e-8, err_msg=name)


def test_mask_bit_packing_order():
    mask = np.zeros((2, 16), dtype=bool)
    mask[0, 0] = mask[0, 9] = mask[1, 15] = True
    assert o.pack_mask_bits(mask).tolist() == [0x01, 0x02, 0x00, 0x80]


# ------------------------------------------------------------------- AdamW
def test_adamw_first_step_is_a_sign_step():
    # with zero moments the bias-corrected first step is lr * g / (|g| + eps): a sign step for |g| >> eps
    rng = np.random.default_rng(21)
    p0, g = rng.normal(0, 1, 1000), rng.normal(0, 1e-2, 1000)
    p1, m1, v1 = o.adamw_step(p0, g, np.zeros(1000), np.zeros(1000), step=1, lr=2e-4, eps=1e-8)
    np.testing.assert_allclose(p1, p0 - 2e-4 * g / (np.abs(g) + 1e-8), rtol=0, atol=1e-15)
    np.testing.assert_allclose(m1, 0.1 * g, rtol=1e-15)
    np.testing.assert_allclose(v1, 0.001 * g * g, rtol=1e-12)


def test_adamw_constant_gradient_closed_form():
    # a constant gradient keeps the bias-corrected moments at g and g^2 for every t, so each step
    # moves by lr * g / (|g| + eps); with weight decay the parameter follows a geometric recursion
    g, lr, wd, eps, T = np.array([3e-3, -2e-2, 5e-1]), 1e-3, 0.01, 1e-8, 25
    p = np.array([0.5, -1.0, 2.0])
    m = np.zeros(3)
    v = np.zeros(3)
    for t in range(1, T + 1):
        p, m, v = o.adamw_step(p, g, m, v, step=t, lr=lr, weight_decay=wd, eps=eps)
    u = lr * g / (np.abs(g) + eps)
    a = 1 - lr * wd
    want = np.array([0.5, -1.0, 2.0]) * a ** T - u * (1 - a ** T) / (1 - a)
    np.testing.assert_allclose(p, want, rtol=1e-10)


def test_adamw_zero_gradient_only_decays():
    p0 = np.array([1.0, -2.0, 0.25])
    p1, m1, v1 = o.adamw_step(p0, np.zeros(3), np.zeros(3), np.zeros(3), step=3, lr=0.1, weight_decay=0.5)
    np.testing.assert_allclose(p1, p0 * (1 - 0.05), rtol=1e-15)
    assert np.all(m1 == 0) and np.all(v1 == 0)
    # grad_scale multiplies the gradient before anything else
    a = o.adamw_step(p0, np.full(3, 2.0), np.zeros(3), np.zeros(3), step=1, lr=0.1, grad_scale=0.5)
    b = o.adamw_step(p0, np.full(3, 1.0), np.zeros(3), np.zeros(3), step=1, lr=0.1)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


# ----------------------------------------------------------- error metrics ---
def test_error_metrics_hand_computed():
    # 2 x 2 case worked by hand: ref = [[3, 0], [0, 4]] has Frobenius norm 5 and
    # RMS sqrt(25 / 4) = 2.5; got differs by +1 at (0, 0) and -2 at (1, 1), so the
    # error has Frobenius norm sqrt(5) and largest magnitude 2.
    ref = np.array([[3.0, 0.0], [0.0, 4.0]])
    got = np.array([[4.0, 0.0], [0.0, 2.0]])
    assert o.rel_frobenius(got, ref) == pytest.approx(math.sqrt(5.0) / 5.0, rel=1e-15)
    assert o.max_abs_over_rms(got, ref) == pytest.approx(2.0 / 2.5, rel=1e-15)
    # identical inputs give exactly zero; a scaled copy gives the scale error
    assert o.rel_frobenius(ref, ref) == 0.0 and o.max_abs_over_rms(ref, ref) == 0.0
    assert o.rel_frobenius(1.5 * ref, ref) == pytest.approx(0.5, rel=1e-15)
    # torch tensors (as the smoke check passes them) give the same numbers
    assert o.rel_frobenius(torch.tensor(got), torch.tensor(ref)) == pytest.approx(math.sqrt(5.0) / 5.0, rel=1e-15)
