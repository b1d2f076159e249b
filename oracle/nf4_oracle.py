"""CPU oracle for the QLoRA frozen-base linear layer (NF4 + double quantization).

TEST INFRASTRUCTURE ONLY. This module defines what the CUDA library must
compute, in plain numpy (fp32 where the format fixes fp32, fp64 for every
matmul). Only the tests, the smoke check in ``__graft_entry__`` and the CPU
baseline leg of ``bench.py`` may import it. It shares no code, constant or
table generator with the CUDA path, and the CUDA path never calls it.

Sources (web pages on QLoRA; cited by title and section):

* [CSD] "QLoRA: Quantized Low-Rank Adaptation" (completesystemdesign.dev):
  Piece 1 (storage: 16-level menu, half a byte per weight, quantized once),
  Piece 2 (compute: blocks of 64 dequantized to BF16 right before the
  multiply), Piece 3 (learning: only the adapter receives gradients),
  the one-block worked example, "NF4: a 4-bit format matched to weight
  statistics", "Double quantization (the label-index-card trick)",
  "Batched 4-bit matmuls".
* [GAMUT] "QLoRA Explained: Fine-Tune 70B+ LLMs on a Single GPU": sections
  "4-Bit NormalFloat (NF4) Quantization" and "Double Quantization".
* [QT] "What is QLoRA?" (qubittool glossary): Key Characteristics
  (backpropagation through quantized weights; adapters in full precision).

Readings taken where the pages are silent or garbled (each is listed in the
design notes of the repository):

1. Levels: the pages say 16 levels at quantiles of a normal distribution
   ([CSD] NF4 section, [GAMUT] NF4 section), with an exact zero and
   normalisation to [-1, 1] (the format's definition here). We take the asymmetric quantile
   construction of the NF4 paper: 8 positive quantiles Phi^-1(p) at p
   equally spaced from delta down to 1/2 (9 points, 1/2 dropped), 7
   negative ones built the same way on 8 points, plus an exact 0, all
   divided by the largest; delta = ((1 - 1/30) + (1 - 1/32)) / 2 keeps the
   outermost quantile finite.
2. Nearest level by fp32 midpoints m_i = fp32(fp32(L_i + L_{i+1}) * 0.5);
   code(x) = #{i : x > m_i}, so a value exactly on a midpoint takes the
   lower level.
3. Normalisation x = fp32(w * fp32(1 / absmax)); a block whose absmax is
   zero or subnormal gets code 7 (the exact zero) everywhere.
4. Packing: byte j holds element 2j in its low nibble and 2j+1 in its high
   nibble; an odd tail leaves the high nibble 0.
5. Plain scale: bf16 (round to nearest even) of the fp32 absmax ([CSD]
   worked example, where each block keeps a single BF16 scale).
6. Double quantization ([CSD] DQ section: the scales become 8-bit floats
   in blocks; the block of 256, the fp32 second-level scale and the mean
   offset are the format's definition here, the pages leaving them open): mu = fp32(S / nblk) with S the fp64 sum of all absmax
   values in a fixed pairwise order; per 256-block d = fp32(a - mu),
   s2 = fp32(max|d| / 448) (1 if max|d| = 0), q = E4M3(fp32(d / s2)) with
   round-to-nearest-even and saturation to +-448 (OCP E4M3, the FP8 whose
   largest normal is 448).
7. Dequantization ([CSD] Piece 2): c = plain ? f32(scale) :
   fp32(fp32(f32(q) * s2) + mu); w' = bf16(fp32(L[code] * c)).
8. Layer: Y = X W'^T + (alpha/r) (X A^T) B^T; backward dX = dY W' +
   (alpha/r)(dY B) A, dB = (alpha/r) dY^T (X A^T), dA = (alpha/r)(dY B)^T X.
   No gradient for W' ([CSD] Piece 3: the quantized base is frozen).
9. Adapter merge ([CSD] "Price 2: deployment friction": the adapter is
   merged onto a dequantized BF16 copy, since a 4-bit matrix cannot absorb
   it; [GAMUT] Step 5 "Save and Merge Adapters"; "QLoRA vs LoRA" FAQ on
   converting back to full precision, FP16 or FP32, and quantizing again
   for deployment): W_merged = W' + (alpha/r) B A, exact in fp64 here; the
   stored BF16 or FP32 copy is that value rounded once (checked by the
   tests with the bound their docstrings derive).
10. LoRA dropout ([GAMUT] Step 3, LoraConfig lora_dropout=0.05, and the
   hyperparameter quick reference; the pages give only the rate): inverted
   dropout on the input of the low-rank branch, as PEFT applies it. With a
   keep mask M and keep scale c = 1/(1 - p): Y = X W'^T + s (c (M*X) A^T) B^T;
   dA = s c (dY B)^T (M*X); dX = dY W' + s c ((dY B) A) * M; dB = s dY^T U
   with U = c (M*X) A^T. The mask is drawn from Philox4x32-10 (Salmon et al.,
   "Parallel Random Numbers: As Easy as 1, 2, 3", SC 2011), counter =
   (e // 8 as two 32-bit words, offset as two 32-bit words), key = seed as
   two 32-bit words; element e (row-major index into X) takes 16-bit lane
   e % 8 of the four output words (word (e % 8) // 2, low half first) and is
   kept iff that value >= round(p * 65536). The effective drop rate is
   round(p * 65536) / 65536 and c = 65536 / (65536 - round(p * 65536)).
11. Paged AdamW, 32-bit ([GAMUT] "Paged Optimizers" and the hyperparameter
   reference, optim="paged_adamw_32bit"; [CSD] "Paged optimizers (the
   storage unit)"): AdamW with decoupled weight decay (Loshchilov and Hutter)
   on fp32 master weights of the adapters with fp32 moment estimates:
   g = grad * grad_scale; m = b1 m + (1 - b1) g; v = b2 v + (1 - b2) g^2;
   p = p (1 - lr wd) - (lr / (1 - b1^t)) m / (sqrt(v) / sqrt(1 - b2^t) + eps).
   "Paged" is where the states live (unified memory that may spill to host
   RAM), not a change to the arithmetic.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import ndtri

BLOCKSIZE = 64          # [CSD] Piece 2 and NF4 section: blocks of 64 weights
DQ_BLOCKSIZE = 256      # second-level block (the format's definition; the pages leave it open)
E4M3_MAX = 448.0        # largest finite OCP E4M3 value
FLT_MIN = np.float32(np.finfo(np.float32).tiny)

MODE_BF16 = 0
MODE_DQ_FP8 = 1


# ----------------------------------------------------------------------------
# bf16 helpers (round to nearest even)
# ----------------------------------------------------------------------------
def bf16_bits(x) -> np.ndarray:
    """Round fp32 values to bf16, nearest-even; returns the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bias = np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    return ((u + bias) >> np.uint64(16)).astype(np.uint16)


def bf16_to_f32(bits) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32)


# ----------------------------------------------------------------------------
# NF4 levels and midpoints  ([CSD] NF4 section; [GAMUT] NF4 section)
# ----------------------------------------------------------------------------
NF4_DELTA = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0))


def nf4_levels_f64() -> np.ndarray:
    """The 16 NF4 levels in fp64, ascending, before rounding to fp32."""
    pos = ndtri(np.linspace(NF4_DELTA, 0.5, 9)[:-1])        # 8 positive quantiles
    neg = -ndtri(np.linspace(NF4_DELTA, 0.5, 8)[:-1])       # 7 negative quantiles
    v = np.sort(np.concatenate([pos, [0.0], neg]))
    return v / v.max()


def nf4_levels() -> np.ndarray:
    """The 16 NF4 levels as fp32 (the values a code dequantizes to)."""
    return nf4_levels_f64().astype(np.float32)


def nf4_midpoints(levels=None) -> np.ndarray:
    """fp32 decision thresholds between neighbouring levels."""
    L = nf4_levels() if levels is None else np.asarray(levels, dtype=np.float32)
    return ((L[:-1] + L[1:]) * np.float32(0.5)).astype(np.float32)


# ----------------------------------------------------------------------------
# First level: blockwise absmax NF4  ([CSD] Piece 1, worked example, NF4 section)
# ----------------------------------------------------------------------------
def _blocks(w_flat: np.ndarray, blocksize: int) -> np.ndarray:
    n = w_flat.size
    nblk = -(-n // blocksize)
    padded = np.zeros(nblk * blocksize, dtype=np.float32)
    padded[:n] = w_flat
    return padded.reshape(nblk, blocksize)


def block_absmax(w, blocksize: int = BLOCKSIZE) -> np.ndarray:
    """fp32 max |w| over each block of `blocksize` consecutive elements.

    A partial last block uses only its present elements (zero padding cannot
    raise a maximum of absolute values)."""
    w = np.ascontiguousarray(w, dtype=np.float32).reshape(-1)
    return np.abs(_blocks(w, blocksize)).max(axis=1).astype(np.float32)


def nf4_code_of(x) -> np.ndarray:
    """Code of already-normalised fp32 values: the number of midpoints below x."""
    x = np.asarray(x, dtype=np.float32)
    codes = np.zeros(x.shape, dtype=np.uint8)
    for m in nf4_midpoints():
        codes += (x > m)
    return codes


def nf4_codes(w, blocksize: int = BLOCKSIZE) -> np.ndarray:
    """One NF4 code (0..15) per element: nearest level of w / absmax."""
    w = np.ascontiguousarray(w, dtype=np.float32).reshape(-1)
    n = w.size
    blocks = _blocks(w, blocksize)
    absmax = np.abs(blocks).max(axis=1).astype(np.float32)
    degenerate = absmax < FLT_MIN
    inv = (np.float32(1.0) / np.where(degenerate, np.float32(1.0), absmax)).astype(np.float32)
    x = (blocks * inv[:, None]).astype(np.float32)
    codes = nf4_code_of(x)
    codes[degenerate, :] = 7
    return codes.reshape(-1)[:n]


def pack_nibbles(codes) -> np.ndarray:
    """Two 4-bit codes per byte: element 2j low nibble, 2j+1 high nibble."""
    c = np.ascontiguousarray(codes, dtype=np.uint8).reshape(-1)
    if c.size % 2:
        c = np.concatenate([c, np.zeros(1, dtype=np.uint8)])
    return (c[0::2] | (c[1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed, n: int) -> np.ndarray:
    p = np.ascontiguousarray(packed, dtype=np.uint8).reshape(-1)
    out = np.empty(p.size * 2, dtype=np.uint8)
    out[0::2] = p & 0x0F
    out[1::2] = p >> 4
    return out[:n]


# ----------------------------------------------------------------------------
# OCP E4M3 (the FP8 of the double quantization)
# ----------------------------------------------------------------------------
def e4m3_decode(code) -> np.ndarray:
    """Exact fp32 value of E4M3 bytes (bias 7, no infinities, S.1111.111 = NaN)."""
    c = np.asarray(code, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return (sign * mag).astype(np.float32)


_E4M3_POS = e4m3_decode(np.arange(0x7F, dtype=np.uint8)).astype(np.float64)  # codes 0..126


def e4m3_encode(v) -> np.ndarray:
    """fp32 -> E4M3 byte: nearest finite value, ties to even mantissa,
    magnitudes above 448 saturate to 448; the sign bit is the input's sign
    (so a negative value that rounds to zero gives 0x80)."""
    v = np.ascontiguousarray(v, dtype=np.float32).reshape(-1)
    a = np.abs(v).astype(np.float64)
    hi = np.searchsorted(_E4M3_POS, a, side="left")
    hi = np.clip(hi, 1, 126)
    lo = hi - 1
    d_lo = a - _E4M3_POS[lo]
    d_hi = _E4M3_POS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(a >= E4M3_MAX, 126, code)
    code = np.where(a <= 0.0, 0, code)
    code = code | np.where(np.signbit(v), 0x80, 0)
    return code.astype(np.uint8)


# ----------------------------------------------------------------------------
# Second level: double quantization of the absmax constants
# ([CSD] "Double quantization (the label-index-card trick)"; [GAMUT] DQ)
# ----------------------------------------------------------------------------
def dq_absmax_sum(absmax) -> float:
    """fp64 sum of all absmax values in a fixed pairwise order: first a
    pairwise tree inside each 256-block (zero padded to 256), then a pairwise
    tree over the block sums in index order (zero padded to a power of two).
    The order is part of the format, so the mean is reproducible bit for bit."""
    v = np.asarray(absmax, dtype=np.float32).astype(np.float64).reshape(-1)
    nb2 = -(-v.size // DQ_BLOCKSIZE)
    t = np.zeros(nb2 * DQ_BLOCKSIZE, dtype=np.float64)
    t[: v.size] = v
    t = t.reshape(nb2, DQ_BLOCKSIZE)
    while t.shape[1] > 1:
        t = t[:, 0::2] + t[:, 1::2]
    s = t[:, 0]
    p = 1
    while p < s.size:
        p *= 2
    s = np.concatenate([s, np.zeros(p - s.size)])
    while s.size > 1:
        s = s[0::2] + s[1::2]
    return float(s[0])


def double_quantize(absmax):
    """Returns (q uint8 [nblk], s2 fp32 [nblk2], mu fp32)."""
    a = np.asarray(absmax, dtype=np.float32).reshape(-1)
    nblk = a.size
    mu = np.float32(dq_absmax_sum(a) / float(nblk))
    d = (a - mu).astype(np.float32)
    nb2 = -(-nblk // DQ_BLOCKSIZE)
    q = np.empty(nblk, dtype=np.uint8)
    s2 = np.empty(nb2, dtype=np.float32)
    for j in range(nb2):
        dj = d[j * DQ_BLOCKSIZE:(j + 1) * DQ_BLOCKSIZE]
        amax = np.float32(np.abs(dj).max())
        sj = np.float32(1.0) if amax == 0 else np.float32(amax / np.float32(E4M3_MAX))
        s2[j] = sj
        q[j * DQ_BLOCKSIZE:(j + 1) * DQ_BLOCKSIZE] = e4m3_encode((dj / sj).astype(np.float32))
    return q, s2, mu


# ----------------------------------------------------------------------------
# Whole-tensor quantize / dequantize
# ----------------------------------------------------------------------------
def quantize(W, mode: int = MODE_DQ_FP8, blocksize: int = BLOCKSIZE) -> dict:
    """NF4-quantize a row-major weight matrix (or any flat array).

    Returns a dict with 'codes' (packed uint8), 'n_elem', 'mode' and either
    'scale_bf16' (uint16 per block) or 'scale_fp8' (uint8 per block),
    'dq_scale' (fp32 per 256 blocks) and 'dq_mean' (fp32 scalar)."""
    w = np.ascontiguousarray(W, dtype=np.float32).reshape(-1)
    absmax = block_absmax(w, blocksize)
    out = {"codes": pack_nibbles(nf4_codes(w, blocksize)), "n_elem": w.size, "mode": mode,
           "absmax": absmax}
    if mode == MODE_BF16:
        out["scale_bf16"] = bf16_bits(absmax)
    elif mode == MODE_DQ_FP8:
        q, s2, mu = double_quantize(absmax)
        out["scale_fp8"], out["dq_scale"], out["dq_mean"] = q, s2, mu
    else:
        raise ValueError("unknown scale mode")
    return out


def block_scales(qw: dict) -> np.ndarray:
    """The fp32 scale c each block dequantizes with."""
    if qw["mode"] == MODE_BF16:
        return bf16_to_f32(qw["scale_bf16"])
    q = e4m3_decode(qw["scale_fp8"])
    s2 = np.repeat(qw["dq_scale"], DQ_BLOCKSIZE)[: q.size]
    return ((q * s2).astype(np.float32) + np.float32(qw["dq_mean"])).astype(np.float32)


def dequantize(qw: dict, blocksize: int = BLOCKSIZE) -> np.ndarray:
    """bf16 bit patterns of w' = bf16(fp32(L[code] * c)), flat, length n_elem."""
    n = qw["n_elem"]
    codes = unpack_nibbles(qw["codes"], n)
    c = np.repeat(block_scales(qw), blocksize)[:n]
    vals = (nf4_levels()[codes] * c).astype(np.float32)
    return bf16_bits(vals)


def dequantize_f64(qw: dict, shape) -> np.ndarray:
    return bf16_to_f32(dequantize(qw)).astype(np.float64).reshape(shape)


# ----------------------------------------------------------------------------
# The frozen-base linear layer with its low-rank branch (fp64)
# ([CSD] Piece 2 and Piece 3, which keep the LoRA math unchanged; the formula is
# the standard LoRA one with scale alpha / r)
# ----------------------------------------------------------------------------
def _f64(t) -> np.ndarray:
    """bf16/fp32 torch tensor or numpy array -> fp64 numpy (exact)."""
    if hasattr(t, "detach"):
        t = t.detach().to("cpu")
        import torch
        if t.dtype == torch.bfloat16:
            t = t.to(torch.float32)
        t = t.numpy()
    return np.asarray(t, dtype=np.float64)


def linear_forward(Wd, X, A, B, alpha: float, rows=None):
    """Y = X W'^T + (alpha/r) (X A^T) B^T in fp64; optional row subset of X.

    Returns (Y, U) with U = X A^T."""
    Wd, X, A, B = _f64(Wd), _f64(X), _f64(A), _f64(B)
    if rows is not None:
        X = X[np.asarray(rows)]
    s = float(alpha) / A.shape[0]
    U = X @ A.T
    Y = X @ Wd.T + s * (U @ B.T)
    return Y, U


def linear_backward(Wd, X, dY, A, B, alpha: float, dx_rows=None):
    """Gradients of the layer w.r.t. X, A and B (W' is frozen), fp64.

    dX = dY W' + s (dY B) A ; dB = s dY^T (X A^T) ; dA = s (dY B)^T X.
    `dx_rows` restricts dX to a subset of rows (dA, dB are always full)."""
    Wd, X, dY, A, B = _f64(Wd), _f64(X), _f64(dY), _f64(A), _f64(B)
    s = float(alpha) / A.shape[0]
    G = dY @ B
    U = X @ A.T
    dB = s * (dY.T @ U)
    dA = s * (G.T @ X)
    if dx_rows is not None:
        r_ = np.asarray(dx_rows)
        dX = dY[r_] @ Wd + s * (G[r_] @ A)
    else:
        dX = dY @ Wd + s * (G @ A)
    return dX, dA, dB


def lora_merge(Wd, A, B, alpha: float) -> np.ndarray:
    """W_merged = W' + (alpha/r) B A in fp64 (reading 9): the dense weight
    that makes the merged layer X W_merged^T equal the adapted layer."""
    Wd, A, B = _f64(Wd), _f64(A), _f64(B)
    s = float(alpha) / A.shape[0]
    return Wd + s * (B @ A)


# ----------------------------------------------------------------------------
# LoRA dropout (reading 10): Philox4x32-10 keep mask and the dropped layer
# ----------------------------------------------------------------------------
PHILOX_M0, PHILOX_M1 = 0xD2511F53, 0xCD9E8D57      # round multipliers
PHILOX_W0, PHILOX_W1 = 0x9E3779B9, 0xBB67AE85      # key increments (Weyl sequence)
M32 = 0xFFFFFFFF


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Philox4x32 with 10 rounds on uint64 numpy arrays holding 32-bit values:
    each round multiplies c0 and c2 by the two constants (64-bit products split
    into high and low words) and mixes the high words with c1, c3 and the key;
    the key advances by the Weyl increments between rounds."""
    c0, c1, c2, c3 = (np.asarray(v, dtype=np.uint64) & M32 for v in (c0, c1, c2, c3))
    k0 = np.asarray(k0, dtype=np.uint64) & M32
    k1 = np.asarray(k1, dtype=np.uint64) & M32
    for rnd in range(10):
        p0 = c0 * np.uint64(PHILOX_M0)
        p1 = c2 * np.uint64(PHILOX_M1)
        hi0, lo0 = p0 >> np.uint64(32), p0 & np.uint64(M32)
        hi1, lo1 = p1 >> np.uint64(32), p1 & np.uint64(M32)
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
        if rnd < 9:
            k0 = (k0 + np.uint64(PHILOX_W0)) & np.uint64(M32)
            k1 = (k1 + np.uint64(PHILOX_W1)) & np.uint64(M32)
    return c0, c1, c2, c3


def dropout_threshold(p: float) -> int:
    """16-bit drop threshold round(p * 65536); p must lie in [0, 1)."""
    t = int(round(float(p) * 65536.0))
    if not 0 <= t < 65536:
        raise ValueError("dropout rate must lie in [0, 1)")
    return t


def dropout_keep_scale(p: float) -> float:
    t = dropout_threshold(p)
    return 65536.0 / (65536.0 - t)


def dropout_random16(count: int, seed: int, offset: int) -> np.ndarray:
    """The 16-bit random value of each element e in [0, count)."""
    e = np.arange(count, dtype=np.uint64)
    g = e >> np.uint64(3)
    words = philox4x32_10(g & np.uint64(M32), g >> np.uint64(32), offset & M32, (offset >> 32) & M32,
                          seed & M32, (seed >> 32) & M32)
    lane = (e & np.uint64(7)).astype(np.int64)
    w = np.choose(lane >> 1, words)
    return ((w >> ((lane & 1) * 16).astype(np.uint64)) & np.uint64(0xFFFF)).astype(np.uint32)


def dropout_mask(m: int, k: int, p: float, seed: int, offset: int) -> np.ndarray:
    """Boolean keep mask [m, k] of reading 10."""
    return (dropout_random16(m * k, seed, offset) >= dropout_threshold(p)).reshape(m, k)


def pack_mask_bits(mask) -> np.ndarray:
    """Row-major bit packing: element e -> bit e % 8 of byte e // 8."""
    return np.packbits(np.asarray(mask, dtype=np.uint8).reshape(-1), bitorder="little")


def linear_forward_dropout(Wd, X, A, B, alpha: float, mask, p: float, rows=None):
    """Y and U of the layer with dropout on the low-rank input (reading 10)."""
    c = dropout_keep_scale(p)
    Wd, X, A, B = _f64(Wd), _f64(X), _f64(A), _f64(B)
    Xm = X * np.asarray(mask, dtype=np.float64)
    if rows is not None:
        X, Xm = X[np.asarray(rows)], Xm[np.asarray(rows)]
    s = float(alpha) / A.shape[0]
    U = c * (Xm @ A.T)
    return X @ Wd.T + s * (U @ B.T), U


def linear_backward_dropout(Wd, X, dY, A, B, alpha: float, mask, p: float, dx_rows=None):
    """dX, dA, dB of the layer with dropout on the low-rank input (reading 10)."""
    c = dropout_keep_scale(p)
    Wd, X, dY, A, B = _f64(Wd), _f64(X), _f64(dY), _f64(A), _f64(B)
    Mf = np.asarray(mask, dtype=np.float64)
    Xm = X * Mf
    s = float(alpha) / A.shape[0]
    G = dY @ B
    U = c * (Xm @ A.T)
    dB = s * (dY.T @ U)
    dA = s * c * (G.T @ Xm)
    if dx_rows is not None:
        r_ = np.asarray(dx_rows)
        dX = dY[r_] @ Wd + s * c * ((G[r_] @ A) * Mf[r_])
    else:
        dX = dY @ Wd + s * c * ((G @ A) * Mf)
    return dX, dA, dB


# ----------------------------------------------------------------------------
# AdamW on the adapter masters (reading 11), fp64
# ----------------------------------------------------------------------------
def adamw_step(param, grad, m, v, step: int, lr: float, beta1: float = 0.9, beta2: float = 0.999,
               eps: float = 1e-8, weight_decay: float = 0.0, grad_scale: float = 1.0):
    """One AdamW step (decoupled weight decay) in fp64; returns (param, m, v)."""
    p, g, m, v = _f64(param), _f64(grad) * grad_scale, _f64(m), _f64(v)
    m = beta1 * m + (1.0 - beta1) * g
    v = beta2 * v + (1.0 - beta2) * g * g
    bc1 = 1.0 - beta1 ** step
    bc2 = 1.0 - beta2 ** step
    p = p * (1.0 - lr * weight_decay) - (lr / bc1) * m / (np.sqrt(v) / math.sqrt(bc2) + eps)
    return p, m, v


def silu_gate_forward(g, u):
    """h = silu(g) * u with silu(g) = g * sigmoid(g), fp64."""
    g, u = _f64(g), _f64(u)
    sig = 1.0 / (1.0 + np.exp(-g))
    return g * sig * u


def silu_gate_backward(dh, g, u):
    """(dg, du) of h = silu(g) * u, fp64."""
    dh, g, u = _f64(dh), _f64(g), _f64(u)
    sig = 1.0 / (1.0 + np.exp(-g))
    du = dh * g * sig
    dg = dh * u * sig * (1.0 + g * (1.0 - sig))
    return dg, du


# ----------------------------------------------------------------------------
# Error metrics used by the parity tests
# ----------------------------------------------------------------------------
def rel_frobenius(got, ref) -> float:
    got, ref = _f64(got), _f64(ref)
    den = math.sqrt(float(np.sum(ref * ref)))
    return math.sqrt(float(np.sum((got - ref) ** 2))) / max(den, 1e-300)


def max_abs_over_rms(got, ref) -> float:
    got, ref = _f64(got), _f64(ref)
    rms = math.sqrt(float(np.mean(ref * ref)))
    return float(np.max(np.abs(got - ref))) / max(rms, 1e-300)
