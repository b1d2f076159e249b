"""Python binding of libqlora (NF4 + double-quant QLoRA linear layer, B200).

Argument marshalling only: every function below forwards to the C entry point
of the same name in libqlora.so (see include/qlora.h); all arithmetic runs in
the library's CUDA kernels. Tensors are torch CUDA tensors (used purely as
device memory); the stream is torch's current stream unless one is given.
There is no CPU fallback: importing the binding without the built library, or
calling it without a CUDA device, raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# QLORA_BOUNDS_CHECK=1 selects the bounds-checking build (python -m bit_nf4_quantized_03_b200.build --bounds-check)
BOUNDS_CHECK = os.environ.get("QLORA_BOUNDS_CHECK", "") not in ("", "0")
LIB_PATH = os.path.join(_PKG, "libqlora_bounds.so" if BOUNDS_CHECK else "libqlora.so")

QLORA_OK = 0
QLORA_ERR_INVALID = 1
QLORA_ERR_UNSUPPORTED = 2
QLORA_ERR_CUDA = 3
QLORA_ERR_WORKSPACE = 4
QLORA_ERR_DEVICE = 5
QLORA_ERR_BOUNDS = 6
QLORA_SCALE_BF16 = 0
QLORA_SCALE_DQ_FP8 = 1
QLORA_DTYPE_BF16 = 0
QLORA_DTYPE_FP32 = 1
QLORA_BWD_ACCUMULATE_GRADS = 1
QLORA_BWD_ACCUMULATE_DX = 2
QLORA_BLOCKSIZE = BLOCKSIZE = 64
QLORA_DQ_BLOCKSIZE = DQ_BLOCKSIZE = 256

# every symbol include/qlora.h declares
EXPORTED = (
    "qlora_status_string", "qlora_version", "qlora_nf4_levels",
    "qlora_nf4_quantize_workspace_bytes", "qlora_nf4_quantize", "qlora_nf4_dequantize",
    "qlora_linear_workspace_bytes", "qlora_linear_fwd", "qlora_linear_bwd",
    "qlora_silu_gate_fwd", "qlora_silu_gate_bwd", "qlora_check_device_error",
    "qlora_launch_count", "qlora_timing_begin", "qlora_timing_end", "qlora_timing_launch",
    "qlora_nf4_quantize_noalloc", "qlora_selftest_wait_timeout", "qlora_lora_merge",
    "qlora_linear_workspace_bytes_ex", "qlora_linear_fwd_ex", "qlora_linear_bwd_ex",
    "qlora_adamw_step", "qlora_paged_alloc", "qlora_paged_free", "qlora_paged_prefetch",
    "qlora_expand_rate", "qlora_bounds_site", "qlora_linear_bwd_group", "qlora_linear_group_workspace_bytes",
)


class QloraError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class NF4Weight(ctypes.Structure):
    """Mirror of qlora_nf4_weight."""
    _fields_ = [
        ("n", ctypes.c_int64), ("k", ctypes.c_int64),
        ("blocksize", ctypes.c_int32), ("dq_blocksize", ctypes.c_int32),
        ("mode", ctypes.c_int32), ("reserved", ctypes.c_int32),
        ("codes", ctypes.c_void_p), ("scale_bf16", ctypes.c_void_p),
        ("scale_fp8", ctypes.c_void_p), ("dq_scale", ctypes.c_void_p),
        ("dq_mean", ctypes.c_void_p),
    ]


class Dropout(ctypes.Structure):
    """Mirror of qlora_dropout: LoRA dropout rate, Philox seed and offset, and the
    device mask buffer (m * k / 8 bytes) the forward writes and the backward reads."""
    _fields_ = [
        ("p", ctypes.c_float), ("reserved", ctypes.c_int32),
        ("seed", ctypes.c_uint64), ("offset", ctypes.c_uint64),
        ("mask", ctypes.c_void_p),
    ]

    def __init__(self, p: float, seed: int, offset: int, mask):
        super().__init__(float(p), 0, int(seed), int(offset), _ptr(mask, allow_addr=True))
        self._mask = mask


class AdamWConfig(ctypes.Structure):
    """Mirror of qlora_adamw_config."""
    _fields_ = [
        ("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float), ("eps", ctypes.c_float),
        ("weight_decay", ctypes.c_float), ("grad_scale", ctypes.c_float), ("step", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
    ]

    def __init__(self, lr: float, step: int, beta1: float = 0.9, beta2: float = 0.999, eps: float = 1e-8,
                 weight_decay: float = 0.0, grad_scale: float = 1.0):
        super().__init__(lr, beta1, beta2, eps, weight_decay, grad_scale, int(step), 0)


_lib = None


def lib() -> ctypes.CDLL:
    """Load libqlora.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libqlora.so not built ({LIB_PATH}); run python -m bit_nf4_quantized_03_b200.build")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, f32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    pw = ctypes.POINTER(NF4Weight)
    pd = ctypes.POINTER(Dropout)
    sig = {
        "qlora_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "qlora_version": (ctypes.c_char_p, []),
        "qlora_nf4_levels": (ctypes.c_int, [vp, vp]),
        "qlora_nf4_quantize_workspace_bytes": (sz, [i64, i64, i32]),
        "qlora_nf4_quantize": (ctypes.c_int, [vp, pw, vp, sz, vp]),
        "qlora_nf4_dequantize": (ctypes.c_int, [pw, vp, vp]),
        "qlora_linear_workspace_bytes": (sz, [i64, i64, i64, i32]),
        "qlora_linear_fwd": (ctypes.c_int, [pw, vp, i64, vp, vp, i32, f32, vp, i32, vp, vp, sz, vp]),
        "qlora_linear_bwd": (ctypes.c_int, [pw, vp, vp, i64, vp, vp, i32, f32, vp, vp, i32, vp, vp, i32,
                                            vp, sz, vp]),
        "qlora_silu_gate_fwd": (ctypes.c_int, [vp, vp, vp, i64, vp]),
        "qlora_silu_gate_bwd": (ctypes.c_int, [vp, vp, vp, vp, vp, i64, vp]),
        "qlora_check_device_error": (ctypes.c_int, [vp]),
        "qlora_launch_count": (ctypes.c_int64, []),
        "qlora_timing_begin": (ctypes.c_int, [i32]),
        "qlora_timing_end": (ctypes.c_int, [vp, vp, vp]),
        "qlora_timing_launch": (ctypes.c_int, [i32, vp, vp]),
        "qlora_nf4_quantize_noalloc": (ctypes.c_int, [vp, pw, vp]),
        "qlora_selftest_wait_timeout": (ctypes.c_int, [i32, vp]),
        "qlora_expand_rate": (ctypes.c_int, [i32, vp, vp]),
        "qlora_bounds_site": (ctypes.c_int, []),
        "qlora_lora_merge": (ctypes.c_int, [pw, vp, vp, i32, f32, vp, i32, vp]),
        "qlora_linear_workspace_bytes_ex": (sz, [i64, i64, i64, i32, pd]),
        "qlora_linear_bwd_group": (ctypes.c_int, [i32, vp, vp, vp, i64, vp, vp, i32, f32, vp, vp, i32, vp, vp, i32,
                                                  vp, sz, vp]),
        "qlora_linear_group_workspace_bytes": (sz, [i32, i64, vp, i64, i32]),
        "qlora_adamw_step": (ctypes.c_int, [vp, vp, vp, vp, vp, i64, ctypes.POINTER(AdamWConfig), vp]),
        "qlora_paged_alloc": (ctypes.c_int, [sz, ctypes.POINTER(ctypes.c_void_p)]),
        "qlora_paged_free": (ctypes.c_int, [vp]),
        "qlora_paged_prefetch": (ctypes.c_int, [vp, sz, i32, vp]),
        "qlora_linear_fwd_ex": (ctypes.c_int, [pw, vp, i64, vp, vp, i32, f32, vp, i32, vp, pd, vp, sz, vp]),
        "qlora_linear_bwd_ex": (ctypes.c_int, [pw, vp, vp, i64, vp, vp, i32, f32, vp, vp, i32, vp, vp, i32,
                                               pd, vp, sz, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def status_string(status: int) -> str:
    return lib().qlora_status_string(int(status)).decode()


def _ptr(t, allow_addr: bool = False) -> int | None:
    """Device address of a CUDA tensor. Raw integer addresses are accepted only where
    an entry point documents them (paged memory), so a stray integer cannot stand in
    for a tensor argument."""
    if t is None:
        return None
    if isinstance(t, int):
        if not allow_addr:
            raise TypeError("expected a CUDA tensor, got an integer address")
        return t
    if not t.is_cuda:
        raise ValueError("libqlora takes CUDA tensors only (no CPU fallback)")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, where: str) -> None:
    if rc != QLORA_OK:
        raise QloraError(rc, where)


# ----------------------------------------------------------------- weight --
class QuantizedWeight:
    """Device buffers of one NF4 weight plus the C struct that points at them."""

    def __init__(self, n: int, k: int, mode: int = QLORA_SCALE_DQ_FP8, device="cuda"):
        self.n, self.k, self.mode = int(n), int(k), int(mode)
        ne = self.n * self.k
        nblk = -(-ne // BLOCKSIZE)
        nblk2 = -(-nblk // DQ_BLOCKSIZE)
        u8 = torch.uint8
        self.codes = torch.zeros((ne + 1) // 2, dtype=u8, device=device)
        self.scale_bf16 = self.scale_fp8 = self.dq_scale = self.dq_mean = None
        if self.mode == QLORA_SCALE_BF16:
            self.scale_bf16 = torch.zeros(nblk, dtype=torch.int16, device=device)
        else:
            self.scale_fp8 = torch.zeros(nblk, dtype=u8, device=device)
            self.dq_scale = torch.zeros(nblk2, dtype=torch.float32, device=device)
            self.dq_mean = torch.zeros(1, dtype=torch.float32, device=device)
        self.struct = NF4Weight(self.n, self.k, BLOCKSIZE, DQ_BLOCKSIZE, self.mode, 0,
                                _ptr(self.codes), _ptr(self.scale_bf16), _ptr(self.scale_fp8),
                                _ptr(self.dq_scale), _ptr(self.dq_mean))

    def ref(self):
        return ctypes.byref(self.struct)

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in
                   (self.codes, self.scale_bf16, self.scale_fp8, self.dq_scale, self.dq_mean) if t is not None)


# ------------------------------------------------------------ entry points --
def qlora_version() -> str:
    return lib().qlora_version().decode()


def qlora_nf4_levels():
    lv = (ctypes.c_float * 16)()
    mid = (ctypes.c_float * 15)()
    _check(lib().qlora_nf4_levels(ctypes.addressof(lv), ctypes.addressof(mid)), "qlora_nf4_levels")
    return list(lv), list(mid)


def qlora_nf4_quantize_workspace_bytes(n: int, k: int, mode: int) -> int:
    return int(lib().qlora_nf4_quantize_workspace_bytes(n, k, mode))


def qlora_nf4_quantize(W: torch.Tensor, w: QuantizedWeight, ws: torch.Tensor | None = None, stream=None):
    """Quantize fp32 W [n, k] into w (allocates a workspace tensor if none is given)."""
    need = qlora_nf4_quantize_workspace_bytes(w.n, w.k, w.mode)
    if ws is None and need > 0:
        ws = torch.empty(need, dtype=torch.uint8, device=W.device)
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib().qlora_nf4_quantize(_ptr(W), w.ref(), _ptr(ws), ws_bytes, _stream(stream)), "qlora_nf4_quantize")
    return w


def qlora_nf4_dequantize(w: QuantizedWeight, out: torch.Tensor, stream=None) -> torch.Tensor:
    _check(lib().qlora_nf4_dequantize(w.ref(), _ptr(out), _stream(stream)), "qlora_nf4_dequantize")
    return out


def qlora_lora_merge(w: QuantizedWeight, A, B, r: int, alpha: float, out, out_dtype: int, stream=None):
    """out[n, k] = dequant(w) + (alpha / r) B A, in bf16 or fp32 (out_dtype)."""
    _check(lib().qlora_lora_merge(w.ref(), _ptr(A), _ptr(B), r, alpha, _ptr(out), out_dtype, _stream(stream)),
           "qlora_lora_merge")
    return out


def qlora_linear_workspace_bytes(m: int, n: int, k: int, r: int) -> int:
    return int(lib().qlora_linear_workspace_bytes(m, n, k, r))


def qlora_linear_fwd(w: QuantizedWeight, X, A, B, r: int, alpha: float, Y, y_dtype: int,
                     U_save=None, ws=None, stream=None):
    m = X.shape[0]
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    rc = lib().qlora_linear_fwd(w.ref(), _ptr(X), m, _ptr(A), _ptr(B), r, float(alpha), _ptr(Y), y_dtype,
                                _ptr(U_save), _ptr(ws), ws_bytes, _stream(stream))
    _check(rc, "qlora_linear_fwd")
    return Y


def qlora_linear_bwd(w: QuantizedWeight, X, dY, A, B, r: int, alpha: float, U_saved, dX, dx_dtype: int,
                     dA, dB, flags: int = 0, ws=None, stream=None):
    m = X.shape[0]
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    rc = lib().qlora_linear_bwd(w.ref(), _ptr(X), _ptr(dY), m, _ptr(A), _ptr(B), r, float(alpha), _ptr(U_saved),
                                _ptr(dX), dx_dtype, _ptr(dA), _ptr(dB), flags, _ptr(ws), ws_bytes,
                                _stream(stream))
    _check(rc, "qlora_linear_bwd")


def _dref(drop):
    return None if drop is None else ctypes.byref(drop)


def qlora_linear_workspace_bytes_ex(m: int, n: int, k: int, r: int, drop=None) -> int:
    return int(lib().qlora_linear_workspace_bytes_ex(m, n, k, r, _dref(drop)))


def qlora_linear_fwd_ex(w: QuantizedWeight, X, A, B, r: int, alpha: float, Y, y_dtype: int,
                        U_save=None, drop=None, ws=None, stream=None):
    m = X.shape[0]
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    rc = lib().qlora_linear_fwd_ex(w.ref(), _ptr(X), m, _ptr(A), _ptr(B), r, float(alpha), _ptr(Y), y_dtype,
                                   _ptr(U_save), _dref(drop), _ptr(ws), ws_bytes, _stream(stream))
    _check(rc, "qlora_linear_fwd_ex")
    return Y


def qlora_linear_bwd_ex(w: QuantizedWeight, X, dY, A, B, r: int, alpha: float, U_saved, dX, dx_dtype: int,
                        dA, dB, flags: int = 0, drop=None, ws=None, stream=None):
    m = X.shape[0]
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    rc = lib().qlora_linear_bwd_ex(w.ref(), _ptr(X), _ptr(dY), m, _ptr(A), _ptr(B), r, float(alpha),
                                   _ptr(U_saved), _ptr(dX), dx_dtype, _ptr(dA), _ptr(dB), flags, _dref(drop),
                                   _ptr(ws), ws_bytes, _stream(stream))
    _check(rc, "qlora_linear_bwd_ex")


def _ptr_array(items):
    """A C array of device addresses (None entries stay NULL)."""
    return (ctypes.c_void_p * len(items))(*[_ptr(t) for t in items])


def qlora_linear_group_workspace_bytes(m: int, ns, k: int, r: int) -> int:
    arr = (ctypes.c_int64 * len(ns))(*[int(n) for n in ns])
    return int(lib().qlora_linear_group_workspace_bytes(len(ns), m, ctypes.addressof(arr), k, r))


def qlora_linear_bwd_group(ws_list, X, dYs, As, Bs, r: int, alpha: float, U_saved, dX, dx_dtype: int,
                           dAs, dBs, flags: int = 0, ws=None, stream=None):
    """Backward of len(ws_list) layers sharing the input X: dX (+)= sum of the layers' terms,
    each layer's dA, dB as qlora_linear_bwd gives them."""
    count = len(ws_list)
    wp = (ctypes.POINTER(NF4Weight) * count)(*[ctypes.pointer(w.struct) for w in ws_list])
    dy, a, b, da, db = (_ptr_array(t) for t in (dYs, As, Bs, dAs, dBs))
    us = None if U_saved is None else _ptr_array(U_saved)
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    rc = lib().qlora_linear_bwd_group(count, ctypes.addressof(wp), _ptr(X), ctypes.addressof(dy), X.shape[0],
                                      ctypes.addressof(a), ctypes.addressof(b), r, float(alpha),
                                      None if us is None else ctypes.addressof(us), _ptr(dX), dx_dtype,
                                      ctypes.addressof(da), ctypes.addressof(db), flags, _ptr(ws), ws_bytes,
                                      _stream(stream))
    _check(rc, "qlora_linear_bwd_group")


def qlora_adamw_step(param, grad, m, v, param_bf16, count: int, cfg: AdamWConfig, stream=None):
    """One AdamW step on fp32 masters (tensors or device-accessible addresses)."""
    _check(lib().qlora_adamw_step(_ptr(param, True), _ptr(grad, True), _ptr(m, True), _ptr(v, True),
                                  _ptr(param_bf16, True), int(count), ctypes.byref(cfg), _stream(stream)),
           "qlora_adamw_step")


def qlora_paged_alloc(nbytes: int) -> int:
    """Managed (pageable unified) memory for optimizer states; returns its address."""
    out = ctypes.c_void_p(0)
    _check(lib().qlora_paged_alloc(int(nbytes), ctypes.byref(out)), "qlora_paged_alloc")
    return int(out.value)


def qlora_paged_free(addr: int):
    _check(lib().qlora_paged_free(addr), "qlora_paged_free")


def qlora_paged_prefetch(addr: int, nbytes: int, to_host: bool = False, stream=None):
    _check(lib().qlora_paged_prefetch(addr, int(nbytes), 1 if to_host else 0, _stream(stream)),
           "qlora_paged_prefetch")


def qlora_silu_gate_fwd(g, u, h, stream=None):
    _check(lib().qlora_silu_gate_fwd(_ptr(g), _ptr(u), _ptr(h), g.numel(), _stream(stream)), "qlora_silu_gate_fwd")
    return h


def qlora_silu_gate_bwd(dh, g, u, dg, du, stream=None):
    _check(lib().qlora_silu_gate_bwd(_ptr(dh), _ptr(g), _ptr(u), _ptr(dg), _ptr(du), g.numel(), _stream(stream)),
           "qlora_silu_gate_bwd")


def qlora_selftest_wait_timeout(limit_ms: int = 100, stream=None) -> None:
    _check(lib().qlora_selftest_wait_timeout(int(limit_ms), _stream(stream)), "qlora_selftest_wait_timeout")


def qlora_expand_rate(iters: int = 2048):
    """(weights expanded per SM-clock, per second) of the NF4 table expansion alone."""
    per_clk, per_s = ctypes.c_double(0), ctypes.c_double(0)
    _check(lib().qlora_expand_rate(int(iters), ctypes.addressof(per_clk), ctypes.addressof(per_s)),
           "qlora_expand_rate")
    return per_clk.value, per_s.value


def qlora_bounds_site() -> int:
    """Site of the first failed bounds check since the last call (0: none); bounds-check build only."""
    return int(lib().qlora_bounds_site())


def qlora_check_device_error(stream=None) -> None:
    rc = lib().qlora_check_device_error(_stream(stream))
    if rc != QLORA_OK and BOUNDS_CHECK:
        raise QloraError(rc, f"qlora_check_device_error (first failed bounds check: site {qlora_bounds_site()})")
    _check(rc, "qlora_check_device_error")


def qlora_launch_count() -> int:
    return int(lib().qlora_launch_count())


def qlora_timing_begin(max_launches: int) -> None:
    _check(lib().qlora_timing_begin(int(max_launches)), "qlora_timing_begin")


def qlora_timing_end():
    """Returns (total device ms, launches timed, algorithmic flops) of the fused GEMMs."""
    ms, n, fl = ctypes.c_double(0), ctypes.c_int32(0), ctypes.c_double(0)
    _check(lib().qlora_timing_end(ctypes.addressof(ms), ctypes.addressof(n), ctypes.addressof(fl)),
           "qlora_timing_end")
    return ms.value, n.value, fl.value


def qlora_timing_launches(count: int):
    """Per-launch (device ms, algorithmic flops) of the last qlora_timing_end, in launch order."""
    out = []
    for i in range(int(count)):
        ms, fl = ctypes.c_double(0), ctypes.c_double(0)
        _check(lib().qlora_timing_launch(i, ctypes.addressof(ms), ctypes.addressof(fl)), "qlora_timing_launch")
        out.append((ms.value, fl.value))
    return out


def qlora_nf4_quantize_noalloc(W: torch.Tensor, w: QuantizedWeight, stream=None):
    """qlora_nf4_quantize for callers that cannot allocate: no workspace, the
    library's fixed scratch array is used (calls must not overlap on the GPU)."""
    _check(lib().qlora_nf4_quantize_noalloc(_ptr(W), w.ref(), _stream(stream)), "qlora_nf4_quantize_noalloc")
    return w
