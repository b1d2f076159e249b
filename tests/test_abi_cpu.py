"""Host-only checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/qlora.h declares, its host-side NF4 level table
equals the oracle's bit for bit, workspace queries are consistent, and bad
arguments are rejected on the host before anything is launched."""
import ctypes
import os
import re

import numpy as np
import pytest

import bit_nf4_quantized_03_b200 as q
from oracle import nf4_oracle as o

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "qlora.h")


def _declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qlora_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    from bit_nf4_quantized_03_b200 import build
    build.build()
    return q.lib()


def test_library_exports_every_declared_symbol(L):
    syms = _declared_symbols()
    assert len(syms) >= 12
    for s in syms:
        assert hasattr(L, s), s
    assert sorted(q.EXPORTED) == syms


def test_bounds_checking_build_exports_the_same_symbols():
    # the -DQLORA_BOUNDS_CHECK variant is the same ABI (built by the build step next to libqlora.so)
    from bit_nf4_quantized_03_b200 import build
    if not os.path.exists(build.LIB_BOUNDS):
        pytest.skip("bounds-checking build not present (python -m bit_nf4_quantized_03_b200.build --bounds-check)")
    LB = ctypes.CDLL(build.LIB_BOUNDS)
    for s in _declared_symbols():
        assert hasattr(LB, s), s


def test_timing_launch_rejects_indexes_without_a_record(L):
    # host bookkeeping only: before any timed launch there is no record to read (1 = QLORA_ERR_INVALID)
    ms, fl = ctypes.c_double(0), ctypes.c_double(0)
    assert L.qlora_timing_launch(0, ctypes.addressof(ms), ctypes.addressof(fl)) == 1
    assert L.qlora_timing_launch(-1, ctypes.addressof(ms), ctypes.addressof(fl)) == 1
    assert L.qlora_timing_launch(0, None, None) == 1


def test_host_level_table_matches_oracle_bitwise(L):
    lv, mid = q.qlora_nf4_levels()
    lv = np.array(lv, dtype=np.float32)
    mid = np.array(mid, dtype=np.float32)
    assert np.array_equal(lv.view(np.uint32), o.nf4_levels().view(np.uint32))
    assert np.array_equal(mid.view(np.uint32), o.nf4_midpoints().view(np.uint32))


def test_status_strings_and_version(L):
    assert q.qlora_version().startswith("qlora-nf4-b200")
    assert q.status_string(0) == "ok"
    assert "invalid" in q.status_string(1)
    assert q.status_string(99) == "unknown status"


def test_workspace_queries(L):
    assert q.qlora_nf4_quantize_workspace_bytes(4096, 4096, q.QLORA_SCALE_BF16) == 0
    dq = q.qlora_nf4_quantize_workspace_bytes(4096, 4096, q.QLORA_SCALE_DQ_FP8)
    assert dq >= 4096 * 4096 // 64 * 4           # fp32 absmax per block
    assert q.qlora_linear_workspace_bytes(2048, 4096, 4096, 64) > 0
    assert q.qlora_linear_workspace_bytes(0, 4096, 4096, 64) == 0
    a = q.qlora_linear_workspace_bytes(16, 8192, 8192, 64)
    b = q.qlora_linear_workspace_bytes(16, 8192, 8192, 64)
    assert a == b > 0


def _weight(n=256, k=256, mode=0, codes=1 << 20, scale=1 << 21):
    return q.NF4Weight(n, k, 64, 256, mode, 0, codes, scale if mode == 0 else None,
                       scale if mode == 1 else None, scale if mode == 1 else None, scale if mode == 1 else None)


def test_invalid_arguments_rejected_on_host(L):
    w = _weight()
    # null / misaligned input
    assert L.qlora_nf4_quantize(None, ctypes.byref(w), None, 0, None) == 1
    assert L.qlora_nf4_quantize(1 << 20 | 4, ctypes.byref(w), None, 0, None) == 1
    # wrong block sizes
    bad = _weight()
    bad.blocksize = 32
    assert L.qlora_nf4_quantize(1 << 22, ctypes.byref(bad), None, 0, None) == 1
    bad = _weight()
    bad.dq_blocksize = 128
    assert L.qlora_nf4_dequantize(ctypes.byref(bad), 1 << 22, None) == 1
    # double-quant without workspace
    wd = _weight(mode=1)
    assert L.qlora_nf4_quantize(1 << 22, ctypes.byref(wd), None, 0, None) == 4
    # linear: unsupported rank, k not a multiple of 64, n not a multiple of 8
    for n, k, r, want in ((256, 256, 12, 2), (256, 200, 8, 2), (260, 256, 8, 2)):
        ww = _weight(n=n, k=k)
        rc = L.qlora_linear_fwd(ctypes.byref(ww), 1 << 23, 128, 1 << 24, 1 << 25, r, 16.0, 1 << 26, 0, None,
                                1 << 27, 1 << 30, None)
        assert rc == want, (n, k, r, rc)
    # workspace too small
    ww = _weight()
    rc = L.qlora_linear_fwd(ctypes.byref(ww), 1 << 23, 128, 1 << 24, 1 << 25, 8, 16.0, 1 << 26, 0, None,
                            1 << 27, 16, None)
    assert rc == 4
    # bwd: bad flags, null grads
    rc = L.qlora_linear_bwd(ctypes.byref(ww), 1 << 23, 1 << 24, 128, 1 << 25, 1 << 26, 8, 16.0, None, None, 0,
                            1 << 27, 1 << 28, 8, 1 << 29, 1 << 30, None)
    assert rc == 1
    rc = L.qlora_linear_bwd(ctypes.byref(ww), 1 << 23, 1 << 24, 128, 1 << 25, 1 << 26, 8, 16.0, None, None, 0,
                            None, 1 << 28, 0, 1 << 29, 1 << 30, None)
    assert rc == 1
    # adapter merge: null adapter, bad output dtype, unsupported rank or k
    ww = _weight()
    assert L.qlora_lora_merge(ctypes.byref(ww), None, 1 << 25, 8, 16.0, 1 << 26, 0, None) == 1
    assert L.qlora_lora_merge(ctypes.byref(ww), 1 << 24, 1 << 25, 8, 16.0, 1 << 26 | 8, 0, None) == 1
    assert L.qlora_lora_merge(ctypes.byref(ww), 1 << 24, 1 << 25, 8, 16.0, 1 << 26, 7, None) == 1
    assert L.qlora_lora_merge(ctypes.byref(ww), 1 << 24, 1 << 25, 12, 16.0, 1 << 26, 0, None) == 2
    wk = _weight(k=200)
    assert L.qlora_lora_merge(ctypes.byref(wk), 1 << 24, 1 << 25, 8, 16.0, 1 << 26, 1, None) == 2
    # dropout: rate outside [0, 1), missing or misaligned mask; the workspace grows by m * k * 2
    ww = _weight()
    for p_, mask_ in ((1.5, 1 << 28), (-0.1, 1 << 28), (0.05, None), (0.05, (1 << 28) | 4)):
        d = q.Dropout(p_, 1, 0, mask_)
        rc = L.qlora_linear_fwd_ex(ctypes.byref(ww), 1 << 23, 128, 1 << 24, 1 << 25, 8, 16.0, 1 << 26, 0, None,
                                   ctypes.byref(d), 1 << 27, 1 << 30, None)
        assert rc == 1, (p_, mask_, rc)
    base = q.qlora_linear_workspace_bytes(128, 256, 256, 8)
    assert q.qlora_linear_workspace_bytes_ex(128, 256, 256, 8, None) == base
    assert q.qlora_linear_workspace_bytes_ex(128, 256, 256, 8, q.Dropout(0.0, 1, 0, None)) == base
    assert q.qlora_linear_workspace_bytes_ex(128, 256, 256, 8, q.Dropout(0.05, 1, 0, 1 << 28)) == base + 128 * 256 * 2
    # AdamW: bad hyperparameters or step, misaligned arrays; count 0 is a no-op
    good = q.AdamWConfig(lr=2e-4, step=1)
    args = (1 << 20, 1 << 21, 1 << 22, 1 << 23, None, 100)
    assert L.qlora_adamw_step(*args[:5], 0, ctypes.byref(good), None) == 0
    for bad in (q.AdamWConfig(lr=2e-4, step=0), q.AdamWConfig(lr=2e-4, step=1, beta1=1.0),
                q.AdamWConfig(lr=2e-4, step=1, beta2=0.0), q.AdamWConfig(lr=2e-4, step=1, eps=0.0),
                q.AdamWConfig(lr=float("nan"), step=1)):
        assert L.qlora_adamw_step(*args, ctypes.byref(bad), None) == 1
    assert L.qlora_adamw_step((1 << 20) | 4, *args[1:], ctypes.byref(good), None) == 1
    assert L.qlora_adamw_step(*args[:4], (1 << 24) | 2, 100, ctypes.byref(good), None) == 1
    assert L.qlora_adamw_step(*args, None, None) == 1
    assert L.qlora_paged_free(None) == 0
    assert L.qlora_paged_prefetch(None, 16, 0, None) == 1
    # elementwise
    assert L.qlora_silu_gate_fwd(None, None, None, 16, None) == 1
    assert L.qlora_silu_gate_fwd(None, None, None, 0, None) == 0
    assert L.qlora_silu_gate_bwd(None, None, None, None, None, -1, None) == 1


def test_binding_refuses_cpu_tensors(L):
    import torch
    w = torch.zeros(64, 64)
    with pytest.raises(ValueError):
        q._ptr(w)
    # an integer stands in for a tensor only where an entry point documents raw addresses
    with pytest.raises(TypeError):
        q._ptr(1 << 20)
    assert q._ptr(1 << 20, allow_addr=True) == 1 << 20


def test_binding_constants_match_the_header_enums():
    # every QLORA_* enum value the header defines, as the binding spells it
    import re
    text = open(HEADER).read()
    vals = dict((name, int(v)) for name, v in re.findall(r"\b(QLORA_[A-Z0-9_]+)\s*=\s*(\d+)", text))
    assert vals, "no enum values found"
    for name, v in vals.items():
        assert getattr(q, name) == v, name
