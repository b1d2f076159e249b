#!/usr/bin/env python3
"""Throughput of the NF4 + double-quant QLoRA frozen-base linear layer on B200.

One step = the hot path of one 65B-shape decoder layer (q/k/v/o 8192x8192,
gate/up 22016x8192, down 8192x22016; NF4 blocks of 64 with FP8 double
quantization; LoRA r = 64, alpha = 16) over 8192 tokens per GPU:

  * forward + backward of q, k, v (shared input, dX accumulated) and o;
  * the SiLU-gated MLP: gate and up forward, h = silu(g) * u, down forward,
    then down backward, SiLU-gate backward, gate and up backward (dX accumulated);
  * forward of all seven projections at M = 16 tokens (weight-stream bound);
  * with N > 1 ranks (data parallel, 8192 tokens per rank): an all-reduce of
    every adapter gradient dA, dB over NCCL.

The weights are quantized once before timing (the pages quantize the frozen
base once, offline); quantize / dequantize throughput is measured as separate
components. Inputs are seeded synthetic tensors.

Prints one JSON line on rank 0. `--impl reference` times the CPU oracle on a
bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "QLoRA linear fwd+bwd TFLOP/s & tokens/s (7B/65B shapes), % of roofline"
WORKLOAD = "65B-shape decoder linears (q/k/v/o 8192x8192, gate/up 22016x8192, down 8192x22016), NF4+DQ, r=64"
M_TOKENS = 8192
M_SMALL = 16
RANK_R = 64
ALPHA = 16.0
LAYERS = [("q_proj", 8192, 8192), ("k_proj", 8192, 8192), ("v_proj", 8192, 8192), ("o_proj", 8192, 8192),
          ("gate_proj", 22016, 8192), ("up_proj", 22016, 8192), ("down_proj", 8192, 22016)]
L2_FLUSH_BYTES = 512 << 20
PAIR_FLOPS_MIN = 1e12      # a fused GEMM at 8192 tokens has >= 2*8192^3 (1.1e12) flops, one at 16 tokens <= 5.8e9

# DRAM bytes (read + write) per launch of the CTA-pair fused GEMM, averaged over its 11 launches of one step, from the
# 1-pass ncu launch list of this benchmark (dram__bytes_read.sum + dram__bytes_write.sum). Printed only while the
# kernel's sources hash to the value recorded with it; any change to them prints null until the counters are taken
# again. (Recorded again, without a new capture, after changes confined to the single-CTA kernel's configuration,
# warp roles and epilogue in the same file: the CTA-pair kernel's code is as captured.)
WGEMM_TRAFFIC = {"bytes_per_launch": 1212925451,
                 "sources_sha256": "59baa132bf327a400c85079d6f4d74c77418a0571252d5e70ab3e85f5a61f4c2"}
WGEMM_SOURCES = ("bit_nf4_quantized_03_b200/csrc/nf4_wgemm.cu", "bit_nf4_quantized_03_b200/csrc/qlora_device.cuh")


def wgemm_sources_sha256() -> str:
    h = hashlib.sha256()
    for rel in WGEMM_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def pair_algo_bytes(m: int = M_TOKENS, r: int = RANK_R) -> float:
    """Algorithmic DRAM bytes per CTA-pair launch of one step, averaged over its launches:
    every operand counted once at its stored size (bf16 activations and outputs, packed
    codes, E4M3 scales with their fp32 second-level scales, the adapter tiles of the K
    extension). Forward: X, W, Y per layer; backward: the layers of a group (q/k/v, and
    gate/up) in one launch reading every layer's dY and W and writing dX once."""
    def w_bytes(n, k):
        return n * k * (0.5 + 1.0 / 64 + 4.0 / 16384)
    dims = {nm: (n, k) for nm, n, k in LAYERS}
    launches = []
    for nm, n, k in LAYERS:                                        # forwards
        launches.append(2 * m * k + w_bytes(n, k) + 2 * m * n + 2 * m * r + 2 * n * r)
    for group in (("down_proj",), ("gate_proj", "up_proj"), ("o_proj",), ("q_proj", "k_proj", "v_proj")):
        k = dims[group[0]][1]
        launches.append(2 * m * k + sum(2 * m * dims[g][0] + w_bytes(*dims[g]) + 2 * m * r + 2 * r * k
                                        for g in group))
    return sum(launches) / len(launches)


def wgemm_traffic():
    if WGEMM_TRAFFIC["sources_sha256"] is None or WGEMM_TRAFFIC["sources_sha256"] != wgemm_sources_sha256():
        return None
    return WGEMM_TRAFFIC["bytes_per_launch"]


# ------------------------------------------------------------------ helpers --
def linear_flops(m: int, n: int, k: int, r: int, backward: bool) -> float:
    """Algorithmic flops: forward 2MNK + 2Mr(K+N); backward adds dX (2MNK + 2MKr),
    G = dY B (2MNr), dB (2MNr) and dA (2MKr). No dequant work, no dW."""
    f = 2.0 * m * n * k + 2.0 * m * r * (k + n)
    if backward:
        f += 2.0 * m * n * k + 4.0 * m * r * (k + n)
    return f


def step_flops(m: int = M_TOKENS, m_small: int = M_SMALL, r: int = RANK_R) -> float:
    total = 0.0
    for _, n, k in LAYERS:
        total += linear_flops(m, n, k, r, True) + linear_flops(m_small, n, k, r, False)
    return total


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["_source"] = "measured"
        return d
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "_source": "fallback"}


def max_over_ranks(x: float) -> float:
    from bit_nf4_quantized_03_b200 import dp
    return dp.max_over_ranks(x)


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples taken while the timed region runs.
    The sampler is started, and its first sample awaited, before the region; each
    sample carries nvidia-smi's timestamp, and only those stamped inside the region
    (plus one interval after it, which still reports the region's last moments)
    are summarised."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    INTERVAL_MS = 50

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.first = ""
        self.out = ""
        self.t0 = self.t1 = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader",
                                          "-lms", str(self.INTERVAL_MS), "-i", str(self.dev)],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        if self.proc is not None:
            try:
                import select
                ready, _, _ = select.select([self.proc.stdout], [], [], 5.0)
                if ready:
                    self.first = self.proc.stdout.readline()
            except (OSError, ValueError):
                pass
        self.t0 = time.time()
        return self

    def __exit__(self, *a):
        self.t1 = time.time()
        rest = ""
        if self.proc is not None:
            time.sleep(2.0 * self.INTERVAL_MS / 1000.0)
            self.proc.terminate()
            try:
                rest, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                rest, _ = self.proc.communicate()
        self.out = (self.first or "") + (rest or "")

    @staticmethod
    def _stamp(text: str):
        import datetime
        try:
            return datetime.datetime.strptime(text.strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()
        except ValueError:
            return None

    def summary(self) -> dict:
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        rows = []
        for line in (self.out or "").splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                sm = float(parts[2].split()[0])
                smax = float(parts[3].split()[0])
            except (ValueError, IndexError):
                continue
            active = {nm for nm, v in zip(names, parts[6:10]) if v.lower().startswith("active")}
            rows.append((self._stamp(parts[0]), sm, smax, active))
        window = "timed region"
        if self.t0 is not None and self.t1 is not None:
            late = self.t1 + self.INTERVAL_MS / 1000.0
            inside = [r for r in rows if r[0] is not None and self.t0 <= r[0] <= late]
        else:
            inside = []
        if not inside:             # region shorter than the sampling interval, or no timestamps
            inside, window = rows, "all samples"
        sm = [r[1] for r in inside]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": inside[-1][2] if inside else None,
                "reasons": sorted(set().union(*[r[3] for r in inside])) if inside else [],
                "samples": len(sm), "window": window}


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 0) for d in threadpool_info() if d.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


# ---------------------------------------------------------- CPU oracle leg --
class OracleSample:
    """The oracle on a bounded sample of the workload: q_proj (8192 x 8192,
    r = 64) with the weight quantized and dequantized once (setup), then per
    step: forward for `rows` sampled tokens, backward dX for those rows, and
    the adapter gradients dA, dB over all 8192 tokens."""

    def __init__(self, rows: int = 32):
        from bit_nf4_quantized_03_b200 import synth
        from oracle import nf4_oracle as o
        self.o = o
        name, n, k = LAYERS[0]
        W = synth.weight(n, k, layer=0)
        self.Wd = o.dequantize_f64(o.quantize(W.numpy(), o.MODE_DQ_FP8), (n, k))
        self.X = synth.activations(M_TOKENS, k, layer=0)
        self.A, self.B = synth.lora_pair(RANK_R, k, n, layer=0)
        self.dY = synth.grad_output(M_TOKENS, n, layer=0)
        self.rows = synth.sample_rows(M_TOKENS, rows).numpy()
        m = M_TOKENS
        r = RANK_R
        nr = len(self.rows)
        self.flops = (2.0 * nr * n * k + 2.0 * nr * r * (k + n)        # Y rows
                      + 2.0 * nr * n * k + 2.0 * nr * r * k            # dX rows
                      + 2.0 * m * n * r + 2.0 * m * k * r              # G, U over all tokens
                      + 2.0 * m * n * r + 2.0 * m * k * r)             # dB, dA
        self.desc = (f"q_proj 8192x8192 r=64: forward and dX for {nr} sampled token rows of 8192, "
                     f"dA/dB over all 8192 tokens (fp64 numpy); weight quantized/dequantized once before timing")

    def step(self) -> float:
        t0 = time.perf_counter()
        self.o.linear_forward(self.Wd, self.X, self.A, self.B, ALPHA, rows=self.rows)
        self.o.linear_backward(self.Wd, self.X, self.dY, self.A, self.B, ALPHA, dx_rows=self.rows)
        return time.perf_counter() - t0


def oracle_configs() -> dict:
    """The oracle, as it stands, timed per workload on the host cores: quantize and
    dequantize of the 4096 x 4096 weight with outliers (both scale modes) and the
    single 256 x 256 layer and the 7B q_proj (fwd+bwd) in full; the 7B SiLU MLP at
    4096 tokens on 64 sampled token rows (forward and dX through the whole chain),
    reported as measured and as a flop-rate extrapolation to the full config."""
    from bit_nf4_quantized_03_b200 import synth
    from oracle import nf4_oracle as o
    res = {}
    W = synth.weight(4096, 4096, outlier_frac=0.001).numpy()
    ne = W.size
    for mode, tag, scale_b in ((o.MODE_BF16, "bf16", 2.0 / 64), (o.MODE_DQ_FP8, "dq_fp8", 1.0 / 64 + 4.0 / 16384)):
        t0 = time.perf_counter()
        qw = o.quantize(W, mode)
        t1 = time.perf_counter()
        o.dequantize(qw)
        t2 = time.perf_counter()
        res[f"quantize_{tag}"] = {"s": t1 - t0, "gbs": ne * (4.5 + scale_b) / (t1 - t0) / 1e9, "sample": "full"}
        res[f"dequantize_{tag}"] = {"s": t2 - t1, "gbs": ne * (2.5 + scale_b) / (t2 - t1) / 1e9, "sample": "full"}
    for name, (m, n, k, r) in (("single_256_r8", (128, 256, 256, 8)), ("q_proj_7b", (2048, 4096, 4096, 64))):
        Wd = o.dequantize_f64(o.quantize(synth.weight(n, k).numpy(), o.MODE_DQ_FP8), (n, k))
        X = synth.activations(m, k)
        A, B = synth.lora_pair(r, k, n)
        dY = synth.grad_output(m, n)
        t0 = time.perf_counter()
        o.linear_forward(Wd, X, A, B, ALPHA)
        o.linear_backward(Wd, X, dY, A, B, ALPHA)
        dt = time.perf_counter() - t0
        fl = linear_flops(m, n, k, r, True)
        res[name] = {"s": dt, "tflops": fl / dt / 1e12, "tokens_per_s": m / dt, "sample": "full"}
    # 7B MLP chain on sampled token rows: every row's forward and dX are independent of
    # the other rows; dA, dB are sums over tokens, so the sample computes those rows' share
    M, H, I, rows = 4096, 4096, 11008, 64
    idx = synth.sample_rows(M, rows).numpy()
    Wg = o.dequantize_f64(o.quantize(synth.weight(I, H, layer=41).numpy(), o.MODE_DQ_FP8), (I, H))
    Wu = o.dequantize_f64(o.quantize(synth.weight(I, H, layer=42).numpy(), o.MODE_DQ_FP8), (I, H))
    Wdn = o.dequantize_f64(o.quantize(synth.weight(H, I, layer=43).numpy(), o.MODE_DQ_FP8), (H, I))
    Ag, Bg = synth.lora_pair(RANK_R, H, I, layer=41)
    Au, Bu = synth.lora_pair(RANK_R, H, I, layer=42)
    Ad, Bd = synth.lora_pair(RANK_R, I, H, layer=43)
    Xs = synth.activations(M, H, layer=41).float().numpy()[idx]
    dYs = synth.grad_output(M, H, layer=43).float().numpy()[idx]
    t0 = time.perf_counter()
    g, _ = o.linear_forward(Wg, Xs, Ag, Bg, ALPHA)
    u, _ = o.linear_forward(Wu, Xs, Au, Bu, ALPHA)
    hh = o.silu_gate_forward(g, u)
    o.linear_forward(Wdn, hh, Ad, Bd, ALPHA)
    dh, _, _ = o.linear_backward(Wdn, hh, dYs, Ad, Bd, ALPHA)
    dg, du = o.silu_gate_backward(dh, g, u)
    o.linear_backward(Wg, Xs, dg, Ag, Bg, ALPHA)
    o.linear_backward(Wu, Xs, du, Au, Bu, ALPHA)
    dt = time.perf_counter() - t0
    sample_fl = (2 * linear_flops(rows, I, H, RANK_R, True) + linear_flops(rows, H, I, RANK_R, True))
    full_fl = 2 * linear_flops(M, I, H, RANK_R, True) + linear_flops(M, H, I, RANK_R, True)
    rate = sample_fl / dt
    res["mlp_7b"] = {"s": dt, "tflops": rate / 1e12, "sample": f"{rows} of {M} token rows through the whole chain "
                     "(forward, dX, and those rows' share of dA and dB)", "extrapolated_full_s": full_fl / rate,
                     "extrapolated_tokens_per_s": M / (full_fl / rate)}
    return res


def run_reference(args) -> None:
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    s = OracleSample()
    for _ in range(args.warmup):
        s.step()
    times = [s.step() for _ in range(args.steps)]
    total = sum(times)
    value = s.flops * len(times) / total / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / len(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample": s.desc},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": s.desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------ native arm --
class Workload:
    def __init__(self, dev):
        import torch
        import bit_nf4_quantized_03_b200 as q
        from bit_nf4_quantized_03_b200 import synth
        self.q, self.dev = q, dev
        rank = int(os.environ.get("RANK", "0"))
        off = 1000 * rank                      # every rank gets its own tokens
        bf, f32 = torch.bfloat16, torch.float32
        self.w, self.A, self.B = {}, {}, {}
        for i, (name, n, k) in enumerate(LAYERS):
            W = synth.weight(n, k, layer=i).to(dev)
            qw = q.QuantizedWeight(n, k, q.QLORA_SCALE_DQ_FP8, device=dev)
            q.qlora_nf4_quantize(W, qw)
            del W
            a, b = synth.lora_pair(RANK_R, k, n, layer=i)
            self.w[name], self.A[name], self.B[name] = qw, a.to(dev), b.to(dev)
        torch.cuda.synchronize()
        M, H, I = M_TOKENS, 8192, 22016
        # host copies (pinned) of every input a step consumes, in the order the step first reads them
        self.host = {
            "x_attn": synth.activations(M, H, layer=off + 10), "x_o": synth.activations(M, H, layer=off + 11),
            "x_mlp": synth.activations(M, H, layer=off + 12), "dy_mlp": synth.grad_output(M, H, layer=off + 24),
            "dy_o": synth.grad_output(M, H, layer=off + 23), "dy_q": synth.grad_output(M, H, layer=off + 20),
            "dy_k": synth.grad_output(M, H, layer=off + 21), "dy_v": synth.grad_output(M, H, layer=off + 22),
            "x16": synth.activations(M_SMALL, H, layer=off + 30), "h16": synth.activations(M_SMALL, I, layer=off + 31),
        }
        # per-input copy events of the current input set (end-to-end timing only): the step
        # waits for each input just before its first use
        self.in_events = None
        self.host = {k_: v.pin_memory() for k_, v in self.host.items()}
        self.d = {k_: v.to(dev) for k_, v in self.host.items()}
        e = lambda *s, dt=bf: torch.empty(*s, dtype=dt, device=dev)
        self.y = {nm: e(M, n) for nm, n, _ in LAYERS if nm not in ("gate_proj", "up_proj", "down_proj")}
        self.g, self.u, self.h, self.y_mlp = e(M, I), e(M, I), e(M, I), e(M, H)
        self.dh, self.dg, self.du = e(M, I), e(M, I), e(M, I)
        self.dx_attn, self.dx_o, self.dx_mlp = e(M, H), e(M, H), e(M, H)
        self.U = {nm: e(M, RANK_R, dt=f32) for nm, _, _ in LAYERS}
        self.y16 = {nm: e(M_SMALL, n) for nm, n, _ in LAYERS}
        # adapter gradients live in one flat buffer (one all-reduce for the data-parallel exchange)
        from bit_nf4_quantized_03_b200 import dp
        self.adapter_grads = dp.AdapterGrads(LAYERS, RANK_R, device=dev)
        self.grads, self.dA, self.dB = self.adapter_grads.flat, self.adapter_grads.dA, self.adapter_grads.dB
        self.host_grads = torch.empty(self.grads.shape, dtype=f32).pin_memory()
        ws = max(max(q.qlora_linear_workspace_bytes(M, n, k, RANK_R),
                     q.qlora_linear_workspace_bytes(M_SMALL, n, k, RANK_R)) for _, n, k in LAYERS)
        ws = max(ws, q.qlora_linear_group_workspace_bytes(M, [H, H, H], H, RANK_R),
                 q.qlora_linear_group_workspace_bytes(M, [I, I], H, RANK_R))
        self.ws = torch.empty(ws, dtype=torch.uint8, device=dev)
        self.flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.h2d_bytes = sum(v.numel() * v.element_size() for v in self.host.values())
        self.d2h_bytes = self.host_grads.numel() * 4

    def _fwd(self, nm, X, Y, U):
        q = self.q
        q.qlora_linear_fwd(self.w[nm], X, self.A[nm], self.B[nm], RANK_R, ALPHA, Y, q.QLORA_DTYPE_BF16, U, self.ws)

    def _bwd(self, nm, X, dY, dX, acc_dx):
        q = self.q
        flags = q.QLORA_BWD_ACCUMULATE_DX if acc_dx else 0
        q.qlora_linear_bwd(self.w[nm], X, dY, self.A[nm], self.B[nm], RANK_R, ALPHA, self.U[nm], dX,
                           q.QLORA_DTYPE_BF16, self.dA[nm], self.dB[nm], flags, self.ws)

    def _bwd_group(self, names, X, dYs, dX):
        """Backward of the layers in `names`, which share the input X: one fused dX GEMM."""
        q = self.q
        q.qlora_linear_bwd_group([self.w[nm] for nm in names], X, list(dYs), [self.A[nm] for nm in names],
                                 [self.B[nm] for nm in names], RANK_R, ALPHA, [self.U[nm] for nm in names], dX,
                                 q.QLORA_DTYPE_BF16, [self.dA[nm] for nm in names], [self.dB[nm] for nm in names],
                                 0, self.ws)

    def _inputs(self):
        """The input set, as a mapping whose lookup first makes the compute stream wait
        for that input's host copy when one is in flight."""
        import torch
        d, evs = self.d, self.in_events

        class _Waiting:
            def __getitem__(self, key):
                if evs is not None:
                    torch.cuda.current_stream().wait_event(evs[key])
                return d[key]
        return d if evs is None else _Waiting()

    def step(self):
        q, d = self.q, self._inputs()
        for nm in ("q_proj", "k_proj", "v_proj"):
            self._fwd(nm, d["x_attn"], self.y[nm], self.U[nm])
        self._fwd("o_proj", d["x_o"], self.y["o_proj"], self.U["o_proj"])
        self._fwd("gate_proj", d["x_mlp"], self.g, self.U["gate_proj"])
        self._fwd("up_proj", d["x_mlp"], self.u, self.U["up_proj"])
        q.qlora_silu_gate_fwd(self.g, self.u, self.h)
        self._fwd("down_proj", self.h, self.y_mlp, self.U["down_proj"])
        self._bwd("down_proj", self.h, d["dy_mlp"], self.dh, False)
        q.qlora_silu_gate_bwd(self.dh, self.g, self.u, self.dg, self.du)
        self._bwd_group(("gate_proj", "up_proj"), d["x_mlp"], (self.dg, self.du), self.dx_mlp)
        self._bwd("o_proj", d["x_o"], d["dy_o"], self.dx_o, False)
        self._bwd_group(("q_proj", "k_proj", "v_proj"), d["x_attn"], (d["dy_q"], d["dy_k"], d["dy_v"]),
                        self.dx_attn)
        for nm, _, _ in LAYERS:
            x = d["h16"] if nm == "down_proj" else d["x16"]
            self._fwd(nm, x, self.y16[nm], None)
        self.adapter_grads.all_reduce()

    def h2d(self):
        for k_, v in self.host.items():
            self.d[k_].copy_(v, non_blocking=True)

    def d2h(self):
        self.host_grads.copy_(self.grads, non_blocking=True)


def time_e2e_pipelined(wl, steps, sync_barrier=None):
    """End-to-end ms per step with the host copies of every step inside the timed region:
    the pinned-host inputs of step i+1 go to a second device input set on a copy stream
    while step i computes, and step i's adapter gradients are copied device-side to a
    staging buffer (so step i+1 cannot overwrite them) and read back to pinned host
    memory on a third stream, so the read-back never queues behind the next input
    copy (the two directions use separate copy engines). Timed by CUDA events from
    the first copy to the last read-back; the inputs of every step exceed L2, so
    nothing is flushed in between."""
    import torch
    comp = torch.cuda.current_stream()
    cs = torch.cuda.Stream()
    rs = torch.cuda.Stream()
    sets = [wl.d, {k_: torch.empty_like(v) for k_, v in wl.d.items()}]
    stage = [torch.empty_like(wl.grads), torch.empty_like(wl.grads)]
    ev = lambda: torch.cuda.Event()
    done, staged, read = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    copied = [{k_: ev() for k_ in wl.host}, {k_: ev() for k_ in wl.host}]   # one event per input and set

    def copy_inputs(dst):
        for k_, v in wl.host.items():
            sets[dst][k_].copy_(v, non_blocking=True)
            copied[dst][k_].record(cs)

    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    base = wl.d
    if sync_barrier:
        sync_barrier()
    torch.cuda.synchronize()
    t0.record(comp)
    cs.wait_event(t0)
    with torch.cuda.stream(cs):
        copy_inputs(0)
    for i in range(steps):
        cur, nxt = i % 2, (i + 1) % 2
        if i + 1 < steps:
            with torch.cuda.stream(cs):
                if i >= 1:
                    cs.wait_event(done[nxt])          # step i-1 is finished with that input set
                copy_inputs(nxt)
        if i >= 2:
            comp.wait_event(read[cur])                # staging buffer free again
        wl.d, wl.in_events = sets[cur], copied[cur]   # the step waits on each input before its first use
        wl.step()
        wl.in_events = None
        done[cur].record(comp)
        stage[cur].copy_(wl.grads, non_blocking=True)
        staged[cur].record(comp)
        with torch.cuda.stream(rs):
            rs.wait_event(staged[cur])
            wl.host_grads.copy_(stage[cur], non_blocking=True)
            read[cur].record(rs)
    comp.wait_stream(cs)
    comp.wait_stream(rs)
    t1.record(comp)
    torch.cuda.synchronize()
    wl.d = base
    if sync_barrier:
        sync_barrier()
    return t0.elapsed_time(t1) / steps


def time_h2d_alone(wl, reps, sync_barrier=None):
    """Device time of one step's pinned-host input copies with no compute beside them
    (the floor of the end-to-end step when the host link is the bottleneck)."""
    import torch
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if sync_barrier:
        sync_barrier()
    torch.cuda.synchronize()
    t0.record()
    for _ in range(reps):
        wl.h2d()
    t1.record()
    torch.cuda.synchronize()
    if sync_barrier:
        sync_barrier()
    return t0.elapsed_time(t1) / reps


def time_steps(fn, steps, flush=None, sync_barrier=None):
    """Device time of `steps` calls of fn (CUDA events on the current stream),
    L2 flushed between calls outside the events. Returns ms per call."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    if sync_barrier:
        sync_barrier()
    torch.cuda.synchronize()
    for a, b in evs:
        if flush is not None:
            flush.fill_(1)
        a.record()
        fn()
        b.record()
    torch.cuda.synchronize()
    if sync_barrier:
        sync_barrier()
    return sum(a.elapsed_time(b) for a, b in evs) / steps


def graph_time(fn, iters, flush) -> float:
    """Device ms per call of fn without host overhead: CUDA-graph replay of
    [L2 flush, fn] x iters minus replay of [L2 flush] x iters."""
    import torch
    fn()
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    g_op, g_flush = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_op, stream=side):
        for _ in range(iters):
            flush.fill_(1)
            fn()
    with torch.cuda.graph(g_flush, stream=side):
        for _ in range(iters):
            flush.fill_(1)

    def replay_ms(g):
        g.replay()
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(3):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        return best

    return max(replay_ms(g_op) - replay_ms(g_flush), 1e-6) / iters


def _quant_components(q, synth, torch, dev, flush, peaks, out, qn, qk, sfx):
    """Quantize (plain and double quant) and dequantize of one [qn, qk] weight with outliers."""
    W = synth.weight(qn, qk, outlier_frac=0.001).to(dev)
    ne = W.numel()
    for mode, tag in ((q.QLORA_SCALE_BF16, "bf16"), (q.QLORA_SCALE_DQ_FP8, "dq_fp8")):
        qw = q.QuantizedWeight(qn, qk, mode, device=dev)
        ws = torch.empty(max(1, q.qlora_nf4_quantize_workspace_bytes(qn, qk, mode)), dtype=torch.uint8,
                         device=dev)
        fn = lambda: q.qlora_nf4_quantize(W, qw, ws)
        for _ in range(3):
            fn()
        ms = graph_time(fn, 20, flush)
        scale_b = 2.0 / 64 if mode == q.QLORA_SCALE_BF16 else 1.0 / 64 + 4.0 / 16384
        algo = ne * (4.0 + 0.5 + scale_b)
        out[f"quantize_{tag}{sfx}"] = {"us": ms * 1e3, "gbs": algo / ms / 1e6,
                                       "frac": algo / ms / 1e6 / peaks["hbm_gbs"], "algo_bytes": algo}
        o_ = torch.empty(qn, qk, dtype=torch.bfloat16, device=dev)
        fn = lambda: q.qlora_nf4_dequantize(qw, o_)
        for _ in range(3):
            fn()
        ms = graph_time(fn, 20, flush)
        algo = ne * (0.5 + scale_b + 2.0)
        out[f"dequantize_{tag}{sfx}"] = {"us": ms * 1e3, "gbs": algo / ms / 1e6,
                                         "frac": algo / ms / 1e6 / peaks["hbm_gbs"], "algo_bytes": algo}


def _seven_b_components(q, synth, torch, dev, flush, peaks, out):
    """7B shapes: q_proj fwd+bwd at 2048 tokens (4096 x 4096) and the SiLU-gated MLP
    (gate/up 11008 x 4096, down 4096 x 11008) fwd+bwd at 4096 tokens, r = 64."""
    bf, f32 = torch.bfloat16, torch.float32
    peak = peaks.get("bf16_tflops", 1590.0)

    def mk(n, k, layer):
        W = synth.weight(n, k, layer=layer).to(dev)
        qw = q.QuantizedWeight(n, k, q.QLORA_SCALE_DQ_FP8, device=dev)
        q.qlora_nf4_quantize(W, qw)
        a, b = synth.lora_pair(RANK_R, k, n, layer=layer)
        return qw, a.to(dev), b.to(dev)

    # config 3: 7B q_proj, X 2048 x 4096
    M, N, K = 2048, 4096, 4096
    qw, a, b = mk(N, K, 40)
    X = synth.activations(M, K, layer=40).to(dev)
    dY = synth.grad_output(M, N, layer=40).to(dev)
    Y = torch.empty(M, N, dtype=bf, device=dev)
    U = torch.empty(M, RANK_R, dtype=f32, device=dev)
    dX = torch.empty(M, K, dtype=bf, device=dev)
    dA = torch.empty(RANK_R, K, dtype=f32, device=dev)
    dB = torch.empty(N, RANK_R, dtype=f32, device=dev)
    ws = torch.empty(q.qlora_linear_workspace_bytes(M, N, K, RANK_R), dtype=torch.uint8, device=dev)

    def qproj():
        q.qlora_linear_fwd(qw, X, a, b, RANK_R, ALPHA, Y, q.QLORA_DTYPE_BF16, U, ws)
        q.qlora_linear_bwd(qw, X, dY, a, b, RANK_R, ALPHA, U, dX, q.QLORA_DTYPE_BF16, dA, dB, 0, ws)
    for _ in range(3):
        qproj()
    ms = graph_time(qproj, 10, flush)
    fl = linear_flops(M, N, K, RANK_R, True)
    out["q_proj_7b_fwd_bwd"] = {"us": ms * 1e3, "tflops": fl / ms / 1e9, "tokens_per_s": M / (ms * 1e-3),
                                "frac_bf16_burst": fl / ms / 1e9 / peak, "flops": fl, "tokens": M}
    del qw, X, dY, Y, U, dX, dA, dB, ws
    # config 4: 7B MLP, 4096 tokens, gate/up 11008 x 4096, down 4096 x 11008, SiLU between
    M, H, I = 4096, 4096, 11008
    lay = {"gate": mk(I, H, 41), "up": mk(I, H, 42), "down": mk(H, I, 43)}
    X = synth.activations(M, H, layer=41).to(dev)
    dY = synth.grad_output(M, H, layer=43).to(dev)
    e = lambda *sh, dt=bf: torch.empty(*sh, dtype=dt, device=dev)
    g, u, h, y, dh, dg, du, dx = e(M, I), e(M, I), e(M, I), e(M, H), e(M, I), e(M, I), e(M, I), e(M, H)
    Us = {nm: e(M, RANK_R, dt=f32) for nm in lay}
    dAs = {nm: e(RANK_R, lay[nm][0].k, dt=f32) for nm in lay}
    dBs = {nm: e(lay[nm][0].n, RANK_R, dt=f32) for nm in lay}
    ws = torch.empty(max(q.qlora_linear_workspace_bytes(M, I, H, RANK_R), q.qlora_linear_workspace_bytes(M, H, I, RANK_R),
                         q.qlora_linear_group_workspace_bytes(M, [I, I], H, RANK_R)), dtype=torch.uint8, device=dev)

    def fwd(nm, x, yy):
        qw_, a_, b_ = lay[nm]
        q.qlora_linear_fwd(qw_, x, a_, b_, RANK_R, ALPHA, yy, q.QLORA_DTYPE_BF16, Us[nm], ws)

    def bwd(nm, x, dy, dxx, acc):
        qw_, a_, b_ = lay[nm]
        q.qlora_linear_bwd(qw_, x, dy, a_, b_, RANK_R, ALPHA, Us[nm], dxx, q.QLORA_DTYPE_BF16, dAs[nm], dBs[nm],
                           q.QLORA_BWD_ACCUMULATE_DX if acc else 0, ws)

    def mlp():
        fwd("gate", X, g)
        fwd("up", X, u)
        q.qlora_silu_gate_fwd(g, u, h)
        fwd("down", h, y)
        bwd("down", h, dY, dh, False)
        q.qlora_silu_gate_bwd(dh, g, u, dg, du)
        # gate and up read the same X: one grouped backward forms dX
        gu = ("gate", "up")
        q.qlora_linear_bwd_group([lay[nm][0] for nm in gu], X, [dg, du], [lay[nm][1] for nm in gu],
                                 [lay[nm][2] for nm in gu], RANK_R, ALPHA, [Us[nm] for nm in gu], dx,
                                 q.QLORA_DTYPE_BF16, [dAs[nm] for nm in gu], [dBs[nm] for nm in gu], 0, ws)
    for _ in range(2):
        mlp()
    ms = graph_time(mlp, 3, flush)
    fl = 2 * linear_flops(M, I, H, RANK_R, True) + linear_flops(M, H, I, RANK_R, True)
    out["mlp_7b_fwd_bwd"] = {"us": ms * 1e3, "tflops": fl / ms / 1e9, "tokens_per_s": M / (ms * 1e-3),
                             "frac_bf16_burst": fl / ms / 1e9 / peak, "flops": fl, "tokens": M}


def components(dev, peaks) -> dict:
    """Quantize / dequantize (4096 x 4096 and 22016 x 8192, with outliers) and M = 16 forward of
    the 65B q_proj, each against the measured HBM copy bandwidth. Timed by
    CUDA-graph replay so per-call host work (binding, tensor-map encoding)
    does not count; L2 is flushed before every call."""
    import torch
    import bit_nf4_quantized_03_b200 as q
    from bit_nf4_quantized_03_b200 import synth
    out = {}
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for qn, qk, sfx in ((4096, 4096, ""), (22016, 8192, "_65b_gate")):
        _quant_components(q, synth, torch, dev, flush, peaks, out, qn, qk, sfx)
    # what a plain device copy reaches when it moves the same bytes as the 4096 x 4096
    # quantize (76 MB) and dequantize (42 MB), timed the same way: the bandwidth a kernel of
    # this size can see, beside the 2 GB copy the peak comes from
    for tag in ("quantize_bf16", "dequantize_bf16"):
        half = int(out[tag]["algo_bytes"]) // 2 // 16 * 16
        src = torch.empty(half, dtype=torch.uint8, device=dev)
        dst = torch.empty(half, dtype=torch.uint8, device=dev)
        fn = lambda: dst.copy_(src)
        for _ in range(3):
            fn()
        ms = graph_time(fn, 20, flush)
        out[f"copy_same_bytes_as_{tag}"] = {"us": ms * 1e3, "gbs": 2 * half / ms / 1e6,
                                            "frac": 2 * half / ms / 1e6 / peaks["hbm_gbs"], "bytes_moved": 2 * half}
        del src, dst
    _seven_b_components(q, synth, torch, dev, flush, peaks, out)
    # the NF4 expansion alone on every SM: the ceiling on the weight rate of any kernel that
    # turns each weight into BF16 through the per-block table
    per_clk, per_s = q.qlora_expand_rate(4096)
    out["expansion_ceiling"] = {"weights_per_sm_clock": per_clk, "gweights_per_s": per_s / 1e9,
                                "note": "nf4_build_lut + nf4_lookup8 per 64-block, codes from shared memory, "
                                        "one CTA of 512 threads per SM, nothing else running"}
    # weight-stream bound forward at M = 16 (65B q_proj)
    n, k = 8192, 8192
    W = synth.weight(n, k).to(dev)
    qw = q.QuantizedWeight(n, k, q.QLORA_SCALE_DQ_FP8, device=dev)
    q.qlora_nf4_quantize(W, qw)
    del W
    a, b = synth.lora_pair(RANK_R, k, n)
    a, b = a.to(dev), b.to(dev)
    x = synth.activations(M_SMALL, k).to(dev)
    y = torch.empty(M_SMALL, n, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(q.qlora_linear_workspace_bytes(M_SMALL, n, k, RANK_R), dtype=torch.uint8, device=dev)
    fn = lambda: q.qlora_linear_fwd(qw, x, a, b, RANK_R, ALPHA, y, q.QLORA_DTYPE_BF16, None, ws)
    for _ in range(3):
        fn()
    ms = graph_time(fn, 50, flush)
    algo = n * k * (0.5 + 1.0 / 64 + 4.0 / 16384) + 2.0 * M_SMALL * (k + n) + 2.0 * RANK_R * (k + n)
    out["fwd_m16_q_proj"] = {"us": ms * 1e3, "gbs": algo / ms / 1e6, "frac": algo / ms / 1e6 / peaks["hbm_gbs"],
                             "algo_bytes": algo,
                             "expansion_frac": n * k / (ms * 1e-3) / per_s,
                             "expansion_bound_us": n * k / per_s * 1e6}
    # LoRA dropout (p = 0.05): q_proj forward + backward at 8192 tokens with and without it
    M = M_TOKENS
    X = synth.activations(M, k).to(dev)
    dY = synth.grad_output(M, n).to(dev)
    Yb = torch.empty(M, n, dtype=torch.bfloat16, device=dev)
    dXb = torch.empty(M, k, dtype=torch.bfloat16, device=dev)
    Ub = torch.empty(M, RANK_R, dtype=torch.float32, device=dev)
    dAb = torch.empty(RANK_R, k, dtype=torch.float32, device=dev)
    dBb = torch.empty(n, RANK_R, dtype=torch.float32, device=dev)
    mask = torch.empty(M * k // 8, dtype=torch.uint8, device=dev)
    drop = q.Dropout(0.05, 1234, 0, mask)
    wsd = torch.empty(q.qlora_linear_workspace_bytes_ex(M, n, k, RANK_R, drop), dtype=torch.uint8, device=dev)
    times = {}
    for tag, d in (("plain", None), ("dropout", drop)):
        def fb(d=d):
            q.qlora_linear_fwd_ex(qw, X, a, b, RANK_R, ALPHA, Yb, q.QLORA_DTYPE_BF16, Ub, d, wsd)
            q.qlora_linear_bwd_ex(qw, X, dY, a, b, RANK_R, ALPHA, Ub, dXb, q.QLORA_DTYPE_BF16, dAb, dBb, 0, d, wsd)
        for _ in range(2):
            fb()
        times[tag] = graph_time(fb, 3, flush)
    out["dropout_fwd_bwd_q_proj"] = {"us": times["dropout"] * 1e3, "us_without": times["plain"] * 1e3,
                                     "overhead": times["dropout"] / times["plain"] - 1.0, "p": 0.05,
                                     "tokens": M}
    del X, dY, Yb, dXb, wsd
    # paged AdamW over one decoder layer's adapters (r = 64: q/k/v/o 64 x (8192 + 8192), gate/up/down
    # 64 x (8192 + 22016)); 30 bytes per parameter: p, g, m, v read; p, m, v and the bf16 copy written
    count = sum(RANK_R * (nn + kk) for _, nn, kk in LAYERS)
    algo = 30.0 * count
    grad = torch.randn(count, device=dev) * 1e-2
    pbf = torch.empty(count, dtype=torch.bfloat16, device=dev)
    dev_states = [torch.zeros(count, device=dev) for _ in range(3)]
    cfg = q.AdamWConfig(2e-4, 10, weight_decay=0.01)
    fn = lambda: q.qlora_adamw_step(dev_states[0], grad, dev_states[1], dev_states[2], pbf, count, cfg)
    for _ in range(3):
        fn()
    ms = graph_time(fn, 20, flush)
    out["adamw_layer_adapters"] = {"us": ms * 1e3, "gbs": algo / ms / 1e6, "frac": algo / ms / 1e6 / peaks["hbm_gbs"],
                                   "algo_bytes": algo, "params": count}
    nbytes = count * 4
    addrs = [q.qlora_paged_alloc(nbytes) for _ in range(3)]
    try:
        for addr in addrs:
            q.qlora_paged_prefetch(addr, nbytes)
        fnp = lambda: q.qlora_adamw_step(addrs[0], grad, addrs[1], addrs[2], pbf, count, cfg)
        for _ in range(3):
            fnp()
        msp = graph_time(fnp, 20, flush)
        # page the three state arrays out to host RAM and back in (the paging cost of one step)
        torch.cuda.synchronize()
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        e0.record()
        for addr in addrs:
            q.qlora_paged_prefetch(addr, nbytes, to_host=True)
        e1.record()
        for addr in addrs:
            q.qlora_paged_prefetch(addr, nbytes)
        e2.record()
        torch.cuda.synchronize()
        out["adamw_layer_adapters_paged"] = {
            "us": msp * 1e3, "gbs": algo / msp / 1e6, "frac": algo / msp / 1e6 / peaks["hbm_gbs"],
            "algo_bytes": algo, "params": count, "page_out_us": e0.elapsed_time(e1) * 1e3,
            "page_in_us": e1.elapsed_time(e2) * 1e3, "paged_bytes": 3 * nbytes}
    finally:
        torch.cuda.synchronize()
        for addr in addrs:
            q.qlora_paged_free(addr)
    del grad, pbf, dev_states
    # adapter merge onto the dequantized weight (65B q_proj, bf16 output)
    wm = torch.empty(n, k, dtype=torch.bfloat16, device=dev)
    fn = lambda: q.qlora_lora_merge(qw, a, b, RANK_R, ALPHA, wm, q.QLORA_DTYPE_BF16)
    for _ in range(3):
        fn()
    ms = graph_time(fn, 10, flush)
    algo = n * k * (0.5 + 1.0 / 64 + 4.0 / 16384 + 2.0) + 2.0 * RANK_R * (k + n)
    out["merge_q_proj"] = {"us": ms * 1e3, "gbs": algo / ms / 1e6, "frac": algo / ms / 1e6 / peaks["hbm_gbs"],
                           "algo_bytes": algo}
    return out


def run_case(args) -> None:
    """One named launch sequence for profiling (a few launches, no JSON line)."""
    import torch
    import bit_nf4_quantized_03_b200 as q
    from bit_nf4_quantized_03_b200 import build, synth
    build.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    name = args.case
    if name in ("fwd_q_65b", "bwd_q_65b", "fwd_m16_q_65b", "fwd_gate_65b", "bwd_down_65b"):
        lay = {"fwd_q_65b": LAYERS[0], "bwd_q_65b": LAYERS[0], "fwd_m16_q_65b": LAYERS[0],
               "fwd_gate_65b": LAYERS[4], "bwd_down_65b": LAYERS[6]}[name]
        _, n, k = lay
        m = M_SMALL if name == "fwd_m16_q_65b" else M_TOKENS
        W = synth.weight(n, k).to(dev)
        qw = q.QuantizedWeight(n, k, q.QLORA_SCALE_DQ_FP8, device=dev)
        q.qlora_nf4_quantize(W, qw)
        del W
        a, b = (t.to(dev) for t in synth.lora_pair(RANK_R, k, n))
        x = synth.activations(m, k).to(dev)
        dy = synth.grad_output(m, n).to(dev)
        y = torch.empty(m, n, dtype=torch.bfloat16, device=dev)
        dx = torch.empty(m, k, dtype=torch.bfloat16, device=dev)
        u = torch.empty(m, RANK_R, dtype=torch.float32, device=dev)
        da = torch.empty(RANK_R, k, dtype=torch.float32, device=dev)
        db = torch.empty(n, RANK_R, dtype=torch.float32, device=dev)
        ws = torch.empty(q.qlora_linear_workspace_bytes(m, n, k, RANK_R), dtype=torch.uint8, device=dev)
        q.qlora_linear_fwd(qw, x, a, b, RANK_R, ALPHA, y, q.QLORA_DTYPE_BF16, u, ws)
        for _ in range(args.case_iters):
            if name.startswith("bwd"):
                q.qlora_linear_bwd(qw, x, dy, a, b, RANK_R, ALPHA, u, dx, q.QLORA_DTYPE_BF16, da, db, 0, ws)
            else:
                q.qlora_linear_fwd(qw, x, a, b, RANK_R, ALPHA, y, q.QLORA_DTYPE_BF16, u, ws)
    elif name == "bwd_qkv_group_65b":
        # the grouped q/k/v backward at 8192 tokens (three 8192 x 8192 weights sharing X)
        n, k = LAYERS[0][1], LAYERS[0][2]
        mem = []
        for i in range(3):
            W = synth.weight(n, k, layer=i).to(dev)
            qw = q.QuantizedWeight(n, k, q.QLORA_SCALE_DQ_FP8, device=dev)
            q.qlora_nf4_quantize(W, qw)
            del W
            a, b = (t.to(dev) for t in synth.lora_pair(RANK_R, k, n, layer=i))
            mem.append((qw, a, b, synth.grad_output(M_TOKENS, n, layer=20 + i).to(dev)))
        x = synth.activations(M_TOKENS, k).to(dev)
        dx = torch.empty(M_TOKENS, k, dtype=torch.bfloat16, device=dev)
        grads = [(torch.empty(RANK_R, k, device=dev), torch.empty(n, RANK_R, device=dev)) for _ in mem]
        ws = torch.empty(q.qlora_linear_group_workspace_bytes(M_TOKENS, [n] * 3, k, RANK_R), dtype=torch.uint8,
                         device=dev)
        for _ in range(1 + args.case_iters):
            q.qlora_linear_bwd_group([m_[0] for m_ in mem], x, [m_[3] for m_ in mem], [m_[1] for m_ in mem],
                                     [m_[2] for m_ in mem], RANK_R, ALPHA, None, dx, q.QLORA_DTYPE_BF16,
                                     [g[0] for g in grads], [g[1] for g in grads], 0, ws)
    elif name == "q_proj_7b":
        # 7B q_proj fwd+bwd at 2048 tokens (4096 x 4096, r = 64)
        M, N, K = 2048, 4096, 4096
        W = synth.weight(N, K, layer=40).to(dev)
        qw = q.QuantizedWeight(N, K, q.QLORA_SCALE_DQ_FP8, device=dev)
        q.qlora_nf4_quantize(W, qw)
        del W
        a, b = (t.to(dev) for t in synth.lora_pair(RANK_R, K, N, layer=40))
        x = synth.activations(M, K, layer=40).to(dev)
        dy = synth.grad_output(M, N, layer=40).to(dev)
        y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        dx = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
        u = torch.empty(M, RANK_R, dtype=torch.float32, device=dev)
        da = torch.empty(RANK_R, K, dtype=torch.float32, device=dev)
        db = torch.empty(N, RANK_R, dtype=torch.float32, device=dev)
        ws = torch.empty(q.qlora_linear_workspace_bytes(M, N, K, RANK_R), dtype=torch.uint8, device=dev)
        for _ in range(1 + args.case_iters):
            q.qlora_linear_fwd(qw, x, a, b, RANK_R, ALPHA, y, q.QLORA_DTYPE_BF16, u, ws)
            q.qlora_linear_bwd(qw, x, dy, a, b, RANK_R, ALPHA, u, dx, q.QLORA_DTYPE_BF16, da, db, 0, ws)
    elif name == "dropout_q_65b":
        n, k = LAYERS[0][1], LAYERS[0][2]
        m = M_TOKENS
        W = synth.weight(n, k).to(dev)
        qw = q.QuantizedWeight(n, k, q.QLORA_SCALE_DQ_FP8, device=dev)
        q.qlora_nf4_quantize(W, qw)
        del W
        a, b = (t.to(dev) for t in synth.lora_pair(RANK_R, k, n))
        x = synth.activations(m, k).to(dev)
        dy = synth.grad_output(m, n).to(dev)
        y = torch.empty(m, n, dtype=torch.bfloat16, device=dev)
        dx = torch.empty(m, k, dtype=torch.bfloat16, device=dev)
        u = torch.empty(m, RANK_R, dtype=torch.float32, device=dev)
        da = torch.empty(RANK_R, k, dtype=torch.float32, device=dev)
        db = torch.empty(n, RANK_R, dtype=torch.float32, device=dev)
        mask = torch.empty(m * k // 8, dtype=torch.uint8, device=dev)
        drop = q.Dropout(0.05, 1234, 0, mask)
        ws = torch.empty(q.qlora_linear_workspace_bytes_ex(m, n, k, RANK_R, drop), dtype=torch.uint8, device=dev)
        for _ in range(1 + args.case_iters):
            q.qlora_linear_fwd_ex(qw, x, a, b, RANK_R, ALPHA, y, q.QLORA_DTYPE_BF16, u, drop, ws)
            q.qlora_linear_bwd_ex(qw, x, dy, a, b, RANK_R, ALPHA, u, dx, q.QLORA_DTYPE_BF16, da, db, 0, drop, ws)
    elif name == "adamw_layer":
        count = sum(RANK_R * (nn + kk) for _, nn, kk in LAYERS)
        grad = torch.randn(count, device=dev) * 1e-2
        pbf = torch.empty(count, dtype=torch.bfloat16, device=dev)
        st = [torch.zeros(count, device=dev) for _ in range(3)]
        for t in range(1 + args.case_iters):
            q.qlora_adamw_step(st[0], grad, st[1], st[2], pbf, count, q.AdamWConfig(2e-4, t + 1, weight_decay=0.01))
    elif name == "merge_q_65b":
        n, k = LAYERS[0][1], LAYERS[0][2]
        W = synth.weight(n, k).to(dev)
        qw = q.QuantizedWeight(n, k, q.QLORA_SCALE_DQ_FP8, device=dev)
        q.qlora_nf4_quantize(W, qw)
        del W
        a, b = (t.to(dev) for t in synth.lora_pair(RANK_R, k, n))
        wm = torch.empty(n, k, dtype=torch.bfloat16, device=dev)
        for _ in range(1 + args.case_iters):
            q.qlora_lora_merge(qw, a, b, RANK_R, ALPHA, wm, q.QLORA_DTYPE_BF16)
    elif name == "quantize_8192":
        # plain (BF16-scale) quantize of a 65B q/k/v/o-shaped weight
        W = synth.weight(8192, 8192, outlier_frac=0.001).to(dev)
        qw = q.QuantizedWeight(8192, 8192, q.QLORA_SCALE_BF16, device=dev)
        for _ in range(1 + args.case_iters):
            q.qlora_nf4_quantize(W, qw)
    elif name in ("quantize_4096", "dequantize_4096"):
        W = synth.weight(4096, 4096, outlier_frac=0.001).to(dev)
        qw = q.QuantizedWeight(4096, 4096, q.QLORA_SCALE_DQ_FP8, device=dev)
        out = torch.empty(4096, 4096, dtype=torch.bfloat16, device=dev)
        q.qlora_nf4_quantize(W, qw)
        for _ in range(args.case_iters):
            if name == "quantize_4096":
                q.qlora_nf4_quantize(W, qw)
            else:
                q.qlora_nf4_dequantize(qw, out)
    else:
        raise SystemExit(f"unknown case {name}")
    torch.cuda.synchronize()
    q.qlora_check_device_error()
    print(f"case {name}: ok, {q.qlora_launch_count()} library launches", flush=True)


def run_native(args) -> None:
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from bit_nf4_quantized_03_b200 import build
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    import bit_nf4_quantized_03_b200 as q
    peaks = measured_peaks()
    barrier = (lambda: dist.barrier()) if world > 1 else None

    wl = Workload(dev)
    for _ in range(args.warmup):
        wl.step()
    q.qlora_check_device_error()

    # timed region: device time per step, L2 flushed between steps
    launches0 = q.qlora_launch_count()
    q.qlora_timing_begin(32 * args.steps)
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        ms = time_steps(wl.step, args.steps, wl.flush, barrier)
    gemm_ms_all, gemm_n_all, gemm_flops_all = q.qlora_timing_end()
    # the roofline's kernel: the fused-GEMM launches at 8192 tokens (CTA-pair kernel); the
    # 16-token forwards (single-CTA kernel, HBM-bound) are reported apart
    per_launch = q.qlora_timing_launches(gemm_n_all)
    big = [(t, f) for t, f in per_launch if f >= PAIR_FLOPS_MIN]
    small = [(t, f) for t, f in per_launch if f < PAIR_FLOPS_MIN]
    gemm_ms, gemm_n, gemm_flops = sum(t for t, _ in big), len(big), sum(f for _, f in big)
    launches = q.qlora_launch_count() - launches0
    q.qlora_check_device_error()
    ms = max_over_ranks(ms)
    flops = step_flops() * world
    value = flops / (ms * 1e-3) / 1e12
    tokens_per_s = M_TOKENS * world / (ms * 1e-3)

    # end to end through the public API: pinned host inputs -> device -> step -> gradients back to host
    def e2e_step():
        wl.h2d()
        wl.step()
        wl.d2h()
    e2e = None
    if not args.no_e2e:
        for _ in range(2):
            e2e_step()
        ms_e2e = max_over_ranks(time_e2e_pipelined(wl, args.steps, barrier))
        ms_h2d = max_over_ranks(time_h2d_alone(wl, 3, barrier))
        e2e = {"value": flops / (ms_e2e * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": wl.h2d_bytes,
               "d2h_bytes_per_step": wl.d2h_bytes, "ms_per_step": ms_e2e,
               "h2d_alone_ms": ms_h2d, "h2d_alone_gbs": wl.h2d_bytes / (ms_h2d * 1e-3) / 1e9,
               "copies": "every step's inputs H2D from pinned host on a copy stream and its adapter gradients D2H "
                         "on a second one, both overlapped with the neighbouring step's compute (double-buffered); "
                         "each input is awaited just before its first use, so the first step starts once its first "
                         "input has landed; h2d_alone_ms is one step's input copies with nothing else running"}

    peak_tc = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
    achieved = gemm_flops / (gemm_ms * 1e-3) / 1e12 if gemm_ms > 0 else None
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak_tc, "unit": "TFLOP/s",
                "frac": (achieved / peak_tc) if achieved else None, "traffic": wgemm_traffic(),
                "traffic_unit": "DRAM bytes per launch, average over the step's 11 CTA-pair launches (ncu): seven "
                                "forwards, four backwards (q/k/v and gate/up grouped)",
                "algorithmic_bytes_per_launch": pair_algo_bytes(),
                "kernel": "qlora_wgemm_pair_kernel (fused NF4 dequant + tcgen05 cta_group::2, 256 weight rows x 512 "
                          "tokens per CTA pair; forward Y and backward dX at 8192 tokens)",
                "launches_timed": gemm_n, "avg_launch_ms": gemm_ms / max(gemm_n, 1),
                "m16_launches": {"kernel": "qlora_wgemm_kernel (single CTA, 16 tokens)", "launches": len(small),
                                 "avg_launch_ms": sum(t for t, _ in small) / max(len(small), 1)},
                "peak_kind": f"bf16_tflops_sustained ({peaks['_source']})"}
    comp = None
    cpu = None
    if rank == 0 and world == 1:
        comp = None if args.no_components else components(dev, peaks)
        if not args.no_cpu_baseline:
            s = OracleSample()
            times = [s.step() for _ in range(args.cpu_steps)]
            v = s.flops * len(times) / sum(times) / 1e12
            cpu = {"value": v, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle", "sample": s.desc,
                   "extrapolated_step_ms": step_flops() / (v * 1e12) * 1e3,
                   "configs": oracle_configs()}
    if world > 1:
        dist.barrier()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD, "tokens_per_gpu": M_TOKENS, "small_m": M_SMALL, "r": RANK_R,
                       "alpha": ALPHA, "weights": "NF4 blk64 + DQ E4M3 blk256", "activations": "bf16",
                       "l2": "inputs larger than L2; 512 MiB written between timed steps",
                       "parallelism": f"dp{world}", "step_tflop": flops / 1e12 / world},
            "tokens_per_s": tokens_per_s,
            "roofline": roofline, "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches, "clocks": clk.summary(), "components": comp,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--cpu-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-components", action="store_true")
    ap.add_argument("--case", default=None, help="run one named launch sequence for profiling and exit")
    ap.add_argument("--case-iters", type=int, default=3)
    args = ap.parse_args(argv)
    if args.case:
        run_case(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_native(args)


if __name__ == "__main__":
    main()
