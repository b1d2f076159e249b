"""Token-sharded data parallelism on CPU ranks (gloo).

Each rank runs the oracle layer on its own contiguous slice of the tokens,
writes its adapter gradients into the flat buffer of
`bit_nf4_quantized_03_b200.dp.AdapterGrads`, and the ranks sum them with one
all-reduce. The summed dA, dB must equal the full-batch oracle's, and each
rank's Y, U and dX must equal the matching rows of the full-batch result
(those need no exchange). The exchange itself is the library's helper, the
layer arithmetic the oracle's, so this checks the partitioning, not the
kernels (the GPU side of the same contract is tests/test_gpu_linear.py::
test_token_shards_sum_to_full_batch)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

LAYERS = [("q_proj", 48, 128), ("down_proj", 64, 192)]
M_TOTAL = 37          # ragged: 19 + 18 tokens on two ranks, 13 + 12 + 12 on three
R, ALPHA = 8, 16.0


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _layer_inputs(i, n, k):
    from bit_nf4_quantized_03_b200 import synth
    from oracle import nf4_oracle as o
    W = synth.weight(n, k, layer=i).numpy()
    Wd = o.dequantize_f64(o.quantize(W, o.MODE_DQ_FP8), (n, k))
    X = synth.activations(M_TOTAL, k, layer=i)
    dY = synth.grad_output(M_TOTAL, n, layer=i)
    A, B = synth.lora_pair(R, k, n, layer=i)
    return Wd, X, dY, A, B


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from bit_nf4_quantized_03_b200 import dp
    from oracle import nf4_oracle as o
    assert dp.world() == (rank, world)
    lo, hi = dp.token_shard(M_TOTAL, rank, world)
    grads = dp.AdapterGrads(LAYERS, R)
    local = {}
    for i, (name, n, k) in enumerate(LAYERS):
        Wd, X, dY, A, B = _layer_inputs(i, n, k)
        Y, U = o.linear_forward(Wd, X[lo:hi], A, B, ALPHA)
        dX, dA, dB = o.linear_backward(Wd, X[lo:hi], dY[lo:hi], A, B, ALPHA)
        grads.dA[name].copy_(torch.from_numpy(dA))
        grads.dB[name].copy_(torch.from_numpy(dB))
        local[name] = (Y, U, dX)
    grads.all_reduce()
    t = dp.max_over_ranks(1.5 + rank)
    out[rank] = {"range": (lo, hi), "t": t,
                 "dA": {nm: grads.dA[nm].double().numpy() for nm, _, _ in LAYERS},
                 "dB": {nm: grads.dB[nm].double().numpy() for nm, _, _ in LAYERS},
                 "local": local}
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_token_shards_sum_to_the_full_batch(world):
    from oracle import nf4_oracle as o
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    ranges = [out[r]["range"] for r in range(world)]
    # the shards tile the tokens in order, sizes differing by at most one
    assert ranges[0][0] == 0 and ranges[-1][1] == M_TOTAL
    assert all(ranges[i][1] == ranges[i + 1][0] for i in range(world - 1))
    sizes = [b - a for a, b in ranges]
    assert max(sizes) - min(sizes) <= 1
    for i, (name, n, k) in enumerate(LAYERS):
        Wd, X, dY, A, B = _layer_inputs(i, n, k)
        Y, U = o.linear_forward(Wd, X, A, B, ALPHA)
        dX, dA, dB = o.linear_backward(Wd, X, dY, A, B, ALPHA)
        for r in range(world):
            # fp32 buffer: the sum of fp32-rounded partials, so compare at fp32 resolution
            assert np.allclose(out[r]["dA"][name], dA, rtol=1e-6, atol=1e-6 * np.abs(dA).max())
            assert np.allclose(out[r]["dB"][name], dB, rtol=1e-6, atol=1e-6 * np.abs(dB).max())
            lo, hi = ranges[r]
            Yl, Ul, dXl = out[r]["local"][name]
            np.testing.assert_allclose(Yl, Y[lo:hi], rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(Ul, U[lo:hi], rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(dXl, dX[lo:hi], rtol=1e-12, atol=1e-12)
    for r in range(world):
        assert out[r]["t"] == 1.5 + (world - 1)       # max over ranks


def test_sum_of_shard_gradients_in_fp64_is_the_full_batch():
    # the exchange is a plain sum: in fp64 the shard partials add up to the full
    # batch to rounding (no process group needed for the arithmetic)
    from bit_nf4_quantized_03_b200 import dp
    from oracle import nf4_oracle as o
    name, n, k = LAYERS[0]
    Wd, X, dY, A, B = _layer_inputs(0, n, k)
    _, dA, dB = o.linear_backward(Wd, X, dY, A, B, ALPHA)
    sA, sB = np.zeros_like(dA), np.zeros_like(dB)
    for r in range(4):
        lo, hi = dp.token_shard(M_TOTAL, r, 4)
        _, a, b = o.linear_backward(Wd, X[lo:hi], dY[lo:hi], A, B, ALPHA)
        sA += a
        sB += b
    np.testing.assert_allclose(sA, dA, rtol=1e-12, atol=1e-12 * np.abs(dA).max())
    np.testing.assert_allclose(sB, dB, rtol=1e-12, atol=1e-12 * np.abs(dB).max())


def test_token_shard_edges():
    from bit_nf4_quantized_03_b200 import dp
    assert [dp.token_shard(5, r, 8) for r in range(8)] == [(0, 1), (1, 2), (2, 3), (3, 4), (4, 5), (5, 5),
                                                           (5, 5), (5, 5)]
    assert dp.token_shard(8192, 3, 8) == (3072, 4096)
    with pytest.raises(ValueError):
        dp.token_shard(10, 2, 2)


def test_single_process_helpers_are_identity():
    from bit_nf4_quantized_03_b200 import dp
    g = dp.AdapterGrads(LAYERS, R)
    g.flat.fill_(1.0)
    g.all_reduce()
    assert torch.all(g.flat == 1.0)
    assert g.dA["q_proj"].shape == (R, 128) and g.dB["down_proj"].shape == (64, R)
    assert dp.max_over_ranks(3.25) == 3.25
    assert dp.world() == (0, 1)
