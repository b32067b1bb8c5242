"""Data-parallel replicas on disjoint token shards (the layout `bench.py --gpus
N` runs: every rank owns its own tokens and the full weights, no collective on
the data path), checked with the oracle on two `gloo` ranks on the CPU.

Tokens are independent units of the layer: a token's output row and its dX row
depend only on that token and the weights (x, h, dY and da are quantised
along H, I and 2I, within the token's own row), so each shard's rows equal the
full batch's rows bit for bit.  The weight gradients are sums over tokens: an
all-reduce of the shards' dW gives the full batch's dW -- exactly without
quantisation, and within the MXFP8 rounding when the wgrad operands are
quantised along tokens in 32-token blocks (blocks then run over each shard's
tokens of an expert rather than the whole batch's)."""
import os
import socket

import numpy as np

from mxfp8_grouped_gemm_x32_b200.workloads import bf16_bits_to_f32, get_config, make_inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    cfg = get_config("tiny", T=96, H=64, I=64, E=4, k=2)
    inp = make_inputs(cfg, seed=41)
    f64 = lambda k: bf16_bits_to_f32(inp[k]).astype(np.float64)
    return f64("x"), f64("w1"), f64("w2"), f64("dy"), inp["topk_idx"], inp["topk_prob"]


def _run(x, w1, w2, dy, idx, prob, quantize):
    from oracle import moe as omoe
    f = omoe.forward(x, w1, w2, idx, prob, quantize=quantize)
    b = omoe.backward(f, x, w1, w2, prob, dy, quantize=quantize)
    return f["out"], b["dX"], b["dW1"], b["dW2"]


def _rank_main(rank, world, port, out_dir):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x, w1, w2, dy, idx, prob = _inputs()
        sl = slice(rank * x.shape[0] // world, (rank + 1) * x.shape[0] // world)   # this rank's tokens
        for quantize in (False, True):
            out, dX, dW1, dW2 = _run(x[sl], w1, w2, dy[sl], idx[sl], prob[sl], quantize)
            g1, g2 = torch.from_numpy(dW1.copy()), torch.from_numpy(dW2.copy())
            dist.all_reduce(g1)
            dist.all_reduce(g2)
            np.savez(os.path.join(out_dir, f"r{rank}_q{int(quantize)}.npz"), out=out, dX=dX, dW1=g1.numpy(),
                     dW2=g2.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_data_parallel_shards_gloo(tmp_path):
    import torch.multiprocessing as mp
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    x, w1, w2, dy, idx, prob = _inputs()
    T = x.shape[0]
    for quantize in (False, True):
        out, dX, dW1, dW2 = _run(x, w1, w2, dy, idx, prob, quantize)
        shards = [np.load(tmp_path / f"r{r}_q{int(quantize)}.npz") for r in range(world)]
        assert np.array_equal(np.concatenate([s["out"] for s in shards]), out)
        assert np.array_equal(np.concatenate([s["dX"] for s in shards]), dX)
        for key, full in (("dW1", dW1), ("dW2", dW2)):
            red = shards[0][key]
            assert np.array_equal(red, shards[1][key])               # every rank holds the same sum
            rms = np.sqrt(np.mean(full ** 2))
            err = np.sqrt(np.mean((red - full) ** 2)) / rms
            if quantize:
                assert err <= 0.1, (key, err)                        # token blocks differ per shard
            else:
                assert err <= 1e-12, (key, err)                      # fp64 summation order only
    assert T % world == 0
