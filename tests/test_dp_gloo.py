"""Data-parallel decomposition of the layer on CPU ranks (gloo, world size 2).

Each rank takes its own slice of the tokens, computes the adapter gradients
with the oracle, and the ranks sum dA and dB with an all-reduce: the result
equals the gradients of the whole batch.  This is the one exchange of the
multi-GPU path (the frozen weight needs none), exercised here without GPUs.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import synthetic
from oracle import lora, nf4


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        lay = synthetic.custom_layer(seed=1234, d=128, k=192, r=8, T=96, alpha=16.0)
        X = nf4.bf16_to_f64(lay.X)
        A = nf4.bf16_to_f64(lay.A)
        B = nf4.bf16_to_f64(lay.B)
        dY = nf4.bf16_to_f64(lay.dY)
        shard = np.array_split(np.arange(lay.T), world)[rank]
        g = lora.grad_adapters(X[shard], A, B, lay.s, dY[shard])
        dA = torch.from_numpy(g["dA"].copy())
        dB = torch.from_numpy(g["dB"].copy())
        dist.all_reduce(dA)
        dist.all_reduce(dB)
        if rank == 0:
            full = lora.grad_adapters(X, A, B, lay.s, dY)
            ok = (np.allclose(dA.numpy(), full["dA"], rtol=1e-12, atol=1e-12) and
                  np.allclose(dB.numpy(), full["dB"], rtol=1e-12, atol=1e-12))
            with open(out_path, "w") as f:
                f.write("ok" if ok else "mismatch")
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_token_sharding_sums_to_full_batch(tmp_path):
    out = str(tmp_path / "result.txt")
    mp.start_processes(_worker, args=(2, _free_port(), out), nprocs=2, join=True,
                       start_method="spawn")
    assert open(out).read() == "ok"
