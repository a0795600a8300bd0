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


def _adam_worker(rank, world, port, out_path):
    """Two data-parallel ranks take three optimiser steps: per step each rank forms
    the adapter gradients of its token shard, the ranks sum them (the one
    exchange), and each applies the same Adam step to its own replica of A
    and B.  The replicas stay identical and equal a single process that sees
    the whole batch."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import adam
        lay = synthetic.custom_layer(seed=77, d=96, k=64, r=4, T=64, alpha=8.0)
        X = nf4.bf16_to_f64(lay.X)
        dY = nf4.bf16_to_f64(lay.dY)
        Wp = np.zeros((lay.d, lay.k))
        shard = np.array_split(np.arange(lay.T), world)[rank]
        mine = {"A": nf4.bf16_to_f64(lay.A), "B": nf4.bf16_to_f64(lay.B)}
        ref = {n: v.copy() for n, v in mine.items()}
        st_m = {n: (np.zeros_like(v), np.zeros_like(v)) for n, v in mine.items()}
        ref_m = {n: (np.zeros_like(v), np.zeros_like(v)) for n, v in ref.items()}
        for t in range(1, 4):
            g = lora.grad_adapters(X[shard], mine["A"], mine["B"], lay.s, dY[shard])
            grads = {"A": torch.from_numpy(g["dA"].copy()), "B": torch.from_numpy(g["dB"].copy())}
            for n in ("A", "B"):
                dist.all_reduce(grads[n])
                out = adam.adam_step(mine[n], *st_m[n], grads[n].numpy(), t=t, lr=1e-3)
                mine[n], st_m[n] = out["theta"], (out["m"], out["v"])
            gf = lora.grad_adapters(X, ref["A"], ref["B"], lay.s, dY)
            for n, gn in (("A", gf["dA"]), ("B", gf["dB"])):
                out = adam.adam_step(ref[n], *ref_m[n], gn, t=t, lr=1e-3)
                ref[n], ref_m[n] = out["theta"], (out["m"], out["v"])
        # replicas agree across ranks bit for bit, and match the whole-batch run
        both = {n: [torch.zeros(v.shape, dtype=torch.float64) for _ in range(world)] for n, v in mine.items()}
        for n in mine:
            dist.all_gather(both[n], torch.from_numpy(mine[n].copy()))
        if rank == 0:
            same = all(torch.equal(both[n][0], both[n][1]) for n in mine)
            close = all(np.allclose(mine[n], ref[n], rtol=1e-10, atol=1e-12) for n in mine)
            with open(out_path, "w") as f:
                f.write("ok" if same and close else f"same={same} close={close}")
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_adam_keeps_replicas_identical(tmp_path):
    out = str(tmp_path / "adam.txt")
    mp.start_processes(_adam_worker, args=(2, _free_port(), out), nprocs=2, join=True,
                       start_method="spawn")
    assert open(out).read() == "ok"


def _id_worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import parameter_efficient_fine_nf4_b200 as q4
        # the library's communicator set-up without a GPU: rank 0 draws the
        # NCCL id, the group shares it, every rank gets (id, nranks, rank)
        got = q4.communicator_from_process_group(make=lambda uid, n, r: (uid, n, r))
        with open(os.path.join(out_dir, f"rank{rank}.bin"), "wb") as f:
            f.write(got[0] + bytes([got[1], got[2]]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_communicator_id_is_shared_by_all_ranks(tmp_path):
    q4 = pytest.importorskip("parameter_efficient_fine_nf4_b200")
    q4.lib()
    mp.start_processes(_id_worker, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    r0 = open(tmp_path / "rank0.bin", "rb").read()
    r1 = open(tmp_path / "rank1.bin", "rb").read()
    assert len(r0) == len(r1) == q4.NCCL_ID_BYTES + 2
    assert r0[:q4.NCCL_ID_BYTES] == r1[:q4.NCCL_ID_BYTES]          # one id for the group
    assert (r0[-2], r0[-1]) == (2, 0) and (r1[-2], r1[-1]) == (2, 1)
