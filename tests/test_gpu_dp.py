"""The library's adapter-gradient all-reduce ([P1] "The update LoRA is allowed
to learn": the data-parallel layer's one exchange is the sum of dA and dB over
the ranks), on a one-rank NCCL communicator: the only form one GPU allows.
The sum over one rank is the input itself, bit for bit."""
import pytest
import torch

pytestmark = pytest.mark.gpu

q4 = pytest.importorskip("parameter_efficient_fine_nf4_b200")


def test_one_rank_allreduce_is_identity():
    torch.cuda.set_device(0)
    comm = q4.Communicator(q4.qlora_comm_unique_id(), 1, 0)
    try:
        g = torch.Generator(device="cuda").manual_seed(7)
        dA = torch.randn(64, 4096, device="cuda", generator=g)
        dB = torch.randn(11008, 64, device="cuda", generator=g)
        a0, b0 = dA.clone(), dB.clone()
        q4.qlora_grad_allreduce(comm, dA, dB)
        torch.cuda.synchronize()
        assert torch.equal(dA, a0) and torch.equal(dB, b0)
        # empty counts are allowed
        e = torch.empty(0, device="cuda")
        q4.qlora_grad_allreduce(comm, e, dB)
        torch.cuda.synchronize()
        assert torch.equal(dB, b0)
    finally:
        comm.close()
