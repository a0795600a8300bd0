"""The C-ABI library loads, exports every symbol include/qlora.h declares, and
its host-only parts agree with the oracle.  No kernel is launched here."""
import ctypes
import os
import re

import numpy as np
import pytest

import parameter_efficient_fine_nf4_b200 as q4
from oracle import nf4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from parameter_efficient_fine_nf4_b200 import build
    build.build()
    return q4.lib()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "qlora.h")).read()
    return sorted(set(re.findall(r"^QLORA_API\s+[\w\s\*]+?\b((?:qlora|lora)_\w+)\s*\(", text, re.M)))


def test_header_declares_the_path():
    names = declared_symbols()
    for required in ("qlora_nf4_quantize", "qlora_nf4_dequantize", "qlora_fwd", "qlora_bwd",
                     "lora_merge", "lora_unmerge"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert len(names) >= 18
    for n in names:
        assert hasattr(lib, n), n
    # the binding wraps exactly the declared set
    assert set(q4.EXPORTED) == set(names)


def test_library_levels_equal_oracle_bit_for_bit(lib):
    levels, thr = q4.qlora_nf4_levels()
    lv = np.array(levels, np.float32)
    assert np.array_equal(lv.view(np.uint32), nf4.nf4_levels().view(np.uint32))
    # thresholds: counting thresholds <= x equals the oracle's nearest level
    # (ties low) for every fp32 x within 2048 ulps of each threshold
    t = np.array(thr, np.float32)
    xs = []
    for ti in t:
        bits = ti.view(np.uint32).astype(np.int64)
        if ti > 0:
            rng_bits = np.arange(bits - 2048, bits + 2048)
        else:
            rng_bits = np.arange(bits - 2048, bits + 2048)   # negative: bit order reversed, same set
        xs.append(rng_bits.astype(np.uint32).view(np.float32))
    x = np.concatenate(xs)
    x = x[np.abs(x) <= 1]
    x = x[: (x.size // 64) * 64]
    oracle_codes = nf4.encode_blocks(x.reshape(-1, 64), np.ones(x.size // 64, np.float32)).ravel()
    lib_codes = (x[:, None] >= t[None, :]).sum(axis=1)
    assert np.array_equal(oracle_codes, lib_codes)


def test_workspace_queries(lib):
    assert q4.qlora_quantize_workspace_bytes(256, 256) >= (256 * 256 // 64) * 4
    assert q4.lora_merge_workspace_bytes(256, 256, 8) >= 256 * 8 * 2
    assert q4.qlora_fwd_workspace_bytes(0, 256, 8, 16) == 0
    # the weight is dequantised inside the GEMM: neither workspace holds a
    # 16-bit copy of it (sU / hi-lo pairs, padded B and split-K partials only)
    # and the QLoRA workspaces equal the plain-LoRA ones
    d, k, r, T = 22016, 8192, 64, 16384
    for fn_q, fn_p in ((q4.qlora_fwd_workspace_bytes, q4.lora_fwd_workspace_bytes),
                       (q4.qlora_bwd_workspace_bytes, q4.lora_bwd_workspace_bytes)):
        assert fn_q(d, k, r, T) == fn_p(d, k, r, T)
        assert fn_q(d, k, r, T) < d * k * 2 // 4
    assert q4.qlora_fwd_workspace_bytes(d, k, r, T) >= T * r * 2
    assert q4.lora_fwd_workspace_bytes(4096, 4096, 8, 0) > 0


def test_argument_validation_without_device(lib):
    L = lib
    # unsupported shapes and bad arguments are rejected on the host before any launch
    nf = q4._NF4(16, 16, 16, 16, 256, 100, 64, 256)              # k % 64 != 0
    st = L.qlora_fwd(ctypes.byref(nf), 16, 16, 8, 16.0, 16, 16, 16, 16, 16, 1 << 20, None)
    assert st == 2
    nf = q4._NF4(16, 16, 16, 16, 256, 256, 64, 256)
    assert L.qlora_fwd(ctypes.byref(nf), 16, 16, 0, 16.0, 16, 16, 16, 16, 16, 1 << 20, None) == 2   # r = 0
    assert L.qlora_fwd(ctypes.byref(nf), 16, 16, 8, -1.0, 16, 16, 16, 16, 16, 1 << 20, None) == 1   # alpha
    assert L.qlora_fwd(ctypes.byref(nf), None, 16, 8, 16.0, 16, 16, 16, 16, 16, 1 << 20, None) == 1  # null A
    assert L.qlora_fwd(ctypes.byref(nf), 16, 16, 8, 16.0, 17, 16, 16, 16, 16, 1 << 20, None) == 3   # misaligned X
    assert L.qlora_fwd(ctypes.byref(nf), 16, 16, 8, 16.0, 16, 16, 16, 16, 16, 64, None) == 4        # workspace
    assert L.qlora_nf4_quantize(16, 256, 100, 64, ctypes.byref(nf), 16, 1 << 20, None) == 2
    assert L.qlora_nf4_quantize(16, 256, 256, 32, ctypes.byref(nf), 16, 1 << 20, None) == 2
    nf_bad = q4._NF4(16, 16, 16, 16, 256, 256, 32, 256)           # block != 64
    assert L.qlora_nf4_dequantize(ctypes.byref(nf_bad), 16, None) == 2
    assert q4.strerror(6) == "device wait timed out"
    # plain LoRA: k % 8, alignment, rank and workspace are checked on the host
    assert L.lora_fwd(16, 256, 100, 16, 16, 8, 16.0, 16, 16, 16, 16, 16, 1 << 20, None) == 2      # k % 8
    assert L.lora_fwd(17, 256, 256, 16, 16, 8, 16.0, 16, 16, 16, 16, 16, 1 << 20, None) == 3      # W
    assert L.lora_fwd(16, 256, 256, 16, 16, 0, 16.0, 16, 16, 16, 16, 16, 1 << 20, None) == 2      # r = 0
    assert L.lora_fwd(16, 256, 256, 16, 16, 8, 16.0, 16, 16, 16, 16, 16, 64, None) == 4           # workspace
    assert L.lora_bwd(16, 130, 256, 16, 16, 8, 16.0, 16, 16, 16, 16, 16, 16, 16, 16, 1 << 20,
                      None) == 2                                                                  # d % 8
    assert L.lora_bwd(None, 256, 256, 16, 16, 8, 16.0, 16, 16, 16, 16, 16, 16, 16, 16, 1 << 20,
                      None) == 1                                                                  # null W
    # LoRA dropout: the rate and the mask are checked on the host first
    nf = q4._NF4(16, 16, 16, 16, 256, 256, 64, 256)
    for p in (1.0, 1.5, -0.1, float("nan")):
        assert L.qlora_fwd_dropout(ctypes.byref(nf), 16, 16, 8, 16.0, 16, 16, p, 16, 16, 16, 16,
                                   1 << 20, None) == 1
    assert L.qlora_fwd_dropout(ctypes.byref(nf), 16, 16, 8, 16.0, 16, None, 0.1, 16, 16, 16, 16,
                               1 << 20, None) == 1                                             # no mask
    assert L.qlora_fwd_dropout(ctypes.byref(nf), 16, 16, 8, 16.0, 16, 17, 0.1, 16, 16, 16, 16,
                               1 << 20, None) == 3                                             # misaligned mask
    assert L.qlora_bwd_dropout(ctypes.byref(nf), 16, 16, 8, 16.0, 16, None, 0.1, 16, 16, 16, 16, 16, 16,
                               16, 1 << 20, None) == 1
    assert L.qlora_fwd_dropout(ctypes.byref(nf), 16, 16, 8, 16.0, 16, 16, 0.1, 16, 16, 16, 16,
                               64, None) == 4                                                  # workspace
    assert q4.qlora_fwd_dropout_workspace_bytes(256, 256, 8, 16) > q4.qlora_fwd_workspace_bytes(256, 256, 8, 16)
    # several adapters: count, total rank and alphas are checked on the host
    al = (ctypes.c_float * 4)(16.0, 16.0, 16.0, 16.0)
    assert L.qlora_fwd_multi(ctypes.byref(nf), 0, 16, 16, 8, ctypes.addressof(al), 16, 16, 16, 16, 16,
                             16, 1 << 20, None) == 1                                           # n = 0
    assert L.qlora_fwd_multi(ctypes.byref(nf), 65, 16, 16, 1, ctypes.addressof(al), 16, 16, 16, 16, 16,
                             16, 1 << 20, None) == 1                                           # n > 64
    assert L.qlora_fwd_multi(ctypes.byref(nf), 4, 16, 16, 65, ctypes.addressof(al), 16, 16, 16, 16, 16,
                             16, 1 << 20, None) == 2                                           # n r > 256
    bad = (ctypes.c_float * 2)(16.0, -1.0)
    assert L.qlora_fwd_multi(ctypes.byref(nf), 2, 16, 16, 8, ctypes.addressof(bad), 16, 16, 16, 16, 16,
                             16, 1 << 20, None) == 1                                           # alpha <= 0
    assert L.qlora_bwd_multi(ctypes.byref(nf), 2, 16, 16, 8, ctypes.addressof(al), 18, 16, 16, 16, 16, 16,
                             16, 16, 16, 1 << 20, None) == 3                                   # misaligned idx
    # data parallel: communicator and gradient all-reduce arguments
    assert L.qlora_grad_allreduce(None, 16, 4, 16, 4, None) == 1                 # no communicator
    assert L.qlora_grad_allreduce(16, 16, -1, 16, 4, None) == 1                  # negative count
    assert L.qlora_grad_allreduce(16, None, 4, 16, 4, None) == 1                 # null dA
    assert L.qlora_comm_init(None, 2, 0, ctypes.byref(ctypes.c_void_p())) == 1
    assert L.qlora_comm_init(16, 2, 2, ctypes.byref(ctypes.c_void_p())) == 1     # rank outside [0, nranks)
    assert L.qlora_comm_destroy(None) == 1
    assert q4.strerror(9) == "NCCL unavailable or an NCCL call failed"
    # the NF4 GEMM build selector takes 0, 1 or 2
    assert L.qlora_set_nf4_gemm_mode(3) == 1 and L.qlora_set_nf4_gemm_mode(-1) == 1
    assert L.qlora_set_nf4_gemm_mode(2) == 0 and L.qlora_set_nf4_gemm_mode(0) == 0
    # Adam: step, betas, lr and alignment are checked on the host; n = 0 is a no-op
    assert L.lora_adam_step(16, 16, 16, 16, 16, 8, 0, 1e-3, 0.9, 0.999, 1e-8, 0.0, None) == 1     # step 0
    assert L.lora_adam_step(16, 16, 16, 16, 16, 8, 1, 1e-3, 1.0, 0.999, 1e-8, 0.0, None) == 1     # beta1 = 1
    assert L.lora_adam_step(16, 16, 16, 16, 16, 8, 1, -1.0, 0.9, 0.999, 1e-8, 0.0, None) == 1     # lr < 0
    assert L.lora_adam_step(16, 16, 16, 16, 16, 8, 1, float("nan"), 0.9, 0.999, 1e-8, 0.0, None) == 1
    assert L.lora_adam_step(16, 20, 16, 16, 16, 8, 1, 1e-3, 0.9, 0.999, 1e-8, 0.0, None) == 3     # bf16 copy
    assert L.lora_adam_step(None, 16, 16, 16, 16, 8, 1, 1e-3, 0.9, 0.999, 1e-8, 0.0, None) == 1   # null
    assert L.lora_adam_step(16, 16, 16, 16, 16, 0, 1, 1e-3, 0.9, 0.999, 1e-8, 0.0, None) == 0     # n = 0
