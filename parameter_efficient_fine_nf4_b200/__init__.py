"""Python binding of libqlora (the QLoRA linear layer on B200).

Argument marshalling only: every step runs in the CUDA kernels of
``libqlora.so``, reached through its C ABI (``include/qlora.h``).  PyTorch
provides device memory and the current stream.  If the shared library is
missing the import of any call raises; there is no CPU fallback.

Names mirror the C entry points.  bf16 tensors are ``torch.bfloat16``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlora.so")

QLORA_OK = 0
QLORA_ERR_TIMEOUT = 6
BLOCK = 64
BLOCK2 = 256


class QloraError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {strerror(status)} (status {status})")


class _NF4(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("absmax_q", ctypes.c_void_p),
                ("scale2", ctypes.c_void_p), ("mean", ctypes.c_void_p),
                ("d", ctypes.c_int64), ("k", ctypes.c_int64),
                ("block", ctypes.c_int32), ("block2", ctypes.c_int32)]


class KernelStat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 48), ("launches", ctypes.c_int64),
                ("total_ms", ctypes.c_double), ("flops", ctypes.c_double),
                ("bytes", ctypes.c_double)]


_lib = None

_VP = ctypes.c_void_p
_I64 = ctypes.c_int64
_SIZE = ctypes.c_size_t
_INT = ctypes.c_int
_F = ctypes.c_float
_NF4P = ctypes.POINTER(_NF4)

_SIGNATURES = {
    "qlora_strerror": (ctypes.c_char_p, [_INT]),
    "qlora_version": (_INT, []),
    "qlora_nf4_levels": (_INT, [_VP, _VP]),
    "qlora_quantize_workspace_bytes": (_SIZE, [_I64, _I64]),
    "qlora_nf4_quantize": (_INT, [_VP, _I64, _I64, _INT, _NF4P, _VP, _SIZE, _VP]),
    "qlora_nf4_dequantize": (_INT, [_NF4P, _VP, _VP]),
    "qlora_nf4_quantize_noalloc": (_INT, [_VP, _I64, _I64, _INT, _NF4P, _VP]),
    "qlora_fwd_workspace_bytes": (_SIZE, [_I64, _I64, _INT, _I64]),
    "qlora_fwd": (_INT, [_NF4P, _VP, _VP, _INT, _F, _VP, _I64, _VP, _VP, _VP, _SIZE, _VP]),
    "qlora_bwd_workspace_bytes": (_SIZE, [_I64, _I64, _INT, _I64]),
    "qlora_bwd": (_INT, [_NF4P, _VP, _VP, _INT, _F, _VP, _VP, _VP, _I64, _VP, _VP, _VP, _VP,
                         _SIZE, _VP]),
    "qlora_fwd_dropout_workspace_bytes": (_SIZE, [_I64, _I64, _INT, _I64]),
    "qlora_fwd_dropout": (_INT, [_NF4P, _VP, _VP, _INT, _F, _VP, _VP, _F, _I64, _VP, _VP, _VP, _SIZE, _VP]),
    "qlora_bwd_dropout_workspace_bytes": (_SIZE, [_I64, _I64, _INT, _I64]),
    "qlora_bwd_dropout": (_INT, [_NF4P, _VP, _VP, _INT, _F, _VP, _VP, _F, _VP, _VP, _I64, _VP, _VP, _VP, _VP,
                                 _SIZE, _VP]),
    "qlora_fwd_multi_workspace_bytes": (_SIZE, [_I64, _I64, _INT, _INT, _I64]),
    "qlora_fwd_multi": (_INT, [_NF4P, _INT, _VP, _VP, _INT, _VP, _VP, _VP, _I64, _VP, _VP, _VP, _SIZE, _VP]),
    "qlora_bwd_multi_workspace_bytes": (_SIZE, [_I64, _I64, _INT, _INT, _I64]),
    "qlora_bwd_multi": (_INT, [_NF4P, _INT, _VP, _VP, _INT, _VP, _VP, _VP, _VP, _VP, _I64, _VP, _VP, _VP, _VP,
                               _SIZE, _VP]),
    "lora_fwd_workspace_bytes": (_SIZE, [_I64, _I64, _INT, _I64]),
    "lora_fwd": (_INT, [_VP, _I64, _I64, _VP, _VP, _INT, _F, _VP, _I64, _VP, _VP, _VP, _SIZE, _VP]),
    "lora_bwd_workspace_bytes": (_SIZE, [_I64, _I64, _INT, _I64]),
    "lora_bwd": (_INT, [_VP, _I64, _I64, _VP, _VP, _INT, _F, _VP, _VP, _VP, _I64, _VP, _VP, _VP, _VP,
                        _SIZE, _VP]),
    "lora_adam_step": (_INT, [_VP, _VP, _VP, _VP, _VP, _I64, _I64, _F, _F, _F, _F, _F, _VP]),
    "lora_merge_workspace_bytes": (_SIZE, [_I64, _I64, _INT]),
    "lora_merge": (_INT, [_NF4P, _VP, _VP, _INT, _F, _VP, _VP, _SIZE, _VP]),
    "lora_unmerge": (_INT, [_VP, _VP, _VP, _INT, _F, _I64, _I64, _VP, _VP, _SIZE, _VP]),
    "qlora_get_device_status": (_INT, [_VP, ctypes.POINTER(_INT)]),
    "qlora_selftest_wait_timeout": (_INT, [_INT, _VP]),
    "qlora_profile_begin": (_INT, []),
    "qlora_profile_end": (_INT, [ctypes.POINTER(KernelStat), _INT, ctypes.POINTER(_INT)]),
    "qlora_launch_count": (_I64, []),
    "qlora_set_nf4_gemm_mode": (_INT, [_INT]),
    "qlora_comm_unique_id": (_INT, [_VP]),
    "qlora_comm_init": (_INT, [_VP, _INT, _INT, ctypes.POINTER(_VP)]),
    "qlora_comm_destroy": (_INT, [_VP]),
    "qlora_grad_allreduce": (_INT, [_VP, _VP, _I64, _VP, _I64, _VP]),
}

EXPORTED = tuple(_SIGNATURES)


def lib() -> ctypes.CDLL:
    """Load libqlora.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"libqlora.so not found at {LIB_PATH}; build it with "
                "`python -m parameter_efficient_fine_nf4_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def strerror(status: int) -> str:
    return lib().qlora_strerror(int(status)).decode()


def _check(status: int, what: str):
    if status != QLORA_OK:
        raise QloraError(status, what)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(int(stream.cuda_stream))


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libqlora must be contiguous")
    return t.data_ptr()


def _need(t: torch.Tensor, dtype, shape, name):
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")


class NF4Weight:
    """Device buffers of one NF4 + double-quant weight (the qlora_nf4_t)."""

    def __init__(self, d: int, k: int, device=None):
        device = torch.device("cuda") if device is None else torch.device(device)
        n_b = d * k // BLOCK
        n_g = (n_b + BLOCK2 - 1) // BLOCK2
        self.d, self.k = d, k
        self.codes = torch.empty(d * k // 2, dtype=torch.uint8, device=device)
        self.absmax_q = torch.empty(n_b, dtype=torch.uint8, device=device)
        self.scale2 = torch.empty(n_g, dtype=torch.float32, device=device)
        self.mean = torch.empty(1, dtype=torch.float32, device=device)
        self._c = _NF4(self.codes.data_ptr(), self.absmax_q.data_ptr(), self.scale2.data_ptr(),
                       self.mean.data_ptr(), d, k, BLOCK, BLOCK2)

    @property
    def cstruct(self) -> _NF4:
        return self._c

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.codes, self.absmax_q, self.scale2, self.mean))


def workspace(nbytes: int, device=None) -> torch.Tensor:
    device = torch.device("cuda") if device is None else torch.device(device)
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


# ------------------------------------------------------------------- host-only
def qlora_version() -> int:
    return lib().qlora_version()


def qlora_nf4_levels():
    lv = (ctypes.c_float * 16)()
    th = (ctypes.c_float * 15)()
    _check(lib().qlora_nf4_levels(ctypes.addressof(lv), ctypes.addressof(th)), "qlora_nf4_levels")
    return list(lv), list(th)


def qlora_quantize_workspace_bytes(d: int, k: int) -> int:
    return lib().qlora_quantize_workspace_bytes(d, k)


def qlora_fwd_workspace_bytes(d: int, k: int, r: int, T: int) -> int:
    return lib().qlora_fwd_workspace_bytes(d, k, r, T)


def qlora_bwd_workspace_bytes(d: int, k: int, r: int, T: int) -> int:
    return lib().qlora_bwd_workspace_bytes(d, k, r, T)


def lora_merge_workspace_bytes(d: int, k: int, r: int) -> int:
    return lib().lora_merge_workspace_bytes(d, k, r)


def qlora_launch_count() -> int:
    return lib().qlora_launch_count()


def qlora_set_nf4_gemm_mode(mode: int) -> None:
    """0 = by shape, 1 = one CTA per tile, 2 = CTA pairs (same bits, other speed)."""
    _check(lib().qlora_set_nf4_gemm_mode(mode), "qlora_set_nf4_gemm_mode")


# ------------------------------------------------------------------- device calls
def qlora_nf4_quantize(W0: torch.Tensor, out: Optional[NF4Weight] = None,
                       ws: Optional[torch.Tensor] = None, stream=None) -> NF4Weight:
    d, k = W0.shape
    _need(W0, torch.float32, (d, k), "W0")
    out = NF4Weight(d, k, W0.device) if out is None else out
    nbytes = qlora_quantize_workspace_bytes(d, k)
    ws = workspace(nbytes, W0.device) if ws is None else ws
    st = lib().qlora_nf4_quantize(_ptr(W0), d, k, BLOCK, ctypes.byref(out.cstruct), _ptr(ws),
                                  ws.numel(), _stream(stream))
    _check(st, "qlora_nf4_quantize")
    return out


NOALLOC_MAX_WEIGHTS = 1 << 28


def qlora_nf4_quantize_noalloc(W0: torch.Tensor, out: NF4Weight, stream=None) -> NF4Weight:
    """Quantise using the library's static device scratch (no workspace).

    For callers that cannot allocate device memory: pass preallocated output
    buffers in ``out``; nothing else is allocated.  d*k is limited to 2^28.
    Calls share one scratch array, so calls that overlap on the GPU race.
    """
    d, k = W0.shape
    _need(W0, torch.float32, (d, k), "W0")
    st = lib().qlora_nf4_quantize_noalloc(_ptr(W0), d, k, BLOCK, ctypes.byref(out.cstruct),
                                          _stream(stream))
    _check(st, "qlora_nf4_quantize_noalloc")
    return out


def qlora_nf4_dequantize(q: NF4Weight, W_out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    W_out = torch.empty(q.d, q.k, dtype=torch.bfloat16, device=q.codes.device) if W_out is None else W_out
    _need(W_out, torch.bfloat16, (q.d, q.k), "W_out")
    _check(lib().qlora_nf4_dequantize(ctypes.byref(q.cstruct), _ptr(W_out), _stream(stream)),
           "qlora_nf4_dequantize")
    return W_out


def qlora_fwd(q: NF4Weight, A: torch.Tensor, B: torch.Tensor, alpha: float, X: torch.Tensor,
              Y: Optional[torch.Tensor] = None, U_save: Optional[torch.Tensor] = None,
              ws: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    r = A.shape[0]
    T = X.shape[0]
    _need(A, torch.bfloat16, (r, q.k), "A")
    _need(B, torch.bfloat16, (q.d, r), "B")
    _need(X, torch.bfloat16, (T, q.k), "X")
    dev = X.device
    Y = torch.empty(T, q.d, dtype=torch.bfloat16, device=dev) if Y is None else Y
    U_save = torch.empty(T, r, dtype=torch.float32, device=dev) if U_save is None else U_save
    _need(Y, torch.bfloat16, (T, q.d), "Y")
    _need(U_save, torch.float32, (T, r), "U_save")
    nbytes = qlora_fwd_workspace_bytes(q.d, q.k, r, T)
    ws = workspace(nbytes, dev) if ws is None else ws
    st = lib().qlora_fwd(ctypes.byref(q.cstruct), _ptr(A), _ptr(B), r, float(alpha), _ptr(X), T,
                         _ptr(Y), _ptr(U_save), _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "qlora_fwd")
    return Y, U_save


def qlora_bwd(q: NF4Weight, A: torch.Tensor, B: torch.Tensor, alpha: float, X: torch.Tensor,
              U_saved: torch.Tensor, dY: torch.Tensor, dX: Optional[torch.Tensor] = None,
              dA: Optional[torch.Tensor] = None, dB: Optional[torch.Tensor] = None,
              ws: Optional[torch.Tensor] = None, stream=None):
    r = A.shape[0]
    T = X.shape[0]
    _need(A, torch.bfloat16, (r, q.k), "A")
    _need(B, torch.bfloat16, (q.d, r), "B")
    _need(X, torch.bfloat16, (T, q.k), "X")
    _need(U_saved, torch.float32, (T, r), "U_saved")
    _need(dY, torch.bfloat16, (T, q.d), "dY")
    dev = X.device
    dX = torch.empty(T, q.k, dtype=torch.bfloat16, device=dev) if dX is None else dX
    dA = torch.empty(r, q.k, dtype=torch.float32, device=dev) if dA is None else dA
    dB = torch.empty(q.d, r, dtype=torch.float32, device=dev) if dB is None else dB
    _need(dX, torch.bfloat16, (T, q.k), "dX")
    _need(dA, torch.float32, (r, q.k), "dA")
    _need(dB, torch.float32, (q.d, r), "dB")
    nbytes = qlora_bwd_workspace_bytes(q.d, q.k, r, T)
    ws = workspace(nbytes, dev) if ws is None else ws
    st = lib().qlora_bwd(ctypes.byref(q.cstruct), _ptr(A), _ptr(B), r, float(alpha), _ptr(X),
                         _ptr(U_saved), _ptr(dY), T, _ptr(dX), _ptr(dA), _ptr(dB), _ptr(ws),
                         ws.numel(), _stream(stream))
    _check(st, "qlora_bwd")
    return dX, dA, dB


def qlora_fwd_dropout_workspace_bytes(d: int, k: int, r: int, T: int) -> int:
    return lib().qlora_fwd_dropout_workspace_bytes(d, k, r, T)


def qlora_bwd_dropout_workspace_bytes(d: int, k: int, r: int, T: int) -> int:
    return lib().qlora_bwd_dropout_workspace_bytes(d, k, r, T)


def _need_keep(keep: Optional[torch.Tensor], T: int, k: int, p: float):
    if p == 0.0 and keep is None:
        return None
    _need(keep, torch.uint8, (T * k // 8,), "keep")
    return _ptr(keep)


def qlora_fwd_dropout(q: NF4Weight, A: torch.Tensor, B: torch.Tensor, alpha: float, X: torch.Tensor,
                      keep: Optional[torch.Tensor], p: float, Y: Optional[torch.Tensor] = None,
                      U_save: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                      stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Forward with LoRA dropout on the adapter input (keep: bit-packed T*k/8 bytes)."""
    r = A.shape[0]
    T = X.shape[0]
    _need(A, torch.bfloat16, (r, q.k), "A")
    _need(B, torch.bfloat16, (q.d, r), "B")
    _need(X, torch.bfloat16, (T, q.k), "X")
    kp = _need_keep(keep, T, q.k, p)
    dev = X.device
    Y = torch.empty(T, q.d, dtype=torch.bfloat16, device=dev) if Y is None else Y
    U_save = torch.empty(T, r, dtype=torch.float32, device=dev) if U_save is None else U_save
    _need(Y, torch.bfloat16, (T, q.d), "Y")
    _need(U_save, torch.float32, (T, r), "U_save")
    ws = workspace(qlora_fwd_dropout_workspace_bytes(q.d, q.k, r, T), dev) if ws is None else ws
    st = lib().qlora_fwd_dropout(ctypes.byref(q.cstruct), _ptr(A), _ptr(B), r, float(alpha), _ptr(X), kp,
                                 float(p), T, _ptr(Y), _ptr(U_save), _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "qlora_fwd_dropout")
    return Y, U_save


def qlora_bwd_dropout(q: NF4Weight, A: torch.Tensor, B: torch.Tensor, alpha: float, X: torch.Tensor,
                      keep: Optional[torch.Tensor], p: float, U_saved: torch.Tensor, dY: torch.Tensor,
                      dX: Optional[torch.Tensor] = None, dA: Optional[torch.Tensor] = None,
                      dB: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None, stream=None):
    """Backward of qlora_fwd_dropout with the same keep mask."""
    r = A.shape[0]
    T = X.shape[0]
    _need(A, torch.bfloat16, (r, q.k), "A")
    _need(B, torch.bfloat16, (q.d, r), "B")
    _need(X, torch.bfloat16, (T, q.k), "X")
    _need(U_saved, torch.float32, (T, r), "U_saved")
    _need(dY, torch.bfloat16, (T, q.d), "dY")
    kp = _need_keep(keep, T, q.k, p)
    dev = X.device
    dX = torch.empty(T, q.k, dtype=torch.bfloat16, device=dev) if dX is None else dX
    dA = torch.empty(r, q.k, dtype=torch.float32, device=dev) if dA is None else dA
    dB = torch.empty(q.d, r, dtype=torch.float32, device=dev) if dB is None else dB
    _need(dX, torch.bfloat16, (T, q.k), "dX")
    _need(dA, torch.float32, (r, q.k), "dA")
    _need(dB, torch.float32, (q.d, r), "dB")
    ws = workspace(qlora_bwd_dropout_workspace_bytes(q.d, q.k, r, T), dev) if ws is None else ws
    st = lib().qlora_bwd_dropout(ctypes.byref(q.cstruct), _ptr(A), _ptr(B), r, float(alpha), _ptr(X), kp,
                                 float(p), _ptr(U_saved), _ptr(dY), T, _ptr(dX), _ptr(dA), _ptr(dB), _ptr(ws),
                                 ws.numel(), _stream(stream))
    _check(st, "qlora_bwd_dropout")
    return dX, dA, dB


def _host_alphas(alphas):
    arr = (ctypes.c_float * len(alphas))(*[float(a) for a in alphas])
    return arr


def qlora_fwd_multi(q: NF4Weight, As: torch.Tensor, Bs: torch.Tensor, alphas, idx: torch.Tensor,
                    X: torch.Tensor, Y: Optional[torch.Tensor] = None, U_save: Optional[torch.Tensor] = None,
                    ws: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Forward with a stack of n adapters (As n x r x k, Bs n x d x r), token t
    using adapter idx[t] (int32, device) with scale alphas[idx[t]] / r."""
    n, r = As.shape[0], As.shape[1]
    T = X.shape[0]
    _need(As, torch.bfloat16, (n, r, q.k), "As")
    _need(Bs, torch.bfloat16, (n, q.d, r), "Bs")
    _need(idx, torch.int32, (T,), "idx")
    _need(X, torch.bfloat16, (T, q.k), "X")
    if len(alphas) != n:
        raise ValueError("one alpha per adapter")
    dev = X.device
    Y = torch.empty(T, q.d, dtype=torch.bfloat16, device=dev) if Y is None else Y
    U_save = torch.empty(T, r, dtype=torch.float32, device=dev) if U_save is None else U_save
    _need(Y, torch.bfloat16, (T, q.d), "Y")
    _need(U_save, torch.float32, (T, r), "U_save")
    ws = workspace(lib().qlora_fwd_multi_workspace_bytes(q.d, q.k, n, r, T), dev) if ws is None else ws
    al = _host_alphas(alphas)
    st = lib().qlora_fwd_multi(ctypes.byref(q.cstruct), n, _ptr(As), _ptr(Bs), r, ctypes.addressof(al), _ptr(idx),
                               _ptr(X), T, _ptr(Y), _ptr(U_save), _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "qlora_fwd_multi")
    return Y, U_save


def qlora_bwd_multi(q: NF4Weight, As: torch.Tensor, Bs: torch.Tensor, alphas, idx: torch.Tensor,
                    X: torch.Tensor, U_saved: torch.Tensor, dY: torch.Tensor, dX: Optional[torch.Tensor] = None,
                    dAs: Optional[torch.Tensor] = None, dBs: Optional[torch.Tensor] = None,
                    ws: Optional[torch.Tensor] = None, stream=None):
    """Backward of qlora_fwd_multi: dX and per-adapter dAs (n x r x k), dBs (n x d x r)."""
    n, r = As.shape[0], As.shape[1]
    T = X.shape[0]
    _need(As, torch.bfloat16, (n, r, q.k), "As")
    _need(Bs, torch.bfloat16, (n, q.d, r), "Bs")
    _need(idx, torch.int32, (T,), "idx")
    _need(X, torch.bfloat16, (T, q.k), "X")
    _need(U_saved, torch.float32, (T, r), "U_saved")
    _need(dY, torch.bfloat16, (T, q.d), "dY")
    if len(alphas) != n:
        raise ValueError("one alpha per adapter")
    dev = X.device
    dX = torch.empty(T, q.k, dtype=torch.bfloat16, device=dev) if dX is None else dX
    dAs = torch.empty(n, r, q.k, dtype=torch.float32, device=dev) if dAs is None else dAs
    dBs = torch.empty(n, q.d, r, dtype=torch.float32, device=dev) if dBs is None else dBs
    _need(dX, torch.bfloat16, (T, q.k), "dX")
    _need(dAs, torch.float32, (n, r, q.k), "dAs")
    _need(dBs, torch.float32, (n, q.d, r), "dBs")
    ws = workspace(lib().qlora_bwd_multi_workspace_bytes(q.d, q.k, n, r, T), dev) if ws is None else ws
    al = _host_alphas(alphas)
    st = lib().qlora_bwd_multi(ctypes.byref(q.cstruct), n, _ptr(As), _ptr(Bs), r, ctypes.addressof(al), _ptr(idx),
                               _ptr(X), _ptr(U_saved), _ptr(dY), T, _ptr(dX), _ptr(dAs), _ptr(dBs), _ptr(ws),
                               ws.numel(), _stream(stream))
    _check(st, "qlora_bwd_multi")
    return dX, dAs, dBs


def lora_fwd_workspace_bytes(d: int, k: int, r: int, T: int) -> int:
    return lib().lora_fwd_workspace_bytes(d, k, r, T)


def lora_bwd_workspace_bytes(d: int, k: int, r: int, T: int) -> int:
    return lib().lora_bwd_workspace_bytes(d, k, r, T)


def lora_fwd(W: torch.Tensor, A: torch.Tensor, B: torch.Tensor, alpha: float, X: torch.Tensor,
             Y: Optional[torch.Tensor] = None, U_save: Optional[torch.Tensor] = None,
             ws: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Plain LoRA forward on a bf16 base W (d x k); see lora_fwd in qlora.h."""
    d, k = W.shape
    r = A.shape[0]
    T = X.shape[0]
    _need(W, torch.bfloat16, (d, k), "W")
    _need(A, torch.bfloat16, (r, k), "A")
    _need(B, torch.bfloat16, (d, r), "B")
    _need(X, torch.bfloat16, (T, k), "X")
    dev = X.device
    Y = torch.empty(T, d, dtype=torch.bfloat16, device=dev) if Y is None else Y
    U_save = torch.empty(T, r, dtype=torch.float32, device=dev) if U_save is None else U_save
    _need(Y, torch.bfloat16, (T, d), "Y")
    _need(U_save, torch.float32, (T, r), "U_save")
    ws = workspace(lora_fwd_workspace_bytes(d, k, r, T), dev) if ws is None else ws
    st = lib().lora_fwd(_ptr(W), d, k, _ptr(A), _ptr(B), r, float(alpha), _ptr(X), T, _ptr(Y),
                        _ptr(U_save), _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "lora_fwd")
    return Y, U_save


def lora_bwd(W: torch.Tensor, A: torch.Tensor, B: torch.Tensor, alpha: float, X: torch.Tensor,
             U_saved: torch.Tensor, dY: torch.Tensor, dX: Optional[torch.Tensor] = None,
             dA: Optional[torch.Tensor] = None, dB: Optional[torch.Tensor] = None,
             ws: Optional[torch.Tensor] = None, stream=None):
    """Plain LoRA backward on a bf16 base W (d x k); see lora_bwd in qlora.h."""
    d, k = W.shape
    r = A.shape[0]
    T = X.shape[0]
    _need(W, torch.bfloat16, (d, k), "W")
    _need(A, torch.bfloat16, (r, k), "A")
    _need(B, torch.bfloat16, (d, r), "B")
    _need(X, torch.bfloat16, (T, k), "X")
    _need(U_saved, torch.float32, (T, r), "U_saved")
    _need(dY, torch.bfloat16, (T, d), "dY")
    dev = X.device
    dX = torch.empty(T, k, dtype=torch.bfloat16, device=dev) if dX is None else dX
    dA = torch.empty(r, k, dtype=torch.float32, device=dev) if dA is None else dA
    dB = torch.empty(d, r, dtype=torch.float32, device=dev) if dB is None else dB
    _need(dX, torch.bfloat16, (T, k), "dX")
    _need(dA, torch.float32, (r, k), "dA")
    _need(dB, torch.float32, (d, r), "dB")
    ws = workspace(lora_bwd_workspace_bytes(d, k, r, T), dev) if ws is None else ws
    st = lib().lora_bwd(_ptr(W), d, k, _ptr(A), _ptr(B), r, float(alpha), _ptr(X), _ptr(U_saved),
                        _ptr(dY), T, _ptr(dX), _ptr(dA), _ptr(dB), _ptr(ws), ws.numel(),
                        _stream(stream))
    _check(st, "lora_bwd")
    return dX, dA, dB


def lora_adam_step(master: torch.Tensor, weight_bf16: torch.Tensor, m: torch.Tensor, v: torch.Tensor,
                   grad: torch.Tensor, step: int, lr: float, beta1: float = 0.9, beta2: float = 0.999,
                   eps: float = 1e-8, weight_decay: float = 0.0, stream=None) -> None:
    """One Adam step in place on (master, m, v) and the bf16 copy; see qlora.h."""
    n = master.numel()
    _need(master, torch.float32, tuple(master.shape), "master")
    for t, dt, name in ((weight_bf16, torch.bfloat16, "weight_bf16"), (m, torch.float32, "m"),
                        (v, torch.float32, "v"), (grad, torch.float32, "grad")):
        _need(t, dt, tuple(master.shape), name)
    _check(lib().lora_adam_step(_ptr(master), _ptr(weight_bf16), _ptr(m), _ptr(v), _ptr(grad), n, int(step),
                                float(lr), float(beta1), float(beta2), float(eps), float(weight_decay),
                                _stream(stream)), "lora_adam_step")


def lora_merge(q: NF4Weight, A: torch.Tensor, B: torch.Tensor, alpha: float,
               W_out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
               stream=None) -> torch.Tensor:
    r = A.shape[0]
    _need(A, torch.bfloat16, (r, q.k), "A")
    _need(B, torch.bfloat16, (q.d, r), "B")
    W_out = torch.empty(q.d, q.k, dtype=torch.bfloat16, device=A.device) if W_out is None else W_out
    _need(W_out, torch.bfloat16, (q.d, q.k), "W_out")
    nbytes = lora_merge_workspace_bytes(q.d, q.k, r)
    ws = workspace(nbytes, A.device) if ws is None else ws
    st = lib().lora_merge(ctypes.byref(q.cstruct), _ptr(A), _ptr(B), r, float(alpha), _ptr(W_out),
                          _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "lora_merge")
    return W_out


def lora_unmerge(W: torch.Tensor, A: torch.Tensor, B: torch.Tensor, alpha: float,
                 W0_out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
    d, k = W.shape
    r = A.shape[0]
    _need(W, torch.bfloat16, (d, k), "W")
    _need(A, torch.bfloat16, (r, k), "A")
    _need(B, torch.bfloat16, (d, r), "B")
    W0_out = torch.empty(d, k, dtype=torch.bfloat16, device=W.device) if W0_out is None else W0_out
    _need(W0_out, torch.bfloat16, (d, k), "W0_out")
    nbytes = lora_merge_workspace_bytes(d, k, r)
    ws = workspace(nbytes, W.device) if ws is None else ws
    st = lib().lora_unmerge(_ptr(W), _ptr(A), _ptr(B), r, float(alpha), d, k, _ptr(W0_out),
                            _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "lora_unmerge")
    return W0_out


def qlora_get_device_status(stream=None) -> int:
    v = ctypes.c_int(0)
    _check(lib().qlora_get_device_status(_stream(stream), ctypes.byref(v)), "qlora_get_device_status")
    return v.value


def qlora_selftest_wait_timeout(limit_us: int, stream=None) -> None:
    _check(lib().qlora_selftest_wait_timeout(int(limit_us), _stream(stream)), "qlora_selftest_wait_timeout")


# ------------------------------------------------------------------ data parallel
NCCL_ID_BYTES = 128


def qlora_comm_unique_id() -> bytes:
    """A new NCCL unique id for the caller to share with every rank."""
    buf = (ctypes.c_uint8 * NCCL_ID_BYTES)()
    _check(lib().qlora_comm_unique_id(ctypes.addressof(buf)), "qlora_comm_unique_id")
    return bytes(buf)


class Communicator:
    """This rank's NCCL communicator for the adapter-gradient sum (owned by
    the caller; release it with close() after its last collective)."""

    def __init__(self, unique_id: bytes, nranks: int, rank: int):
        if len(unique_id) != NCCL_ID_BYTES:
            raise ValueError(f"unique_id must be {NCCL_ID_BYTES} bytes")
        buf = (ctypes.c_uint8 * NCCL_ID_BYTES).from_buffer_copy(unique_id)
        h = ctypes.c_void_p()
        _check(lib().qlora_comm_init(ctypes.addressof(buf), int(nranks), int(rank), ctypes.byref(h)),
               "qlora_comm_init")
        self.handle = h.value
        self.nranks, self.rank = nranks, rank

    def close(self) -> None:
        if self.handle:
            _check(lib().qlora_comm_destroy(self.handle), "qlora_comm_destroy")
            self.handle = None


def communicator_from_process_group(group=None, make=Communicator):
    """This rank's communicator over the ranks of a torch.distributed group:
    rank 0 draws the NCCL id and the group broadcasts it (any backend)."""
    import torch.distributed as dist
    rank, n = dist.get_rank(group), dist.get_world_size(group)
    box = [qlora_comm_unique_id() if rank == 0 else None]
    dist.broadcast_object_list(box, src=dist.get_global_rank(group, 0) if group is not None else 0, group=group)
    return make(box[0], n, rank)


def qlora_grad_allreduce(comm: "Communicator", dA: torch.Tensor, dB: torch.Tensor, stream=None) -> None:
    """dA and dB (fp32, device) become their sums over the ranks, in place."""
    for name, t in (("dA", dA), ("dB", dB)):
        if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous fp32 CUDA tensor")
    _check(lib().qlora_grad_allreduce(comm.handle, _ptr(dA), dA.numel(), _ptr(dB), dB.numel(), _stream(stream)),
           "qlora_grad_allreduce")


def qlora_profile_begin() -> None:
    _check(lib().qlora_profile_begin(), "qlora_profile_begin")


def qlora_profile_end():
    cap = 64
    arr = (KernelStat * cap)()
    n = ctypes.c_int(0)
    _check(lib().qlora_profile_end(arr, cap, ctypes.byref(n)), "qlora_profile_end")
    return [{"name": arr[i].name.decode(), "launches": arr[i].launches, "total_ms": arr[i].total_ms,
             "flops": arr[i].flops, "bytes": arr[i].bytes} for i in range(min(n.value, cap))]
