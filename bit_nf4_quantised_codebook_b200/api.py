"""ctypes binding over libqlora_nf4.so (the C ABI in include/qlora_nf4.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch provides device memory (the caller side of the ABI allocates
outputs and the workspace) and the current CUDA stream.  If the library is
missing the first call raises; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libqlora_nf4.so")

QLORA_OP_QUANTIZE, QLORA_OP_FORWARD, QLORA_OP_BACKWARD, QLORA_OP_MERGE = 0, 1, 2, 3
QLORA_DEVERR_NONFINITE, QLORA_DEVERR_TIMEOUT = 1, 2
QLORA_ERR_CUDA = 4
CODEBOOKS = {"nf4": 0, "int4": 1, "fp4_e2m1": 2, "fp4_e3m0": 3}
DQ_MODES = {"none": 0, "e4m3": 1, "int8": 2}

EXPORTED = [
    "qlora_status_string", "qlora_build_codebook", "qlora_nf4_sizes", "qlora_workspace_size",
    "qlora_quantize", "qlora_dequantize", "qlora_linear_forward", "qlora_linear_backward",
    "qlora_kernel_launch_count", "qlora_set_timing_events", "qlora_quantize_noalloc",
    "qlora_selftest_bounded_wait", "qlora_adamw_step", "qlora_merge_requantize",
    "qlora_format_codebook", "qlora_format_sizes", "qlora_format_workspace_size", "qlora_quantize_format",
    "qlora_dequantize_format", "qlora_quant_error", "qlora_last_cuda_error",
]


class QloraError(RuntimeError):
    pass


class _Weight(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("K", ctypes.c_int64), ("codes", ctypes.c_void_p),
                ("c2q", ctypes.c_void_p), ("c1", ctypes.c_void_p), ("mean", ctypes.c_void_p)]


class _AdamwTensor(ctypes.Structure):
    _fields_ = [("param", ctypes.c_void_p), ("param_bf16", ctypes.c_void_p), ("grad", ctypes.c_void_p),
                ("m", ctypes.c_void_p), ("v", ctypes.c_void_p), ("n", ctypes.c_int64)]


class _Format(ctypes.Structure):
    _fields_ = [("codebook", ctypes.c_int), ("block", ctypes.c_int), ("dq", ctypes.c_int)]


class _QWeight(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("K", ctypes.c_int64), ("fmt", _Format), ("codes", ctypes.c_void_p),
                ("consts", ctypes.c_void_p), ("c1", ctypes.c_void_p), ("mean", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load the shared library (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise QloraError(f"{LIB_PATH} is missing: run `python -m bit_nf4_quantised_codebook_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, i32, f32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.qlora_status_string.restype = ctypes.c_char_p
        L.qlora_status_string.argtypes = [i32]
        L.qlora_build_codebook.argtypes = [vp, vp]
        L.qlora_nf4_sizes.argtypes = [i64, i64, vp, vp, vp]
        L.qlora_workspace_size.argtypes = [i32, i64, i64, i64, i32, vp]
        L.qlora_quantize.argtypes = [vp, ctypes.POINTER(_Weight), vp, sz, vp, vp]
        L.qlora_dequantize.argtypes = [ctypes.POINTER(_Weight), vp, vp]
        L.qlora_linear_forward.argtypes = [ctypes.POINTER(_Weight), vp, i64, vp, vp, i32, f32, vp, vp, vp, sz,
                                           vp, vp]
        L.qlora_linear_backward.argtypes = [ctypes.POINTER(_Weight), vp, vp, i64, vp, vp, i32, f32, vp, vp, vp,
                                            vp, vp, sz, vp, vp]
        L.qlora_kernel_launch_count.restype = ctypes.c_uint64
        L.qlora_kernel_launch_count.argtypes = []
        L.qlora_set_timing_events.argtypes = [vp, vp, vp, vp]
        L.qlora_quantize_noalloc.argtypes = [vp, ctypes.POINTER(_Weight), vp, vp]
        L.qlora_selftest_bounded_wait.argtypes = [ctypes.c_uint, vp, vp, vp]
        L.qlora_adamw_step.argtypes = [ctypes.POINTER(_AdamwTensor), i32, f32, f32, f32, f32, f32, i64, vp]
        L.qlora_format_codebook.argtypes = [i32, vp, vp]
        L.qlora_format_sizes.argtypes = [ctypes.POINTER(_Format), i64, i64, vp, vp, vp]
        L.qlora_format_workspace_size.argtypes = [ctypes.POINTER(_Format), i64, i64, vp]
        L.qlora_quantize_format.argtypes = [vp, ctypes.POINTER(_QWeight), vp, sz, vp, vp]
        L.qlora_dequantize_format.argtypes = [ctypes.POINTER(_QWeight), vp, vp]
        L.qlora_quant_error.argtypes = [vp, vp, i64, vp, vp]
        L.qlora_merge_requantize.argtypes = [ctypes.POINTER(_Weight), vp, vp, i32, f32, ctypes.POINTER(_Weight),
                                             vp, vp, sz, vp, vp]
        L.qlora_last_cuda_error.argtypes = [vp]
        for name in EXPORTED[1:]:
            if name not in ("qlora_kernel_launch_count", "qlora_last_cuda_error"):
                getattr(L, name).restype = i32
        L.qlora_last_cuda_error.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _check(st: int, what: str) -> None:
    if st != 0:
        msg = f"{what}: {lib().qlora_status_string(st).decode()} (status {st})"
        if st == QLORA_ERR_CUDA:
            msg += f": {lib().qlora_last_cuda_error(None).decode()}"
        raise QloraError(msg)


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _need(t: torch.Tensor, dtype: torch.dtype, shape: tuple, name: str) -> None:
    if not t.is_cuda or t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise QloraError(f"{name}: expected contiguous CUDA {dtype} {tuple(shape)}, got {t.dtype} "
                         f"{tuple(t.shape)} on {t.device}")


@dataclass
class NF4Weight:
    """A quantised frozen weight: device buffers of the stored format."""
    N: int
    K: int
    codes: torch.Tensor   # uint8 [N*K/2]
    c2q: torch.Tensor     # uint8 [N*K/64]
    c1: torch.Tensor      # float32 [ceil(N*K/16384)]
    mean: torch.Tensor    # float32 [1] (padded to 4 floats for alignment)

    def c_struct(self) -> _Weight:
        return _Weight(self.N, self.K, self.codes.data_ptr(), self.c2q.data_ptr(), self.c1.data_ptr(),
                       self.mean.data_ptr())

    def nbytes(self) -> int:
        return self.codes.numel() + self.c2q.numel() + 4 * self.c1.numel() + 4


# ---------------------------------------------------------------- the C ABI, one call each
def qlora_build_codebook() -> tuple[list[float], list[float]]:
    lv = (ctypes.c_float * 16)()
    th = (ctypes.c_float * 15)()
    _check(lib().qlora_build_codebook(lv, th), "qlora_build_codebook")
    return list(lv), list(th)


def qlora_nf4_sizes(N: int, K: int) -> tuple[int, int, int]:
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().qlora_nf4_sizes(N, K, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)), "qlora_nf4_sizes")
    return a.value, b.value, c.value


def qlora_workspace_size(op: int, M: int, N: int, K: int, r: int) -> int:
    n = ctypes.c_size_t()
    _check(lib().qlora_workspace_size(op, M, N, K, r, ctypes.byref(n)), "qlora_workspace_size")
    return n.value


def alloc_weight(N: int, K: int, device=None) -> NF4Weight:
    cb, qb, sb = qlora_nf4_sizes(N, K)
    dev = device or torch.device("cuda")
    return NF4Weight(N, K, torch.empty(cb, dtype=torch.uint8, device=dev),
                     torch.empty(qb, dtype=torch.uint8, device=dev),
                     torch.empty(sb // 4, dtype=torch.float32, device=dev),
                     torch.zeros(4, dtype=torch.float32, device=dev))


def new_error_word(device=None) -> torch.Tensor:
    return torch.zeros(4, dtype=torch.int32, device=device or torch.device("cuda"))


def _workspace(op, M, N, K, r, ws, device):
    need = qlora_workspace_size(op, M, N, K, r)
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=device)
    elif ws.numel() < need:
        raise QloraError(f"workspace too small: {ws.numel()} < {need}")
    return ws


def qlora_quantize(W: torch.Tensor, out: NF4Weight | None = None, ws: torch.Tensor | None = None,
                   dev_err: torch.Tensor | None = None) -> NF4Weight:
    N, K = W.shape
    _need(W, torch.bfloat16, (N, K), "W")
    out = out or alloc_weight(N, K, W.device)
    ws = _workspace(QLORA_OP_QUANTIZE, 0, N, K, 0, ws, W.device)
    s = out.c_struct()
    _check(lib().qlora_quantize(W.data_ptr(), ctypes.byref(s), ws.data_ptr(), ws.numel(), _ptr(dev_err),
                                _stream()), "qlora_quantize")
    return out


def qlora_quantize_noalloc(W: torch.Tensor, out: NF4Weight, dev_err: torch.Tensor | None = None) -> NF4Weight:
    """Quantise into the caller's buffers `out` without any workspace: the
    library keeps the scratch in a static device array (N*K <= 2^26).  For
    callers that cannot allocate device memory; see include/qlora_nf4.h."""
    N, K = W.shape
    _need(W, torch.bfloat16, (N, K), "W")
    if (out.N, out.K) != (N, K):
        raise QloraError(f"out is {out.N}x{out.K}, W is {N}x{K}")
    s = out.c_struct()
    _check(lib().qlora_quantize_noalloc(W.data_ptr(), ctypes.byref(s), _ptr(dev_err), _stream()),
           "qlora_quantize_noalloc")
    return out


def qlora_dequantize(w: NF4Weight, out: torch.Tensor | None = None) -> torch.Tensor:
    out = out if out is not None else torch.empty(w.N, w.K, dtype=torch.bfloat16, device=w.codes.device)
    _need(out, torch.bfloat16, (w.N, w.K), "W_out")
    s = w.c_struct()
    _check(lib().qlora_dequantize(ctypes.byref(s), out.data_ptr(), _stream()), "qlora_dequantize")
    return out


@dataclass
class FormatWeight:
    """A weight stored in one of the format variants (code book, block size,
    treatment of the block constants)."""
    N: int
    K: int
    codebook: str
    block: int
    dq: str
    codes: torch.Tensor            # uint8 [N*K/2]
    consts: torch.Tensor           # float32 [N*K/block] (dq "none") or uint8 [N*K/block]
    c1: torch.Tensor | None        # float32 [ceil(N*K/block/256)]
    mean: torch.Tensor | None      # float32 [4] (element 0)

    def c_fmt(self) -> _Format:
        return _Format(CODEBOOKS[self.codebook], self.block, DQ_MODES[self.dq])

    def c_struct(self) -> _QWeight:
        return _QWeight(self.N, self.K, self.c_fmt(), self.codes.data_ptr(), self.consts.data_ptr(), _ptr(self.c1),
                        _ptr(self.mean))

    def nbytes(self) -> int:
        return (self.codes.numel() + self.consts.numel() * self.consts.element_size()
                + (0 if self.c1 is None else 4 * self.c1.numel() + 4))


def qlora_format_codebook(codebook: str) -> tuple[list[float], list[float]]:
    lv = (ctypes.c_float * 16)()
    th = (ctypes.c_float * 15)()
    _check(lib().qlora_format_codebook(CODEBOOKS[codebook], lv, th), "qlora_format_codebook")
    return list(lv), list(th)


def alloc_format_weight(N: int, K: int, codebook: str, block: int, dq: str, device=None) -> FormatWeight:
    f = _Format(CODEBOOKS[codebook], block, DQ_MODES[dq])
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().qlora_format_sizes(ctypes.byref(f), N, K, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)),
           "qlora_format_sizes")
    dev = device or torch.device("cuda")
    consts = (torch.empty(b.value // 4, dtype=torch.float32, device=dev) if dq == "none"
              else torch.empty(b.value, dtype=torch.uint8, device=dev))
    c1 = None if dq == "none" else torch.empty(max(1, c.value // 4), dtype=torch.float32, device=dev)
    mean = None if dq == "none" else torch.zeros(4, dtype=torch.float32, device=dev)
    return FormatWeight(N, K, codebook, block, dq, torch.empty(a.value, dtype=torch.uint8, device=dev), consts, c1,
                        mean)


def qlora_quantize_format(W: torch.Tensor, codebook: str, block: int, dq: str, out: FormatWeight | None = None,
                          ws: torch.Tensor | None = None, dev_err: torch.Tensor | None = None) -> FormatWeight:
    N, K = W.shape
    _need(W, torch.bfloat16, (N, K), "W")
    out = out or alloc_format_weight(N, K, codebook, block, dq, W.device)
    f = out.c_fmt()
    need = ctypes.c_size_t()
    _check(lib().qlora_format_workspace_size(ctypes.byref(f), N, K, ctypes.byref(need)),
           "qlora_format_workspace_size")
    if ws is None:
        ws = torch.empty(max(16, need.value), dtype=torch.uint8, device=W.device)
    s = out.c_struct()
    _check(lib().qlora_quantize_format(W.data_ptr(), ctypes.byref(s), ws.data_ptr(), ws.numel(), _ptr(dev_err),
                                       _stream()), "qlora_quantize_format")
    return out


def qlora_dequantize_format(w: FormatWeight, out: torch.Tensor | None = None) -> torch.Tensor:
    out = out if out is not None else torch.empty((w.N, w.K), dtype=torch.bfloat16, device=w.codes.device)
    _need(out, torch.bfloat16, (w.N, w.K), "W_out")
    s = w.c_struct()
    _check(lib().qlora_dequantize_format(ctypes.byref(s), out.data_ptr(), _stream()), "qlora_dequantize_format")
    return out


def qlora_quant_error(W: torch.Tensor, W_hat: torch.Tensor, stats: torch.Tensor | None = None) -> torch.Tensor:
    """Device float64 [3]: sum (w - w_hat)^2, sum w^2, max |w - w_hat|."""
    _need(W_hat, torch.bfloat16, tuple(W.shape), "W_hat")
    stats = stats if stats is not None else torch.empty(3, dtype=torch.float64, device=W.device)
    _check(lib().qlora_quant_error(W.data_ptr(), W_hat.data_ptr(), W.numel(), stats.data_ptr(), _stream()),
           "qlora_quant_error")
    return stats


def qlora_merge_requantize(w: NF4Weight, A: torch.Tensor, B: torch.Tensor, s: float, out: NF4Weight | None = None,
                           W_merged: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                           dev_err: torch.Tensor | None = None) -> NF4Weight:
    """W_eff = bf16(float32(W_hat + s·(A·B)ᵀ)) requantised into ``out`` (a new
    weight by default; ``out=w`` merges in place).  ``W_merged`` (N x K bf16)
    optionally receives W_eff."""
    r = A.shape[1]
    _need(A, torch.bfloat16, (w.K, r), "A")
    _need(B, torch.bfloat16, (r, w.N), "B")
    if W_merged is not None:
        _need(W_merged, torch.bfloat16, (w.N, w.K), "W_merged")
    out = out or alloc_weight(w.N, w.K, A.device)
    ws = _workspace(QLORA_OP_MERGE, 0, w.N, w.K, r, ws, A.device)
    sw, so = w.c_struct(), out.c_struct()
    _check(lib().qlora_merge_requantize(ctypes.byref(sw), A.data_ptr(), B.data_ptr(), r, s, ctypes.byref(so),
                                        _ptr(W_merged), ws.data_ptr(), ws.numel(), _ptr(dev_err), _stream()),
           "qlora_merge_requantize")
    return out


def qlora_linear_forward(w: NF4Weight, X: torch.Tensor, A: torch.Tensor, B: torch.Tensor, s: float,
                         Y: torch.Tensor | None = None, T_save: torch.Tensor | None = None,
                         save_t: bool = True, ws: torch.Tensor | None = None,
                         dev_err: torch.Tensor | None = None):
    """Returns (Y, T_save) with T_save = bf16(s·X·A) (None if save_t is False)."""
    M, K = X.shape
    r = A.shape[1]
    _need(X, torch.bfloat16, (M, w.K), "X")
    _need(A, torch.bfloat16, (w.K, r), "A")
    _need(B, torch.bfloat16, (r, w.N), "B")
    dev = X.device
    Y = Y if Y is not None else torch.empty(M, w.N, dtype=torch.bfloat16, device=dev)
    _need(Y, torch.bfloat16, (M, w.N), "Y")
    if T_save is None and save_t:
        T_save = torch.empty(M, r, dtype=torch.bfloat16, device=dev)
    ws = _workspace(QLORA_OP_FORWARD, M, w.N, w.K, r, ws, dev)
    st = w.c_struct()
    _check(lib().qlora_linear_forward(ctypes.byref(st), X.data_ptr(), M, A.data_ptr(), B.data_ptr(), r,
                                      float(s), Y.data_ptr(), _ptr(T_save), ws.data_ptr(), ws.numel(),
                                      _ptr(dev_err), _stream()), "qlora_linear_forward")
    return Y, T_save


def qlora_linear_backward(w: NF4Weight, X: torch.Tensor, dY: torch.Tensor, A: torch.Tensor, B: torch.Tensor,
                          s: float, T_saved: torch.Tensor | None = None, dX: torch.Tensor | None = None,
                          dA: torch.Tensor | None = None, dB: torch.Tensor | None = None,
                          want_dx: bool = True, ws: torch.Tensor | None = None,
                          dev_err: torch.Tensor | None = None):
    """Returns (dX bf16 [M,K] or None, dA f32 [K,r], dB f32 [r,N])."""
    M = X.shape[0]
    r = A.shape[1]
    _need(X, torch.bfloat16, (M, w.K), "X")
    _need(dY, torch.bfloat16, (M, w.N), "dY")
    _need(A, torch.bfloat16, (w.K, r), "A")
    _need(B, torch.bfloat16, (r, w.N), "B")
    dev = X.device
    if want_dx and dX is None:
        dX = torch.empty(M, w.K, dtype=torch.bfloat16, device=dev)
    dA = dA if dA is not None else torch.empty(w.K, r, dtype=torch.float32, device=dev)
    dB = dB if dB is not None else torch.empty(r, w.N, dtype=torch.float32, device=dev)
    if T_saved is not None:
        _need(T_saved, torch.bfloat16, (M, r), "T_saved")
    ws = _workspace(QLORA_OP_BACKWARD, M, w.N, w.K, r, ws, dev)
    st = w.c_struct()
    _check(lib().qlora_linear_backward(ctypes.byref(st), X.data_ptr(), dY.data_ptr(), M, A.data_ptr(),
                                       B.data_ptr(), r, float(s), _ptr(T_saved), _ptr(dX), dA.data_ptr(),
                                       dB.data_ptr(), ws.data_ptr(), ws.numel(), _ptr(dev_err), _stream()),
           "qlora_linear_backward")
    return dX, dA, dB


def qlora_kernel_launch_count() -> int:
    return int(lib().qlora_kernel_launch_count())


def qlora_set_timing_events(fwd_begin=None, fwd_end=None, bwd_begin=None, bwd_end=None) -> None:
    """Events (torch.cuda.Event, created with enable_timing) recorded around the fused GEMMs."""
    h = lambda e: None if e is None else e.cuda_event
    _check(lib().qlora_set_timing_events(h(fwd_begin), h(fwd_end), h(bwd_begin), h(bwd_end)),
           "qlora_set_timing_events")


def qlora_selftest_bounded_wait(timeout_us: int, dev_err: torch.Tensor, gave_up: torch.Tensor | None = None) -> None:
    """Run the device self-test of the bounded-wait error path (see the C header)."""
    _check(lib().qlora_selftest_bounded_wait(timeout_us, dev_err.data_ptr(),
                                             None if gave_up is None else gave_up.data_ptr(), _stream()),
           "qlora_selftest_bounded_wait")


class AdamwGroup:
    """Up to 16 adapter tensors prepared once for qlora_adamw_step: the tensors are
    checked and the descriptor array is built here, so that each step() is only
    the C call.  ``tensors`` is a list of (param float32, param_bf16 bfloat16 or
    None, grad float32, m float32, v float32) CUDA tensors; the caller keeps
    them alive and in place (param, m, v are updated in place)."""

    def __init__(self, tensors):
        self.count = len(tensors)
        self.arr = (_AdamwTensor * max(1, self.count))()
        self.keep = list(tensors)
        for k, (p, pb, g, m, v) in enumerate(tensors):
            for t, name in ((p, "param"), (g, "grad"), (m, "m"), (v, "v")):
                _need(t, torch.float32, tuple(p.shape), name)
            if pb is not None:
                _need(pb, torch.bfloat16, tuple(p.shape), "param_bf16")
            self.arr[k] = _AdamwTensor(p.data_ptr(), _ptr(pb), g.data_ptr(), m.data_ptr(), v.data_ptr(), p.numel())

    def step(self, lr: float, beta1: float = 0.9, beta2: float = 0.999, eps: float = 1e-8,
             weight_decay: float = 0.0, step: int = 1) -> None:
        _check(lib().qlora_adamw_step(self.arr, self.count, lr, beta1, beta2, eps, weight_decay, step, _stream()),
               "qlora_adamw_step")


def qlora_adamw_step(tensors, lr: float, beta1: float = 0.9, beta2: float = 0.999, eps: float = 1e-8,
                     weight_decay: float = 0.0, step: int = 1) -> None:
    """One AdamW step over up to 16 tensors in one launch (see AdamwGroup for the
    tensor list); for repeated steps on the same tensors, keep an AdamwGroup."""
    AdamwGroup(tensors).step(lr, beta1, beta2, eps, weight_decay, step)


def bits_to_tensor(bits, device="cuda") -> torch.Tensor:
    """numpy uint16 bfloat16 bit patterns -> CUDA bfloat16 tensor (same bits)."""
    import numpy as np
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).to(device)


def tensor_to_bits(t: torch.Tensor):
    import numpy as np
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
