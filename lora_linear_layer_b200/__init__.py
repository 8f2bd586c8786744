"""Python binding of the B200 fused LoRA linear layer library.

Argument marshalling only: each function takes torch CUDA tensors (bf16,
contiguous), passes their device pointers, sizes and the current CUDA stream
to the C ABI of ``include/lora.h`` (``_lib/liblora_b200.so``) and raises
``LoraError`` on a non-OK status.  Every step of the layer runs in the
library's kernels; there is no fallback of any kind.  If the shared library
is missing, the first call raises ``LoraLibraryMissing``.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Sequence, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "liblora_b200.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "lora.h")

STATUS = {
    0: "LORA_OK", 1: "LORA_ERR_NULL", 2: "LORA_ERR_SHAPE", 3: "LORA_ERR_ALIGN",
    4: "LORA_ERR_RANK", 5: "LORA_ERR_WORKSPACE", 6: "LORA_ERR_CUDA",
    7: "LORA_ERR_TIMEOUT", 8: "LORA_ERR_UNSUPPORTED_DEVICE", 9: "LORA_ERR_ALIAS", 10: "LORA_ERR_FLAGS",
}
LORA_BWD_FP32_GRADS = 1
LORA_BWD_T_SAVED = 2
STATUS_CODE = {v: k for k, v in STATUS.items()}


class LoraError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = int(code)
        super().__init__(f"{what}: {STATUS.get(self.code, self.code)} ({lora_status_string(self.code)})")


class LoraLibraryMissing(ImportError):
    pass


class _FwdDesc(ctypes.Structure):
    _fields_ = [("X", ctypes.c_void_p), ("W", ctypes.c_void_p), ("A", ctypes.c_void_p), ("B", ctypes.c_void_p),
                ("Y", ctypes.c_void_p), ("M", ctypes.c_int64), ("d_in", ctypes.c_int64), ("d_out", ctypes.c_int64)]


class _MergeDesc(ctypes.Structure):
    _fields_ = [("W_src", ctypes.c_void_p), ("A", ctypes.c_void_p), ("B", ctypes.c_void_p),
                ("W_dst", ctypes.c_void_p), ("d_out", ctypes.c_int64), ("d_in", ctypes.c_int64)]


class _Plan(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("fwd_kind", "fwd_bn", "fwd_cg", "fwd_stages", "fwd_run_l",
                                              "fwd_num_m", "fwd_num_n", "fwd_splits")] + \
               [("fwd_smem", ctypes.c_uint32)] + \
               [(n, ctypes.c_int32) for n in ("bwd1_splits_dt", "bwd1_splits_t", "bwd1_saved_splits")] + \
               [("bwd1_smem", ctypes.c_uint32), ("bwd2_splits_db", ctypes.c_int32),
                ("bwd2_splits_da", ctypes.c_int32), ("bwd2_smem", ctypes.c_uint32),
                ("dx_bn", ctypes.c_int32), ("dx_cg", ctypes.c_int32), ("dx_stages", ctypes.c_int32),
                ("dx_smem", ctypes.c_uint32), ("workspace_bytes", ctypes.c_uint64),
                ("fwd_seeded", ctypes.c_int32), ("fwd_tx", ctypes.c_int32)]


_lib_handle = None
_lock = threading.Lock()


def lib() -> ctypes.CDLL:
    """Load (once) and return the shared library; raise if it is missing."""
    global _lib_handle
    if _lib_handle is not None:
        return _lib_handle
    with _lock:
        if _lib_handle is not None:
            return _lib_handle
        if not os.path.exists(LIB_PATH):
            raise LoraLibraryMissing(
                f"{LIB_PATH} not found: build it with lora_linear_layer_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        i64, i32, f32, vp, sz = ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t
        L.lora_abi_version.restype = ctypes.c_int
        L.lora_abi_version.argtypes = []
        L.lora_status_string.restype = ctypes.c_char_p
        L.lora_status_string.argtypes = [ctypes.c_int]
        L.lora_fwd.restype = ctypes.c_int
        L.lora_fwd.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i32, f32, vp]
        L.lora_fwd_save.restype = ctypes.c_int
        L.lora_fwd_save.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i32, f32, vp, sz, vp]
        L.lora_fwd_batched.restype = ctypes.c_int
        L.lora_fwd_batched.argtypes = [ctypes.POINTER(_FwdDesc), i32, i32, f32, vp]
        L.lora_bwd_workspace_size.restype = sz
        L.lora_bwd_workspace_size.argtypes = [i64, i64, i64, i32]
        L.lora_bwd.restype = ctypes.c_int
        L.lora_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i32, f32, vp, sz, vp]
        L.lora_bwd_ex.restype = ctypes.c_int
        L.lora_bwd_ex.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i32, f32, vp, sz, ctypes.c_uint32, vp]
        L.lora_bwd_grads.restype = ctypes.c_int
        L.lora_bwd_grads.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i32, f32, vp, sz, ctypes.c_uint32, vp]
        L.lora_bwd_dx.restype = ctypes.c_int
        L.lora_bwd_dx.argtypes = [vp, vp, vp, vp, i64, i64, i64, i32, vp, sz, vp]
        L.lora_bwd_noalloc.restype = ctypes.c_int
        L.lora_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i32, f32, vp]
        L.lora_merge.restype = ctypes.c_int
        L.lora_merge.argtypes = [vp, vp, vp, vp, i64, i64, i32, f32, vp]
        L.lora_merge_batched.restype = ctypes.c_int
        L.lora_merge_batched.argtypes = [ctypes.POINTER(_MergeDesc), i32, i32, f32, vp]
        L.lora_restore.restype = ctypes.c_int
        L.lora_restore.argtypes = [vp, vp, i64, vp]
        L.lora_get_device_status.restype = ctypes.c_int
        L.lora_get_device_status.argtypes = []
        L.lora_check_args.restype = ctypes.c_int
        L.lora_check_args.argtypes = [i32, ctypes.POINTER(vp), i32, i64, i64, i64, i32, sz]
        L.lora_plan.restype = ctypes.c_int
        L.lora_plan.argtypes = [i64, i64, i64, i32, i32, ctypes.POINTER(_Plan)]
        L.lora_selftest_wait_timeout.restype = ctypes.c_int
        L.lora_selftest_wait_timeout.argtypes = [i64]
        # explicit-scale forms: the same argument lists with `scale` in place of alpha
        for name, base in (("lora_fwd_scaled", "lora_fwd"), ("lora_fwd_save_scaled", "lora_fwd_save"),
                           ("lora_fwd_batched_scaled", "lora_fwd_batched"), ("lora_bwd_scaled", "lora_bwd_ex"),
                           ("lora_bwd_grads_scaled", "lora_bwd_grads"), ("lora_merge_scaled", "lora_merge"),
                           ("lora_merge_batched_scaled", "lora_merge_batched")):
            fn = getattr(L, name)
            fn.restype = ctypes.c_int
            fn.argtypes = list(getattr(L, base).argtypes)
        _lib_handle = L
        return L


# ------------------------------------------------------------ helpers ----

def _ptr(t) -> int:
    return int(t.data_ptr())


_torch = None
_raw_stream = None


def _tm():
    global _torch, _raw_stream
    if _torch is None:
        import torch
        # the current stream's handle without building a torch.cuda.Stream
        # object (about 3 us of host time per call); the public API otherwise
        _raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)
        _torch = torch
    return _torch


def _stream(stream) -> int:
    if stream is None:
        torch = _tm()
        if _raw_stream is not None:
            return int(_raw_stream(torch.cuda.current_device()))
        return int(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return stream
    return int(stream.cuda_stream)


def _check_tensor(t, name: str, shape: Optional[Tuple[int, ...]] = None):
    torch = _tm()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bf16, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and t.shape != shape:
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _raise(code: int, what: str):
    if code != 0:
        raise LoraError(code, what)


# --------------------------------------------------------------- ABI ----

def lora_abi_version() -> int:
    return int(lib().lora_abi_version())


def lora_status_string(code: int) -> str:
    return lib().lora_status_string(int(code)).decode()


def _fwd_call(name, X, W, A, B, Y, value, stream):
    M, d_in = X.shape
    d_out, r = B.shape
    for t, n, s in ((X, "X", (M, d_in)), (W, "W", (d_out, d_in)), (A, "A", (r, d_in)),
                    (B, "B", (d_out, r)), (Y, "Y", (M, d_out))):
        _check_tensor(t, n, s)
    code = getattr(lib(), name)(_ptr(X), _ptr(W), _ptr(A), _ptr(B), _ptr(Y), M, d_in, d_out, r,
                                float(value), _stream(stream))
    _raise(code, name)


def lora_fwd(X, W, A, B, Y, alpha: float, stream=None) -> None:
    """Y = X W^T + (alpha/r) (X A^T) B^T (see include/lora.h)."""
    _fwd_call("lora_fwd", X, W, A, B, Y, alpha, stream)


def lora_fwd_scaled(X, W, A, B, Y, scale: float, stream=None) -> None:
    """Y = X W^T + scale (X A^T) B^T with the scale given (e.g. rsLoRA's
    alpha / sqrt(r)); see include/lora.h."""
    _fwd_call("lora_fwd_scaled", X, W, A, B, Y, scale, stream)


def lora_fwd_save(X, W, A, B, Y, alpha: float, workspace, stream=None) -> None:
    """lora_fwd that also writes T = X A^T into the backward's workspace
    (see include/lora.h); pass that workspace to lora_bwd_ex or
    lora_bwd_grads with LORA_BWD_T_SAVED."""
    _fwd_save_call("lora_fwd_save", X, W, A, B, Y, alpha, workspace, stream)


def lora_fwd_save_scaled(X, W, A, B, Y, scale: float, workspace, stream=None) -> None:
    """lora_fwd_save with the scale given instead of alpha."""
    _fwd_save_call("lora_fwd_save_scaled", X, W, A, B, Y, scale, workspace, stream)


def _fwd_save_call(name, X, W, A, B, Y, value, workspace, stream):
    M, d_in = X.shape
    d_out, r = B.shape
    for t, n, s in ((X, "X", (M, d_in)), (W, "W", (d_out, d_in)), (A, "A", (r, d_in)),
                    (B, "B", (d_out, r)), (Y, "Y", (M, d_out))):
        _check_tensor(t, n, s)
    ws_bytes = int(workspace.numel() * workspace.element_size())
    code = getattr(lib(), name)(_ptr(X), _ptr(W), _ptr(A), _ptr(B), _ptr(Y), M, d_in, d_out, r, float(value),
                                _ptr(workspace), ws_bytes, _stream(stream))
    _raise(code, name)


def lora_fwd_batched(items: Sequence[Tuple], alpha: float, stream=None) -> None:
    """One launch for several independent forwards (X, W, A, B, Y) that share
    the rank r and alpha (see include/lora.h)."""
    _fwd_batched_call("lora_fwd_batched", items, alpha, stream)


def lora_fwd_batched_scaled(items: Sequence[Tuple], scale: float, stream=None) -> None:
    """lora_fwd_batched with the scale given instead of alpha."""
    _fwd_batched_call("lora_fwd_batched_scaled", items, scale, stream)


def _fwd_batched_call(name, items, value, stream):
    n = len(items)
    arr = (_FwdDesc * max(n, 1))()
    r = None
    for i, (X, W, A, B, Y) in enumerate(items):
        M, d_in = X.shape
        d_out, r_i = B.shape
        if r is None:
            r = r_i
        elif r_i != r:
            raise ValueError(f"lora_fwd_batched: every problem needs the same rank ({r} vs {r_i})")
        for t, nm, sh in ((X, "X", (M, d_in)), (W, "W", (d_out, d_in)), (A, "A", (r, d_in)),
                          (B, "B", (d_out, r)), (Y, "Y", (M, d_out))):
            _check_tensor(t, nm, sh)
        arr[i] = _FwdDesc(_ptr(X), _ptr(W), _ptr(A), _ptr(B), _ptr(Y), M, d_in, d_out)
    code = getattr(lib(), name)(arr, n, int(r or 8), float(value), _stream(stream))
    _raise(code, name)


def lora_bwd_workspace_size(M: int, d_in: int, d_out: int, r: int) -> int:
    return int(lib().lora_bwd_workspace_size(int(M), int(d_in), int(d_out), int(r)))


def lora_bwd(X, W, A, B, dY, dX, dA, dB, alpha: float, workspace, stream=None) -> None:
    """dX = dY W + dT A, dA = dT^T X, dB = s dY^T T (see include/lora.h).

    ``workspace`` is a CUDA tensor (any dtype) of at least
    ``lora_bwd_workspace_size(M, d_in, d_out, r)`` bytes."""
    M, d_in = X.shape
    d_out, r = B.shape
    for t, n, s in ((X, "X", (M, d_in)), (W, "W", (d_out, d_in)), (A, "A", (r, d_in)),
                    (B, "B", (d_out, r)), (dY, "dY", (M, d_out)), (dX, "dX", (M, d_in)),
                    (dA, "dA", (r, d_in)), (dB, "dB", (d_out, r))):
        _check_tensor(t, n, s)
    ws_bytes = int(workspace.numel() * workspace.element_size())
    code = lib().lora_bwd(_ptr(X), _ptr(W), _ptr(A), _ptr(B), _ptr(dY), _ptr(dX), _ptr(dA), _ptr(dB),
                          M, d_in, d_out, r, float(alpha), _ptr(workspace), ws_bytes, _stream(stream))
    _raise(code, "lora_bwd")


def lora_bwd_ex(X, W, A, B, dY, dX, dA, dB, alpha: float, workspace, flags: int = 0, stream=None) -> None:
    """lora_bwd with flags (see include/lora.h).  With LORA_BWD_FP32_GRADS,
    dA and dB are float32 tensors and receive the fp32 reductions that
    lora_bwd would round to bf16."""
    _bwd_ex_call("lora_bwd_ex", X, W, A, B, dY, dX, dA, dB, alpha, workspace, flags, stream)


def lora_bwd_scaled(X, W, A, B, dY, dX, dA, dB, scale: float, workspace, flags: int = 0, stream=None) -> None:
    """lora_bwd_ex with the scale given instead of alpha."""
    _bwd_ex_call("lora_bwd_scaled", X, W, A, B, dY, dX, dA, dB, scale, workspace, flags, stream)


def _bwd_ex_call(name, X, W, A, B, dY, dX, dA, dB, value, workspace, flags, stream):
    import torch
    M, d_in = X.shape
    d_out, r = B.shape
    for t, n, s in ((X, "X", (M, d_in)), (W, "W", (d_out, d_in)), (A, "A", (r, d_in)),
                    (B, "B", (d_out, r)), (dY, "dY", (M, d_out)), (dX, "dX", (M, d_in))):
        _check_tensor(t, n, s)
    gdt = torch.float32 if int(flags) & LORA_BWD_FP32_GRADS else torch.bfloat16
    for t, n, s in ((dA, "dA", (r, d_in)), (dB, "dB", (d_out, r))):
        if not isinstance(t, torch.Tensor) or t.dtype != gdt:
            raise TypeError(f"{n} must be a {gdt} tensor with these flags")
        if not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != s:
            raise ValueError(f"{n} must be a contiguous CUDA tensor of shape {s}")
    ws_bytes = int(workspace.numel() * workspace.element_size())
    code = getattr(lib(), name)(_ptr(X), _ptr(W), _ptr(A), _ptr(B), _ptr(dY), _ptr(dX), _ptr(dA), _ptr(dB),
                                M, d_in, d_out, r, float(value), _ptr(workspace), ws_bytes, int(flags),
                                _stream(stream))
    _raise(code, name)


def _check_grads(dA, dB, r: int, d_in: int, d_out: int, flags: int):
    torch = _tm()
    gdt = torch.float32 if int(flags) & LORA_BWD_FP32_GRADS else torch.bfloat16
    for t, n, s in ((dA, "dA", (r, d_in)), (dB, "dB", (d_out, r))):
        if not isinstance(t, torch.Tensor) or t.dtype != gdt:
            raise TypeError(f"{n} must be a {gdt} tensor with these flags")
        if not t.is_cuda or not t.is_contiguous() or t.shape != s:
            raise ValueError(f"{n} must be a contiguous CUDA tensor of shape {s}")


def lora_bwd_grads(X, A, B, dY, dA, dB, alpha: float, workspace, flags: int = 0, stream=None) -> None:
    """First half of the backward (see include/lora.h): T (unless
    LORA_BWD_T_SAVED) and dT into the workspace, then dA and dB.  lora_bwd_dx
    with the same workspace gives dX."""
    _bwd_grads_call("lora_bwd_grads", X, A, B, dY, dA, dB, alpha, workspace, flags, stream)


def lora_bwd_grads_scaled(X, A, B, dY, dA, dB, scale: float, workspace, flags: int = 0, stream=None) -> None:
    """lora_bwd_grads with the scale given instead of alpha."""
    _bwd_grads_call("lora_bwd_grads_scaled", X, A, B, dY, dA, dB, scale, workspace, flags, stream)


def _bwd_grads_call(name, X, A, B, dY, dA, dB, value, workspace, flags, stream):
    M, d_in = X.shape
    d_out, r = B.shape
    for t, n, s in ((X, "X", (M, d_in)), (A, "A", (r, d_in)), (B, "B", (d_out, r)), (dY, "dY", (M, d_out))):
        _check_tensor(t, n, s)
    _check_grads(dA, dB, r, d_in, d_out, flags)
    ws_bytes = int(workspace.numel() * workspace.element_size())
    code = getattr(lib(), name)(_ptr(X), _ptr(A), _ptr(B), _ptr(dY), _ptr(dA), _ptr(dB), M, d_in, d_out, r,
                                float(value), _ptr(workspace), ws_bytes, int(flags), _stream(stream))
    _raise(code, name)


def lora_bwd_dx(W, A, dY, dX, workspace, stream=None) -> None:
    """Second half of the backward: dX = dY W + dT A from the dT that the
    preceding lora_bwd_grads call of the same shape left in `workspace`."""
    M, d_out = dY.shape
    r, d_in = A.shape
    for t, n, s in ((W, "W", (d_out, d_in)), (A, "A", (r, d_in)), (dY, "dY", (M, d_out)), (dX, "dX", (M, d_in))):
        _check_tensor(t, n, s)
    ws_bytes = int(workspace.numel() * workspace.element_size())
    code = lib().lora_bwd_dx(_ptr(W), _ptr(A), _ptr(dY), _ptr(dX), M, d_in, d_out, r, _ptr(workspace), ws_bytes,
                             _stream(stream))
    _raise(code, "lora_bwd_dx")


def lora_bwd_noalloc(X, W, A, B, dY, dX, dA, dB, alpha: float, stream=None) -> None:
    """lora_bwd for callers that cannot allocate device memory: the scratch
    is the library's own fixed 32 MiB per-device array (see include/lora.h).
    Calls that may overlap on the GPU share that array; keep them on one
    stream."""
    M, d_in = X.shape
    d_out, r = B.shape
    for t, n, s in ((X, "X", (M, d_in)), (W, "W", (d_out, d_in)), (A, "A", (r, d_in)),
                    (B, "B", (d_out, r)), (dY, "dY", (M, d_out)), (dX, "dX", (M, d_in)),
                    (dA, "dA", (r, d_in)), (dB, "dB", (d_out, r))):
        _check_tensor(t, n, s)
    code = lib().lora_bwd_noalloc(_ptr(X), _ptr(W), _ptr(A), _ptr(B), _ptr(dY), _ptr(dX), _ptr(dA), _ptr(dB),
                                  M, d_in, d_out, r, float(alpha), _stream(stream))
    _raise(code, "lora_bwd_noalloc")


def lora_merge(W_src, A, B, W_dst, alpha: float, stream=None) -> None:
    """W_dst = bf16(W_src + (alpha/r) B A); W_dst may be W_src (in place)."""
    _merge_call("lora_merge", W_src, A, B, W_dst, alpha, stream)


def lora_merge_scaled(W_src, A, B, W_dst, scale: float, stream=None) -> None:
    """W_dst = bf16(W_src + scale B A) with the scale given."""
    _merge_call("lora_merge_scaled", W_src, A, B, W_dst, scale, stream)


def _merge_call(name, W_src, A, B, W_dst, value, stream):
    d_out, d_in = W_src.shape
    r = A.shape[0]
    for t, n, s in ((W_src, "W_src", (d_out, d_in)), (A, "A", (r, d_in)), (B, "B", (d_out, r)),
                    (W_dst, "W_dst", (d_out, d_in))):
        _check_tensor(t, n, s)
    code = getattr(lib(), name)(_ptr(W_src), _ptr(A), _ptr(B), _ptr(W_dst), d_out, d_in, r, float(value),
                                _stream(stream))
    _raise(code, name)


class MergeBatch:
    """A batched merge prepared once for fixed buffers: the tensors are
    checked and the descriptor array is built here, and every call passes the
    same array to ``lora_merge_batched``.  This fits the adapter refresh,
    which re-merges the same (pristine, A, B, W_inf) buffers each cycle after
    updating A and B in place.  The tensors must stay alive and in place."""

    def __init__(self, items: Sequence[Tuple], r: int):
        self.n = len(items)
        self.r = int(r)
        self._arr = (_MergeDesc * max(self.n, 1))()
        self._keep = []
        for i, (W_src, A, B, W_dst) in enumerate(items):
            d_out, d_in = W_src.shape
            for t, nm, s in ((W_src, "W_src", (d_out, d_in)), (A, "A", (self.r, d_in)), (B, "B", (d_out, self.r)),
                             (W_dst, "W_dst", (d_out, d_in))):
                _check_tensor(t, nm, s)
            self._arr[i] = _MergeDesc(_ptr(W_src), _ptr(A), _ptr(B), _ptr(W_dst), d_out, d_in)
            self._keep.append((W_src, A, B, W_dst))

    def __call__(self, alpha: float, stream=None, *, scale: Optional[float] = None) -> None:
        """Merge with s = alpha / r, or with s = ``scale`` when it is given
        (then ``alpha`` is ignored)."""
        if scale is None:
            code = lib().lora_merge_batched(self._arr, self.n, self.r, float(alpha), _stream(stream))
            _raise(code, "lora_merge_batched")
        else:
            code = lib().lora_merge_batched_scaled(self._arr, self.n, self.r, float(scale), _stream(stream))
            _raise(code, "lora_merge_batched_scaled")


def lora_merge_batched(items: Sequence[Tuple], r: int, alpha: float, stream=None) -> None:
    """Merge every (W_src, A, B, W_dst) of ``items`` (shared r, alpha)."""
    MergeBatch(items, r)(alpha, stream)


def lora_merge_batched_scaled(items: Sequence[Tuple], r: int, scale: float, stream=None) -> None:
    """lora_merge_batched with the scale given instead of alpha."""
    MergeBatch(items, r)(0.0, stream, scale=scale)


def lora_restore(W_src, W_dst, stream=None) -> None:
    """W_dst <- W_src (bit copy)."""
    _check_tensor(W_src, "W_src")
    _check_tensor(W_dst, "W_dst", tuple(W_src.shape))
    code = lib().lora_restore(_ptr(W_src), _ptr(W_dst), W_src.numel(), _stream(stream))
    _raise(code, "lora_restore")


def lora_get_device_status() -> int:
    """Synchronize the device; return the status code (0 = OK)."""
    return int(lib().lora_get_device_status())


def lora_check_args(op: int, ptrs: Sequence[int], M: int, d_in: int, d_out: int, r: int,
                    workspace_bytes: int = 0) -> int:
    """Host-only validation (no GPU): returns the status code."""
    n = len(ptrs)
    arr = (ctypes.c_void_p * max(n, 1))(*[ctypes.c_void_p(p) if p else None for p in ptrs])
    return int(lib().lora_check_args(int(op), arr, n, int(M), int(d_in), int(d_out), int(r),
                                     int(workspace_bytes)))


def lora_plan(M: int, d_in: int, d_out: int, r: int, sm_count: int = 148) -> dict:
    """The launch plan the library would use for this shape (host only; see
    include/lora.h), as a dict of lora_plan_t's fields."""
    out = _Plan()
    _raise(lib().lora_plan(int(M), int(d_in), int(d_out), int(r), int(sm_count), ctypes.byref(out)), "lora_plan")
    return {name: int(getattr(out, name)) for name, _ in _Plan._fields_}


def lora_selftest_wait_timeout(limit_ns: int) -> int:
    return int(lib().lora_selftest_wait_timeout(int(limit_ns)))


def header_functions() -> list:
    """Names of the functions include/lora.h declares (for export checks)."""
    import re
    with open(HEADER_PATH) as f:
        txt = f.read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\**\s+\**(lora_[a-z0-9_]+)\s*\(",
                                 txt, flags=re.M)))
