"""ctypes binding of libfa.so: the C ABI of include/fa.h under the same names,
plus ``forward``/``backward`` helpers that marshal torch CUDA tensors.

Every computation runs in the library's kernels. There is no fallback: if
libfa.so is missing, or a tensor is not a CUDA tensor, the call raises.
torch is used only to allocate device memory and to name the stream. The
helpers check every buffer against the shapes that q and k imply (the C ABI
receives only pointers and those sizes) and launch on q's device.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa.so")
# The same library built with device-side index and bounds checks (FA_CHECK=1;
# see fa_last_device_status in include/fa.h). Selected with use_library().
LIB_CHECK_PATH = os.path.join(_HERE, "libfa_check.so")

FA_FP16, FA_BF16 = 0, 1
FA_OK = 0
FA_ERR_MISALIGNED = -3
FA_ERR_WORKSPACE = -7
STATUS = {
    0: "FA_OK", -1: "FA_ERR_INVALID_ARG", -2: "FA_ERR_UNSUPPORTED", -3: "FA_ERR_MISALIGNED",
    -4: "FA_ERR_CUDA", -5: "FA_ERR_TIMEOUT", -6: "FA_ERR_NOT_IMPLEMENTED", -7: "FA_ERR_WORKSPACE",
    -8: "FA_ERR_SCRATCH_LIMIT", -9: "FA_ERR_BOUNDS",
}
FA_NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024
EXPORTED = ("fa_fwd", "fa_fwd_ex", "fa_fwd_fp8", "fa_fwd_fp8_ex", "fa_bwd", "fa_bwd_ex", "fa_bwd_noalloc",
            "fa_fwd_workspace_size", "fa_fwd_workspace_size_ex", "fa_fwd_split_plan",
            "fa_bwd_workspace_size", "fa_bwd_workspace_size_ex", "fa_selftest_wait_timeout",
            "fa_last_device_status", "fa_strerror", "fa_version")


class FaTensor(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("stride_b", ctypes.c_int64),
                ("stride_s", ctypes.c_int64), ("stride_h", ctypes.c_int64)]


class FwdParams(ctypes.Structure):
    _fields_ = [("q", FaTensor), ("k", FaTensor), ("v", FaTensor), ("o", FaTensor),
                ("lse", ctypes.c_void_p),
                ("B", ctypes.c_int), ("H", ctypes.c_int), ("Sq", ctypes.c_int), ("Sk", ctypes.c_int),
                ("D", ctypes.c_int), ("scale", ctypes.c_float), ("causal", ctypes.c_int),
                ("dtype", ctypes.c_int),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
                ("split_ranks", ctypes.c_int)]


class FwdFp8Params(ctypes.Structure):
    _fields_ = [("q", FaTensor), ("k", FaTensor), ("v", FaTensor), ("o", FaTensor),
                ("lse", ctypes.c_void_p),
                ("B", ctypes.c_int), ("H", ctypes.c_int), ("Sq", ctypes.c_int), ("Sk", ctypes.c_int),
                ("D", ctypes.c_int), ("scale", ctypes.c_float),
                ("q_descale", ctypes.c_float), ("k_descale", ctypes.c_float), ("v_descale", ctypes.c_float),
                ("causal", ctypes.c_int), ("o_dtype", ctypes.c_int)]


class BwdParams(ctypes.Structure):
    _fields_ = [("q", FaTensor), ("k", FaTensor), ("v", FaTensor), ("o", FaTensor), ("dO", FaTensor),
                ("lse", ctypes.c_void_p),
                ("dq", FaTensor), ("dk", FaTensor), ("dv", FaTensor),
                ("B", ctypes.c_int), ("H", ctypes.c_int), ("Sq", ctypes.c_int), ("Sk", ctypes.c_int),
                ("D", ctypes.c_int), ("scale", ctypes.c_float), ("causal", ctypes.c_int),
                ("dtype", ctypes.c_int), ("workspace", ctypes.c_void_p),
                ("workspace_bytes", ctypes.c_size_t), ("deterministic", ctypes.c_int)]


class FaError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)} ({fa_strerror(status)})")


_lib = None


def use_library(path: str) -> None:
    """Route every call of this module through the library at `path` from now
    on (LIB_PATH, or LIB_CHECK_PATH for the check build). The library is
    loaded at the next call."""
    global _lib, LIB_PATH
    LIB_PATH = path
    _lib = None


def lib():
    """Load libfa.so (once). Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m exact_io_aware_96_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp]
        L.fa_fwd.restype = i
        L.fa_fwd_ex.argtypes = [ctypes.POINTER(FwdParams), vp]
        L.fa_fwd_ex.restype = i
        L.fa_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, f, f, f, i, i, vp]
        L.fa_fwd_fp8.restype = i
        L.fa_fwd_fp8_ex.argtypes = [ctypes.POINTER(FwdFp8Params), vp]
        L.fa_fwd_fp8_ex.restype = i
        L.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp, sz, vp]
        L.fa_bwd.restype = i
        L.fa_bwd_ex.argtypes = [ctypes.POINTER(BwdParams), vp]
        L.fa_bwd_ex.restype = i
        L.fa_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp]
        L.fa_bwd_noalloc.restype = i
        L.fa_fwd_workspace_size.argtypes = [i, i, i, i, i, i]
        L.fa_fwd_workspace_size.restype = sz
        L.fa_fwd_workspace_size_ex.argtypes = [i, i, i, i, i, i, i, ctypes.POINTER(ctypes.c_int)]
        L.fa_fwd_workspace_size_ex.restype = sz
        L.fa_fwd_split_plan.argtypes = [i, i, i, i, i, i, i, i, ctypes.POINTER(ctypes.c_int), ctypes.c_void_p, i]
        L.fa_fwd_split_plan.restype = i
        L.fa_bwd_workspace_size.argtypes = [i, i, i, i]
        L.fa_bwd_workspace_size.restype = sz
        L.fa_bwd_workspace_size_ex.argtypes = [i, i, i, i, i, i]
        L.fa_bwd_workspace_size_ex.restype = sz
        L.fa_selftest_wait_timeout.argtypes = [ctypes.c_uint, vp]
        L.fa_selftest_wait_timeout.restype = i
        L.fa_last_device_status.argtypes = [ctypes.POINTER(ctypes.c_int)]
        L.fa_last_device_status.restype = i
        L.fa_strerror.argtypes = [i]
        L.fa_strerror.restype = ctypes.c_char_p
        L.fa_version.argtypes = []
        L.fa_version.restype = i
        _lib = L
    return _lib


# ---------------------------------------------------------------- raw C ABI
def fa_fwd(q, k, v, o, lse, B, H, Sq, Sk, D, scale, causal, dtype, stream=0) -> int:
    return lib().fa_fwd(q, k, v, o, lse, B, H, Sq, Sk, D, scale, causal, dtype, stream)


def fa_fwd_ex(params: FwdParams, stream=0) -> int:
    return lib().fa_fwd_ex(ctypes.byref(params), stream)


def fa_fwd_fp8(q, k, v, o, lse, B, H, Sq, Sk, D, scale, q_descale, k_descale, v_descale, causal, o_dtype,
               stream=0) -> int:
    return lib().fa_fwd_fp8(q, k, v, o, lse, B, H, Sq, Sk, D, scale, q_descale, k_descale, v_descale, causal,
                            o_dtype, stream)


def fa_fwd_fp8_ex(params: FwdFp8Params, stream=0) -> int:
    return lib().fa_fwd_fp8_ex(ctypes.byref(params), stream)


def fa_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, H, Sq, Sk, D, scale, causal, dtype,
           workspace, workspace_bytes, stream=0) -> int:
    return lib().fa_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, H, Sq, Sk, D, scale, causal, dtype,
                        workspace, workspace_bytes, stream)


def fa_bwd_ex(params: BwdParams, stream=0) -> int:
    return lib().fa_bwd_ex(ctypes.byref(params), stream)


def fa_bwd_noalloc(q, k, v, o, lse, dO, dq, dk, dv, B, H, Sq, Sk, D, scale, causal, dtype, stream=0) -> int:
    """Backward with the library's built-in scratch instead of a workspace
    (for callers that cannot allocate device memory; see include/fa.h)."""
    return lib().fa_bwd_noalloc(q, k, v, o, lse, dO, dq, dk, dv, B, H, Sq, Sk, D, scale, causal, dtype, stream)


def fa_bwd_workspace_size(B, H, Sq, D) -> int:
    return lib().fa_bwd_workspace_size(B, H, Sq, D)


def fa_bwd_workspace_size_ex(B, H, Sq, Sk, D, deterministic) -> int:
    return lib().fa_bwd_workspace_size_ex(B, H, Sq, Sk, D, deterministic)


def fa_selftest_wait_timeout(limit_us, stream=0) -> int:
    """Launch the failure-path self-test (see include/fa.h)."""
    return lib().fa_selftest_wait_timeout(limit_us, stream)


def fa_last_device_status():
    """(status, [code, block, role, iteration]) — synchronises the device."""
    d = (ctypes.c_int * 4)()
    st = lib().fa_last_device_status(d)
    return st, list(d)


def fa_strerror(status: int) -> str:
    return lib().fa_strerror(status).decode()


def fa_version() -> int:
    return lib().fa_version()


# ------------------------------------------------------------ torch helpers
_DT = {torch.float16: FA_FP16, torch.bfloat16: FA_BF16}


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype not in _DT:
        raise TypeError(f"fp16/bf16 tensors only, got {t.dtype}")
    return _DT[t.dtype]


def _view(t: torch.Tensor) -> FaTensor:
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device (the library has no CPU path)")
    if t.dim() != 4 or t.stride(3) != 1:
        raise ValueError("expected a [B, S, H, D] view with a contiguous last axis")
    return FaTensor(t.data_ptr(), t.stride(0), t.stride(1), t.stride(2))


def _expect(name: str, t: torch.Tensor, shape, dtype, device) -> None:
    """The C ABI takes raw pointers and the sizes of q and k only, so every
    other buffer must have exactly the shape, dtype and device they imply
    (a smaller one would be read or written past its end)."""
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, q on {device}")


def _expect_lse(lse: torch.Tensor, B: int, H: int, Sq: int, device) -> None:
    _expect("lse", lse, (B, H, Sq), torch.float32, device)
    if not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 [B, H, Sq] tensor")


def _dims(q: torch.Tensor, k: torch.Tensor):
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q and k must be [B, S, H, D] tensors")
    B, Sq, H, D = q.shape
    if (k.shape[0], k.shape[2], k.shape[3]) != (B, H, D):
        raise ValueError(f"k: expected [B={B}, Sk, H={H}, D={D}], got {tuple(k.shape)}")
    return B, Sq, H, D, k.shape[1]


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def fwd_workspace_size(B, H, Sq, Sk, D, causal, split_ranks=0, device=None):
    """(bytes, split ranks) of the forward's key-range split on `device`
    (default: the current one); (0, 0) when no split is chosen."""
    ns = ctypes.c_int(0)
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        n = lib().fa_fwd_workspace_size_ex(B, H, Sq, Sk, D, int(bool(causal)), int(split_ranks), ctypes.byref(ns))
    return int(n), ns.value


def fwd_split_plan(B, H, Sq, Sk, D, causal, split_ranks=0, sms=0):
    """(n_split, [(rank, kind), ...]) of the forward's key-range split for
    `sms` SMs (0: the current device); kind 0 whole rank, 1/2 its key halves."""
    ns = ctypes.c_int(0)
    buf = (ctypes.c_ubyte * 256)()
    n = lib().fa_fwd_split_plan(B, H, Sq, Sk, D, int(bool(causal)), int(split_ranks), int(sms), ctypes.byref(ns),
                                buf, 256)
    if n < 0:
        raise FaError(n, "fa_fwd_split_plan")
    return ns.value, [(buf[i] // 3, buf[i] % 3) for i in range(n)]


def fwd_workspace_for(B, H, Sq, Sk, D, causal, device, split_ranks=0):
    """A workspace for forward(..., workspace=...), or None when no split is chosen."""
    n, _ = fwd_workspace_size(B, H, Sq, Sk, D, causal, split_ranks, device)
    return torch.empty(n, dtype=torch.uint8, device=device) if n else None


def forward(q, k, v, causal=False, scale=None, out=None, lse=None, stream=None, workspace=None, split_ranks=0):
    """O, LSE = attention(q, k, v) on [B, S, H, D] CUDA tensors (strided views allowed).

    split_ranks: 0 lets the library choose a key-range split of the heaviest
    query blocks (it then needs a workspace, taken from torch's allocator
    unless one is given), k > 0 splits the first k query-block ranks, -1
    never splits."""
    B, Sq, H, D, Sk = _dims(q, k)
    dt = _dtype_code(q)
    dev = q.device
    _expect("k", k, (B, Sk, H, D), q.dtype, dev)
    _expect("v", v, (B, Sk, H, D), q.dtype, dev)
    if scale is None:
        scale = D ** -0.5
    if out is None:
        out = torch.empty((B, Sq, H, D), dtype=q.dtype, device=dev)
    if lse is None:
        lse = torch.empty((B, H, Sq), dtype=torch.float32, device=dev)
    _expect("out", out, (B, Sq, H, D), q.dtype, dev)
    _expect_lse(lse, B, H, Sq, dev)
    views = (_view(q), _view(k), _view(v), _view(out))  # refuses non-CUDA tensors first
    if workspace is None and split_ranks >= 0:
        workspace = fwd_workspace_for(B, H, Sq, Sk, D, causal, dev, split_ranks)
    if workspace is not None:
        if workspace.device != dev or workspace.dtype != torch.uint8 or not workspace.is_contiguous():
            raise ValueError("workspace: expected a contiguous uint8 tensor on q's device")
    p = FwdParams(*views, lse.data_ptr(),
                  B, H, Sq, Sk, D, float(scale), int(bool(causal)), dt,
                  workspace.data_ptr() if workspace is not None else None,
                  workspace.numel() if workspace is not None else 0, int(split_ranks))
    with torch.cuda.device(dev):
        st = fa_fwd_ex(p, _stream(stream))
    if st != FA_OK:
        raise FaError(st, "fa_fwd_ex")
    return out, lse


def forward_fp8(q, k, v, q_descale, k_descale, v_descale, causal=False, scale=None,
                out_dtype=torch.bfloat16, out=None, lse=None, stream=None):
    """O, LSE from e4m3 tensors: the values attended over are q * q_descale,
    k * k_descale, v * v_descale. q, k, v are torch.float8_e4m3fn (or uint8
    holding E4M3 bytes) [B, S, H, D] CUDA views; O is ``out_dtype``."""
    B, Sq, H, D, Sk = _dims(q, k)
    if q.dtype not in (torch.float8_e4m3fn, torch.uint8):
        raise TypeError(f"e4m3 tensors (torch.float8_e4m3fn or uint8 bytes) only, got {q.dtype}")
    dev = q.device
    _expect("k", k, (B, Sk, H, D), q.dtype, dev)
    _expect("v", v, (B, Sk, H, D), q.dtype, dev)
    od = _DT.get(out_dtype)
    if od is None:
        raise TypeError(f"out_dtype must be fp16 or bf16, got {out_dtype}")
    if scale is None:
        scale = D ** -0.5
    if out is None:
        out = torch.empty((B, Sq, H, D), dtype=out_dtype, device=dev)
    if lse is None:
        lse = torch.empty((B, H, Sq), dtype=torch.float32, device=dev)
    _expect("out", out, (B, Sq, H, D), out_dtype, dev)
    _expect_lse(lse, B, H, Sq, dev)
    p = FwdFp8Params(_view(q), _view(k), _view(v), _view(out), lse.data_ptr(),
                     B, H, Sq, Sk, D, float(scale), float(q_descale), float(k_descale), float(v_descale),
                     int(bool(causal)), od)
    with torch.cuda.device(dev):
        st = fa_fwd_fp8_ex(p, _stream(stream))
    if st != FA_OK:
        raise FaError(st, "fa_fwd_fp8_ex")
    return out, lse


def backward_noalloc(q, k, v, o, lse, do, causal=False, scale=None, dq=None, dk=None, dv=None, stream=None):
    """dQ, dK, dV through fa_bwd_noalloc: the backward that takes no workspace
    and uses the library's built-in device scratch (64 MiB per device;
    larger problems raise with FA_ERR_SCRATCH_LIMIT). The tensors must be
    dense [B, S, H, D] (the entry point takes no strides). Calls that overlap
    on the GPU share that scratch and race: see include/fa.h."""
    B, Sq, H, D, Sk = _dims(q, k)
    dt = _dtype_code(q)
    dev = q.device
    if not q.is_cuda:
        raise ValueError("tensors must live on a CUDA device (the library has no CPU path)")
    for name, t, S in (("q", q, Sq), ("k", k, Sk), ("v", v, Sk), ("o", o, Sq), ("do", do, Sq)):
        _expect(name, t, (B, S, H, D), q.dtype, dev)
        if not t.is_contiguous():
            raise ValueError(f"{name} must be a dense [B, S, H, D] tensor for fa_bwd_noalloc")
    _expect_lse(lse, B, H, Sq, dev)
    if scale is None:
        scale = D ** -0.5
    dq = torch.empty((B, Sq, H, D), dtype=q.dtype, device=dev) if dq is None else dq
    dk = torch.empty((B, Sk, H, D), dtype=q.dtype, device=dev) if dk is None else dk
    dv = torch.empty((B, Sk, H, D), dtype=q.dtype, device=dev) if dv is None else dv
    for name, t, S in (("dq", dq, Sq), ("dk", dk, Sk), ("dv", dv, Sk)):
        _expect(name, t, (B, S, H, D), q.dtype, dev)
        if not t.is_contiguous():
            raise ValueError(f"{name} must be a dense [B, S, H, D] tensor for fa_bwd_noalloc")
    with torch.cuda.device(dev):
        st = fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                            dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, Sq, Sk, D, float(scale),
                            int(bool(causal)), dt, _stream(stream))
    if st != FA_OK:
        raise FaError(st, "fa_bwd_noalloc")
    return dq, dk, dv


def workspace_for(B, H, Sq, D, device, Sk=None, deterministic=False) -> torch.Tensor:
    if deterministic:
        n = fa_bwd_workspace_size_ex(B, H, Sq, Sq if Sk is None else Sk, D, 1)
    else:
        n = fa_bwd_workspace_size(B, H, Sq, D)
    return torch.empty(n, dtype=torch.uint8, device=device)


def backward(q, k, v, o, lse, do, causal=False, scale=None, dq=None, dk=None, dv=None,
             workspace=None, stream=None, deterministic=False):
    """dQ, dK, dV of L = sum(dO * O) for O = attention(q, k, v).
    ``deterministic=True`` sums dQ in a fixed order (bit-identical runs; more
    workspace and time)."""
    B, Sq, H, D, Sk = _dims(q, k)
    dt = _dtype_code(q)
    dev = q.device
    _expect("k", k, (B, Sk, H, D), q.dtype, dev)
    _expect("v", v, (B, Sk, H, D), q.dtype, dev)
    _expect("o", o, (B, Sq, H, D), q.dtype, dev)
    _expect("do", do, (B, Sq, H, D), q.dtype, dev)
    _expect_lse(lse, B, H, Sq, dev)
    if scale is None:
        scale = D ** -0.5
    dq = torch.empty((B, Sq, H, D), dtype=q.dtype, device=dev) if dq is None else dq
    dk = torch.empty((B, Sk, H, D), dtype=q.dtype, device=dev) if dk is None else dk
    dv = torch.empty((B, Sk, H, D), dtype=q.dtype, device=dev) if dv is None else dv
    _expect("dq", dq, (B, Sq, H, D), q.dtype, dev)
    _expect("dk", dk, (B, Sk, H, D), q.dtype, dev)
    _expect("dv", dv, (B, Sk, H, D), q.dtype, dev)
    if workspace is None:
        workspace = workspace_for(B, H, Sq, D, dev, Sk=Sk, deterministic=deterministic)
    if workspace.device != dev or not workspace.is_contiguous():
        raise ValueError(f"workspace must be a contiguous buffer on {dev}")
    ws_bytes = workspace.numel() * workspace.element_size()
    p = BwdParams(_view(q), _view(k), _view(v), _view(o), _view(do), lse.data_ptr(),
                  _view(dq), _view(dk), _view(dv), B, H, Sq, Sk, D, float(scale),
                  int(bool(causal)), dt, workspace.data_ptr(), ws_bytes, int(bool(deterministic)))
    with torch.cuda.device(dev):
        st = fa_bwd_ex(p, _stream(stream))
    if st != FA_OK:
        raise FaError(st, "fa_bwd_ex")
    return dq, dk, dv
