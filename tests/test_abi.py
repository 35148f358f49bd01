"""The C ABI without a GPU: libfa.so loads, exports what include/fa.h declares,
and rejects bad arguments on the host (no CUDA call is reached)."""
import ctypes
import os
import re

import pytest

from exact_io_aware_96_b200 import fa

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "fa.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(fa_\w+)\s*\(", src, flags=re.M)))


def test_header_lists_expected_entry_points():
    assert set(declared_functions()) == set(fa.EXPORTED)


def test_library_exports_every_declared_symbol(fa_lib):
    for name in declared_functions():
        assert hasattr(fa_lib, name), name


def test_check_build_exports_every_declared_symbol():
    """libfa_check.so (FA_CHECK=1) is the same library: same entry points."""
    from exact_io_aware_96_b200 import build
    if not os.path.exists(fa.LIB_CHECK_PATH):
        build.build(check=True)
    L = ctypes.CDLL(fa.LIB_CHECK_PATH)
    for name in declared_functions():
        assert hasattr(L, name), name
    L.fa_strerror.restype = ctypes.c_char_p
    assert b"bounds check" in L.fa_strerror(-9)


def test_version_and_strerror(fa_lib):
    assert fa.fa_version() >= 100
    for code in fa.STATUS:
        assert fa.fa_strerror(code)
    assert fa.fa_strerror(12345) == "unknown status"


def test_workspace_size(fa_lib):
    # dq accumulator (fp32, rows padded to 128) + Dvec + base-2 LSE (fp32)
    assert fa.fa_bwd_workspace_size(1, 2, 128, 64) == 2 * 128 * 64 * 4 + 2 * 2 * 128 * 4
    assert fa.fa_bwd_workspace_size(2, 12, 2000, 64) == 24 * 2048 * 64 * 4 + 2 * 24 * 2048 * 4
    # head_dim below 64 uses the 64-wide accumulator, above 64 the 128-wide one
    assert fa.fa_bwd_workspace_size(1, 1, 128, 32) == fa.fa_bwd_workspace_size(1, 1, 128, 64)
    assert fa.fa_bwd_workspace_size(1, 1, 128, 96) == 128 * (128 + 2) * 4
    assert fa.fa_bwd_workspace_size(0, 1, 1, 64) == 0
    assert fa.fa_bwd_workspace_size(1, 1, -5, 64) == 0


def test_workspace_size_ex(fa_lib):
    # mode 0 is the plain size; mode 1 adds (rounded to 256 B) one fp32 [128][Dk] slot per block pair
    assert fa.fa_bwd_workspace_size_ex(2, 12, 2000, 2000, 64, 0) == fa.fa_bwd_workspace_size(2, 12, 2000, 64)
    base = fa.fa_bwd_workspace_size(1, 8, 8192, 128)
    assert base % 256 == 0
    assert fa.fa_bwd_workspace_size_ex(1, 8, 8192, 8192, 128, 1) == base + 8 * 64 * 64 * 128 * 128 * 4
    base = fa.fa_bwd_workspace_size(2, 3, 129, 32)   # not a multiple of 256: rounded up
    off = (base + 255) // 256 * 256
    assert fa.fa_bwd_workspace_size_ex(2, 3, 129, 700, 32, 1) == off + 6 * 2 * 6 * 128 * 64 * 4
    assert fa.fa_bwd_workspace_size_ex(1, 1, 128, 0, 64, 1) == 0
    assert fa.fa_bwd_workspace_size_ex(1, 1, 128, 128, 64, 2) == 0


A = 0x10000  # a 16-byte aligned fake address: validation fails before any use


def fwd(**kw):
    args = dict(q=A, k=A, v=A, o=A, lse=A, B=1, H=2, Sq=128, Sk=128, D=64, scale=0.125,
                causal=0, dtype=fa.FA_FP16)
    args.update(kw)
    return fa.fa_fwd(*args.values())


def bwd(**kw):
    args = dict(q=A, k=A, v=A, o=A, lse=A, dO=A, dq=A, dk=A, dv=A, B=1, H=2, Sq=128, Sk=128, D=64,
                scale=0.125, causal=0, dtype=fa.FA_FP16, ws=A, ws_bytes=1 << 30)
    args.update(kw)
    return fa.fa_bwd(*args.values())


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), -1), (dict(o=None), -1), (dict(lse=None), -1),
    (dict(B=0), -1), (dict(H=-1), -1), (dict(Sq=0), -1), (dict(Sk=0), -1),
    (dict(scale=0.0), -1), (dict(scale=-1.0), -1), (dict(scale=float("nan")), -1), (dict(scale=float("inf")), -1),
    (dict(causal=2), -1),
    (dict(D=4), -2), (dict(D=100), -2), (dict(D=136), -2), (dict(D=256), -2), (dict(D=0), -2),
    (dict(dtype=2), -2), (dict(dtype=-1), -2),
    (dict(q=A + 8), -3), (dict(v=A + 2), -3), (dict(o=A + 4), -3), (dict(lse=A + 2), -3),
    (dict(B=1 << 16, H=1 << 16, Sq=1 << 10), -1),
])
def test_fwd_rejects(fa_lib, kw, code):
    assert fwd(**kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(dO=None), -1), (dict(dq=None), -1), (dict(dk=None), -1), (dict(dv=None), -1), (dict(lse=None), -1),
    (dict(D=81), -2), (dict(D=144), -2), (dict(dtype=3), -2), (dict(dk=A + 8), -3), (dict(dO=A + 4), -3),
    (dict(ws=None), -7), (dict(ws_bytes=100), -7), (dict(ws=A + 16), -3),
])
def test_bwd_rejects(fa_lib, kw, code):
    assert bwd(**kw) == code


def fwd_fp8(**kw):
    args = dict(q=A, k=A, v=A, o=A, lse=A, B=1, H=2, Sq=128, Sk=128, D=64, scale=0.125,
                qd=0.01, kd=0.02, vd=0.03, causal=0, o_dtype=fa.FA_BF16)
    args.update(kw)
    return fa.fa_fwd_fp8(*args.values())


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), -1), (dict(v=None), -1), (dict(lse=None), -1), (dict(Sk=0), -1), (dict(causal=-1), -1),
    (dict(scale=0.0), -1), (dict(qd=0.0), -1), (dict(kd=-1.0), -1), (dict(vd=float("nan")), -1),
    (dict(vd=float("inf")), -1), (dict(scale=1e30, qd=1e30), -1),
    (dict(D=8), -2), (dict(D=72), -2), (dict(D=144), -2), (dict(o_dtype=2), -2), (dict(o_dtype=-1), -2),
    (dict(q=A + 8), -3), (dict(o=A + 2), -3), (dict(lse=A + 1), -3),
])
def test_fwd_fp8_rejects(fa_lib, kw, code):
    assert fwd_fp8(**kw) == code


def test_fwd_fp8_strides(fa_lib):
    t = fa.FaTensor(A, 3 * 512 * 12 * 64, 3 * 12 * 64, 64)
    o = fa.FaTensor(A, 512 * 12 * 64, 12 * 64, 64)
    p = fa.FwdFp8Params(t, t, t, o, A, 2, 12, 512, 512, 64, 0.125, 1.0, 1.0, 1.0, 0, fa.FA_BF16)
    p.v = fa.FaTensor(A, 3 * 512 * 12 * 64, 3 * 12 * 64 + 8, 64)  # a multiple of 8 but not of 16 bytes
    assert fa.fa_fwd_fp8_ex(p) == -3
    p.v = t
    p.o = fa.FaTensor(A, 512 * 12 * 64, 12 * 64 + 4, 64)
    assert fa.fa_fwd_fp8_ex(p) == -3
    assert fa_lib.fa_fwd_fp8_ex(None, None) == -1


def test_strided_views_checked(fa_lib):
    t = fa.FaTensor(A, 3 * 512 * 12 * 64, 3 * 12 * 64, 64)
    p = fa.FwdParams(t, t, t, t, A, 2, 12, 512, 512, 64, 0.125, 0, fa.FA_FP16)
    bad = fa.FaTensor(A, 3 * 512 * 12 * 64, 3 * 12 * 64 + 4, 64)  # seq stride not a multiple of 8
    p.k = bad
    assert fa.fa_fwd_ex(p) == -3
    p.k = fa.FaTensor(A, -1, 64, 64)
    assert fa.fa_fwd_ex(p) == -1
    assert fa_lib.fa_fwd_ex(None, None) == -1
    assert fa_lib.fa_bwd_ex(None, None) == -1


def test_fwd_workspace_sizes(fa_lib):
    """Forced key-range splits: tickets (8 B per split (b, h, rank)), then per
    split CTA 256 rows of (m, l) and of fp32 O at the kernel width, each
    section 256-byte aligned. No device is needed for a forced split."""
    import ctypes
    ns = ctypes.c_int(-1)
    n = fa_lib.fa_fwd_workspace_size_ex(2, 3, 1000, 1000, 128, 1, 2, ctypes.byref(ns))
    pairs, ctas = 2 * 3 * 2, 2 * 2 * 3 * 2
    off_o = 256 + (ctas * 256 * 8 + 255) // 256 * 256
    assert ns.value == 2 and n == off_o + ctas * 256 * 128 * 4 and pairs * 8 <= 256
    # split_ranks above the number of 256-row ranks is capped (1000 rows: 4
    # ranks); D = 40 runs the 64-wide kernel
    n = fa_lib.fa_fwd_workspace_size_ex(2, 3, 1000, 1000, 40, 0, 9, ctypes.byref(ns))
    ctas = 2 * 2 * 3 * 4
    assert ns.value == 4 and n == 256 + (ctas * 256 * 8 + 255) // 256 * 256 + ctas * 256 * 64 * 4
    assert fa_lib.fa_fwd_workspace_size_ex(2, 3, 1000, 1000, 64, 0, -1, ctypes.byref(ns)) == 0 and ns.value == 0
    assert fa_lib.fa_fwd_workspace_size_ex(0, 3, 1000, 1000, 64, 0, 2, None) == 0
    # no split past 64 ranks of 256 rows
    assert fa_lib.fa_fwd_workspace_size_ex(1, 1, 64 * 256, 64 * 256, 64, 0, 2, ctypes.byref(ns)) > 0 and ns.value == 2
    assert fa_lib.fa_fwd_workspace_size_ex(1, 1, 64 * 256 + 1, 64 * 256, 64, 0, 2, ctypes.byref(ns)) == 0
    assert ns.value == 0
    assert fa_lib.fa_fwd_workspace_size_ex(1, 1, 10, 10, 72, 0, 2, None) > 0    # D <= 128: the 128-wide kernel
    assert fa_lib.fa_fwd_workspace_size_ex(1, 1, 10, 10, 144, 0, 2, None) == 0  # unsupported head_dim


def test_fwd_workspace_alignment_checked(fa_lib):
    t = fa.FaTensor(A, 512 * 12 * 64, 12 * 64, 64)
    p = fa.FwdParams(t, t, t, t, A, 2, 12, 512, 512, 64, 0.125, 0, fa.FA_FP16, A + 16, 1 << 20, 1)
    assert fa.fa_fwd_ex(p) == -3                 # workspace must be 256-byte aligned


def test_bwd_ex_deterministic_flag_checked(fa_lib):
    t = fa.FaTensor(A, 512 * 12 * 64, 12 * 64, 64)
    ws = fa.fa_bwd_workspace_size_ex(2, 12, 512, 512, 64, 1)
    p = fa.BwdParams(t, t, t, t, t, A, t, t, t, 2, 12, 512, 512, 64, 0.125, 0, fa.FA_FP16, A, ws, 2)
    assert fa.fa_bwd_ex(p) == -1                 # flag must be 0 or 1
    p.deterministic = 1
    p.workspace_bytes = fa.fa_bwd_workspace_size(2, 12, 512, 64)
    assert fa.fa_bwd_ex(p) == -7                 # the plain workspace is too small for mode 1


def test_selftest_limit_checked(fa_lib):
    assert fa.fa_selftest_wait_timeout(0) == -1
    assert fa.fa_selftest_wait_timeout(4000001) == -1


def test_torch_helpers_refuse_cpu_tensors(fa_lib):
    import torch
    q = torch.zeros(1, 8, 1, 64, dtype=torch.float16)
    with pytest.raises(ValueError):
        fa.forward(q, q, q)
    with pytest.raises(TypeError):
        fa.forward(q.float(), q.float(), q.float())


def test_host_pipeline_needs_a_gpu():
    import torch
    from exact_io_aware_96_b200.host_pipeline import HostAttentionPipeline
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    with pytest.raises(RuntimeError):
        HostAttentionPipeline(1, 128, 2, 64)


def test_torch_helpers_check_every_buffer_against_q_and_k():
    """The C ABI sizes everything from q and k; the helpers refuse any other
    buffer whose shape, dtype or device differs (checked before the CUDA
    check, so it runs on CPU tensors)."""
    import torch
    f16 = torch.float16
    B, Sq, Sk, H, D = 1, 8, 12, 2, 64
    q = torch.zeros(B, Sq, H, D, dtype=f16)
    k = torch.zeros(B, Sk, H, D, dtype=f16)
    v = torch.zeros(B, Sk, H, D, dtype=f16)
    cases = [
        (ValueError, "k: expected", dict(q=q, k=torch.zeros(B, Sk, H + 1, D, dtype=f16), v=v)),
        (ValueError, "v: expected shape", dict(q=q, k=k, v=torch.zeros(B, Sk - 1, H, D, dtype=f16))),
        (TypeError, "v: expected", dict(q=q, k=k, v=v.bfloat16())),
        (ValueError, "out: expected shape", dict(q=q, k=k, v=v, out=torch.zeros(B, Sq - 1, H, D, dtype=f16))),
        (TypeError, "out: expected", dict(q=q, k=k, v=v, out=torch.zeros(B, Sq, H, D, dtype=torch.bfloat16))),
        (ValueError, "lse: expected shape", dict(q=q, k=k, v=v, lse=torch.zeros(B, Sq, H))),
        (ValueError, "contiguous", dict(q=q, k=k, v=v, lse=torch.zeros(B, Sq, H).transpose(1, 2))),
    ]
    for exc, msg, kw in cases:
        with pytest.raises(exc, match=msg):
            fa.forward(**kw)
    o = torch.zeros(B, Sq, H, D, dtype=f16)
    lse = torch.zeros(B, H, Sq)
    bwd_cases = [
        (ValueError, "o: expected shape", dict(o=torch.zeros(B, Sk, H, D, dtype=f16))),
        (TypeError, "do: expected", dict(do=o.bfloat16())),
        (ValueError, "lse: expected shape", dict(lse=torch.zeros(B, H, Sk))),
        (ValueError, "dq: expected shape", dict(dq=torch.zeros(B, Sk, H, D, dtype=f16))),
        (ValueError, "dk: expected shape", dict(dk=torch.zeros(B, Sq, H, D, dtype=f16))),
        (TypeError, "dv: expected", dict(dv=torch.zeros(B, Sk, H, D))),
    ]
    for exc, msg, kw in bwd_cases:
        args = dict(q=q, k=k, v=v, o=o, lse=lse, do=o)
        args.update(kw)
        with pytest.raises(exc, match=msg):
            fa.backward(**args)
    # well-formed CPU tensors get as far as the device check
    with pytest.raises(ValueError, match="CUDA device"):
        fa.backward(q, k, v, o, lse, o, workspace=torch.zeros(16, dtype=torch.uint8))
    u8 = torch.uint8
    with pytest.raises(TypeError, match="k: expected"):
        fa.forward_fp8(torch.zeros(B, Sq, H, D, dtype=u8), torch.zeros(B, Sk, H, D, dtype=torch.float8_e4m3fn),
                       torch.zeros(B, Sk, H, D, dtype=u8), 1.0, 1.0, 1.0)
    with pytest.raises(ValueError, match="v: expected shape"):
        fa.forward_fp8(torch.zeros(B, Sq, H, D, dtype=u8), torch.zeros(B, Sk, H, D, dtype=u8),
                       torch.zeros(B, Sq, H, D, dtype=u8), 1.0, 1.0, 1.0)


def test_torch_helpers_marshal_well_formed_calls(monkeypatch):
    """The argument marshalling of forward/backward/forward_fp8 for
    well-formed buffers, with the device parts stubbed: the structs get the
    sizes of q and k and the workspace size in bytes."""
    import contextlib

    import torch
    seen = {}
    monkeypatch.setattr(fa, "_view", lambda t: fa.FaTensor(0, t.stride(0), t.stride(1), t.stride(2)))
    monkeypatch.setattr(fa, "_stream", lambda s: 0)
    monkeypatch.setattr(torch.cuda, "device", lambda d: contextlib.nullcontext())
    for name in ("fa_fwd_ex", "fa_fwd_fp8_ex", "fa_bwd_ex"):
        monkeypatch.setattr(fa, name, lambda p, s, name=name: seen.__setitem__(name, p) or 0)
    B, Sq, Sk, H, D = 2, 8, 12, 3, 64
    q = torch.zeros(B, Sq, H, D, dtype=torch.bfloat16)
    k = torch.zeros(B, Sk, H, D, dtype=torch.bfloat16)
    o, lse = fa.forward(q, k, k.clone(), causal=True)
    p = seen["fa_fwd_ex"]
    assert (p.B, p.H, p.Sq, p.Sk, p.D, p.causal, p.dtype) == (B, H, Sq, Sk, D, 1, fa.FA_BF16)
    assert o.shape == q.shape and lse.shape == (B, H, Sq)
    ws = torch.zeros(100, dtype=torch.float32)
    dq, dk, dv = fa.backward(q, k, k.clone(), o, lse, o.clone(), workspace=ws)
    p = seen["fa_bwd_ex"]
    assert (p.B, p.H, p.Sq, p.Sk, p.D, p.workspace_bytes) == (B, H, Sq, Sk, D, 400)
    assert dq.shape == q.shape and dk.shape == k.shape and dv.shape == k.shape
    q8 = torch.zeros(B, Sq, H, D, dtype=torch.uint8)
    k8 = torch.zeros(B, Sk, H, D, dtype=torch.uint8)
    o8, _ = fa.forward_fp8(q8, k8, k8.clone(), 0.5, 0.25, 2.0, out_dtype=torch.float16)
    p = seen["fa_fwd_fp8_ex"]
    assert (p.Sq, p.Sk, p.o_dtype, p.v_descale) == (Sq, Sk, fa.FA_FP16, 2.0) and o8.dtype == torch.float16


def test_backward_noalloc_helper_checks_and_marshals(monkeypatch):
    """backward_noalloc (the torch helper over fa_bwd_noalloc) refuses CPU
    tensors, buffers whose shape or dtype differ from what q and k imply, and
    strided views (the entry point takes no strides); for well-formed buffers
    it passes the sizes of q and k and the data pointers."""
    import contextlib

    import torch
    f16 = torch.float16
    B, Sq, Sk, H, D = 1, 8, 12, 2, 64
    q = torch.zeros(B, Sq, H, D, dtype=f16)
    k = torch.zeros(B, Sk, H, D, dtype=f16)
    o = torch.zeros(B, Sq, H, D, dtype=f16)
    lse = torch.zeros(B, H, Sq)
    with pytest.raises(ValueError, match="CUDA device"):
        fa.backward_noalloc(q, k, k, o, lse, o)
    # pretend the tensors are on the GPU to reach the shape and layout checks
    monkeypatch.setattr(torch.Tensor, "is_cuda", property(lambda self: True))
    with pytest.raises(ValueError, match="v: expected shape"):
        fa.backward_noalloc(q, k, torch.zeros(B, Sq, H, D, dtype=f16), o, lse, o)
    with pytest.raises(TypeError, match="do: expected"):
        fa.backward_noalloc(q, k, k, o, lse, o.bfloat16())
    with pytest.raises(ValueError, match="lse: expected shape"):
        fa.backward_noalloc(q, k, k, o, torch.zeros(B, H, Sk), o)
    strided = torch.zeros(B, H, Sq, D, dtype=f16).transpose(1, 2)
    with pytest.raises(ValueError, match="o must be a dense"):
        fa.backward_noalloc(q, k, k, strided, lse, o)
    with pytest.raises(ValueError, match="dk: expected shape"):
        fa.backward_noalloc(q, k, k, o, lse, o, dk=torch.zeros(B, Sq, H, D, dtype=f16))
    seen = {}
    monkeypatch.setattr(fa, "_stream", lambda s: 0)
    monkeypatch.setattr(torch.cuda, "device", lambda d: contextlib.nullcontext())
    monkeypatch.setattr(fa, "fa_bwd_noalloc", lambda *a: seen.__setitem__("args", a) or 0)
    dq, dk, dv = fa.backward_noalloc(q, k, k, o, lse, o, causal=True)
    a = seen["args"]
    assert a[0] == q.data_ptr() and a[6] == dq.data_ptr() and a[8] == dv.data_ptr()
    assert a[9:17] == (B, H, Sq, Sk, D, D ** -0.5, 1, fa.FA_FP16)
    assert dq.shape == q.shape and dk.shape == k.shape and dv.shape == k.shape
