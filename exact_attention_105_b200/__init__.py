"""Python binding of the sm_100a exact-attention library (libattn_sm100.so).

The binding only marshals arguments. It takes shapes, data pointers and the
current CUDA stream from torch tensors and calls the C ABI declared in
``include/attn.h``. All arithmetic runs in the library's CUDA kernels. There
is no fallback: if the shared library is missing or the device is not an
sm_100 part, every call raises.

Layout: q, o, dO, dq are [B, Hq, Nq, d]. k, v, dk, dv are [B, Hkv, Nk, d].
All are contiguous bfloat16 CUDA tensors. lse is [B, Hq, Nq] float32.
``attn_fwd``/``attn_bwd`` need Nq == Nk; the ``*_masked`` calls take
Nq != Nk (bottom-right causal alignment), a sliding window and softcapping.
The ``*_varlen`` calls take a packed batch: q/o/dO/dq [total_q, Hq, d],
k/v/dk/dv [total_k, Hkv, d], lse [Hq, total_q], with int32 cu_seqlens.
"""
from __future__ import annotations

import ctypes
import math
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libattn_sm100.so")

ATTN_OK, ATTN_ERR_ARG, ATTN_ERR_UNSUPPORTED, ATTN_ERR_CUDA, ATTN_ERR_TIMEOUT = range(5)
_STATUS_NAMES = {0: "ATTN_OK", 1: "ATTN_ERR_ARG", 2: "ATTN_ERR_UNSUPPORTED",
                 3: "ATTN_ERR_CUDA", 4: "ATTN_ERR_TIMEOUT"}

# Every symbol include/attn.h declares, with its ctypes signature.
_P, _I, _F, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "attn_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _P]),
    "attn_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ,
                      _I, _I, _I, _I, _I, _F, _I, _P]),
    "attn_bwd_workspace_size": (_SZ, [_I, _I, _I, _I]),
    "attn_bwd_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P,
                              _I, _I, _I, _I, _I, _F, _I, _P]),
    "attn_fwd_masked": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _I, _I, _F,
                             _P]),
    "attn_bwd_masked": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ,
                             _I, _I, _I, _I, _I, _I, _F, _I, _I, _I, _F, _P]),
    "attn_fwd_varlen": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F,
                             _I, _I, _I, _F, _P]),
    "attn_bwd_varlen": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ,
                             _I, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I, _I, _F, _P]),
    "attn_check_status": (_I, [_P]),
    "attn_selftest_wait_timeout": (_I, [_P]),
    "attn_get_last_error": (ctypes.c_char_p, []),
    "attn_abi_version": (_I, []),
    "attn_profile_enable": (None, [_I]),
    "attn_profile_reset": (None, []),
    "attn_profile_read": (_I, [_I, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(_I),
                               ctypes.POINTER(ctypes.c_double)]),
}

PROFILED_KERNELS = ("fwd_kernel", "bwd_pre_kernel", "bwd_dkdv_kernel", "bwd_dq_kernel")

_lib = None


class AttnError(RuntimeError):
    """A non-OK status from the library, with its message."""

    def __init__(self, status: int, message: str):
        super().__init__(f"{_STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def load_library():
    """Load (once) and return the ctypes handle; raise if it was never built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m exact_attention_105_b200.build` "
                "(there is no CPU fallback)")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _check(status: int):
    if status != ATTN_OK:
        msg = load_library().attn_get_last_error().decode(errors="replace")
        raise AttnError(status, msg)


class _OnDevice:
    """Makes CUDA device `index` current for the duration of a call, and
    exposes its current stream. When the device is already current (the
    usual case) it changes nothing, which keeps the per-call host cost low."""

    __slots__ = ("index", "prev")

    def __init__(self, index):
        self.index = index
        self.prev = None

    def __enter__(self):
        cur = _current_device()
        if cur != self.index:
            import torch
            self.prev = cur
            torch.cuda.set_device(self.index)
        return self

    def __exit__(self, *exc):
        if self.prev is not None:
            import torch
            torch.cuda.set_device(self.prev)
        return False

    def stream(self, stream):
        """The handle to launch on: `stream` if given, else the device's current stream."""
        if stream is not None:
            return stream.cuda_stream
        return _raw_stream()(self.index)


_RAW_STREAM = None
_GET_DEVICE = None


def _current_device():
    """The current CUDA device index. After the first call (which goes through
    torch.cuda.current_device() and so initialises CUDA) it uses torch's C-level
    getter, skipping the Python-side initialisation checks on every call."""
    global _GET_DEVICE
    if _GET_DEVICE is None:
        import torch
        idx = torch.cuda.current_device()
        _GET_DEVICE = getattr(torch._C, "_cuda_getDevice", None) or torch.cuda.current_device
        return idx
    return _GET_DEVICE()


def _raw_stream():
    """A function from a device index to the raw handle of its current stream.
    torch's C-level accessor costs a fraction of building a Stream object."""
    global _RAW_STREAM
    if _RAW_STREAM is None:
        import torch
        fn = getattr(torch._C, "_cuda_getCurrentRawStream", None)
        _RAW_STREAM = fn if fn is not None else \
            (lambda i: torch.cuda.current_stream(i).cuda_stream)
    return _RAW_STREAM


def _device_guard(*tensors):
    """All tensor arguments must live on one CUDA device. The call then runs
    with that device current (the library launches on the current device)."""
    import torch
    idx = None
    for t in tensors:
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"expected torch.Tensor arguments, got {type(t).__name__}")
        i = t.get_device()
        if idx is None:
            idx = i
        elif i != idx:
            devs = sorted({str(x.device) for x in tensors if isinstance(x, torch.Tensor)})
            raise ValueError(f"all tensors must be on one device, got {devs}")
    if idx is None or idx < 0:
        raise ValueError("tensors must be CUDA tensors (the library takes device pointers), "
                         f"got {tensors[0].device if tensors else None}")
    return _OnDevice(idx)


def _stream_handle(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dev_ptr(t, name):
    """The data pointer of a contiguous tensor, as an int (ctypes passes it as
    void*). Callers run this inside _device_guard, which has already checked
    that every tensor is a CUDA tensor on one device."""
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _check_dtype(t, dtype, name):
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


# Per-step fast path of attn_fwd / attn_bwd. After one call has gone through
# the full checks (which also loads the library and caches torch's device and
# stream getters), calls whose tensors are plainly valid (exact torch.Tensor,
# expected shapes and dtypes, contiguous, all on the current device) skip the
# Python-side helpers and are marshalled by the _pycall module when it is
# built (ctypes otherwise). Anything else takes the checked path, which raises
# the specific error. The library repeats every check that matters for safety.
_FAST = None      # (library handle, Tensor type, bf16, fp32, fwd caller, bwd caller)


def _enable_fast():
    global _FAST
    import torch
    lib = _lib
    if lib is None or _GET_DEVICE is None or _RAW_STREAM is None:
        return
    try:
        from . import _pycall
    except ImportError:
        _pycall = None
    if _pycall is not None:
        fa = ctypes.cast(lib.attn_fwd, ctypes.c_void_p).value
        ba = ctypes.cast(lib.attn_bwd, ctypes.c_void_p).value
        cf, cb = _pycall.call_fwd, _pycall.call_bwd
        fwd = lambda *a: cf(fa, *a)  # noqa: E731
        bwd = lambda *a: cb(ba, *a)  # noqa: E731
    else:
        fwd, bwd = lib.attn_fwd, lib.attn_bwd
    _FAST = (lib, torch.Tensor, torch.bfloat16, torch.float32, fwd, bwd)


def attn_fwd(q, k, v, o=None, lse=None, scale=None, causal=False, stream=None):
    """Forward pass; returns (o, lse). Allocates o/lse with torch if not given."""
    fast = _FAST
    if fast is not None and fast[0] is _lib:
        T = fast[1]
        if type(q) is T and type(k) is T and type(v) is T and type(o) is T and type(lse) is T:
            qs, ks = q.shape, k.shape
            if len(qs) == 4 and len(ks) == 4:
                B, Hq, N, d = qs
                bf = fast[2]
                dev = q.get_device()
                if (ks[0] == B and ks[2] == N and ks[3] == d and v.shape == ks and o.shape == qs
                        and lse.shape == (B, Hq, N) and q.dtype is bf and k.dtype is bf
                        and v.dtype is bf and o.dtype is bf and lse.dtype is fast[3] and dev >= 0
                        and dev == _GET_DEVICE() and k.get_device() == dev
                        and v.get_device() == dev and o.get_device() == dev
                        and lse.get_device() == dev and q.is_contiguous() and k.is_contiguous()
                        and v.is_contiguous() and o.is_contiguous() and lse.is_contiguous()):
                    st = fast[4](q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                 lse.data_ptr(), B, Hq, ks[1], N, d,
                                 1.0 / math.sqrt(d) if scale is None else float(scale),
                                 1 if causal else 0,
                                 _RAW_STREAM(dev) if stream is None else stream.cuda_stream)
                    if st != ATTN_OK:
                        _check(st)
                    return o, lse
    return _attn_fwd_checked(q, k, v, o, lse, scale, causal, stream)


def _attn_fwd_checked(q, k, v, o, lse, scale, causal, stream):
    import torch
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    kshape = (B, Hkv, N, d)
    if k.shape != kshape or v.shape != kshape:
        raise ValueError(f"k/v shape {tuple(k.shape)}/{tuple(v.shape)} does not match q {tuple(q.shape)}")
    bf16 = torch.bfloat16
    if q.dtype != bf16 or k.dtype != bf16 or v.dtype != bf16:
        for t, n in ((q, "q"), (k, "k"), (v, "v")):
            _check_dtype(t, bf16, n)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    if o.dtype != bf16 or lse.dtype != torch.float32:
        _check_dtype(o, bf16, "o")
        _check_dtype(lse, torch.float32, "lse")
    if o.shape != q.shape or lse.shape != (B, Hq, N):
        raise ValueError("o/lse shape mismatch")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    lib = _lib if _lib is not None else load_library()
    with _device_guard(q, k, v, o, lse) as g:
        _check(lib.attn_fwd(_dev_ptr(q, "q"), _dev_ptr(k, "k"), _dev_ptr(v, "v"), _dev_ptr(o, "o"),
                            _dev_ptr(lse, "lse"), B, Hq, Hkv, N, d, scale, int(bool(causal)),
                            g.stream(stream)))
    if _FAST is None or _FAST[0] is not _lib:
        _enable_fast()
    return o, lse


def attn_bwd_workspace_size(B, Hq, N, d) -> int:
    return int(load_library().attn_bwd_workspace_size(B, Hq, N, d))


def _check_bwd_inputs(q, k, v, o, lse, dO):
    """Shapes and dtypes of the fixed-length backward's inputs. The library
    builds its tensor maps from q's and k's shapes, so a smaller o, dO or lse
    would be read past its end: it is refused here, before any launch."""
    import torch
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (lse, "lse"), (dO, "dO")):
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{n} must be a torch.Tensor")
    if q.dim() != 4:
        raise ValueError(f"q must be [B, Hq, N, d], got shape {tuple(q.shape)}")
    B, Hq, N, d = q.shape
    Hkv = k.shape[1] if k.dim() == 4 else -1
    if k.shape != (B, Hkv, N, d) or v.shape != k.shape or o.shape != q.shape \
            or dO.shape != q.shape or lse.shape != (B, Hq, N):
        raise ValueError("shape mismatch among q, k, v, o, lse, dO")
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dO, "dO")):
        _check_dtype(t, torch.bfloat16, n)
    _check_dtype(lse, torch.float32, "lse")
    return B, Hq, Hkv, N, d


def _check_grad_outputs(dq, dk, dv, q, k, v):
    """The gradient outputs must match q, k, v in shape and be bf16: the
    kernels store whole tiles into them through tensor maps sized from q/k."""
    import torch
    for t, n, ref in ((dq, "dq", q), (dk, "dk", k), (dv, "dv", v)):
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{n} must be a torch.Tensor")
        _check_dtype(t, torch.bfloat16, n)
        if t.shape != ref.shape:
            raise ValueError(f"{n} shape {tuple(t.shape)} does not match {tuple(ref.shape)}")


def attn_bwd(q, k, v, o, lse, dO, dq=None, dk=None, dv=None, workspace=None, scale=None,
             causal=False, stream=None):
    """Backward pass; returns (dq, dk, dv). Allocates outputs/workspace if not given."""
    fast = _FAST
    if (fast is not None and fast[0] is _lib and type(q) is fast[1] and type(k) is fast[1]
            and type(lse) is fast[1] and type(workspace) is fast[1]):
        T, bf = fast[1], fast[2]
        qs, ks = q.shape, k.shape
        if len(qs) == 4 and len(ks) == 4 and workspace.is_contiguous():
            B, Hq, N, d = qs
            dev = q.get_device()
            ptrs = []
            if (ks[0] == B and ks[2] == N and ks[3] == d and lse.shape == (B, Hq, N)
                    and lse.dtype is fast[3] and dev >= 0 and dev == _GET_DEVICE()):
                for t, shape in ((q, qs), (k, ks), (v, ks), (o, qs), (lse, None), (dO, qs),
                                 (dq, qs), (dk, ks), (dv, ks)):
                    if (type(t) is not T or t.get_device() != dev or not t.is_contiguous()
                            or (shape is not None and (t.shape != shape or t.dtype is not bf))):
                        break
                    ptrs.append(t.data_ptr())
            if len(ptrs) == 9 and workspace.get_device() == dev:
                st = fast[5](*ptrs, workspace.data_ptr(),
                             workspace.numel() * workspace.element_size(), B, Hq, ks[1], N, d,
                             1.0 / math.sqrt(d) if scale is None else float(scale),
                             1 if causal else 0,
                             _RAW_STREAM(dev) if stream is None else stream.cuda_stream)
                if st != ATTN_OK:
                    _check(st)
                return dq, dk, dv
    return _attn_bwd_checked(q, k, v, o, lse, dO, dq, dk, dv, workspace, scale, causal, stream)


def _attn_bwd_checked(q, k, v, o, lse, dO, dq, dk, dv, workspace, scale, causal, stream):
    import torch
    B, Hq, Hkv, N, d = _check_bwd_inputs(q, k, v, o, lse, dO)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check_grad_outputs(dq, dk, dv, q, k, v)
    need = attn_bwd_workspace_size(B, Hq, N, d)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    lib = load_library()
    with _device_guard(q, k, v, o, lse, dO, dq, dk, dv, workspace) as g:
        _check(lib.attn_bwd(_dev_ptr(q, "q"), _dev_ptr(k, "k"), _dev_ptr(v, "v"), _dev_ptr(o, "o"),
                            _dev_ptr(lse, "lse"), _dev_ptr(dO, "dO"), _dev_ptr(dq, "dq"),
                            _dev_ptr(dk, "dk"), _dev_ptr(dv, "dv"), _dev_ptr(workspace, "workspace"),
                            workspace.numel() * workspace.element_size(),
                            B, Hq, Hkv, N, d, scale, int(bool(causal)), g.stream(stream)))
    if _FAST is None or _FAST[0] is not _lib:
        _enable_fast()
    return dq, dk, dv


NOALLOC_SCRATCH_BYTES = (8 << 20) + 64


def attn_bwd_noalloc(q, k, v, o, lse, dO, dq, dk, dv, scale=None, causal=False, stream=None):
    """attn_bwd without a workspace, for callers that must not allocate device
    memory when the backward runs. The scratch is a fixed 8 MiB + 64 byte device array
    inside the library (shapes with B * Hq * ceil128(N) > 1048576 are rejected),
    and the output tensors must be passed in. Calls that
    overlap on the GPU share that array and race. Returns (dq, dk, dv).
    Shapes and dtypes are checked as in attn_bwd before anything is launched."""
    B, Hq, Hkv, N, d = _check_bwd_inputs(q, k, v, o, lse, dO)
    _check_grad_outputs(dq, dk, dv, q, k, v)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    lib = load_library()
    with _device_guard(q, k, v, o, lse, dO, dq, dk, dv) as g:
        _check(lib.attn_bwd_noalloc(_dev_ptr(q, "q"), _dev_ptr(k, "k"), _dev_ptr(v, "v"),
                                    _dev_ptr(o, "o"), _dev_ptr(lse, "lse"), _dev_ptr(dO, "dO"),
                                    _dev_ptr(dq, "dq"), _dev_ptr(dk, "dk"), _dev_ptr(dv, "dv"),
                                    B, Hq, Hkv, N, d, scale, int(bool(causal)),
                                    g.stream(stream)))
    return dq, dk, dv


def _window(window):
    left, right = (int(window[0]), int(window[1]))
    return max(left, -1), max(right, -1)


def _softcap(softcap):
    c = 0.0 if softcap is None else float(softcap)
    if not math.isfinite(c) or c < 0:
        raise ValueError(f"softcap must be finite and >= 0, got {softcap}")
    return c


def attn_fwd_masked(q, k, v, o=None, lse=None, scale=None, causal=False, window=(-1, -1),
                    softcap=0.0, stream=None):
    """Forward with Nq = q.shape[2] queries, Nk = k.shape[2] keys and a sliding
    window (left, right); a negative side is unbounded. Query i sees key j iff
    i + Nk - Nq - left <= j <= i + Nk - Nq + right (and j <= i + Nk - Nq when
    causal). softcap = c > 0 caps each scaled logit z to c * tanh(z / c).
    Rows that see no key get o = 0, lse = -inf. Returns (o, lse)."""
    import torch
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if k.shape != (B, Hkv, Nk, d) or v.shape != k.shape:
        raise ValueError(f"k/v shape {tuple(k.shape)}/{tuple(v.shape)} does not match q {tuple(q.shape)}")
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check_dtype(t, torch.bfloat16, n)
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device) if lse is None else lse
    _check_dtype(o, torch.bfloat16, "o")
    _check_dtype(lse, torch.float32, "lse")
    if o.shape != q.shape or lse.shape != (B, Hq, Nq):
        raise ValueError("o/lse shape mismatch")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    wl, wr = _window(window)
    lib = load_library()
    with _device_guard(q, k, v, o, lse) as g:
        _check(lib.attn_fwd_masked(_dev_ptr(q, "q"), _dev_ptr(k, "k"), _dev_ptr(v, "v"),
                                   _dev_ptr(o, "o"), _dev_ptr(lse, "lse"), B, Hq, Hkv, Nq, Nk, d,
                                   scale, int(bool(causal)), wl, wr, _softcap(softcap),
                                   g.stream(stream)))
    return o, lse


def attn_bwd_masked(q, k, v, o, lse, dO, dq=None, dk=None, dv=None, workspace=None, scale=None,
                    causal=False, window=(-1, -1), softcap=0.0, stream=None):
    """Backward of attn_fwd_masked with the same causal/window/softcap; returns (dq, dk, dv)."""
    import torch
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if k.shape != (B, Hkv, Nk, d) or v.shape != k.shape or o.shape != q.shape \
            or dO.shape != q.shape or lse.shape != (B, Hq, Nq):
        raise ValueError("shape mismatch among q, k, v, o, lse, dO")
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dO, "dO")):
        _check_dtype(t, torch.bfloat16, n)
    _check_dtype(lse, torch.float32, "lse")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for t, n, ref in ((dq, "dq", q), (dk, "dk", k), (dv, "dv", v)):
        _check_dtype(t, torch.bfloat16, n)
        if t.shape != ref.shape:
            raise ValueError(f"{n} shape mismatch")
    need = attn_bwd_workspace_size(B, Hq, Nq, d)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    wl, wr = _window(window)
    lib = load_library()
    with _device_guard(q, k, v, o, lse, dO, dq, dk, dv, workspace) as g:
        _check(lib.attn_bwd_masked(_dev_ptr(q, "q"), _dev_ptr(k, "k"), _dev_ptr(v, "v"),
                                   _dev_ptr(o, "o"), _dev_ptr(lse, "lse"), _dev_ptr(dO, "dO"),
                                   _dev_ptr(dq, "dq"), _dev_ptr(dk, "dk"), _dev_ptr(dv, "dv"),
                                   _dev_ptr(workspace, "workspace"),
                                   workspace.numel() * workspace.element_size(),
                                   B, Hq, Hkv, Nq, Nk, d, scale, int(bool(causal)), wl, wr,
                                   _softcap(softcap), g.stream(stream)))
    return dq, dk, dv


def _check_cu(cu, name, device):
    import torch
    if not isinstance(cu, torch.Tensor) or cu.dtype != torch.int32 or cu.dim() != 1:
        raise TypeError(f"{name} must be a 1-D int32 tensor")
    if not cu.is_cuda or cu.device != device or not cu.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor on {device}")
    return ctypes.c_void_p(cu.data_ptr())


def attn_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, o=None,
                    lse=None, scale=None, causal=False, window=(-1, -1), softcap=0.0, stream=None):
    """Packed batch forward: q [total_q, Hq, d], k/v [total_k, Hkv, d], int32
    cu_seqlens of length B + 1 on the device. Returns (o [total_q, Hq, d],
    lse [Hq, total_q]). Offsets are checked on the GPU: invalid ones make the
    next attn_check_status() raise."""
    import torch
    total_q, Hq, d = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    if k.shape != (total_k, Hkv, d) or v.shape != k.shape:
        raise ValueError("k/v must be [total_k, Hkv, d] with q's d")
    if cu_seqlens_q.shape != cu_seqlens_k.shape:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must have the same length (B + 1)")
    B = cu_seqlens_q.shape[0] - 1
    cq = _check_cu(cu_seqlens_q, "cu_seqlens_q", q.device)
    ck = _check_cu(cu_seqlens_k, "cu_seqlens_k", q.device)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check_dtype(t, torch.bfloat16, n)
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty((Hq, total_q), dtype=torch.float32, device=q.device) if lse is None else lse
    _check_dtype(o, torch.bfloat16, "o")
    _check_dtype(lse, torch.float32, "lse")
    if o.shape != q.shape or lse.shape != (Hq, total_q):
        raise ValueError("o/lse shape mismatch")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    wl, wr = _window(window)
    lib = load_library()
    with _device_guard(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k) as g:
        _check(lib.attn_fwd_varlen(_dev_ptr(q, "q"), _dev_ptr(k, "k"), _dev_ptr(v, "v"),
                                   _dev_ptr(o, "o"), _dev_ptr(lse, "lse"), cq, ck, B, Hq, Hkv,
                                   total_q, total_k, int(max_seqlen_q), int(max_seqlen_k), d, scale,
                                   int(bool(causal)), wl, wr, _softcap(softcap),
                                   g.stream(stream)))
    return o, lse


def attn_bwd_varlen(q, k, v, o, lse, dO, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                    dq=None, dk=None, dv=None, workspace=None, scale=None, causal=False,
                    window=(-1, -1), softcap=0.0, stream=None):
    """Backward of attn_fwd_varlen with the same arguments; returns (dq, dk, dv)."""
    import torch
    total_q, Hq, d = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    if k.shape != (total_k, Hkv, d) or v.shape != k.shape or o.shape != q.shape \
            or dO.shape != q.shape or lse.shape != (Hq, total_q):
        raise ValueError("shape mismatch among q, k, v, o, lse, dO")
    if cu_seqlens_q.shape != cu_seqlens_k.shape:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must have the same length (B + 1)")
    B = cu_seqlens_q.shape[0] - 1
    cq = _check_cu(cu_seqlens_q, "cu_seqlens_q", q.device)
    ck = _check_cu(cu_seqlens_k, "cu_seqlens_k", q.device)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dO, "dO")):
        _check_dtype(t, torch.bfloat16, n)
    _check_dtype(lse, torch.float32, "lse")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for t, n, ref in ((dq, "dq", q), (dk, "dk", k), (dv, "dv", v)):
        _check_dtype(t, torch.bfloat16, n)
        if t.shape != ref.shape:
            raise ValueError(f"{n} shape mismatch")
    need = attn_bwd_workspace_size(B, Hq, int(max_seqlen_q), d)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    wl, wr = _window(window)
    lib = load_library()
    with _device_guard(q, k, v, o, lse, dO, dq, dk, dv, workspace, cu_seqlens_q, cu_seqlens_k) as g:
        _check(lib.attn_bwd_varlen(_dev_ptr(q, "q"), _dev_ptr(k, "k"), _dev_ptr(v, "v"),
                                   _dev_ptr(o, "o"), _dev_ptr(lse, "lse"), _dev_ptr(dO, "dO"),
                                   _dev_ptr(dq, "dq"), _dev_ptr(dk, "dk"), _dev_ptr(dv, "dv"), cq, ck,
                                   _dev_ptr(workspace, "workspace"),
                                   workspace.numel() * workspace.element_size(), B, Hq, Hkv, total_q,
                                   total_k, int(max_seqlen_q), int(max_seqlen_k), d, scale,
                                   int(bool(causal)), wl, wr, _softcap(softcap),
                                   g.stream(stream)))
    return dq, dk, dv


def profile_enable(on: bool = True):
    """Turn per-kernel CUDA-event timing inside the library on or off."""
    load_library().attn_profile_enable(int(bool(on)))


def profile_reset():
    load_library().attn_profile_reset()


def profile_read():
    """{kernel name: (launches, total milliseconds)} since the last reset."""
    lib = load_library()
    out = {}
    for idx in range(len(PROFILED_KERNELS)):
        name = ctypes.c_char_p()
        n = ctypes.c_int()
        ms = ctypes.c_double()
        _check(lib.attn_profile_read(idx, ctypes.byref(name), ctypes.byref(n), ctypes.byref(ms)))
        out[name.value.decode()] = (n.value, ms.value)
    return out


def selftest_wait_timeout(stream=None):
    """Launch the failure-detection self-test. A kernel waits on a barrier
    that is never signalled, gives up after two seconds, and records a timeout.
    The next attn_check_status() raises AttnError(ATTN_ERR_TIMEOUT)."""
    _check(load_library().attn_selftest_wait_timeout(_stream_handle(stream)))


def attn_check_status(stream=None):
    """Synchronise the stream and raise AttnError if a kernel reported a timeout."""
    _check(load_library().attn_check_status(_stream_handle(stream)))
