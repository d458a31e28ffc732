"""The C-ABI boundary on the CPU: the library loads, exports every symbol the
header declares, and rejects bad arguments with status codes before touching
a GPU. No compute call is made here (there is no GPU on the build machine)."""
import ctypes
import os
import re

import pytest

import exact_attention_105_b200 as ea
from exact_attention_105_b200 import build as eabuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


@pytest.fixture(scope="module")
def lib():
    eabuild.build()
    return ea.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("attn_fwd", "attn_bwd", "attn_bwd_workspace_size", "attn_check_status",
                     "attn_get_last_error"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) <= set(ea.SIGNATURES)
    assert lib.attn_abi_version() == 102


FAKE = 1 << 20          # aligned, non-null, but not device memory


def fwd(lib, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Hq=2, Hkv=1, N=128, d=64,
        scale=0.125, causal=0):
    return lib.attn_fwd(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, causal, None)


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=3, Hkv=2), ea.ATTN_ERR_ARG),          # GQA needs Hq % Hkv == 0
    (dict(Hkv=0), ea.ATTN_ERR_ARG),
    (dict(B=-1), ea.ATTN_ERR_ARG),
    (dict(N=-5), ea.ATTN_ERR_ARG),
    (dict(d=96), ea.ATTN_ERR_UNSUPPORTED),
    (dict(d=256), ea.ATTN_ERR_UNSUPPORTED),
    (dict(scale=0.0), ea.ATTN_ERR_ARG),
    (dict(scale=float("nan")), ea.ATTN_ERR_ARG),
    (dict(scale=float("inf")), ea.ATTN_ERR_ARG),
    (dict(causal=2), ea.ATTN_ERR_ARG),
    (dict(q=None), ea.ATTN_ERR_ARG),
    (dict(lse=None), ea.ATTN_ERR_ARG),
    (dict(k=FAKE + 8), ea.ATTN_ERR_ARG),           # TMA needs 16-byte alignment
])
def test_fwd_argument_errors(lib, kw, code):
    assert fwd(lib, **kw) == code
    assert lib.attn_get_last_error().decode() != ""


def test_empty_problem_is_a_no_op(lib):
    assert fwd(lib, B=0) == ea.ATTN_OK
    assert fwd(lib, N=0) == ea.ATTN_OK
    assert fwd(lib, q=None, k=None, v=None, o=None, lse=None, N=0) == ea.ATTN_OK


def test_no_cpu_fallback_without_a_device(lib):
    """Valid arguments on a machine without an sm_100 device: an error, never a CPU path."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert fwd(lib) == ea.ATTN_ERR_CUDA
    assert "device" in lib.attn_get_last_error().decode().lower() or \
        "cuda" in lib.attn_get_last_error().decode().lower()


def bwd(lib, ws=FAKE, ws_bytes=1 << 30, B=1, Hq=2, Hkv=1, N=128, d=64, scale=0.125, causal=0,
        **ptrs):
    p = {n: FAKE for n in ("q", "k", "v", "o", "lse", "dO", "dq", "dk", "dv")}
    p.update(ptrs)
    return lib.attn_bwd(p["q"], p["k"], p["v"], p["o"], p["lse"], p["dO"], p["dq"], p["dk"],
                        p["dv"], ws, ws_bytes, B, Hq, Hkv, N, d, scale, causal, None)


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=4, Hkv=3), ea.ATTN_ERR_ARG),
    (dict(d=32), ea.ATTN_ERR_UNSUPPORTED),
    (dict(dO=None), ea.ATTN_ERR_ARG),
    (dict(dv=FAKE + 4), ea.ATTN_ERR_ARG),
    (dict(ws=None), ea.ATTN_ERR_ARG),
    (dict(ws_bytes=16), ea.ATTN_ERR_ARG),          # smaller than attn_bwd_workspace_size
    (dict(causal=-1), ea.ATTN_ERR_ARG),
])
def test_bwd_argument_errors(lib, kw, code):
    assert bwd(lib, **kw) == code


def test_marshalling_module_calls_the_library(lib):
    """_pycall converts the ints and floats the binding passes and calls the
    function at the address it is given. With arguments the library rejects
    before touching a device, the library's status and message come back."""
    from exact_attention_105_b200 import _pycall
    fa = ctypes.cast(lib.attn_fwd, ctypes.c_void_p).value
    ba = ctypes.cast(lib.attn_bwd, ctypes.c_void_p).value
    assert _pycall.call_fwd(fa, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 3, 2, 128, 64, 0.125, 0,
                            None) == ea.ATTN_ERR_ARG
    assert "divisible" in lib.attn_get_last_error().decode()
    assert _pycall.call_fwd(fa, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 1, 128, 64, 0.125, 2,
                            None) == ea.ATTN_ERR_ARG
    assert "causal" in lib.attn_get_last_error().decode()
    assert _pycall.call_bwd(ba, *([FAKE] * 10), 1 << 30, 1, 2, 1, 128, 96, 0.125, 0,
                            None) == ea.ATTN_ERR_UNSUPPORTED
    assert _pycall.call_bwd(ba, *([FAKE] * 10), 1 << 30, 1, 2, 1, 128, 64, 0.125, 0,
                            None) in (ea.ATTN_ERR_ARG, ea.ATTN_ERR_CUDA)
    with pytest.raises(TypeError):
        _pycall.call_fwd(fa, FAKE)
    with pytest.raises(OverflowError):
        _pycall.call_fwd(fa, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 40, 2, 1, 128, 64, 0.125, 0, None)
    with pytest.raises(ValueError):
        _pycall.call_fwd(0, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 1, 128, 64, 0.125, 0, None)


def test_workspace_size(lib):
    assert lib.attn_bwd_workspace_size(0, 4, 128, 64) == 0
    small = lib.attn_bwd_workspace_size(1, 1, 128, 64)
    assert small >= 128 * 4                         # at least one fp32 per query row
    assert lib.attn_bwd_workspace_size(8, 16, 2048, 128) >= 8 * 16 * 2048 * 4


def test_binding_rejects_cpu_tensors():
    import torch
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        ea.attn_fwd(q, q, q, o=q.clone(), lse=torch.zeros(1, 1, 128), causal=False)


def fwd_masked(lib, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Hq=2, Hkv=1, Nq=128, Nk=256,
               d=64, scale=0.125, causal=0, wl=-1, wr=-1, softcap=0.0):
    return lib.attn_fwd_masked(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, wl, wr,
                               softcap, None)


def bwd_masked(lib, ws=FAKE, ws_bytes=1 << 30, B=1, Hq=2, Hkv=1, Nq=128, Nk=256, d=64,
               scale=0.125, causal=0, wl=-1, wr=-1, softcap=0.0, **ptrs):
    p = {n: FAKE for n in ("q", "k", "v", "o", "lse", "dO", "dq", "dk", "dv")}
    p.update(ptrs)
    return lib.attn_bwd_masked(p["q"], p["k"], p["v"], p["o"], p["lse"], p["dO"], p["dq"],
                               p["dk"], p["dv"], ws, ws_bytes, B, Hq, Hkv, Nq, Nk, d, scale,
                               causal, wl, wr, softcap, None)


@pytest.mark.parametrize("kw,code", [
    (dict(Nq=-1), ea.ATTN_ERR_ARG),
    (dict(Nk=-1), ea.ATTN_ERR_ARG),
    (dict(Nk=(1 << 24) + 1), ea.ATTN_ERR_ARG),
    (dict(causal=3), ea.ATTN_ERR_ARG),
    (dict(Hq=3, Hkv=2), ea.ATTN_ERR_ARG),
    (dict(d=80), ea.ATTN_ERR_UNSUPPORTED),
    (dict(q=None), ea.ATTN_ERR_ARG),
    (dict(v=FAKE + 2), ea.ATTN_ERR_ARG),
    (dict(o=None, Nk=0), ea.ATTN_ERR_ARG),        # Nk == 0 still writes o and lse
    (dict(softcap=-1.0), ea.ATTN_ERR_ARG),
    (dict(softcap=float("inf")), ea.ATTN_ERR_ARG),
    (dict(softcap=float("nan")), ea.ATTN_ERR_ARG),
])
def test_fwd_masked_argument_errors(lib, kw, code):
    assert fwd_masked(lib, **kw) == code
    assert lib.attn_get_last_error().decode() != ""


def test_masked_empty_problems(lib):
    # No query rows: nothing is written, so no pointer is needed.
    assert fwd_masked(lib, q=None, k=None, v=None, o=None, lse=None, Nq=0) == ea.ATTN_OK
    assert fwd_masked(lib, B=0) == ea.ATTN_OK
    assert bwd_masked(lib, B=0) == ea.ATTN_OK
    assert bwd_masked(lib, Nq=0, Nk=0, q=None, k=None, v=None, o=None, lse=None, dO=None,
                      dq=None, dk=None, dv=None, ws=None) == ea.ATTN_OK


def test_masked_no_keys_needs_no_key_pointers(lib):
    """Nk == 0 with rows to write: k and v are not read, so null is accepted;
    without a device the call then fails as a CUDA error, not an argument one."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert fwd_masked(lib, k=None, v=None, Nk=0) == ea.ATTN_ERR_CUDA
    assert bwd_masked(lib, Nk=0, k=None, v=None, dk=None, dv=None, o=None, lse=None, dO=None,
                      ws=None, ws_bytes=0) == ea.ATTN_ERR_CUDA


@pytest.mark.parametrize("kw,code", [
    (dict(Nq=-3), ea.ATTN_ERR_ARG),
    (dict(dk=None), ea.ATTN_ERR_ARG),
    (dict(ws=None), ea.ATTN_ERR_ARG),
    (dict(ws_bytes=2 * 2 * 128 * 4 - 4), ea.ATTN_ERR_ARG),   # workspace sized by Nq
    (dict(causal=-1), ea.ATTN_ERR_ARG),
])
def test_bwd_masked_argument_errors(lib, kw, code):
    assert bwd_masked(lib, **kw) == code


def test_bwd_masked_workspace_is_sized_by_queries(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    need = lib.attn_bwd_workspace_size(1, 2, 128, 64)
    # Exactly the Nq-sized workspace passes the argument checks (then: no device).
    assert bwd_masked(lib, Nq=128, Nk=4096, ws_bytes=need) == ea.ATTN_ERR_CUDA


CU = 1 << 21            # 4-byte aligned, non-null, but not device memory


def fwd_varlen(lib, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, cu_q=CU, cu_k=CU, B=2, Hq=2, Hkv=1,
               total_q=300, total_k=500, max_q=200, max_k=300, d=128, scale=0.1, causal=1,
               wl=-1, wr=-1, softcap=0.0):
    return lib.attn_fwd_varlen(q, k, v, o, lse, cu_q, cu_k, B, Hq, Hkv, total_q, total_k, max_q,
                               max_k, d, scale, causal, wl, wr, softcap, None)


def bwd_varlen(lib, ws=FAKE, ws_bytes=1 << 30, cu_q=CU, cu_k=CU, B=2, Hq=2, Hkv=1, total_q=300,
               total_k=500, max_q=200, max_k=300, d=128, scale=0.1, causal=1, wl=-1, wr=-1,
               softcap=0.0, **ptrs):
    p = {n: FAKE for n in ("q", "k", "v", "o", "lse", "dO", "dq", "dk", "dv")}
    p.update(ptrs)
    return lib.attn_bwd_varlen(p["q"], p["k"], p["v"], p["o"], p["lse"], p["dO"], p["dq"],
                               p["dk"], p["dv"], cu_q, cu_k, ws, ws_bytes, B, Hq, Hkv, total_q,
                               total_k, max_q, max_k, d, scale, causal, wl, wr, softcap, None)


@pytest.mark.parametrize("kw,code", [
    (dict(total_q=-1), ea.ATTN_ERR_ARG),
    (dict(total_k=-5), ea.ATTN_ERR_ARG),
    (dict(max_q=0), ea.ATTN_ERR_ARG),                # rows but no room for them
    (dict(max_k=-1), ea.ATTN_ERR_ARG),
    (dict(max_q=(1 << 24) + 1), ea.ATTN_ERR_ARG),
    (dict(B=-1), ea.ATTN_ERR_ARG),
    (dict(Hq=3, Hkv=2), ea.ATTN_ERR_ARG),
    (dict(d=96), ea.ATTN_ERR_UNSUPPORTED),
    (dict(softcap=-2.0), ea.ATTN_ERR_ARG),
    (dict(causal=5), ea.ATTN_ERR_ARG),
    (dict(q=None), ea.ATTN_ERR_ARG),
    (dict(lse=FAKE + 4), ea.ATTN_ERR_ARG),
])
def test_fwd_varlen_argument_errors(lib, kw, code):
    assert fwd_varlen(lib, **kw) == code
    assert lib.attn_get_last_error().decode() != ""


@pytest.mark.parametrize("kw,code", [
    (dict(total_q=-1), ea.ATTN_ERR_ARG),
    (dict(ws=None), ea.ATTN_ERR_ARG),
    (dict(ws_bytes=2 * 2 * 256 * 4 - 4), ea.ATTN_ERR_ARG),   # sized by B, Hq and max_seqlen_q
    (dict(dk=None), ea.ATTN_ERR_ARG),
    (dict(softcap=float("nan")), ea.ATTN_ERR_ARG),
])
def test_bwd_varlen_argument_errors(lib, kw, code):
    assert bwd_varlen(lib, **kw) == code


def test_varlen_empty_batches(lib):
    assert fwd_varlen(lib, B=0, q=None, k=None, v=None, o=None, lse=None, cu_q=None,
                      cu_k=None) == ea.ATTN_OK
    assert fwd_varlen(lib, total_q=0, q=None, o=None, lse=None) == ea.ATTN_OK
    assert bwd_varlen(lib, total_q=0, total_k=0) == ea.ATTN_OK


def test_varlen_offsets_checks(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    # Valid arguments: without a device the call fails as a CUDA error. Null or
    # misaligned offsets are argument errors found on the host.
    assert fwd_varlen(lib) == ea.ATTN_ERR_CUDA
    assert fwd_varlen(lib, cu_q=None) == ea.ATTN_ERR_ARG
    assert fwd_varlen(lib, cu_k=CU + 2) == ea.ATTN_ERR_ARG
    assert bwd_varlen(lib, cu_k=None) == ea.ATTN_ERR_ARG
