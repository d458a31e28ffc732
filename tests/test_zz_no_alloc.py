"""attn_bwd_noalloc: the backward pass for callers that cannot allocate.

Some callers cannot call cudaMalloc when the backward runs. Plugins whose
execute step must not allocate, code inside an allocator callback, and
processes with a fixed device-memory budget set at start-up are examples.
They cannot supply attn_bwd's workspace. attn_bwd_noalloc keeps that scratch
in a fixed 8 MiB device array inside the library. These tests check, through
the C ABI, that it returns the same gradients as attn_bwd with a caller
workspace on two calls in a row, and that it rejects shapes whose scratch
would not fit. This file is collected last on purpose. It must also pass in
a fresh process on its own, because the library's first call on a device sets
up the array's address."""
import ctypes

import pytest
import torch

import exact_attention_105_b200 as ea
import workloads
from exact_attention_105_b200 import build as eabuild

GRAD_REL_TOL = 2e-2          # the same bound the backward parity tests use
FAKE = 1 << 20


def test_noalloc_rejects_shapes_beyond_the_static_scratch():
    """8 MiB holds B*Hq*ceil128(N) <= 1048576 rows. One more 128-row block is refused
    with an argument error before any device work (runs without a GPU too)."""
    eabuild.build()
    lib = ea.load_library()
    # B=1, Hq=8193, N=128 -> 8193 * 128 rows > 1048576: too big.
    st = lib.attn_bwd_noalloc(*([FAKE] * 9), 1, 8193, 1, 128, 64, 0.125, 0, None)
    assert st == ea.ATTN_ERR_ARG
    assert "static" in lib.attn_get_last_error().decode()
    assert ea.attn_bwd_workspace_size(1, 8193, 128, 64) > ea.NOALLOC_SCRATCH_BYTES
    assert ea.attn_bwd_workspace_size(1, 8192, 128, 64) == ea.NOALLOC_SCRATCH_BYTES


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls():
    lib = ea.load_library()
    w = workloads.small("noalloc", 2, 4, 2, 300, 128, True, seed=77)
    q, k, v, do = (t.cuda() for t in workloads.make_inputs(w))
    o, lse = ea.attn_fwd(q, k, v, scale=w.scale, causal=True)
    ref = ea.attn_bwd(q, k, v, o, lse, do, scale=w.scale, causal=True)
    ea.attn_check_status()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    for call in range(2):
        dq, dk, dv = torch.full_like(q, float("nan")), torch.full_like(k, float("nan")), \
            torch.full_like(v, float("nan"))
        st = lib.attn_bwd_noalloc(ptr(q), ptr(k), ptr(v), ptr(o), ptr(lse), ptr(do), ptr(dq),
                                  ptr(dk), ptr(dv), w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, 1, stream)
        assert st == ea.ATTN_OK, lib.attn_get_last_error().decode()
        ea.attn_check_status()
        for name, got, want in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
            assert torch.isfinite(got.float()).all(), (call, name)
            err = (got.float() - want.float()).abs().max().item()
            bound = GRAD_REL_TOL * want.float().abs().max().item()
            assert err <= bound, (call, name, err, bound)
