"""attn_bwd_noalloc: the backward pass for callers that cannot allocate.

Some callers cannot call cudaMalloc when the backward runs. Plugins whose
execute step must not allocate, code inside an allocator callback, and
processes with a fixed device-memory budget set at start-up are examples.
They cannot supply attn_bwd's workspace. attn_bwd_noalloc keeps that scratch
in a fixed 8 MiB device array inside the library.

These tests check that it returns exactly attn_bwd's gradients (the same
deterministic kernels run, only the scratch address differs) on two calls in
a row: one through the C ABI with ctypes, one through the Python wrapper.
The gradients are also compared with the float64 oracle at the backward
parity bound. Shapes whose scratch would not fit, and mis-shaped or
wrongly typed outputs, are refused before any launch.

This file is collected last on purpose. It must also pass in a fresh process
on its own, because the library's first call on a device sets up the array's
address."""
import ctypes

import numpy as np
import pytest
import torch

import exact_attention_105_b200 as ea
import oracle
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


def test_noalloc_wrapper_rejects_bad_outputs_before_launch():
    """The Python wrapper checks shapes and dtypes as attn_bwd does, before it
    looks at devices, so these raise on CPU tensors without touching a GPU."""
    w = workloads.small("noalloc_args", 1, 2, 1, 64, 64, True, seed=5)
    q, k, v, do = workloads.make_inputs(w)
    o = torch.zeros_like(q)
    lse = torch.zeros((1, 2, 64), dtype=torch.float32)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    with pytest.raises(ValueError, match="dq shape"):
        ea.attn_bwd_noalloc(q, k, v, o, lse, do, dq[:, :, :32], dk, dv)
    with pytest.raises(TypeError, match="dq must be"):
        ea.attn_bwd_noalloc(q, k, v, o, lse, do, dq.float(), dk, dv)
    with pytest.raises(TypeError, match="lse must be"):
        ea.attn_bwd_noalloc(q, k, v, o, lse.bfloat16(), do, dq, dk, dv)
    with pytest.raises(ValueError, match="shape mismatch"):
        ea.attn_bwd_noalloc(q, k, v, o[:, :, :10], lse, do, dq, dk, dv)
    with pytest.raises(ValueError, match="dv shape"):
        ea.attn_bwd_noalloc(q, k, v, o, lse, do, dq, dk, dv[:, :, 1:])


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls():
    lib = ea.load_library()
    w = workloads.small("noalloc", 2, 4, 2, 300, 128, True, seed=77)
    q_h, k_h, v_h, do_h = workloads.make_inputs(w)
    q, k, v, do = (t.cuda() for t in (q_h, k_h, v_h, do_h))
    o, lse = ea.attn_fwd(q, k, v, scale=w.scale, causal=True)
    want = ea.attn_bwd(q, k, v, o, lse, do, scale=w.scale, causal=True)
    ea.attn_check_status()
    refs = oracle.attention_backward(q_h, k_h, v_h, do_h, w.scale, True)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    for call in range(2):
        dq, dk, dv = torch.full_like(q, float("nan")), torch.full_like(k, float("nan")), \
            torch.full_like(v, float("nan"))
        if call == 0:                          # the C ABI, as a C caller makes it
            st = lib.attn_bwd_noalloc(ptr(q), ptr(k), ptr(v), ptr(o), ptr(lse), ptr(do), ptr(dq),
                                      ptr(dk), ptr(dv), w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, 1,
                                      stream)
            assert st == ea.ATTN_OK, lib.attn_get_last_error().decode()
        else:                                  # the Python wrapper users call
            ea.attn_bwd_noalloc(q, k, v, o, lse, do, dq, dk, dv, scale=w.scale, causal=True)
        ea.attn_check_status()
        for name, got, ref_gpu, ref64 in zip(("dq", "dk", "dv"), (dq, dk, dv), want, refs):
            assert torch.equal(got, ref_gpu), (call, name, "differs from attn_bwd")
            g = got.float().cpu().numpy()
            err = float(np.abs(g - ref64).max())
            bound = GRAD_REL_TOL * float(np.abs(ref64).max())
            assert err <= bound, (call, name, err, bound)
