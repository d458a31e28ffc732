"""Failure detection without a GPU fault.

Every pipeline wait in the kernels is bounded. When a wait runs out, the
kernel records a timeout in a device status word and returns; it never
traps. On the GPU, the self-test kernel waits on a barrier nothing signals.
The host must see ATTN_ERR_TIMEOUT, and the context must stay usable. On
the host side, a failing call reports an error code and a message, and a
missing device is an error, never a CPU fallback (see test_boundary.py)."""
import numpy as np
import pytest

import exact_attention_105_b200 as ea
import oracle
import workloads


@pytest.mark.gpu
def test_bounded_wait_reports_timeout_and_context_survives():
    ea.attn_check_status()                    # start from a clean status word
    ea.selftest_wait_timeout()
    with pytest.raises(ea.AttnError) as err:
        ea.attn_check_status()
    assert err.value.status == ea.ATTN_ERR_TIMEOUT
    assert "gave up" in str(err.value)
    ea.attn_check_status()                    # the word was cleared
    # The context still works: a small forward matches the oracle.
    w = workloads.small("after_timeout", 1, 2, 2, 200, 64, True, seed=3, backward=False)
    q, k, v = workloads.make_inputs(w, with_grad_out=False)
    o, lse = ea.attn_fwd(q.cuda(), k.cuda(), v.cuda(), scale=w.scale, causal=True)
    ea.attn_check_status()
    o_ref, lse_ref = oracle.attention_forward(q, k, v, w.scale, True)
    assert np.abs(o.float().cpu().numpy() - o_ref).max() <= 1e-2
    assert np.abs(lse.cpu().numpy() - lse_ref).max() <= 1e-3


def test_host_errors_carry_a_message():
    from exact_attention_105_b200 import build as eabuild
    eabuild.build()
    lib = ea.load_library()
    st = lib.attn_fwd(1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 1, 6, 4, 128, 64, 0.1, 0, None)
    assert st == ea.ATTN_ERR_ARG
    assert "divisible" in lib.attn_get_last_error().decode()
