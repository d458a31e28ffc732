"""GPU: the kernels write their outputs only inside the output tensors.

Each output tile leaves the kernel either as one 128-row TMA store (the rows
past the tensor are clipped by the tensor map) or row by row (a packed tile
that runs past its sequence). Here every output (O, lse, dQ, dK, dV) is a view
at the start of a larger buffer whose tail holds a sentinel bit pattern. After
a forward and a backward the tail must be unchanged, and the outputs must
still match the float64 oracle. The shapes make the last tile of the last head
(fixed layout) or of the last sequence (packed layout) ragged, and mix packed
sequences whose tiles are whole with ones whose last tile is not."""
import numpy as np
import pytest
import torch

import exact_attention_105_b200 as ea
import oracle
import workloads
from tests.gpu_helpers import GRAD_REL_TOL, LSE_TOL, O_TOL, max_err

pytestmark = pytest.mark.gpu

TAIL = 8192                     # sentinel elements after each output
SENTINEL16 = 0x5A5A             # as bf16 about 1.5e16: no output here is near it
SENTINEL32 = 0x5A5A5A5A


def padded(shape, dtype):
    """(buffer, view): the view is the first prod(shape) elements of a buffer
    whose remaining TAIL elements hold the sentinel."""
    n = int(np.prod(shape))
    buf = torch.empty(n + TAIL, dtype=dtype, device="cuda")
    if dtype == torch.bfloat16:
        buf.view(torch.int16).fill_(SENTINEL16)
    else:
        buf.view(torch.int32).fill_(SENTINEL32)
    return buf, buf[:n].view(shape)


def tail_intact(buf, n):
    if buf.dtype == torch.bfloat16:
        t = buf[n:].view(torch.int16)
        return bool((t == SENTINEL16).all().item())
    t = buf[n:].view(torch.int32)
    return bool((t == SENTINEL32).all().item())


def err(got, ref):
    return max_err(got.float().cpu().numpy(), ref)[0]


def check_grads(got, ref, label):
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        e = err(g, r)
        assert e <= GRAD_REL_TOL * float(np.abs(r).max()), (label, name, e)


@pytest.mark.parametrize("N,d,causal", [(300, 128, True), (300, 128, False), (200, 64, True)])
def test_fixed_layout_writes_stay_inside(N, d, causal):
    B, Hq, Hkv = 2, 4, 2
    q, k, v, do = workloads.make_inputs_qk(B, Hq, Hkv, N, N, d, seed=91)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    scale = d ** -0.5
    ob, o = padded((B, Hq, N, d), torch.bfloat16)
    lb, lse = padded((B, Hq, N), torch.float32)
    ea.attn_fwd(qd, kd, vd, o, lse, scale=scale, causal=causal)
    qb, dq = padded((B, Hq, N, d), torch.bfloat16)
    kb, dk = padded((B, Hkv, N, d), torch.bfloat16)
    vb, dv = padded((B, Hkv, N, d), torch.bfloat16)
    ea.attn_bwd(qd, kd, vd, o, lse, dod, dq, dk, dv, scale=scale, causal=causal)
    ea.attn_check_status()
    torch.cuda.synchronize()
    for buf, view, name in ((ob, o, "o"), (lb, lse, "lse"), (qb, dq, "dq"), (kb, dk, "dk"),
                            (vb, dv, "dv")):
        assert tail_intact(buf, view.numel()), f"{name}: write past the tensor"
    o_ref, lse_ref = oracle.attention_forward(q, k, v, scale, causal)
    assert err(o, o_ref) <= O_TOL
    assert err(lse, lse_ref) <= LSE_TOL
    check_grads((dq, dk, dv), oracle.attention_backward(q, k, v, do, scale, causal),
                f"fixed N={N} d={d}")


@pytest.mark.parametrize("lens,causal", [([128, 200, 256, 77], True),
                                          ([256, 128, 130], False)])
def test_packed_layout_writes_stay_inside(lens, causal):
    Hq, Hkv, d = 4, 2, 128
    q, k, v, do, cq, ck = workloads.make_packed_inputs(lens, lens, Hq, Hkv, d, seed=92)
    qd, kd, vd, dod, cqd, ckd = (t.cuda() for t in (q, k, v, do, cq, ck))
    total = sum(lens)
    mx = max(lens)
    scale = d ** -0.5
    ob, o = padded((total, Hq, d), torch.bfloat16)
    lb, lse = padded((Hq, total), torch.float32)
    ea.attn_fwd_varlen(qd, kd, vd, cqd, ckd, mx, mx, o, lse, scale=scale, causal=causal)
    qb, dq = padded((total, Hq, d), torch.bfloat16)
    kb, dk = padded((total, Hkv, d), torch.bfloat16)
    vb, dv = padded((total, Hkv, d), torch.bfloat16)
    ea.attn_bwd_varlen(qd, kd, vd, o, lse, dod, cqd, ckd, mx, mx, dq, dk, dv, scale=scale,
                       causal=causal)
    ea.attn_check_status()
    torch.cuda.synchronize()
    for buf, view, name in ((ob, o, "o"), (lb, lse, "lse"), (qb, dq, "dq"), (kb, dk, "dk"),
                            (vb, dv, "dv")):
        assert tail_intact(buf, view.numel()), f"{name}: write past the tensor"
    o_ref, lse_ref = oracle.attention_forward_varlen(q, k, v, cq.numpy(), ck.numpy(), scale,
                                                     causal)
    assert err(o, o_ref) <= O_TOL
    assert err(lse, lse_ref) <= LSE_TOL
    check_grads((dq, dk, dv),
                oracle.attention_backward_varlen(q, k, v, do, cq.numpy(), ck.numpy(), scale,
                                                 causal),
                f"packed {lens}")
