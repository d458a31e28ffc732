"""GPU backward parity: dQ, dK, dV from the sm_100a kernels against the float64
oracle's exact gradient, on the same seeded bf16 inputs. The forward outputs
(o, lse) fed to the backward come from the GPU forward, as in training.

Tolerance: for each of dQ, dK, dV, max|got - ref| <= 2e-2 * max|ref|. When
the reference is identically zero (N = 1: the single weight is 1, so
dS = P * (dP - D) = 0 and dQ = 0), the relative bound is 0, and an absolute
floor of 1e-5 applies instead. That is far below the bf16 resolution of any
nonzero gradient here."""
import numpy as np
import pytest
import torch

import exact_attention_105_b200 as ea
import oracle
import workloads
from tests.gpu_helpers import GRAD_REL_TOL, max_err, to_dev

ZERO_REF_FLOOR = 1e-5

pytestmark = pytest.mark.gpu


def gpu_fwd_bwd(q, k, v, do, scale, causal):
    """Forward and backward into gradients pre-filled with NaN (see
    assert_grads_close, which checks the whole of each gradient is finite)."""
    qd, kd, vd, dod = to_dev(q, k, v, do)
    o, lse = ea.attn_fwd(qd, kd, vd, scale=scale, causal=causal)
    dq, dk, dv = (torch.full_like(t, float("nan")) for t in (qd, kd, vd))
    ea.attn_bwd(qd, kd, vd, o, lse, dod, dq, dk, dv, scale=scale, causal=causal)
    ea.attn_check_status()
    return dq, dk, dv


def assert_grads_close(got, refs, label, heads=None):
    errs = {}
    for name, g, ref in zip(("dq", "dk", "dv"), got, refs):
        g = g.float().cpu().numpy()
        assert np.all(np.isfinite(g)), f"{label}: non-finite {name} (an element left unwritten?)"
        if heads is not None:
            sel = heads[name]
            g = np.stack([g[b, h] for b, h in sel])
            ref = np.stack([ref[b, h] for b, h in sel])
        assert np.all(np.isfinite(g)), f"{label}: non-finite {name}"
        e, idx = max_err(g, ref)
        bound = max(GRAD_REL_TOL * float(np.abs(ref).max()), ZERO_REF_FLOOR)
        assert e <= bound, f"{label}: {name} max err {e:.3e} at {idx} > {bound:.3e}"
        errs[name] = e / max(float(np.abs(ref).max()), 1e-30)
    return errs


def check(w):
    q, k, v, do = workloads.make_inputs(w)
    got = gpu_fwd_bwd(q, k, v, do, w.scale, w.causal)
    refs = oracle.attention_backward(q, k, v, do, w.scale, w.causal)
    return assert_grads_close(got, refs, w.name), (q, k, v, do, got, refs)


SHAPES = []
for d in (64, 128):
    for causal in (False, True):
        for n in (1, 100, 128, 129, 300, 512):
            SHAPES.append(workloads.small(f"bwd_N{n}_d{d}_c{int(causal)}", 1, 2, 2, n, d, causal,
                                          seed=3 * n + d))


@pytest.mark.parametrize("w", SHAPES, ids=lambda w: w.name)
def test_bwd_small_shapes(w):
    check(w)


@pytest.mark.parametrize("hq,hkv,causal", [(4, 1, True), (4, 2, False), (6, 3, True), (8, 2, True)])
def test_bwd_gqa(hq, hkv, causal):
    """GQA backward: dK and dV of a KV head sum over its query-head group."""
    check(workloads.small(f"bwd_gqa_{hq}_{hkv}", 2, hq, hkv, 384, 128, causal, seed=hq + 7 * hkv))


def test_bwd_large_logits():
    check(workloads.small("bwd_q4", 1, 2, 2, 700, 128, True, q_mult=4.0, seed=21))


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_d64_many_items(causal):
    """d = 64 with more work items than SMs (dK/dV: 2 x 16 x 9 = 288, items of
    odd and even step counts in a row), so the dK/dV kernel's alternating S^T
    buffers run across item boundaries; three whole heads against the oracle."""
    w = workloads.small(f"bwd_d64_items_c{int(causal)}", 2, 16, 16, 1100, 64, causal,
                        seed=51 + int(causal))
    q, k, v, do = workloads.make_inputs(w)
    got = gpu_fwd_bwd(q, k, v, do, w.scale, w.causal)
    picks = [(0, 0), (0, 9), (1, 15)]
    refs = oracle.attention_backward(q, k, v, do, w.scale, w.causal, heads=picks)
    assert_grads_close(got, refs, w.name, heads={"dq": picks, "dk": picks, "dv": picks})


def test_bwd_c5_full_size_sampled_heads():
    """The training-step workload at full size; three whole heads compared exactly."""
    w = workloads.C5
    q, k, v, do = workloads.make_inputs(w)
    got = gpu_fwd_bwd(q, k, v, do, w.scale, w.causal)
    picks = [(0, 0), (3, 7), (w.B - 1, w.Hq - 1)]
    refs = oracle.attention_backward(q, k, v, do, w.scale, w.causal, heads=picks)
    heads = {"dq": picks, "dk": picks, "dv": picks}
    assert_grads_close(got, refs, w.name, heads=heads)
    for g in got:
        assert torch.isfinite(g.float()).all()


def test_bwd_workspace_contents_ignored():
    """The backward's workspace (the lse/D rows and the work counters that the
    persistent dK/dV and dQ kernels hand items out from) may hold anything on
    entry: a workspace of 0xFF bytes (counters at -1), reused twice in a row,
    gives the same gradients bit for bit as a zeroed one. The shape has more
    work items than SMs (dK/dV: 4 x 4 x 18 = 288, dQ: 4 x 16 x 18 = 1152), so
    the CTAs take items from the counters; two heads are checked against the
    oracle as well."""
    w = workloads.small("bwd_persistent", 4, 16, 4, 2304, 64, True, seed=41)
    q, k, v, do = workloads.make_inputs(w)
    qd, kd, vd, dod = to_dev(q, k, v, do)
    o, lse = ea.attn_fwd(qd, kd, vd, scale=w.scale, causal=True)
    need = ea.attn_bwd_workspace_size(w.B, w.Hq, w.N, w.d)
    clean = torch.zeros(need, dtype=torch.uint8, device="cuda")
    ref = ea.attn_bwd(qd, kd, vd, o, lse, dod, workspace=clean, scale=w.scale, causal=True)
    dirty = torch.full((need,), 0xFF, dtype=torch.uint8, device="cuda")
    for _ in range(2):
        got = ea.attn_bwd(qd, kd, vd, o, lse, dod, workspace=dirty, scale=w.scale, causal=True)
        ea.attn_check_status()
        for x, y in zip(got, ref):
            assert torch.equal(x, y)
    # The oracle computes the listed KV heads and every query head of their groups.
    kv_picks = [(0, 0), (w.B - 1, w.Hkv - 1)]
    refs = oracle.attention_backward(q, k, v, do, w.scale, True, heads=kv_picks)
    heads = {"dq": [(0, 0), (w.B - 1, w.Hq - 1)], "dk": kv_picks, "dv": kv_picks}
    assert_grads_close(ref, refs, w.name, heads=heads)


def test_bwd_deterministic():
    w = workloads.small("bwd_det", 2, 4, 2, 640, 128, True, seed=5)
    q, k, v, do = workloads.make_inputs(w)
    a = gpu_fwd_bwd(q, k, v, do, w.scale, True)
    b = gpu_fwd_bwd(q, k, v, do, w.scale, True)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_bwd_within_twice_naive_bf16_baseline():
    """Upstream methodology: gradient error at most twice that of plain bf16
    torch attention (autograd through materialised bf16 ops) against the same
    float64 reference."""
    w = workloads.small("bwd_naive", 2, 4, 4, 1024, 128, True, seed=17)
    errs, (q, k, v, do, got, refs) = check(w)
    qd, kd, vd, dod = (t.cuda().requires_grad_(True) for t in (q, k, v, do))
    s = torch.matmul(qd, kd.transpose(-1, -2)) * w.scale
    n = s.shape[-1]
    s = s.masked_fill(torch.ones(n, n, dtype=torch.bool, device="cuda").triu(1), float("-inf"))
    out = torch.matmul(torch.softmax(s, dim=-1).to(torch.bfloat16), vd)
    out.backward(dod.detach())
    for name, g, ref in zip(("dq", "dk", "dv"), (qd.grad, kd.grad, vd.grad), refs):
        e_naive = max_err(g.float().cpu().numpy(), ref)[0] / float(np.abs(ref).max())
        assert errs[name] <= 2.0 * e_naive + 1e-4, (name, errs[name], e_naive)
