"""Long sequences, beyond what the oracle can materialise whole.

Forward at N = 131072: sampled rows against the oracle, which computes each
row over all of its keys. Backward at N = 32768 with GQA: sampled dQ rows
against the oracle's row-wise gradient, and two identities that hold at any
size (pinned in the oracle tests): sum_k dV[k] = sum_q dO[q] over the query
heads of a KV group, and sum_k dK[k] = 0."""
import numpy as np
import pytest
import torch

import exact_attention_105_b200 as ea
import oracle
import workloads
from tests.gpu_helpers import GRAD_REL_TOL, LSE_TOL, O_TOL, max_err

pytestmark = pytest.mark.gpu


def test_forward_n131072_sampled_rows():
    B, Hq, Hkv, N, d = 1, 2, 1, 131072, 128
    q, k, v = workloads.make_inputs_qk(B, Hq, Hkv, N, N, d, seed=131, with_grad_out=False)
    o, lse = ea.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True)
    ea.attn_check_status()
    o = o.float().cpu().numpy()
    lse = lse.cpu().numpy()
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 65535, 65536, N - 2, N - 1],
                                     rng.integers(0, N, 16)]))
    for h in range(Hq):
        o_ref, l_ref = oracle.attention_forward_rows(q, k, v, d ** -0.5, True, 0, h, rows)
        eo, _ = max_err(o[0, h][rows], o_ref)
        el, _ = max_err(lse[0, h][rows], l_ref)
        assert eo <= O_TOL and el <= LSE_TOL, (h, eo, el)


def test_backward_n32768_gqa():
    B, Hq, Hkv, N, d = 1, 4, 2, 32768, 128
    G = Hq // Hkv
    q, k, v, do = workloads.make_inputs_qk(B, Hq, Hkv, N, N, d, seed=327)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = ea.attn_fwd(qd, kd, vd, causal=True)
    dq, dk, dv = ea.attn_bwd(qd, kd, vd, o, lse, dod, causal=True)
    ea.attn_check_status()
    dq, dk, dv = (t.double().cpu().numpy() for t in (dq, dk, dv))
    for t in (dq, dk, dv):
        assert np.all(np.isfinite(t))
    do64 = do.double().numpy()
    for hk in range(Hkv):
        want_dv = do64[0, hk * G:(hk + 1) * G].sum(axis=(0, 1))
        got_dv = dv[0, hk].sum(axis=0)
        scale_dv = np.abs(dv[0, hk]).sum(axis=0).max()
        assert np.abs(got_dv - want_dv).max() <= 2e-3 * scale_dv, "sum_k dV != sum_q dO"
        got_dk = dk[0, hk].sum(axis=0)
        scale_dk = np.abs(dk[0, hk]).sum(axis=0).max()
        assert np.abs(got_dk).max() <= 2e-3 * scale_dk, "sum_k dK != 0"
    rng = np.random.default_rng(1)
    rows = np.unique(np.concatenate([[0, 1, 128, N // 2, N - 1], rng.integers(0, N, 11)]))
    for h in (0, Hq - 1):
        ref = oracle.attention_backward_dq_rows(q, k, v, do, d ** -0.5, True, 0, h, rows)
        e, idx = max_err(dq[0, h][rows], ref)
        assert e <= GRAD_REL_TOL * np.abs(ref).max(), (h, e, idx)
