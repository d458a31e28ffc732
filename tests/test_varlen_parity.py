"""GPU parity of the packed ("varlen") calls against the float64 oracle.

The pages (hysenlabs.com "FlashAttention: exakte Attention-Kernel fuer CUDA
und ROCm", section "Von 2.0 bis 2.7") name the varlen functions of release
2.0. The layout read here is the one the oracle pins: q/o [total_q, Hq, d],
k/v [total_k, Hkv, d], lse [Hq, total_q], int32 cu_seqlens. Each sequence
attends within itself with its own bottom-right causal alignment, window
and softcap. Tolerances are those of the other calls."""
import numpy as np
import pytest
import torch

import exact_attention_105_b200 as ea
import oracle
import workloads
from tests.gpu_helpers import GRAD_REL_TOL, LSE_TOL, O_TOL, max_err

pytestmark = pytest.mark.gpu

ZERO_REF_FLOOR = 1e-5


def run(lens_q, lens_k, Hq, Hkv, d, causal, window, softcap, seed, q_mult=1.0, backward=True):
    q, k, v, do, cq, ck = workloads.make_packed_inputs(lens_q, lens_k, Hq, Hkv, d, seed, q_mult)
    dev = [t.cuda() for t in (q, k, v, do, cq, ck)]
    qd, kd, vd, dod, cqd, ckd = dev
    mq, mk = max(lens_q), max(lens_k)
    scale = d ** -0.5
    o, lse = ea.attn_fwd_varlen(qd, kd, vd, cqd, ckd, mq, mk, scale=scale, causal=causal,
                                window=window, softcap=softcap)
    grads = None
    if backward:
        grads = ea.attn_bwd_varlen(qd, kd, vd, o, lse, dod, cqd, ckd, mq, mk, scale=scale,
                                   causal=causal, window=window, softcap=softcap)
    ea.attn_check_status()
    return (q, k, v, do, cq, ck, scale), (o, lse), grads


def check_fwd(inputs, o, lse, causal, window, softcap, label):
    q, k, v, _, cq, ck, scale = inputs
    o_ref, lse_ref = oracle.attention_forward_varlen(q, k, v, cq.numpy(), ck.numpy(), scale,
                                                     causal, window, softcap)
    o = o.float().cpu().numpy()
    lse = lse.cpu().numpy()
    assert np.all(np.isfinite(o)), f"{label}: non-finite O"
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), empty), f"{label}: rows with lse = -inf differ"
    eo, io = max_err(o, o_ref)
    assert eo <= O_TOL, f"{label}: max|O-O_ref| = {eo:.3e} at {io}"
    if (~empty).any():
        el, _ = max_err(lse[~empty], lse_ref[~empty])
        assert el <= LSE_TOL, f"{label}: max|lse-lse_ref| = {el:.3e}"


def check_bwd(inputs, grads, causal, window, softcap, label):
    q, k, v, do, cq, ck, scale = inputs
    refs = oracle.attention_backward_varlen(q, k, v, do, cq.numpy(), ck.numpy(), scale, causal,
                                            window, softcap)
    for name, g, ref in zip(("dq", "dk", "dv"), grads, refs):
        g = g.float().cpu().numpy()
        assert np.all(np.isfinite(g)), f"{label}: non-finite {name}"
        e, idx = max_err(g, ref)
        bound = max(GRAD_REL_TOL * float(np.abs(ref).max(initial=0.0)), ZERO_REF_FLOOR)
        assert e <= bound, f"{label}: {name} max err {e:.3e} at {idx} > {bound:.3e}"


# (lens_q, lens_k, Hq, Hkv, d, causal, window, softcap)
CASES = [
    ([300, 128, 1, 517], [300, 128, 1, 517], 2, 2, 128, True, (-1, -1), 0.0),
    ([300, 128, 1, 517], [300, 128, 1, 517], 2, 2, 64, False, (-1, -1), 0.0),
    ([100, 0, 250, 7], [400, 33, 0, 129], 4, 2, 128, True, (-1, -1), 0.0),   # empty sequences
    ([129, 640], [1000, 64], 2, 1, 128, True, (200, -1), 0.0),
    ([256, 300, 5], [256, 300, 5], 4, 4, 64, False, (31, 17), 0.0),
    ([384, 200], [384, 700], 8, 2, 128, True, (-1, -1), 30.0),
    ([777], [777], 2, 2, 128, False, (-1, -1), 5.0),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"q{'-'.join(map(str, c[0]))}_k{'-'.join(map(str, c[1]))}_H{c[2]}_{c[3]}_d{c[4]}_c{int(c[5])}_w{c[6][0]}_{c[6][1]}_cap{c[7]:g}")
def test_varlen_fwd_bwd(case):
    lens_q, lens_k, Hq, Hkv, d, causal, window, cap = case
    inputs, (o, lse), grads = run(lens_q, lens_k, Hq, Hkv, d, causal, window, cap,
                                  seed=sum(lens_q) + 3 * sum(lens_k) + d,
                                  q_mult=2.0 if cap else 1.0)
    check_fwd(inputs, o, lse, causal, window, cap, str(case))
    check_bwd(inputs, grads, causal, window, cap, str(case))


def test_varlen_equal_lengths_match_the_fixed_layout():
    """Packed equal-length sequences give the fixed-layout results (a different
    tensor map and the general mask mode; the same arithmetic)."""
    B, H, N, d = 3, 4, 333, 128
    q, k, v, do = workloads.make_inputs_qk(B, H, H, N, N, d, seed=9)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o1, l1 = ea.attn_fwd(qd, kd, vd, causal=True)
    g1 = ea.attn_bwd(qd, kd, vd, o1, l1, dod, causal=True)
    pack = lambda x: x.transpose(1, 2).reshape(B * N, H, d).contiguous()
    cu = torch.arange(0, (B + 1) * N, N, dtype=torch.int32, device="cuda")
    o2, l2 = ea.attn_fwd_varlen(pack(qd), pack(kd), pack(vd), cu, cu, N, N, causal=True)
    g2 = ea.attn_bwd_varlen(pack(qd), pack(kd), pack(vd), o2, l2, pack(dod), cu, cu, N, N,
                            causal=True)
    ea.attn_check_status()
    assert (pack(o1).float() - o2.float()).abs().max().item() <= 1e-2
    assert (l1.transpose(0, 1).reshape(H, B * N) - l2).abs().max().item() <= 1e-3
    for a, b in zip(g1, g2):
        a = pack(a).float()
        assert (a - b.float()).abs().max().item() <= 2e-2 * a.abs().max().item()


def test_varlen_deterministic():
    lens = [500, 123, 900]
    r1 = run(lens, lens, 4, 2, 128, True, (-1, -1), 0.0, seed=3)
    r2 = run(lens, lens, 4, 2, 128, True, (-1, -1), 0.0, seed=3)
    assert torch.equal(r1[1][0], r2[1][0]) and torch.equal(r1[1][1], r2[1][1])
    for a, b in zip(r1[2], r2[2]):
        assert torch.equal(a, b)


def test_varlen_mixed_lengths_larger():
    """A longer mix (about 7k tokens, lengths from 1 to 3000) in the forward
    and backward."""
    lens = [1000, 3000, 517, 2048, 1, 129]
    inputs, (o, lse), grads = run(lens, lens, 4, 2, 128, True, (-1, -1), 0.0, seed=17)
    check_fwd(inputs, o, lse, True, (-1, -1), 0.0, "mix")
    check_bwd(inputs, grads, True, (-1, -1), 0.0, "mix")


def test_invalid_offsets_are_reported_and_clipped():
    """Offsets that decrease are found on the GPU: the call stays in bounds,
    the status check raises ATTN_ERR_ARG, and the next valid call is clean."""
    q, k, v, do, cq, ck = workloads.make_packed_inputs([200, 100], [200, 100], 2, 2, 128, seed=5)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    bad = torch.tensor([0, 250, 150], dtype=torch.int32, device="cuda")   # 250 > 150
    ea.attn_fwd_varlen(qd, kd, vd, bad, bad, 200, 200, causal=True)
    with pytest.raises(ea.AttnError) as err:
        ea.attn_check_status()
    assert err.value.status == ea.ATTN_ERR_ARG
    ea.attn_fwd_varlen(qd, kd, vd, cq.cuda(), ck.cuda(), 200, 200, causal=True)
    ea.attn_check_status()


def test_sequence_longer_than_max_seqlen_is_reported():
    q, k, v, do, cq, ck = workloads.make_packed_inputs([300], [300], 2, 2, 64, seed=6)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    ea.attn_fwd_varlen(qd, kd, vd, cq.cuda(), ck.cuda(), 256, 300)      # max_seqlen_q too small
    with pytest.raises(ea.AttnError) as err:
        ea.attn_check_status()
    assert err.value.status == ea.ATTN_ERR_ARG
