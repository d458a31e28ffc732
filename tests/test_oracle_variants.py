"""Pins of the oracle's softcapping and varlen (packed batch) readings.

Softcapping (hysenlabs.com "FlashAttention: exakte Attention-Kernel fuer CUDA
und ROCm", section "Von 2.0 bis 2.7", release 2.6) has no formula on the pages;
the oracle reads it as c * tanh(z / c) on the scaled logits. Varlen (release
2.0, "unpadded" functions) is read as sequences packed token by token with
cu_seqlens offsets. These tests pin both readings to limits with closed forms,
to pure-Python brute force, to torch float64 library routines with an
independently built mask, and to finite differences.
"""
import math

import numpy as np
import pytest
import torch

import oracle

rng = np.random.default_rng(4321)


def rand(*shape, scale=1.0):
    return rng.standard_normal(shape) * scale


# ---------------------------------------------------------------- softcapping

@pytest.mark.parametrize("causal", [False, True])
def test_huge_cap_is_plain_attention(causal):
    """c tanh(z/c) = z - z^3/(3c^2) + ...: with c = 1e7 the change is below 1e-13."""
    q, k, v = rand(1, 2, 9, 8), rand(1, 2, 9, 8), rand(1, 2, 9, 8)
    o1, l1 = oracle.attention_forward(q, k, v, 0.4, causal)
    o2, l2 = oracle.attention_forward(q, k, v, 0.4, causal, softcap=1e7)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l2, l1, rtol=0, atol=1e-12)


@pytest.mark.parametrize("nq,nk,causal,window", [(7, 7, False, (-1, -1)), (5, 9, True, (-1, -1)),
                                                 (8, 8, False, (2, 1))])
def test_tiny_cap_is_uniform_attention(nq, nk, causal, window):
    """As c -> 0 every capped logit is within c of 0, so each row's weights are
    uniform over its visible keys: O = mean of those V rows, lse = ln(count)."""
    q, k, v = rand(nq, 8, scale=3.0), rand(nk, 8), rand(nk, 8)
    c = 1e-10
    o, lse = oracle.attention_head(q, k, v, 1.0, causal, window=window, softcap=c)
    vis = oracle.visible(np.arange(nq), nq, nk, causal, window)
    for i in range(nq):
        cnt = int(vis[i].sum())
        if cnt == 0:
            assert lse[i] == -np.inf and np.all(o[i] == 0)
            continue
        np.testing.assert_allclose(o[i], v[vis[i]].mean(axis=0), rtol=0, atol=1e-8)
        assert abs(lse[i] - math.log(cnt)) <= 2 * c


def test_capped_logits_bound_lse():
    """|c tanh(z/c)| < c, so ln(n) - c < lse < ln(n) + c for a row over n keys."""
    q, k, v = rand(16, 8, scale=5.0), rand(40, 8, scale=5.0), rand(40, 8)
    for c in (0.5, 3.0, 30.0):
        _, lse = oracle.attention_head(q, k, v, 1.0, False, softcap=c)
        assert np.all(lse < math.log(40) + c) and np.all(lse > math.log(40) - c)


@pytest.mark.parametrize("window", [(-1, -1), (2, 0)])
@pytest.mark.parametrize("nq,nk,causal", [(4, 4, False), (3, 6, True), (6, 3, True)])
def test_softcap_bruteforce(nq, nk, causal, window):
    q, k, v = rand(nq, 5, scale=2.0), rand(nk, 5, scale=2.0), rand(nk, 3)
    o, lse = oracle.attention_head(q, k, v, 0.7, causal, window=window, softcap=1.3)
    ob, lb = oracle.attention_bruteforce(q.tolist(), k.tolist(), v.tolist(), 0.7, causal, window,
                                         softcap=1.3)
    np.testing.assert_allclose(o, np.array(ob), rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, np.array(lb), rtol=0, atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_softcap_backward_matches_torch_autograd(causal):
    """torch float64 autograd differentiates the capped forward on its own; the
    oracle's backward carries a hand-derived 1 - tanh^2 factor."""
    B, Hq, Hkv, N, d, c = 1, 4, 2, 11, 8, 2.5
    q = torch.randn(B, Hq, N, d, dtype=torch.float64, requires_grad=True)
    k = torch.randn(B, Hkv, N, d, dtype=torch.float64, requires_grad=True)
    v = torch.randn(B, Hkv, N, d, dtype=torch.float64, requires_grad=True)
    do = torch.randn(B, Hq, N, d, dtype=torch.float64)
    kk = k.repeat_interleave(Hq // Hkv, dim=1)
    vv = v.repeat_interleave(Hq // Hkv, dim=1)
    z = torch.tanh((q @ kk.transpose(-1, -2)) * 0.6 / c) * c
    if causal:
        z = z.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
    out = torch.softmax(z, dim=-1) @ vv
    (out * do).sum().backward()
    o, _ = oracle.attention_forward(q.detach(), k.detach(), v.detach(), 0.6, causal, softcap=c)
    np.testing.assert_allclose(o, out.detach().numpy(), rtol=0, atol=1e-12)
    dq, dk, dv = oracle.attention_backward(q.detach(), k.detach(), v.detach(), do, 0.6, causal,
                                           softcap=c)
    np.testing.assert_allclose(dq, q.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk, k.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv, v.grad.numpy(), rtol=0, atol=1e-12)


def _numeric_grads(f, arrays, eps=1e-5):
    out = []
    for x in arrays:
        g = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            keep = x[idx]
            x[idx] = keep + eps
            fp = f()
            x[idx] = keep - eps
            fm = f()
            x[idx] = keep
            g[idx] = (fp - fm) / (2 * eps)
        out.append(g)
    return out


@pytest.mark.parametrize("window", [(-1, -1), (1, 1)])
def test_softcap_gradients_by_central_differences(window):
    q, k, v, do = rand(1, 2, 5, 3, scale=2.0), rand(1, 1, 6, 3, scale=2.0), rand(1, 1, 6, 3), rand(1, 2, 5, 3)
    c = 0.9

    def loss():
        o, _ = oracle.attention_forward(q, k, v, 0.8, True, window=window, softcap=c)
        return float(np.sum(o * do))

    num = _numeric_grads(loss, [q, k, v])
    got = oracle.attention_backward(q, k, v, do, 0.8, True, window=window, softcap=c)
    for n, g in zip(num, got):
        assert np.max(np.abs(n - g)) / np.max(np.abs(g)) <= 1e-6


def test_dropping_the_tanh_derivative_is_caught():
    """A planted mistake (the backward without the 1 - tanh^2 factor, i.e. the
    uncapped gradient) differs from finite differences of the capped forward."""
    q, k, v, do = rand(4, 3, scale=2.0), rand(4, 3, scale=2.0), rand(4, 3), rand(4, 3)
    c = 0.7

    def loss():
        o, _ = oracle.attention_head(q, k, v, 1.0, False, softcap=c)
        return float(np.sum(o * do))

    num = _numeric_grads(loss, [q])[0]
    s = oracle.scores(q, k, 1.0, False, softcap=c)
    p, _, _ = oracle.softmax_rows(s)
    dp = do @ v.T
    ds_wrong = p * (dp - np.sum(p * dp, axis=1, keepdims=True))     # factor missing
    assert np.max(np.abs(ds_wrong @ k - num)) > 1e-3
    good = oracle.attention_head_bwd(q, k, v, do, 1.0, False, softcap=c)[0]
    assert np.max(np.abs(good - num)) < 1e-8


def test_softcap_rejects_negative():
    with pytest.raises(ValueError):
        oracle.capped(np.zeros(3), -1.0)


# ---------------------------------------------------------------- varlen

def _pack(lens, H, d, scale=1.0):
    return rand(int(sum(lens)), H, d, scale=scale)


def _cu(lens):
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)


def block_diagonal_mask(lens_q, lens_k, causal, window):
    """[total_q, total_k] mask over the whole packed batch, built token by
    token from each token's sequence id and position within its sequence."""
    seq_q = np.repeat(np.arange(len(lens_q)), lens_q)
    seq_k = np.repeat(np.arange(len(lens_k)), lens_k)
    pos_q = np.concatenate([np.arange(n) for n in lens_q]) if sum(lens_q) else np.zeros(0, int)
    pos_k = np.concatenate([np.arange(n) for n in lens_k]) if sum(lens_k) else np.zeros(0, int)
    m = np.zeros((len(seq_q), len(seq_k)), dtype=bool)
    for a in range(len(seq_q)):
        for b in range(len(seq_k)):
            s = seq_q[a]
            if seq_k[b] != s:
                continue
            shift = lens_k[s] - lens_q[s]           # bottom-right alignment per sequence
            i, j = pos_q[a], pos_k[b]
            ok = True
            if causal and j > i + shift:
                ok = False
            if window[1] >= 0 and j > i + shift + window[1]:
                ok = False
            if window[0] >= 0 and j < i + shift - window[0]:
                ok = False
            m[a, b] = ok
    return m


CASES = [
    ([5, 9, 1], [5, 9, 1], False, (-1, -1), 0.0),
    ([5, 9, 1], [7, 4, 3], True, (-1, -1), 0.0),
    ([3, 0, 6, 2], [4, 2, 0, 5], True, (-1, -1), 0.0),      # empty query and key sequences
    ([8, 6], [8, 11], False, (2, 1), 0.0),
    ([8, 6], [8, 11], True, (3, -1), 1.5),
]


@pytest.mark.parametrize("lens_q,lens_k,causal,window,softcap", CASES)
def test_varlen_matches_one_attention_with_a_block_diagonal_mask(lens_q, lens_k, causal, window,
                                                                  softcap):
    """Library routine on the whole packed batch: torch float64 softmax over
    the capped logits with the block-diagonal mask, and its autograd."""
    Hq, Hkv, d, scale = 4, 2, 8, 0.5
    qn, kn, vn, don = (_pack(lens_q, Hq, d), _pack(lens_k, Hkv, d), _pack(lens_k, Hkv, d),
                       _pack(lens_q, Hq, d))
    cq, ck = _cu(lens_q), _cu(lens_k)
    mask = torch.from_numpy(block_diagonal_mask(lens_q, lens_k, causal, window))
    q = torch.from_numpy(qn).requires_grad_()
    k = torch.from_numpy(kn).requires_grad_()
    v = torch.from_numpy(vn).requires_grad_()
    G = Hq // Hkv
    qh = q.permute(1, 0, 2)                                   # [Hq, total_q, d]
    kh = k.permute(1, 0, 2).repeat_interleave(G, dim=0)
    vh = v.permute(1, 0, 2).repeat_interleave(G, dim=0)
    z = (qh @ kh.transpose(-1, -2)) * scale
    if softcap > 0:
        z = torch.tanh(z / softcap) * softcap
    z = z.masked_fill(~mask, float("-inf"))
    rows_ok = mask.any(dim=1)
    p = torch.softmax(torch.where(rows_ok[None, :, None], z, torch.zeros_like(z)), dim=-1)
    p = torch.where(mask[None], p, torch.zeros_like(p))
    out = (p @ vh).permute(1, 0, 2)                           # [total_q, Hq, d]
    lse_t = torch.logsumexp(z, dim=-1)                        # -inf on empty rows
    (out * torch.from_numpy(don)).sum().backward()

    o, lse = oracle.attention_forward_varlen(qn, kn, vn, cq, ck, scale, causal, window, softcap)
    np.testing.assert_allclose(o, out.detach().numpy(), rtol=0, atol=1e-12)
    np.testing.assert_array_equal(np.isneginf(lse), np.isneginf(lse_t.detach().numpy()))
    fin = np.isfinite(lse)
    np.testing.assert_allclose(lse[fin], lse_t.detach().numpy()[fin], rtol=0, atol=1e-12)
    dq, dk, dv = oracle.attention_backward_varlen(qn, kn, vn, don, cq, ck, scale, causal, window,
                                                  softcap)
    np.testing.assert_allclose(dq, q.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk, k.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv, v.grad.numpy(), rtol=0, atol=1e-12)


def test_varlen_with_equal_lengths_is_the_padded_batch():
    B, H, N, d = 3, 2, 7, 4
    q, k, v = rand(B, H, N, d), rand(B, H, N, d), rand(B, H, N, d)
    o_b, l_b = oracle.attention_forward(q, k, v, 0.5, True)
    pack = lambda x: x.transpose(0, 2, 1, 3).reshape(B * N, H, d)   # [B,H,N,d] -> [B*N,H,d]
    cu = _cu([N] * B)
    o_v, l_v = oracle.attention_forward_varlen(pack(q), pack(k), pack(v), cu, cu, 0.5, True)
    np.testing.assert_allclose(o_v, pack(o_b), rtol=0, atol=1e-14)
    np.testing.assert_allclose(l_v, l_b.transpose(1, 0, 2).reshape(H, B * N), rtol=0, atol=1e-14)


def test_varlen_bruteforce_per_sequence():
    lens_q, lens_k = [2, 3, 0, 1], [3, 1, 2, 4]
    q, k, v = _pack(lens_q, 1, 3), _pack(lens_k, 1, 3), _pack(lens_k, 1, 2)
    cq, ck = _cu(lens_q), _cu(lens_k)
    o, lse = oracle.attention_forward_varlen(q, k, v, cq, ck, 0.9, True)
    for b in range(4):
        qs = q[cq[b]:cq[b + 1], 0].tolist()
        if not qs:
            continue
        ob, lb = oracle.attention_bruteforce(qs, k[ck[b]:ck[b + 1], 0].tolist(),
                                             v[ck[b]:ck[b + 1], 0].tolist(), 0.9, True)
        np.testing.assert_allclose(o[cq[b]:cq[b + 1], 0], np.array(ob), rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse[0, cq[b]:cq[b + 1]], np.array(lb), rtol=0, atol=1e-14)


@pytest.mark.parametrize("cu", [[1, 3], [0, 4, 3], [0, 2]])
def test_varlen_rejects_bad_offsets(cu):
    q = rand(3, 1, 2)
    with pytest.raises(ValueError):
        oracle.attention_forward_varlen(q, q, q, cu, [0, 3] if len(cu) == 2 else [0, 1, 3], 1.0, False)


# ---------------------------------------------------------------- row-wise dQ

@pytest.mark.parametrize("causal,window,softcap", [(True, (-1, -1), 0.0), (False, (3, 2), 0.0),
                                                   (True, (-1, -1), 1.5)])
def test_dq_rows_equal_the_full_backward(causal, window, softcap):
    """The row-wise dQ used for full-size spot checks is the same gradient the
    whole-head backward gives (which central differences pin above)."""
    B, Hq, Hkv, N, d = 1, 4, 2, 23, 8
    q, k, v, do = rand(B, Hq, N, d), rand(B, Hkv, N, d), rand(B, Hkv, N, d), rand(B, Hq, N, d)
    dq, _, _ = oracle.attention_backward(q, k, v, do, 0.6, causal, window=window, softcap=softcap)
    rows = [0, 1, 7, 21, 22]
    for b, h in ((0, 0), (0, 3)):
        got = oracle.attention_backward_dq_rows(q, k, v, do, 0.6, causal, b, h, rows,
                                                window=window, softcap=softcap)
        np.testing.assert_allclose(got, dq[b, h][rows], rtol=0, atol=1e-12)


def test_gradient_identities_hold_in_the_oracle():
    """Identities the GPU tests use at sizes the oracle cannot run whole:
    the weights of a row sum to one, so sum_k dV[k] = sum_q dO[q]; the entries
    of a row of dS sum to zero, so sum_k dK[k] = 0."""
    q, k, v, do = rand(1, 2, 30, 8), rand(1, 2, 30, 8), rand(1, 2, 30, 8), rand(1, 2, 30, 8)
    _, dk, dv = oracle.attention_backward(q, k, v, do, 0.5, True)
    np.testing.assert_allclose(dv.sum(axis=2), do.sum(axis=2), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, rtol=0, atol=1e-12)
