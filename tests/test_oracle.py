"""Pins for the float64 oracle, against facts that do not come from the oracle itself.

Each test states what fixes the expected value. Sources are the worked numbers
printed on the pages (tests/golden), closed forms, invariants of the
definition, independent library routines (scipy, torch's float64 CPU
attention and autograd), brute force and finite differences. The "mutants"
tests at the end plant plausible mistakes in copies of the oracle's formulas
and check that some pin catches each one.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from oracle import attention_ref as ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


def rand(*shape, scale=1.0):
    return rng.standard_normal(shape) * scale


# ---------------------------------------------------------------- sizing pins

def test_sizing_matches_printed_table():
    """tokenwerk.de, 'Warum Kacheln beim Speicherzugriff helfen': 2 MiB, 32 MiB, 128 KiB."""
    with open(os.path.join(GOLDEN, "dense_matrix_sizing.json")) as f:
        g = json.load(f)
    for row in g["rows"]:
        assert oracle.dense_score_matrix_cells(row["n"]) == row["cells"]
        assert oracle.dense_score_matrix_bytes(row["n"], bytes_per_cell=g["bytes_per_cell"]) == row["bytes"]
        unit, div = ("MiB", 2**20) if row["printed"].endswith("MiB") else ("KiB", 2**10)
        assert f"{row['bytes'] // div} {unit}" == row["printed"]
    big = oracle.dense_score_matrix_bytes(1024 * g["length_ratio"])
    assert big == g["size_ratio"] * oracle.dense_score_matrix_bytes(1024)


@pytest.mark.parametrize("n,expect_mib", [(1024, 2), (4096, 32)])
def test_materialised_scores_have_printed_size(n, expect_mib):
    """The oracle really materialises the N x N matrix the pages size (as 2-byte cells)."""
    q = rand(n, 2)
    s = oracle.scores(q, q, 1.0, causal=False)
    assert s.shape == (n, n)
    assert s.size == oracle.dense_score_matrix_cells(n)
    assert s.astype(np.float16).nbytes == expect_mib * 2**20


# ------------------------------------------------------------- softmax pins

@pytest.mark.parametrize("causal", [False, True])
def test_softmax_rows_are_distributions(causal):
    q, k = rand(37, 8), rand(37, 8)
    s = oracle.scores(q, k, 0.3, causal)
    p, _, _ = oracle.softmax_rows(s)
    assert np.all(p >= 0)
    assert np.max(np.abs(p.sum(axis=1) - 1.0)) <= 1e-12
    if causal:
        assert np.all(p[~oracle.causal_visible(37, 37)] == 0.0)


def test_softmax_and_lse_match_scipy():
    """Library routines: scipy.special.softmax and logsumexp of the scaled logits."""
    q, k, v = rand(50, 16), rand(50, 16), rand(50, 16)
    scale = 0.25
    s = q @ k.T * scale
    p, _, _ = oracle.softmax_rows(s)
    np.testing.assert_allclose(p, scipy.special.softmax(s, axis=1), rtol=0, atol=1e-13)
    o, lse = oracle.attention_head(q, k, v, scale, causal=False)
    np.testing.assert_allclose(lse, scipy.special.logsumexp(s, axis=1), rtol=0, atol=1e-12)
    np.testing.assert_allclose(o, scipy.special.softmax(s, axis=1) @ v, rtol=0, atol=1e-12)


# ------------------------------------------------------ value-path pins

@pytest.mark.parametrize("causal", [False, True])
def test_constant_v_gives_constant_o(causal):
    n, d = 40, 8
    c = rand(d)
    v = np.tile(c, (n, 1))
    o, _ = oracle.attention_head(rand(n, d), rand(n, d), v, 0.5, causal)
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-13)


def test_single_position():
    """N = 1: the only weight is 1, so O = V and lse = q.k * scale."""
    q, k, v = rand(1, 8), rand(1, 8), rand(1, 8)
    for causal in (False, True):
        o, lse = oracle.attention_head(q, k, v, 0.7, causal)
        np.testing.assert_allclose(o, v, rtol=0, atol=1e-15)
        assert abs(lse[0] - 0.7 * float(q[0] @ k[0])) <= 1e-14


def test_key_permutation_invariance():
    q, k, v = rand(30, 8), rand(45, 8), rand(45, 8)
    perm = rng.permutation(45)
    o1, l1 = oracle.attention_head(q, k, v, 0.4, causal=False)
    o2, l2 = oracle.attention_head(q, k[perm], v[perm], 0.4, causal=False)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)


def test_hand_checked_two_by_two():
    """q = k = identity, scale 1, causal: row 0 sees key 0 only; row 1 weights [1, e]/(1+e)."""
    eye = np.eye(2)
    v = np.array([[3.0, -1.0], [5.0, 2.0]])
    o, lse = oracle.attention_head(eye, eye, v, 1.0, causal=True)
    np.testing.assert_allclose(o[0], v[0], rtol=0, atol=1e-15)
    w = np.array([1.0, math.e]) / (1.0 + math.e)
    np.testing.assert_allclose(o[1], w @ v, rtol=0, atol=1e-15)
    assert abs(lse[0] - 1.0) <= 1e-15          # ln(exp(q0.k0)) = 1
    assert abs(lse[1] - math.log(1.0 + math.e)) <= 1e-15


def test_causal_bottom_right_alignment():
    """hysenlabs.com, 'Von 2.0 bis 2.7': with Nq < Nk the mask ends at the bottom-right corner."""
    vis = oracle.causal_visible(2, 5)
    assert vis.tolist() == [[True, True, True, True, False], [True, True, True, True, True]]
    vis_short_k = oracle.causal_visible(4, 2)   # first two queries see nothing
    assert vis_short_k.sum(axis=1).tolist() == [0, 0, 1, 2]
    o, lse = oracle.attention_head(rand(4, 3), rand(2, 3), rand(2, 3), 1.0, causal=True)
    assert np.all(o[:2] == 0.0) and np.all(np.isneginf(lse[:2]))


# ------------------------------------------------------------ brute force

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("nq,nk", [(1, 1), (3, 3), (4, 4), (2, 4), (4, 2)])
def test_bruteforce_tiny(causal, nq, nk):
    q, k, v = rand(nq, 3), rand(nk, 3), rand(nk, 2)
    o, lse = oracle.attention_head(q, k, v, 0.9, causal)
    ob, lb = oracle.attention_bruteforce(q.tolist(), k.tolist(), v.tolist(), 0.9, causal)
    np.testing.assert_allclose(o, np.array(ob), rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, np.array(lb), rtol=0, atol=1e-14)


# ------------------------------------------------ online recurrence pins

@pytest.mark.parametrize("block", [1, 7, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("threshold", [0.0, 8.0 * math.log(2.0)])
def test_online_softmax_equals_two_pass(block, causal, threshold):
    n, d = 300, 16
    q, k, v = rand(n, d, scale=2.0), rand(n, d), rand(n, d)
    o1, l1 = oracle.attention_head(q, k, v, 0.5, causal)
    o2, l2 = oracle.online_softmax_attention_head(q, k, v, 0.5, causal, block, threshold)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l2, l1, rtol=0, atol=1e-12)


def test_row_chunking_is_invisible():
    q, k, v = rand(100, 8), rand(100, 8), rand(100, 8)
    o1, l1 = oracle.attention_head(q, k, v, 0.5, True, row_chunk=100)
    o2, l2 = oracle.attention_head(q, k, v, 0.5, True, row_chunk=7)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-14)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-14)


def test_sampled_rows_match_full():
    q = torch.randn(1, 2, 200, 8)
    k = torch.randn(1, 2, 200, 8)
    v = torch.randn(1, 2, 200, 8)
    o, lse = oracle.attention_forward(q, k, v, 0.3, True)
    rows = [0, 1, 127, 128, 199]
    o_r, l_r = oracle.attention_forward_rows(q, k, v, 0.3, True, 0, 1, rows)
    np.testing.assert_allclose(o_r, o[0, 1, rows], rtol=0, atol=1e-14)
    np.testing.assert_allclose(l_r, lse[0, 1, rows], rtol=0, atol=1e-14)


# ------------------------------------------------------------ GQA pins

def test_gqa_equals_repeated_kv_heads():
    """hysenlabs.com, 'Die Schnittstellen...': fewer KV heads than Q heads, contiguous groups."""
    B, Hq, Hkv, N, d = 2, 6, 2, 20, 8
    q = torch.randn(B, Hq, N, d, dtype=torch.float64)
    k = torch.randn(B, Hkv, N, d, dtype=torch.float64)
    v = torch.randn(B, Hkv, N, d, dtype=torch.float64)
    o, lse = oracle.attention_forward(q, k, v, 0.35, True)
    k_rep = k.repeat_interleave(Hq // Hkv, dim=1)
    v_rep = v.repeat_interleave(Hq // Hkv, dim=1)
    o2, lse2 = oracle.attention_forward(q, k_rep, v_rep, 0.35, True)
    np.testing.assert_allclose(o, o2, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, lse2, rtol=0, atol=1e-14)
    with pytest.raises(ValueError):
        oracle.attention_forward(q, k[:, :1].repeat(1, 4, 1, 1), v[:, :1].repeat(1, 4, 1, 1), 1.0, False)


# -------------------------------------- independent library: torch float64

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("hq,hkv", [(2, 2), (4, 1), (6, 3)])
def test_forward_matches_torch_float64_sdpa(causal, hq, hkv):
    B, N, d = 2, 33, 16
    q = torch.randn(B, hq, N, d, dtype=torch.float64)
    k = torch.randn(B, hkv, N, d, dtype=torch.float64)
    v = torch.randn(B, hkv, N, d, dtype=torch.float64)
    scale = 1.0 / math.sqrt(d)
    expect = torch.nn.functional.scaled_dot_product_attention(
        q, k, v, is_causal=causal, scale=scale, enable_gqa=True)
    o, lse = oracle.attention_forward(q, k, v, scale, causal)
    np.testing.assert_allclose(o, expect.numpy(), rtol=0, atol=1e-13)
    s = torch.einsum("bhnd,bhmd->bhnm", q, k.repeat_interleave(hq // hkv, 1)) * scale
    if causal:
        s = s.masked_fill(~torch.ones(N, N, dtype=torch.bool).tril(), -math.inf)
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("hq,hkv", [(2, 2), (4, 2)])
def test_backward_matches_torch_autograd(causal, hq, hkv):
    B, N, d = 1, 29, 8
    q = torch.randn(B, hq, N, d, dtype=torch.float64, requires_grad=True)
    k = torch.randn(B, hkv, N, d, dtype=torch.float64, requires_grad=True)
    v = torch.randn(B, hkv, N, d, dtype=torch.float64, requires_grad=True)
    do = torch.randn(B, hq, N, d, dtype=torch.float64)
    scale = 0.4
    out = torch.nn.functional.scaled_dot_product_attention(
        q, k, v, is_causal=causal, scale=scale, enable_gqa=True)
    out.backward(do)
    dq, dk, dv = oracle.attention_backward(q.detach(), k.detach(), v.detach(), do, scale, causal)
    np.testing.assert_allclose(dq, q.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk, k.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv, v.grad.numpy(), rtol=0, atol=1e-12)


# ------------------------------------------------- finite differences

def _loss(q, k, v, do, scale, causal):
    o, _ = oracle.attention_forward(q, k, v, scale, causal)
    return float(np.sum(o * do))


@pytest.mark.parametrize("causal", [False, True])
def test_gradients_by_central_differences(causal):
    """B=1, Hq=2, Hkv=1, N=5, d=3: also pins the GQA gradient sum over the group."""
    B, Hq, Hkv, N, d = 1, 2, 1, 5, 3
    q, k, v = rand(B, Hq, N, d), rand(B, Hkv, N, d), rand(B, Hkv, N, d)
    do = rand(B, Hq, N, d)
    scale = 0.8
    dq, dk, dv = oracle.attention_backward(q, k, v, do, scale, causal)
    eps = 1e-5
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            fp = _loss(args["q"], args["k"], args["v"], do, scale, causal)
            args[name] = xm
            fm = _loss(args["q"], args["k"], args["v"], do, scale, causal)
            num[idx] = (fp - fm) / (2 * eps)
        rel = np.max(np.abs(num - g)) / max(1e-30, np.max(np.abs(g)))
        assert rel <= 1e-6, (name, rel)


# ---------------------------------------------------------------- mutants
# Plausible mistakes, planted in copies of the oracle's formulas, each of which
# a pin above must catch. The planted copies live only here; the oracle is untouched.

def _head_mutant(kind):
    def f(q, k, v, scale, causal):
        if kind == "no_scale":
            s = q @ k.T
        elif kind == "transposed_scores":
            s = (k @ q.T) * scale
        else:
            s = (q @ k.T) * scale
        if causal:
            i = np.arange(q.shape[0])[:, None]
            j = np.arange(k.shape[0])[None, :]
            keep = (j < i) | (i == 0) if kind == "strict_mask" else (j <= i)
            if kind == "mask_transposed":
                keep = j >= i
            s = np.where(keep, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        if kind == "no_normalise":
            return e @ v
        p = e / e.sum(axis=1, keepdims=True)
        if kind == "v_transposed":
            return p @ v.T[: p.shape[1]].T if v.shape[0] == v.shape[1] else p @ v[::-1]
        return p @ v
    return f


@pytest.mark.parametrize("kind", ["no_scale", "transposed_scores", "strict_mask",
                                  "mask_transposed", "no_normalise", "v_transposed"])
def test_forward_mutants_are_caught_by_brute_force(kind):
    q, k, v = rand(4, 3), rand(4, 3), rand(4, 3)
    ob, _ = oracle.attention_bruteforce(q.tolist(), k.tolist(), v.tolist(), 0.7, True)
    bad = _head_mutant(kind)(q, k, v, 0.7, True)
    assert np.max(np.abs(bad - np.array(ob))) > 1e-6


def test_backward_mutant_without_row_dot_is_caught():
    """Dropping the rowsum(P*dP) term of dS must break the finite-difference pin."""
    q, k, v, do = rand(5, 3), rand(5, 3), rand(5, 3), rand(5, 3)
    s = oracle.scores(q, k, 0.8, False)
    p, _, _ = oracle.softmax_rows(s)
    dq_bad = 0.8 * ((p * (do @ v.T)) @ k)
    dq, _, _ = ref.attention_head_bwd(q, k, v, do, 0.8, False)
    assert np.max(np.abs(dq_bad - dq)) > 1e-3


# ------------------------------------------- sliding window and Nq != Nk
# hysenlabs.com, 'Von 2.0 bis 2.7': sliding-window attention (2.3) and the
# bottom-right causal alignment for Nq != Nk (2.1).

def test_window_reduces_to_known_masks():
    n = 50
    q, k, v = rand(n, 8), rand(n, 8), rand(n, 8)
    full = oracle.attention_head(q, k, v, 0.5, False)
    causal = oracle.attention_head(q, k, v, 0.5, True)
    wide = oracle.attention_head(q, k, v, 0.5, False, window=(n, n))
    left_only = oracle.attention_head(q, k, v, 0.5, False, window=(n, 0))
    for a, b in ((full, wide), (causal, left_only)):
        np.testing.assert_allclose(a[0], b[0], rtol=0, atol=1e-14)
        np.testing.assert_allclose(a[1], b[1], rtol=0, atol=1e-14)


def test_window_zero_is_identity_on_v():
    """window (0, 0) with Nq == Nk: each query sees only its own key, so O = V."""
    n = 20
    q, k, v = rand(n, 4), rand(n, 4), rand(n, 3)
    o, lse = oracle.attention_head(q, k, v, 0.7, False, window=(0, 0))
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, 0.7 * np.sum(q * k, axis=1), rtol=0, atol=1e-14)


def test_visible_counts_closed_form():
    """With Nq == Nk == n, window (l, r): row i sees min(i, l) + 1 + min(n-1-i, r) keys."""
    n, l, r = 30, 5, 3
    vis = oracle.visible(np.arange(n), n, n, False, (l, r))
    expect = [min(i, l) + 1 + min(n - 1 - i, r) for i in range(n)]
    assert vis.sum(axis=1).tolist() == expect


@pytest.mark.parametrize("window", [(2, 1), (0, 3), (3, -1), (-1, 2)])
@pytest.mark.parametrize("nq,nk,causal", [(5, 5, False), (4, 6, True), (6, 4, True), (3, 7, False)])
def test_window_bruteforce(window, nq, nk, causal):
    q, k, v = rand(nq, 3), rand(nk, 3), rand(nk, 2)
    o, lse = oracle.attention_head(q, k, v, 0.9, causal, window=window)
    ob, lb = oracle.attention_bruteforce(q.tolist(), k.tolist(), v.tolist(), 0.9, causal, window)
    np.testing.assert_allclose(o, np.array(ob), rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, np.array(lb), rtol=0, atol=1e-14)


@pytest.mark.parametrize("nq,nk,causal,window", [(40, 70, True, (-1, -1)), (70, 40, True, (-1, -1)),
                                                 (50, 50, False, (7, 3)), (33, 61, True, (9, -1))])
def test_masked_forward_and_backward_match_torch(nq, nk, causal, window):
    """Library routine: torch float64 SDPA with the explicit boolean mask, and its autograd."""
    q = torch.randn(1, 2, nq, 8, dtype=torch.float64, requires_grad=True)
    k = torch.randn(1, 2, nk, 8, dtype=torch.float64, requires_grad=True)
    v = torch.randn(1, 2, nk, 8, dtype=torch.float64, requires_grad=True)
    do = torch.randn(1, 2, nq, 8, dtype=torch.float64)
    mask = torch.from_numpy(oracle.visible(np.arange(nq), nq, nk, causal, window))
    rows_ok = mask.any(dim=1)
    out = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=0.3)
    out = torch.where(rows_ok[None, None, :, None], out, torch.zeros_like(out))
    (out * do).sum().backward()
    o, lse = oracle.attention_forward(q.detach(), k.detach(), v.detach(), 0.3, causal, window=window)
    np.testing.assert_allclose(o, out.detach().numpy(), rtol=0, atol=1e-12)
    assert np.all(np.isneginf(lse[..., ~rows_ok.numpy()]))
    dq, dk, dv = oracle.attention_backward(q.detach(), k.detach(), v.detach(), do, 0.3, causal,
                                           window=window)
    np.testing.assert_allclose(dq, q.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk, k.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv, v.grad.numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("window", [(0, 0), (4, 2), (10, -1)])
def test_online_softmax_with_window(window):
    q, k, v = rand(60, 8), rand(60, 8), rand(60, 8)
    o1, l1 = oracle.attention_head(q, k, v, 0.5, False, window=window)
    o2, l2 = oracle.online_softmax_attention_head(q, k, v, 0.5, False, 16, 8 * math.log(2), window)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l2, l1, rtol=0, atol=1e-12)
