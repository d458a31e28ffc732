"""Shared helpers for the GPU parity tests: run the CUDA path through the
binding, run the oracle on the same bf16 inputs, and report errors with the
location of the worst element so a breach can be diagnosed."""
from __future__ import annotations

import numpy as np
import torch

import exact_attention_105_b200 as ea
import oracle

# Tolerances fixed before measuring (forward: absolute on O and lse;
# backward: absolute, relative to the largest reference magnitude).
O_TOL = 1e-2
LSE_TOL = 1e-3
GRAD_REL_TOL = 2e-2


def to_dev(*ts):
    return [t.to("cuda", non_blocking=False).contiguous() for t in ts]


def gpu_fwd(q, k, v, scale, causal):
    """Forward through the binding into outputs pre-filled with NaN, so a
    finiteness check over the whole output shows every element was written."""
    qd, kd, vd = to_dev(q, k, v)
    o = torch.full_like(qd, float("nan"))
    lse = torch.full(qd.shape[:3], float("nan"), dtype=torch.float32, device=qd.device)
    ea.attn_fwd(qd, kd, vd, o, lse, scale=scale, causal=causal)
    ea.attn_check_status()
    return o, lse


def max_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    diff = np.abs(got - ref)
    if diff.size == 0:
        return 0.0, None
    idx = np.unravel_index(int(np.argmax(diff)), diff.shape)
    return float(diff[idx]), idx


def assert_fwd_close(o_gpu, lse_gpu, o_ref, lse_ref, label=""):
    o_np = o_gpu.float().cpu().numpy() if hasattr(o_gpu, "cpu") else o_gpu
    l_np = lse_gpu.float().cpu().numpy() if hasattr(lse_gpu, "cpu") else lse_gpu
    assert np.all(np.isfinite(o_np)), f"{label}: non-finite O"
    assert np.all(np.isfinite(l_np)), f"{label}: non-finite lse"
    eo, io = max_err(o_np, o_ref)
    el, il = max_err(l_np, lse_ref)
    assert eo <= O_TOL, f"{label}: max|O-O_ref| = {eo:.3e} at {io} (ref {o_ref[io]:.4f}, max|O_ref| {np.abs(o_ref).max():.3f})"
    assert el <= LSE_TOL, f"{label}: max|lse-lse_ref| = {el:.3e} at {il}"
    return eo, el


def naive_bf16_attention(q, k, v, scale, causal):
    """Materialised attention in bf16 torch ops on the GPU: the 'baseline
    implementation' of the upstream test methodology (hysenlabs.com, section
    'Tests, BSD-3-Clause und Zitierpraxis'). It is used only to bound the
    kernel's error at two times the baseline's, never as the reference."""
    qd, kd, vd = to_dev(q, k, v)
    G = qd.shape[1] // kd.shape[1]
    kd = kd.repeat_interleave(G, dim=1)
    vd = vd.repeat_interleave(G, dim=1)
    s = torch.matmul(qd, kd.transpose(-1, -2)) * scale
    if causal:
        n = s.shape[-1]
        s = s.masked_fill(torch.ones(n, n, dtype=torch.bool, device=s.device).triu(1), float("-inf"))
    p = torch.softmax(s, dim=-1).to(torch.bfloat16)
    return torch.matmul(p, vd)


def sample_rows(N, rng, extra=24):
    """Tile edges, the ragged tail and random rows of a length-N sequence."""
    rows = {0, 1, 2, N - 1, N - 2}
    for edge in range(128, N, 128):
        rows.update({edge - 1, edge})
    rows = sorted(r for r in rows if 0 <= r < N)
    if len(rows) > 48:
        keep = rng.choice(len(rows), 48, replace=False)
        rows = sorted(rows[i] for i in keep) + [0, N - 1]
    rows += list(rng.integers(0, N, size=extra))
    return np.array(sorted(set(int(r) for r in rows)))


# Relative error of one bf16 round-to-nearest: the unit roundoff 2^-p of a
# p = 8 bit significand (7 stored bits and the implicit one). It is reached
# just above a power of two: 2.0078 rounds to 2.0, an error of 2^-8 * 2.0078.
BF16_HALF_ULP_REL = 2.0 ** -8
# Slack for the kernel's fp32 arithmetic around P: ex2.approx and the softcap's
# rcp.approx (relative errors near 2^-22), the fp32 tensor-core accumulation,
# and the fp32 row sums. Far above their sum at these sizes, far below 2^-8.
FP32_PATH_REL = 2e-4


def p_rounding_bound(q, k, v, scale, causal, window=(-1, -1), softcap=0.0):
    """Element-wise error bound for O when P is rounded to bf16 before the PV
    product and the output is rounded to bf16 once.

    Derivation (own, from the arithmetic; the pages give the definition only).
    Let w_j be the exact softmax weights of a row and O = sum_j w_j v_j. The
    kernel multiplies V by p_j (1 + d_j), |d_j| <= u with u = 2^-8 + fp32
    slack, and divides by the sum of the same rounded p_j. Then
        O_kernel - O = sum_j w_j d_j (v_j - O) / (1 + sum_j w_j d_j),
    so |O_kernel - O| <= u / (1 - u) * sum_j w_j |v_j - O| per output column.
    Rounding the fp32 result to bf16 adds at most 2^-8 |O_kernel|. Returns the
    bound with the float64 oracle's weights, shaped like O [B, Hq, Nq, d]."""
    q64, k64, v64 = (oracle.to_f64(t) for t in (q, k, v))
    B, Hq, Nq, d = q64.shape
    G = Hq // k64.shape[1]
    u = BF16_HALF_ULP_REL + FP32_PATH_REL
    out = np.empty((B, Hq, Nq, d))
    for b in range(B):
        for h in range(Hq):
            kk, vv = k64[b, h // G], v64[b, h // G]
            s = oracle.scores(q64[b, h], kk, scale, causal, window=window, softcap=softcap)
            w, _, _ = oracle.softmax_rows(s)
            o = w @ vv
            spread = np.einsum("ij,ijc->ic", w, np.abs(vv[None, :, :] - o[:, None, :]))
            out[b, h] = u / (1.0 - u) * spread + BF16_HALF_ULP_REL * (np.abs(o) + u * spread)
    return out
