"""Float64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY. Only the test suite, the package smoke check and the
benchmark's CPU-baseline leg may import this module. The CUDA library never
calls it, and it imports nothing from the CUDA side.

What it computes is the plain definition the FlashAttention pages state,
written out directly and slowly so it can be checked by eye:

* hysenlabs.com, "FlashAttention: exakte Attention-Kernel fuer CUDA und ROCm",
  section "Die Schnittstellen von flash_attn_func bis KV-Cache": every entry
  point computes ``softmax(Q @ K^T * softmax_scale) @ V``. The same section
  lets K/V have fewer heads than Q when the Q head count divides evenly
  (MQA/GQA). Grouping is contiguous: query head ``h`` reads KV head
  ``h // (Hq // Hkv)``.
* Same page, section "Von 2.0 bis 2.7": the causal mask is aligned to the
  bottom-right corner when the query and key lengths differ. Query ``i`` may
  see key ``j`` iff ``j <= i + (Nk - Nq)``. With ``Nq == Nk`` this is ``j <= i``.
  Release 2.3 there adds sliding-window attention, and the interface section
  lists a ``window_size`` parameter. Read plainly, with the same bottom-right
  alignment: ``window = (left, right)`` keeps key ``j`` for query ``i`` iff
  ``i + off - left <= j <= i + off + right`` with ``off = Nk - Nq``. A negative
  side means unbounded. Causal is the case ``right = 0``.
  Release 2.6 there adds softcapping "as used in Gemma-2 and Grok" without a
  formula. Read plainly (the form those models use): with ``softcap = c > 0``
  each scaled logit ``z = scale * q . k`` becomes ``c * tanh(z / c)`` before
  masking and the softmax; ``c = 0`` turns it off. lse is then the
  logsumexp of the capped logits.
* Release 2.0 there renames the unpadded functions to "varlen". Read plainly:
  a batch of sequences of different lengths is packed token by token with no
  padding, Q as ``[total_q, Hq, d]`` and K/V as ``[total_k, Hkv, d]``, and
  ``cu_seqlens_q/k`` (length B+1, starting at 0) give each sequence's first
  row. Sequence b attends only within itself, with its own ``Nq_b`` and
  ``Nk_b`` (bottom-right causal alignment and window per sequence). lse is
  ``[Hq, total_q]``.
* tokenwerk.de "FlashAttention", section "Was FlashAttention veraendert", and
  unite.ai "Was ist FlashAttention?", the worked example: the method is exact,
  not an approximation. So the oracle is the definition itself. S and P are
  materialised in full, the softmax is the textbook two-pass one, and there
  is no blocking or online recurrence. The one exception is
  ``online_softmax_attention_head``, which restates the tiled algorithm
  separately so that tests can pin it against the definition.

Readings where the pages are silent (each is listed in the design notes):

* The pages never define the logsumexp output. Here
  ``lse_i = ln sum_j exp(scale * q_i . k_j)`` over the unmasked keys, in
  natural log, of the *scaled* logits.
* A row with no visible key has ``O = 0`` and ``lse = -inf``.
* The pages do not write out the backward pass. The oracle uses the exact
  gradient of the definition. ``dV = P^T dO``, ``dP = dO V^T`` and
  ``dS = P * (dP - rowsum(P * dP))``. Then ``dQ = scale * dS K`` and
  ``dK = scale * dS^T Q``. Under GQA, dK and dV of a KV head are summed over
  the query heads that read it. With softcapping the chain rule adds the
  factor ``d(c tanh(z/c))/dz = 1 - tanh(z/c)^2`` to dS.

Inputs may be torch tensors (any dtype, e.g. bfloat16) or numpy arrays. They
are upcast to float64 once, so the oracle sees the same rounded values the
GPU sees.
"""
from __future__ import annotations

import math

import numpy as np

ROW_CHUNK = 2048  # query rows per materialised block of S (bounds memory at N=16384)


def to_f64(x) -> np.ndarray:
    """Upcast a torch tensor or array-like to a float64 numpy array."""
    if hasattr(x, "detach"):
        import torch  # local: the oracle itself only needs numpy
        return x.detach().to(device="cpu", dtype=torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


# --------------------------------------------------------------------------
# Sizing of the dense per-head score matrix that the tiled method avoids.
# tokenwerk.de "FlashAttention", section "Warum Kacheln beim Speicherzugriff
# helfen", table of matrix and tile sizes (two bytes per cell).
# --------------------------------------------------------------------------

def dense_score_matrix_cells(n_q: int, n_k: int | None = None) -> int:
    """Cells of one head's full score matrix: Nq * Nk."""
    return n_q * (n_q if n_k is None else n_k)


def dense_score_matrix_bytes(n_q: int, n_k: int | None = None, bytes_per_cell: int = 2) -> int:
    """Bytes of one head's full score matrix at ``bytes_per_cell`` per entry."""
    return dense_score_matrix_cells(n_q, n_k) * bytes_per_cell


# --------------------------------------------------------------------------
# The definition, one head at a time.
# --------------------------------------------------------------------------

def causal_visible(n_q: int, n_k: int) -> np.ndarray:
    """Boolean [Nq, Nk]: True where query i may attend to key j (bottom-right)."""
    i = np.arange(n_q)[:, None]
    j = np.arange(n_k)[None, :]
    return j <= i + (n_k - n_q)


def visible(rows, n_q_total: int, n_k: int, causal: bool, window=(-1, -1)) -> np.ndarray:
    """Boolean [len(rows), Nk]: query row i (of n_q_total) may see key j.

    Bottom-right alignment with off = Nk - Nq: causal keeps j <= i + off, and
    window (left, right) keeps i + off - left <= j <= i + off + right. A
    negative window side is unbounded.
    """
    i = np.asarray(rows)[:, None]
    j = np.arange(n_k)[None, :]
    off = n_k - n_q_total
    keep = np.ones((i.shape[0], n_k), dtype=bool)
    left, right = window
    if causal:
        keep &= j <= i + off
    if right >= 0:
        keep &= j <= i + off + right
    if left >= 0:
        keep &= j >= i + off - left
    return keep


def capped(z: np.ndarray, softcap: float) -> np.ndarray:
    """Softcapping of scaled logits: c * tanh(z / c) for c > 0, identity for c = 0."""
    if softcap < 0:
        raise ValueError("softcap must be >= 0")
    return softcap * np.tanh(z / softcap) if softcap > 0 else z


def scores(q: np.ndarray, k: np.ndarray, scale: float, causal: bool,
           row_offset: int = 0, n_q_total: int | None = None, window=(-1, -1),
           softcap: float = 0.0) -> np.ndarray:
    """S = (Q K^T) * scale (softcapped when softcap > 0), masked entries -inf.

    ``q`` holds query rows ``row_offset .. row_offset + len(q)`` of a sequence
    of ``n_q_total`` queries (default: just these rows). That is how the
    row-chunked and row-sampled callers keep the causal/window mask right.
    """
    s = capped((q @ k.T) * scale, softcap)
    if causal or window[0] >= 0 or window[1] >= 0:
        n_q_total = q.shape[0] if n_q_total is None else n_q_total
        rows = np.arange(row_offset, row_offset + q.shape[0])
        s = np.where(visible(rows, n_q_total, k.shape[0], causal, window), s, -np.inf)
    return s


def softmax_rows(s: np.ndarray):
    """Two-pass softmax of each row of S: returns (P, row max m, row sum l).

    Fully masked rows (all -inf) give P = 0, m = -inf, l = 0.
    """
    m = np.max(s, axis=1)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(s - m_safe[:, None])          # exp(-inf) = 0 for masked entries
    l = np.sum(e, axis=1)
    l_safe = np.where(l > 0, l, 1.0)
    p = e / l_safe[:, None]
    return p, m, l


def attention_head(q, k, v, scale: float, causal: bool, row_chunk: int = ROW_CHUNK,
                   window=(-1, -1), softcap: float = 0.0):
    """O and lse for one (query head, KV head) pair; q [Nq,d], k/v [Nk,d] float64."""
    n_q = q.shape[0]
    o = np.empty((n_q, v.shape[1]), dtype=np.float64)
    lse = np.empty(n_q, dtype=np.float64)
    for r0 in range(0, n_q, row_chunk):
        r1 = min(n_q, r0 + row_chunk)
        s = scores(q[r0:r1], k, scale, causal, row_offset=r0, n_q_total=n_q, window=window,
                   softcap=softcap)
        p, m, l = softmax_rows(s)
        o[r0:r1] = p @ v
        with np.errstate(divide="ignore"):
            lse[r0:r1] = np.where(l > 0, m + np.log(np.where(l > 0, l, 1.0)), -np.inf)
    return o, lse


def attention_head_rows(q_rows, k, v, scale: float, causal: bool, rows, n_q_total: int,
                        window=(-1, -1), softcap: float = 0.0):
    """O and lse for selected query rows (indices ``rows`` of ``n_q_total``)."""
    rows = np.asarray(rows)
    s = capped((q_rows @ k.T) * scale, softcap)
    if causal or window[0] >= 0 or window[1] >= 0:
        s = np.where(visible(rows, n_q_total, k.shape[0], causal, window), s, -np.inf)
    p, m, l = softmax_rows(s)
    with np.errstate(divide="ignore"):
        lse = np.where(l > 0, m + np.log(np.where(l > 0, l, 1.0)), -np.inf)
    return p @ v, lse


def attention_head_bwd(q, k, v, do, scale: float, causal: bool, window=(-1, -1),
                       softcap: float = 0.0):
    """dQ, dK, dV for one head pair, from explicit S and P (no recompute trick)."""
    s = scores(q, k, scale, causal, window=window, softcap=softcap)
    p, _, _ = softmax_rows(s)
    dv = p.T @ do
    dp = do @ v.T
    row_dot = np.sum(p * dp, axis=1, keepdims=True)
    ds = p * (dp - row_dot)                      # gradient with respect to the (capped) logits
    if softcap > 0:
        t = np.tanh((q @ k.T) * scale / softcap)
        ds = ds * (1.0 - t * t)                  # chain rule through c * tanh(z / c)
    dq = scale * (ds @ k)
    dk = scale * (ds.T @ q)
    return dq, dk, dv


# --------------------------------------------------------------------------
# Batched entry points over [B, H, N, d].
# --------------------------------------------------------------------------

def _kv_head(hq: int, n_q_heads: int, n_kv_heads: int) -> int:
    if n_q_heads % n_kv_heads != 0:
        raise ValueError("query head count must be divisible by the KV head count")
    return hq // (n_q_heads // n_kv_heads)


def attention_forward(q, k, v, scale: float, causal: bool, window=(-1, -1),
                      softcap: float = 0.0):
    """O [B,Hq,Nq,d] and lse [B,Hq,Nq] in float64 (K/V may have Nk != Nq rows)."""
    q, k, v = to_f64(q), to_f64(k), to_f64(v)
    B, Hq, Nq, _ = q.shape
    Hkv = k.shape[1]
    o = np.empty((B, Hq, Nq, v.shape[3]), dtype=np.float64)
    lse = np.empty((B, Hq, Nq), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            hk = _kv_head(h, Hq, Hkv)
            o[b, h], lse[b, h] = attention_head(q[b, h], k[b, hk], v[b, hk], scale, causal,
                                                window=window, softcap=softcap)
    return o, lse


def attention_forward_rows(q, k, v, scale: float, causal: bool, b: int, hq: int, rows,
                           window=(-1, -1), softcap: float = 0.0):
    """O and lse of the listed query rows of head (b, hq), for full-size spot checks."""
    Hq, Nq = q.shape[1], q.shape[2]
    hk = _kv_head(hq, Hq, k.shape[1])
    rows = np.asarray(rows)
    q_rows = to_f64(q[b, hq][rows])
    return attention_head_rows(q_rows, to_f64(k[b, hk]), to_f64(v[b, hk]), scale, causal,
                               rows, Nq, window=window, softcap=softcap)


def attention_backward(q, k, v, do, scale: float, causal: bool, heads=None, window=(-1, -1),
                       softcap: float = 0.0):
    """dQ [B,Hq,N,d], dK and dV [B,Hkv,N,d] in float64.

    ``heads``: optional list of (b, hkv) KV heads to compute (the others are
    left as NaN). All query heads of each listed group are included, which is
    what a sampled full-size check needs.
    """
    q, k, v, do = to_f64(q), to_f64(k), to_f64(v), to_f64(do)
    B, Hq = q.shape[:2]
    Hkv = k.shape[1]
    G = Hq // Hkv
    if Hq % Hkv != 0:
        raise ValueError("query head count must be divisible by the KV head count")
    dq = np.full(q.shape, np.nan)
    dk = np.full(k.shape, np.nan)
    dv = np.full(v.shape, np.nan)
    todo = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hkv)]
    for b, hk in todo:
        dk[b, hk] = 0.0
        dv[b, hk] = 0.0
        for h in range(hk * G, (hk + 1) * G):
            gq, gk, gv = attention_head_bwd(q[b, h], k[b, hk], v[b, hk], do[b, h], scale, causal,
                                            window=window, softcap=softcap)
            dq[b, h] = gq
            dk[b, hk] += gk
            dv[b, hk] += gv
    return dq, dk, dv


def attention_backward_dq_rows(q, k, v, do, scale: float, causal: bool, b: int, hq: int, rows,
                               window=(-1, -1), softcap: float = 0.0):
    """dQ of the listed query rows of head (b, hq), for full-size spot checks.

    Every quantity dQ needs is local to the row: its scores over all keys,
    P from their softmax, dP = dO_row V^T, D = sum(P * dP), dS = P * (dP - D)
    (times 1 - tanh^2 with softcapping) and dQ = scale * dS K.
    """
    Hq, Nq = q.shape[1], q.shape[2]
    hk = _kv_head(hq, Hq, k.shape[1])
    rows = np.asarray(rows)
    qr = to_f64(q[b, hq][rows])
    kk, vv = to_f64(k[b, hk]), to_f64(v[b, hk])
    dor = to_f64(do[b, hq][rows])
    z = (qr @ kk.T) * scale
    s = capped(z, softcap)
    if causal or window[0] >= 0 or window[1] >= 0:
        s = np.where(visible(rows, Nq, kk.shape[0], causal, window), s, -np.inf)
    p, _, _ = softmax_rows(s)
    dp = dor @ vv.T
    ds = p * (dp - np.sum(p * dp, axis=1, keepdims=True))
    if softcap > 0:
        t = np.tanh(z / softcap)
        ds = ds * (1.0 - t * t)
    return scale * (ds @ kk)


# --------------------------------------------------------------------------
# The tiled algorithm, restated separately so tests can pin it to the
# definition. unite.ai "Was ist FlashAttention?", section "Eine fuenfstufige
# Betriebsuebersicht": stage 1 partitions Q, K and V into tiles, stage 3
# computes local scores with a running normalisation, and stage 4 accumulates
# outputs without materialising the full matrix. The running normalisation
# is named there but not written out. It is read here as the usual running
# max/sum rescaling.
# --------------------------------------------------------------------------

def online_softmax_attention_head(q, k, v, scale: float, causal: bool, block: int,
                                  rescale_threshold: float = 0.0, window=(-1, -1)):
    """One head, keys visited in blocks of ``block`` with a running max and sum.

    ``rescale_threshold`` (natural-log units) lets the running max lag the
    true max by up to that much before the accumulator is rescaled. The
    result is the same in exact arithmetic, because the final division uses
    the same stale max. The GPU kernel uses the same lazy update with its
    own threshold, and the tests pin this variant too.
    """
    n_q, n_k = q.shape[0], k.shape[0]
    m = np.full(n_q, -np.inf)
    l = np.zeros(n_q)
    acc = np.zeros((n_q, v.shape[1]))
    vis = visible(np.arange(n_q), n_q, n_k, causal, window)
    for c0 in range(0, n_k, block):
        c1 = min(n_k, c0 + block)
        s = (q @ k[c0:c1].T) * scale
        s = np.where(vis[:, c0:c1], s, -np.inf)
        m_blk = np.max(s, axis=1)
        m_new = np.maximum(m, m_blk)
        move = m_new > m + rescale_threshold
        m_use = np.where(move, m_new, m)
        with np.errstate(invalid="ignore"):
            alpha = np.where(np.isfinite(m), np.exp(m - m_use), 0.0)
        m_use_safe = np.where(np.isfinite(m_use), m_use, 0.0)
        p = np.exp(s - m_use_safe[:, None])
        p = np.where(np.isfinite(s), p, 0.0)
        l = l * alpha + p.sum(axis=1)
        acc = acc * alpha[:, None] + p @ v[c0:c1]
        m = m_use
    l_safe = np.where(l > 0, l, 1.0)
    o = acc / l_safe[:, None]
    with np.errstate(divide="ignore"):
        lse = np.where(l > 0, m + np.log(l_safe), -np.inf)
    return o, lse


# --------------------------------------------------------------------------
# Brute force for tiny inputs: scalar loops and math.exp, nothing vectorised.
# --------------------------------------------------------------------------

def attention_bruteforce(q, k, v, scale: float, causal: bool, window=(-1, -1),
                         softcap: float = 0.0):
    """Pure-Python O and lse for one head; q [Nq][d], k/v [Nk][d] nested lists."""
    n_q, n_k, d_v = len(q), len(k), len(v[0])
    out, lses = [], []
    for i in range(n_q):
        logits = []
        for j in range(n_k):
            if causal and j > i + (n_k - n_q):
                continue
            if window[1] >= 0 and j > i + (n_k - n_q) + window[1]:
                continue
            if window[0] >= 0 and j < i + (n_k - n_q) - window[0]:
                continue
            dot = 0.0
            for c in range(len(q[i])):
                dot += q[i][c] * k[j][c]
            z = dot * scale
            if softcap > 0:
                z = softcap * math.tanh(z / softcap)
            logits.append((j, z))
        if not logits:
            out.append([0.0] * d_v)
            lses.append(-math.inf)
            continue
        big = max(x for _, x in logits)
        weights = [(j, math.exp(x - big)) for j, x in logits]
        total = sum(w for _, w in weights)
        row = [0.0] * d_v
        for j, w in weights:
            for c in range(d_v):
                row[c] += (w / total) * v[j][c]
        out.append(row)
        lses.append(big + math.log(total))
    return out, lses


# --------------------------------------------------------------------------
# Varlen (unpadded) batches: sequences packed token by token.
# --------------------------------------------------------------------------

def _check_cu(cu, total: int, name: str):
    cu = [int(x) for x in np.asarray(cu).tolist()]
    if not cu or cu[0] != 0 or cu[-1] != total or any(b < a for a, b in zip(cu, cu[1:])):
        raise ValueError(f"{name} must start at 0, be non-decreasing and end at {total}")
    return cu


def attention_forward_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, scale: float, causal: bool,
                             window=(-1, -1), softcap: float = 0.0):
    """Packed batch: q [total_q, Hq, d], k/v [total_k, Hkv, d] -> O [total_q, Hq, d] and
    lse [Hq, total_q], float64. Sequence b is rows cu_q[b]:cu_q[b+1] of q and
    cu_k[b]:cu_k[b+1] of k/v, and attends only within itself."""
    q, k, v = to_f64(q), to_f64(k), to_f64(v)
    total_q, Hq, _ = q.shape
    total_k, Hkv, _ = k.shape
    cq = _check_cu(cu_seqlens_q, total_q, "cu_seqlens_q")
    ck = _check_cu(cu_seqlens_k, total_k, "cu_seqlens_k")
    if len(cq) != len(ck):
        raise ValueError("cu_seqlens_q and cu_seqlens_k describe different batch sizes")
    o = np.zeros((total_q, Hq, v.shape[2]))
    lse = np.full((Hq, total_q), -np.inf)
    for b in range(len(cq) - 1):
        q0, q1, k0, k1 = cq[b], cq[b + 1], ck[b], ck[b + 1]
        if q1 == q0:
            continue
        for h in range(Hq):
            hk = _kv_head(h, Hq, Hkv)
            if k1 == k0:                      # no keys: O = 0, lse = -inf (already set)
                continue
            o[q0:q1, h], lse[h, q0:q1] = attention_head(q[q0:q1, h], k[k0:k1, hk], v[k0:k1, hk],
                                                        scale, causal, window=window,
                                                        softcap=softcap)
    return o, lse


def attention_backward_varlen(q, k, v, do, cu_seqlens_q, cu_seqlens_k, scale: float,
                              causal: bool, window=(-1, -1), softcap: float = 0.0):
    """dQ [total_q, Hq, d], dK and dV [total_k, Hkv, d] of the packed batch, float64."""
    q, k, v, do = to_f64(q), to_f64(k), to_f64(v), to_f64(do)
    total_q, Hq, _ = q.shape
    total_k, Hkv, _ = k.shape
    cq = _check_cu(cu_seqlens_q, total_q, "cu_seqlens_q")
    ck = _check_cu(cu_seqlens_k, total_k, "cu_seqlens_k")
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    for b in range(len(cq) - 1):
        q0, q1, k0, k1 = cq[b], cq[b + 1], ck[b], ck[b + 1]
        if q1 == q0 or k1 == k0:
            continue
        for h in range(Hq):
            hk = _kv_head(h, Hq, Hkv)
            gq, gk, gv = attention_head_bwd(q[q0:q1, h], k[k0:k1, hk], v[k0:k1, hk],
                                            do[q0:q1, h], scale, causal, window=window,
                                            softcap=softcap)
            dq[q0:q1, h] = gq
            dk[k0:k1, hk] += gk
            dv[k0:k1, hk] += gv
    return dq, dk, dv
