"""CPU float64 oracle for scaled-dot-product attention, forward and backward.

TEST INFRASTRUCTURE ONLY.  This module is imported by ``tests/``, by
``__graft_entry__.smoke()`` and by the CPU-baseline leg of ``bench.py``; the
product path (the CUDA library and its Python binding) never imports, calls or
links it, and it imports nothing from the product.  It is deliberately plain
and slow: one explicit L x L score matrix per (batch, query head), an explicit
boolean mask matrix, an explicit softmax and explicit chain-rule gradients, all
in numpy float64.  No blocking, no online softmax, no fusion.

What it computes, and where each piece comes from:

* The attention definition softmax(Q K^T / sqrt(d_k)) V, its four steps
  (score, scale + softmax, weighted sum, output shaped like Q) -- codelab
  "jax-gpu-05-attention-gpu", section 1 ("Dikkat nasil calisir?") and the
  naive reference of section 4 ("Dikkat mekanizmasini sifirdan uygulama");
  Medium "Simplified Explanation of Attention ...", "Scaled Dot Product
  Operation" Steps 1-4.
* (B, T, N, H) layout of Q, K, V and the output -- codelab section 3.
* Causal masking (query i sees keys j <= i) -- codelab section 7 ("Nedensel
  maskeleme ekleme").
* Causal sliding window (Mistral, window 4096) -- HF transformers issue #30461
  "Slowdown in Training Speed Due to SDPA Mask Fix in Version 4.40.0".
  The pages never say whether the window bound is inclusive; this oracle takes
  the bound explicitly: key j is visible from query i iff
  i - window_left <= j <= i + window_right (a negative bound = unbounded).
* MHA / GQA / MQA: KV heads shared by contiguous groups of query heads,
  g = hq // (Hq / Hkv) -- codelab section 9 ("MHA, GQA ve MQA'yi
  karsilastirma").
* Additive attention biases: a full (dense) bias tensor and a T5-style
  relative-position bias looked up from a [num_buckets, H] table -- catie-aq/
  flashT5 README (the "Full attention biases" and "T5-like relative position
  encoding biases" implementations, and the 3 October 2024 "fa2-rpe" item).
  The bias is added after the 1/sqrt(d) scaling and is not itself scaled.
* T5 bucketing: the pages name the bias but print no formula.  The oracle
  uses the published T5 closed form (Raffel et al. 2020) in its log form,
  evaluated in float64 (see ``t5_relative_bucket``).
* Backward: the pages print no gradient formulas; the oracle applies the chain
  rule to the definition above (dP = dO V^T, dS = P * (dP - rowsum(P*dP)),
  dQ = scale dS K, dK = scale dS^T Q, dV = P^T dO, with dK / dV summed over
  the query heads that share a KV head).
* ALiBi: the flashT5 README names it among the supported positional
  schemes but prints no formula.  The oracle takes the linear bias of Press
  et al. 2022 ("Train Short, Test Long"), bias = -m_h |j - i| with one slope
  m_h per query head given by the caller; under a causal mask this is the
  paper's -m_h (i - j), and the absolute value extends it to keys after the
  query.
* A relative-position table (any per-head function of the distance j - i,
  given as a table [Lq + Lk - 1, Hq], entry j - i + Lq - 1): the general form
  of which T5 and ALiBi are special cases.
* FIRE: the flashT5 README names it among the positional schemes it plans
  to support, without a formula.  The oracle takes the bias of Li et al.
  (2023, "Functional Interpolation for Relative Positions Improves Long
  Context Transformers"): f(psi(i - j) / psi(max(T, i))) with
  psi(x) = log(c x + 1) and f a one-hidden-layer ReLU MLP from the scalar to
  one value per head.  Reading: the threshold T is at least the longest
  query position (T >= Lq - 1), so max(T, i) = T on every row and the bias
  is a function of the distance alone -- a relative-position table; keys
  after the query (bidirectional use) take the same function of |i - j|.
* Bias gradients: the scores are linear in the bias with coefficient 1, so
  the gradient of a dense bias is dS itself, summed over every index along
  which the bias is broadcast, and the gradient of a T5 table entry
  table[k, h] is the sum of dS over all (b, i, j) with bucket(j - i) = k in
  head h (chain rule through the table lookup).  The pages name a learnable
  relative-position bias for training (catie-aq/flashT5 README, "T5-like
  relative position encoding biases") but print no gradient.
* Cross-attention (a query sequence attending to a key/value sequence of
  another length, as in T5's encoder-decoder): the same definition with
  K, V of Lk rows.  The pages do not say how positions of the two
  sequences line up; the oracle counts both from 0, so masks and
  relative-position biases read the absolute indices i and j.  (T5's own
  cross-attention uses neither a causal mask nor a position bias.)
* Packed variable-length sequences (HF transformers issue #30461: the
  reporter's fine-tune packs its examples, ``packing=True``; catie-aq/flashT5
  README: dynamic batching to cut padding): the pages do not say how
  attention treats the boundaries of packed examples.  The oracle's reading:
  the sequences lie end to end on one axis, cut by cumulative lengths
  ``cu_seqlens``; a query attends only to keys of its own sequence; positions
  count from 0 at each sequence's first row, and the masks and relative-
  position biases use those local positions.  ``attention_forward_packed``
  and ``attention_backward_packed`` write this out over the whole packed
  axis with one explicit block-diagonal mask.
* LSE is the natural-log log-sum-exp of each score row (bias included); a row
  with no visible key has LSE = -inf, output 0 and zero gradients.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "t5_relative_bucket",
    "visibility_mask",
    "head_scores",
    "attention_forward",
    "attention_backward",
    "attention_probs",
    "dense_bias_gradient",
    "t5_table_gradient",
    "alibi_slope_gradient",
    "rel_table_gradient",
    "fire_table",
    "fire_gradients",
    "packed_positions",
    "packed_visibility_mask",
    "attention_forward_packed",
    "attention_backward_packed",
]


# --------------------------------------------------------------------------
# T5 relative-position bucketing (catie-aq/flashT5 README, "T5-like relative
# position encoding biases"; closed form of Raffel et al. 2020).
# --------------------------------------------------------------------------
def t5_relative_bucket(rel, num_buckets: int = 32, max_distance: int = 128,
                       bidirectional: bool = True) -> np.ndarray:
    """Bucket id of the signed distance ``rel = key_pos - query_pos``.

    Bidirectional: half the buckets hold keys after the query (rel > 0,
    ids offset by num_buckets/2), half the rest; within a half, distances
    below max_exact = half/2 get one bucket each, larger distances share
    logarithmically wider buckets up to max_distance, beyond which all
    distances fall in the last bucket of the half.

    Unidirectional (decoder): only keys at or before the query matter,
    n = max(-rel, 0), all num_buckets are used, max_exact = num_buckets/2.

    The log is evaluated in float64 and truncated toward zero.
    """
    rel = np.asarray(rel, dtype=np.int64)
    nb = int(num_buckets)
    if bidirectional:
        nb = nb // 2
        offset = np.where(rel > 0, nb, 0).astype(np.int64)
        n = np.abs(rel)
    else:
        offset = np.zeros_like(rel)
        n = np.maximum(-rel, 0)
    max_exact = nb // 2
    out = np.empty_like(rel)
    small = n < max_exact
    out[small] = n[small]
    big = ~small
    if np.any(big):
        nf = n[big].astype(np.float64)
        v = np.log(nf / max_exact) / math.log(max_distance / max_exact) * (nb - max_exact)
        large = max_exact + np.trunc(v).astype(np.int64)
        out[big] = np.minimum(large, nb - 1)
    return out + offset


# --------------------------------------------------------------------------
# Mask (codelab section 7; transformers issue #30461 sliding window).
# --------------------------------------------------------------------------
def visibility_mask(L: int, causal: bool, window_left: int = -1,
                    window_right: int = -1, Lk: int | None = None) -> np.ndarray:
    """Boolean [L, Lk] matrix, True where query i may attend to key j."""
    Lk = L if Lk is None else Lk
    i = np.arange(L)[:, None]
    j = np.arange(Lk)[None, :]
    m = np.ones((L, Lk), dtype=bool)
    if causal:
        m &= j <= i
    if window_left is not None and window_left >= 0:
        m &= j >= i - window_left
    if window_right is not None and window_right >= 0:
        m &= j <= i + window_right
    return m


def _as64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # a torch tensor
        x = x.detach().to("cpu")
        import torch  # local: only to read torch inputs
        x = x.to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def _bias_matrix(b: int, hq: int, L: int, bias, t5_table, t5_num_buckets,
                 t5_max_distance, t5_bidirectional, alibi_slopes=None, Lk=None,
                 rel_table=None):
    """Additive bias for one (batch, query head), [L, Lk] float64 (or 0)."""
    Lk = L if Lk is None else Lk
    out = 0.0
    if rel_table is not None:
        i = np.arange(L)[:, None]
        j = np.arange(Lk)[None, :]
        out = out + rel_table[j - i + L - 1, hq]
    if alibi_slopes is not None:
        i = np.arange(L)[:, None]
        j = np.arange(Lk)[None, :]
        out = out - alibi_slopes[hq] * np.abs(j - i)
    if bias is not None:
        # a bias row of extent 1 is broadcast over the query rows
        out = out + np.broadcast_to(
            bias[b if bias.shape[0] > 1 else 0, hq if bias.shape[1] > 1 else 0], (L, Lk))
    if t5_table is not None:
        i = np.arange(L)[:, None]
        j = np.arange(Lk)[None, :]
        bucket = t5_relative_bucket(j - i, t5_num_buckets, t5_max_distance, t5_bidirectional)
        out = out + t5_table[bucket, hq]
    return out


def head_scores(q, k, b, hq, *, scale, causal=False, window_left=-1,
                window_right=-1, bias=None, t5_table=None, t5_num_buckets=32,
                t5_max_distance=128, t5_bidirectional=True, alibi_slopes=None,
                rel_table=None, rows=None):
    """Masked score matrix S for one (b, hq): scale * Q K^T + bias, -inf where
    masked.  q: [B, L, Hq, d], k: [B, Lk, Hkv, d] float64 arrays (Lk = L for
    self-attention; positions of both sequences count from 0).  With
    ``rows`` (an index array), only those query rows of S are formed."""
    B, L, Hq, d = q.shape
    Lk = k.shape[1]
    Hkv = k.shape[2]
    g = hq // (Hq // Hkv)
    r = np.arange(L) if rows is None else np.asarray(rows)
    S = scale * (q[b, r, hq, :] @ k[b, :, g, :].T)
    if bias is not None or t5_table is not None or alibi_slopes is not None or \
            rel_table is not None:
        S = S + _bias_matrix(b, hq, L, bias, t5_table, t5_num_buckets, t5_max_distance,
                             t5_bidirectional, alibi_slopes, Lk, rel_table)[r]
    M = visibility_mask(L, causal, window_left, window_right, Lk)[r]
    S = np.where(M, S, -np.inf)
    return S


def _softmax_rows(S):
    """Row softmax of a masked score matrix and its natural-log LSE."""
    m = np.max(S, axis=1)
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    E = np.exp(S - m_safe[:, None])           # exp(-inf) = 0 for masked
    ssum = E.sum(axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        lse = np.where(ssum > 0, m_safe + np.log(ssum), -np.inf)
        P = np.where(ssum[:, None] > 0, E / ssum[:, None], 0.0)
    return P, lse


def _select(B, Hkv, batches, kv_heads):
    bs = range(B) if batches is None else list(batches)
    gs = range(Hkv) if kv_heads is None else list(kv_heads)
    return bs, gs


def _scale_of(d, scale):
    return 1.0 / math.sqrt(d) if scale is None else float(scale)


def attention_probs(q, k, b, hq, *, scale=None, **mask_bias):
    """Probability matrix P (rows sum to 1 over visible keys) for one head."""
    q = _as64(q)
    k = _as64(k)
    for name in ("bias", "t5_table", "alibi_slopes", "rel_table"):
        if name in mask_bias:
            mask_bias[name] = _as64(mask_bias[name])
    S = head_scores(q, k, b, hq, scale=_scale_of(q.shape[-1], scale), **mask_bias)
    P, _ = _softmax_rows(S)
    return P


def attention_forward(q, k, v, *, scale=None, causal=False, window_left=-1,
                      window_right=-1, bias=None, t5_table=None,
                      t5_num_buckets=32, t5_max_distance=128,
                      t5_bidirectional=True, alibi_slopes=None, rel_table=None,
                      batches=None, kv_heads=None, query_rows=None):
    """O = softmax(scale Q K^T + bias, masked) V and LSE, in float64.

    q: [B, L, Hq, d]; k, v: [B, Lk, Hkv, d] (Lk = L for self-attention);
    bias: [B|1, Hq|1, L|1, Lk] or None;
    t5_table: [num_buckets, Hq] or None; alibi_slopes: [Hq] or None;
    rel_table: [L + Lk - 1, Hq] (row j - i + L - 1) or None.
    Returns O [B, L, Hq, d] and
    LSE [B, Hq, L]; when ``batches`` / ``kv_heads`` restrict the work to a
    subset, entries outside it are NaN.
    """
    q, k, v = _as64(q), _as64(k), _as64(v)
    bias, t5_table, alibi_slopes = _as64(bias), _as64(t5_table), _as64(alibi_slopes)
    rel_table = _as64(rel_table)
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    assert Hq % Hkv == 0
    G = Hq // Hkv
    sc = _scale_of(d, scale)
    O = np.full((B, L, Hq, v.shape[-1]), np.nan)
    LSE = np.full((B, Hq, L), np.nan)
    kw = dict(causal=causal, window_left=window_left, window_right=window_right,
              bias=bias, t5_table=t5_table, t5_num_buckets=t5_num_buckets,
              t5_max_distance=t5_max_distance, t5_bidirectional=t5_bidirectional,
              alibi_slopes=alibi_slopes, rel_table=rel_table)
    r = np.arange(L) if query_rows is None else np.asarray(query_rows)
    bs, gs = _select(B, Hkv, batches, kv_heads)
    for b in bs:
        for g in gs:
            for hq in range(g * G, (g + 1) * G):
                S = head_scores(q, k, b, hq, scale=sc, rows=r, **kw)
                P, lse = _softmax_rows(S)
                O[b, r, hq, :] = P @ v[b, :, g, :]
                LSE[b, hq, r] = lse
    return O, LSE


def attention_backward(q, k, v, do, *, scale=None, causal=False,
                       window_left=-1, window_right=-1, bias=None,
                       t5_table=None, t5_num_buckets=32, t5_max_distance=128,
                       t5_bidirectional=True, alibi_slopes=None, rel_table=None,
                       batches=None, kv_heads=None, return_dbias=False):
    """Gradients of sum(O * dO) with respect to Q, K, V (float64).

    Returns dQ [B, L, Hq, d], dK and dV [B, Lk, Hkv, d] (and, with
    ``return_dbias``, dS per head as [B, Hq, L, Lk], the gradient of a dense
    additive bias).  Subset selection as in ``attention_forward``.
    """
    q, k, v, do = _as64(q), _as64(k), _as64(v), _as64(do)
    bias, t5_table, alibi_slopes = _as64(bias), _as64(t5_table), _as64(alibi_slopes)
    rel_table = _as64(rel_table)
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    sc = _scale_of(d, scale)
    dQ = np.full(q.shape, np.nan)
    dK = np.full(k.shape, np.nan)
    dV = np.full(v.shape, np.nan)
    dB = np.full((B, Hq, L, k.shape[1]), np.nan) if return_dbias else None
    kw = dict(causal=causal, window_left=window_left, window_right=window_right,
              bias=bias, t5_table=t5_table, t5_num_buckets=t5_num_buckets,
              t5_max_distance=t5_max_distance, t5_bidirectional=t5_bidirectional,
              alibi_slopes=alibi_slopes, rel_table=rel_table)
    bs, gs = _select(B, Hkv, batches, kv_heads)
    for b in bs:
        for g in gs:
            dK[b, :, g, :] = 0.0
            dV[b, :, g, :] = 0.0
            Kg = k[b, :, g, :]
            Vg = v[b, :, g, :]
            for hq in range(g * G, (g + 1) * G):
                S = head_scores(q, k, b, hq, scale=sc, **kw)
                P, _ = _softmax_rows(S)
                dO = do[b, :, hq, :]
                dP = dO @ Vg.T                               # dL/dP
                Dv = np.sum(P * dP, axis=1)                  # rowsum(P * dP)
                dS = P * (dP - Dv[:, None])                  # softmax Jacobian
                dQ[b, :, hq, :] = sc * (dS @ Kg)
                dK[b, :, g, :] += sc * (dS.T @ q[b, :, hq, :])
                dV[b, :, g, :] += P.T @ dO
                if dB is not None:
                    dB[b, hq] = dS
    if return_dbias:
        return dQ, dK, dV, dB
    return dQ, dK, dV


# --------------------------------------------------------------------------
# Bias gradients (chain rule through the additive bias; catie-aq/flashT5
# README, "Full attention biases" and "T5-like relative position encoding
# biases").
# --------------------------------------------------------------------------
def dense_bias_gradient(dS, bias_shape):
    """Gradient of a dense bias of shape ``bias_shape`` = [B|1, Hq|1, L|1, L]
    from dS [B, Hq, L, L]: dS summed over each index where the bias has
    extent 1 (it was broadcast there), in float64."""
    dS = np.asarray(dS, dtype=np.float64)
    assert len(bias_shape) == 4 and bias_shape[3] == dS.shape[3]
    axes = tuple(a for a in range(3) if bias_shape[a] == 1 and dS.shape[a] != 1)
    out = dS.sum(axis=axes, keepdims=True) if axes else dS.copy()
    assert out.shape == tuple(bias_shape)
    return out


def t5_table_gradient(dS, num_buckets: int = 32, max_distance: int = 128,
                      bidirectional: bool = True):
    """Gradient of a T5 table [num_buckets, Hq] from dS [B, Hq, L, L]:
    grad[k, h] = sum of dS[b, h, i, j] over every (b, i, j) whose distance
    j - i falls in bucket k (one explicit scatter-add per head)."""
    dS = np.asarray(dS, dtype=np.float64)
    B, Hq, L, Lk = dS.shape
    i = np.arange(L)[:, None]
    j = np.arange(Lk)[None, :]
    bucket = t5_relative_bucket(j - i, num_buckets, max_distance, bidirectional)
    grad = np.zeros((num_buckets, Hq))
    for h in range(Hq):
        np.add.at(grad[:, h], bucket.ravel(), dS[:, h].sum(axis=0).ravel())
    return grad


def alibi_slope_gradient(dS):
    """Gradient of the ALiBi slopes [Hq] from dS [B, Hq, L, L]: the bias
    -m_h |j - i| is linear in m_h, so dm_h = -sum over (b, i, j) of
    |j - i| dS[b, h, i, j]."""
    dS = np.asarray(dS, dtype=np.float64)
    L, Lk = dS.shape[2], dS.shape[3]
    dist = np.abs(np.arange(Lk)[None, :] - np.arange(L)[:, None])
    return -np.einsum("bhij,ij->h", dS, dist)


def rel_table_gradient(dS):
    """Gradient of a relative-position table [L + Lk - 1, Hq] from dS
    [B, Hq, L, Lk]: entry j - i + L - 1 collects every dS[b, h, i, j] at that
    distance (chain rule through the lookup; one explicit scatter-add)."""
    dS = np.asarray(dS, dtype=np.float64)
    B, Hq, L, Lk = dS.shape
    row = (np.arange(Lk)[None, :] - np.arange(L)[:, None] + L - 1).ravel()
    grad = np.zeros((L + Lk - 1, Hq))
    for h in range(Hq):
        np.add.at(grad[:, h], row, dS[:, h].sum(axis=0).ravel())
    return grad


def _fire_inputs(L, Lk, c, threshold):
    """FIRE's normalized distance x = psi(|i - j|) / psi(threshold) for the
    rows j - i = -(L - 1) .. Lk - 1, psi(t) = log(c t + 1)."""
    if threshold < L - 1:
        raise ValueError("the FIRE threshold must be at least the last query position")
    dist = np.abs(np.arange(-(L - 1), Lk, dtype=np.float64))
    return np.log(c * dist + 1.0) / np.log(c * threshold + 1.0), dist


def fire_table(L, Lk, c, threshold, w1, b1, w2, b2):
    """FIRE bias as a relative-position table [L + Lk - 1, H] (Li et al.
    2023): f(x) = w2 relu(w1 x + b1) + b2 per head, x = psi(|i - j|) /
    psi(threshold), psi(t) = log(c t + 1).  w1, b1: [W]; w2: [H, W]; b2: [H]."""
    w1, b1, w2, b2 = (np.asarray(a, dtype=np.float64) for a in (w1, b1, w2, b2))
    x, _ = _fire_inputs(L, Lk, c, threshold)
    hidden = np.maximum(np.outer(x, w1) + b1[None, :], 0.0)      # [R, W]
    return hidden @ w2.T + b2[None, :]                             # [R, H]


def fire_gradients(d_table, L, Lk, c, threshold, w1, b1, w2, b2):
    """Gradients of sum(d_table * fire_table(...)) with respect to w1, b1, w2,
    b2, c and threshold (chain rule through the MLP and psi).  Returns a dict
    of float64 arrays (c and threshold as scalars)."""
    g = np.asarray(d_table, dtype=np.float64)                      # [R, H]
    w1, b1, w2, b2 = (np.asarray(a, dtype=np.float64) for a in (w1, b1, w2, b2))
    x, dist = _fire_inputs(L, Lk, c, threshold)
    pre = np.outer(x, w1) + b1[None, :]
    hidden = np.maximum(pre, 0.0)
    d_hidden = g @ w2                                              # [R, W]
    d_pre = np.where(pre > 0.0, d_hidden, 0.0)
    dx = d_pre @ w1                                                # [R]
    num = np.log(c * dist + 1.0)
    den = np.log(c * threshold + 1.0)
    dx_dc = (dist / (c * dist + 1.0)) / den - num * (threshold / (c * threshold + 1.0)) / den ** 2
    dx_dt = -num * (c / (c * threshold + 1.0)) / den ** 2
    return {"w1": d_pre.T @ x, "b1": d_pre.sum(axis=0), "w2": g.T @ hidden,
            "b2": g.sum(axis=0), "c": float(dx @ dx_dc), "threshold": float(dx @ dx_dt)}


# --------------------------------------------------------------------------
# Packed variable-length sequences (transformers issue #30461, packing=True;
# catie-aq/flashT5 README, dynamic batching).
# --------------------------------------------------------------------------
def packed_positions(cu_seqlens):
    """Sequence id and local position (from 0) of every row of a packed axis."""
    cu = [int(x) for x in np.asarray(cu_seqlens)]
    total = cu[-1]
    seq = np.empty(total, dtype=np.int64)
    pos = np.empty(total, dtype=np.int64)
    for b in range(len(cu) - 1):
        seq[cu[b]:cu[b + 1]] = b
        pos[cu[b]:cu[b + 1]] = np.arange(cu[b + 1] - cu[b])
    return seq, pos


def packed_visibility_mask(cu_seqlens_q, cu_seqlens_k, causal, window_left=-1,
                           window_right=-1):
    """Boolean [total_q, total_k]: packed query row r sees packed key row c
    iff both belong to the same sequence and their local positions i, j
    satisfy the mask (j <= i if causal, j >= i - window_left, j <= i +
    window_right; negative bounds unbounded)."""
    sq, i = packed_positions(cu_seqlens_q)
    sk, j = packed_positions(cu_seqlens_k)
    i = i[:, None]
    j = j[None, :]
    m = sq[:, None] == sk[None, :]
    if causal:
        m &= j <= i
    if window_left is not None and window_left >= 0:
        m &= j >= i - window_left
    if window_right is not None and window_right >= 0:
        m &= j <= i + window_right
    return m


def _packed_scores(q, k, hq, G, sc, M, rel, t5_table, t5_num_buckets, t5_max_distance,
                   t5_bidirectional, alibi_slopes):
    S = sc * (q[:, hq, :] @ k[:, hq // G, :].T)
    if t5_table is not None:
        S = S + t5_table[t5_relative_bucket(rel, t5_num_buckets, t5_max_distance,
                                            t5_bidirectional), hq]
    if alibi_slopes is not None:
        S = S - alibi_slopes[hq] * np.abs(rel)
    return np.where(M, S, -np.inf)


def attention_forward_packed(q, k, v, cu_seqlens_q, cu_seqlens_k, *, scale=None,
                             causal=False, window_left=-1, window_right=-1, t5_table=None,
                             t5_num_buckets=32, t5_max_distance=128, t5_bidirectional=True,
                             alibi_slopes=None):
    """O [total_q, Hq, d] and LSE [Hq, total_q] of a packed batch: the
    definition over the whole packed axis with the block-diagonal mask of
    ``packed_visibility_mask`` and the relative position j - i of the local
    positions.  q: [total_q, Hq, d]; k, v: [total_k, Hkv, d]."""
    q, k, v = _as64(q), _as64(k), _as64(v)
    t5_table, alibi_slopes = _as64(t5_table), _as64(alibi_slopes)
    Tq, Hq, d = q.shape
    G = Hq // k.shape[1]
    sc = _scale_of(d, scale)
    M = packed_visibility_mask(cu_seqlens_q, cu_seqlens_k, causal, window_left, window_right)
    _, pi = packed_positions(cu_seqlens_q)
    _, pj = packed_positions(cu_seqlens_k)
    rel = pj[None, :] - pi[:, None]
    O = np.zeros((Tq, Hq, v.shape[-1]))
    LSE = np.zeros((Hq, Tq))
    for hq in range(Hq):
        S = _packed_scores(q, k, hq, G, sc, M, rel, t5_table, t5_num_buckets, t5_max_distance,
                           t5_bidirectional, alibi_slopes)
        P, lse = _softmax_rows(S)
        O[:, hq, :] = P @ v[:, hq // G, :]
        LSE[hq] = lse
    return O, LSE


def attention_backward_packed(q, k, v, do, cu_seqlens_q, cu_seqlens_k, *, scale=None,
                              causal=False, window_left=-1, window_right=-1, t5_table=None,
                              t5_num_buckets=32, t5_max_distance=128, t5_bidirectional=True,
                              alibi_slopes=None, return_intermediates=False):
    """dQ [total_q, Hq, d], dK and dV [total_k, Hkv, d] of sum(O * dO) for a
    packed batch, by the chain rule over the packed axis (as in
    ``attention_backward``).  With ``return_intermediates`` also P and dS,
    each [Hq, total_q, total_k]."""
    q, k, v, do = _as64(q), _as64(k), _as64(v), _as64(do)
    t5_table, alibi_slopes = _as64(t5_table), _as64(alibi_slopes)
    Tq, Hq, d = q.shape
    G = Hq // k.shape[1]
    sc = _scale_of(d, scale)
    M = packed_visibility_mask(cu_seqlens_q, cu_seqlens_k, causal, window_left, window_right)
    _, pi = packed_positions(cu_seqlens_q)
    _, pj = packed_positions(cu_seqlens_k)
    rel = pj[None, :] - pi[:, None]
    dQ = np.zeros(q.shape)
    dK = np.zeros(k.shape)
    dV = np.zeros(v.shape)
    Ps, dSs = [], []
    for hq in range(Hq):
        g = hq // G
        S = _packed_scores(q, k, hq, G, sc, M, rel, t5_table, t5_num_buckets, t5_max_distance,
                           t5_bidirectional, alibi_slopes)
        P, _ = _softmax_rows(S)
        dP = do[:, hq, :] @ v[:, g, :].T
        Dv = np.sum(P * dP, axis=1)
        dS = P * (dP - Dv[:, None])
        dQ[:, hq, :] = sc * (dS @ k[:, g, :])
        dK[:, g, :] += sc * (dS.T @ q[:, hq, :])
        dV[:, g, :] += P.T @ do[:, hq, :]
        if return_intermediates:
            Ps.append(P)
            dSs.append(dS)
    if return_intermediates:
        return dQ, dK, dV, np.stack(Ps), np.stack(dSs)
    return dQ, dK, dV
