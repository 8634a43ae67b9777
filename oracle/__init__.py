"""fp64 CPU oracle for block-sparse causal prefill attention (test infrastructure).

This package is test infrastructure, not product code. Only the tests, the smoke check
in ``__graft_entry__`` and the ``cpu_baseline`` / ``--impl reference`` legs of
``bench.py`` may import it. It shares no code with the CUDA path and imports nothing
from the product package. Its inputs are the exact values the kernels read (bf16, or
e4m3 codes times their per-head scale), widened to float64.

It follows the three stages in the order the pages give them:

1. ``pool_blocks``  -- block-mean pooling ("FlashPrefill: Instantaneous Pattern Discovery
   and Thresholding for Ultra-Fast Long-Context Prefilling", technical summary 2.A,
   "Block Approximation": keys averaged per block; the skeleton of queries is read as
   block means of Q as well, so that the pooled score is the mean of the raw block of
   scaled Q K^T, which is what the fused 2-D reduction of 2.A computes in one pass).
2. ``block_scores`` and ``block_keep`` -- the pooled block-score matrix and the max-based
   dynamic threshold thresh_I = alpha * max_{J<=I} Score_{I,J} (same page, 2.B), with
   Score read as the softmax probability over the causal pooled row, an inclusive
   comparison, and the diagonal and first blocks always kept.
3. ``masked_causal_attention`` -- exact softmax attention of each query over the keys
   j <= i whose block was kept for (head, query block); skipped blocks take no part at
   all (same page, 2.C, physical skip).

GQA: query head h reads KV head h // (Hq / Hkv). Requests of a varlen batch are
independent; blocks restart at each request's first token and a request's last block
may hold fewer than ``block`` tokens (its mean runs over the valid tokens only).

Chunked (prefix-cached) prefill: with ``cu_k`` given, request b holds kv_len_b keys and its
q_len_b queries are the LAST q_len_b positions P0_b = kv_len_b - q_len_b .. kv_len_b - 1
(causality aligned at the bottom right). Blocks are defined on absolute positions, so the
request's query blocks run from I0_b = P0_b // block to the last kv block; a query block's
pooled mean runs over the queries it holds. Without ``cu_k``, q_len = kv_len (P0 = 0).

Pins: every function here is pinned by ``tests/test_oracle_pins.py`` against brute
force, closed forms and special cases (see the docstrings there). The V2 mean-correction
term is named by the pages but never defined, so it is not implemented here.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = ["pool_blocks", "pool_query_blocks", "block_scores", "block_keep", "keep_ratio",
           "masked_causal_attention", "request_blocks", "query_blocks"]


def request_blocks(cu_seqlens, block):
    """Per-request block counts and the offsets of each request's first block."""
    cu = [int(x) for x in cu_seqlens]
    nb = [(cu[b + 1] - cu[b] + block - 1) // block for b in range(len(cu) - 1)]
    off = [0]
    for n in nb:
        off.append(off[-1] + n)
    return nb, off


def query_blocks(cu_q, cu_k, block):
    """Per request: (first query position P0, first absolute query block I0, number of query
    blocks nq), and the offsets of each request's first query block."""
    cq = [int(x) for x in cu_q]
    ck = [int(x) for x in (cu_k if cu_k is not None else cu_q)]
    info, off = [], [0]
    for b in range(len(cq) - 1):
        L, n = ck[b + 1] - ck[b], cq[b + 1] - cq[b]
        assert 0 <= n <= L
        P0 = L - n
        I0 = P0 // block
        nq = (L + block - 1) // block - I0 if n > 0 else 0
        info.append((P0, I0, nq))
        off.append(off[-1] + nq)
    return info, off


def _widen(x, lo, hi, heads, scale):
    """Rows lo..hi-1 of x[:, heads] as float64, times the per-head scale if given."""
    y = np.asarray(x[lo:hi, heads], dtype=np.float64)
    if scale is not None:
        sc = np.asarray(scale, dtype=np.float64)[heads]
        y = y * (sc[None, :, None] if y.ndim == 3 else sc)
    return y


def pool_blocks(x, block, cu_seqlens, scale=None):
    """Block means of ``x`` [T, H, d] -> float64 [H, total_blocks, d].

    Block I of request b averages tokens cu[b] + I*block ... min(cu[b+1], cu[b]+(I+1)*block)-1
    of x * scale[h] (scale: optional per-head dequantisation factor).
    """
    T, H, d = x.shape
    nb, off = request_blocks(cu_seqlens, block)
    out = np.zeros((H, off[-1], d), dtype=np.float64)
    cu = [int(c) for c in cu_seqlens]
    heads = np.arange(H)
    for b in range(len(nb)):
        for I in range(nb[b]):
            lo = cu[b] + I * block
            hi = min(cu[b + 1], lo + block)
            out[:, off[b] + I, :] = _widen(x, lo, hi, heads, scale).mean(axis=0)
    return out


def pool_query_blocks(q, block, cu_q, cu_k, scale=None):
    """Chunked prefill: means of the queries each query block holds -> [Hq, total_qblocks, d].
    Query block I of request b holds positions max(P0, I*block) .. min(L, (I+1)*block) - 1,
    stored at rows cu_q[b] + (position - P0)."""
    T, H, d = q.shape
    info, off = query_blocks(cu_q, cu_k, block)
    ck = [int(x) for x in cu_k]
    cq = [int(x) for x in cu_q]
    out = np.zeros((H, off[-1], d), dtype=np.float64)
    heads = np.arange(H)
    for b, (P0, I0, nq) in enumerate(info):
        L = ck[b + 1] - ck[b]
        for i in range(nq):
            I = I0 + i
            lo, hi = max(P0, I * block), min(L, (I + 1) * block)
            out[:, off[b] + i, :] = _widen(q, cq[b] + lo - P0, cq[b] + hi - P0, heads,
                                           scale).mean(axis=0)
    return out


def block_scores(q_pool, k_pool, cu_seqlens, block, scale, cu_k=None):
    """Pooled block scores per request: list of [Hq, nq, nk] float64 arrays with
    s[h, i, J] = scale * qbar[h, I] . kbar[h // G, J] for J <= I and -inf for J > I, where
    I = I0 + i is the absolute block of query-block row i (I0 = 0 without ``cu_k``, and then
    nq = nk). ``cu_seqlens`` are the query lengths; ``cu_k`` the key lengths if they differ."""
    Hq = q_pool.shape[0]
    Hkv = k_pool.shape[0]
    G = Hq // Hkv
    nk, koff = request_blocks(cu_k if cu_k is not None else cu_seqlens, block)
    info, qoff = query_blocks(cu_seqlens, cu_k, block)
    out = []
    for b in range(len(nk)):
        P0, I0, nq = info[b]
        n = nk[b]
        s = np.full((Hq, nq, n), -np.inf)
        causal = np.arange(n)[None, :] <= (I0 + np.arange(nq))[:, None]
        for h in range(Hq):
            qb = q_pool[h, qoff[b]:qoff[b] + nq]
            kb = k_pool[h // G, koff[b]:koff[b] + n]
            full = scale * (qb @ kb.T)
            s[h][causal] = full[causal]
        out.append(s)
    return out


def _row_softmax(s):
    """Softmax over the last axis of a score array whose masked entries are -inf. A request
    without tokens has no blocks: its (empty) array is returned as it is."""
    if s.shape[-1] == 0:
        return s.copy()
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=-1, keepdims=True)


def block_keep(scores, alpha, force_first=True, force_diag=True, row0=0):
    """Keep set for one request: bool [Hq, nq, nk] (row i is absolute query block row0 + i).

    p = softmax over the causal pooled row; keep J iff p[J] >= alpha * max_J p, plus the
    diagonal block J = I and the first block J = 0 when forced."""
    nq, n = scores.shape[-2:]
    if n == 0:
        return np.zeros(scores.shape, dtype=bool)
    p = _row_softmax(scores)
    keep = p >= alpha * p.max(axis=-1, keepdims=True)
    rows = row0 + np.arange(nq)
    causal = np.arange(n)[None, :] <= rows[:, None]
    keep &= causal[None]
    if force_diag:
        keep[:, np.arange(nq), rows] = True
    if force_first:
        keep[:, :, 0] = True
    return keep


def keep_ratio(scores):
    """p[J] / max p over each causal row (float64; 0 above the diagonal). A block whose
    ratio lies within a relative 1e-3 of alpha sits on the threshold, where fp32 and fp64
    may legitimately decide differently."""
    if scores.shape[-1] == 0:
        return scores.copy()
    p = _row_softmax(scores)
    return p / p.max(axis=-1, keepdims=True)


def masked_causal_attention(q, k, v, keeps, cu_seqlens, block, scale, rows=None,
                            q_scale=None, k_scale=None, v_scale=None, cu_k=None):
    """Exact masked causal softmax attention in float64.

    q [Tq, Hq, d], k/v [Tk, Hkv, d] (times the optional per-head ``*_scale``); ``keeps`` is the
    list of per-request bool keep sets [Hq, nq, nk] (row i = absolute query block I0 + i).
    Query i of request b at absolute position p (row cu_q[b] + p - P0) in block I = p // block
    attends to the keys j <= p of that request whose block J = j // block is kept for (h, I).
    Without ``cu_k`` the queries are the whole request (P0 = 0, cu_k = cu_seqlens).

    ``rows``: None for every (head, global query block), else an iterable of (h, Ig).
    Returns (out [Tq, Hq, d] float64 with NaN where not computed, lse [Hq, Tq] natural log
    of the sum of exp(scaled logits), NaN where not computed).
    """
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    cq = [int(c) for c in cu_seqlens]
    ck = [int(c) for c in (cu_k if cu_k is not None else cu_seqlens)]
    info, off = query_blocks(cu_seqlens, cu_k, block)
    if rows is None:
        rows = [(h, Ig) for h in range(Hq) for Ig in range(off[-1])]
    out = np.full((T, Hq, d), np.nan)
    lse = np.full((Hq, T), np.nan)
    for h, Ig in rows:
        b = int(np.searchsorted(off, Ig, side="right") - 1)
        P0, I0, nq = info[b]
        i = Ig - off[b]
        I = I0 + i
        kbase = ck[b]
        L = ck[b + 1] - kbase
        p_lo, p_hi = max(P0, I * block), min(L, (I + 1) * block)   # query positions
        kept = [J for J in range(I + 1) if keeps[b][h, i, J]]
        if not kept:
            continue
        key_pos = np.concatenate([np.arange(J * block, min(L, (J + 1) * block)) for J in kept])
        qrows = slice(cq[b] + p_lo - P0, cq[b] + p_hi - P0)
        qi = np.asarray(q[qrows, h], dtype=np.float64)
        kj = np.asarray(k[kbase + key_pos, h // G], dtype=np.float64)
        vj = np.asarray(v[kbase + key_pos, h // G], dtype=np.float64)
        if q_scale is not None:
            qi = qi * float(q_scale[h])
        if k_scale is not None:
            kj = kj * float(k_scale[h // G])
        if v_scale is not None:
            vj = vj * float(v_scale[h // G])
        s = scale * (qi @ kj.T)
        s[key_pos[None, :] > np.arange(p_lo, p_hi)[:, None]] = -np.inf
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        z = e.sum(axis=1, keepdims=True)
        out[qrows, h] = (e @ vj) / z
        lse[h, qrows] = (m + np.log(z))[:, 0]
    return out, lse


def default_scale(d):
    """Softmax scale 1/sqrt(d), used both for the pooled scores and for attention."""
    return 1.0 / math.sqrt(d)
