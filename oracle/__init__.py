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

Pins: every function here is pinned by ``tests/test_oracle_pins.py`` against brute
force, closed forms and special cases (see the docstrings there). The V2 mean-correction
term is named by the pages but never defined, so it is not implemented here.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = ["pool_blocks", "block_scores", "block_keep", "keep_ratio",
           "masked_causal_attention", "request_blocks"]


def request_blocks(cu_seqlens, block):
    """Per-request block counts and the offsets of each request's first block."""
    cu = [int(x) for x in cu_seqlens]
    nb = [(cu[b + 1] - cu[b] + block - 1) // block for b in range(len(cu) - 1)]
    off = [0]
    for n in nb:
        off.append(off[-1] + n)
    return nb, off


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


def block_scores(q_pool, k_pool, cu_seqlens, block, scale):
    """Pooled block scores per request: list of [Hq, nb, nb] float64 arrays with
    s[h, I, J] = scale * qbar[h, I] . kbar[h // G, J] for J <= I and -inf for J > I."""
    Hq = q_pool.shape[0]
    Hkv = k_pool.shape[0]
    G = Hq // Hkv
    nb, off = request_blocks(cu_seqlens, block)
    out = []
    for b in range(len(nb)):
        n = nb[b]
        s = np.full((Hq, n, n), -np.inf)
        causal = np.tril(np.ones((n, n), dtype=bool))
        for h in range(Hq):
            qb = q_pool[h, off[b]:off[b] + n]
            kb = k_pool[h // G, off[b]:off[b] + n]
            full = scale * (qb @ kb.T)
            s[h][causal] = full[causal]
        out.append(s)
    return out


def _row_softmax(s):
    """Softmax over the last axis of a score array whose masked entries are -inf."""
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=-1, keepdims=True)


def block_keep(scores, alpha, force_first=True, force_diag=True):
    """Keep set for one request: bool [Hq, nb, nb].

    p = softmax over the causal pooled row; keep J iff p[J] >= alpha * max_J p, plus the
    diagonal block J = I and the first block J = 0 when forced."""
    p = _row_softmax(scores)
    keep = p >= alpha * p.max(axis=-1, keepdims=True)
    n = scores.shape[-1]
    causal = np.tril(np.ones((n, n), dtype=bool))
    keep &= causal[None]
    if force_diag:
        idx = np.arange(n)
        keep[:, idx, idx] = True
    if force_first:
        keep[:, :, 0] = True
    return keep


def keep_ratio(scores):
    """p[J] / max p over each causal row (float64; 0 above the diagonal). A block whose
    ratio lies within a relative 1e-3 of alpha sits on the threshold, where fp32 and fp64
    may legitimately decide differently."""
    p = _row_softmax(scores)
    return p / p.max(axis=-1, keepdims=True)


def masked_causal_attention(q, k, v, keeps, cu_seqlens, block, scale, rows=None,
                            q_scale=None, k_scale=None, v_scale=None):
    """Exact masked causal softmax attention in float64.

    q [T, Hq, d], k/v [T, Hkv, d] (times the optional per-head ``*_scale``); ``keeps`` is the list of per-request bool keep sets
    [Hq, nb, nb]. Query i of request b (local index t) in block I = t // block attends to
    the keys j <= t of that request whose block J = j // block has keeps[b][h, I, J].

    ``rows``: None for every (head, global query block), else an iterable of (h, Ig).
    Returns (out [T, Hq, d] float64 with NaN where not computed, lse [Hq, T] natural log
    of the sum of exp(scaled logits), NaN where not computed).
    """
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    nb, off = request_blocks(cu_seqlens, block)
    cu = [int(c) for c in cu_seqlens]
    if rows is None:
        rows = [(h, Ig) for h in range(Hq) for Ig in range(off[-1])]
    out = np.full((T, Hq, d), np.nan)
    lse = np.full((Hq, T), np.nan)
    for h, Ig in rows:
        b = int(np.searchsorted(off, Ig, side="right") - 1)
        I = Ig - off[b]
        base = cu[b]
        L = cu[b + 1] - base
        q_lo, q_hi = base + I * block, base + min(L, (I + 1) * block)
        kept = [J for J in range(I + 1) if keeps[b][h, I, J]]
        if not kept:
            continue
        key_idx = np.concatenate([np.arange(base + J * block, base + min(L, (J + 1) * block))
                                  for J in kept])
        qi = np.asarray(q[q_lo:q_hi, h], dtype=np.float64)
        kj = np.asarray(k[key_idx, h // G], dtype=np.float64)
        vj = np.asarray(v[key_idx, h // G], dtype=np.float64)
        if q_scale is not None:
            qi = qi * float(q_scale[h])
        if k_scale is not None:
            kj = kj * float(k_scale[h // G])
        if v_scale is not None:
            vj = vj * float(v_scale[h // G])
        s = scale * (qi @ kj.T)
        s[key_idx[None, :] > np.arange(q_lo, q_hi)[:, None]] = -np.inf
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        z = e.sum(axis=1, keepdims=True)
        out[q_lo:q_hi, h] = (e @ vj) / z
        lse[h, q_lo:q_hi] = (m + np.log(z))[:, 0]
    return out, lse


def default_scale(d):
    """Softmax scale 1/sqrt(d), used both for the pooled scores and for attention."""
    return 1.0 / math.sqrt(d)
