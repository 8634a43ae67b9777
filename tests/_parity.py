"""Shared helpers of the GPU parity tests: run the oracle on a workload's exact inputs, turn
an oracle keep set into kernel index lists (host code), and compare results.

Tolerances (stated by the workload specification for this path):
  block mask : bit-identical except blocks whose oracle ratio p_J / max p lies within a
               relative 1e-3 of alpha (there fp32 and fp64 may decide differently);
  attention  : bf16 max-abs <= 1e-2 and relative L2 <= 5e-3; e4m3 <= 6e-2 and <= 3e-2.
               The output format is bf16 for both, and rounding a value to bf16 alone moves
               it by up to half a bf16 ulp (2^-8 of its magnitude: 0.0078 in [2, 4), 0.0156
               in [4, 8)), so an exact result stored as bf16 could miss a plain 1e-2 bound.
               The max-abs bound is therefore read as a bound on the error of the value the
               kernel rounds to bf16: each element's error counts beyond half an ulp of the
               stored bf16 value (at most 0.0039 below magnitude 2). The relative L2 bound is
               taken as it stands.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle as O

TOL = {"bf16": (1e-2, 5e-3), "e4m3": (6e-2, 3e-2)}
EXEMPT_REL = 1e-3


class OracleRun:
    """The oracle's pooling, scores and keep sets for one workload's inputs. For a chunked
    workload (``inp.cu_q`` set) the queries are the last q_len positions of each request and
    query-side arrays are indexed by query block (request b's rows start at absolute block
    I0[b])."""

    def __init__(self, inp, alpha, force_first=True, force_diag=True):
        w = inp.workload
        self.inp = inp
        self.block = w.block
        self.cu = inp.cu_seqlens.tolist()
        self.chunked = inp.cu_q is not None
        self.cu_q = inp.cu_q.tolist() if self.chunked else self.cu
        cu_k = self.cu if self.chunked else None
        self.scale = 1.0 / math.sqrt(w.d)
        self.q = inp.codes_f32("q")
        self.k = inp.codes_f32("k")
        self.v = inp.codes_f32("v")
        self.qs, self.ks, self.vs = inp.scale_f64("q"), inp.scale_f64("k"), inp.scale_f64("v")
        if self.chunked:
            self.q_pool = O.pool_query_blocks(self.q, w.block, self.cu_q, self.cu, scale=self.qs)
        else:
            self.q_pool = O.pool_blocks(self.q, w.block, self.cu, scale=self.qs)
        self.k_pool = O.pool_blocks(self.k, w.block, self.cu, scale=self.ks)
        self.scores = O.block_scores(self.q_pool, self.k_pool, self.cu_q, w.block, self.scale,
                                     cu_k=cu_k)
        info, self.qoff = O.query_blocks(self.cu_q, cu_k, w.block)
        self.I0 = [i[1] for i in info]
        self.nq = [i[2] for i in info]
        self.keeps = [O.block_keep(s, alpha, force_first, force_diag, row0=i0)
                      for s, i0 in zip(self.scores, self.I0)]
        self.ratios = [O.keep_ratio(s) for s in self.scores]
        self.alpha = alpha
        self.nb, self.off = O.request_blocks(self.cu, w.block)

    def causal(self, r):
        """bool [nq, nk] of request r: key block J <= absolute query block I0 + i."""
        return (np.arange(self.nb[r])[None, :] <=
                (self.I0[r] + np.arange(self.nq[r]))[:, None])

    def attention(self, rows=None, keeps=None):
        return O.masked_causal_attention(self.q, self.k, self.v,
                                         self.keeps if keeps is None else keeps, self.cu_q,
                                         self.block, self.scale, rows=rows, q_scale=self.qs,
                                         k_scale=self.ks, v_scale=self.vs,
                                         cu_k=self.cu if self.chunked else None)


def keep_to_lists(keeps, Hq):
    """Kernel index lists (kv_cnt [Hq, nq], kv_idx [Hq, nq, max_kv_blocks]) of a keep set."""
    total = sum(k.shape[1] for k in keeps)
    mb = max(k.shape[-1] for k in keeps)
    cnt = np.zeros((Hq, total), dtype=np.int32)
    idx = np.full((Hq, total, mb), -7, dtype=np.int32)
    g0 = 0
    for kk in keeps:
        for h in range(Hq):
            for I in range(kk.shape[1]):
                js = np.nonzero(kk[h, I])[0]
                cnt[h, g0 + I] = len(js)
                idx[h, g0 + I, :len(js)] = js
        g0 += kk.shape[1]
    return torch.from_numpy(cnt), torch.from_numpy(idx)


def bits_to_keeps(bits, run: OracleRun):
    """GPU bitmask [Hq, nq, words] -> per-request bool keep sets [Hq, nq_b, nk_b]."""
    b = bits.cpu().numpy().view(np.uint32)
    Hq = b.shape[0]
    out = []
    for r, n in enumerate(run.nb):
        q0, nq = run.qoff[r], run.nq[r]
        kk = np.zeros((Hq, nq, n), dtype=bool)
        for J in range(n):
            kk[:, :, J] = (b[:, q0:q0 + nq, J // 32] >> np.uint32(J % 32)) & 1
        out.append(kk)
    return out


def lists_to_keeps(cnt, idx, run: OracleRun):
    c = cnt.cpu().numpy()
    ix = idx.cpu().numpy()
    Hq = c.shape[0]
    out = []
    for r, n in enumerate(run.nb):
        kk = np.zeros((Hq, run.nq[r], n), dtype=bool)
        for h in range(Hq):
            for i in range(run.nq[r]):
                g = run.qoff[r] + i
                js = ix[h, g, :c[h, g]]
                assert (np.diff(js) > 0).all(), "index list not ascending"
                kk[h, i, js] = True
        out.append(kk)
    return out


def mask_mismatches(gpu_keeps, run: OracleRun):
    """(non-exempt mismatches, exempt mismatches, total causal blocks)."""
    bad = ex = tot = 0
    for r, (gk, ok, ratio) in enumerate(zip(gpu_keeps, run.keeps, run.ratios)):
        tri = run.causal(r)[None]
        diff = (gk != ok)
        assert not (gk & ~tri).any(), "bit above the diagonal"
        near = np.abs(ratio - run.alpha) <= EXEMPT_REL * run.alpha
        bad += int((diff & ~near & tri).sum())
        ex += int((diff & near & tri).sum())
        tot += int(tri.sum()) * ok.shape[0]
    return bad, ex, tot


def bf16_half_ulp(g):
    """Half the spacing of bf16 values at each (bf16-representable) element of ``g``: the most
    that rounding a real number to that bf16 value can have moved it. 0 at zero."""
    g = np.abs(np.asarray(g, dtype=np.float64))
    _, e = np.frexp(g)                 # g = m * 2^e, 0.5 <= m < 1; bf16 keeps 8 bits of m
    return np.where(g > 0, np.ldexp(1.0, e - 9), 0.0)


def attn_errors(out_gpu, out_ref, rows_mask=None):
    """(max-abs error beyond the bf16 output rounding, relative L2) over the computed (non-NaN)
    entries of the oracle output: max |gpu - ref| - half_ulp_bf16(gpu), floored at 0."""
    g = out_gpu.float().cpu().double().numpy()
    r = out_ref
    sel = ~np.isnan(r)
    if rows_mask is not None:
        sel &= rows_mask
    gs = g[sel]
    d = gs - r[sel]
    net = np.maximum(np.abs(d) - bf16_half_ulp(gs), 0.0)
    return float(net.max()), float(np.linalg.norm(d) / max(np.linalg.norm(r[sel]), 1e-30))


def stratified_rows(run, gpu_keeps, Hq, seed, per_head=16):
    """(head, global query block) rows for a sampled attention comparison: for every head, one
    row in each tenth of the batch's query blocks, the batch's last query block, the last query
    block of one request (a different one per head) and random rows up to ``per_head``; only
    rows whose GPU and oracle masks agree (the others differ only at near-threshold blocks)."""
    rng = np.random.default_rng(seed)
    nrows = run.qoff[-1]
    ends = [run.qoff[r + 1] - 1 for r in range(len(run.nq)) if run.nq[r] > 0]
    edges = np.linspace(0, nrows, 11).astype(int)
    rows = []
    for h in range(Hq):
        picks = [nrows - 1, ends[h % len(ends)]]
        picks += [int(rng.integers(a, max(a + 1, b))) for a, b in zip(edges[:-1], edges[1:])]
        picks = list(dict.fromkeys(picks))
        for _ in range(50 * per_head):
            if len(picks) >= min(per_head, nrows):
                break
            Ig = int(rng.integers(nrows))
            if Ig not in picks:
                picks.append(Ig)
        for Ig in picks:
            r = int(np.searchsorted(run.qoff, Ig, side="right") - 1)
            i = Ig - run.qoff[r]
            if np.array_equal(gpu_keeps[r][h, i], run.keeps[r][h, i]):
                rows.append((h, Ig))
    return rows


def device_inputs(inp, dev):
    q = inp.q.to(dev)
    k = inp.k.to(dev)
    v = inp.v.to(dev)
    sc = {}
    for n in ("q_scale", "k_scale", "v_scale"):
        t = getattr(inp, n)
        sc[n] = None if t is None else t.to(dev)
    return q, k, v, sc
