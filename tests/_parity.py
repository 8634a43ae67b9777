"""Shared helpers of the GPU parity tests: run the oracle on a workload's exact inputs, turn
an oracle keep set into kernel index lists (host code), and compare results.

Tolerances (stated by the workload specification for this path):
  block mask : bit-identical except blocks whose oracle ratio p_J / max p lies within a
               relative 1e-3 of alpha (there fp32 and fp64 may decide differently);
  attention  : bf16 max-abs <= 1e-2 and relative L2 <= 5e-3; e4m3 <= 6e-2 and <= 3e-2.
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


def attn_errors(out_gpu, out_ref, rows_mask=None):
    """(max-abs, relative L2) over the computed (non-NaN) entries of the oracle output."""
    g = out_gpu.float().cpu().double().numpy()
    r = out_ref
    sel = ~np.isnan(r)
    if rows_mask is not None:
        sel &= rows_mask
    d = g[sel] - r[sel]
    return float(np.abs(d).max()), float(np.linalg.norm(d) / max(np.linalg.norm(r[sel]), 1e-30))


def device_inputs(inp, dev):
    q = inp.q.to(dev)
    k = inp.k.to(dev)
    v = inp.v.to(dev)
    sc = {}
    for n in ("q_scale", "k_scale", "v_scale"):
        t = getattr(inp, n)
        sc[n] = None if t is None else t.to(dev)
    return q, k, v, sc
