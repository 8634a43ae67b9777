"""GPU parity of chunked (prefix-cached) prefill against the fp64 oracle, through the C ABI.

Request b holds kv_len_b keys and prefills its last q_len_b positions: the pooled query means,
the block mask on absolute block positions and the attention of the chunk's queries over the
whole request (cached prefix included) are compared with the oracle on the same inputs. The
attention runs on index lists the host writes from the oracle's own keep set.
"""
import dataclasses

import numpy as np
import pytest
import torch

import block_sparse_long_qk_b200 as fp
from block_sparse_long_qk_b200 import synthetic as S

from _parity import (TOL, OracleRun, attn_errors, bits_to_keeps, device_inputs, keep_to_lists,
                     lists_to_keeps, mask_mismatches)

pytestmark = pytest.mark.gpu

W = S.WORKLOADS
BASE = dataclasses.replace(W["chunked"], Hq=8, Hkv=2, structure="iid", page_size=0)

# (workload, kv_lens, q_lens, alpha). The q_lens cover: a whole request (q_len = kv_len), an
# empty chunk, chunks that start inside a block (partial first query block), a chunk inside a
# single block, one query, block-aligned starts, and a ragged last block.
CASES = {
    "mixed": (BASE, (1000, 700, 300, 1500, 129), (1000, 0, 37, 641, 1), 0.5),
    "aligned": (BASE, (1024, 640), (512, 128), 0.5),
    "one_block": (BASE, (900, 200), (50, 100), 0.5),
    "band": (dataclasses.replace(BASE, structure="band"), (3000, 2500), (900, 1300), 0.1),
    "dense_alpha0": (BASE, (777, 400), (300, 399), 0.0),
    "paged": (dataclasses.replace(BASE, page_size=64), (1000, 700, 300), (333, 700, 65), 0.5),
    "fp8": (dataclasses.replace(BASE, dtype="e4m3"), (1100, 600), (450, 130), 0.5),
    "b64_d64": (dataclasses.replace(BASE, block=64, d=64), (700, 333), (250, 90), 0.5),
    "gqa3": (dataclasses.replace(BASE, Hq=6), (800, 500), (300, 77), 0.5),
    "gqa5": (dataclasses.replace(BASE, Hq=10, structure="band"), (900, 1300), (450, 129), 0.1),
    # one query head per KV head: query-block pairs. 6 + 7 + 2 query blocks: the pair (6, 5)
    # holds the first block of request 1 and the last of request 0
    "mha": (dataclasses.replace(BASE, Hq=2, Hkv=2), (1000, 850, 300), (744, 850, 65), 0.5),
    # many key blocks per row (several score chunks in the mask kernel), long cached prefix
    "long_prefix": (dataclasses.replace(W["llama128k"], Hq=8, Hkv=2), (20000, 9000),
                    (1500, 2700), 0.1),
}


def _inputs(name):
    w, kv, ql, alpha = CASES[name]
    return S.make_inputs(w, seed=9, seqlens=kv, q_lens=ql), alpha


def _cb(inp, dev):
    w = inp.workload
    return fp.ChunkedBatch.make(w.q_lens, w.seqlens, w.block, dev)


def _paged(inp, dev):
    if not inp.workload.page_size:
        return None
    return fp.PagedKV(inp.k_cache.to(dev), inp.v_cache.to(dev), inp.page_table.to(dev))


@pytest.mark.parametrize("name", list(CASES))
def test_chunked_pool_and_mask_match_oracle(name, cuda_device):
    inp, alpha = _inputs(name)
    w = inp.workload
    run = OracleRun(inp, alpha)
    q, k, _, sc = device_inputs(inp, cuda_device)
    cb = _cb(inp, cuda_device)
    paged = _paged(inp, cuda_device)
    split = torch.empty(fp.k_split_shape(w.Hkv, cb.total_kblocks, w.d), dtype=torch.bfloat16,
                        device=cuda_device)
    qp, kp = fp.pool_qk_chunked(q, k, cb, q_scale=sc["q_scale"], k_scale=sc["k_scale"],
                                paged=paged, k_split_out=split)
    torch.cuda.synchronize()
    for got, ref in ((qp, run.q_pool), (kp, run.k_pool)):
        g = got.cpu().double().numpy()
        assert g.shape == ref.shape
        assert np.abs(g - ref).max() <= 1e-5 * max(1.0, np.abs(ref).max())
    bits, cnt, idx = fp.build_block_mask_chunked(qp, kp, cb, alpha)
    torch.cuda.synchronize()
    gk = bits_to_keeps(bits, run)
    bad, ex, tot = mask_mismatches(gk, run)
    assert bad == 0, f"{bad} non-exempt mask mismatches of {tot}"
    assert ex <= max(2, tot // 1000)
    lk = lists_to_keeps(cnt, idx, run)
    for a_, b_ in zip(gk, lk):
        assert np.array_equal(a_, b_)
    # the TMA-fed mask (pooled keys pre-split by the pool kernel) gives the same lists
    bits2, cnt2, idx2 = fp.build_block_mask_chunked(qp, kp, cb, alpha, k_split=split)
    torch.cuda.synchronize()
    assert torch.equal(bits2, bits) and torch.equal(cnt2, cnt)
    for a_, b_ in zip(lk, lists_to_keeps(cnt2, idx2, run)):
        assert np.array_equal(a_, b_)


@pytest.mark.parametrize("name", list(CASES))
def test_chunked_attention_matches_oracle(name, cuda_device):
    inp, alpha = _inputs(name)
    w = inp.workload
    run = OracleRun(inp, alpha)
    rows = None
    if name == "long_prefix":
        rows = [(h, Ig) for h in range(w.Hq) for Ig in range(0, run.qoff[-1], 3)]
    ref, ref_lse = run.attention(rows=rows)
    cnt, idx = keep_to_lists(run.keeps, w.Hq)
    q, k, v, sc = device_inputs(inp, cuda_device)
    cb = _cb(inp, cuda_device)
    sentinel = torch.full((cb.total_q, w.Hq, w.d), 7.0, dtype=torch.bfloat16, device=cuda_device)
    out, lse = fp.sparse_prefill_attn_chunked(
        q, k, v, cnt.to(cuda_device), idx.to(cuda_device), cb, paged=_paged(inp, cuda_device),
        q_scale=sc["q_scale"], k_scale=sc["k_scale"], v_scale=sc["v_scale"], return_lse=True,
        out=sentinel)
    fp.check_status(cuda_device)
    amax, rel = attn_errors(out, ref)
    tol = TOL[w.dtype]
    assert amax <= tol[0] and rel <= tol[1], (amax, rel)
    dl = np.abs(lse.cpu().double().numpy() - ref_lse)
    assert np.nanmax(dl) <= (2e-3 if w.dtype == "bf16" else 3e-2)
    if rows is None:
        # every query row was written (no row of the chunk is left at the sentinel)
        assert not bool((out == 7.0).all(dim=-1).any())


def test_whole_requests_equal_plain_prefill(cuda_device):
    """q_len = kv_len for every request: the chunked calls compute what the plain calls do,
    bit for bit (same blocks, same lists, same tiles)."""
    w = dataclasses.replace(BASE, structure="band")
    kv = (1000, 129, 640)
    inp = S.make_inputs(w, seed=4, seqlens=kv, q_lens=kv)
    q, k, v, _ = device_inputs(inp, cuda_device)
    cb = fp.ChunkedBatch.make(kv, kv, w.block, cuda_device)
    b = fp.Batch.make(kv, w.block, cuda_device)
    qp, kp = fp.pool_qk_chunked(q, k, cb)
    qp0, kp0 = fp.pool_qk(q, k, w.block, batch=b)
    bits, cnt, idx = fp.build_block_mask_chunked(qp, kp, cb, 0.1)
    bits0, cnt0, idx0 = fp.build_block_mask(qp0, kp0, 0.1, block=w.block, batch=b)
    out, lse = fp.sparse_prefill_attn_chunked(q, k, v, cnt, idx, cb, return_lse=True)
    out0, lse0 = fp.sparse_prefill_attn(q, k, v, cnt0, idx0, w.block, batch=b, return_lse=True)
    fp.check_status(cuda_device)
    assert torch.equal(qp, qp0) and torch.equal(kp, kp0)
    assert torch.equal(bits, bits0) and torch.equal(cnt, cnt0)
    for h in range(w.Hq):
        for g in range(cb.total_qblocks):
            n = int(cnt[h, g])
            assert torch.equal(idx[h, g, :n], idx0[h, g, :n])
    assert torch.equal(out, out0) and torch.equal(lse, lse0)


def test_chunk_rows_equal_full_prefill_rows_when_dense(cuda_device):
    """alpha = 0 keeps every causal block: a chunk's rows then see exactly the keys they see in
    a full prefill of the same request, in the same tiles, so the outputs agree bit for bit."""
    w = dataclasses.replace(BASE, structure="band", q_lens=None)
    kv, ql = (1000, 700), (333, 128)
    full = S.make_inputs(w, seed=5, seqlens=kv)
    q, k, v, _ = device_inputs(full, cuda_device)
    out0, lse0, _, _ = fp.sparse_prefill(q, k, v, 0.0, w.block,
                                         batch=fp.Batch.make(kv, w.block, cuda_device),
                                         return_lse=True)
    rows = torch.cat([torch.arange(kv[0] - ql[0], kv[0]),
                      kv[0] + torch.arange(kv[1] - ql[1], kv[1])]).to(cuda_device)
    qc = q[rows].contiguous()
    cb = fp.ChunkedBatch.make(ql, kv, w.block, cuda_device)
    out, lse, _, _ = fp.sparse_prefill_chunked(qc, k, v, cb, 0.0, return_lse=True)
    fp.check_status(cuda_device)
    assert torch.equal(out, out0[rows]) and torch.equal(lse, lse0[:, rows])


def test_chunked_argument_errors(cuda_device):
    q = torch.zeros((10, 4, 128), dtype=torch.bfloat16, device=cuda_device)
    k = torch.zeros((5, 2, 128), dtype=torch.bfloat16, device=cuda_device)
    cb = fp.ChunkedBatch.make((10,), (5 + 5,), 128, cuda_device)
    bad = dataclasses.replace(cb, total_k=5)   # more queries than keys
    with pytest.raises(fp.FpError) as e:
        fp.pool_qk_chunked(q, k, bad)
    assert e.value.code == -1
    with pytest.raises(ValueError):
        fp.ChunkedBatch.make((11,), (10,), 128, cuda_device)


def _chunk_rows(inp):
    """Host rows of K and V at each request's new (chunk) positions, in request order."""
    w = inp.workload
    cu = inp.cu_seqlens.tolist()
    idx = torch.cat([torch.arange(cu[b] + L - n, cu[b] + L)
                     for b, (n, L) in enumerate(zip(w.q_lens, w.seqlens))])
    return inp.k[idx].contiguous(), inp.v[idx].contiguous()


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_append_writes_chunk_rows_into_the_paged_cache(dtype, cuda_device):
    """The append kernel writes the chunk's K/V rows exactly where the full cache has them,
    and nothing else; the chunked prefill on the appended cache equals the one on the full
    cache bit for bit."""
    w = dataclasses.replace(BASE, page_size=64, dtype=dtype)
    inp = S.make_inputs(w, seed=12, seqlens=(1000, 700, 300, 129), q_lens=(333, 700, 65, 1))
    w = inp.workload
    cb = _cb(inp, cuda_device)
    full = _paged(inp, cuda_device)
    # a cache holding the prefixes only: every chunk slot cleared
    k_cache, v_cache = full.k_cache.clone(), full.v_cache.clone()
    P = w.page_size
    for b, (n, L) in enumerate(zip(w.q_lens, w.seqlens)):
        for p in range(L - n, L):
            page = int(inp.page_table[b, p // P])
            k_cache.view(torch.uint8)[page, p % P].zero_()
            v_cache.view(torch.uint8)[page, p % P].zero_()
    kn, vn = _chunk_rows(inp)
    cache = fp.PagedKV(k_cache, v_cache, full.page_table)
    fp.append_paged_kv(kn.to(cuda_device), vn.to(cuda_device), cb, cache)
    fp.check_status(cuda_device)
    assert torch.equal(k_cache.view(torch.uint8), full.k_cache.view(torch.uint8))
    assert torch.equal(v_cache.view(torch.uint8), full.v_cache.view(torch.uint8))
    q, _, _, sc = device_inputs(inp, cuda_device)
    kw = dict(q_scale=sc["q_scale"], k_scale=sc["k_scale"], v_scale=sc["v_scale"])
    out_a, _, _, _ = fp.sparse_prefill_chunked(q, None, None, cb, 0.5, paged=cache, **kw)
    out_b, _, _, _ = fp.sparse_prefill_chunked(q, None, None, cb, 0.5, paged=full, **kw)
    fp.check_status(cuda_device)
    assert torch.equal(out_a, out_b)


def test_append_reports_a_bad_page_entry(cuda_device):
    w = dataclasses.replace(BASE, page_size=64)
    inp = S.make_inputs(w, seed=13, seqlens=(300,), q_lens=(100,))
    cb = _cb(inp, cuda_device)
    full = _paged(inp, cuda_device)
    pt = full.page_table.clone()
    pt[0, 299 // 64] = 10 ** 6          # the page of the last rows points past the cache
    kn, vn = _chunk_rows(inp)
    before = full.k_cache.clone()
    fp.append_paged_kv(kn.to(cuda_device), vn.to(cuda_device), cb,
                       fp.PagedKV(full.k_cache, full.v_cache, pt))
    with pytest.raises(fp.FpError) as e:
        fp.check_status(cuda_device)
    assert e.value.code == -5
    # rows whose page is valid were written (with the values they already had)
    assert torch.equal(full.k_cache, before)


@pytest.mark.parametrize("name", ["paged", "fp8_paged"])
def test_paged_output_layout_equals_the_contiguous_output(name, cuda_device):
    """FP_OUT_PAGED: the attention epilogue writes each new query's output row into the K/V
    caches' page layout (slot p % page_size of page page_table[b, p // page_size]). Gathered
    back through the page table on the host, it equals the contiguous output bit for bit,
    slots that hold no new query stay as they were, and lse is unchanged."""
    if name == "fp8_paged":
        w = dataclasses.replace(BASE, page_size=64, dtype="e4m3")
        inp = S.make_inputs(w, seed=13, seqlens=(1100, 600, 257), q_lens=(450, 600, 64))
    else:
        inp, _ = _inputs(name)
    w = inp.workload
    q, _, _, sc = device_inputs(inp, cuda_device)
    cb = _cb(inp, cuda_device)
    paged = _paged(inp, cuda_device)
    kw = dict(q_scale=sc["q_scale"], k_scale=sc["k_scale"], v_scale=sc["v_scale"])
    qp, kp = fp.pool_qk_chunked(q, None, cb, q_scale=sc["q_scale"], k_scale=sc["k_scale"],
                                paged=paged)
    _, cnt, idx = fp.build_block_mask_chunked(qp, kp, cb, 0.5, mask_bits=False)
    out, lse = fp.sparse_prefill_attn_chunked(q, None, None, cnt, idx, cb, paged=paged,
                                              return_lse=True, **kw)
    pages = torch.full((paged.k_cache.shape[0], paged.page_size, w.Hq, w.d), 5.0,
                       dtype=torch.bfloat16, device=cuda_device)
    out_p, lse_p = fp.sparse_prefill_attn_chunked(q, None, None, cnt, idx, cb, paged=paged,
                                                  return_lse=True, out=pages, out_paged=True,
                                                  **kw)
    fp.check_status(cuda_device)
    assert out_p.data_ptr() == pages.data_ptr()
    assert torch.equal(lse_p, lse)
    pt = inp.page_table
    ps = paged.page_size
    written = torch.zeros(pages.shape[:2], dtype=torch.bool)
    cu_q = inp.cu_q.tolist()
    for b, (n, L) in enumerate(zip(w.q_lens, w.seqlens)):
        pos = torch.arange(L - n, L)
        slots = pt[b, pos // ps].long() * ps + pos % ps
        got = pages.view(-1, w.Hq, w.d)[slots.to(cuda_device)]
        assert torch.equal(got, out[cu_q[b]:cu_q[b + 1]])
        written.view(-1)[slots] = True
    rest = pages.view(-1, w.Hq, w.d)[~written.view(-1).to(cuda_device)]
    assert bool((rest == 5.0).all())


@pytest.mark.parametrize("name", ["mixed", "paged", "fp8", "b64_d64", "gqa3", "gqa5", "mha",
                                  "long_prefix", "paged_out"])
def test_query_block_pairing_gives_the_same_output(name, cuda_device):
    """FP_PAIR_QBLOCKS: every CTA runs one head over two neighbouring query blocks (both tiles
    read each KV block they both kept once) instead of two heads of a GQA group at one query
    block. Each tile still accumulates its own kept blocks in ascending order with the same
    instructions, so out and lse equal the default split's bit for bit, for pairs inside a
    request and across request boundaries, contiguous or paged K/V, bf16 or e4m3."""
    inp, alpha = _inputs("paged" if name == "paged_out" else name)
    q, k, v, sc = device_inputs(inp, cuda_device)
    cb = _cb(inp, cuda_device)
    paged = _paged(inp, cuda_device)
    kw = dict(q_scale=sc["q_scale"], k_scale=sc["k_scale"], v_scale=sc["v_scale"],
              return_lse=True, paged=paged)
    kk, vv = (None, None) if paged is not None else (k, v)
    qp, kp = fp.pool_qk_chunked(q, kk, cb, q_scale=sc["q_scale"], k_scale=sc["k_scale"],
                                paged=paged)
    _, cnt, idx = fp.build_block_mask_chunked(qp, kp, cb, alpha, mask_bits=False)
    out_paged = name == "paged_out"
    outs = []
    for pair in (False, True):
        out = None
        if out_paged:
            out = torch.full((paged.k_cache.shape[0], paged.page_size, q.shape[1], q.shape[2]),
                             5.0, dtype=torch.bfloat16, device=cuda_device)
        outs.append(fp.sparse_prefill_attn_chunked(q, kk, vv, cnt, idx, cb, out=out,
                                                   out_paged=out_paged, pair_qblocks=pair,
                                                   **kw))
    fp.check_status(cuda_device)
    (o0, l0), (o1, l1) = outs
    assert torch.equal(o0, o1)
    assert torch.equal(l0, l1)
