"""Failure paths of the pool, mask, attention and append kernels on the GPU, made on the host: a
mask-operand load that is never issued (one-shot test hook) and prefix sums or page-table
entries that do not describe the batch. Each is reported through the caller's status word, none
is followed to an out-of-range access, the requests the fault does not touch keep their exact
results, and the context stays usable for the next call.
"""
import dataclasses

import pytest
import torch

import block_sparse_long_qk_b200 as fp
from block_sparse_long_qk_b200 import synthetic as S

pytestmark = pytest.mark.gpu

W = S.WORKLOADS


def _inputs(seqlens, seed, paged=False, q_lens=None):
    base = W["paged"] if paged else W["llama32k"]
    w = dataclasses.replace(base, Hq=8, Hkv=2, structure="iid")
    return S.make_inputs(w, seed=seed, seqlens=seqlens, q_lens=q_lens)


def _status(dev):
    """The status word's error code (0 if clean); reading it clears it."""
    try:
        fp.check_status(dev)
        return 0
    except fp.FpError as e:
        return e.code


def test_mask_timeout_is_reported_sticky_and_cleared(cuda_device):
    """A key-operand load of the mask kernel that never arrives: its bounded wait runs out, the
    status reads FP_ERR_TIMEOUT, a mask launch before the check does no work at all, and after
    the check the same call gives the clean results bit for bit."""
    dev = cuda_device
    inp = _inputs((1000,), 41)
    q, k = inp.q.to(dev), inp.k.to(dev)
    b = fp.Batch.make((1000,), 128, dev)
    split = torch.empty(fp.k_split_shape(2, b.total_blocks, 128), dtype=torch.bfloat16,
                        device=dev)
    qp, kp = fp.pool_qk(q, k, 128, batch=b, k_split_out=split)
    bits0, cnt0, idx0 = fp.build_block_mask(qp, kp, 0.5, block=128, batch=b, k_split=split)
    assert _status(dev) == 0
    lib = fp.library()
    assert lib.fp_debug_skip_mask_load(0) == 0
    fp.build_block_mask(qp, kp, 0.5, block=128, batch=b, k_split=split)
    # sticky: the next launch on the same workspace leaves its outputs untouched
    bits = torch.full_like(bits0, -7)
    cnt = torch.full_like(cnt0, -7)
    idx = torch.full_like(idx0, -7)
    rc = lib.fp_build_block_mask(
        fp._ptr(qp), fp._ptr(kp), fp._ptr(split), None, 1, b.total_blocks, b.max_blocks, 8, 2,
        128, 0.5, 128 ** -0.5, fp.FORCE_FIRST | fp.FORCE_DIAG, fp._ptr(bits), fp._ptr(cnt),
        fp._ptr(idx), fp._ptr(fp.workspace(dev)), fp._stream(dev))
    assert rc == 0
    torch.cuda.synchronize()
    assert bool((bits == -7).all()) and bool((cnt == -7).all()) and bool((idx == -7).all())
    assert _status(dev) == -4
    bits2, cnt2, idx2 = fp.build_block_mask(qp, kp, 0.5, block=128, batch=b, k_split=split)
    assert _status(dev) == 0
    assert torch.equal(bits2, bits0) and torch.equal(cnt2, cnt0)
    for h in range(8):
        for i in range(b.total_blocks):
            n = int(cnt0[h, i])
            assert torch.equal(idx2[h, i, :n], idx0[h, i, :n])


def _bad_blocks(good, dev):
    """Request 0 (300 tokens, 3 blocks) stays consistent; request 1 (129 tokens) claims 3 blocks
    and request 2 (640 tokens) 4, with the totals unchanged."""
    return dataclasses.replace(good, cu_blocks=torch.tensor([0, 3, 6, 10], dtype=torch.int32,
                                                            device=dev))


def test_pool_refuses_inconsistent_prefix_sums(cuda_device):
    dev = cuda_device
    seqlens = (300, 129, 640)
    inp = _inputs(seqlens, 43)
    q, k = inp.q.to(dev), inp.k.to(dev)
    good = fp.Batch.make(seqlens, 128, dev)
    qp0, kp0 = fp.pool_qk(q, k, 128, batch=good)
    assert _status(dev) == 0
    qp, kp = fp.pool_qk(q, k, 128, batch=_bad_blocks(good, dev))
    assert _status(dev) == -5
    assert torch.equal(qp[:, :3], qp0[:, :3]) and torch.equal(kp[:, :3], kp0[:, :3])
    # token prefix sums past the tokens passed, and a negative request length
    for cu in ([0, 300, 429, 1200], [0, 300, 200, 1069]):
        bad = dataclasses.replace(good, cu_seqlens=torch.tensor(cu, dtype=torch.int32,
                                                                device=dev))
        qp, kp = fp.pool_qk(q, k, 128, batch=bad)
        assert _status(dev) == -5
        assert torch.equal(qp[:, :3], qp0[:, :3])
    qp1, _ = fp.pool_qk(q, k, 128, batch=good)
    assert _status(dev) == 0 and torch.equal(qp1, qp0)


def test_mask_refuses_inconsistent_prefix_sums(cuda_device):
    """The mask call sees block prefix sums only (no token counts), so what it can check is
    that they ascend, stay within total_blocks and give no request more than max_blocks blocks
    (a longer request would overflow its index-list rows)."""
    dev = cuda_device
    seqlens = (300, 129, 640)
    inp = _inputs(seqlens, 44)
    q, k = inp.q.to(dev), inp.k.to(dev)
    good = fp.Batch.make(seqlens, 128, dev)
    qp, kp = fp.pool_qk(q, k, 128, batch=good)
    bits0, cnt0, _ = fp.build_block_mask(qp, kp, 0.5, block=128, batch=good)
    assert _status(dev) == 0
    for cb in ([0, 3, 4, 10],        # request 2 claims 6 blocks, max_blocks is 5
               [0, 3, 2, 10],        # decreasing
               [0, 3, 5, 11]):       # past total_blocks
        bad = dataclasses.replace(good, cu_blocks=torch.tensor(cb, dtype=torch.int32, device=dev))
        for flags in (fp.FORCE_FIRST | fp.FORCE_DIAG,
                      fp.FORCE_FIRST | fp.FORCE_DIAG | fp.MASK_FP32):
            fp.build_block_mask(qp, kp, 0.5, block=128, batch=bad, flags=flags)
            assert _status(dev) == -5, (cb, flags)
    bits1, cnt1, _ = fp.build_block_mask(qp, kp, 0.5, block=128, batch=good)
    assert _status(dev) == 0
    assert torch.equal(bits1, bits0) and torch.equal(cnt1, cnt0)


def test_attention_refuses_inconsistent_prefix_sums(cuda_device):
    dev = cuda_device
    seqlens = (300, 129, 640)
    inp = _inputs(seqlens, 45)
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    good = fp.Batch.make(seqlens, 128, dev)
    out0, _, cnt, idx = fp.sparse_prefill(q, k, v, 0.5, 128, batch=good)
    assert _status(dev) == 0
    out = torch.full_like(out0, 3.0)
    fp.sparse_prefill_attn(q, k, v, cnt, idx, 128, batch=_bad_blocks(good, dev), out=out)
    assert _status(dev) == -5
    assert torch.equal(out[:300], out0[:300])        # request 0 is unaffected
    assert bool((out[300:] == 3.0).all())            # the others are not written


def test_pool_reports_out_of_range_page_entries(cuda_device):
    dev = cuda_device
    inp = _inputs((300, 129), 46, paged=True)
    q = inp.q.to(dev)
    b = fp.Batch.make((300, 129), 128, dev)
    pt = inp.page_table.to(dev).clone()
    paged = fp.PagedKV(inp.k_cache.to(dev), inp.v_cache.to(dev), pt)
    _, kp0 = fp.pool_qk(q, None, 128, batch=b, paged=paged)
    assert _status(dev) == 0
    pt[0, 1] = -1                          # tokens 64..127 of request 0
    _, kp = fp.pool_qk(q, None, 128, batch=b, paged=paged)
    assert _status(dev) == -5
    assert torch.equal(kp[:, 1:], kp0[:, 1:])          # other blocks unchanged
    pt[0, 1] = paged.k_cache.shape[0]                  # one past the last page
    fp.pool_qk(q, None, 128, batch=b, paged=paged)
    assert _status(dev) == -5


def test_chunked_stages_refuse_inconsistent_prefix_sums(cuda_device):
    """Chunked batch whose query-block prefix sums disagree with the query and key rows: every
    stage reports FP_ERR_BAD_INDEX, and a consistent batch runs cleanly afterwards."""
    dev = cuda_device
    q_lens, kv_lens = (100, 50), (1000, 300)
    inp = _inputs(kv_lens, 47, q_lens=q_lens)
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    cb = fp.ChunkedBatch.make(q_lens, kv_lens, 128, dev)
    out0, _, cnt, idx = fp.sparse_prefill_chunked(q, k, v, cb, 0.5)
    assert _status(dev) == 0
    qb = cb.cu_qblocks.clone()
    qb[1] += 1                       # request 0 claims one query block too many
    bad = dataclasses.replace(cb, cu_qblocks=qb)
    qp, kp = fp.pool_qk_chunked(q, k, bad)
    assert _status(dev) == -5
    fp.build_block_mask_chunked(qp, kp, bad, 0.5)
    assert _status(dev) == -5
    fp.sparse_prefill_attn_chunked(q, k, v, cnt, idx, bad)
    assert _status(dev) == -5
    out1, _, _, _ = fp.sparse_prefill_chunked(q, k, v, cb, 0.5)
    assert _status(dev) == 0 and torch.equal(out1, out0)


def test_append_refuses_more_new_rows_than_keys(cuda_device):
    """A request that claims more new rows than it has keys: its rows are not written and the
    status reads FP_ERR_BAD_INDEX; the other request's rows land as usual."""
    dev = cuda_device
    q_lens, kv_lens = (100, 50), (1000, 300)
    inp = _inputs(kv_lens, 48, paged=True, q_lens=q_lens)
    cb = fp.ChunkedBatch.make(q_lens, kv_lens, 128, dev)
    kc = torch.zeros_like(inp.k_cache).to(dev)
    vc = torch.zeros_like(inp.v_cache).to(dev)
    paged = fp.PagedKV(kc, vc, inp.page_table.to(dev))
    k_new = torch.randn((150, 2, 128), device=dev).to(torch.bfloat16)
    v_new = torch.randn((150, 2, 128), device=dev).to(torch.bfloat16)
    ck = cb.cu_k.clone()
    ck[2] = ck[1] + 40               # request 1: 50 new rows but only 40 keys
    bad = dataclasses.replace(cb, cu_k=ck)
    fp.append_paged_kv(k_new, v_new, bad, paged)
    assert _status(dev) == -5
    torch.cuda.synchronize()
    pt = inp.page_table
    page_size = kc.shape[1]
    for r in (0, 99):                # request 0's rows: positions 900 .. 999
        p = 900 + r
        slot = int(pt[0, p // page_size]) * page_size + p % page_size
        row = kc.view(-1, 2, 128)[slot]
        assert torch.equal(row, k_new[r])
    assert int((vc.view(-1, 2, 128).float().abs().sum(dim=(1, 2)) > 0).sum()) == 100


def test_mask_timeout_stops_the_attention_of_the_same_step(cuda_device):
    """A step's calls share one workspace: after the mask kernel's wait ran out, its lists are
    incomplete, and the attention launch that follows on the same workspace does no work (its
    output buffer stays as it was) until fp_check_status reports the timeout and clears it."""
    dev = cuda_device
    inp = _inputs((640,), 49)
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    b = fp.Batch.make((640,), 128, dev)
    good, _, _, _ = fp.sparse_prefill(q, k, v, 0.5, 128, batch=b)
    assert _status(dev) == 0
    split = torch.empty(fp.k_split_shape(2, b.total_blocks, 128), dtype=torch.bfloat16,
                        device=dev)
    qp, kp = fp.pool_qk(q, k, 128, batch=b, k_split_out=split)
    assert fp.library().fp_debug_skip_mask_load(0) == 0
    _, cnt, idx = fp.build_block_mask(qp, kp, 0.5, block=128, batch=b, k_split=split)
    out = torch.full_like(good, 7.0)
    fp.sparse_prefill_attn(q, k, v, cnt, idx, 128, batch=b, out=out)
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())
    assert _status(dev) == -4
    again, _, _, _ = fp.sparse_prefill(q, k, v, 0.5, 128, batch=b)
    assert _status(dev) == 0 and torch.equal(again, good)
