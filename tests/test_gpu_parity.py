"""GPU parity of the three kernels against the fp64 oracle (through the C ABI).

Every case draws seeded synthetic inputs, runs the CUDA path, and compares element by
element with the oracle on the same inputs: pooled means, the block mask (bit-identical
up to near-threshold blocks), and the attention output computed from the oracle's own keep
set (index lists written on the host from that set), so that no oracle input ever comes
from the CUDA path.
"""
import dataclasses
import math

import numpy as np
import pytest
import torch

import block_sparse_long_qk_b200 as fp
from block_sparse_long_qk_b200 import synthetic as S

from _parity import (TOL, OracleRun, attn_errors, bits_to_keeps, device_inputs, keep_to_lists,
                     lists_to_keeps, mask_mismatches, stratified_rows)

pytestmark = pytest.mark.gpu

W = S.WORKLOADS


def _case(name):
    """Small workloads: several tiles, ragged tails, every kernel variant."""
    base = W["llama32k"]
    cases = {
        "tiny": (W["tiny"], None, 0.1),
        "tiny_a09": (W["tiny"], None, 0.9),
        "gqa_ragged": (dataclasses.replace(base, Hq=8, Hkv=2, structure="band"), (1000,), 0.1),
        "gqa_ragged_a05": (dataclasses.replace(base, Hq=8, Hkv=2, structure="iid"), (1000,), 0.5),
        "varlen": (dataclasses.replace(base, Hq=8, Hkv=2, structure="iid"), (300, 129, 640), 0.5),
        "paged": (dataclasses.replace(W["paged"], Hq=8, Hkv=2, structure="iid"),
                  (300, 129, 640), 0.5),
        "fp8": (dataclasses.replace(W["fp8_128k"], Hq=8, Hkv=2, structure="iid"), (1000,), 0.5),
        "mha_d128": (dataclasses.replace(base, Hq=4, Hkv=4, structure="iid"), (700,), 0.5),
        "dense_alpha0": (dataclasses.replace(base, Hq=4, Hkv=2, structure="iid"), (600,), 0.0),
        "d128_b64": (dataclasses.replace(base, Hq=4, Hkv=2, block=64, structure="iid"),
                     (500,), 0.5),
        "d64_b128": (dataclasses.replace(base, Hq=4, Hkv=2, d=64, structure="iid"), (500,), 0.5),
        # more than 128 key blocks per row: several score chunks per pass in the mask kernel
        "long_ragged": (dataclasses.replace(W["llama128k"], Hq=8, Hkv=2), (20000,), 0.1),
        # mask CTAs whose rows straddle requests, several chunks
        "varlen_long": (dataclasses.replace(base, Hq=8, Hkv=2, structure="iid"),
                        (17000, 300, 9000), 0.5),
        # group of 8 query heads per KV head
        "gqa8": (dataclasses.replace(base, Hq=16, Hkv=2, structure="iid"), (3000,), 0.5),
        # groups of 3, 5 and 7: mask row tiles with idle rows (G does not divide 128), and
        # attention CTAs holding a pair of heads or a single one
        "gqa3": (dataclasses.replace(base, Hq=6, Hkv=2, structure="iid"), (1500,), 0.5),
        "gqa5": (dataclasses.replace(base, Hq=10, Hkv=2, structure="band"), (1300, 700), 0.1),
        "gqa7": (dataclasses.replace(base, Hq=7, Hkv=1, structure="band"), (1500,), 0.1),
        # i.i.d. twins of the two above: every causal block is kept (pooled logits of i.i.d.
        # inputs are ~0.01 apart), so the first query rows of a request attend to one or two
        # keys and their outputs are nearly single V rows (|o| up to ~3), where the bf16
        # output rounding alone reaches 0.0078
        "gqa5_iid": (dataclasses.replace(base, Hq=10, Hkv=2, structure="iid"), (1300, 700), 0.5),
        "gqa7_iid": (dataclasses.replace(base, Hq=7, Hkv=1, structure="iid"), (1500,), 0.5),
        # a request without tokens between two others (no blocks, no rows)
        "varlen_empty": (dataclasses.replace(base, Hq=8, Hkv=2, structure="iid"),
                         (300, 0, 129), 0.5),
        "paged_empty": (dataclasses.replace(W["paged"], Hq=8, Hkv=2, structure="iid"),
                        (0, 200, 0, 65), 0.5),
        # one query head per KV head (and below, an odd group): at these sizes each CTA runs a
        # single tile (query-block pairs, which straddle request boundaries in these length
        # mixes, are taken on problems of two waves or more: `mha128k` at full size, and the
        # FP_PAIR_QBLOCKS tests of test_gpu_chunked.py on small ones)
        "mha_varlen": (dataclasses.replace(base, Hq=2, Hkv=2, structure="iid"),
                       (300, 129, 640), 0.5),
        "mha_paged": (dataclasses.replace(W["paged"], Hq=2, Hkv=2, structure="iid"),
                      (300, 129, 640, 77), 0.5),
        "mha_fp8": (dataclasses.replace(W["fp8_128k"], Hq=3, Hkv=3, structure="iid"),
                    (300, 129, 640, 77), 0.5),
        "gqa3_varlen": (dataclasses.replace(base, Hq=6, Hkv=2, structure="band"),
                        (300, 129, 640, 77), 0.1),
    }
    w, seqlens, alpha = cases[name]
    return S.make_inputs(w, seed=7, seqlens=seqlens), alpha


SMALL = ["tiny", "tiny_a09", "gqa_ragged", "gqa_ragged_a05", "varlen", "paged", "fp8",
         "mha_d128", "dense_alpha0", "d128_b64", "d64_b128", "long_ragged", "varlen_long", "gqa8",
         "gqa3", "gqa5", "gqa7", "gqa5_iid", "gqa7_iid", "varlen_empty", "paged_empty", "mha_varlen",
         "mha_paged", "mha_fp8", "gqa3_varlen"]
# cases whose full fp64 attention would be slow: the oracle runs on every 5th query block
SAMPLED = {"long_ragged", "varlen_long"}


def _batch(inp, dev):
    return fp.Batch.make(inp.workload.seqlens, inp.workload.block, dev)


def _paged(inp, dev):
    if not inp.workload.page_size:
        return None
    return fp.PagedKV(inp.k_cache.to(dev), inp.v_cache.to(dev), inp.page_table.to(dev))


@pytest.mark.parametrize("name", SMALL)
def test_pool_and_mask_match_oracle(name, cuda_device):
    inp, alpha = _case(name)
    run = OracleRun(inp, alpha)
    q, k, v, sc = device_inputs(inp, cuda_device)
    b = _batch(inp, cuda_device)
    qp, kp = fp.pool_qk(q, k, inp.workload.block, batch=b, q_scale=sc["q_scale"],
                        k_scale=sc["k_scale"], paged=_paged(inp, cuda_device))
    torch.cuda.synchronize()
    for got, ref in ((qp, run.q_pool), (kp, run.k_pool)):
        g = got.cpu().double().numpy()
        assert np.abs(g - ref).max() <= 1e-5 * max(1.0, np.abs(ref).max())
    bits, cnt, idx = fp.build_block_mask(qp, kp, alpha, block=inp.workload.block, batch=b)
    torch.cuda.synchronize()
    gk = bits_to_keeps(bits, run)
    bad, ex, tot = mask_mismatches(gk, run)
    assert bad == 0, f"{bad} non-exempt mask mismatches of {tot}"
    assert ex <= max(2, tot // 1000)
    # the index lists say the same as the bits
    lk = lists_to_keeps(cnt, idx, run)
    for a_, b_ in zip(gk, lk):
        assert np.array_equal(a_, b_)
    # with the pool kernel's hi / lo split of k_pool (TMA-fed mask kernel) the results are the
    # same bits and lists
    split = torch.empty(fp.k_split_shape(inp.workload.Hkv, b.total_blocks, inp.workload.d),
                        dtype=torch.bfloat16, device=cuda_device)
    qp2, kp2 = fp.pool_qk(q, k, inp.workload.block, batch=b, q_scale=sc["q_scale"],
                          k_scale=sc["k_scale"], paged=_paged(inp, cuda_device), k_split_out=split)
    bits2, cnt2, idx2 = fp.build_block_mask(qp2, kp2, alpha, block=inp.workload.block, batch=b,
                                            k_split=split)
    torch.cuda.synchronize()
    assert torch.equal(qp2, qp) and torch.equal(kp2, kp)
    assert torch.equal(bits2, bits) and torch.equal(cnt2, cnt)
    for a_, b_ in zip(lk, lists_to_keeps(cnt2, idx2, run)):
        assert np.array_equal(a_, b_)


@pytest.mark.parametrize("name", SMALL)
def test_attention_matches_oracle(name, cuda_device):
    inp, alpha = _case(name)
    w = inp.workload
    run = OracleRun(inp, alpha)
    rows = None
    if name in SAMPLED:
        rows = [(h, Ig) for h in range(w.Hq) for Ig in range(0, run.off[-1], 5)]
    ref, ref_lse = run.attention(rows=rows)
    cnt, idx = keep_to_lists(run.keeps, w.Hq)
    q, k, v, sc = device_inputs(inp, cuda_device)
    b = _batch(inp, cuda_device)
    kw = dict(q_scale=sc["q_scale"], k_scale=sc["k_scale"], v_scale=sc["v_scale"],
              return_lse=True)
    if w.page_size:
        out, lse = fp.sparse_prefill_attn_paged(q, _paged(inp, cuda_device), cnt.to(cuda_device),
                                                idx.to(cuda_device), b, **kw)
    else:
        out, lse = fp.sparse_prefill_attn(q, k, v, cnt.to(cuda_device), idx.to(cuda_device),
                                          w.block, batch=b, **kw)
    fp.check_status(cuda_device)
    amax, rel = attn_errors(out, ref)
    tol = TOL[w.dtype]
    assert amax <= tol[0] and rel <= tol[1], (amax, rel)
    dl = np.abs(lse.cpu().double().numpy() - ref_lse)
    assert np.nanmax(dl) <= (2e-3 if w.dtype == "bf16" else 3e-2)


def test_skipped_blocks_are_never_read(cuda_device):
    """Physical skip: query blocks 3..7 do not keep KV blocks 1 and 2, whose K/V rows are then
    poisoned with NaN. Those query blocks' outputs stay finite and bit-identical."""
    w = dataclasses.replace(W["llama32k"], Hq=4, Hkv=2, structure="iid")
    inp = S.make_inputs(w, seed=3, seqlens=(1024,))
    keep = np.tril(np.ones((4, 8, 8), dtype=bool))
    keep[:, 3:, 1:3] = False
    cnt, idx = keep_to_lists([keep], 4)
    cnt, idx = cnt.to(cuda_device), idx.to(cuda_device)
    q, k, v, _ = device_inputs(inp, cuda_device)
    out0, _ = fp.sparse_prefill_attn(q, k, v, cnt, idx, 128)
    kp, vp = k.clone(), v.clone()
    kp[128:384] = float("nan")
    vp[128:384] = float("nan")
    out1, _ = fp.sparse_prefill_attn(q, kp, vp, cnt, idx, 128)
    torch.cuda.synchronize()
    assert torch.isfinite(out1[384:].float()).all()
    assert torch.equal(out0[384:], out1[384:])


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_lane_divergent_rescale(dtype, cuda_device):
    """Even query rows of the last block see a score jump of ~10 log2 units at KV block 2 (the
    running max is rescaled), odd rows do not: rows of one warp take different paths through
    the lazy O rescale and must still match the oracle."""
    L, d = 512, 128
    g = torch.Generator().manual_seed(9)
    q = torch.randn(L, 2, d, generator=g) * 0.1
    k = torch.randn(L, 1, d, generator=g) * 0.1
    v = torch.randn(L, 1, d, generator=g)
    u = torch.zeros(d)
    u[3] = 1.0
    k[256:384, 0] += 9.0 * u
    q[384::2, :] += 9.0 * u
    w = dataclasses.replace(W["llama32k"], Hq=2, Hkv=1, seqlens=(L,), dtype=dtype)
    inp = S.Inputs(w, q, k, v, torch.tensor([0, L], dtype=torch.int32))
    if dtype == "e4m3":
        inp.q, inp.q_scale = S.quantize_e4m3(q)
        inp.k, inp.k_scale = S.quantize_e4m3(k)
        inp.v, inp.v_scale = S.quantize_e4m3(v)
    else:
        inp.q, inp.k, inp.v = q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)
    run = OracleRun(inp, 0.0)        # every causal block kept, ascending order 0, 1, 2, 3
    ref, _ = run.attention()
    cnt, idx = keep_to_lists(run.keeps, 2)
    dq, dk, dv, sc = device_inputs(inp, cuda_device)
    out, _ = fp.sparse_prefill_attn(dq, dk, dv, cnt.to(cuda_device), idx.to(cuda_device), 128,
                                    q_scale=sc["q_scale"], k_scale=sc["k_scale"],
                                    v_scale=sc["v_scale"])
    fp.check_status(cuda_device)
    amax, rel = attn_errors(out, ref)
    tol = TOL[dtype]
    assert amax <= tol[0] and rel <= tol[1], (amax, rel)


def test_band_workload_16k(cuda_device):
    """The 128K recipe (vertical stripes + local band, alpha 0.1) at 16K tokens: realistic
    sparse lists whose two heads per CTA differ, many CTA waves, full pipeline."""
    w = dataclasses.replace(W["llama128k"], seqlens=(16384,))
    inp = S.make_inputs(w, seed=31)
    run = OracleRun(inp, w.alpha)
    q, k, v, _ = device_inputs(inp, cuda_device)
    b = _batch(inp, cuda_device)
    qp, kp = fp.pool_qk(q, k, w.block, batch=b)
    bits, cnt, idx = fp.build_block_mask(qp, kp, w.alpha, block=w.block, batch=b)
    out, _ = fp.sparse_prefill_attn(q, k, v, cnt, idx, w.block, batch=b)
    fp.check_status(cuda_device)
    gk = bits_to_keeps(bits, run)
    bad, ex, tot = mask_mismatches(gk, run)
    assert bad == 0 and ex <= max(4, tot // 10000), (bad, ex, tot)
    rows = [(h, I) for h in range(w.Hq) for I in range(0, 128, 9)
            if np.array_equal(gk[0][h, I], run.keeps[0][h, I])]
    ref, _ = run.attention(rows=rows)
    amax, rel = attn_errors(out, ref)
    assert amax <= TOL["bf16"][0] and rel <= TOL["bf16"][1], (amax, rel)


def test_bad_index_is_reported_not_read(cuda_device):
    w = dataclasses.replace(W["llama32k"], Hq=2, Hkv=1, structure="iid")
    inp = S.make_inputs(w, seed=4, seqlens=(512,))
    keep = np.tril(np.ones((2, 4, 4), dtype=bool))
    cnt, idx = keep_to_lists([keep], 2)
    idx[0, 1, 1] = 3   # a non-causal block for query block 1
    q, k, v, _ = device_inputs(inp, cuda_device)
    fp.sparse_prefill_attn(q, k, v, cnt.to(cuda_device), idx.to(cuda_device), 128)
    with pytest.raises(fp.FpError) as e:
        fp.check_status(cuda_device)
    assert e.value.code == -5
    fp.check_status(cuda_device)   # cleared


def test_pipeline_timeout_is_reported_and_cleared(cuda_device):
    """A K load that never arrives (test hook, first CTA only): the MMA issuer's bounded wait
    runs out, the status reads FP_ERR_TIMEOUT, the timeout is sticky until cleared, and the
    next call on the same context is correct again."""
    w = dataclasses.replace(W["llama32k"], Hq=2, Hkv=1, structure="iid")
    inp = S.make_inputs(w, seed=5, seqlens=(256,))
    keep = np.tril(np.ones((2, 2, 2), dtype=bool))
    cnt, idx = keep_to_lists([keep], 2)
    cnt, idx = cnt.to(cuda_device), idx.to(cuda_device)
    q, k, v, _ = device_inputs(inp, cuda_device)
    good, _ = fp.sparse_prefill_attn(q, k, v, cnt, idx, 128)
    fp.check_status(cuda_device)
    lib = fp.library()
    assert lib.fp_debug_skip_k_load(-1) == -1
    assert lib.fp_debug_skip_k_load(0) == 0
    fp.sparse_prefill_attn(q, k, v, cnt, idx, 128)
    # sticky: a launch on the same workspace before the check does no work at all
    sentinel = torch.full_like(good, 7.0)
    fp.sparse_prefill_attn(q, k, v, cnt, idx, 128, out=sentinel)
    torch.cuda.synchronize()
    assert bool((sentinel == 7.0).all())
    with pytest.raises(fp.FpError) as e:
        fp.check_status(cuda_device)
    assert e.value.code == -4
    # cleared by the check: the same call now completes and matches
    again, _ = fp.sparse_prefill_attn(q, k, v, cnt, idx, 128)
    fp.check_status(cuda_device)
    assert torch.equal(again, good)


def _full_size(name, cuda_device):
    inp = S.make_inputs(name)
    w = inp.workload
    run = OracleRun(inp, w.alpha)
    q, k, v, sc = device_inputs(inp, cuda_device)
    paged = _paged(inp, cuda_device)
    kw = dict(q_scale=sc["q_scale"], k_scale=sc["k_scale"], v_scale=sc["v_scale"])
    if run.chunked:
        cb = fp.ChunkedBatch.make(w.q_lens, w.seqlens, w.block, cuda_device)
        qp, kp = fp.pool_qk_chunked(q, k, cb, q_scale=sc["q_scale"], k_scale=sc["k_scale"],
                                    paged=paged)
        bits, cnt, idx = fp.build_block_mask_chunked(qp, kp, cb, w.alpha)
        out, _ = fp.sparse_prefill_attn_chunked(q, k, v, cnt, idx, cb, paged=paged, **kw)
    else:
        b = _batch(inp, cuda_device)
        qp, kp = fp.pool_qk(q, k, w.block, batch=b, q_scale=sc["q_scale"],
                            k_scale=sc["k_scale"], paged=paged)
        bits, cnt, idx = fp.build_block_mask(qp, kp, w.alpha, block=w.block, batch=b)
        if paged is not None:
            out, _ = fp.sparse_prefill_attn_paged(q, paged, cnt, idx, b, **kw)
        else:
            out, _ = fp.sparse_prefill_attn(q, k, v, cnt, idx, w.block, batch=b, **kw)
    fp.check_status(cuda_device)
    gk = bits_to_keeps(bits, run)
    bad, ex, tot = mask_mismatches(gk, run)
    assert bad == 0 and ex <= max(4, tot // 100000), (bad, ex, tot)
    rows = stratified_rows(run, gk, w.Hq, seed=11)
    assert len(rows) >= 15 * w.Hq, len(rows)
    ref, _ = run.attention(rows=rows)
    amax, rel = attn_errors(out, ref)
    tol = TOL[w.dtype]
    assert amax <= tol[0] and rel <= tol[1], (amax, rel)
    return run


@pytest.mark.parametrize("name", ["llama32k", "llama128k", "fp8_128k", "paged", "chunked",
                                  "mha128k"])
def test_full_size_workloads(name, cuda_device):
    _full_size(name, cuda_device)


@pytest.mark.parametrize("name", ["llama128k", "fp8_128k"])
def test_query_block_pairing_at_full_size(name, cuda_device):
    """The general work split (two neighbouring query blocks of one head per CTA, forced with
    FP_PAIR_QBLOCKS) on the full 128K GQA layers: the same output, bit for bit, as the default
    head-pair split that the full-size oracle comparison checks (16,384 CTAs, kept lists up to
    ~80 blocks per row)."""
    inp = S.make_inputs(name)
    w = inp.workload
    q, k, v, sc = device_inputs(inp, cuda_device)
    kw = dict(q_scale=sc["q_scale"], k_scale=sc["k_scale"], v_scale=sc["v_scale"],
              return_lse=True)
    b = _batch(inp, cuda_device)
    qp, kp = fp.pool_qk(q, k, w.block, batch=b, q_scale=sc["q_scale"], k_scale=sc["k_scale"])
    _, cnt, idx = fp.build_block_mask(qp, kp, w.alpha, block=w.block, batch=b, mask_bits=False)
    out, lse = fp.sparse_prefill_attn(q, k, v, cnt, idx, w.block, batch=b, **kw)
    T = q.shape[0]
    cb = fp.ChunkedBatch.make((T,), (T,), w.block, cuda_device)
    out_q, lse_q = fp.sparse_prefill_attn_chunked(q, k, v, cnt, idx, cb, pair_qblocks=True, **kw)
    fp.check_status(cuda_device)
    assert torch.equal(out, out_q)
    assert torch.equal(lse, lse_q)


def test_longest_sequence_512k(cuda_device):
    """One 524,288-token sequence (4,096 blocks per row): the largest single layer the tests
    run. Pooled means and the mask against the oracle in full, the attention on sampled rows."""
    w = dataclasses.replace(W["llama128k"], Hq=8, Hkv=2)
    inp = S.make_inputs(w, seed=19, seqlens=(524288,))
    run = OracleRun(inp, w.alpha)
    q, k, v, _ = device_inputs(inp, cuda_device)
    b = _batch(inp, cuda_device)
    qp, kp = fp.pool_qk(q, k, w.block, batch=b)
    bits, cnt, idx = fp.build_block_mask(qp, kp, w.alpha, block=w.block, batch=b)
    out, _ = fp.sparse_prefill_attn(q, k, v, cnt, idx, w.block, batch=b)
    fp.check_status(cuda_device)
    for got, ref in ((qp, run.q_pool), (kp, run.k_pool)):
        g = got.cpu().double().numpy()
        assert np.abs(g - ref).max() <= 1e-5 * max(1.0, np.abs(ref).max())
    gk = bits_to_keeps(bits, run)
    bad, ex, tot = mask_mismatches(gk, run)
    assert bad == 0 and ex <= max(4, tot // 100000), (bad, ex, tot)
    rows = stratified_rows(run, gk, w.Hq, seed=23)
    assert len(rows) >= 15 * w.Hq, len(rows)
    ref, _ = run.attention(rows=rows)
    amax, rel = attn_errors(out, ref)
    assert amax <= TOL["bf16"][0] and rel <= TOL["bf16"][1], (amax, rel)


def test_strided_views_and_host_prefix_sums_are_refused(cuda_device):
    q = torch.zeros((256, 4, 128), dtype=torch.bfloat16, device=cuda_device)
    k = torch.zeros((256, 2, 128), dtype=torch.bfloat16, device=cuda_device)
    with pytest.raises(ValueError, match="contiguous"):
        fp.pool_qk(q[:, :, :64], k[:, :, :64], 128)
    b = fp.Batch.make((200, 56), 128, cuda_device)
    host_b = dataclasses.replace(b, cu_seqlens=b.cu_seqlens.cpu().pin_memory().cuda(),
                                 cu_blocks=b.cu_blocks.cpu())
    with pytest.raises(ValueError, match="CUDA tensor"):
        fp.pool_qk(q, k, 128, batch=host_b)
    # at the C ABI: a host array is refused with a message, nothing is launched
    import numpy as np
    cu = np.array([0, 200, 256], dtype=np.int32)
    qp = torch.empty((4, 3, 128), device=cuda_device)
    kp = torch.empty((2, 3, 128), device=cuda_device)
    rc = fp.library().fp_pool_qk(fp._ptr(q), fp._ptr(k), 0, None, None, cu.ctypes.data,
                                 fp._ptr(b.cu_blocks), 2, 256, 3, 4, 2, 128, 128, None, 0, 0,
                                 0, fp._ptr(qp), fp._ptr(kp), None, None,
                                 fp._stream(q.device))
    assert rc == -1 and b"host memory" in fp.library().fp_last_error_string()
    torch.cuda.synchronize()


@pytest.mark.parametrize("name", ["tiny", "gqa3", "varlen", "gqa8"])
def test_fp32_mask_matches_oracle_and_tensor_core_mask(name, cuda_device):
    """FP_MASK_FP32 runs the fp32 FFMA scores: the same keep sets as the oracle (up to the
    near-threshold exemption), and as the tensor-core kernel away from the threshold."""
    inp, alpha = _case(name)
    run = OracleRun(inp, alpha)
    q, k, _, sc = device_inputs(inp, cuda_device)
    b = _batch(inp, cuda_device)
    qp, kp = fp.pool_qk(q, k, inp.workload.block, batch=b, q_scale=sc["q_scale"],
                        k_scale=sc["k_scale"], paged=_paged(inp, cuda_device))
    flags = fp.FORCE_FIRST | fp.FORCE_DIAG
    bits32, cnt32, idx32 = fp.build_block_mask(qp, kp, alpha, block=inp.workload.block, batch=b,
                                               flags=flags | fp.MASK_FP32)
    bits, _, _ = fp.build_block_mask(qp, kp, alpha, block=inp.workload.block, batch=b,
                                     flags=flags)
    torch.cuda.synchronize()
    g32 = bits_to_keeps(bits32, run)
    bad, ex, tot = mask_mismatches(g32, run)
    assert bad == 0 and ex <= max(2, tot // 1000), (bad, ex, tot)
    for a_, b_ in zip(g32, lists_to_keeps(cnt32, idx32, run)):
        assert np.array_equal(a_, b_)
    gtc = bits_to_keeps(bits, run)
    for r, (x, y, ratio) in enumerate(zip(g32, gtc, run.ratios)):
        near = np.abs(ratio - alpha) <= 1e-3 * alpha
        assert not ((x != y) & ~near).any()


@pytest.mark.parametrize("world", [2, 4])
def test_head_split_equals_whole_layer(world, cuda_device):
    """The multi-GPU head split (each rank the whole path on its KV-head groups, no exchange),
    run here slice after slice on one GPU: the slices' masks and outputs, put side by side,
    are the whole layer's bit for bit (every stage works per head, and a slice holds whole GQA
    groups, so the attention CTAs pair the same heads)."""
    import bench
    w = dataclasses.replace(W["llama128k"], Hq=16, Hkv=4)
    inp = S.make_inputs(w, seed=29, seqlens=(3000, 1700))
    dev = cuda_device
    b = _batch(inp, dev)
    q, k, v, _ = device_inputs(inp, dev)
    out, _, cnt, idx = fp.sparse_prefill(q, k, v, w.alpha, w.block, batch=b)
    outs, cnts = [], []
    for r in range(world):
        part = bench.shard_inputs(inp, r, world)
        pq, pk, pv, _ = device_inputs(part, dev)
        o, _, c, _ = fp.sparse_prefill(pq, pk, pv, w.alpha, w.block, batch=b)
        outs.append(o)
        cnts.append(c)
    fp.check_status(dev)
    assert torch.equal(torch.cat(outs, dim=1), out)
    assert torch.equal(torch.cat(cnts, dim=0), cnt)
