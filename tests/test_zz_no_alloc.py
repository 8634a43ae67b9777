"""fp_pool_and_mask_noalloc against the regular two calls, through the C ABI.

The no-allocation entry exists for callers that cannot allocate device memory while they run
(for example a serving engine whose free HBM all belongs to its KV-cache pool, or code that
must not pay the device synchronisation of cudaMalloc). It keeps the pooled means in a static
device array of the library instead of caller buffers. Here it must produce exactly the block
mask and index lists that fp_pool_qk + fp_build_block_mask produce (integer results: bit for
bit), on two calls in a row with different shapes, so that nothing left in the shared array
by the first call leaks into the second. This file is collected last on purpose.
"""
import ctypes
import dataclasses

import pytest
import torch

import block_sparse_long_qk_b200 as fp
from block_sparse_long_qk_b200 import synthetic as S

pytestmark = pytest.mark.gpu

_p = ctypes.c_void_p


def _ptr(t):
    return None if t is None else _p(t.data_ptr())


def _noalloc_raw(inp, b, dev, alpha):
    """Calls the C entry point directly (no Python helper in between)."""
    w = inp.workload
    q = inp.q.to(dev)
    paged = w.page_size > 0
    kk = (inp.k_cache if paged else inp.k).to(dev)
    pt = inp.page_table.to(dev) if paged else None
    words = (b.max_blocks + 31) // 32
    bits = torch.zeros((w.Hq, b.total_blocks, words), dtype=torch.int32, device=dev)
    cnt = torch.full((w.Hq, b.total_blocks), -1, dtype=torch.int32, device=dev)
    idx = torch.full((w.Hq, b.total_blocks, b.max_blocks), -1, dtype=torch.int32, device=dev)
    cu, cb = (None, None) if (b.size == 1 and not paged) else (_ptr(b.cu_seqlens),
                                                               _ptr(b.cu_blocks))
    lib = fp.library()
    rc = lib.fp_pool_and_mask_noalloc(
        _ptr(q), _ptr(kk), 0, None, None, cu, cb, b.size, b.total_tokens, b.total_blocks,
        b.max_blocks, w.Hq, w.Hkv, w.d, w.block, _ptr(pt), w.page_size if paged else 0,
        pt.shape[1] if paged else 0, kk.shape[0] if paged else 0, float(alpha),
        float(w.d ** -0.5), fp.FORCE_FIRST | fp.FORCE_DIAG, _ptr(bits), _ptr(cnt), _ptr(idx),
        _p(torch.cuda.current_stream(dev).cuda_stream))
    assert rc == 0, lib.fp_last_error_string()
    return bits, cnt, idx


def _regular(inp, b, dev, alpha):
    w = inp.workload
    paged = None
    if w.page_size:
        paged = fp.PagedKV(inp.k_cache.to(dev), inp.v_cache.to(dev), inp.page_table.to(dev))
    qp, kp = fp.pool_qk(inp.q.to(dev), inp.k.to(dev), w.block, batch=b, paged=paged)
    return fp.build_block_mask(qp, kp, alpha, block=w.block, batch=b)


CALLS = [
    # one sequence, GQA, ragged tail
    (dataclasses.replace(S.WORKLOADS["llama128k"], Hq=8, Hkv=2), (5000,), 41, 0.1),
    # a paged varlen batch with other head counts and lengths (shape differs from call 1)
    (dataclasses.replace(S.WORKLOADS["paged"], Hq=4, Hkv=1, structure="iid"),
     (700, 129, 2100), 42, 0.5),
]


def test_noalloc_matches_regular_calls_twice_in_a_row(cuda_device):
    for w, seqlens, seed, alpha in CALLS:
        inp = S.make_inputs(w, seed=seed, seqlens=seqlens)
        b = fp.Batch.make(seqlens, w.block, cuda_device)
        ref_bits, ref_cnt, ref_idx = _regular(inp, b, cuda_device, alpha)
        bits, cnt, idx = _noalloc_raw(inp, b, cuda_device, alpha)
        torch.cuda.synchronize(cuda_device)
        assert torch.equal(bits, ref_bits)
        assert torch.equal(cnt, ref_cnt)
        n = ref_cnt.long()
        valid = torch.arange(b.max_blocks, device=cuda_device)[None, None, :] < n[:, :, None]
        assert torch.equal(idx[valid], ref_idx[valid])


def test_noalloc_rejects_problems_beyond_its_scratch(cuda_device):
    lib = fp.library()
    # (32 + 8) * 2048 blocks * 128 = 10.5 Mi floats > 8 Mi floats of static scratch
    rc = lib.fp_pool_and_mask_noalloc(
        _p(256), _p(256), 0, None, None, None, None, 1, 2048 * 128, 2048, 2048, 32, 8, 128, 128,
        None, 0, 0, 0, 0.1, 0.088, 3, None, _p(256), _p(256), None)
    assert rc == -1
    msg = lib.fp_last_error_string().decode()
    assert "static scratch" in msg and "32 MiB" in msg
