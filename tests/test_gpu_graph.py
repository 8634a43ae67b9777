"""The path captures into a CUDA graph: replays on new data give exactly the eager results."""
import dataclasses

import pytest
import torch

import block_sparse_long_qk_b200 as fp
from block_sparse_long_qk_b200 import synthetic as S

pytestmark = pytest.mark.gpu


def test_plain_varlen_step_replays_bit_exact(cuda_device):
    w = dataclasses.replace(S.WORKLOADS["llama32k"], Hq=8, Hkv=2, structure="band")
    seqlens = (1000, 129, 640)
    b = fp.Batch.make(seqlens, w.block, cuda_device)
    xs = [S.make_inputs(w, seed=60 + i, seqlens=seqlens) for i in range(3)]
    q, k, v = (t.to(cuda_device) for t in (xs[0].q, xs[0].k, xs[0].v))

    def run(q, k, v):
        out, _, _, _ = fp.sparse_prefill(q, k, v, 0.1, w.block, batch=b)
        return out

    step = fp.GraphStep(run, (q, k, v))
    for x in xs[1:] + xs[:1]:
        for dst, src in zip(step.inputs, (x.q, x.k, x.v)):
            dst.copy_(src)
        got = step.replay().clone()
        ref = run(*(t.to(cuda_device) for t in (x.q, x.k, x.v)))
        torch.cuda.synchronize()
        assert torch.equal(got, ref)
    fp.check_status(cuda_device)


def test_chunked_paged_step_with_append_replays_bit_exact(cuda_device):
    w = dataclasses.replace(S.WORKLOADS["chunked"], Hq=8, Hkv=2, structure="band")
    kv, ql = (1000, 700, 300), (333, 700, 65)
    inp = S.make_inputs(w, seed=70, seqlens=kv, q_lens=ql)
    cb = fp.ChunkedBatch.make(ql, kv, w.block, cuda_device)
    cache = fp.PagedKV(inp.k_cache.to(cuda_device), inp.v_cache.to(cuda_device),
                       inp.page_table.to(cuda_device))
    cu = inp.cu_seqlens.tolist()
    rows = torch.cat([torch.arange(cu[b] + L - n, cu[b] + L)
                      for b, (n, L) in enumerate(zip(ql, kv))])
    kn, vn = inp.k[rows].to(cuda_device), inp.v[rows].to(cuda_device)
    q = inp.q.to(cuda_device)

    def run(q, kn, vn):
        fp.append_paged_kv(kn, vn, cb, cache)
        out, _, _, _ = fp.sparse_prefill_chunked(q, None, None, cb, 0.1, paged=cache)
        return out

    ref = run(q.clone(), kn.clone(), vn.clone()).clone()
    step = fp.GraphStep(run, (q, kn, vn))
    got = step.replay().clone()
    torch.cuda.synchronize()
    fp.check_status(cuda_device)
    assert torch.equal(got, ref)
