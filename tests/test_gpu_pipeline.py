"""The pipelined host-buffer API gives, step for step, exactly what the direct calls give."""
import dataclasses

import pytest
import torch

import block_sparse_long_qk_b200 as fp
from block_sparse_long_qk_b200 import synthetic as S

pytestmark = pytest.mark.gpu


def test_host_pipeline_matches_direct_calls(cuda_device):
    w = dataclasses.replace(S.WORKLOADS["llama32k"], Hq=8, Hkv=2, structure="band")
    seqlens = (1000, 129, 640)
    b = fp.Batch.make(seqlens, w.block, cuda_device)
    inputs = [S.make_inputs(w, seed=30 + i, seqlens=seqlens) for i in range(5)]

    def run(q, k, v, out):
        fp.sparse_prefill(q, k, v, 0.1, w.block, batch=b, out=out)

    host_in = [(x.q.pin_memory(), x.k.pin_memory(), x.v.pin_memory()) for x in inputs]
    host_out = [torch.empty(x.q.shape, dtype=torch.bfloat16).pin_memory() for x in inputs]
    pipe = fp.HostPipeline(run, host_in[0], host_out[0], cuda_device, depth=2)
    for hi, ho in zip(host_in, host_out):
        pipe.submit(hi, ho)
    pipe.synchronize()
    fp.check_status(cuda_device)
    for x, ho in zip(inputs, host_out):
        ref, _, _, _ = fp.sparse_prefill(x.q.to(cuda_device), x.k.to(cuda_device),
                                         x.v.to(cuda_device), 0.1, w.block, batch=b)
        torch.cuda.synchronize()
        assert torch.equal(ho, ref.cpu())
