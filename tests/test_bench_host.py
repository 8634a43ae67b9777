"""Host-side accounting of bench.py: query blocks, work counts and bytes agree with the
definitions the oracle uses (no GPU)."""
import numpy as np
import torch

import oracle as O
from block_sparse_long_qk_b200 import synthetic as S

import bench


def test_query_blocks_match_the_oracle():
    for name in ("llama128k", "paged", "chunked"):
        w = S.WORKLOADS[name]
        cu_k = np.concatenate([[0], np.cumsum(w.seqlens)]).astype(int)
        q_lens = w.q_lens if w.q_lens is not None else w.seqlens
        cu_q = np.concatenate([[0], np.cumsum(q_lens)]).astype(int)
        info, off = O.query_blocks(cu_q, cu_k if w.q_lens is not None else None, w.block)
        I, lo, hi = bench._query_blocks(w)
        assert len(I) == off[-1]
        exp_I = [i0 + i for (_, i0, nq) in info for i in range(nq)]
        assert I.tolist() == exp_I
        assert int((hi - lo).sum()) == int(sum(q_lens))


def test_work_counts_dense_closed_form():
    """With every causal block kept, the algorithmic FLOPs are 4 d times the number of causal
    (query, key) pairs, L (L + 1) / 2 per head for one sequence."""
    w = S.Workload("t", (1000,), 4, 2, 64, 128)
    nq = (1000 + 127) // 128
    cnt = torch.tensor([[I + 1 for I in range(nq)]] * w.Hq, dtype=torch.int32)
    alg, executed, density = bench.work_counts(w, cnt, None)
    assert alg == 4.0 * w.d * w.Hq * (1000 * 1001 // 2)
    assert executed == 4.0 * 128 * 128 * w.d * float(cnt.sum())
    assert density == 1.0


def test_pool_mask_bytes():
    w = S.WORKLOADS["llama128k"]
    pool, total = bench.pool_mask_bytes(w)
    assert pool == 131072 * (32 + 8) * 128 * 2 + (1024 * 32 + 1024 * 8) * 128 * 4 + 1024 * 8 * 128 * 4
    assert total - pool == (1024 * 32 + 1024 * 8) * 128 * 4 + 1024 * 8 * 128 * 4


def test_head_pairs_share_more_kept_blocks_than_query_block_pairs():
    """The attention CTA pairs the two query heads of a GQA group at one query block; the
    QUILT-style alternative pairs two neighbouring query blocks of one head. The kernel's steps
    and K/V loads are one per block in the union of the pair's kept lists, so the pairing with
    the smaller union does less work. On the 128K recipe (at 16K tokens here; 4.1 % at 128K)
    the head pairs' union is several percent smaller."""
    import dataclasses
    from _parity import OracleRun
    w = dataclasses.replace(S.WORKLOADS["llama128k"], seqlens=(16384,))
    K = OracleRun(S.make_inputs(w, seed=31), w.alpha).keeps[0]       # [Hq, nq, nk]
    Hq, nq, _ = K.shape
    head_union = sum(int((K[h] | K[h + 1]).sum()) for h in range(0, Hq, 2))
    qblk_union = sum(int((K[h, i] | K[h, i - 1]).sum()) for h in range(Hq)
                     for i in range(nq - 1, 0, -2))
    assert nq % 2 == 0
    assert qblk_union > 1.02 * head_union
    assert head_union < 0.51 * int(K.sum())      # the two heads' lists nearly coincide


def test_every_full_size_workload_has_a_traffic_figure():
    """bench.py reports the attention kernel's measured DRAM bytes per launch as
    roofline.traffic; every workload bench.py can run at full size has its figure (the tiny
    layer fits in L2 and reports none)."""
    import json
    import os
    with open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                           "profiles", "attn_traffic.json")) as f:
        traffic = json.load(f)
    for name in S.WORKLOADS:
        if name == "tiny":
            continue
        assert name in traffic and traffic[name] > 0, name
