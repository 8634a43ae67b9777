"""The binding's host-side checks of tensor shapes and dtypes (no GPU needed).

The C ABI receives pointers and sizes only, so a tensor smaller than the sizes the other
arguments imply would be read or written past its end by a kernel. The binding refuses such
calls before anything reaches the library. Correct calls made here with host tensors get past
every check and stop at the refusal of host memory, which shows that the checks accept them.
"""
import dataclasses

import pytest
import torch

import block_sparse_long_qk_b200 as fp

T, HQ, HKV, D, B = 256, 4, 2, 128, 128
WS = torch.zeros(256, dtype=torch.uint8)


def _qkv(dtype=torch.bfloat16, t=T):
    return (torch.zeros((t, HQ, D), dtype=dtype), torch.zeros((t, HKV, D), dtype=dtype),
            torch.zeros((t, HKV, D), dtype=dtype))


def _lists(nblk=2, mb=2):
    return (torch.zeros((HQ, nblk), dtype=torch.int32),
            torch.zeros((HQ, nblk, mb), dtype=torch.int32))


def _reaches_library(fn):
    with pytest.raises(ValueError, match="CUDA tensor"):
        fn()


def test_correct_calls_pass_every_check():
    q, k, v = _qkv()
    cnt, idx = _lists()
    _reaches_library(lambda: fp.pool_qk(q, k, B))
    _reaches_library(lambda: fp.pool_qk(q, k, B, k_split_out=torch.empty(
        fp.k_split_shape(HKV, 2, D), dtype=torch.bfloat16)))
    qp, kp = torch.zeros((HQ, 2, D)), torch.zeros((HKV, 2, D))
    _reaches_library(lambda: fp.build_block_mask(qp, kp, 0.1, block=B))
    _reaches_library(lambda: fp.sparse_prefill_attn(q, k, v, cnt, idx, B, ws=WS))
    _reaches_library(lambda: fp.sparse_prefill_attn(
        q, k, v, cnt, idx, B, ws=WS, out=torch.empty((T, HQ, D), dtype=torch.bfloat16)))
    e4 = torch.float8_e4m3fn
    q8, k8, v8 = _qkv(e4)
    _reaches_library(lambda: fp.sparse_prefill_attn(
        q8, k8, v8, cnt, idx, B, ws=WS, q_scale=torch.ones(HQ), k_scale=torch.ones(HKV),
        v_scale=torch.ones(HKV)))


@pytest.mark.parametrize("case,err,msg", [
    ("k_rows", ValueError, "k: expected shape"),
    ("v_dim", ValueError, "v: expected shape"),
    ("cnt_dtype", TypeError, "kv_cnt: expected dtype"),
    ("idx_small", ValueError, "kv_idx: expected at least"),
    ("out_dtype", TypeError, "out: expected dtype"),
    ("out_shape", ValueError, "out: expected shape"),
    ("q_scale_len", ValueError, "q_scale: expected shape"),
    ("k_scale_dtype", TypeError, "k_scale: expected dtype"),
    ("batch_tokens", ValueError, "the batch holds 200 tokens"),
    ("heads", ValueError, "not a multiple"),
    ("q_rank", ValueError, "q: expected"),
])
def test_attention_refuses_mismatched_tensors(case, err, msg):
    e4 = case in ("q_scale_len", "k_scale_dtype")
    q, k, v = _qkv(torch.float8_e4m3fn if e4 else torch.bfloat16)
    cnt, idx = _lists()
    kw = dict(ws=WS)
    if e4:
        kw.update(q_scale=torch.ones(HQ), k_scale=torch.ones(HKV), v_scale=torch.ones(HKV))
    if case == "k_rows":
        k = k[:-1].contiguous()
    elif case == "v_dim":
        v = torch.zeros((T, HKV, 64), dtype=v.dtype)
    elif case == "cnt_dtype":
        cnt = cnt.long()
    elif case == "idx_small":
        idx = idx[:, :, :1].contiguous()
    elif case == "out_dtype":
        kw["out"] = torch.empty((T, HQ, D), dtype=torch.float32)
    elif case == "out_shape":
        kw["out"] = torch.empty((T - 1, HQ, D), dtype=torch.bfloat16)
    elif case == "q_scale_len":
        kw["q_scale"] = torch.ones(HQ - 1)
    elif case == "k_scale_dtype":
        kw["k_scale"] = torch.ones(HKV, dtype=torch.float64)
    elif case == "batch_tokens":
        kw["batch"] = fp.Batch.make((200,), B, "cpu")
    elif case == "heads":
        q = torch.zeros((T, 3, D), dtype=q.dtype)
    elif case == "q_rank":
        q = q.reshape(T, HQ * D)
    with pytest.raises(err, match=msg):
        fp.sparse_prefill_attn(q, k, v, cnt, idx, B, **kw)


def test_pool_and_mask_refuse_mismatched_tensors():
    q, k, _ = _qkv()
    with pytest.raises(ValueError, match="k_split_out: expected shape"):
        fp.pool_qk(q, k, B, k_split_out=torch.empty((2, HKV, 3, D), dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="expected head dim"):
        fp.pool_qk(q, torch.zeros((T, HKV, 64), dtype=q.dtype), B)
    qp, kp = torch.zeros((HQ, 2, D)), torch.zeros((HKV, 3, D))
    with pytest.raises(ValueError, match="k_pool: expected shape"):
        fp.build_block_mask(qp, kp, 0.1, block=B)
    with pytest.raises(TypeError, match="q_pool: expected dtype"):
        fp.build_block_mask(qp.double(), kp[:, :2].contiguous(), 0.1, block=B)
    b = fp.Batch.make((200, 300), B, "cpu")            # 2 + 3 blocks
    with pytest.raises(ValueError, match="the batch holds 5 blocks"):
        fp.build_block_mask(qp, kp[:, :2].contiguous(), 0.1, block=B, batch=b)


def _paged(pages=8, page=64, rows=1, dtype=torch.bfloat16, pt_dtype=torch.int32):
    return fp.PagedKV(torch.zeros((pages, page, HKV, D), dtype=dtype),
                      torch.zeros((pages, page, HKV, D), dtype=dtype),
                      torch.zeros((rows, 4), dtype=pt_dtype))


def test_paged_calls_check_caches_and_page_table():
    q, _, _ = _qkv()
    b = fp.Batch.make((T,), B, "cpu")
    cnt, idx = _lists()
    _reaches_library(lambda: fp.sparse_prefill_attn_paged(q, _paged(), cnt, idx, b, ws=WS))
    _reaches_library(lambda: fp.pool_qk(q, None, B, paged=_paged()))
    with pytest.raises(TypeError, match="page_table: expected dtype"):
        fp.sparse_prefill_attn_paged(q, _paged(pt_dtype=torch.int64), cnt, idx, b, ws=WS)
    b2 = fp.Batch.make((128, 128), B, "cpu")
    with pytest.raises(ValueError, match="page_table: expected"):
        fp.sparse_prefill_attn_paged(q, _paged(rows=1), cnt, idx, b2, ws=WS)
    bad_v = dataclasses.replace(_paged(), v_cache=torch.zeros((7, 64, HKV, D),
                                                              dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="v_cache: expected shape"):
        fp.sparse_prefill_attn_paged(q, bad_v, cnt, idx, b, ws=WS)
    with pytest.raises(ValueError, match="k_cache: expected head dim"):
        fp.pool_qk(q, None, B, paged=fp.PagedKV(torch.zeros((8, 64, HKV * D)),
                                                 torch.zeros((8, 64, HKV * D)),
                                                 torch.zeros((1, 4), dtype=torch.int32)))


def test_chunked_calls_check_rows_against_the_batch():
    cb = fp.ChunkedBatch.make((100, 50), (300, 200), B, "cpu")
    q = torch.zeros((150, HQ, D), dtype=torch.bfloat16)
    k = torch.zeros((500, HKV, D), dtype=torch.bfloat16)
    cnt, idx = _lists(cb.total_qblocks, cb.max_kblocks)
    _reaches_library(lambda: fp.pool_qk_chunked(q, k, cb))
    _reaches_library(lambda: fp.sparse_prefill_attn_chunked(q, k, k, cnt, idx, cb, ws=WS))
    with pytest.raises(ValueError, match="the batch holds 150 queries"):
        fp.pool_qk_chunked(q[:149].contiguous(), k, cb)
    with pytest.raises(ValueError, match="k: expected shape"):
        fp.sparse_prefill_attn_chunked(q, k[:499].contiguous(), k, cnt, idx, cb, ws=WS)
    with pytest.raises(ValueError, match="kv_idx: expected at least"):
        fp.sparse_prefill_attn_chunked(q, k, k, cnt, idx[:, :, :1].contiguous(), cb, ws=WS)
    qp = torch.zeros((HQ, cb.total_qblocks + 1, D))
    with pytest.raises(ValueError, match="query blocks but q_pool"):
        fp.build_block_mask_chunked(qp, torch.zeros((HKV, cb.total_kblocks, D)), cb)


def test_append_checks_rows_and_heads():
    cb = fp.ChunkedBatch.make((100,), (300,), B, "cpu")
    kn = torch.zeros((100, HKV, D), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="100 new rows"):
        fp.append_paged_kv(kn[:99].contiguous(), kn[:99].contiguous(), cb, _paged(), ws=WS)
    with pytest.raises(ValueError, match="KV heads"):
        fp.append_paged_kv(kn[:, :1].contiguous(), kn[:, :1].contiguous(), cb, _paged(), ws=WS)
    _reaches_library(lambda: fp.append_paged_kv(kn, kn, cb, _paged(), ws=WS))
