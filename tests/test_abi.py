"""The C-ABI library loads, exports every symbol its header declares, and rejects bad
arguments on the host before touching a GPU (no compute call here)."""
import ctypes

import pytest

import block_sparse_long_qk_b200 as fp


def test_library_exports_every_header_symbol():
    lib = fp.library()
    names = fp.header_symbols()
    assert "fp_pool_qk" in names and "fp_sparse_prefill_attn_paged" in names
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) <= set(fp._SIGNATURES), "binding lacks a signature for a header symbol"


def test_version_and_workspace():
    lib = fp.library()
    assert lib.fp_version() >= 100
    assert lib.fp_workspace_size() >= 4


def _bad_attn(**over):
    """Arguments of a well-formed single-sequence attention call with fake pointers; only
    host-side validation runs for the failing cases below."""
    a = dict(q=16, k=16, v=16, dtype=0, qs=None, ks=None, vs=None, cu=None, cb=None, batch=1,
             T=256, tb=2, mb=2, Hq=8, Hkv=2, d=128, block=128, scale=0.1, cnt=16, idx=16,
             out=16, lse=None, ws=256, stream=None)
    a.update(over)
    lib = fp.library()
    return lib.fp_sparse_prefill_attn(*[a[k] for k in (
        "q", "k", "v", "dtype", "qs", "ks", "vs", "cu", "cb", "batch", "T", "tb", "mb", "Hq",
        "Hkv", "d", "block", "scale", "cnt", "idx", "out", "lse", "ws", "stream")])


@pytest.mark.parametrize("over,code", [
    (dict(dtype=7), -1),             # unknown dtype
    (dict(Hq=6, Hkv=4), -1),         # Hq not a multiple of Hkv
    (dict(d=96), -2),                # unsupported head dim
    (dict(block=32), -2),            # unsupported block
    (dict(tb=3), -1),                # total_blocks != ceil(T / block)
    (dict(q=8), -1),                 # misaligned pointer
    (dict(ws=128), -1),              # misaligned workspace
    (dict(dtype=1), -1),             # e4m3 without scales
    (dict(batch=2), -1),             # varlen without cu arrays
])
def test_attention_rejects_bad_arguments(over, code):
    assert _bad_attn(**over) == code
    assert fp.library().fp_last_error_string()


@pytest.mark.parametrize("over,code,msg", [
    (dict(qs=16), -1, b"no scales"),                  # bf16 with a scale pointer
    (dict(cu=16), -1, b"both given or both NULL"),    # one prefix-sum array without the other
    (dict(T=-1, tb=0, mb=0), -1, b"negative"),
    (dict(mb=3), -1, b"max_blocks must equal"),       # one sequence: max_blocks = total_blocks
    (dict(Hq=0), -1, b"multiple of Hkv"),
    (dict(out=None), -1, b"null pointer"),
    (dict(ws=None), -1, b"null pointer"),
    (dict(d=64, block=64, T=128, tb=2, mb=2, dtype=1, qs=16, ks=16, vs=16), -2, b"e4m3"),
])
def test_attention_error_messages(over, code, msg):
    assert _bad_attn(**over) == code
    assert msg in fp.library().fp_last_error_string()


def _bad_paged(**over):
    """A well-formed paged attention call with fake pointers (host validation only)."""
    a = dict(q=16, k=16, v=16, dtype=0, qs=None, ks=None, vs=None, cu=16, cb=16, batch=2,
             T=300, tb=3, mb=2, Hq=8, Hkv=2, d=128, block=128, pt=16, ps=64, mp=4, npg=8,
             scale=0.1, cnt=16, idx=16, out=16, lse=None, ws=256, stream=None)
    a.update(over)
    return fp.library().fp_sparse_prefill_attn_paged(*a.values())


@pytest.mark.parametrize("over,msg", [
    (dict(pt=None), b"page table"),
    (dict(cu=None, cb=None, batch=1, T=256, tb=2, mb=2), b"prefix sums"),
    (dict(ps=48), b"page_size 48"),
    (dict(ps=256), b"page_size 256"),                 # larger than the block
    (dict(npg=0), b"num_pages (0)"),
    (dict(mp=0), b"max_pages (0)"),
])
def test_paged_attention_rejects_bad_paging(over, msg):
    assert _bad_paged(**over) == -1
    assert msg in fp.library().fp_last_error_string()


@pytest.mark.parametrize("args,code,msg", [
    # (q_pool, k_pool, split, cu_blocks, batch, total_blocks, max_blocks, Hq, Hkv, d, alpha)
    ((16, 16, None, None, 0, 4, 4, 8, 2, 128, 0.1), -1, b"batch"),
    ((16, 16, None, None, 1, 4, 5, 8, 2, 128, 0.1), -1, b"max_blocks must equal"),
    ((16, 16, None, None, 1, 4, 4, 6, 4, 128, 0.1), -1, b"multiple of Hkv"),
    ((16, 16, None, None, 1, 4, 4, 8, 2, 96, 0.1), -2, b"head dim 96"),
    ((8, 16, None, None, 1, 4, 4, 8, 2, 128, 0.1), -1, b"16-byte aligned"),
    ((16, 16, 8, None, 1, 4, 4, 8, 2, 128, 0.1), -1, b"16-byte aligned"),
    ((16, 16, None, None, 1, 4, 4, 8, 2, 128, float("nan")), -1, b"alpha"),
    ((16, 16, None, None, 1, 4, 4, 8, 2, 128, -0.5), -1, b"alpha"),
])
def test_mask_error_messages(args, code, msg):
    lib = fp.library()
    rc = lib.fp_build_block_mask(*args, 0.1, 3, None, 16, 16, None, None)
    assert rc == code
    assert msg in lib.fp_last_error_string()


def test_noalloc_refuses_problems_past_its_scratch():
    """(Hq + Hkv) * total_blocks * d above 8 Mi floats: refused with a message, before any
    CUDA call (this runs without a GPU)."""
    lib = fp.library()
    T = 2048 * 128
    rc = lib.fp_pool_and_mask_noalloc(16, 16, 0, None, None, None, None, 1, T, 2048, 2048, 32, 8,
                                      128, 128, None, 0, 0, 0, 0.1, 0.1, 3, None, 16, 16, None)
    assert rc == -1
    assert b"static scratch" in lib.fp_last_error_string()


def test_debug_hook_and_status_reject_bad_arguments():
    lib = fp.library()
    assert lib.fp_debug_skip_k_load(-1) == -1
    assert lib.fp_debug_skip_mask_load(-1) == -1
    assert lib.fp_check_status(None, None) == -1
    assert b"workspace" in lib.fp_last_error_string()


def test_mask_rejects_alpha_out_of_range():
    lib = fp.library()
    rc = lib.fp_build_block_mask(16, 16, None, None, 1, 4, 4, 8, 2, 128, 1.5, 0.1, 3, None, 16,
                                 16, None, None)
    assert rc == -1
    assert b"alpha" in lib.fp_last_error_string()


def test_chunked_batch_layout():
    """Host-side prefix sums of a chunked batch (query blocks start at floor(P0 / block))."""
    cb = fp.ChunkedBatch.make((1000, 0, 37, 641, 1), (1000, 700, 300, 1500, 129), 128, "cpu")
    # query blocks: [0, 8), none, [2, 3), [6, 12), [1, 2)
    assert cb.cu_qblocks.tolist() == [0, 8, 8, 9, 15, 16]
    assert cb.cu_kblocks.tolist() == [0, 8, 14, 17, 29, 31]
    assert (cb.total_q, cb.total_k, cb.max_kblocks) == (1679, 3629, 12)


def _bad_chunked_attn(**over):
    """A well-formed chunked attention call with fake pointers (host validation only)."""
    a = dict(q=16, k=16, v=16, dtype=0, qs=None, ks=None, vs=None, cq=16, cqb=16, ck=16, ckb=16,
             batch=2, Tq=300, Tk=1000, tqb=4, tkb=9, mkb=5, Hq=8, Hkv=2, d=128, block=128,
             pt=None, ps=0, mp=0, npg=0, scale=0.1, cnt=16, idx=16, out=16, lse=None, of=0,
             ws=256, stream=None)
    a.update(over)
    return fp.library().fp_sparse_prefill_attn_chunked(*a.values())


@pytest.mark.parametrize("over,code", [
    (dict(cq=None), -1),             # chunked calls need every prefix-sum array
    (dict(ckb=None), -1),
    (dict(Tq=1001), -1),             # more queries than keys
    (dict(tqb=10), -1),              # more query blocks than key blocks
    (dict(mkb=0), -1),               # no room for a kept-block list
    (dict(block=96), -2),
    (dict(pt=16, ps=48), -1),        # page size not dividing the block
    (dict(dtype=1, qs=16, ks=16, vs=16, d=64), -2),   # e4m3 needs d = 128
    (dict(of=1), -1),                # paged output without a page table
    (dict(of=3), -1),                # the same with query-block pairing (FP_PAIR_QBLOCKS = 2)
    (dict(of=4), -1),                # unknown flag
])
def test_chunked_attention_rejects_bad_arguments(over, code):
    assert _bad_chunked_attn(**over) == code
    assert fp.library().fp_last_error_string()


def test_chunked_attention_flag_messages():
    """FP_OUT_PAGED (1) and FP_PAIR_QBLOCKS (2) are the only flags; any other bit is refused
    as unknown, and the paged output is refused for its missing page table, not its flag."""
    assert fp.OUT_PAGED == 1 and fp.PAIR_QBLOCKS == 2
    for of in (4, 8, 1 << 30):
        assert _bad_chunked_attn(of=of) == -1
        assert b"unknown flags" in fp.library().fp_last_error_string()
    for of in (1, 3):
        assert _bad_chunked_attn(of=of) == -1
        assert b"page table" in fp.library().fp_last_error_string()


def test_chunked_mask_and_pool_reject_bad_arguments():
    lib = fp.library()
    # mask: block size is needed to place query blocks
    rc = lib.fp_build_block_mask_chunked(16, 16, None, 16, 16, 16, 16, 2, 4, 9, 5, 8, 2, 128, 96,
                                         0.1, 0.1, 3, None, 16, 16, None, None)
    assert rc == -2
    rc = lib.fp_build_block_mask_chunked(16, 16, None, None, 16, 16, 16, 2, 4, 9, 5, 8, 2, 128,
                                         128, 0.1, 0.1, 3, None, 16, 16, None, None)
    assert rc == -1
    rc = lib.fp_pool_qk_chunked(16, 16, 0, None, None, 16, 16, 16, 16, 2, 1001, 1000, 4, 9, 8, 2,
                                128, 128, None, 0, 0, 0, 16, 16, None, None, None)
    assert rc == -1 and b"total_q" in lib.fp_last_error_string()


def test_append_rejects_bad_arguments():
    lib = fp.library()
    args = [16, 16, 0, 16, 16, 2, 300, 2, 128, 16, 64, 8, 40, 16, 16, 256, None]
    bad_d = list(args); bad_d[8] = 96
    assert lib.fp_append_paged_kv(*bad_d) == -2
    null_pt = list(args); null_pt[9] = None
    assert lib.fp_append_paged_kv(*null_pt) == -1
    bad_page = list(args); bad_page[10] = 0
    assert lib.fp_append_paged_kv(*bad_page) == -1
    misaligned = list(args); misaligned[13] = 8
    assert lib.fp_append_paged_kv(*misaligned) == -1


def test_empty_inputs_return_ok_without_launching():
    """No tokens: every stage returns FP_OK before any CUDA call (this runs without a GPU)."""
    lib = fp.library()
    assert lib.fp_pool_qk(16, 16, 0, None, None, None, None, 1, 0, 0, 8, 2, 128, 128, None, 0, 0,
                          0, 16, 16, None, None, None) == 0
    assert lib.fp_build_block_mask(16, 16, None, None, 1, 0, 0, 8, 2, 128, 0.1, 0.1, 3, None, 16,
                                   16, None, None) == 0
    assert _bad_attn(T=0, tb=0, mb=0) == 0
    assert lib.fp_append_paged_kv(16, 16, 0, 16, 16, 1, 0, 2, 128, 16, 64, 1, 1, 16, 16, 256,
                                  None) == 0


def test_host_index_arrays_are_refused_before_launch():
    """Prefix sums left in host memory would make a kernel fault the GPU; the library
    refuses them (on a machine without a GPU the pointer cannot even be queried)."""
    import numpy as np
    cu = np.array([0, 200, 300], dtype=np.int32)
    cb = np.array([0, 2, 3], dtype=np.int32)
    lib = fp.library()
    rc = lib.fp_pool_qk(16, 16, 0, None, None, cu.ctypes.data, cb.ctypes.data, 2, 300, 3, 8, 2,
                        128, 128, None, 0, 0, 0, 16, 16, None, None, None)
    assert rc == -1
    assert b"cu_" in lib.fp_last_error_string()


def test_binding_refuses_cpu_tensors_views_and_mixed_dtypes():
    import torch
    q = torch.zeros((256, 4, 128), dtype=torch.bfloat16)
    k = torch.zeros((256, 2, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        fp._ptr(q)
    with pytest.raises(TypeError, match="same dtype"):
        fp._same_dtype(q, k.to(torch.float8_e4m3fn))
    fp._same_dtype(q, k, None)
    assert fp._ptr(None) is None


def test_pool_and_mask_refuse_a_misaligned_workspace():
    """The pool and mask calls take the status workspace (NULL allowed); a misaligned one is
    refused before anything is enqueued."""
    lib = fp.library()
    rc = lib.fp_pool_qk(16, 16, 0, None, None, None, None, 1, 256, 2, 8, 2, 128, 128, None, 0, 0,
                        0, 16, 16, None, 128, None)
    assert rc == -1 and b"workspace" in lib.fp_last_error_string()
    rc = lib.fp_build_block_mask(16, 16, None, None, 1, 2, 2, 8, 2, 128, 0.1, 0.1, 3, None, 16,
                                 16, 128, None)
    assert rc == -1 and b"workspace" in lib.fp_last_error_string()
    rc = lib.fp_pool_qk_chunked(16, 16, 0, None, None, 16, 16, 16, 16, 2, 300, 1000, 4, 9, 8, 2,
                                128, 128, None, 0, 0, 0, 16, 16, None, 64, None)
    assert rc == -1 and b"workspace" in lib.fp_last_error_string()
    rc = lib.fp_build_block_mask_chunked(16, 16, None, 16, 16, 16, 16, 2, 4, 9, 5, 8, 2, 128, 128,
                                         0.1, 0.1, 3, None, 16, 16, 64, None)
    assert rc == -1 and b"workspace" in lib.fp_last_error_string()
