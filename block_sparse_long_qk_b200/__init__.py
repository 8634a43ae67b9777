"""Block-sparse causal prefill attention for B200 (FlashPrefill-style), Python binding.

Thin ctypes layer over ``libfpsparse.so`` (declared in ``include/fpsparse.h``). It only
marshals arguments: torch is used for device memory and streams, and every step of the
path runs in the library's CUDA kernels. There is no CPU fallback: if the library is
missing or fails to load, every call raises.

The path (names follow "FlashPrefill: Instantaneous Pattern Discovery and Thresholding for
Ultra-Fast Long-Context Prefilling", technical summary section 2):

    q_pool, k_pool     = pool_qk(q, k, block)                      # 2.A block means
    mask, kv_cnt, kv_idx = build_block_mask(q_pool, k_pool, alpha)   # 2.B max-based threshold
    out, lse           = sparse_prefill_attn(q, k, v, kv_cnt, kv_idx)  # 2.C physical skip

``sparse_prefill`` runs all three. Paged K/V (``PagedKV``) and varlen batches (``Batch``)
follow "FlashPrefill V2: Block-Sparse Prefill Attention for Long-Context LLM Serving",
Abstract (paged KV cache, continuous batching); so do the ``*_chunked`` calls with a
``ChunkedBatch``, whose requests prefill only the last q_len of their kv_len positions (a
chunk after a cached prefix).
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
import re

import torch

__all__ = ["Batch", "PagedKV", "pool_qk", "build_block_mask", "sparse_prefill_attn",
           "sparse_prefill_attn_paged", "sparse_prefill", "check_status", "workspace",
           "library", "FpError", "FORCE_FIRST", "FORCE_DIAG", "MASK_FP32", "OUT_PAGED", "PAIR_QBLOCKS", "header_symbols",
           "pool_and_mask_noalloc", "k_split_shape", "ChunkedBatch", "pool_qk_chunked",
           "build_block_mask_chunked", "sparse_prefill_attn_chunked", "sparse_prefill_chunked",
           "HostPipeline", "append_paged_kv", "GraphStep", "head_shard"]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfpsparse.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "fpsparse.h")

FP_OK = 0
FP_DTYPE_BF16, FP_DTYPE_E4M3 = 0, 1
FORCE_FIRST, FORCE_DIAG, MASK_FP32 = 1, 2, 4
OUT_PAGED, PAIR_QBLOCKS = 1, 2
_ERRORS = {-1: "FP_ERR_INVALID_ARG", -2: "FP_ERR_UNSUPPORTED", -3: "FP_ERR_CUDA",
           -4: "FP_ERR_TIMEOUT", -5: "FP_ERR_BAD_INDEX"}

_p, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_SIGNATURES = {
    "fp_version": (_i, []),
    "fp_last_error_string": (ctypes.c_char_p, []),
    "fp_workspace_size": (_sz, []),
    "fp_pool_qk": (_i, [_p, _p, _i, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _p, _i, _i,
                        _i, _p, _p, _p, _p, _p]),
    "fp_build_block_mask": (_i, [_p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _f, _f, _i, _p, _p,
                                 _p, _p, _p]),
    "fp_sparse_prefill_attn": (_i, [_p, _p, _p, _i, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i,
                                    _i, _i, _i, _f, _p, _p, _p, _p, _p, _p]),
    "fp_sparse_prefill_attn_paged": (_i, [_p, _p, _p, _i, _p, _p, _p, _p, _p, _i, _i, _i, _i,
                                          _i, _i, _i, _i, _p, _i, _i, _i, _f, _p, _p, _p, _p,
                                          _p, _p]),
    "fp_check_status": (_i, [_p, _p]),
    "fp_debug_skip_k_load": (_i, [_i]),
    "fp_debug_skip_mask_load": (_i, [_i]),
    "fp_pool_and_mask_noalloc": (_i, [_p, _p, _i, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i,
                                      _i, _p, _i, _i, _i, _f, _f, _i, _p, _p, _p, _p]),
    "fp_pool_qk_chunked": (_i, [_p, _p, _i, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i,
                                _i, _i, _p, _i, _i, _i, _p, _p, _p, _p, _p]),
    "fp_build_block_mask_chunked": (_i, [_p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i,
                                         _i, _i, _f, _f, _i, _p, _p, _p, _p, _p]),
    "fp_append_paged_kv": (_i, [_p, _p, _i, _p, _p, _i, _i, _i, _i, _p, _i, _i, _i, _p, _p, _p,
                                _p]),
    "fp_sparse_prefill_attn_chunked": (_i, [_p, _p, _p, _i, _p, _p, _p, _p, _p, _p, _p, _i, _i,
                                            _i, _i, _i, _i, _i, _i, _i, _i, _p, _i, _i, _i, _f,
                                            _p, _p, _p, _p, _i, _p, _p]),
}


class FpError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"{_ERRORS.get(code, code)}: {msg}")
        self.code = code


_lib = None


def library():
    """The loaded C library. Raises if it is missing (build it with
    ``python -m block_sparse_long_qk_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise FpError(-3, f"{LIB_PATH} not found; build it with "
                              "`python -m block_sparse_long_qk_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def header_symbols():
    """Names of the functions declared in include/fpsparse.h."""
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:int|size_t|const char\*)\s+(fp_\w+)\s*\(", txt,
                                 flags=re.M)))


def _check(rc):
    if rc != FP_OK:
        raise FpError(rc, library().fp_last_error_string().decode())


def _ptr(t):
    """Device address of a contiguous CUDA tensor (None passes NULL). The kernels read plain
    row-major device memory, so host tensors and strided views are refused here rather than
    read wrongly on the GPU."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"expected a CUDA tensor, got one on {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"expected a contiguous tensor, got shape {tuple(t.shape)} with "
                         f"strides {t.stride()}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _same_dtype(*ts):
    """Q, K and V (or a cache) must share one storage type: the kernels read them as one."""
    ts = [t for t in ts if t is not None]
    if any(t.dtype != ts[0].dtype for t in ts):
        raise TypeError("Q, K and V must have the same dtype, got "
                        + ", ".join(str(t.dtype) for t in ts))


def _expect(t, name, shape=None, dtype=None, min_numel=None):
    """Host-side check of a tensor the kernels read or write: the C ABI receives only a
    pointer and the sizes derived from the other arguments, so a tensor smaller than those
    sizes would be read or written past its end on the GPU. Refused here instead."""
    if t is None:
        return
    if shape is not None and tuple(t.shape) != tuple(int(x) for x in shape):
        raise ValueError(f"{name}: expected shape {tuple(int(x) for x in shape)}, got "
                         f"{tuple(t.shape)}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: expected dtype {dtype}, got {t.dtype}")
    if min_numel is not None and t.numel() < min_numel:
        raise ValueError(f"{name}: expected at least {int(min_numel)} elements, got "
                         f"{t.numel()}")


def _expect_heads(q, k, name_k="k"):
    """Q [T, Hq, d] and K [*, Hkv, d]: same head dim, Hq a multiple of Hkv."""
    if q.dim() != 3:
        raise ValueError(f"q: expected [tokens, Hq, d], got shape {tuple(q.shape)}")
    if k.dim() < 3 or k.shape[-1] != q.shape[-1]:
        raise ValueError(f"{name_k}: expected head dim {q.shape[-1]}, got shape "
                         f"{tuple(k.shape)}")
    if q.shape[1] % k.shape[-2] != 0:
        raise ValueError(f"Hq = {q.shape[1]} is not a multiple of Hkv = {k.shape[-2]}")


def _expect_scales(q_scale, k_scale, v_scale, Hq, Hkv):
    _expect(q_scale, "q_scale", (Hq,), torch.float32)
    _expect(k_scale, "k_scale", (Hkv,), torch.float32)
    _expect(v_scale, "v_scale", (Hkv,), torch.float32)


def _expect_paged(paged, d, batch_size, need_v):
    """Caches [num_pages, page_size, Hkv, d] and an int32 page table with a row per request."""
    kc = paged.k_cache
    if kc.dim() != 4 or kc.shape[-1] != d:
        raise ValueError(f"k_cache: expected [num_pages, page_size, Hkv, {d}], got shape "
                         f"{tuple(kc.shape)}")
    if need_v:
        _expect(paged.v_cache, "v_cache", kc.shape)
    pt = paged.page_table
    if pt.dim() != 2 or pt.shape[0] < batch_size:
        raise ValueError(f"page_table: expected [batch >= {batch_size}, max_pages], got shape "
                         f"{tuple(pt.shape)}")
    _expect(pt, "page_table", dtype=torch.int32)


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return FP_DTYPE_BF16
    if t.dtype == torch.float8_e4m3fn:
        return FP_DTYPE_E4M3
    raise TypeError(f"unsupported storage dtype {t.dtype} (bf16 or float8_e4m3fn)")


@dataclasses.dataclass
class Batch:
    """A varlen batch: host lengths plus the device index arrays the kernels read."""
    seqlens: tuple
    block: int
    cu_seqlens: torch.Tensor    # int32 [B+1] on the device
    cu_blocks: torch.Tensor     # int32 [B+1] on the device
    total_tokens: int
    total_blocks: int
    max_blocks: int

    @staticmethod
    def make(seqlens, block, device):
        seqlens = tuple(int(s) for s in seqlens)
        nb = [(s + block - 1) // block for s in seqlens]
        cu = [0]
        for s in seqlens:
            cu.append(cu[-1] + s)
        cb = [0]
        for n in nb:
            cb.append(cb[-1] + n)
        return Batch(seqlens, block, torch.tensor(cu, dtype=torch.int32, device=device),
                     torch.tensor(cb, dtype=torch.int32, device=device), cu[-1], cb[-1],
                     max(nb) if nb else 0)

    @property
    def size(self):
        return len(self.seqlens)

    def _ptrs(self):
        if self.size == 1:
            return None, None
        return _ptr(self.cu_seqlens), _ptr(self.cu_blocks)


@dataclasses.dataclass
class PagedKV:
    """K/V caches [num_pages, page_size, Hkv, d] and the int32 page table [B, max_pages]."""
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    page_table: torch.Tensor

    @property
    def page_size(self):
        return self.k_cache.shape[1]


def head_shard(Hq, Hkv, rank, world):
    """The heads that rank ``rank`` of ``world`` owns when one layer is split by KV-head group:
    (query-head slice, KV-head slice). A query head reads only its own KV head in all three
    stages (pooled scores, mask and attention), so each rank runs the whole path on its slice
    with no exchange between ranks. Groups are dealt as evenly as they go: the first
    Hkv % world ranks take one group more. At most Hkv ranks."""
    if Hq <= 0 or Hkv <= 0 or Hq % Hkv:
        raise ValueError(f"Hq ({Hq}) must be a positive multiple of Hkv ({Hkv})")
    if not 1 <= world <= Hkv or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of {world}: a head split needs 1 <= world <= Hkv ({Hkv})")
    base, extra = divmod(Hkv, world)
    g0 = rank * base + min(rank, extra)
    g1 = g0 + base + (1 if rank < extra else 0)
    G = Hq // Hkv
    return slice(g0 * G, g1 * G), slice(g0, g1)


_workspaces = {}


def workspace(device):
    """A zeroed per-device status workspace (allocated once by torch)."""
    device = torch.device(device)
    key = device.index if device.index is not None else torch.cuda.current_device()
    ws = _workspaces.get(key)
    if ws is None:
        n = library().fp_workspace_size()
        ws = torch.zeros(max(256, n), dtype=torch.uint8, device=device)
        _workspaces[key] = ws
    return ws


def check_status(device=None, ws=None):
    """Waits for the current stream and raises if a launch on the workspace recorded a
    pipeline timeout, an out-of-range index or inconsistent prefix sums since the last check."""
    if ws is None:
        ws = workspace(device if device is not None else torch.device("cuda"))
    _check(library().fp_check_status(_ptr(ws), _stream(ws.device)))


def _batch_for(q, block, batch):
    if batch is None:
        return Batch.make((q.shape[0],), block, q.device)
    if batch.block != block:
        raise ValueError("batch was built for a different block size")
    return batch


def _expect_tokens(b, T):
    if b.total_tokens != T:
        raise ValueError(f"the batch holds {b.total_tokens} tokens but q has {T} rows")


def pool_qk(q, k, block=128, *, batch: Batch | None = None, q_scale=None, k_scale=None,
            paged: PagedKV | None = None, k_split_out=None, ws=None):
    """Block means of Q [T,Hq,d] and K [T,Hkv,d] (or the paged K cache) -> float32
    q_pool [Hq, nblk, d], k_pool [Hkv, nblk, d]. With ``k_split_out`` (bf16 tensor of
    ``k_split_shape``) the kernel also writes the hi / lo bf16 split of k_pool there, which
    ``build_block_mask(k_split=...)`` then loads instead of converting."""
    kk = paged.k_cache if paged is not None else k
    _expect_heads(q, kk, "k_cache" if paged is not None else "k")
    T, Hq, d = q.shape
    _same_dtype(q, kk)
    Hkv = kk.shape[-2]
    b = _batch_for(q, block, batch)
    _expect_tokens(b, T)
    if paged is not None:
        _expect_paged(paged, d, b.size, need_v=False)
    else:
        _expect(k, "k", (T, Hkv, d))
    _expect_scales(q_scale, k_scale, None, Hq, Hkv)
    _expect(k_split_out, "k_split_out", k_split_shape(Hkv, b.total_blocks, d), torch.bfloat16)
    q_pool = torch.empty((Hq, b.total_blocks, d), dtype=torch.float32, device=q.device)
    k_pool = torch.empty((Hkv, b.total_blocks, d), dtype=torch.float32, device=q.device)
    cu, cb = b._ptrs()
    if paged is not None and cu is None:
        cu, cb = _ptr(b.cu_seqlens), _ptr(b.cu_blocks)
    pt = paged.page_table if paged is not None else None
    _check(library().fp_pool_qk(
        _ptr(q), _ptr(kk), _dtype_code(q), _ptr(q_scale), _ptr(k_scale), cu, cb, b.size, T,
        b.total_blocks, Hq, Hkv, d, block, _ptr(pt), paged.page_size if paged else 0,
        pt.shape[1] if pt is not None else 0, kk.shape[0] if pt is not None else 0,
        _ptr(q_pool), _ptr(k_pool), _ptr(k_split_out),
        _ptr(workspace(q.device) if ws is None else ws), _stream(q.device)))
    return q_pool, k_pool


def k_split_shape(Hkv, total_blocks, d):
    """Shape of the bf16 hi / lo split of the pooled keys: [2, Hkv, total_blocks, d]."""
    return (2, Hkv, total_blocks, d)


def build_block_mask(q_pool, k_pool, alpha=0.1, *, block=128, batch: Batch | None = None,
                     scale=None, flags=FORCE_FIRST | FORCE_DIAG, mask_bits=True, k_split=None,
                     ws=None):
    """Max-based dynamic threshold on the pooled block scores -> (mask_bits or None
    [Hq, nblk, words] uint32 viewed as int32, kv_cnt [Hq, nblk] int32, kv_idx
    [Hq, nblk, max_blocks] int32)."""
    Hq, nblk, d = q_pool.shape
    Hkv = k_pool.shape[0]
    _expect(q_pool, "q_pool", dtype=torch.float32)
    _expect(k_pool, "k_pool", (Hkv, nblk, d), torch.float32)
    _expect(k_split, "k_split", k_split_shape(Hkv, nblk, d), torch.bfloat16)
    if batch is None:
        batch = Batch.make((nblk * block,), block, q_pool.device)
        batch = dataclasses.replace(batch, total_blocks=nblk, max_blocks=nblk)
    elif batch.total_blocks != nblk:
        raise ValueError(f"the batch holds {batch.total_blocks} blocks but q_pool has {nblk}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    words = (batch.max_blocks + 31) // 32
    dev = q_pool.device
    bits = torch.zeros((Hq, nblk, words), dtype=torch.int32, device=dev) if mask_bits else None
    kv_cnt = torch.empty((Hq, nblk), dtype=torch.int32, device=dev)
    kv_idx = torch.empty((Hq, nblk, batch.max_blocks), dtype=torch.int32, device=dev)
    cb = _ptr(batch.cu_blocks) if batch.size > 1 else None
    _check(library().fp_build_block_mask(
        _ptr(q_pool), _ptr(k_pool), _ptr(k_split), cb, batch.size, nblk, batch.max_blocks, Hq,
        Hkv, d,
        float(alpha), float(scale), int(flags), _ptr(bits), _ptr(kv_cnt), _ptr(kv_idx),
        _ptr(workspace(dev) if ws is None else ws), _stream(dev)))
    return bits, kv_cnt, kv_idx


def _expect_lists(kv_cnt, kv_idx, Hq, nblk, max_blocks):
    """kv_cnt int32 [Hq, nblk] and kv_idx int32 [Hq, nblk, max_blocks] (or larger buffers)."""
    if kv_cnt is None or kv_idx is None:
        raise ValueError("kv_cnt and kv_idx are required")
    _expect(kv_cnt, "kv_cnt", dtype=torch.int32, min_numel=Hq * nblk)
    _expect(kv_idx, "kv_idx", dtype=torch.int32, min_numel=Hq * nblk * max_blocks)


def sparse_prefill_attn(q, k, v, kv_cnt, kv_idx, block=128, *, batch: Batch | None = None,
                        scale=None, q_scale=None, k_scale=None, v_scale=None,
                        return_lse=False, out=None, ws=None):
    """Causal attention over the kept KV blocks -> (out bf16 [T,Hq,d], lse [Hq,T] or None)."""
    _same_dtype(q, k, v)
    _expect_heads(q, k)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    b = _batch_for(q, block, batch)
    _expect_tokens(b, T)
    _expect(k, "k", (T, Hkv, d))
    _expect(v, "v", (T, Hkv, d))
    _expect_lists(kv_cnt, kv_idx, Hq, b.total_blocks, b.max_blocks)
    _expect_scales(q_scale, k_scale, v_scale, Hq, Hkv)
    _expect(out, "out", (T, Hq, d), torch.bfloat16)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((T, Hq, d), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((Hq, T), dtype=torch.float32, device=q.device) if return_lse else None
    ws = workspace(q.device) if ws is None else ws
    cu, cb = b._ptrs()
    _check(library().fp_sparse_prefill_attn(
        _ptr(q), _ptr(k), _ptr(v), _dtype_code(q), _ptr(q_scale), _ptr(k_scale), _ptr(v_scale),
        cu, cb, b.size, T, b.total_blocks, b.max_blocks, Hq, Hkv, d, block, float(scale),
        _ptr(kv_cnt), _ptr(kv_idx), _ptr(out), _ptr(lse), _ptr(ws), _stream(q.device)))
    return out, lse


def sparse_prefill_attn_paged(q, paged: PagedKV, kv_cnt, kv_idx, batch: Batch, *,
                              scale=None, q_scale=None, k_scale=None, v_scale=None,
                              return_lse=False, out=None, ws=None):
    """Same as ``sparse_prefill_attn`` with K/V read through the page table."""
    _same_dtype(q, paged.k_cache, paged.v_cache)
    _expect_heads(q, paged.k_cache, "k_cache")
    T, Hq, d = q.shape
    Hkv = paged.k_cache.shape[2]
    _expect_tokens(batch, T)
    _expect_paged(paged, d, batch.size, need_v=True)
    _expect_lists(kv_cnt, kv_idx, Hq, batch.total_blocks, batch.max_blocks)
    _expect_scales(q_scale, k_scale, v_scale, Hq, Hkv)
    _expect(out, "out", (T, Hq, d), torch.bfloat16)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((T, Hq, d), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((Hq, T), dtype=torch.float32, device=q.device) if return_lse else None
    ws = workspace(q.device) if ws is None else ws
    pt = paged.page_table
    _check(library().fp_sparse_prefill_attn_paged(
        _ptr(q), _ptr(paged.k_cache), _ptr(paged.v_cache), _dtype_code(q), _ptr(q_scale),
        _ptr(k_scale), _ptr(v_scale), _ptr(batch.cu_seqlens), _ptr(batch.cu_blocks),
        batch.size, T, batch.total_blocks, batch.max_blocks, Hq, Hkv, d, batch.block, _ptr(pt),
        paged.page_size, pt.shape[1], paged.k_cache.shape[0], float(scale), _ptr(kv_cnt),
        _ptr(kv_idx), _ptr(out), _ptr(lse), _ptr(ws), _stream(q.device)))
    return out, lse


def sparse_prefill(q, k=None, v=None, alpha=0.1, block=128, *, batch: Batch | None = None,
                   paged: PagedKV | None = None, scale=None, q_scale=None, k_scale=None,
                   v_scale=None, return_lse=False, flags=FORCE_FIRST | FORCE_DIAG, out=None):
    """The whole path: pool -> threshold/mask -> sparse attention. Returns
    (out, lse or None, kv_cnt, kv_idx); ``out`` may be a preallocated bf16 [T, Hq, d]."""
    b = _batch_for(q, block, batch)
    d = q.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    Hkv = (paged.k_cache if paged is not None else k).shape[-2]
    k_split = torch.empty(k_split_shape(Hkv, b.total_blocks, d), dtype=torch.bfloat16,
                          device=q.device)
    q_pool, k_pool = pool_qk(q, k, block, batch=b, q_scale=q_scale, k_scale=k_scale, paged=paged,
                             k_split_out=k_split)
    _, kv_cnt, kv_idx = build_block_mask(q_pool, k_pool, alpha, block=block, batch=b,
                                         scale=scale, flags=flags, mask_bits=False,
                                         k_split=k_split)
    if paged is not None:
        out, lse = sparse_prefill_attn_paged(q, paged, kv_cnt, kv_idx, b, scale=scale,
                                             q_scale=q_scale, k_scale=k_scale, v_scale=v_scale,
                                             return_lse=return_lse, out=out)
    else:
        out, lse = sparse_prefill_attn(q, k, v, kv_cnt, kv_idx, block, batch=b, scale=scale,
                                       q_scale=q_scale, k_scale=k_scale, v_scale=v_scale,
                                       return_lse=return_lse, out=out)
    return out, lse, kv_cnt, kv_idx


def pool_and_mask_noalloc(q, k, alpha=0.1, block=128, *, batch: Batch | None = None,
                          scale=None, q_scale=None, k_scale=None, paged: PagedKV | None = None,
                          flags=FORCE_FIRST | FORCE_DIAG, mask_bits=True):
    """``pool_qk`` + ``build_block_mask`` with the pooled means kept in the library's static
    device scratch (for callers that cannot allocate them). Returns (mask_bits or None,
    kv_cnt, kv_idx); the output tensors are allocated here by torch for convenience."""
    kk = paged.k_cache if paged is not None else k
    _expect_heads(q, kk, "k_cache" if paged is not None else "k")
    T, Hq, d = q.shape
    _same_dtype(q, kk)
    Hkv = kk.shape[-2]
    b = _batch_for(q, block, batch)
    _expect_tokens(b, T)
    if paged is not None:
        _expect_paged(paged, d, b.size, need_v=False)
    else:
        _expect(k, "k", (T, Hkv, d))
    _expect_scales(q_scale, k_scale, None, Hq, Hkv)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dev = q.device
    words = (b.max_blocks + 31) // 32
    bits = torch.zeros((Hq, b.total_blocks, words), dtype=torch.int32, device=dev) \
        if mask_bits else None
    kv_cnt = torch.empty((Hq, b.total_blocks), dtype=torch.int32, device=dev)
    kv_idx = torch.empty((Hq, b.total_blocks, b.max_blocks), dtype=torch.int32, device=dev)
    cu, cb = b._ptrs()
    if paged is not None and cu is None:
        cu, cb = _ptr(b.cu_seqlens), _ptr(b.cu_blocks)
    pt = paged.page_table if paged is not None else None
    _check(library().fp_pool_and_mask_noalloc(
        _ptr(q), _ptr(kk), _dtype_code(q), _ptr(q_scale), _ptr(k_scale), cu, cb, b.size, T,
        b.total_blocks, b.max_blocks, Hq, Hkv, d, block, _ptr(pt),
        paged.page_size if paged else 0, pt.shape[1] if pt is not None else 0,
        kk.shape[0] if pt is not None else 0, float(alpha), float(scale), int(flags),
        _ptr(bits), _ptr(kv_cnt), _ptr(kv_idx), _stream(dev)))
    return bits, kv_cnt, kv_idx


@dataclasses.dataclass
class ChunkedBatch:
    """A chunked / prefix-cached varlen batch: request b has kv_lens[b] keys and prefills its
    last q_lens[b] positions. Blocks lie on absolute positions; the query blocks of request b
    are the absolute blocks (kv_len - q_len) // block .. ceil(kv_len / block) - 1."""
    q_lens: tuple
    kv_lens: tuple
    block: int
    cu_q: torch.Tensor        # int32 [B+1] on the device
    cu_qblocks: torch.Tensor  # int32 [B+1]
    cu_k: torch.Tensor        # int32 [B+1]
    cu_kblocks: torch.Tensor  # int32 [B+1]
    total_q: int
    total_k: int
    total_qblocks: int
    total_kblocks: int
    max_kblocks: int

    @staticmethod
    def make(q_lens, kv_lens, block, device):
        q_lens = tuple(int(x) for x in q_lens)
        kv_lens = tuple(int(x) for x in kv_lens)
        if len(q_lens) != len(kv_lens) or not q_lens:
            raise ValueError("q_lens and kv_lens need one entry per request")
        nk, nq = [], []
        for n, L in zip(q_lens, kv_lens):
            if not 0 <= n <= L:
                raise ValueError(f"q_len {n} must lie in [0, kv_len {L}]")
            nk.append((L + block - 1) // block)
            nq.append(nk[-1] - (L - n) // block if n > 0 else 0)

        def cum(xs):
            out = [0]
            for x in xs:
                out.append(out[-1] + x)
            return out
        cq, ck, cqb, ckb = cum(q_lens), cum(kv_lens), cum(nq), cum(nk)

        def dev(xs):
            return torch.tensor(xs, dtype=torch.int32, device=device)
        return ChunkedBatch(q_lens, kv_lens, block, dev(cq), dev(cqb), dev(ck), dev(ckb),
                            cq[-1], ck[-1], cqb[-1], ckb[-1], max(nk))

    @property
    def size(self):
        return len(self.q_lens)

    def _args(self):
        return (_ptr(self.cu_q), _ptr(self.cu_qblocks), _ptr(self.cu_k), _ptr(self.cu_kblocks),
                self.size)


def _expect_chunk_rows(cb, q, k, v, paged, need_v):
    """Q [total_q, Hq, d]; K and V [total_k, Hkv, d] or the caches of ``paged``."""
    T, Hq, d = q.shape
    if T != cb.total_q:
        raise ValueError(f"the batch holds {cb.total_q} queries but q has {T} rows")
    if paged is not None:
        _expect_paged(paged, d, cb.size, need_v)
    else:
        Hkv = k.shape[-2]
        _expect(k, "k", (cb.total_k, Hkv, d))
        if need_v:
            _expect(v, "v", (cb.total_k, Hkv, d))


def pool_qk_chunked(q, k, cb: ChunkedBatch, *, q_scale=None, k_scale=None,
                    paged: PagedKV | None = None, k_split_out=None, ws=None):
    """Block means for a chunked batch: q_pool [Hq, total_qblocks, d] over the queries each
    query block holds, k_pool [Hkv, total_kblocks, d] over all keys (cached prefix included)."""
    kk = paged.k_cache if paged is not None else k
    _expect_heads(q, kk, "k_cache" if paged is not None else "k")
    _, Hq, d = q.shape
    _same_dtype(q, kk)
    Hkv = kk.shape[-2]
    _expect_chunk_rows(cb, q, k, None, paged, need_v=False)
    _expect_scales(q_scale, k_scale, None, Hq, Hkv)
    _expect(k_split_out, "k_split_out", k_split_shape(Hkv, cb.total_kblocks, d), torch.bfloat16)
    q_pool = torch.empty((Hq, cb.total_qblocks, d), dtype=torch.float32, device=q.device)
    k_pool = torch.empty((Hkv, cb.total_kblocks, d), dtype=torch.float32, device=q.device)
    pt = paged.page_table if paged is not None else None
    _check(library().fp_pool_qk_chunked(
        _ptr(q), _ptr(kk), _dtype_code(q), _ptr(q_scale), _ptr(k_scale), *cb._args(),
        cb.total_q, cb.total_k, cb.total_qblocks, cb.total_kblocks, Hq, Hkv, d, cb.block,
        _ptr(pt), paged.page_size if paged else 0, pt.shape[1] if pt is not None else 0,
        kk.shape[0] if pt is not None else 0, _ptr(q_pool), _ptr(k_pool), _ptr(k_split_out),
        _ptr(workspace(q.device) if ws is None else ws), _stream(q.device)))
    return q_pool, k_pool


def build_block_mask_chunked(q_pool, k_pool, cb: ChunkedBatch, alpha=0.1, *, scale=None,
                             flags=FORCE_FIRST | FORCE_DIAG, mask_bits=True, k_split=None,
                             ws=None):
    """Threshold for a chunked batch -> (mask_bits or None [Hq, total_qblocks, words],
    kv_cnt [Hq, total_qblocks], kv_idx [Hq, total_qblocks, max_kblocks])."""
    Hq, nqb, d = q_pool.shape
    Hkv = k_pool.shape[0]
    if nqb != cb.total_qblocks:
        raise ValueError(f"the batch holds {cb.total_qblocks} query blocks but q_pool has {nqb}")
    _expect(q_pool, "q_pool", dtype=torch.float32)
    _expect(k_pool, "k_pool", (Hkv, cb.total_kblocks, d), torch.float32)
    _expect(k_split, "k_split", k_split_shape(Hkv, cb.total_kblocks, d), torch.bfloat16)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dev = q_pool.device
    words = (cb.max_kblocks + 31) // 32
    bits = torch.zeros((Hq, nqb, words), dtype=torch.int32, device=dev) if mask_bits else None
    kv_cnt = torch.empty((Hq, nqb), dtype=torch.int32, device=dev)
    kv_idx = torch.empty((Hq, nqb, cb.max_kblocks), dtype=torch.int32, device=dev)
    _check(library().fp_build_block_mask_chunked(
        _ptr(q_pool), _ptr(k_pool), _ptr(k_split), *cb._args(), cb.total_qblocks,
        cb.total_kblocks, cb.max_kblocks, Hq, Hkv, d, cb.block, float(alpha), float(scale),
        int(flags), _ptr(bits), _ptr(kv_cnt), _ptr(kv_idx),
        _ptr(workspace(dev) if ws is None else ws), _stream(dev)))
    return bits, kv_cnt, kv_idx


def sparse_prefill_attn_chunked(q, k, v, kv_cnt, kv_idx, cb: ChunkedBatch, *,
                                paged: PagedKV | None = None, scale=None, q_scale=None,
                                k_scale=None, v_scale=None, return_lse=False, out=None, ws=None,
                                out_paged=False, pair_qblocks=False):
    """Attention of the chunk's queries over the kept KV blocks of the whole request ->
    (out bf16 [total_q, Hq, d], lse [Hq, total_q] or None). K/V are contiguous [total_k, Hkv,
    d] (``k``, ``v``) or the caches of ``paged``. With ``out_paged`` (paged K/V only) the output
    is written in the caches' page layout instead: out [num_pages, page_size, Hq, d], the row
    of position p of request b at slot p % page_size of page page_table[b, p // page_size].
    ``pair_qblocks`` runs every CTA on two neighbouring query blocks of one head instead of two
    heads of a GQA group (the same output, bit for bit)."""
    kk = paged.k_cache if paged is not None else k
    vv = paged.v_cache if paged is not None else v
    _same_dtype(q, kk, vv)
    _expect_heads(q, kk, "k_cache" if paged is not None else "k")
    T, Hq, d = q.shape
    Hkv = kk.shape[-2]
    _expect_chunk_rows(cb, q, k, v, paged, need_v=True)
    _expect_lists(kv_cnt, kv_idx, Hq, cb.total_qblocks, cb.max_kblocks)
    _expect_scales(q_scale, k_scale, v_scale, Hq, Hkv)
    if out_paged and paged is None:
        raise ValueError("out_paged writes through the K/V page table: pass paged=")
    out_shape = (paged.k_cache.shape[0], paged.page_size, Hq, d) if out_paged else (T, Hq, d)
    _expect(out, "out", out_shape, torch.bfloat16)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty(out_shape, dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((Hq, T), dtype=torch.float32, device=q.device) if return_lse else None
    ws = workspace(q.device) if ws is None else ws
    pt = paged.page_table if paged is not None else None
    _check(library().fp_sparse_prefill_attn_chunked(
        _ptr(q), _ptr(kk), _ptr(vv), _dtype_code(q), _ptr(q_scale), _ptr(k_scale),
        _ptr(v_scale), *cb._args(), cb.total_q, cb.total_k, cb.total_qblocks, cb.total_kblocks,
        cb.max_kblocks, Hq, Hkv, d, cb.block, _ptr(pt), paged.page_size if paged else 0,
        pt.shape[1] if pt is not None else 0, kk.shape[0] if pt is not None else 0,
        float(scale), _ptr(kv_cnt), _ptr(kv_idx), _ptr(out), _ptr(lse),
        (OUT_PAGED if out_paged else 0) | (PAIR_QBLOCKS if pair_qblocks else 0), _ptr(ws),
        _stream(q.device)))
    return out, lse


def append_paged_kv(k_new, v_new, cb: ChunkedBatch, paged: PagedKV, *, ws=None):
    """Writes the chunk's new K and V rows [total_q, Hkv, d] into the paged caches at their
    absolute positions (before the chunked prefill reads them)."""
    T, Hkv, d = k_new.shape
    _same_dtype(k_new, v_new, paged.k_cache, paged.v_cache)
    if T != cb.total_q:
        raise ValueError(f"the batch holds {cb.total_q} new rows but k_new has {T}")
    _expect(v_new, "v_new", (T, Hkv, d))
    _expect_paged(paged, d, cb.size, need_v=True)
    if paged.k_cache.shape[2] != Hkv:
        raise ValueError(f"k_cache holds {paged.k_cache.shape[2]} KV heads, k_new {Hkv}")
    ws = workspace(k_new.device) if ws is None else ws
    pt = paged.page_table
    _check(library().fp_append_paged_kv(
        _ptr(k_new), _ptr(v_new), _dtype_code(k_new), _ptr(cb.cu_q), _ptr(cb.cu_k), cb.size, T,
        Hkv, d, _ptr(pt), paged.page_size, pt.shape[1], paged.k_cache.shape[0],
        _ptr(paged.k_cache), _ptr(paged.v_cache), _ptr(ws), _stream(k_new.device)))


def sparse_prefill_chunked(q, k, v, cb: ChunkedBatch, alpha=0.1, *,
                           paged: PagedKV | None = None, scale=None, q_scale=None,
                           k_scale=None, v_scale=None, return_lse=False,
                           flags=FORCE_FIRST | FORCE_DIAG, out=None, out_paged=False):
    """The whole path for a chunked batch. Returns (out, lse or None, kv_cnt, kv_idx);
    ``out_paged`` as for ``sparse_prefill_attn_chunked``."""
    d = q.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    Hkv = (paged.k_cache if paged is not None else k).shape[-2]
    k_split = torch.empty(k_split_shape(Hkv, cb.total_kblocks, d), dtype=torch.bfloat16,
                          device=q.device)
    q_pool, k_pool = pool_qk_chunked(q, k, cb, q_scale=q_scale, k_scale=k_scale, paged=paged,
                                     k_split_out=k_split)
    _, kv_cnt, kv_idx = build_block_mask_chunked(q_pool, k_pool, cb, alpha, scale=scale,
                                                 flags=flags, mask_bits=False, k_split=k_split)
    out, lse = sparse_prefill_attn_chunked(q, k, v, kv_cnt, kv_idx, cb, paged=paged, scale=scale,
                                           q_scale=q_scale, k_scale=k_scale, v_scale=v_scale,
                                           return_lse=return_lse, out=out, out_paged=out_paged)
    return out, lse, kv_cnt, kv_idx


class HostPipeline:
    """Runs the path step after step on inputs and outputs in pinned host memory, overlapping
    each step's host-to-device copies and the previous step's device-to-host copy with the
    kernels (three CUDA streams: copy-in, compute, copy-out; ``depth`` device buffer sets).

    ``run(*device_inputs, out=device_out)`` enqueues one step on the current stream (e.g. a
    call of ``sparse_prefill`` with the layer's fixed arguments bound). ``submit`` copies the
    host inputs in, runs the step and copies its output back into ``host_out``; it returns at
    once. ``synchronize`` waits for every submitted step. Host tensors must not be changed
    until the step that reads or writes them has completed."""

    def __init__(self, run, input_like, out_like, device, depth=2):
        self.run = run
        self.device = torch.device(device)
        self.depth = depth
        self.h2d = torch.cuda.Stream(self.device)
        self.comp = torch.cuda.Stream(self.device)
        self.d2h = torch.cuda.Stream(self.device)
        self.dev_in = [[torch.empty(t.shape, dtype=t.dtype, device=self.device)
                        for t in input_like] for _ in range(depth)]
        self.dev_out = [torch.empty(out_like.shape, dtype=out_like.dtype, device=self.device)
                        for _ in range(depth)]
        self.in_free = [None] * depth    # compute of the step that last read buffer set i
        self.out_free = [None] * depth   # copy-out of the step that last wrote buffer set i
        self.n = 0

    def submit(self, host_inputs, host_out):
        i = self.n % self.depth
        self.n += 1
        ev_in, ev_done, ev_out = (torch.cuda.Event() for _ in range(3))
        with torch.cuda.stream(self.h2d):
            if self.in_free[i] is not None:
                self.h2d.wait_event(self.in_free[i])
            for d, h in zip(self.dev_in[i], host_inputs):
                d.copy_(h, non_blocking=True)
            ev_in.record(self.h2d)
        with torch.cuda.stream(self.comp):
            self.comp.wait_event(ev_in)
            if self.out_free[i] is not None:
                self.comp.wait_event(self.out_free[i])
            self.run(*self.dev_in[i], out=self.dev_out[i])
            ev_done.record(self.comp)
        with torch.cuda.stream(self.d2h):
            self.d2h.wait_event(ev_done)
            host_out.copy_(self.dev_out[i], non_blocking=True)
            ev_out.record(self.d2h)
        self.in_free[i] = ev_done
        self.out_free[i] = ev_out

    def synchronize(self):
        for st in (self.h2d, self.comp, self.d2h):
            st.synchronize()


class GraphStep:
    """One step of the path captured into a CUDA graph: ``run(*inputs)`` (device tensors of
    fixed shape, the call's other arguments bound) is run ``warmup`` times eagerly, then
    captured; ``replay()`` relaunches all of its kernels at once and returns the tensors the
    captured call returned. New data goes into the captured input tensors in place
    (``inputs[i].copy_(...)``) before a replay. The library's calls allocate nothing on the
    device and never synchronise, so they capture as they are."""

    def __init__(self, run, inputs, warmup=2):
        self.inputs = tuple(inputs)
        dev = self.inputs[0].device
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            for _ in range(warmup):
                run(*self.inputs)
        torch.cuda.current_stream(dev).wait_stream(side)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.outputs = run(*self.inputs)

    def replay(self):
        self.graph.replay()
        return self.outputs
