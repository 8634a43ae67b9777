// extern "C" entry points of libfpsparse.so: argument checks, then one kernel launch each.
// Declarations and the contract of every call are in include/fpsparse.h.
#include <atomic>
#include <limits.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>

#include <initializer_list>
#include <string>
#include <utility>

#include "fp_common.cuh"
#include "fp_launch.h"

namespace {

thread_local std::string g_err;
thread_local int g_fault_skip_k = -1;  // one-shot test hook for the next attention call
thread_local int g_fault_skip_mask = -1;  // one-shot test hook for the next mask call

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(FP_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The workspace holds the status word; NULL is allowed where the call says so.
int check_workspace(const void* workspace) {
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(FP_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  return FP_OK;
}

// The small index arrays (prefix sums, page tables) are the arguments most easily left in
// host memory by a caller; a kernel reading one would fault the GPU. Each non-NULL one must
// be memory the device can address. While `stream` is being captured into a CUDA graph the
// query is skipped (it is not a stream operation; the same call run eagerly checks it).
int check_device_arrays(void* stream,
                        std::initializer_list<std::pair<const void*, const char*>> arrays) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(static_cast<cudaStream_t>(stream), &cs) != cudaSuccess) {
    cudaGetLastError();
    cs = cudaStreamCaptureStatusNone;
  }
  if (cs != cudaStreamCaptureStatusNone) return FP_OK;
  for (const auto& a : arrays) {
    if (a.first == nullptr) continue;
    cudaPointerAttributes at{};
    const cudaError_t e = cudaPointerGetAttributes(&at, a.first);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return fail(FP_ERR_INVALID_ARG, "%s: cannot query the pointer (%s)", a.second,
                  cudaGetErrorString(e));
    }
    if (at.type == cudaMemoryTypeUnregistered || at.devicePointer == nullptr)
      return fail(FP_ERR_INVALID_ARG, "%s is host memory; pass device memory", a.second);
  }
  return FP_OK;
}

// Shared checks of the varlen description and head layout.
int check_common(int dtype, const float* qs, const float* ks, const float* vs, bool need_v,
                 const int32_t* cu_seqlens, const int32_t* cu_blocks, int batch,
                 int total_tokens, int total_blocks, int Hq, int Hkv, int d, int block) {
  if (dtype != FP_DTYPE_BF16 && dtype != FP_DTYPE_E4M3)
    return fail(FP_ERR_INVALID_ARG, "dtype %d is neither FP_DTYPE_BF16 nor FP_DTYPE_E4M3", dtype);
  if (dtype == FP_DTYPE_BF16 && (qs || ks || vs))
    return fail(FP_ERR_INVALID_ARG, "bf16 inputs take no scales (pass NULL)");
  if (dtype == FP_DTYPE_E4M3 && (!qs || !ks || (need_v && !vs)))
    return fail(FP_ERR_INVALID_ARG, "e4m3 inputs need per-head scales");
  if (d != 64 && d != 128) return fail(FP_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", d);
  if (block != 64 && block != 128)
    return fail(FP_ERR_UNSUPPORTED, "block %d (supported: 64, 128)", block);
  if (batch < 1) return fail(FP_ERR_INVALID_ARG, "batch must be >= 1 (got %d)", batch);
  if (batch > 1 && (!cu_seqlens || !cu_blocks))
    return fail(FP_ERR_INVALID_ARG, "batch > 1 needs cu_seqlens and cu_blocks");
  if ((cu_seqlens == nullptr) != (cu_blocks == nullptr))
    return fail(FP_ERR_INVALID_ARG, "cu_seqlens and cu_blocks are both given or both NULL");
  if (total_tokens < 0 || total_blocks < 0)
    return fail(FP_ERR_INVALID_ARG, "negative token or block count");
  if (cu_blocks == nullptr && total_blocks != (total_tokens + block - 1) / block)
    return fail(FP_ERR_INVALID_ARG, "total_blocks %d != ceil(T / block) for one sequence",
                total_blocks);
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0)
    return fail(FP_ERR_INVALID_ARG, "Hq (%d) must be a positive multiple of Hkv (%d)", Hq, Hkv);
  return FP_OK;
}

}  // namespace

namespace fp {
EncodeTiledFn tensor_map_encoder() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

int set_error(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}
}  // namespace fp

extern "C" {

int fp_version(void) { return 300; }

const char* fp_last_error_string(void) { return g_err.c_str(); }

size_t fp_workspace_size(void) { return 256; }

}  // extern "C"

namespace {

// The varlen description of plain prefill: queries and keys are the same rows.
fp::Seqs plain_seqs(const int32_t* cu_seqlens, const int32_t* cu_blocks, int batch,
                    int total_tokens, int total_blocks, int max_blocks, int block) {
  fp::Seqs s{};
  s.cu_q = s.cu_k = cu_seqlens;
  s.cu_qb = s.cu_kb = cu_blocks;
  s.batch = batch;
  s.total_q = s.total_k = total_tokens;
  s.total_qb = s.total_kb = total_blocks;
  s.max_kb = max_blocks;
  s.block = block;
  return s;
}

// Checks of a chunked varlen description (all four prefix-sum arrays are required).
int check_chunked(const int32_t* cu_q, const int32_t* cu_qblocks, const int32_t* cu_k,
                  const int32_t* cu_kblocks, int batch, int total_q, int total_k, int total_qb,
                  int total_kb, int max_kb) {
  if (batch < 1) return fail(FP_ERR_INVALID_ARG, "batch must be >= 1 (got %d)", batch);
  if (!cu_q || !cu_qblocks || !cu_k || !cu_kblocks)
    return fail(FP_ERR_INVALID_ARG, "chunked prefill needs cu_q, cu_qblocks, cu_k, cu_kblocks");
  if (total_q < 0 || total_k < 0 || total_qb < 0 || total_kb < 0 || max_kb < 0)
    return fail(FP_ERR_INVALID_ARG, "negative token or block count");
  if (total_q > total_k)
    return fail(FP_ERR_INVALID_ARG, "total_q %d exceeds total_k %d", total_q, total_k);
  if (total_qb > total_kb)
    return fail(FP_ERR_INVALID_ARG, "total_qblocks %d exceeds total_kblocks %d", total_qb,
                total_kb);
  if (total_kb > 0 && max_kb < 1) return fail(FP_ERR_INVALID_ARG, "bad block counts");
  return FP_OK;
}

int check_paging(const int32_t* page_table, int page_size, int max_pages, int num_pages,
                 int block) {
  if (page_table &&
      (page_size < 16 || page_size % 16 || block % page_size || max_pages < 1 || num_pages < 1))
    return fail(FP_ERR_INVALID_ARG,
                "page_size %d must be a multiple of 16 dividing block %d, and max_pages (%d) "
                "and num_pages (%d) at least 1", page_size, block, max_pages, num_pages);
  return FP_OK;
}

int pool_impl(const void* q, const void* k, int dtype, const float* q_scale,
              const float* k_scale, const fp::Seqs& s, int Hq, int Hkv, int d,
              const int32_t* k_page_table, int page_size, int max_pages, int num_pages,
              float* q_pool, float* k_pool, void* k_pool_split, void* workspace, void* stream) {
  if (!q || !k || !q_pool || !k_pool) return fail(FP_ERR_INVALID_ARG, "null tensor pointer");
  if (check_workspace(workspace)) return FP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q_pool) || !aligned16(k_pool) ||
      !aligned16(k_pool_split))
    return fail(FP_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  int rc = check_paging(k_page_table, page_size, max_pages, num_pages, s.block);
  if (rc) return rc;
  if (k_page_table && s.cu_k == nullptr)
    return fail(FP_ERR_INVALID_ARG, "a paged K needs the varlen prefix sums");
  if (s.total_kb == 0) return FP_OK;
  rc = check_device_arrays(stream, {{s.cu_q, "cu_q / cu_seqlens"},
                                    {s.cu_qb, "cu_qblocks / cu_blocks"}, {s.cu_k, "cu_k"},
                                    {s.cu_kb, "cu_kblocks"}, {k_page_table, "k_page_table"},
                                    {workspace, "workspace"}});
  if (rc) return rc;
  fp::PoolArgs a{};
  a.status = static_cast<uint32_t*>(workspace);
  a.q = static_cast<const uint8_t*>(q);
  a.k = static_cast<const uint8_t*>(k);
  a.q_scale = q_scale;
  a.k_scale = k_scale;
  a.page_table = k_page_table;
  a.q_pool = q_pool;
  a.k_pool = k_pool;
  a.k_split = static_cast<__nv_bfloat16*>(k_pool_split);
  a.s = s;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.d = d;
  a.page_size = page_size;
  a.max_pages = max_pages;
  a.num_pages = num_pages;
  cudaError_t e = fp::launch_pool(a, dtype == FP_DTYPE_E4M3, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FP_OK : cuda_fail(e, "pool kernel launch");
}

int mask_impl(const float* q_pool, const float* k_pool, const void* k_pool_split,
              const fp::Seqs& s, int Hq, int Hkv, int d, float alpha, float scale, int flags,
              uint32_t* mask_bits, int32_t* kv_cnt, int32_t* kv_idx, void* workspace,
              void* stream) {
  const int skip_chunk = g_fault_skip_mask;
  g_fault_skip_mask = -1;
  if (!q_pool || !k_pool || !kv_cnt || !kv_idx) return fail(FP_ERR_INVALID_ARG, "null pointer");
  if (check_workspace(workspace)) return FP_ERR_INVALID_ARG;
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv)
    return fail(FP_ERR_INVALID_ARG, "Hq (%d) must be a positive multiple of Hkv (%d)", Hq, Hkv);
  if (d != 64 && d != 128) return fail(FP_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", d);
  if (!(alpha >= 0.f && alpha <= 1.f)) return fail(FP_ERR_INVALID_ARG, "alpha must be in [0, 1]");
  if (!aligned16(q_pool) || !aligned16(k_pool) || !aligned16(k_pool_split))
    return fail(FP_ERR_INVALID_ARG, "pooled tensors must be 16-byte aligned");
  if (s.total_qb == 0) return FP_OK;
  int rc = check_device_arrays(stream, {{s.cu_q, "cu_q"}, {s.cu_qb, "cu_qblocks / cu_blocks"},
                                        {s.cu_k, "cu_k"}, {s.cu_kb, "cu_kblocks"},
                                        {workspace, "workspace"}});
  if (rc) return rc;
  const int G = Hq / Hkv;
  const int nb = fp::mask_blocks_per_cta(G, d, s.max_kb);
  const bool fp32 = (flags & FP_MASK_FP32) != 0 || !fp::mask_tc_supported(G, d);
  if (fp32 && nb == 0)
    return fail(FP_ERR_UNSUPPORTED, "%d blocks per request with %d heads per KV head exceed the "
                "shared-memory score rows of the fp32 mask kernel", s.max_kb, G);
  fp::MaskArgs a{};
  a.q_pool = q_pool;
  a.k_pool = k_pool;
  a.k_split = k_pool_split;
  a.mask_bits = mask_bits;
  a.kv_cnt = kv_cnt;
  a.kv_idx = kv_idx;
  a.status = static_cast<uint32_t*>(workspace);
  a.fault_skip_chunk = skip_chunk;
  a.s = s;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.d = d;
  a.G = G;
  a.NB = nb;
  a.log_alpha = alpha > 0.f ? logf(alpha) : -INFINITY;
  a.scale = scale;
  a.flags = flags;
  cudaError_t e = fp::launch_mask(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FP_OK : cuda_fail(e, "mask kernel launch");
}

// SMs of the calling thread's current device (cached per device; 148 if the query fails).
int device_sm_count() {
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n <= 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

int attn_impl(const void* q, const void* k, const void* v, int dtype, const float* q_scale,
              const float* k_scale, const float* v_scale, const fp::Seqs& s, int Hq, int Hkv,
              int d, const int32_t* page_table, int page_size, int max_pages, int num_pages,
              float scale, const int32_t* kv_cnt, const int32_t* kv_idx, void* out, float* lse,
              int out_flags, void* workspace, void* stream) {
  if (!q || !k || !v || !out || !kv_cnt || !kv_idx || !workspace)
    return fail(FP_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return fail(FP_ERR_INVALID_ARG, "Q, K, V and out must be 16-byte aligned");
  if (check_workspace(workspace)) return FP_ERR_INVALID_ARG;
  if (dtype == FP_DTYPE_E4M3 && !(d == 128 && s.block == 128))
    return fail(FP_ERR_UNSUPPORTED, "e4m3 attention supports d = 128, block = 128");
  int rc = check_paging(page_table, page_size, max_pages, num_pages, s.block);
  if (rc) return rc;
  if (page_table && s.cu_k == nullptr)
    return fail(FP_ERR_INVALID_ARG, "paged attention needs the varlen prefix sums");
  if (out_flags & ~(FP_OUT_PAGED | FP_PAIR_QBLOCKS))
    return fail(FP_ERR_INVALID_ARG, "unknown flags %d", out_flags);
  if ((out_flags & FP_OUT_PAGED) && !page_table)
    return fail(FP_ERR_INVALID_ARG, "FP_OUT_PAGED writes through the K/V page table: pass one");
  const int G = Hq / Hkv;
  fp::AttnArgs a{};
  a.kv_cnt = kv_cnt;
  a.kv_idx = kv_idx;
  a.page_table = page_table;
  a.q_scale = q_scale;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.lse = lse;
  a.status = static_cast<uint32_t*>(workspace);
  a.s = s;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.page_size = page_size;
  a.max_pages = max_pages;
  a.num_pages = num_pages;
  a.G = G;
  // Two heads of a GQA group per CTA. A head left over (odd G, all heads for G = 1) runs alone
  // in its CTA or pairs two neighbouring query blocks: pairing halves those heads' CTAs and
  // makes each ~1.2x longer, which pays once their single tiles would fill the GPU at least
  // twice (with fewer, SMs would idle); FP_PAIR_QBLOCKS pairs query blocks for every head.
  // Head-pair kernel: Hkv * ceil(G / 2) items per query block (the odd head alone). General
  // split: per level of two query blocks and KV head, head_pairs items at each block and
  // qpair_heads over both (at the last level of an odd total_qb the second block's head pairs
  // have no work and end at once).
  const long long single_items = static_cast<long long>(Hkv) * ((G + 1) / 2) * s.total_qb;
  const bool pair_q = (out_flags & FP_PAIR_QBLOCKS) ||
                      (G % 2 == 1 && single_items >= 2LL * device_sm_count());
  a.head_pairs = (out_flags & FP_PAIR_QBLOCKS) ? 0 : G / 2;
  a.qpair_heads = pair_q ? G - 2 * a.head_pairs : 0;
  {
    const long long levels = (static_cast<long long>(s.total_qb) + 1) / 2;
    const long long items =
        a.qpair_heads == 0 ? single_items
                           : levels * Hkv * (2 * a.head_pairs + a.qpair_heads);
    if (items > INT_MAX) return fail(FP_ERR_INVALID_ARG, "too many attention work items");
    a.num_items = static_cast<int>(items);
  }
  a.scale_log2 = scale * 1.4426950408889634f;
  a.fault_skip_k = g_fault_skip_k;
  a.out_paged = (out_flags & FP_OUT_PAGED) ? 1 : 0;
  g_fault_skip_k = -1;
  fp::AttnLaunch L{};
  L.q = q;
  L.k = k;
  L.v = v;
  L.e4m3 = dtype == FP_DTYPE_E4M3;
  L.paged = page_table != nullptr;
  L.d = d;
  L.kv_rows = page_table ? static_cast<long long>(num_pages) * page_size : s.total_k;
  L.seg_rows = page_table ? page_size : s.block;
  if (s.total_qb == 0) return FP_OK;
  rc = check_device_arrays(stream, {{s.cu_q, "cu_q / cu_seqlens"},
                                    {s.cu_qb, "cu_qblocks / cu_blocks"}, {s.cu_k, "cu_k"},
                                    {s.cu_kb, "cu_kblocks"}, {page_table, "page_table"},
                                    {kv_cnt, "kv_cnt"}, {kv_idx, "kv_idx"},
                                    {workspace, "workspace"}});
  if (rc) return rc;
  cudaError_t e = fp::launch_attn(a, L, s.block, static_cast<cudaStream_t>(stream));
  if (e == cudaErrorNotSupported) return fail(FP_ERR_UNSUPPORTED, "unsupported d/block/dtype");
  return e == cudaSuccess ? FP_OK : cuda_fail(e, "attention kernel launch");
}

}  // namespace

extern "C" {

int fp_pool_qk(const void* q, const void* k, int dtype, const float* q_scale,
               const float* k_scale, const int32_t* cu_seqlens, const int32_t* cu_blocks,
               int batch, int total_tokens, int total_blocks, int Hq, int Hkv, int d,
               int block, const int32_t* k_page_table, int page_size, int max_pages,
               int num_pages, float* q_pool, float* k_pool, void* k_pool_split,
               void* workspace, void* stream) {
  g_err.clear();
  int rc = check_common(dtype, q_scale, k_scale, nullptr, false, cu_seqlens, cu_blocks, batch,
                        total_tokens, total_blocks, Hq, Hkv, d, block);
  if (rc) return rc;
  return pool_impl(q, k, dtype, q_scale, k_scale,
                   plain_seqs(cu_seqlens, cu_blocks, batch, total_tokens, total_blocks,
                              total_blocks, block),
                   Hq, Hkv, d, k_page_table, page_size, max_pages, num_pages, q_pool, k_pool,
                   k_pool_split, workspace, stream);
}

int fp_build_block_mask(const float* q_pool, const float* k_pool, const void* k_pool_split,
                        const int32_t* cu_blocks, int batch, int total_blocks, int max_blocks,
                        int Hq, int Hkv, int d, float alpha, float scale, int flags,
                        uint32_t* mask_bits, int32_t* kv_cnt, int32_t* kv_idx, void* workspace,
                        void* stream) {
  g_err.clear();
  if (batch < 1 || (batch > 1 && !cu_blocks))
    return fail(FP_ERR_INVALID_ARG, "batch > 1 needs cu_blocks");
  if (total_blocks < 0 || max_blocks < 0 || (total_blocks > 0 && max_blocks < 1))
    return fail(FP_ERR_INVALID_ARG, "bad block counts");
  if (cu_blocks == nullptr && max_blocks != total_blocks)
    return fail(FP_ERR_INVALID_ARG, "one sequence: max_blocks must equal total_blocks");
  // The mask needs only block indices: with no token counts, the query and key block lists of
  // a plain prefill coincide (P0 = 0), which the block prefix sums alone describe.
  const fp::Seqs s = plain_seqs(cu_blocks, cu_blocks, batch, total_blocks, total_blocks,
                                max_blocks, 1);
  return mask_impl(q_pool, k_pool, k_pool_split, s, Hq, Hkv, d, alpha, scale, flags, mask_bits,
                   kv_cnt, kv_idx, workspace, stream);
}

int fp_sparse_prefill_attn(const void* q, const void* k, const void* v, int dtype,
                           const float* q_scale, const float* k_scale, const float* v_scale,
                           const int32_t* cu_seqlens, const int32_t* cu_blocks, int batch,
                           int total_tokens, int total_blocks, int max_blocks, int Hq,
                           int Hkv, int d, int block, float scale, const int32_t* kv_cnt,
                           const int32_t* kv_idx, void* out, float* lse, void* workspace,
                           void* stream) {
  g_err.clear();
  int rc = check_common(dtype, q_scale, k_scale, v_scale, true, cu_seqlens, cu_blocks, batch,
                        total_tokens, total_blocks, Hq, Hkv, d, block);
  if (rc) return rc;
  if (cu_blocks == nullptr && max_blocks != total_blocks)
    return fail(FP_ERR_INVALID_ARG, "one sequence: max_blocks must equal total_blocks");
  return attn_impl(q, k, v, dtype, q_scale, k_scale, v_scale,
                   plain_seqs(cu_seqlens, cu_blocks, batch, total_tokens, total_blocks,
                              max_blocks, block),
                   Hq, Hkv, d, nullptr, 0, 0, 0, scale, kv_cnt, kv_idx, out, lse, 0, workspace,
                   stream);
}

int fp_sparse_prefill_attn_paged(const void* q, const void* k_cache, const void* v_cache,
                                 int dtype, const float* q_scale, const float* k_scale,
                                 const float* v_scale, const int32_t* cu_seqlens,
                                 const int32_t* cu_blocks, int batch, int total_tokens,
                                 int total_blocks, int max_blocks, int Hq, int Hkv, int d,
                                 int block, const int32_t* page_table, int page_size,
                                 int max_pages, int num_pages, float scale,
                                 const int32_t* kv_cnt, const int32_t* kv_idx, void* out,
                                 float* lse, void* workspace, void* stream) {
  g_err.clear();
  if (!page_table) return fail(FP_ERR_INVALID_ARG, "paged attention needs a page table");
  int rc = check_common(dtype, q_scale, k_scale, v_scale, true, cu_seqlens, cu_blocks, batch,
                        total_tokens, total_blocks, Hq, Hkv, d, block);
  if (rc) return rc;
  if (cu_blocks == nullptr && max_blocks != total_blocks)
    return fail(FP_ERR_INVALID_ARG, "one sequence: max_blocks must equal total_blocks");
  return attn_impl(q, k_cache, v_cache, dtype, q_scale, k_scale, v_scale,
                   plain_seqs(cu_seqlens, cu_blocks, batch, total_tokens, total_blocks,
                              max_blocks, block),
                   Hq, Hkv, d, page_table, page_size, max_pages, num_pages, scale, kv_cnt,
                   kv_idx, out, lse, 0, workspace, stream);
}

static fp::Seqs chunked_seqs(const int32_t* cu_q, const int32_t* cu_qblocks,
                             const int32_t* cu_k, const int32_t* cu_kblocks, int batch,
                             int total_q, int total_k, int total_qblocks, int total_kblocks,
                             int max_kblocks, int block) {
  fp::Seqs s{};
  s.cu_q = cu_q;
  s.cu_qb = cu_qblocks;
  s.cu_k = cu_k;
  s.cu_kb = cu_kblocks;
  s.batch = batch;
  s.total_q = total_q;
  s.total_k = total_k;
  s.total_qb = total_qblocks;
  s.total_kb = total_kblocks;
  s.max_kb = max_kblocks;
  s.block = block;
  return s;
}

int fp_pool_qk_chunked(const void* q, const void* k, int dtype, const float* q_scale,
                       const float* k_scale, const int32_t* cu_q, const int32_t* cu_qblocks,
                       const int32_t* cu_k, const int32_t* cu_kblocks, int batch, int total_q,
                       int total_k, int total_qblocks, int total_kblocks, int Hq, int Hkv,
                       int d, int block, const int32_t* k_page_table, int page_size,
                       int max_pages, int num_pages, float* q_pool, float* k_pool,
                       void* k_pool_split, void* workspace, void* stream) {
  g_err.clear();
  int rc = check_common(dtype, q_scale, k_scale, nullptr, false, cu_q, cu_qblocks, batch,
                        total_q, total_qblocks, Hq, Hkv, d, block);
  if (rc) return rc;
  rc = check_chunked(cu_q, cu_qblocks, cu_k, cu_kblocks, batch, total_q, total_k, total_qblocks,
                     total_kblocks, total_kblocks > 0 ? 1 : 0);
  if (rc) return rc;
  // The pool kernel needs no per-row list length: any request's block count is at most
  // total_kblocks.
  return pool_impl(q, k, dtype, q_scale, k_scale,
                   chunked_seqs(cu_q, cu_qblocks, cu_k, cu_kblocks, batch, total_q, total_k,
                                total_qblocks, total_kblocks, total_kblocks, block),
                   Hq, Hkv, d, k_page_table, page_size, max_pages, num_pages, q_pool, k_pool,
                   k_pool_split, workspace, stream);
}

int fp_build_block_mask_chunked(const float* q_pool, const float* k_pool,
                                const void* k_pool_split, const int32_t* cu_q,
                                const int32_t* cu_qblocks, const int32_t* cu_k,
                                const int32_t* cu_kblocks, int batch, int total_qblocks,
                                int total_kblocks, int max_kblocks, int Hq, int Hkv, int d,
                                int block, float alpha, float scale, int flags,
                                uint32_t* mask_bits, int32_t* kv_cnt, int32_t* kv_idx,
                                void* workspace, void* stream) {
  g_err.clear();
  if (block != 64 && block != 128)
    return fail(FP_ERR_UNSUPPORTED, "block %d (supported: 64, 128)", block);
  int rc = check_chunked(cu_q, cu_qblocks, cu_k, cu_kblocks, batch, 0, 0, total_qblocks,
                         total_kblocks, max_kblocks);
  if (rc) return rc;
  // The mask reads no token rows, and this call is not given the token totals: the device-side
  // checks of the prefix sums bound the rows by INT_MAX and the blocks by the totals passed.
  return mask_impl(q_pool, k_pool, k_pool_split,
                   chunked_seqs(cu_q, cu_qblocks, cu_k, cu_kblocks, batch, INT_MAX, INT_MAX,
                                total_qblocks, total_kblocks, max_kblocks, block),
                   Hq, Hkv, d, alpha, scale, flags, mask_bits, kv_cnt, kv_idx, workspace,
                   stream);
}

int fp_sparse_prefill_attn_chunked(const void* q, const void* k, const void* v, int dtype,
                                   const float* q_scale, const float* k_scale,
                                   const float* v_scale, const int32_t* cu_q,
                                   const int32_t* cu_qblocks, const int32_t* cu_k,
                                   const int32_t* cu_kblocks, int batch, int total_q,
                                   int total_k, int total_qblocks, int total_kblocks,
                                   int max_kblocks, int Hq, int Hkv, int d, int block,
                                   const int32_t* page_table, int page_size, int max_pages,
                                   int num_pages, float scale, const int32_t* kv_cnt,
                                   const int32_t* kv_idx, void* out, float* lse, int out_flags,
                                   void* workspace, void* stream) {
  g_err.clear();
  int rc = check_common(dtype, q_scale, k_scale, v_scale, true, cu_q, cu_qblocks, batch,
                        total_q, total_qblocks, Hq, Hkv, d, block);
  if (rc) return rc;
  rc = check_chunked(cu_q, cu_qblocks, cu_k, cu_kblocks, batch, total_q, total_k, total_qblocks,
                     total_kblocks, max_kblocks);
  if (rc) return rc;
  return attn_impl(q, k, v, dtype, q_scale, k_scale, v_scale,
                   chunked_seqs(cu_q, cu_qblocks, cu_k, cu_kblocks, batch, total_q, total_k,
                                total_qblocks, total_kblocks, max_kblocks, block),
                   Hq, Hkv, d, page_table, page_size, max_pages, num_pages, scale, kv_cnt,
                   kv_idx, out, lse, out_flags, workspace, stream);
}

int fp_append_paged_kv(const void* k_new, const void* v_new, int dtype, const int32_t* cu_q,
                       const int32_t* cu_k, int batch, int total_q, int Hkv, int d,
                       const int32_t* page_table, int page_size, int max_pages, int num_pages,
                       void* k_cache, void* v_cache, void* workspace, void* stream) {
  g_err.clear();
  if (dtype != FP_DTYPE_BF16 && dtype != FP_DTYPE_E4M3)
    return fail(FP_ERR_INVALID_ARG, "dtype %d is neither FP_DTYPE_BF16 nor FP_DTYPE_E4M3", dtype);
  if (d != 64 && d != 128) return fail(FP_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", d);
  if (batch < 1 || Hkv < 1 || total_q < 0)
    return fail(FP_ERR_INVALID_ARG, "batch and Hkv must be >= 1, total_q >= 0");
  if (!k_new || !v_new || !cu_q || !cu_k || !page_table || !k_cache || !v_cache || !workspace)
    return fail(FP_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(FP_ERR_INVALID_ARG, "K/V rows and caches must be 16-byte aligned");
  if (check_workspace(workspace)) return FP_ERR_INVALID_ARG;
  if (page_size < 1 || max_pages < 1 || num_pages < 1)
    return fail(FP_ERR_INVALID_ARG, "page_size, max_pages and num_pages must be >= 1");
  if (total_q == 0) return FP_OK;
  int rc = check_device_arrays(stream, {{cu_q, "cu_q"}, {cu_k, "cu_k"},
                                        {page_table, "page_table"}, {workspace, "workspace"}});
  if (rc) return rc;
  fp::AppendArgs a{};
  a.k_new = static_cast<const uint8_t*>(k_new);
  a.v_new = static_cast<const uint8_t*>(v_new);
  a.k_cache = static_cast<uint8_t*>(k_cache);
  a.v_cache = static_cast<uint8_t*>(v_cache);
  a.page_table = page_table;
  a.status = static_cast<uint32_t*>(workspace);
  a.s.cu_q = cu_q;
  a.s.cu_k = cu_k;
  a.s.batch = batch;
  a.s.total_q = total_q;
  a.row_bytes = Hkv * d * (dtype == FP_DTYPE_E4M3 ? 1 : 2);
  a.page_size = page_size;
  a.max_pages = max_pages;
  a.num_pages = num_pages;
  cudaError_t e = fp::launch_append(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FP_OK : cuda_fail(e, "append kernel launch");
}

int fp_debug_skip_k_load(int union_block) {
  g_err.clear();
  if (union_block < 0) return fail(FP_ERR_INVALID_ARG, "union block index must be >= 0");
  g_fault_skip_k = union_block;
  return FP_OK;
}

int fp_debug_skip_mask_load(int chunk) {
  g_err.clear();
  if (chunk < 0) return fail(FP_ERR_INVALID_ARG, "chunk index must be >= 0");
  g_fault_skip_mask = chunk;
  return FP_OK;
}

int fp_check_status(void* workspace, void* stream) {
  g_err.clear();
  if (!workspace) return fail(FP_ERR_INVALID_ARG, "null workspace");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "reading the status word");
  if (word != 0) {
    e = cudaMemsetAsync(workspace, 0, sizeof(word), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the status word");
  }
  if (word & fp::kStatusTimeout)
    return fail(FP_ERR_TIMEOUT, "a pipeline wait in the mask or attention kernel timed out");
  if (word & fp::kStatusBadIndex)
    return fail(FP_ERR_BAD_INDEX, "an index list, page table entry or prefix sum was out of "
                "range or inconsistent");
  return FP_OK;
}

}  // extern "C"
