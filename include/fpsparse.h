/*
 * fpsparse -- block-sparse causal prefill attention for NVIDIA B200 (sm_100a).
 *
 * C ABI of libfpsparse.so. The three stages of the method, each one CUDA kernel:
 *
 *   fp_pool_qk               block means of Q and K            ("FlashPrefill: Instantaneous
 *                            Pattern Discovery and Thresholding for Ultra-Fast Long-Context
 *                            Prefilling", technical summary 2.A, block approximation and the
 *                            fused 2-D reduction)
 *   fp_build_block_mask      pooled block scores, max-based dynamic threshold, KV-block mask
 *                            and index lists                    (same page, 2.B)
 *   fp_sparse_prefill_attn   causal attention over the kept KV blocks only, index-based
 *                            physical skip                      (same page, 2.C; GQA packing,
 *                            FP8 and paged KV with continuous batching from "FlashPrefill V2:
 *                            Block-Sparse Prefill Attention for Long-Context LLM Serving",
 *                            Abstract)
 *   fp_sparse_prefill_attn_paged   the same with K/V read through a page table
 *   fp_*_chunked             the three stages for chunked / prefix-cached prefill, where each
 *                            request's queries are the last q_len of its kv_len positions
 *   fp_append_paged_kv       writes a chunk's new K/V rows into the paged cache first
 *
 * Conventions for every call:
 *  - Every pointer argument is a DEVICE pointer unless its comment says "host". The caller
 *    owns all memory; the library allocates nothing on these paths. Inputs are read only.
 *  - Token-major activations: Q is [T, Hq, d], K and V are [T, Hkv, d], row-major and
 *    contiguous (element (t, h, c) at ((t * H) + h) * d + c). T is the total token count of
 *    the batch. Query head h reads KV head h / (Hq / Hkv) (grouped-query attention).
 *  - Varlen batches: cu_seqlens is int32 [batch + 1] (cu[0] = 0, cu[batch] = T, ascending)
 *    and cu_blocks is int32 [batch + 1] with cu_blocks[b+1] - cu_blocks[b] =
 *    ceil((cu[b+1] - cu[b]) / block). Blocks restart at each request's first token; a
 *    request's last block may be partial. For one sequence pass batch = 1 and both pointers
 *    NULL. "Global block" Ig indexes the blocks of all requests in order (0 .. total_blocks).
 *  - dtype is FP_DTYPE_BF16 or FP_DTYPE_E4M3. For e4m3 storage the real value of an element
 *    is code * scale[head], with one float32 scale per head (q_scale [Hq], k_scale and
 *    v_scale [Hkv]); for bf16 the scale pointers must be NULL.
 *  - All work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default stream)
 *    and is asynchronous. Argument errors are reported before anything is enqueued.
 *  - Return value: FP_OK (0) or a negative FP_ERR_* code; fp_last_error_string() then holds
 *    a message for the calling thread. Nothing throws across this boundary.
 *  - Faults found on the device (an index or page-table entry out of range, prefix sums that
 *    do not describe the batch consistently, a pipeline wait that ran out) are recorded in the
 *    status word of the caller's `workspace` (fp_workspace_size() bytes of device memory,
 *    256-byte aligned, zeroed once before first use) and read with fp_check_status. The
 *    kernels never turn such a fault into an out-of-range access: the affected block is
 *    skipped and its outputs are left unwritten or incomplete. For the pool and mask calls the
 *    workspace may be NULL (then nothing is recorded); the attention and append calls require
 *    it. One workspace shared by the calls of a step reports the whole step.
 *  - Prefix sums are read on the device only. Each block a kernel maps checks the entries of
 *    its own request: rows and blocks within the totals passed, a non-empty query range no
 *    longer than the key range, and block counts equal to the ceil-divisions stated below (and
 *    at most max_blocks). A violation is FP_ERR_BAD_INDEX.
 */
#ifndef FPSPARSE_H_
#define FPSPARSE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FP_OK 0
#define FP_ERR_INVALID_ARG (-1)  /* a size, pointer or alignment the call cannot accept */
#define FP_ERR_UNSUPPORTED (-2)  /* a valid configuration that this build does not cover */
#define FP_ERR_CUDA (-3)         /* a CUDA runtime or driver call failed */
#define FP_ERR_TIMEOUT (-4)      /* a kernel pipeline wait ran out (reported by fp_check_status) */
#define FP_ERR_BAD_INDEX (-5)    /* an index list or page table entry out of range (fp_check_status) */

#define FP_DTYPE_BF16 0
#define FP_DTYPE_E4M3 1

#define FP_FORCE_FIRST 1 /* always keep KV block 0 of every row */
#define FP_FORCE_DIAG 2  /* always keep the diagonal KV block J = I */
#define FP_MASK_FP32 4   /* pooled scores in fp32 FFMA instead of the tensor cores (slower; the
                            same keep rule, a second implementation to cross-check) */

#define FP_OUT_PAGED 1   /* out_flags of fp_sparse_prefill_attn_chunked: write O in the paged
                            layout of the K/V cache (see there) */
#define FP_PAIR_QBLOCKS 2 /* out_flags of fp_sparse_prefill_attn_chunked: every CTA pairs two
                            neighbouring query blocks of one head instead of two heads of a GQA
                            group (see the work split under fp_sparse_prefill_attn) */

/* Library version, e.g. 300 for 0.3.0. 0.1.1 added the chunked-prefill calls, the paged K/V
 * append and FP_MASK_FP32; 0.2.0 gives the pool and mask calls a workspace (status word) and
 * checks the prefix sums on the device; 0.3.0 pairs query blocks where heads cannot be paired
 * (G = 1, the last head of an odd G) and adds FP_PAIR_QBLOCKS. */
int fp_version(void);

/* Message describing the last error returned on the calling thread ("" if none). */
const char* fp_last_error_string(void);

/*
 * Stage 1: block-mean pooling ("FlashPrefill: Instantaneous Pattern Discovery ...",
 * technical summary 2.A: keys averaged per block; queries read the same way).
 *
 *   q_pool[h, Ig, :] = mean over the valid tokens i of block Ig of Q[i, h, :] * q_scale[h]
 *   k_pool[g, Ig, :] = mean over the valid tokens j of block Ig of K[j, g, :] * k_scale[g]
 *
 * q, k       Q [T, Hq, d], K [T, Hkv, d] in `dtype`; with k_page_table != NULL, k is instead
 *            a paged cache [num_pages, page_size, Hkv, d] and token t of request b lives in
 *            page k_page_table[b * max_pages + t / page_size], slot t % page_size; entries
 *            outside [0, num_pages) and pages past max_pages are not read (those tokens count
 *            as zeros).
 * q_pool     float32 [Hq, total_blocks, d] (written)
 * k_pool     float32 [Hkv, total_blocks, d] (written)
 * k_pool_split  NULL, or bf16 [2, Hkv, total_blocks, d] (written): hi = bf16(k_pool) and
 *            lo = bf16(k_pool - hi), the operand split fp_build_block_mask feeds to the tensor
 *            cores; passing it on to fp_build_block_mask saves that call the conversion.
 * workspace  NULL, or the status workspace: an out-of-range page entry (those tokens then
 *            count as zeros) or an inconsistent request (its blocks are not written) records
 *            FP_ERR_BAD_INDEX.
 * Supported: d in {64, 128}; block in {64, 128}; Hq % Hkv == 0; page_size a multiple of 16
 * that divides block. Q and K must be 16-byte aligned.
 */
int fp_pool_qk(const void* q, const void* k, int dtype, const float* q_scale,
               const float* k_scale, const int32_t* cu_seqlens, const int32_t* cu_blocks,
               int batch, int total_tokens, int total_blocks, int Hq, int Hkv, int d,
               int block, const int32_t* k_page_table, int page_size, int max_pages,
               int num_pages, float* q_pool, float* k_pool, void* k_pool_split,
               void* workspace, void* stream);

/*
 * Stage 2: pooled block scores and the max-based dynamic threshold ("FlashPrefill:
 * Instantaneous Pattern Discovery ...", technical summary 2.B: thresh_I = alpha *
 * max_{J<=I} Score_{I,J}, no sort and no top-k).
 *
 * Per head h and request-local query block I (global row Ig), over the causal blocks J <= I
 * of the same request:
 *   s_J  = scale * dot(q_pool[h, Ig], k_pool[h / (Hq/Hkv), cu_blocks[b] + J])   (float32)
 *   keep J  iff  s_J - max_J s_J >= ln(alpha)          (= softmax(s)_J >= alpha * max softmax)
 *           or (flags & FP_FORCE_FIRST and J == 0) or (flags & FP_FORCE_DIAG and J == I).
 * flags may also hold FP_MASK_FP32 (fp32 FFMA scores instead of the tensor cores; that kernel
 * keeps a request's score rows in shared memory, so very long requests with it return
 * FP_ERR_UNSUPPORTED).
 * alpha in [0, 1]; alpha = 0 keeps every causal block.
 *
 * k_pool_split  NULL, or the split written by fp_pool_qk for this k_pool (results are
 *            identical either way; with it the scores' operands are loaded, not converted)
 * mask_bits  uint32 [Hq, total_blocks, words], words = ceil(max_blocks / 32): bit J % 32 of
 *            word J / 32 is set iff block J is kept (bits above I are 0). May be NULL.
 * kv_cnt     int32 [Hq, total_blocks]: number of kept blocks of the row
 * kv_idx     int32 [Hq, total_blocks, max_blocks]: the kept request-local block indices in
 *            ascending order in the first kv_cnt entries (the rest is left untouched)
 * max_blocks largest per-request block count (host int)
 * workspace  NULL, or the status workspace: a bounded wait that runs out records
 *            FP_ERR_TIMEOUT (the lists of that call are then incomplete), inconsistent block
 *            prefix sums FP_ERR_BAD_INDEX (those rows are not written). A timeout recorded
 *            earlier in the workspace makes the call do nothing until fp_check_status clears it.
 */
int fp_build_block_mask(const float* q_pool, const float* k_pool, const void* k_pool_split,
                        const int32_t* cu_blocks, int batch, int total_blocks, int max_blocks,
                        int Hq, int Hkv, int d, float alpha, float scale, int flags,
                        uint32_t* mask_bits, int32_t* kv_cnt, int32_t* kv_idx, void* workspace,
                        void* stream);

/*
 * Stage 3: causal attention over the kept KV blocks only ("FlashPrefill: Instantaneous
 * Pattern Discovery ...", technical summary 2.C, index-based physical skip; GQA packing and
 * FP8 as in "FlashPrefill V2 ...", Abstract).
 *
 *   out[i, h, :] = sum_j softmax_j(scale * q_i . k_j) v_j   over the keys j <= i of the same
 *                  request whose block J = (j - cu[b]) / block is listed in
 *                  kv_idx[h, Ig, 0 .. kv_cnt[h, Ig]), Ig the global block of query i.
 *   lse[h, i]    = ln sum_j exp(scale * q_i . k_j) over the same keys (may be NULL).
 *
 * Index lists must be ascending, request-local and causal (0 <= J <= I); entries outside that
 * range are skipped and reported as FP_ERR_BAD_INDEX by fp_check_status.
 * q, k, v    as in fp_pool_qk (e4m3: per-head scales; the output is always bf16)
 * out        bf16 [T, Hq, d] (written)
 * lse        float32 [Hq, T] or NULL
 * workspace  at least fp_workspace_size() bytes of device memory, 256-byte aligned, holding
 *            the status word that fp_check_status reads. Concurrent calls need distinct
 *            workspaces.
 * Supported: d in {64, 128}; block in {64, 128} (e4m3: d = 128, block = 128);
 * Hq % Hkv == 0. Q, K, V must be 16-byte aligned.
 * Work split (the output is bit-identical whichever split runs: every tile accumulates its own
 * kept blocks in ascending order with the same instructions): each CTA runs two query tiles
 * that read the same KV head and loads every KV block either tile kept once. With G = Hq / Hkv
 * even, the tiles are two heads of a GQA group at one query block; the head an odd G leaves
 * over, and every head when G = 1, is paired with itself over two neighbouring query blocks
 * (cross-query reuse, "QUILT: Rethinking Sparse-Attention Prefill through Shared Query
 * Execution", Abstract) when those heads' single tiles would fill the GPU's SMs at least twice,
 * and runs one tile per CTA on smaller problems. FP_PAIR_QBLOCKS (chunked call) pairs query
 * blocks for every head.
 */
int fp_sparse_prefill_attn(const void* q, const void* k, const void* v, int dtype,
                           const float* q_scale, const float* k_scale, const float* v_scale,
                           const int32_t* cu_seqlens, const int32_t* cu_blocks, int batch,
                           int total_tokens, int total_blocks, int max_blocks, int Hq,
                           int Hkv, int d, int block, float scale, const int32_t* kv_cnt,
                           const int32_t* kv_idx, void* out, float* lse, void* workspace,
                           void* stream);

/*
 * Stage 3 with a paged KV cache and a continuous (varlen) batch ("FlashPrefill V2 ...",
 * Abstract: paged KV cache and continuous batching). Same definition as
 * fp_sparse_prefill_attn; K and V are read as caches [num_pages, page_size, Hkv, d] through
 * page_table int32 [batch, max_pages] (entry -1 or >= num_pages is FP_ERR_BAD_INDEX when it
 * would be read). page_size must be a multiple of 16 that divides block. Queries are
 * contiguous [T, Hq, d] with cu_seqlens (query length = KV length: prefill from scratch).
 */
int fp_sparse_prefill_attn_paged(const void* q, const void* k_cache, const void* v_cache,
                                 int dtype, const float* q_scale, const float* k_scale,
                                 const float* v_scale, const int32_t* cu_seqlens,
                                 const int32_t* cu_blocks, int batch, int total_tokens,
                                 int total_blocks, int max_blocks, int Hq, int Hkv, int d,
                                 int block, const int32_t* page_table, int page_size,
                                 int max_pages, int num_pages, float scale,
                                 const int32_t* kv_cnt, const int32_t* kv_idx, void* out,
                                 float* lse, void* workspace, void* stream);

/*
 * Chunked (prefix-cached) prefill. "FlashPrefill V2: Block-Sparse Prefill Attention for
 * Long-Context LLM Serving", Abstract: the kernels serve as the attention backend of a
 * continuous-batching engine with a paged KV cache. In such an engine a request's prefill may
 * run in chunks, or start after a cached prefix: its new queries are then the LAST q_len of
 * its kv_len positions, and they attend to the cached keys as well as to each other. These
 * three calls take the stages above to that case; with q_len = kv_len for every request they
 * compute exactly what the plain calls compute.
 *
 * Varlen description (all four arrays int32 [batch + 1], ascending from 0, device memory):
 *  - cu_k: key rows. Request b holds L_b = cu_k[b+1] - cu_k[b] keys (positions 0 .. L_b - 1);
 *    total_k = cu_k[batch].
 *  - cu_q: query rows. Request b holds n_b = cu_q[b+1] - cu_q[b] <= L_b queries, at positions
 *    P0_b = L_b - n_b .. L_b - 1 (causality aligned at the bottom right: query position p sees
 *    keys 0 .. p); total_q = cu_q[batch]. n_b = 0 is allowed (the request has no query block).
 *  - cu_kblocks: ceil(L_b / block) KV blocks per request (blocks of absolute positions,
 *    restarting at each request); total_kblocks = cu_kblocks[batch].
 *  - cu_qblocks: the query blocks of request b are the absolute blocks I = floor(P0_b / block)
 *    .. ceil(L_b / block) - 1, so cu_qblocks[b+1] - cu_qblocks[b] = ceil(L_b / block) -
 *    floor(P0_b / block) (0 when n_b = 0); total_qblocks = cu_qblocks[batch]. The first query
 *    block of a request may hold fewer than `block` queries (positions before P0_b belong to
 *    the prefix); the last one may too (positions past L_b).
 * Every array is indexed by global query block Ig (0 .. total_qblocks - 1) where the plain
 * calls use global block Ig, and key-side arrays by global KV block: q_pool [Hq,
 * total_qblocks, d], k_pool [Hkv, total_kblocks, d], k_pool_split bf16 [2, Hkv, total_kblocks,
 * d] (or NULL), mask_bits uint32 [Hq, total_qblocks, ceil(max_kblocks / 32)] (or NULL), kv_cnt
 * [Hq, total_qblocks], kv_idx [Hq, total_qblocks, max_kblocks] with max_kblocks >= the largest
 * ceil(L_b / block). Kept-block indices are request-local absolute KV blocks J = 0 .. I.
 * The host does not read the prefix sums: they must agree with the totals and with each other
 * as stated here (as cu_seqlens / cu_blocks must for the plain calls).
 *
 * fp_pool_qk_chunked: the pooled mean of query block I of request b runs over the queries it
 * holds (positions max(P0_b, I * block) .. min(L_b, (I + 1) * block) - 1); KV block J averages
 * the keys at positions J * block .. min(L_b, (J + 1) * block) - 1. K is contiguous [total_k,
 * Hkv, d] or, with k_page_table != NULL, the cache [num_pages, page_size, Hkv, d] read through
 * page_table int32 [batch, max_pages] (same rules as fp_pool_qk). Q is contiguous [total_q,
 * Hq, d].
 * fp_build_block_mask_chunked: row Ig (absolute block I of request b) scores KV blocks J = 0 ..
 * I of request b, with the same threshold, flags and outputs as fp_build_block_mask. `block` is
 * needed to place query blocks (64 or 128).
 * fp_sparse_prefill_attn_chunked: out [total_q, Hq, d] bf16 and lse [Hq, total_q] (or NULL) for
 * the queries only. K and V are contiguous [total_k, Hkv, d] (page_table NULL) or caches read
 * through page_table (same rules as fp_sparse_prefill_attn_paged). out_flags is a
 * combination of FP_PAIR_QBLOCKS (the work split above; the output is the same) and
 * FP_OUT_PAGED: with FP_OUT_PAGED out is instead a bf16 buffer [num_pages, page_size, Hq, d] in the page
 * layout of the K/V caches, and the output row of the query at absolute position p of request
 * b goes to slot p % page_size of page page_table[b * max_pages + p / page_size] (the page
 * table must be given; an entry out of range skips the row and records FP_ERR_BAD_INDEX; slots
 * that hold no new query are not written). The epilogue thus writes O where an engine keeping
 * per-token state in its KV page layout expects it, with no gather afterwards. lse stays
 * [Hq, total_q]. Errors and workspaces as fp_pool_qk, fp_build_block_mask and
 * fp_sparse_prefill_attn respectively.
 */
int fp_pool_qk_chunked(const void* q, const void* k, int dtype, const float* q_scale,
                       const float* k_scale, const int32_t* cu_q, const int32_t* cu_qblocks,
                       const int32_t* cu_k, const int32_t* cu_kblocks, int batch, int total_q,
                       int total_k, int total_qblocks, int total_kblocks, int Hq, int Hkv,
                       int d, int block, const int32_t* k_page_table, int page_size,
                       int max_pages, int num_pages, float* q_pool, float* k_pool,
                       void* k_pool_split, void* workspace, void* stream);

int fp_build_block_mask_chunked(const float* q_pool, const float* k_pool,
                                const void* k_pool_split, const int32_t* cu_q,
                                const int32_t* cu_qblocks, const int32_t* cu_k,
                                const int32_t* cu_kblocks, int batch, int total_qblocks,
                                int total_kblocks, int max_kblocks, int Hq, int Hkv, int d,
                                int block, float alpha, float scale, int flags,
                                uint32_t* mask_bits, int32_t* kv_cnt, int32_t* kv_idx,
                                void* workspace, void* stream);

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
                                   void* workspace, void* stream);

/*
 * Chunked prefill, the step before the three stages: writes the new chunk's K and V rows into
 * the paged KV cache ("FlashPrefill V2: Block-Sparse Prefill Attention for Long-Context LLM
 * Serving", Abstract: paged KV cache and continuous batching). Row t of request b (cu_q[b] <=
 * t < cu_q[b+1]) holds absolute position p = L_b - n_b + (t - cu_q[b]), with L_b = cu_k[b+1] -
 * cu_k[b] the request's key count after the append and n_b its new rows (the same description
 * as the fp_*_chunked calls); it is copied bit for bit to slot p % page_size of page
 * page_table[b][p / page_size] of k_cache and v_cache [num_pages, page_size, Hkv, d].
 * k_new, v_new  [total_q, Hkv, d], bf16 or e4m3 codes (dtype), 16-byte aligned
 * workspace     as for the attention calls; a page-table entry outside [0, num_pages) or a
 *               position past max_pages pages skips that row and records FP_ERR_BAD_INDEX
 *               (read with fp_check_status).
 * Supported: d in {64, 128}. Rows of different calls may target the same slots only if the
 * calls are ordered on one stream.
 */
int fp_append_paged_kv(const void* k_new, const void* v_new, int dtype, const int32_t* cu_q,
                       const int32_t* cu_k, int batch, int total_q, int Hkv, int d,
                       const int32_t* page_table, int page_size, int max_pages, int num_pages,
                       void* k_cache, void* v_cache, void* workspace, void* stream);

/*
 * fp_pool_qk followed by fp_build_block_mask, for callers that cannot allocate device memory.
 * The pages have no counterpart: this is a deployment variant of stages 1 and 2, with the same
 * arguments and results as those two calls, minus the q_pool / k_pool buffers.
 *
 * Who needs it: a serving engine that hands nearly all free HBM to its KV-cache pool at start-up
 * and must not allocate while serving; code that cannot afford the device synchronisation that
 * cudaMalloc / cudaFree imply; a host application that passes the library only preallocated
 * input and output buffers. The pooled means then live in a file-scope device array of this
 * library, 32 MiB per GPU that loads the library, held until the process exits.
 *
 * Limit: (Hq + Hkv) * total_blocks * d <= 8 Mi floats; larger problems return
 * FP_ERR_INVALID_ARG with a message (use the two regular calls with caller buffers). The first
 * call on each device looks up the array's device address (cudaGetSymbolAddress) with that
 * device current and keeps it for the life of the process; make that first call before any
 * stream capture, and do not call this entry on a device after cudaDeviceReset. All calls share
 * the array (each call rewrites the pooled values it reads, nothing needs clearing), so calls
 * whose work overlaps on the same GPU race. No device memory is allocated by this call.
 * Differences from the two regular calls: the mask kernel converts the pooled keys to its
 * tensor-core operands itself (there is no k_pool_split buffer to load them from), and there is
 * no workspace, so device-side faults are contained as in the other calls but not reported.
 */
int fp_pool_and_mask_noalloc(const void* q, const void* k, int dtype, const float* q_scale,
                             const float* k_scale, const int32_t* cu_seqlens,
                             const int32_t* cu_blocks, int batch, int total_tokens,
                             int total_blocks, int max_blocks, int Hq, int Hkv, int d, int block,
                             const int32_t* k_page_table, int page_size, int max_pages,
                             int num_pages, float alpha, float scale, int flags,
                             uint32_t* mask_bits, int32_t* kv_cnt, int32_t* kv_idx,
                             void* stream);

/*
 * Test hook for the failure path (the pages have no counterpart). Makes the NEXT attention
 * call issued from this thread skip, in its first CTA, the TMA load of K for the given union
 * block (0 = the first block that CTA visits). That CTA's bounded pipeline wait then runs out
 * after about 2 s and the call's workspace records FP_ERR_TIMEOUT (read it with
 * fp_check_status); nothing faults and the context stays usable. One-shot: later calls are
 * unaffected. Returns FP_ERR_INVALID_ARG for a negative index.
 */
int fp_debug_skip_k_load(int union_block);

/*
 * Test hook for the mask kernel's failure path (the pages have no counterpart). Makes the NEXT
 * fp_build_block_mask / fp_build_block_mask_chunked call issued from this thread that loads its
 * key operands by TMA (k_pool_split given) skip, in its first CTA, the load of the given chunk
 * of 128 key blocks (chunks of the first pass first). That CTA's bounded wait runs out after
 * about 2 s and the workspace records FP_ERR_TIMEOUT. One-shot; FP_ERR_INVALID_ARG for a
 * negative index.
 */
int fp_debug_skip_mask_load(int chunk);

/* Bytes of device workspace (the status word) the calls take (a fixed small size). */
size_t fp_workspace_size(void);

/*
 * Waits for `stream`, reads and clears the status word in `workspace`, and returns FP_OK,
 * FP_ERR_TIMEOUT or FP_ERR_BAD_INDEX (or FP_ERR_CUDA if the stream itself failed).
 * The workspace must have been zeroed once before its first use (e.g. cudaMemset).
 * A recorded timeout is sticky: mask and attention launches on that workspace do no work
 * (their CTAs exit at once) until this call has cleared it.
 */
int fp_check_status(void* workspace, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FPSPARSE_H_ */
