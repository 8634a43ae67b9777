// Argument structs and host launchers shared by the kernel files and the C ABI (internal).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace fp {

// A varlen batch whose queries may be a suffix of each request (chunked / prefix-cached
// prefill): request b holds kv_len_b = cu_k[b+1] - cu_k[b] keys and q_len_b query rows, the
// queries being the last q_len_b positions P0_b = kv_len_b - q_len_b .. kv_len_b - 1. Blocks
// are defined on absolute positions: the request's KV blocks are 0 .. ceil(kv_len/block) - 1,
// its query blocks run from I0_b = P0_b / block to the same last block. With cu_q == nullptr
// the batch is one sequence of total_q = total_k tokens (P0 = 0). The entry points for plain
// prefill pass the same arrays for queries and keys (P0 = 0 everywhere).
struct Seqs {
  const int32_t* cu_q;   // [batch + 1] query rows
  const int32_t* cu_qb;  // [batch + 1] query blocks
  const int32_t* cu_k;   // [batch + 1] key rows
  const int32_t* cu_kb;  // [batch + 1] key blocks
  int batch, total_q, total_k, total_qb, total_kb, max_kb, block;
};

struct PoolArgs {
  const uint8_t* q;
  const uint8_t* k;
  const float* q_scale;
  const float* k_scale;
  const int32_t* page_table;
  float* q_pool;           // [Hq][total_qb][d]
  float* k_pool;           // [Hkv][total_kb][d]
  __nv_bfloat16* k_split;  // optional bf16 [2][Hkv][total_kb][d] hi / lo parts of k_pool
  uint32_t* status;        // caller's status word, or nullptr (nothing recorded)
  Seqs s;
  int Hq, Hkv, d, page_size, max_pages, num_pages;
  int q_slices;  // column slices of Q per block (the rest of gridDim.y are K slices)
};

struct MaskArgs {
  const float* q_pool;
  const float* k_pool;
  const void* k_split;  // bf16 [2][Hkv][total_kb][d] hi / lo parts of k_pool, or nullptr
  uint32_t* mask_bits;  // [Hq][total_qb][ceil(max_kb / 32)]
  int32_t* kv_cnt;      // [Hq][total_qb]
  int32_t* kv_idx;      // [Hq][total_qb][max_kb]
  uint32_t* status;     // caller's status word, or nullptr (nothing recorded)
  Seqs s;
  int Hq, Hkv, d, G, NB;
  int fault_skip_chunk;  // test hook: CTA 0 skips the B-operand TMA load of this chunk
  float log_alpha;  // -inf for alpha = 0
  float scale;
  int flags;
};

struct AttnArgs {
  const int32_t* kv_cnt;
  const int32_t* kv_idx;
  const int32_t* page_table;
  const float* q_scale;
  const float* k_scale;
  const float* v_scale;
  __nv_bfloat16* out;
  float* lse;
  uint32_t* status;
  Seqs s;
  int Hq, Hkv;
  int page_size, max_pages, num_pages;  // paged only
  int G;                               // query heads per KV head
  int head_pairs;                       // per KV head: head pairs (two heads, one query block)
  int qpair_heads;                      // per KV head: heads paired over two query blocks; 0
                                        // selects the head-pair kernel (odd G: last head alone)
  int num_items;                        // CTAs (make_tiles / make_tiles_qp in attn.cu)
  int fault_skip_k;                     // test hook: CTA 0 skips the K load of this union block
  int out_paged;                        // out is [num_pages, page_size, Hq, d] via page_table
  float scale_log2;                     // softmax scale * log2(e)
};

struct AppendArgs {
  const uint8_t* k_new;  // [total_q, Hkv, d] rows of the new chunk
  const uint8_t* v_new;
  uint8_t* k_cache;      // [num_pages, page_size, Hkv, d]
  uint8_t* v_cache;
  const int32_t* page_table;  // [batch, max_pages]
  uint32_t* status;
  Seqs s;
  int row_bytes;  // Hkv * d * element size
  int page_size, max_pages, num_pages;
};

struct AttnLaunch {
  const void *q, *k, *v;
  bool e4m3, paged;
  int d;
  long long kv_rows;  // rows of the K/V tensor map (total_k, or num_pages * page_size)
  int seg_rows;       // rows per K/V TMA box (block, or page_size)
};

cudaError_t launch_pool(const PoolArgs& a, bool e4m3, cudaStream_t stream);
cudaError_t launch_mask(const MaskArgs& a, cudaStream_t stream);
int mask_blocks_per_cta(int G, int d, int max_kb);
bool mask_tc_supported(int G, int d);   // tensor-core scores (mask_tc.cu) apply
cudaError_t launch_mask_tc(const MaskArgs& a, cudaStream_t stream);
cudaError_t launch_attn(const AttnArgs& a, const AttnLaunch& L, int block, cudaStream_t stream);
cudaError_t launch_append(const AppendArgs& a, cudaStream_t stream);

// cuTensorMapEncodeTiled, looked up once through the runtime (no link against libcuda).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);
EncodeTiledFn tensor_map_encoder();

// Records a printf-style message for fp_last_error_string() on this thread; returns `code`.
int set_error(int code, const char* fmt, ...);

}  // namespace fp

namespace fp {

// Query block gq of a batch: request b, absolute block index I, the request's first query
// position P0 and key count L, the query row holding absolute position P0 (qrow0), the key row
// of position 0 (kbase) and the global KV block of the request's block 0 (kb0). `ok` is false
// when the prefix sums of request b do not describe it consistently (see seqs_request_ok);
// then nothing of the block may be read or written.
struct QBlock {
  int b, I, P0, L, qrow0, kbase, kb0;
  bool ok;
};

#ifdef __CUDACC__
__device__ __forceinline__ int seqs_find(const int32_t* cu, int batch, int x) {
  int lo = 0, hi = batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(cu + mid) <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// The prefix sums are caller data that the host does not read. Before a kernel derives rows
// from the entries of request b it checks that they describe a request the buffers can hold:
// query blocks qb0 <= g < qb1 <= total_qb (g the block being mapped), query rows q0 .. q1 - 1
// within [0, total_q) and at least one of them, key rows k0 .. k1 - 1 within [0, total_k) and
// at least as many as queries, ceil(L / block) KV blocks at kb0 .. kb1 - 1 within [0, total_kb)
// and at most max_kb of them, and ceil(L / block) - floor(P0 / block) query blocks. 64-bit
// arithmetic, so that no sum of caller values overflows.
__device__ __forceinline__ bool seqs_request_ok(const Seqs& s, long long g, long long qb0,
                                                long long qb1, long long q0, long long q1,
                                                long long k0, long long k1, long long kb0,
                                                long long kb1) {
  const long long nq = q1 - q0, L = k1 - k0;
  if (!(qb0 <= g && g < qb1 && qb1 <= s.total_qb)) return false;
  if (!(q0 >= 0 && nq >= 1 && q1 <= s.total_q)) return false;
  if (!(k0 >= 0 && L >= nq && k1 <= s.total_k)) return false;
  const long long nkb = (L + s.block - 1) / s.block;
  if (!(kb0 >= 0 && kb1 - kb0 == nkb && kb1 <= s.total_kb && nkb <= s.max_kb)) return false;
  return qb1 - qb0 == nkb - (L - nq) / s.block;
}

__device__ __forceinline__ QBlock query_block(const Seqs& s, int gq) {
  QBlock r;
  r.ok = true;
  if (s.cu_q == nullptr) {
    r.b = 0; r.P0 = 0; r.L = s.total_k; r.qrow0 = 0; r.kbase = 0; r.kb0 = 0; r.I = gq;
    return r;
  }
  r.b = seqs_find(s.cu_qb, s.batch, gq);
  const int qb0 = __ldg(s.cu_qb + r.b), qb1 = __ldg(s.cu_qb + r.b + 1);
  r.qrow0 = __ldg(s.cu_q + r.b);
  const int q1 = __ldg(s.cu_q + r.b + 1);
  r.kbase = __ldg(s.cu_k + r.b);
  const int k1 = __ldg(s.cu_k + r.b + 1);
  r.kb0 = __ldg(s.cu_kb + r.b);
  const int kb1 = __ldg(s.cu_kb + r.b + 1);
  r.ok = seqs_request_ok(s, gq, qb0, qb1, r.qrow0, q1, r.kbase, k1, r.kb0, kb1);
  if (!r.ok) {
    r.b = 0; r.P0 = 0; r.L = 0; r.qrow0 = 0; r.kbase = 0; r.kb0 = 0; r.I = 0;
    return r;
  }
  const int nq = q1 - r.qrow0;
  r.L = k1 - r.kbase;
  r.P0 = r.L - nq;
  r.I = r.P0 / s.block + (gq - qb0);
  return r;
}

// KV block gk of a batch: request b, block index J, key count L, key row of position 0; `ok`
// as for QBlock (key blocks kb0 <= gk < kb1 <= total_kb, ceil(L / block) of them, key rows
// within [0, total_k)).
struct KBlock {
  int b, J, L, kbase;
  bool ok;
};

__device__ __forceinline__ KBlock key_block(const Seqs& s, int gk) {
  KBlock r;
  r.ok = true;
  if (s.cu_k == nullptr) {
    r.b = 0; r.J = gk; r.L = s.total_k; r.kbase = 0;
    return r;
  }
  r.b = seqs_find(s.cu_kb, s.batch, gk);
  const long long kb0 = __ldg(s.cu_kb + r.b), kb1 = __ldg(s.cu_kb + r.b + 1);
  const long long k0 = __ldg(s.cu_k + r.b), k1 = __ldg(s.cu_k + r.b + 1);
  const long long L = k1 - k0;
  r.ok = kb0 <= gk && gk < kb1 && kb1 <= s.total_kb && k0 >= 0 && L >= 1 && k1 <= s.total_k &&
         kb1 - kb0 == (L + s.block - 1) / s.block;
  if (!r.ok) {
    r.b = 0; r.J = 0; r.L = 0; r.kbase = 0;
    return r;
  }
  r.kbase = static_cast<int>(k0);
  r.L = static_cast<int>(L);
  r.J = gk - static_cast<int>(kb0);
  return r;
}
#endif

}  // namespace fp
