// Argument structs and host launchers shared by the kernel files and the C ABI (internal).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace fp {

struct PoolArgs {
  const uint8_t* q;
  const uint8_t* k;
  const float* q_scale;
  const float* k_scale;
  const int32_t* cu_seqlens;
  const int32_t* cu_blocks;
  const int32_t* page_table;
  float* q_pool;
  float* k_pool;
  __nv_bfloat16* k_split;  // optional bf16 [2][Hkv][total_blocks][d] hi / lo parts of k_pool
  int batch, total_tokens, total_blocks, Hq, Hkv, d, block, page_size, max_pages, num_pages;
  int q_slices;  // column slices of Q per block (the rest of gridDim.y are K slices)
};

struct MaskArgs {
  const float* q_pool;
  const float* k_pool;
  const void* k_split;  // bf16 [2][Hkv][total_blocks][d] hi / lo parts of k_pool, or nullptr
  const int32_t* cu_blocks;
  uint32_t* mask_bits;
  int32_t* kv_cnt;
  int32_t* kv_idx;
  int batch, total_blocks, max_blocks, Hq, Hkv, d, G, NB;
  float log_alpha;  // -inf for alpha = 0
  float scale;
  int flags;
};

struct AttnArgs {
  const int32_t* cu_seqlens;
  const int32_t* cu_blocks;
  const int32_t* kv_cnt;
  const int32_t* kv_idx;
  const int32_t* page_table;
  const float* q_scale;
  const float* k_scale;
  const float* v_scale;
  __nv_bfloat16* out;
  float* lse;
  uint32_t* status;
  int batch, total_tokens, total_blocks, max_blocks, Hq, Hkv, block;
  int page_size, max_pages, num_pages;  // paged only
  int pair_heads;                       // 1: the two tiles of a CTA are two heads of one block
  int num_items;
  int fault_skip_k;                     // test hook: CTA 0 skips the K load of this union block
  float scale_log2;                     // softmax scale * log2(e)
};

struct AttnLaunch {
  const void *q, *k, *v;
  bool e4m3, paged;
  int d;
  long long kv_rows;  // rows of the K/V tensor map (T, or num_pages * page_size)
  int seg_rows;       // rows per K/V TMA box (block, or page_size)
};

cudaError_t launch_pool(const PoolArgs& a, bool e4m3, cudaStream_t stream);
cudaError_t launch_mask(const MaskArgs& a, cudaStream_t stream);
int mask_blocks_per_cta(int G, int d, int max_blocks);
bool mask_tc_supported(int G, int d);   // tensor-core scores (mask_tc.cu) apply
cudaError_t launch_mask_tc(const MaskArgs& a, cudaStream_t stream);
cudaError_t launch_attn(const AttnArgs& a, const AttnLaunch& L, int block, cudaStream_t stream);

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
