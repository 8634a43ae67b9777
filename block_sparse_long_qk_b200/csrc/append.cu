// Chunked prefill, the step before attention: the new chunk's K and V rows are written into
// the paged KV cache at their absolute positions ("FlashPrefill V2: Block-Sparse Prefill
// Attention for Long-Context LLM Serving", Abstract: paged KV cache and continuous batching).
//
// Pure data movement: one CTA per new token row, each thread moving 16-byte units of the
// row's Hkv x d elements from the contiguous chunk to (page, slot) of the cache, K and V.
#include "fp_common.cuh"
#include "fp_launch.h"

namespace fp {

constexpr int kAppendThreads = 128;

__global__ void __launch_bounds__(kAppendThreads) append_kernel(AppendArgs a) {
  const int t = blockIdx.x;  // new row
  if (t >= a.s.total_q) return;
  const int b = seqs_find(a.s.cu_q, a.s.batch, t);
  const int q0 = __ldg(a.s.cu_q + b);
  const int n = __ldg(a.s.cu_q + b + 1) - q0;
  const int L = __ldg(a.s.cu_k + b + 1) - __ldg(a.s.cu_k + b);
  const int p = L - n + (t - q0);  // absolute position of the row
  const int lp = p / a.page_size;
  int page = -1;
  if (p >= 0 && lp < a.max_pages) page = __ldg(a.page_table + static_cast<size_t>(b) * a.max_pages + lp);
  if (page < 0 || page >= a.num_pages) {
    if (threadIdx.x == 0) record_status(a.status, kStatusBadIndex);
    return;
  }
  const size_t dst_row = static_cast<size_t>(page) * a.page_size + p % a.page_size;
  const int units = a.row_bytes / 16;
  const int4* ks = reinterpret_cast<const int4*>(a.k_new + static_cast<size_t>(t) * a.row_bytes);
  const int4* vs = reinterpret_cast<const int4*>(a.v_new + static_cast<size_t>(t) * a.row_bytes);
  int4* kd = reinterpret_cast<int4*>(a.k_cache + dst_row * a.row_bytes);
  int4* vd = reinterpret_cast<int4*>(a.v_cache + dst_row * a.row_bytes);
  for (int u = threadIdx.x; u < units; u += blockDim.x) {
    const int4 kv = __ldcs(ks + u), vv = __ldcs(vs + u);
    kd[u] = kv;
    vd[u] = vv;
  }
}

cudaError_t launch_append(const AppendArgs& a, cudaStream_t stream) {
  if (a.s.total_q == 0) return cudaSuccess;
  append_kernel<<<a.s.total_q, kAppendThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace fp
