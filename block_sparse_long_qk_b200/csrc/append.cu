// Chunked prefill, the step before attention: the new chunk's K and V rows are written into
// the paged KV cache at their absolute positions ("FlashPrefill V2: Block-Sparse Prefill
// Attention for Long-Context LLM Serving", Abstract: paged KV cache and continuous batching).
//
// Pure data movement: one CTA per 8 new token rows, each thread moving 16-byte units of the
// rows' Hkv x d elements from the contiguous chunk to (page, slot) of the cache, K and V, with
// the 8 rows' loads in flight together.
#include "fp_common.cuh"
#include "fp_launch.h"

namespace fp {

constexpr int kAppendThreads = 128;
constexpr int kAppendRows = 8;  // new rows per CTA, their loads in flight together

// Destination row of new row t in the cache, or -1 (and the status bit) when its page entry is
// out of range or the prefix sums of its request are inconsistent (q0 <= t < q1 and at most as
// many new rows as keys).
__device__ __forceinline__ long long append_dst_row(const AppendArgs& a, int t) {
  const int b = seqs_find(a.s.cu_q, a.s.batch, t);
  const int q0 = __ldg(a.s.cu_q + b);
  const int n = __ldg(a.s.cu_q + b + 1) - q0;
  const int L = __ldg(a.s.cu_k + b + 1) - __ldg(a.s.cu_k + b);
  if (!(q0 <= t && t - q0 < n && n <= L)) return -1;
  const int p = L - n + (t - q0);  // absolute position of the row
  const int lp = p / a.page_size;
  int page = -1;
  if (p >= 0 && lp < a.max_pages)
    page = __ldg(a.page_table + static_cast<size_t>(b) * a.max_pages + lp);
  if (page < 0 || page >= a.num_pages) return -1;
  return static_cast<long long>(page) * a.page_size + p % a.page_size;
}

__global__ void __launch_bounds__(kAppendThreads) append_kernel(AppendArgs a) {
  const int t0 = blockIdx.x * kAppendRows;
  const int units = a.row_bytes / 16;
  __shared__ long long dst[kAppendRows];
  if (threadIdx.x < kAppendRows) {
    const int t = t0 + threadIdx.x;
    long long d = -2;  // past the end of the chunk: nothing to do
    if (t < a.s.total_q) {
      d = append_dst_row(a, t);
      if (d < 0) record_status(a.status, kStatusBadIndex);
    }
    dst[threadIdx.x] = d;
  }
  __syncthreads();
  for (int u = threadIdx.x; u < units; u += blockDim.x) {
    int4 kv[kAppendRows], vv[kAppendRows];
#pragma unroll
    for (int r = 0; r < kAppendRows; ++r) {
      if (dst[r] >= 0) {
        const size_t src = (static_cast<size_t>(t0 + r) * a.row_bytes) / 16 + u;
        kv[r] = __ldcs(reinterpret_cast<const int4*>(a.k_new) + src);
        vv[r] = __ldcs(reinterpret_cast<const int4*>(a.v_new) + src);
      }
    }
#pragma unroll
    for (int r = 0; r < kAppendRows; ++r) {
      if (dst[r] >= 0) {
        const size_t o = (static_cast<size_t>(dst[r]) * a.row_bytes) / 16 + u;
        reinterpret_cast<int4*>(a.k_cache)[o] = kv[r];
        reinterpret_cast<int4*>(a.v_cache)[o] = vv[r];
      }
    }
  }
}

cudaError_t launch_append(const AppendArgs& a, cudaStream_t stream) {
  if (a.s.total_q == 0) return cudaSuccess;
  const int grid = (a.s.total_q + kAppendRows - 1) / kAppendRows;
  append_kernel<<<grid, kAppendThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace fp
