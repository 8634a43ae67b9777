// Stage 2: pooled block scores, max-based dynamic threshold, block mask and index lists.
//
// "FlashPrefill: Instantaneous Pattern Discovery and Thresholding for Ultra-Fast Long-Context
// Prefilling", technical summary 2.B: per query block I the pruning threshold is alpha times
// the largest pooled score of the row over J <= I; there is no sort and no top-k. With Score
// read as the softmax probability of the pooled row, p_J >= alpha * max p is the same test as
// s_J - max s >= ln(alpha) on the scaled pooled logits, which is what runs here (the softmax
// denominator cancels, so no exponential is needed).
//
// Used when the caller asks for fp32 scores (FP_MASK_FP32), as an independent implementation of
// the same stage next to the tensor-core kernel in mask_tc.cu.
//
// One CTA owns R = G * NB rows: the G query heads that share KV head g, times NB consecutive
// global query blocks. It streams the KV head's pooled keys through shared memory in chunks
// of 64 blocks, so every pooled key row is read from L2 once per CTA and reused by all R rows,
// and keeps the R score rows in shared memory (fp32 FFMA: the threshold compare must hold to
// well under 1e-3 in log space). Then one warp per row takes the row max with shuffles, forms
// the keep bits 32 blocks at a time with a ballot, and compacts the kept indices with popc.
#include <math.h>

#include "fp_common.cuh"
#include "fp_launch.h"

namespace fp {

constexpr int kMaskThreads = 256;
constexpr int kMaskChunk = 64;  // pooled key blocks per shared-memory chunk

__host__ __device__ inline int mask_pad(int d) { return d + 4; }  // row stride, conflict-free

__host__ inline size_t mask_smem_bytes(int R, int d, int max_blocks) {
  return sizeof(float) * (static_cast<size_t>(R) * mask_pad(d) +
                          static_cast<size_t>(kMaskChunk) * mask_pad(d) +
                          static_cast<size_t>(R) * max_blocks) +
         sizeof(int) * 4 * R;
}

__global__ void __launch_bounds__(kMaskThreads) mask_kernel(MaskArgs a) {
  extern __shared__ float4 smem_f4[];
  float* sm = reinterpret_cast<float*>(smem_f4);
  const int R = a.G * a.NB;
  const int dp = mask_pad(a.d);
  float* sq = sm;                                  // [R][dp]
  float* sk = sq + static_cast<size_t>(R) * dp;    // [kMaskChunk][dp]
  float* ss = sk + static_cast<size_t>(kMaskChunk) * dp;  // [R][max_kb]
  int* row_I = reinterpret_cast<int*>(ss + static_cast<size_t>(R) * a.s.max_kb);
  int* row_kb = row_I + R;    // global block index of the row's request block 0
  int* row_h = row_kb + R;
  int* row_g = row_h + R;     // global query block (-1 if past the end)

  const int g = blockIdx.y;
  const int Ig0 = blockIdx.x * a.NB;
  const int tid = threadIdx.x;
  // A timeout recorded in the caller's status word is sticky: do nothing (decided by one read
  // for the whole block).
  const bool stale = tid == 0 && a.status != nullptr &&
                     (*reinterpret_cast<volatile uint32_t*>(a.status) & kStatusTimeout);
  if (__syncthreads_or(stale ? 1 : 0)) return;

  // Row bookkeeping.
  for (int r = tid; r < R; r += kMaskThreads) {
    const int Ig = Ig0 + r / a.G;
    const int h = g * a.G + r % a.G;
    if (Ig < a.s.total_qb) {
      const QBlock qb = query_block(a.s, Ig);
      row_I[r] = qb.ok ? qb.I : -2;  // absolute query block: keys J = 0 .. I of the request
      row_kb[r] = qb.kb0;  // global KV block of the request's block 0
      row_g[r] = Ig;
    } else {
      row_I[r] = -1;
      row_kb[r] = 0;
      row_g[r] = -1;
    }
    row_h[r] = h;
  }
  // Pooled queries of the R rows.
  const int d4 = a.d / 4;
  for (int i = tid; i < R * d4; i += kMaskThreads) {
    const int r = i / d4, c = (i % d4) * 4;
    const int Ig = Ig0 + r / a.G;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (Ig < a.s.total_qb)
      v = __ldg(reinterpret_cast<const float4*>(
          a.q_pool + (static_cast<size_t>(g * a.G + r % a.G) * a.s.total_qb + Ig) * a.d + c));
    *reinterpret_cast<float4*>(sq + r * dp + c) = v;
  }
  __syncthreads();

  // Key-block range this CTA needs: from block 0 of its first row's request to the diagonal
  // block of its last row. With prefix sums that do not describe the requests consistently a
  // row may fall outside it (or be refused outright): the CTA then records kStatusBadIndex and
  // touches nothing.
  const int r_last = (min(Ig0 + a.NB, a.s.total_qb) - 1 - Ig0) * a.G;
  const int Jg_lo = row_kb[0];
  const int Jg_hi = row_kb[r_last] + row_I[r_last];
  bool bad = false;
  for (int r = tid; r < R; r += kMaskThreads)
    bad |= row_I[r] == -2 || (row_g[r] >= 0 && (row_kb[r] < Jg_lo || row_kb[r] + row_I[r] > Jg_hi));
  if (__syncthreads_or(bad ? 1 : 0)) {
    if (tid == 0) record_status(a.status, kStatusBadIndex);
    return;
  }

  // Thread -> (key column within the chunk, row group); rows rg, rg + 4, ... of the R rows.
  const int col = tid % kMaskChunk;
  const int rg = tid / kMaskChunk;
  constexpr int kRowGroups = kMaskThreads / kMaskChunk;  // 4

  for (int Jg0 = Jg_lo; Jg0 <= Jg_hi; Jg0 += kMaskChunk) {
    const int nchunk = min(kMaskChunk, Jg_hi - Jg0 + 1);
    __syncthreads();  // previous chunk fully consumed
    for (int i = tid; i < kMaskChunk * d4; i += kMaskThreads) {
      const int j = i / d4, c = (i % d4) * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j < nchunk)
        v = __ldg(reinterpret_cast<const float4*>(
            a.k_pool + (static_cast<size_t>(g) * a.s.total_kb + Jg0 + j) * a.d + c));
      *reinterpret_cast<float4*>(sk + j * dp + c) = v;
    }
    __syncthreads();
    if (col < nchunk) {
      const int Jg = Jg0 + col;
      const float* kr = sk + col * dp;
      for (int r0 = rg; r0 < R; r0 += kRowGroups * 8) {
        float acc[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) acc[u] = 0.f;
        for (int c = 0; c < a.d; c += 4) {
          const float4 kv = *reinterpret_cast<const float4*>(kr + c);
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int r = r0 + u * kRowGroups;
            if (r < R) {
              const float4 qv = *reinterpret_cast<const float4*>(sq + r * dp + c);
              acc[u] = fmaf(qv.x, kv.x, acc[u]);
              acc[u] = fmaf(qv.y, kv.y, acc[u]);
              acc[u] = fmaf(qv.z, kv.z, acc[u]);
              acc[u] = fmaf(qv.w, kv.w, acc[u]);
            }
          }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int r = r0 + u * kRowGroups;
          if (r < R && row_g[r] >= 0) {
            const int J = Jg - row_kb[r];
            if (J >= 0 && J <= row_I[r]) ss[static_cast<size_t>(r) * a.s.max_kb + J] = acc[u] * a.scale;
          }
        }
      }
    }
  }
  __syncthreads();

  // Threshold, bits and compaction: one warp per row.
  const int warp = tid / 32, lane = tid % 32;
  const int words = (a.s.max_kb + 31) / 32;
  for (int r = warp; r < R; r += kMaskThreads / 32) {
    const int Ig = row_g[r];
    if (Ig < 0) continue;
    const int I = row_I[r];
    const int h = row_h[r];
    const float* srow = ss + static_cast<size_t>(r) * a.s.max_kb;
    float m = -INFINITY;
    for (int J = lane; J <= I; J += 32) m = fmaxf(m, srow[J]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const size_t row = static_cast<size_t>(h) * a.s.total_qb + Ig;
    int32_t* idx = a.kv_idx + row * a.s.max_kb;
    int cnt = 0;
    for (int w = 0; w < words; ++w) {
      const int J = w * 32 + lane;
      bool keep = false;
      if (J <= I) {
        keep = (srow[J] - m >= a.log_alpha) || ((a.flags & FP_FORCE_FIRST) && J == 0) ||
               ((a.flags & FP_FORCE_DIAG) && J == I);
      }
      const uint32_t bits = __ballot_sync(0xffffffffu, keep);
      if (a.mask_bits != nullptr && lane == 0) a.mask_bits[row * words + w] = bits;
      if (keep) idx[cnt + __popc(bits & ((1u << lane) - 1u))] = J;
      cnt += __popc(bits);
    }
    if (lane == 0) a.kv_cnt[row] = cnt;
  }
}

// Picks NB (query blocks per CTA) so that R = G * NB <= 32 rows and the score rows fit in
// about 112 KB of shared memory (two CTAs per SM). Returns 0 if even NB = 1 does not fit.
int mask_blocks_per_cta(int G, int d, int max_blocks) {
  int nb = G >= 32 ? 1 : 32 / G;
  while (nb > 1 && mask_smem_bytes(G * nb, d, max_blocks) > 112 * 1024) nb /= 2;
  if (mask_smem_bytes(G * nb, d, max_blocks) > 200 * 1024) return 0;
  return nb;
}

cudaError_t launch_mask(const MaskArgs& in, cudaStream_t stream) {
  if (!(in.flags & FP_MASK_FP32) && mask_tc_supported(in.G, in.d))
    return launch_mask_tc(in, stream);
  MaskArgs a = in;
  const size_t smem = mask_smem_bytes(a.G * a.NB, a.d, a.s.max_kb);
  cudaError_t e = cudaFuncSetAttribute(mask_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((a.s.total_qb + a.NB - 1) / a.NB, a.Hkv);
  mask_kernel<<<grid, kMaskThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace fp
