// Stage 1: block-mean pooling of Q and K.
//
// "FlashPrefill: Instantaneous Pattern Discovery and Thresholding for Ultra-Fast Long-Context
// Prefilling", technical summary 2.A: keys are averaged per block (block approximation), and
// the query skeleton is read as block means of Q as well, so that the pooled score of stage 2
// equals the mean of the raw scaled Q K^T block (the fused 2-D reduction).
//
// Chunked prefill: query blocks hold only the request's query positions (see Seqs).
//
// Faults in the caller's data are never turned into out-of-range accesses: a block whose
// request the prefix sums do not describe consistently is skipped, and a paged token whose
// page entry is out of range counts as zeros; both record kStatusBadIndex in the caller's
// status word (read by fp_check_status).
//
// HBM-bound stream: every CTA owns one (global block, tensor, 2 KB-wide column slice) and
// its 128 threads each own 16 contiguous bytes of the token row (8 bf16 or 16 e4m3 values),
// walking the block's tokens with 8 independent 16-byte loads in flight per thread. A warp
// therefore reads 512 contiguous bytes of one token row per load. Accumulation is fp32.
#include "fp_common.cuh"
#include "fp_launch.h"

namespace fp {

constexpr int kPoolThreads = 128;

template <bool E4M3>
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(PoolArgs a) {
  constexpr int EPT = E4M3 ? 16 : 8;  // elements per thread (16 bytes)
  const int gb = blockIdx.x;
  const bool is_q = static_cast<int>(blockIdx.y) < a.q_slices;
  const int slice = is_q ? blockIdx.y : blockIdx.y - a.q_slices;
  const int H = is_q ? a.Hq : a.Hkv;
  const int cols = H * a.d;
  const int col = (slice * kPoolThreads + threadIdx.x) * EPT;
  if (col >= cols) return;

  // Query block gb: the query positions it holds (chunked prefill: only those at or after
  // the request's first query position P0). Key block gb: its keys, in a paged cache or at
  // contiguous rows.
  if (gb >= (is_q ? a.s.total_qb : a.s.total_kb)) return;
  int n, b = 0, t0 = 0;
  size_t first_row = 0;
  if (is_q) {
    const QBlock qb = query_block(a.s, gb);
    if (!qb.ok) {
      if (threadIdx.x == 0) record_status(a.status, kStatusBadIndex);
      return;
    }
    const int lo = max(qb.P0, qb.I * a.s.block);
    const int hi = min(qb.L, (qb.I + 1) * a.s.block);
    n = hi - lo;
    first_row = static_cast<size_t>(qb.qrow0) + (lo - qb.P0);
  } else {
    const KBlock kb = key_block(a.s, gb);
    if (!kb.ok) {
      if (threadIdx.x == 0) record_status(a.status, kStatusBadIndex);
      return;
    }
    b = kb.b;
    t0 = kb.J * a.s.block;
    n = min(a.s.block, kb.L - t0);
    first_row = static_cast<size_t>(kb.kbase) + t0;
  }
  const uint8_t* src = is_q ? a.q : a.k;
  const bool paged = (!is_q) && a.page_table != nullptr;
  const size_t row_bytes = static_cast<size_t>(cols) * (E4M3 ? 1 : 2);
  const size_t col_bytes = static_cast<size_t>(col) * (E4M3 ? 1 : 2);

  float acc[EPT];
#pragma unroll
  for (int i = 0; i < EPT; ++i) acc[i] = 0.f;

  // Row base of token r0 of the block (r0 a multiple of the group size, 8 or 16; with page_size
  // % 16 == 0 the group's rows lie in one page, so one page-table lookup serves them); nullptr
  // for a paged
  // token whose page entry is out of range (recorded in the status word).
  auto group_base = [&](int r0) -> const uint8_t* {
    size_t row;
    if (paged) {
      const int tl = t0 + r0;
      const int lp = tl / a.page_size;
      if (lp >= a.max_pages) {
        record_status(a.status, kStatusBadIndex);
        return nullptr;
      }
      const int page = __ldg(a.page_table + static_cast<size_t>(b) * a.max_pages + lp);
      if (page < 0 || page >= a.num_pages) {
        record_status(a.status, kStatusBadIndex);
        return nullptr;
      }
      row = static_cast<size_t>(page) * a.page_size + (tl % a.page_size);
    } else {
      row = first_row + r0;
    }
    return src + row * row_bytes + col_bytes;
  };
  auto load = [&](const uint8_t* gbase, int u) -> int4 {
    return gbase ? __ldcs(reinterpret_cast<const int4*>(gbase + u * row_bytes))
                 : make_int4(0, 0, 0, 0);
  };

  auto accumulate = [&](int4 v) {
    if constexpr (E4M3) {
      const __nv_fp8x2_storage_t* p2 = reinterpret_cast<const __nv_fp8x2_storage_t*>(&v);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(p2[i], __NV_E4M3);
        float2 f = __half22float2(*reinterpret_cast<__half2*>(&h));
        acc[2 * i] += f.x;
        acc[2 * i + 1] += f.y;
      }
    } else {
      const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(p2[i]);
        acc[2 * i] += f.x;
        acc[2 * i + 1] += f.y;
      }
    }
  };

  int r = 0;
  // Rows per group = 16-byte loads in flight per thread. An e4m3 load carries twice the values
  // of a bf16 one, so its decode takes twice as long per byte; with 16 rows in flight the e4m3
  // stream reaches 6.0 TB/s instead of 5.0 with 8 (128K, interleaved A/B, identical results).
  constexpr int kInFlight = E4M3 ? 16 : 8;
  for (; r + kInFlight <= n; r += kInFlight) {
    const uint8_t* gbase = group_base(r);
    int4 v[kInFlight];
#pragma unroll
    for (int u = 0; u < kInFlight; ++u) v[u] = load(gbase, u);
#pragma unroll
    for (int u = 0; u < kInFlight; ++u) accumulate(v[u]);
  }
  if (r < n) {
    const uint8_t* gbase = group_base(r);
    for (int u = 0; r + u < n; ++u) accumulate(load(gbase, u));
  }

  const int h = col / a.d;
  const int c = col % a.d;
  float s = 1.f / static_cast<float>(n);
  const float* scale = is_q ? a.q_scale : a.k_scale;
  if (scale != nullptr) s *= __ldg(scale + h);
  float* dst = (is_q ? a.q_pool : a.k_pool) +
               (static_cast<size_t>(h) * (is_q ? a.s.total_qb : a.s.total_kb) + gb) * a.d + c;
#pragma unroll
  for (int i = 0; i < EPT; ++i) acc[i] *= s;
#pragma unroll
  for (int i = 0; i < EPT; i += 4)
    *reinterpret_cast<float4*>(dst + i) = make_float4(acc[i], acc[i + 1], acc[i + 2], acc[i + 3]);
  if (!is_q && a.k_split != nullptr) {
    // bf16 hi / lo split of the pooled key (the tensor-core operands of the mask kernel).
    const size_t plane = static_cast<size_t>(a.Hkv) * a.s.total_kb * a.d;
    __nv_bfloat16* hi = a.k_split + (static_cast<size_t>(h) * a.s.total_kb + gb) * a.d + c;
#pragma unroll
    for (int i = 0; i < EPT; i += 8) {
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __nv_bfloat162 hh = __floats2bfloat162_rn(acc[i + 2 * j], acc[i + 2 * j + 1]);
        const float2 hf = __bfloat1622float2(hh);
        hw[j] = *reinterpret_cast<const uint32_t*>(&hh);
        lw[j] = pack_bf16x2(acc[i + 2 * j] - hf.x, acc[i + 2 * j + 1] - hf.y);
      }
      *reinterpret_cast<uint4*>(hi + i) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4*>(hi + plane + i) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
  }
}

cudaError_t launch_pool(const PoolArgs& in, bool e4m3, cudaStream_t stream) {
  PoolArgs a = in;
  const int ept = e4m3 ? 16 : 8;
  const int per_cta = kPoolThreads * ept;
  a.q_slices = (a.Hq * a.d + per_cta - 1) / per_cta;
  const int k_slices = (a.Hkv * a.d + per_cta - 1) / per_cta;
  dim3 grid(a.s.total_qb > a.s.total_kb ? a.s.total_qb : a.s.total_kb, a.q_slices + k_slices);
  if (e4m3)
    pool_kernel<true><<<grid, kPoolThreads, 0, stream>>>(a);
  else
    pool_kernel<false><<<grid, kPoolThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace fp
