// Stage 2 on the tensor cores: pooled block scores, max-based threshold, mask and index lists.
//
// Same definition as mask.cu ("FlashPrefill: Instantaneous Pattern Discovery and Thresholding
// for Ultra-Fast Long-Context Prefilling", technical summary 2.B: keep J iff
// s_J - max_{J'<=I} s_J' >= ln(alpha), plus the forced first and diagonal blocks), but the
// scores come from tcgen05.mma instead of fp32 FFMA. The threshold compare has to hold to well
// under 1e-3 in log space, which a single bf16 product does not; each fp32 operand x is split
// into bf16 x_hi = bf16(x) and x_lo = bf16(x - x_hi) (16 significant bits together), and
//   q . k ~= q_hi . k_hi + q_hi . k_lo + q_lo . k_hi       (fp32 accumulation in TMEM),
// which leaves a relative error of about 3 * 2^-18 of sum |q_c k_c| (the dropped q_lo . k_lo and
// the bf16 rounding of the residuals).
//
// One CTA = 128 query rows (the G heads of KV head g times floor(128/G) consecutive query
// blocks; when G does not divide 128 the last 128 mod G rows stay empty) x every key block its
// rows need, in chunks of 128 key blocks: S = Q K^T is an M=128, N=128,
// K=d tile. Pass 0 takes each row's max over its causal, same-request blocks; pass 1 recomputes
// the chunks and writes the keep bits and the ascending index list. Operands are converted
// from fp32 and written to shared memory in the 128-byte-swizzled K-major layout by all 512
// threads, double-buffered against the MMAs; S is double-buffered in TMEM (2 x 128 columns).
// In the epilogue warp w reads TMEM lane quarter w % 4 (32 query rows) and column group w / 4
// (32 key blocks): four threads share a row, combining their partial maxima once at the pass
// boundary and their kept counts through a per-chunk prefix in shared memory.
//
// Failures: every wait is bounded; one that runs out records kStatusTimeout in the caller's
// status word and the CTA stops issuing loads and MMAs (its lists are then incomplete, which
// the status reports). A timeout already recorded in that word makes the kernel do nothing
// (sticky until fp_check_status clears it). A CTA whose rows the prefix sums do not describe
// consistently records kStatusBadIndex and returns before touching any buffer.
#include <math.h>
#include <string.h>

#include "fp_common.cuh"
#include "fp_launch.h"

namespace fp {

namespace {

constexpr int kTcThreads = 512;
constexpr int kTcRows = 128;  // M
constexpr int kTcKeys = 128;  // N per chunk

template <int D>
struct TcCfg {
  static constexpr int kTile = kTcRows * D * 2;      // bytes of one bf16 [128 x D] operand
  static constexpr int kAHi = 0, kALo = kTile;
  static constexpr int kB = 2 * kTile;               // B[buf][hi/lo]
  static constexpr int kMeta = kB + 4 * kTile;
  // row metadata (4 x 128 ints), per-chunk kept counts (2 x 4 x 128 ints), partial maxima
  // (4 x 128 floats), barriers and the TMEM slot, alignment slack
  static constexpr int kSmem = kMeta + (4 + 8 + 4) * kTcRows * 4 + 64 + 1024;
  static constexpr int kBoxBytes = kTcKeys * 128;         // one 128-row x 64-column bf16 box
  static constexpr int kSplitTx = 2 * (D / 64) * kBoxBytes;  // hi + lo tiles of one chunk
  static constexpr int kKSteps = D / 16;
};

// Writes 8 consecutive values (columns k0..k0+7, k0 % 8 == 0) of row r of a K-major,
// 128-byte-swizzled bf16 tile as hi and lo parts.
__device__ __forceinline__ void put8(uint8_t* hi_tile, uint8_t* lo_tile, int rows, int r, int k0,
                                     const float* v) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    // Packed conversions (two values per instruction) for the hi part and the residual.
    const __nv_bfloat162 hh = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    const float2 hf = __bfloat1622float2(hh);
    h[i] = *reinterpret_cast<const uint32_t*>(&hh);
    l[i] = pack_bf16x2(v[2 * i] - hf.x, v[2 * i + 1] - hf.y);
  }
  const int chunk = k0 / 64, unit = (k0 % 64) / 8;
  const int off = chunk * rows * 128 + r * 128 + ((unit ^ (r & 7)) << 4);
  *reinterpret_cast<uint4*>(hi_tile + off) = make_uint4(h[0], h[1], h[2], h[3]);
  *reinterpret_cast<uint4*>(lo_tile + off) = make_uint4(l[0], l[1], l[2], l[3]);
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// kTma: the B operand (pooled keys, split into bf16 hi / lo) is read by TMA from the split that
// the pool kernel wrote (`tm_split`: 2-D map over [2 * Hkv * total_kb, d] bf16 with
// 128-row, 64-column boxes), instead of being converted from fp32 by the threads.
template <int D, bool kTma>
__global__ void __launch_bounds__(kTcThreads, 1)
    mask_tc_kernel(const __grid_constant__ CUtensorMap tm_split, const MaskArgs a) {
  using C = TcCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  int* row_I = reinterpret_cast<int*>(smem + C::kMeta);  // -1: no row
  int* row_kb = row_I + kTcRows;
  int* row_h = row_kb + kTcRows;
  int* row_g = row_h + kTcRows;
  int* cnt_part = row_g + kTcRows;                    // [2][4][128] kept counts per column group
  float* max_part = reinterpret_cast<float*>(cnt_part + 8 * kTcRows);  // [4][128]
  uint64_t* done = reinterpret_cast<uint64_t*>(max_part + 4 * kTcRows);  // [2]
  uint64_t* full = done + 2;                                              // [2] (TMA)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(full + 2);

  const int tid = threadIdx.x, warp = tid / 32;
  // One thread reads the word and the block decides together (another CTA may set it at any
  // time, so separate reads could disagree and leave the barriers below unmatched).
  const bool stale = tid == 0 && a.status != nullptr &&
                     (*reinterpret_cast<volatile uint32_t*>(a.status) & kStatusTimeout);
  if (__syncthreads_or(stale ? 1 : 0)) return;
  // 1-D grid over (row tile, KV head), ordered so that the late row tiles of every KV head --
  // the longest causal rows -- launch first and the short ones fill the tail.
  const int g = blockIdx.x % a.Hkv;
  const int rows_blk = kTcRows / a.G;                 // query blocks per CTA
  const int rows_used = rows_blk * a.G;               // the rest (when G does not divide 128) idle
  const int ntiles = gridDim.x / a.Hkv;
  const int Ig0 = (ntiles - 1 - static_cast<int>(blockIdx.x) / a.Hkv) * rows_blk;

  if (tid < kTcRows) {
    const int Ig = Ig0 + tid / a.G;
    row_h[tid] = g * a.G + tid % a.G;
    if (tid < rows_used && Ig < a.s.total_qb) {
      const QBlock qb = query_block(a.s, Ig);
      row_I[tid] = qb.ok ? qb.I : -2;  // absolute query block: keys J = 0 .. I of the request
      row_kb[tid] = qb.kb0;            // global KV block of the request's block 0
      row_g[tid] = Ig;
    } else {
      row_I[tid] = -1;
      row_kb[tid] = 0;
      row_g[tid] = -1;
    }
  }
  __syncthreads();
  // Key-block range of the CTA: block 0 of its first row's request .. the diagonal block of
  // its last row (rows are ordered by request, then by block). Every row must lie inside it;
  // with inconsistent prefix sums it may not, and the CTA then touches nothing.
  const int r_last = (min(Ig0 + rows_blk, a.s.total_qb) - 1 - Ig0) * a.G;
  const int last = row_kb[r_last] + row_I[r_last];
  const int Jg_lo = row_kb[0];
  const bool bad_row = tid < kTcRows && (row_I[tid] == -2 || (row_I[tid] >= 0 &&
                       (row_kb[tid] < Jg_lo || row_kb[tid] + row_I[tid] > last)));
  if (__syncthreads_or(bad_row ? 1 : 0)) {
    if (tid == 0) record_status(a.status, kStatusBadIndex);
    return;
  }
  if (tid == 0) {
    mbar_init(&done[0], 1);
    mbar_init(&done[1], 1);
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    fence_barrier_init();
    if constexpr (kTma) prefetch_tensormap(&tm_split);
  }
  // The CTA owns its 128 rows of mask words: zero them, keep bits are OR-ed in later.
  if (a.mask_bits != nullptr) {
    const int words = (a.s.max_kb + 31) / 32;
    for (int i = tid; i < kTcRows * words; i += kTcThreads) {
      const int rr = i / words;
      const int Ig = Ig0 + rr / a.G;
      if (rr < rows_used && Ig < a.s.total_qb)
        a.mask_bits[(static_cast<size_t>(g * a.G + rr % a.G) * a.s.total_qb + Ig) * words +
                    i % words] = 0u;
    }
  }
  if (warp == 0) {
    __syncwarp();
    tmem_alloc(tmem_slot, 256);
  }

  // A operand: the 128 rows' pooled queries, split into hi / lo.
  constexpr int kUnits = D / 8;
  for (int u = tid; u < kTcRows * kUnits; u += kTcThreads) {
    const int r = u / kUnits, k0 = (u % kUnits) * 8;
    const int Ig = Ig0 + r / a.G;
    float v[8];
    if (r < rows_used && Ig < a.s.total_qb) {
      const float4* src = reinterpret_cast<const float4*>(
          a.q_pool + (static_cast<size_t>(g * a.G + r % a.G) * a.s.total_qb + Ig) * D + k0);
      const float4 x0 = __ldg(src), x1 = __ldg(src + 1);
      v[0] = x0.x; v[1] = x0.y; v[2] = x0.z; v[3] = x0.w;
      v[4] = x1.x; v[5] = x1.y; v[6] = x1.z; v[7] = x1.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = 0.f;
    }
    put8(smem + C::kAHi, smem + C::kALo, kTcRows, r, k0, v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int nch = (last - Jg_lo) / kTcKeys + 1;
  const int W = 2 * nch;  // pass 0 chunks, then pass 1 chunks

  // Each thread owns kPer 8-value units of a chunk. `fetch` issues all of its global loads into
  // registers (so they are in flight together, and can be in flight while the tensor core
  // works); `store` converts them and writes the chunk's hi / lo tiles.
  constexpr int kPer = kTcKeys * kUnits / kTcThreads;
  float4 xk[kPer][2];
  auto fetch = [&](int w) {
    const int Jg0 = Jg_lo + (w % nch) * kTcKeys;
#pragma unroll
    for (int p = 0; p < kPer; ++p) {
      const int u = tid + p * kTcThreads;
      const int j = u / kUnits, k0 = (u % kUnits) * 8;
      const int Jg = Jg0 + j;
      if (Jg <= last) {
        const float4* src = reinterpret_cast<const float4*>(
            a.k_pool + (static_cast<size_t>(g) * a.s.total_kb + Jg) * D + k0);
        xk[p][0] = __ldg(src);
        xk[p][1] = __ldg(src + 1);
      } else {
        xk[p][0] = xk[p][1] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  };
  auto store = [&](int buf) {
    uint8_t* bh = smem + C::kB + (2 * buf) * C::kTile;
    uint8_t* bl = bh + C::kTile;
#pragma unroll
    for (int p = 0; p < kPer; ++p) {
      const int u = tid + p * kTcThreads;
      const float v[8] = {xk[p][0].x, xk[p][0].y, xk[p][0].z, xk[p][0].w,
                          xk[p][1].x, xk[p][1].y, xk[p][1].z, xk[p][1].w};
      put8(bh, bl, kTcKeys, u / kUnits, (u % kUnits) * 8, v);
    }
  };

  // One chunk of the B operand by TMA: hi rows g * total_kb + Jg0 .. +127 and the same rows
  // of the lo plane (rows past the group's last block carry other data or zeros; their score
  // columns are never valid).
  auto tma_chunk = [&](int w, int buf) {
    // Test hook (fp_debug_skip_mask_load): the load is never issued, so the wait for it runs
    // out and the kernel reports FP_ERR_TIMEOUT.
    if (w == a.fault_skip_chunk && blockIdx.x == 0) return false;
    const int row = g * a.s.total_kb + Jg_lo + (w % nch) * kTcKeys;
    const int lo_row = a.Hkv * a.s.total_kb + row;
    uint8_t* bh = smem + C::kB + (2 * buf) * C::kTile;
    uint8_t* bl = bh + C::kTile;
    mbar_arrive_expect_tx(&full[buf], C::kSplitTx);
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      tma_load_2d(bh + c * C::kBoxBytes, &tm_split, &full[buf], c * 64, row);
      tma_load_2d(bl + c * C::kBoxBytes, &tm_split, &full[buf], c * 64, lo_row);
    }
    return true;
  };

  constexpr uint32_t idesc = make_idesc(1, 1, 0, kTcRows, kTcKeys);
  const uint32_t sbase = smem_u32(smem);
  auto issue = [&](int buf) {
    const uint32_t d_tm = tmem + buf * kTcKeys;
    const uint32_t bh = sbase + C::kB + (2 * buf) * C::kTile, bl = bh + C::kTile;
#pragma unroll
    for (int kk = 0; kk < C::kKSteps; ++kk) {
      const uint32_t off = (kk / 4) * (128 * 128) + (kk % 4) * 32;
      const uint64_t ah = make_sdesc(sbase + C::kAHi + off, 16, 1024);
      const uint64_t al = make_sdesc(sbase + C::kALo + off, 16, 1024);
      const uint64_t dh = make_sdesc(bh + off, 16, 1024);
      const uint64_t dl = make_sdesc(bl + off, 16, 1024);
      mma_f16_ss(d_tm, ah, dh, idesc, kk > 0 ? 1u : 0u);
      mma_f16_ss(d_tm, ah, dl, idesc, 1u);
      mma_f16_ss(d_tm, al, dh, idesc, 1u);
    }
    tc_commit(&done[buf]);
  };

  // Epilogue state: thread (quarter, column group) owns query row r and 32 of the 128 columns
  // of each chunk.
  const int quarter = warp & 3, cgrp = warp >> 2;
  const int r = quarter * 32 + (tid & 31);
  const int I = row_I[r];
  const int kb = row_kb[r];
  float rmax = -INFINITY;
  int cnt = 0;                     // kept blocks of the row so far (same in all 4 threads)
  uint32_t pend_km = 0;            // keep bits of the previous chunk, written one chunk later
  int pend_J = 0, pend_item = -1;
  const int words = (a.s.max_kb + 31) / 32;
  const size_t row = I >= 0 ? static_cast<size_t>(row_h[r]) * a.s.total_qb + row_g[r] : 0;
  int32_t* idx = a.kv_idx + row * a.s.max_kb;
  uint32_t* bits_row = a.mask_bits ? a.mask_bits + row * words : nullptr;

  // Writes the previous chunk's kept indices at their place in the ascending list, using the
  // kept counts of the four column groups of that chunk (visible after the block barrier).
  auto flush = [&]() {
    if (pend_item < 0) return;
    const int* cp = cnt_part + (pend_item & 1) * 4 * kTcRows;
    int before = 0, total = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = cp[q * kTcRows + r];
      before += q < cgrp ? c : 0;
      total += c;
    }
    if (pend_km) {
      int o = cnt + before;
      for (uint32_t t = pend_km; t; t &= t - 1) idx[o++] = pend_J + __ffs(t) - 1;
      if (bits_row) {
        const int w0 = pend_J >> 5, sh = pend_J & 31;
        atomicOr(bits_row + w0, pend_km << sh);
        if (sh && (pend_km >> (32 - sh))) atomicOr(bits_row + w0 + 1, pend_km >> (32 - sh));
      }
    }
    cnt += total;
    pend_item = -1;
  };

  auto process = [&](int w, int buf) {
    tc_fence_after();
    float v[32];
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    tmem_ld32(tmem + lane_base + buf * kTcKeys + cgrp * 32, v);
    tmem_ld_wait();
    flush();
    const bool pass0 = w < nch;
    if (w == nch) {  // first pass-1 chunk: the four partial maxima of pass 0 are in smem
      rmax = fmaxf(fmaxf(max_part[r], max_part[kTcRows + r]),
                   fmaxf(max_part[2 * kTcRows + r], max_part[3 * kTcRows + r]));
    }
    const int Jb = Jg_lo + (w % nch) * kTcKeys - kb + cgrp * 32;  // request-local J of v[0]
    const int lo = max(0, -Jb), hi = min(31, I - Jb);            // valid columns lo..hi
    const bool any = I >= 0 && hi >= lo;
    const uint32_t valid =
        any ? ((hi == 31 ? 0xffffffffu : ((2u << hi) - 1u)) & (~0u << lo)) : 0u;
    if (pass0) {
      if (any) {
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int e = 0; e < 32; e += 2)
          m4[(e / 2) % 4] = fmax3(m4[(e / 2) % 4], ((valid >> e) & 1u) ? v[e] : -INFINITY,
                                  ((valid >> (e + 1)) & 1u) ? v[e + 1] : -INFINITY);
        rmax = fmaxf(rmax, fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * a.scale);
      }
      if (w == nch - 1) max_part[cgrp * kTcRows + r] = rmax;
    } else {
      uint32_t km = 0;
      if (any) {
        // s * scale - max >= ln(alpha)  <=>  s >= (max + ln(alpha)) / scale   (scale > 0)
        const float thr = (rmax + a.log_alpha) / a.scale;
#pragma unroll
        for (int e = 0; e < 32; ++e) km |= (v[e] >= thr ? 1u : 0u) << e;
        if ((a.flags & FP_FORCE_FIRST) && Jb <= 0 && 0 < Jb + 32) km |= 1u << (-Jb);
        if ((a.flags & FP_FORCE_DIAG) && Jb <= I && I < Jb + 32) km |= 1u << (I - Jb);
        km &= valid;
      }
      // Columns before the row's request (Jb < 0) are never valid: drop them so the bits
      // start at J >= 0 (then -Jb <= lo <= 31).
      int Jn = Jb;
      if (km && Jn < 0) {
        km >>= -Jn;
        Jn = 0;
      }
      cnt_part[(w & 1) * 4 * kTcRows + cgrp * kTcRows + r] = __popc(km);
      pend_km = km;
      pend_J = Jn;
      pend_item = w;
    }
  };

  // Thread 0 alone issues loads and MMAs. After a wait of its own has run out it issues
  // nothing more (commits only, so that every barrier the other threads wait for still
  // completes); `lost` is the buffer of a load that was issued and never arrived.
  bool stop = false, issued = false;
  int lost = -1, lost_parity = 0;
  if constexpr (kTma) {
    if (tid == 0) issued = tma_chunk(0, 0);
  } else {
    fetch(0);
    store(0);
    fence_async_smem();
  }
  __syncthreads();
  for (int w = 0; w < W; ++w) {
    const int b = w & 1;
    if constexpr (kTma) {
      if (tid == 0) {
        // chunk w has landed -> its MMAs; then, once chunk w-1's MMAs are done with the
        // other buffer, start loading chunk w+1 into it.
        if (!stop && !mbar_wait(&full[b], (w >> 1) & 1)) {
          record_status(a.status, kStatusTimeout);
          stop = true;
          if (issued) {
            lost = b;
            lost_parity = (w >> 1) & 1;
          }
        }
        tc_fence_after();
        if (!stop) issue(b);
        else tc_commit(&done[b]);
        if (!stop && w + 1 < W) {
          if (w == 0 || mbar_wait(&done[b ^ 1], ((w - 1) >> 1) & 1)) {
            issued = tma_chunk(w + 1, b ^ 1);
          } else {
            record_status(a.status, kStatusTimeout);
            stop = true;
          }
        }
      }
    } else {
      if (tid == 0) {
        tc_fence_after();
        if (!stop) issue(b);
        else tc_commit(&done[b]);
      }
      if (w + 1 < W) fetch(w + 1);  // loads in flight while the MMAs of chunk w run
    }
    if (w >= 1) {
      // All threads wait for the previous chunk's MMAs: its B buffer is rewritten and its
      // TMEM columns are read now. The wait is bounded; every thread stays in the loop
      // either way, so the block barriers below always match.
      const bool ok = mbar_wait(&done[b ^ 1], ((w - 1) >> 1) & 1);
      if (__all_sync(0xffffffffu, ok)) process(w - 1, b ^ 1);
      else if ((tid & 31) == 0) record_status(a.status, kStatusTimeout);
    }
    if constexpr (!kTma) {
      if (w + 1 < W) store(b ^ 1);
      fence_async_smem();
    }
    tc_fence_before();
    __syncthreads();
  }
  {
    const bool ok = mbar_wait(&done[(W - 1) & 1], ((W - 1) >> 1) & 1);
    if (__all_sync(0xffffffffu, ok)) process(W - 1, (W - 1) & 1);
    else if ((tid & 31) == 0) record_status(a.status, kStatusTimeout);
  }
  // A load that was issued but never arrived may still be writing shared memory: give it one
  // more bounded wait before the CTA exits.
  if constexpr (kTma) {
    if (tid == 0 && lost >= 0) mbar_wait(&full[lost], lost_parity);
  }

  __syncthreads();  // the last chunk's kept counts are visible
  flush();
  if (I >= 0 && cgrp == 0) a.kv_cnt[row] = cnt;
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace

bool mask_tc_supported(int G, int d) {
  return (d == 64 || d == 128) && G >= 1 && G <= kTcRows;
}

template <int D, bool kTma>
static cudaError_t launch_tc(const MaskArgs& a, const CUtensorMap& map, dim3 grid,
                             cudaStream_t stream) {
  auto kern = mask_tc_kernel<D, kTma>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       TcCfg<D>::kSmem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kTcThreads, TcCfg<D>::kSmem, stream>>>(map, a);
  return cudaGetLastError();
}

cudaError_t launch_mask_tc(const MaskArgs& a, cudaStream_t stream) {
  const int rows_blk = kTcRows / a.G;
  dim3 grid(((a.s.total_qb + rows_blk - 1) / rows_blk) * a.Hkv);
  CUtensorMap map;
  memset(&map, 0, sizeof(map));
  if (a.k_split != nullptr) {
    EncodeTiledFn enc = tensor_map_encoder();
    if (enc == nullptr) return cudaErrorNotSupported;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.d),
                          2ull * static_cast<cuuint64_t>(a.Hkv) * a.s.total_kb};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.d) * 2};
    cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(kTcKeys)};
    cuuint32_t estr[2] = {1u, 1u};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a.k_split), dims,
            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    return a.d == 128 ? launch_tc<128, true>(a, map, grid, stream)
                      : launch_tc<64, true>(a, map, grid, stream);
  }
  return a.d == 128 ? launch_tc<128, false>(a, map, grid, stream)
                    : launch_tc<64, false>(a, map, grid, stream);
}

}  // namespace fp
