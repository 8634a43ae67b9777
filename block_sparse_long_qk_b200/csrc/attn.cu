// Stage 3: block-sparse causal attention over the kept KV blocks (contiguous and paged KV).
//
// "FlashPrefill: Instantaneous Pattern Discovery and Thresholding for Ultra-Fast Long-Context
// Prefilling", technical summary 2.C: masked blocks are skipped physically -- the kernel walks
// the index list of kept blocks and points its loads straight at them, running no control
// logic for the blocks in between. "FlashPrefill V2: Block-Sparse Prefill Attention for
// Long-Context LLM Serving", Abstract: query heads that share a KV head are packed onto the
// same K/V loads (PackGQA), FP8 inputs, paged KV cache and continuous batching.
//
// B200 design (one CTA = two 128-row query tiles that read the same KV head: two heads of a
// GQA group at one query block, or one head at two neighbouring query blocks; see the work
// items below):
//   warp 0      TMA producer: both Q tiles once, then K and V tiles of the union of the two
//               tiles' kept-block lists into a 2-deep K ring and a 2-deep V ring.
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer. Per union block it issues
//               S_t = Q_t K^T for each tile t that kept the block, and, before that, the
//               pending O_t += P_t V of the tile's previous block. The two tiles therefore
//               alternate on the tensor core while the other tile's softmax runs (the sm_100
//               counterpart of the pages' pingpong schedule).
//   warps 4-7   softmax of tile 0, warps 8-11 softmax of tile 1: one thread per query row reads
//               its S row from TMEM, applies the causal mask on the diagonal block, keeps a
//               running max with lazy rescaling of O (only when the max grows by more than
//               2^8), writes P (bf16 or e4m3) back into the S columns of TMEM, and finally
//               normalises O and writes the bf16 output row (plus the row's log-sum-exp).
// TMEM: S0 | S1 | O0 | O1 (fp32 accumulators, 128 lanes); P_t aliases the first columns of S_t
// and is consumed by the PV MMA straight from TMEM. All waits are bounded (fp_common.cuh).
#include <math.h>

#include <type_traits>

#include "fp_common.cuh"
#include "fp_launch.h"

namespace fp {

template <int D, int BN, bool FP8>
struct AttnCfg {
  static constexpr int kBM = 128;
  static constexpr int kEB = FP8 ? 1 : 2;
  static constexpr int kChunkEl = 128 / kEB;         // elements per 128-byte swizzle row
  static constexpr int kNChunk = D / kChunkEl;
  static constexpr int kQBytes = kBM * D * kEB;
  static constexpr int kKVBytes = BN * D * kEB;
  static constexpr int kKSt = 2, kVSt = 2;
  static constexpr int kKStep = FP8 ? 32 : 16;       // MMA K per instruction
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + 2 * kQBytes;
  static constexpr int kVOff = kKOff + kKSt * kKVBytes;
  static constexpr int kBarOff = kVOff + kVSt * kKVBytes;
  static constexpr int kSmemBytes = kBarOff + 256 + 1024;  // + barriers + alignment slack
  static_assert(kKSt <= 4 && kVSt <= 4, "ring depth");
  static_assert(kSmemBytes <= 232448, "shared memory per block");
  static constexpr int kTmemUsed = 2 * BN + 2 * D;          // S0 S1 O0 O1
  static constexpr int kTmemCols = kTmemUsed <= 256 ? 256 : 512;  // power-of-2 allocation
  static constexpr uint32_t kS0 = 0, kS1 = BN, kO0 = 2 * BN, kO1 = 2 * BN + D;
  static constexpr int kThreads = 384;
  static_assert(kTmemUsed <= 512, "S and O tiles of both query tiles must fit in TMEM");
};

struct Tile {
  // h: query head; Ig: global query block; I: its absolute block in the request (keys J <= I);
  // q_lo: query row of tile row 0 (absolute position I * block; for the first block of a
  // chunked request it precedes the request's first query row); rows r0 .. r1-1 are valid
  // queries (r1 = 0 marks an absent tile); cnt / list: the kept-block list of (h, Ig).
  int h, Ig, I, q_lo, r0, r1, cnt;
  const int32_t* list;
};

// A tile's request, for the work split whose two tiles may lie in different requests: b
// (page-table row), kbase (key row of position 0), len (key count), kb0 (its first KV block in
// the prefix sums; kb0 + J orders the blocks of both tiles in one walk).
struct Req {
  int b, kbase, len, kb0;
};

// Levels (pairs of query blocks) per item window of the general work split (make_tiles_qp).
constexpr int kQpWindow = 32;

struct Shared {  // placed at kBarOff
  uint64_t q_full;
  uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];  // ring slots (kKSt, kVSt <= 4)
  uint64_t s_full[2], p_full[2], o_final[2];
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort_flag;
};

// Next entry of a kept-block list that is a valid causal block index (0 <= J <= I), or -1.
// Invalid entries are skipped; `report` records them once in the status word.
__device__ __forceinline__ int next_valid(const int32_t* list, int cnt, int& i, int I,
                                          uint32_t* status, bool report) {
  while (i < cnt) {
    const int J = __ldg(list + i);
    ++i;
    if (J >= 0 && J <= I) return J;
    if (report) record_status(status, kStatusBadIndex);
  }
  return -1;
}

// Walks the ascending union of two kept-block lists; `bits` says which tiles kept the block.
// With KEYED, the lists are merged on kb0 + J (the tiles' requests may differ: a block both
// tiles kept, same request and same J, comes once with bits = 3; tiles of different requests
// share none).
template <bool KEYED>
struct UnionWalk {
  const int32_t *l0, *l1;
  int c0, c1, i0, i1, I0, I1, a, b, o0, o1;
  __device__ void init(const Tile& t0, const Tile& t1, int off0 = 0, int off1 = 0) {
    l0 = t0.list; l1 = t1.list; c0 = t0.cnt; c1 = t1.cnt; I0 = t0.I; I1 = t1.I;
    o0 = KEYED ? off0 : 0; o1 = KEYED ? off1 : 0;
    i0 = i1 = 0;
    a = next_valid(l0, c0, i0, I0, nullptr, false);
    b = next_valid(l1, c1, i1, I1, nullptr, false);
  }
  __device__ bool next(int& J, int& bits) {
    if (a < 0 && b < 0) return false;
    const int ka = KEYED ? a + o0 : a, kb = KEYED ? b + o1 : b;
    if (b < 0 || (a >= 0 && ka < kb)) { J = a; bits = 1; a = next_valid(l0, c0, i0, I0, nullptr, false); }
    else if (a < 0 || kb < ka) { J = b; bits = 2; b = next_valid(l1, c1, i1, I1, nullptr, false); }
    else { J = a; bits = 3; a = next_valid(l0, c0, i0, I0, nullptr, false); b = next_valid(l1, c1, i1, I1, nullptr, false); }
    return true;
  }
};

// Head-pair split: work item -> two heads of a GQA group at one query block, one request. Items run heaviest-first (late query blocks have the longest causal rows). `kbase`
// / `len`: key row of the request's position 0 and its key count; `b`: the request (page-table
// row). Returns false (both tiles absent) when the prefix sums do not describe the request
// consistently.
__device__ __forceinline__ bool make_tiles(const AttnArgs& a, int item, Tile* t, int& g,
                                           int& b, int& kbase, int& len) {
  // The G query heads of a KV head form ceil(G / 2) items per query block: pairs of heads,
  // and for an odd G one single head (its CTA runs one tile; the host sends an odd G here only
  // when single tiles give the GPU more CTAs than it could otherwise fill).
  const int npair = (a.G + 1) / 2;
  const int per_block = a.Hkv * npair;
  const int Ig = a.s.total_qb - 1 - item / per_block;
  const int rem = item % per_block;
  g = rem / npair;
  const int h0 = g * a.G + 2 * (rem % npair);
  t[0].h = h0; t[0].Ig = Ig;
  t[1].h = h0 + 1; t[1].Ig = (h0 + 1 < (g + 1) * a.G) ? Ig : -1;
  if (t[1].Ig < 0) t[1].h = h0;
  const QBlock qb = query_block(a.s, Ig);
  b = qb.b;
  kbase = qb.kbase;
  len = qb.L;
  for (int s = 0; s < 2; ++s) {
    if (t[s].Ig < 0 || !qb.ok) {
      t[s].r0 = t[s].r1 = 0; t[s].cnt = 0; t[s].list = a.kv_idx; t[s].I = -1; t[s].q_lo = 0;
      continue;
    }
    const int B = a.s.block;
    t[s].I = qb.I;
    t[s].q_lo = qb.qrow0 + qb.I * B - qb.P0;
    t[s].r0 = max(0, qb.P0 - qb.I * B);
    t[s].r1 = min(B, qb.L - qb.I * B);
    const size_t row = static_cast<size_t>(t[s].h) * a.s.total_qb + t[s].Ig;
    t[s].cnt = __ldg(a.kv_cnt + row);
    t[s].cnt = max(0, min(t[s].cnt, a.s.max_kb));
    t[s].list = a.kv_idx + row * a.s.max_kb;
  }
  return qb.ok;
}

// General split: work item -> two tiles that read the same KV head. Two heads of a GQA group
// share a query block (a head pair); a head that pairing leaves over (odd G, every head when
// G = 1, or every head when query-block pairing is forced) is paired with itself over two
// neighbouring query blocks (the QUILT page's cross-query reuse: both tiles read every block
// they both kept once). Levels of two query blocks, Ig0 = total_qb - 1 - 2 * level and
// Ig1 = Ig0 - 1, hold per KV head S = 2 hp + nqh items: hp head pairs at Ig0, nqh query-block
// pairs, hp head pairs at Ig1 (both tiles absent at the last level when total_qb is odd).
// Items run heaviest-first in windows of kQpWindow levels, and inside a window KV head by KV
// head: the CTAs in flight (about one per SM) then cover a few KV heads over many neighbouring
// query blocks, so the K/V blocks those share (the local band, columns every row keeps) stay in
// L2 instead of every KV head's working set at once. Returns false (tiles absent) when the
// prefix sums do not describe a tile's request consistently.
__device__ __forceinline__ bool make_tiles_qp(const AttnArgs& a, int item, Tile* t, Req* rq,
                                              int& g) {
  const int hp = a.head_pairs, nqh = a.qpair_heads, S = 2 * hp + nqh;
  const int levels = (a.s.total_qb + 1) / 2;
  const int per_win = kQpWindow * a.Hkv * S;
  const int win = item / per_win;
  int rem = item % per_win;
  const int wn = min(kQpWindow, levels - win * kQpWindow);  // levels in this window
  g = rem / (wn * S);
  rem %= wn * S;
  const int Ig0 = a.s.total_qb - 1 - 2 * (win * kQpWindow + rem / S);
  const int slot = rem % S;
  int Igs[2];
  if (slot < hp || slot >= hp + nqh) {
    const bool second = slot >= hp;
    t[0].h = g * a.G + 2 * (second ? slot - hp - nqh : slot);
    t[1].h = t[0].h + 1;
    Igs[0] = Igs[1] = second ? Ig0 - 1 : Ig0;
  } else {
    t[0].h = t[1].h = g * a.G + 2 * hp + (slot - hp);
    Igs[0] = Ig0;
    Igs[1] = Ig0 - 1;
  }
  bool ok = true;
  QBlock qb{};
  for (int s = 0; s < 2; ++s) {
    t[s].Ig = Igs[s];
    if (Igs[s] < 0) {
      t[s].r0 = t[s].r1 = 0; t[s].cnt = 0; t[s].list = a.kv_idx; t[s].I = -1; t[s].q_lo = 0;
      rq[s] = Req{0, 0, 0, 0};
      continue;
    }
    if (s == 0 || Igs[1] != Igs[0]) qb = query_block(a.s, Igs[s]);
    if (!qb.ok) {
      ok = false;
      t[s].r0 = t[s].r1 = 0; t[s].cnt = 0; t[s].list = a.kv_idx; t[s].I = -1; t[s].q_lo = 0;
      rq[s] = Req{0, 0, 0, 0};
      continue;
    }
    const int B = a.s.block;
    rq[s] = Req{qb.b, qb.kbase, qb.L, qb.kb0};
    t[s].I = qb.I;
    t[s].q_lo = qb.qrow0 + qb.I * B - qb.P0;
    t[s].r0 = max(0, qb.P0 - qb.I * B);
    t[s].r1 = min(B, qb.L - qb.I * B);
    const size_t row = static_cast<size_t>(t[s].h) * a.s.total_qb + t[s].Ig;
    t[s].cnt = __ldg(a.kv_cnt + row);
    t[s].cnt = max(0, min(t[s].cnt, a.s.max_kb));
    t[s].list = a.kv_idx + row * a.s.max_kb;
  }
  return ok;
}

// OUTP: the output goes through the K/V page table (FP_OUT_PAGED; paged K/V only). A template
// parameter, so that the other instantiations keep no page-table state live through the loop.
// QP: the general work split (query-block pairs, tiles of two requests); without it the
// head-pair split, whose tiles share one request.
template <int D, int BN, bool FP8, bool PAGED, bool OUTP, bool QP>
__global__ void __launch_bounds__(384, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const AttnArgs a) {
  using C = AttnCfg<D, BN, FP8>;
  extern __shared__ uint8_t smem_raw[];
  // Swizzled TMA tiles and UMMA descriptors assume 1024-byte aligned shared addresses.
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  Shared& sh = *reinterpret_cast<Shared*>(smem + C::kBarOff);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  // A timeout recorded earlier in this workspace makes later CTAs exit at once, so one
  // broken pipeline cannot hold the GPU for a 2 s wait per CTA. fp_check_status clears it.
  if (threadIdx.x == 0)
    sh.abort_flag = (a.status != nullptr && (*reinterpret_cast<volatile uint32_t*>(a.status) &
                                             kStatusTimeout)) ? 1 : 0;
  __syncthreads();
  if (sh.abort_flag) return;

  Tile tl[2];
  Req rq[2];
  int g, b = 0, kbase = 0, len = 0;
  bool tiles_ok;
  if constexpr (QP) tiles_ok = make_tiles_qp(a, blockIdx.x, tl, rq, g);
  else tiles_ok = make_tiles(a, blockIdx.x, tl, g, b, kbase, len);
  if (!tiles_ok && threadIdx.x == 0) record_status(a.status, kStatusBadIndex);
  // A head pair past the first query block (odd total_qb, last level) has no work; every
  // thread of the CTA maps the same item, so the whole CTA leaves together.
  if constexpr (QP)
    if (tl[0].Ig < 0 && tl[1].Ig < 0) return;
  // Producer bookkeeping: the last use of each ring slot whose load was issued, so that a CTA
  // that gives up waits (bounded) for its own bulk copies before it exits.
  int k_issued[C::kKSt], v_issued[C::kVSt];
  bool q_issued = false;
#pragma unroll
  for (int i = 0; i < C::kKSt; ++i) k_issued[i] = -1;
#pragma unroll
  for (int i = 0; i < C::kVSt; ++i) v_issued[i] = -1;

  if (threadIdx.x == 0) {
    mbar_init(&sh.q_full, 1);
    for (int i = 0; i < C::kKSt; ++i) {
      mbar_init(&sh.k_full[i], 1);
      mbar_init(&sh.k_empty[i], 1);
    }
    for (int i = 0; i < C::kVSt; ++i) {
      mbar_init(&sh.v_full[i], 1);
      mbar_init(&sh.v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.s_full[i], 1); mbar_init(&sh.p_full[i], 128); mbar_init(&sh.o_final[i], 1);
    }
    mbar_init(&sh.drain, 1);
    sh.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(&sh.tmem_base, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      const int ntiles = tl[1].r1 > 0 ? 2 : 1;
      mbar_arrive_expect_tx(&sh.q_full, ntiles * C::kQBytes);
      for (int s = 0; s < ntiles; ++s)
        for (int c = 0; c < C::kNChunk; ++c)
          tma_load_3d(smem + C::kQOff + s * C::kQBytes + c * (C::kBM * 128), &tm_q, &sh.q_full,
                      c * C::kChunkEl, tl[s].h, tl[s].q_lo);
      q_issued = true;
      UnionWalk<QP> uw;
      if constexpr (QP) uw.init(tl[0], tl[1], rq[0].kb0, rq[1].kb0);
      else uw.init(tl[0], tl[1]);
      int J, bits;
      for (int k = 0; uw.next(J, bits); ++k) {
        if (sh.abort_flag) break;
        const int ks = k % C::kKSt, vs = k % C::kVSt;
        // Row coordinates of the block's segments (whole block, or one per page).
        constexpr int kSegRows = PAGED ? 0 : BN;
        const int seg_rows = PAGED ? a.page_size : kSegRows;
        const int nseg = BN / seg_rows;
        // The block's request (with QP the tiles' requests may differ, and then no block has
        // bits = 3).
        int kb_req = kbase, len_req = len, b_req = b;
        if constexpr (QP) {
          const bool from0 = bits & 1;
          kb_req = from0 ? rq[0].kbase : rq[1].kbase;
          len_req = from0 ? rq[0].len : rq[1].len;
          b_req = from0 ? rq[0].b : rq[1].b;
        }
        for (int which = 0; which < 2; ++which) {
          const int st = which == 0 ? ks : vs;
          uint64_t* full = which == 0 ? &sh.k_full[st] : &sh.v_full[st];
          uint64_t* empty = which == 0 ? &sh.k_empty[st] : &sh.v_empty[st];
          const int use = k / (which == 0 ? C::kKSt : C::kVSt);
          if (use > 0 && !mbar_wait(empty, (use - 1) & 1)) {
            record_status(a.status, kStatusTimeout); sh.abort_flag = 1; break;
          }
          // Test hook (fp_debug_skip_k_load): the load is never issued, so the MMA issuer's
          // bounded wait for it runs out and the kernel reports FP_ERR_TIMEOUT.
          if (which == 0 && k == a.fault_skip_k && blockIdx.x == 0) continue;
          mbar_arrive_expect_tx(full, C::kKVBytes);
          uint8_t* dst = smem + (which == 0 ? C::kKOff : C::kVOff) + st * C::kKVBytes;
          const CUtensorMap* tm = which == 0 ? &tm_k : &tm_v;
          for (int sgi = 0; sgi < nseg; ++sgi) {
            int row;
            const int tok = J * BN + sgi * seg_rows;  // request-local first token
            if constexpr (PAGED) {
              const int pages_req = (len_req + a.page_size - 1) / a.page_size;
              const int lp = tok / a.page_size;
              row = a.num_pages * a.page_size;  // past the end: TMA fills zeros
              if (lp < pages_req && lp < a.max_pages) {
                const int pid = __ldg(a.page_table + static_cast<size_t>(b_req) * a.max_pages + lp);
                if (pid >= 0 && pid < a.num_pages) row = pid * a.page_size;
                else record_status(a.status, kStatusBadIndex);
              }
            } else {
              row = kb_req + tok;
            }
            for (int c = 0; c < C::kNChunk; ++c)
              tma_load_3d(dst + c * (BN * 128) + sgi * (seg_rows * 128), tm, full,
                          c * C::kChunkEl, g, row);
          }
          if (which == 0) k_issued[st] = use;
          else v_issued[st] = use;
        }
        if (sh.abort_flag) break;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t fmt = FP8 ? 0u : 1u;
      constexpr uint32_t idesc_s = make_idesc(fmt, fmt, 0, 128, BN);
      constexpr uint32_t idesc_o = make_idesc(fmt, fmt, 1, 128, D);
      const uint32_t sbase = smem_u32(smem);
      auto s_col = [](int t) -> uint32_t { return t == 0 ? C::kS0 : C::kS1; };
      auto o_col = [](int t) -> uint32_t { return t == 0 ? C::kO0 : C::kO1; };
      bool ok = mbar_wait(&sh.q_full, 0);
      tc_fence_after();
      int n[2] = {0, 0}, pend[2] = {-1, -1};
      int vusers[2] = {0, 0};
      auto issue_pv = [&](int t) -> bool {
        const int k = pend[t];
        const int vs = k % C::kVSt;
        if (!mbar_wait(&sh.p_full[t], (n[t] - 1) & 1)) return false;
        if (!mbar_wait(&sh.v_full[vs], (k / C::kVSt) & 1)) return false;
        tc_fence_after();
        const uint32_t vaddr = sbase + C::kVOff + vs * C::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < BN / C::kKStep; ++kk) {
          const uint64_t bdesc = make_sdesc(vaddr + kk * (C::kKStep / 8) * 1024, BN * 128, 1024);
          const uint32_t a_tm = tmem + s_col(t) + kk * 8;
          const uint32_t acc = (n[t] > 1 || kk > 0) ? 1u : 0u;
          if constexpr (FP8) mma_f8_ts(tmem + o_col(t), a_tm, bdesc, idesc_o, acc);
          else mma_f16_ts(tmem + o_col(t), a_tm, bdesc, idesc_o, acc);
        }
        if (--vusers[vs] == 0) tc_commit(&sh.v_empty[vs]);
        pend[t] = -1;
        return true;
      };
      UnionWalk<QP> uw;
      if constexpr (QP) uw.init(tl[0], tl[1], rq[0].kb0, rq[1].kb0);
      else uw.init(tl[0], tl[1]);
      int J, bits;
      for (int k = 0; ok && uw.next(J, bits); ++k) {
        if (sh.abort_flag) { ok = false; break; }
        const int ks = k % C::kKSt;
        if (!mbar_wait(&sh.k_full[ks], (k / C::kKSt) & 1)) { ok = false; break; }
        tc_fence_after();
        vusers[k % C::kVSt] = __popc(bits);
        const uint32_t kaddr = sbase + C::kKOff + ks * C::kKVBytes;
        // Tiles that kept this block: finish their previous block (PV), then S = Q K^T.
        for (int t = 0; t < 2 && ok; ++t) {
          if (!((bits >> t) & 1)) continue;
          if (pend[t] >= 0 && !issue_pv(t)) { ok = false; break; }
          const uint32_t qaddr = sbase + C::kQOff + t * C::kQBytes;
#pragma unroll
          for (int kk = 0; kk < D / C::kKStep; ++kk) {
            const uint32_t byte = kk * C::kKStep * C::kEB;  // K offset of this step in bytes
            const uint32_t chunk = byte / 128, off = byte % 128;
            const uint64_t adesc = make_sdesc(qaddr + chunk * (128 * 128) + off, 16, 1024);
            const uint64_t bdesc = make_sdesc(kaddr + chunk * (BN * 128) + off, 16, 1024);
            if constexpr (FP8) mma_f8_ss(tmem + s_col(t), adesc, bdesc, idesc_s, kk > 0 ? 1u : 0u);
            else mma_f16_ss(tmem + s_col(t), adesc, bdesc, idesc_s, kk > 0 ? 1u : 0u);
          }
          tc_commit(&sh.s_full[t]);
          ++n[t];
          pend[t] = k;
        }
        if (!ok) break;
        tc_commit(&sh.k_empty[ks]);
        // Tiles that skipped this block: flush their pending PV now, so that no V slot is
        // held past the next block (each V slot is reused two union blocks later).
        for (int t = 0; t < 2 && ok; ++t)
          if (!((bits >> t) & 1) && pend[t] >= 0 && !issue_pv(t)) ok = false;
      }
      for (int t = 0; t < 2; ++t) {
        if (ok && pend[t] >= 0 && !issue_pv(t)) ok = false;
        tc_commit(&sh.o_final[t]);
      }
      if (!ok) { record_status(a.status, kStatusTimeout); sh.abort_flag = 1; }
      // Every MMA of this CTA has completed before TMEM is released (bounded wait).
      tc_commit(&sh.drain);
      if (!mbar_wait(&sh.drain, 0)) record_status(a.status, kStatusTimeout);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ softmax / epilogue
    const int t = (warp - 4) / 4;
    const int r = (warp % 4) * 32 + lane;  // query row of the tile = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp % 4) * 32) << 16;
    const uint32_t s_tm = tmem + lane_base + (t == 0 ? C::kS0 : C::kS1);
    const uint32_t o_tm = tmem + lane_base + (t == 0 ? C::kO0 : C::kO1);
    const Tile T = t == 0 ? tl[0] : tl[1];
    float sl2 = a.scale_log2;
    if constexpr (FP8) sl2 *= __ldg(a.q_scale + T.h) * __ldg(a.k_scale + g);
    float m = -INFINITY, l = 0.f;
    int n = 0;
    bool ok = true;
    int i = 0;
    // P = 2^(s * sl2 - mu) for the row, taken from the S row the max pass left in registers
    // (no second TMEM read: measured 0.8 % fewer cycles per union block than re-reading the
    // upper 64 columns, about 3.5 % fewer than re-reading the whole row), packed and written
    // over the S columns in TMEM; returns the row sum. Four independent partial sums keep the
    // add chain short.
    // With e4m3 inputs the MMAs run twice as fast and the MUFU ex2 unit (4 lanes per clock per
    // SM sub-partition) becomes the limit: there, two column pairs in eight off the diagonal
    // take the FMA-pipe polynomial instead (measured at 128K, interleaved: 7.62 ms median
    // against 8.02 with 1/8 or 3/8 and 8.27 with 1/2). With bf16 the extra FMA work costs
    // more than it saves, so every exponential uses MUFU ex2.
    constexpr bool kPolyExp = FP8;
    auto p_pass = [&](const float* s_row, float mu, auto diag_tag) -> float {
      constexpr bool diag = decltype(diag_tag)::value;
      const float2 sc2 = make_float2(sl2, sl2), nm2 = make_float2(-mu, -mu);
      float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                       make_float2(0.f, 0.f)};
#pragma unroll
      for (int h0 = 0; h0 < BN; h0 += 64) {
        const float* sv = s_row + h0;
#pragma unroll
        for (int c1 = 0; c1 < 64 && h0 + c1 < BN; c1 += 32) {
          const int c0 = h0 + c1;
          float2 pp[16];
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            float2 x = ffma2(make_float2(sv[c1 + c], sv[c1 + c + 1]), sc2, nm2);
            if constexpr (diag) {
              if (c0 + c > r) x.x = -INFINITY;
              if (c0 + c + 1 > r) x.y = -INFINITY;
            }
            pp[c / 2] = (kPolyExp && !diag && (c / 2) % 8 >= 6)
                            ? exp2_poly2(x)
                            : make_float2(ex2(x.x), ex2(x.y));
          }
#pragma unroll
          for (int e = 0; e < 16; ++e) acc[e % 4] = fadd2(acc[e % 4], pp[e]);
          if constexpr (FP8) {
            uint32_t w[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              w[e] = pack_e4m3x4(pp[2 * e].x, pp[2 * e].y, pp[2 * e + 1].x, pp[2 * e + 1].y);
            tmem_st8(s_tm + c0 / 4, w);
          } else {
            uint32_t w[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) w[e] = pack_bf16x2(pp[e].x, pp[e].y);
            tmem_st16(s_tm + c0 / 2, w);
          }
        }
      }
      const float2 t = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
      return t.x + t.y;
    };
    int J = next_valid(T.list, T.cnt, i, T.I, a.status, r == 0);
    while (J >= 0) {
      // The next list entry is fetched before the wait, off the critical path.
      const int J_next = next_valid(T.list, T.cnt, i, T.I, a.status, r == 0);
      const bool got = !sh.abort_flag && mbar_wait(&sh.s_full[t], n & 1);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tc_fence_after();
      const bool diag = (J == T.I);
      // Row max over the S row (causal mask inside the diagonal block: key c > query r), as a
      // tree of 8 independent 3-input maxima. The whole row comes from TMEM in one round trip
      // (measured: 4 % fewer cycles per union block than two 64-column halves).
      float mr[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mr[e] = -INFINITY;
      float sv[BN];
#pragma unroll
      for (int c = 0; c < BN; c += 32) tmem_ld32(s_tm + c, sv + c);
      tmem_ld_wait();
      if (diag) {
#pragma unroll
        for (int c = 0; c < BN; ++c) sv[c] = (c > r) ? -INFINITY : sv[c];
      }
#pragma unroll
      for (int c = 0; c < BN; c += 2) mr[(c / 2) % 8] = fmax3(mr[(c / 2) % 8], sv[c], sv[c + 1]);
      const float mx = fmax3(fmax3(mr[0], mr[1], mr[2]), fmax3(mr[3], mr[4], mr[5]),
                             fmaxf(mr[6], mr[7])) * sl2;  // sl2 > 0: max commutes with scaling
      // Lazy rescaling: keep the stale max m unless the row max grew by more than 2^8, so P
      // stays <= 256 (exact in fp32 accumulation, in range for bf16 and e4m3).
      bool rescale = false;
      float f = 1.f;
      if (n == 0) {
        m = mx;
      } else if (mx > m + 8.f) {
        f = ex2(m - mx);
        l *= f;
        m = mx;
        rescale = true;
      }
      const float mu = (m == -INFINITY) ? 0.f : m;
      const float sum = diag ? p_pass(sv, mu, std::true_type{}) : p_pass(sv, mu, std::false_type{});
      l += sum;
      // tcgen05.ld/st are warp-collective: when any row of the warp rescales, the whole warp
      // runs the pass (f = 1 for rows that keep their max).
      if (__any_sync(0xffffffffu, rescale)) {
        // PV of the previous block has completed (it precedes S of this block on the tensor
        // pipe), and the next PV waits for p_full: O can be rescaled in place.
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          float o[32];
          tmem_ld32(o_tm + c, o);
          tmem_ld_wait();
          uint32_t w[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) w[e] = __float_as_uint(o[e] * f);
          tmem_st32(o_tm + c, w);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&sh.p_full[t]);
      ++n;
      J = J_next;
    }
    // Epilogue: wait for the last PV of this tile, normalise, store.
    const bool fin = ok && !sh.abort_flag && mbar_wait(&sh.o_final[t], 0);
    if (__all_sync(0xffffffffu, fin)) {
      tc_fence_after();
      // Output row of tile row r: its query row, or, with a paged output, the slot of its
      // absolute position in the page the K/V page table gives (an entry out of range skips
      // the row and records kStatusBadIndex).
      bool valid = r >= T.r0 && r < T.r1;
      size_t out_row = static_cast<size_t>(T.q_lo + r);
      if (OUTP && valid) {
        int b_out = b;
        if constexpr (QP) b_out = t == 0 ? rq[0].b : rq[1].b;
        const int pos = T.I * BN + r;
        const int lp = pos / a.page_size;
        const int pg = lp < a.max_pages
                           ? __ldg(a.page_table + static_cast<size_t>(b_out) * a.max_pages + lp) : -1;
        if (pg >= 0 && pg < a.num_pages) {
          out_row = static_cast<size_t>(pg) * a.page_size + pos % a.page_size;
        } else {
          record_status(a.status, kStatusBadIndex);
          valid = false;
        }
      }
      __nv_bfloat16* orow = a.out + (out_row * a.Hq + T.h) * D;
      if (n > 0) {
        float inv = (l > 0.f) ? 1.f / l : 0.f;
        if constexpr (FP8) inv *= __ldg(a.v_scale + g);
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          float o[32];
          tmem_ld32(o_tm + c, o);
          tmem_ld_wait();
          if (valid) {
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint4 v;
              v.x = pack_bf16x2(o[e] * inv, o[e + 1] * inv);
              v.y = pack_bf16x2(o[e + 2] * inv, o[e + 3] * inv);
              v.z = pack_bf16x2(o[e + 4] * inv, o[e + 5] * inv);
              v.w = pack_bf16x2(o[e + 6] * inv, o[e + 7] * inv);
              *reinterpret_cast<uint4*>(orow + c + e) = v;
            }
          }
        }
        if (valid && a.lse != nullptr)
          a.lse[static_cast<size_t>(T.h) * a.s.total_q + T.q_lo + r] =
              (l > 0.f) ? (m + log2f(l)) * 0.69314718055994530942f : -INFINITY;
      } else if (valid) {
        // No kept block at all: the row attends to nothing; write zeros / -inf.
        for (int c = 0; c < D; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(0, 0, 0, 0);
        if (a.lse != nullptr)
          a.lse[static_cast<size_t>(T.h) * a.s.total_q + T.q_lo + r] = -INFINITY;
      }
    } else {
      record_status(a.status, kStatusTimeout);
      sh.abort_flag = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
  // After a failed wait some issued load may never have been consumed: wait (bounded) until
  // every bulk copy of this CTA has landed, so none still writes shared memory after exit.
  if (warp == 0 && lane == 0 && sh.abort_flag) {
    if (q_issued) mbar_wait(&sh.q_full, 0);
    for (int i = 0; i < C::kKSt; ++i)
      if (k_issued[i] >= 0) mbar_wait(&sh.k_full[i], k_issued[i] & 1);
    for (int i = 0; i < C::kVSt; ++i)
      if (v_issued[i] >= 0) mbar_wait(&sh.v_full[i], v_issued[i] & 1);
  }
}

// ------------------------------------------------------------------------------------ host side
// [rows, heads, d] token-major tensor; box = (one 128-byte chunk of d, 1 head, box_rows rows).
static bool make_map(CUtensorMap* m, const void* base, bool e4m3, int d, int heads,
                     long long rows, int box_rows) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  const int eb = e4m3 ? 1 : 2;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(heads),
                        static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * eb,
                           static_cast<cuuint64_t>(d) * heads * eb};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / eb), 1u, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(m, e4m3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                   const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, int BN, bool FP8, bool PAGED, bool OUTP, bool QP>
static cudaError_t launch_s(const AttnArgs& a, const AttnLaunch& L, cudaStream_t stream) {
  using C = AttnCfg<D, BN, FP8>;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, L.q, FP8, D, a.Hq, a.s.total_q, 128) ||
      !make_map(&mk, L.k, FP8, D, a.Hkv, L.kv_rows, L.seg_rows) ||
      !make_map(&mv, L.v, FP8, D, a.Hkv, L.kv_rows, L.seg_rows))
    return cudaErrorInvalidValue;
  auto kern = attn_kernel<D, BN, FP8, PAGED, OUTP, QP>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::kSmemBytes);
  if (e != cudaSuccess) return e;
  if (a.num_items == 0) return cudaSuccess;
  kern<<<a.num_items, C::kThreads, C::kSmemBytes, stream>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

// Work split: the head-pair kernel unless some head pairs query blocks (odd G or G = 1 on
// problems large enough, or FP_PAIR_QBLOCKS).
template <int D, int BN, bool FP8, bool PAGED, bool OUTP = false>
static cudaError_t launch_t(const AttnArgs& a, const AttnLaunch& L, cudaStream_t stream) {
  return a.qpair_heads > 0 ? launch_s<D, BN, FP8, PAGED, OUTP, true>(a, L, stream)
                           : launch_s<D, BN, FP8, PAGED, OUTP, false>(a, L, stream);
}

// Paged K/V: with the paged output layout or without it.
template <int D, int BN, bool FP8>
static cudaError_t launch_paged(const AttnArgs& a, const AttnLaunch& L, cudaStream_t stream) {
  return a.out_paged ? launch_t<D, BN, FP8, true, true>(a, L, stream)
                     : launch_t<D, BN, FP8, true, false>(a, L, stream);
}

cudaError_t launch_attn(const AttnArgs& a, const AttnLaunch& L, int block, cudaStream_t stream) {
  if (a.out_paged && !L.paged) return cudaErrorInvalidValue;
  if (L.e4m3) {
    if (L.d == 128 && block == 128)
      return L.paged ? launch_paged<128, 128, true>(a, L, stream)
                     : launch_t<128, 128, true, false>(a, L, stream);
    return cudaErrorNotSupported;
  }
  if (L.d == 128 && block == 128)
    return L.paged ? launch_paged<128, 128, false>(a, L, stream)
                   : launch_t<128, 128, false, false>(a, L, stream);
  if (L.d == 64 && block == 64)
    return L.paged ? launch_paged<64, 64, false>(a, L, stream)
                   : launch_t<64, 64, false, false>(a, L, stream);
  if (L.d == 128 && block == 64)
    return L.paged ? launch_paged<128, 64, false>(a, L, stream)
                   : launch_t<128, 64, false, false>(a, L, stream);
  if (L.d == 64 && block == 128)
    return L.paged ? launch_paged<64, 128, false>(a, L, stream)
                   : launch_t<64, 128, false, false>(a, L, stream);
  return cudaErrorNotSupported;
}

}  // namespace fp
