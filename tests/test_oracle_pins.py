"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these re-call an oracle routine to produce an expected value. Each pin comes
from outside the oracle: brute-force loops over single tokens, a closed form, the
hand-worked threshold row under ``tests/golden/``, or a reduction to a simpler case
(GQA to repeated heads, a varlen batch to its requests run alone, masked blocks to
NaN-poisoned ones).

Sources: "FlashPrefill: Instantaneous Pattern Discovery and Thresholding for Ultra-Fast
Long-Context Prefilling", technical summary 2.A (block means, fused 2-D reduction), 2.B
(max-based threshold), 2.C (physical skip of masked blocks).
"""
import json
import math
import os

import numpy as np
import pytest

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed):
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(shape)


def _brute_attention(q, k, v, cu, scale):
    """Dense causal softmax attention, one query and one key at a time (pure Python)."""
    T, Hq, d = q.shape
    G = Hq // k.shape[1]
    out = np.zeros((T, Hq, d))
    lse = np.zeros((Hq, T))
    for b in range(len(cu) - 1):
        for h in range(Hq):
            for i in range(cu[b], cu[b + 1]):
                logits = []
                for j in range(cu[b], i + 1):
                    acc = 0.0
                    for c in range(d):
                        acc += q[i, h, c] * k[j, h // G, c]
                    logits.append(scale * acc)
                m = max(logits)
                w = [math.exp(x - m) for x in logits]
                z = sum(w)
                for c in range(d):
                    out[i, h, c] = sum(w[t] * v[cu[b] + t, h // G, c] for t in range(len(w))) / z
                lse[h, i] = m + math.log(z)
    return out, lse


def _all_causal_keep(cu, block, Hq):
    nb, _ = O.request_blocks(cu, block)
    return [np.tril(np.ones((Hq, n, n), dtype=bool)) for n in nb]


def test_alpha0_keeps_every_causal_block_and_equals_dense_bruteforce():
    """With the threshold disabled (alpha = 0) every causal block is kept and the
    masked attention is plain dense causal softmax attention."""
    cu = [0, 37, 37 + 64, 37 + 64 + 50]
    T, Hq, Hkv, d, block = cu[-1], 4, 2, 8, 16
    q, k, v = _rand((T, Hq, d), 1), _rand((T, Hkv, d), 2), _rand((T, Hkv, d), 3)
    scale = 1.0 / math.sqrt(d)
    qp = O.pool_blocks(q, block, cu)
    kp = O.pool_blocks(k, block, cu)
    keeps = [O.block_keep(s, 0.0) for s in O.block_scores(qp, kp, cu, block, scale)]
    for kk, ref in zip(keeps, _all_causal_keep(cu, block, Hq)):
        assert np.array_equal(kk, ref)
    out, lse = O.masked_causal_attention(q, k, v, keeps, cu, block, scale)
    bo, bl = _brute_attention(q, k, v, cu, scale)
    np.testing.assert_allclose(out, bo, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, bl, rtol=0, atol=1e-12)


def test_pooled_score_is_mean_of_raw_block_scores():
    """Linearity behind the fused 2-D reduction: qbar_I . kbar_J * scale equals the mean
    over the (valid) I x J rectangle of the raw scaled scores q_i . k_j. Above the block
    diagonal the pooled row is masked (-inf). Three query heads per KV head, so that a wrong
    head mapping (h % Hkv instead of h // G) changes the scores."""
    cu = [0, 40, 40 + 29]
    Hq, Hkv, d, block = 6, 2, 4, 8
    G = Hq // Hkv
    T = cu[-1]
    q, k = _rand((T, Hq, d), 4), _rand((T, Hkv, d), 5)
    scale = 1.0 / math.sqrt(d)
    s = O.block_scores(O.pool_blocks(q, block, cu), O.pool_blocks(k, block, cu), cu, block,
                       scale)
    for b in range(len(cu) - 1):
        L = cu[b + 1] - cu[b]
        n = (L + block - 1) // block
        for h in range(Hq):
            for I in range(n):
                for J in range(n):
                    if J > I:
                        assert s[b][h, I, J] == -np.inf
                        continue
                    tot, cnt = 0.0, 0
                    for i in range(cu[b] + I * block, cu[b] + min(L, (I + 1) * block)):
                        for j in range(cu[b] + J * block, cu[b] + min(L, (J + 1) * block)):
                            tot += scale * sum(q[i, h, c] * k[j, h // G, c] for c in range(d))
                            cnt += 1
                    assert s[b][h, I, J] == pytest.approx(tot / cnt, abs=1e-12)


def test_partial_last_block_mean_closed_form():
    """x[t] = t: the mean of block [lo, hi) is (lo + hi - 1) / 2, the ragged last block of
    each request included."""
    cu = [0, 21, 21 + 16, 21 + 16 + 5]
    T, block = cu[-1], 8
    x = np.zeros((T, 1, 3))
    for b in range(3):
        for t in range(cu[b], cu[b + 1]):
            x[t, 0, :] = t - cu[b]
    p = O.pool_blocks(x, block, cu)
    expect = []
    for b in range(3):
        L = cu[b + 1] - cu[b]
        for I in range((L + block - 1) // block):
            lo, hi = I * block, min(L, (I + 1) * block)
            expect.append((lo + hi - 1) / 2.0)
    np.testing.assert_array_equal(p[0, :, 0], np.array(expect))


def test_threshold_golden_row():
    g = json.load(open(os.path.join(GOLDEN, "threshold_row.json")))
    s = np.full((1, 6, 6), -np.inf)
    s[0, 5, :] = g["scores"]
    for I in range(5):
        s[0, I, : I + 1] = 0.0
    keep = O.block_keep(s, g["alpha"])[0, 5]
    assert keep.tolist() == g["keep"]
    keep_t = O.block_keep(s, g["alpha"], force_first=False, force_diag=False)[0, 5]
    assert keep_t.tolist() == g["keep_threshold_only"]
    np.testing.assert_allclose(O.keep_ratio(s)[0, 5], g["ratio"], rtol=1e-14)


@pytest.mark.parametrize("alpha", [1e-30, 0.05, 0.1, 0.5, 1.0])
def test_row_max_always_kept_and_alpha_limits(alpha):
    n, Hq = 24, 3
    s = np.full((Hq, n, n), -np.inf)
    r = _rand((Hq, n, n), 6) * 3.0
    tri = np.tril(np.ones((n, n), dtype=bool))
    s[:, tri] = r[:, tri]
    keep = O.block_keep(s, alpha, force_first=False, force_diag=False)
    arg = np.argmax(np.where(tri[None], s, -np.inf), axis=-1)
    for h in range(Hq):
        for I in range(n):
            assert keep[h, I, arg[h, I]]
            assert not keep[h, I, I + 1:].any()
    if alpha == 1.0:   # no ties in continuous random scores: only the argmax survives
        assert (keep.sum(axis=-1) == 1).all()
    if alpha == 1e-30:  # scores of std 3 span far less than ln(1e30) = 69: all kept
        assert np.array_equal(keep, np.broadcast_to(tri, keep.shape))
    # softmax is shift invariant: adding a constant to a row changes nothing, even a constant
    # far past the range of exp (a softmax that does not subtract the row max overflows there)
    for shift in (7.5, 800.0, -800.0):
        keep2 = O.block_keep(s + shift, alpha, force_first=False, force_diag=False)
        assert np.array_equal(keep, keep2)


def test_masked_blocks_contribute_exactly_zero():
    """Physical skip: poisoning the K and V rows of every block that a (head, query
    block) row did not keep with NaN leaves that row's output bit-identical."""
    cu = [0, 96]
    T, Hq, Hkv, d, block = 96, 2, 1, 8, 16
    q, k, v = _rand((T, Hq, d), 7), _rand((T, Hkv, d), 8), _rand((T, Hkv, d), 9)
    scale = 1.0 / math.sqrt(d)
    n = T // block
    keep = np.tril(np.ones((Hq, n, n), dtype=bool))
    keep[0, 5, [1, 2, 4]] = False
    ref, ref_lse = O.masked_causal_attention(q, k, v, [keep], cu, block, scale, rows=[(0, 5)])
    kp, vp = k.copy(), v.copy()
    for J in (1, 2, 4):
        kp[J * block:(J + 1) * block] = np.nan
        vp[J * block:(J + 1) * block] = np.nan
    out, lse = O.masked_causal_attention(q, kp, vp, [keep], cu, block, scale, rows=[(0, 5)])
    rows = slice(5 * block, 6 * block)
    assert np.isfinite(out[rows, 0]).all()
    assert np.array_equal(out[rows, 0], ref[rows, 0])
    assert np.array_equal(lse[0, rows], ref_lse[0, rows])
    # and dropping blocks does change the result (the mask is actually applied)
    full, _ = O.masked_causal_attention(q, k, v, [np.tril(np.ones_like(keep))], cu, block,
                                        scale, rows=[(0, 5)])
    assert not np.allclose(full[rows, 0], ref[rows, 0])


def test_gqa_equals_repeated_kv_heads():
    cu = [0, 70]
    T, Hq, Hkv, d, block = 70, 4, 2, 8, 16
    q, k, v = _rand((T, Hq, d), 10), _rand((T, Hkv, d), 11), _rand((T, Hkv, d), 12)
    rep = [0, 0, 1, 1]
    kr, vr = k[:, rep], v[:, rep]
    scale = 1.0 / math.sqrt(d)
    def run(kk, vv):
        s = O.block_scores(O.pool_blocks(q, block, cu), O.pool_blocks(kk, block, cu), cu,
                           block, scale)
        keeps = [O.block_keep(x, 0.3) for x in s]
        return keeps, O.masked_causal_attention(q, kk, vv, keeps, cu, block, scale)
    k1, (o1, l1) = run(k, v)
    k2, (o2, l2) = run(kr, vr)
    assert all(np.array_equal(a, b) for a, b in zip(k1, k2))
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_varlen_batch_equals_requests_alone():
    lens = [50, 16, 33]
    cu = [0, 50, 66, 99]
    Hq, Hkv, d, block = 2, 1, 8, 16
    q, k, v = _rand((99, Hq, d), 13), _rand((99, Hkv, d), 14), _rand((99, Hkv, d), 15)
    scale = 1.0 / math.sqrt(d)
    def run(qq, kk, vv, c):
        s = O.block_scores(O.pool_blocks(qq, block, c), O.pool_blocks(kk, block, c), c,
                           block, scale)
        keeps = [O.block_keep(x, 0.2) for x in s]
        return keeps, O.masked_causal_attention(qq, kk, vv, keeps, c, block, scale)
    keeps, (o, l) = run(q, k, v, cu)
    for b, L in enumerate(lens):
        sl = slice(cu[b], cu[b + 1])
        kb, (ob, lb) = run(q[sl], k[sl], v[sl], [0, L])
        assert np.array_equal(keeps[b], kb[0])
        assert np.array_equal(o[sl], ob) and np.array_equal(l[:, sl], lb)


def test_per_head_scale_equals_prescaled_values():
    """e4m3 inputs enter as codes times a per-head scale; the product of a 4-bit code
    and a float32 scale is exact in float64, so scaling inside equals scaling outside."""
    cu = [0, 40]
    T, Hq, Hkv, d, block = 40, 6, 2, 8, 8
    rng = np.random.Generator(np.random.PCG64(16))
    codes = lambda s: rng.integers(-16, 17, size=s).astype(np.float64) * 0.5
    q, k, v = codes((T, Hq, d)), codes((T, Hkv, d)), codes((T, Hkv, d))
    qs = np.array([0.013, 0.25, 0.5, 0.0625, 0.125, 2.0])
    ks, vs = np.array([0.031, 0.375]), np.array([0.7, 0.0078125])
    scale = 1.0 / math.sqrt(d)
    a = O.pool_blocks(q, block, cu, scale=qs)
    b = O.pool_blocks(q * qs[None, :, None], block, cu)
    assert np.array_equal(a, b)
    keep = [np.tril(np.ones((Hq, 5, 5), dtype=bool))]
    o1, _ = O.masked_causal_attention(q, k, v, keep, cu, block, scale, q_scale=qs,
                                      k_scale=ks, v_scale=vs)
    o2, _ = O.masked_causal_attention(q * qs[None, :, None], k * ks[None, :, None],
                                      v * vs[None, :, None], keep, cu, block, scale)
    assert np.array_equal(o1, o2)


# ---- chunked (prefix-cached) prefill: the queries are the last q_len positions of each request

def _chunked_case(seed=17):
    kv_lens, q_lens = [70, 45, 33], [30, 45, 10]     # prefixes 40, 0, 23 (not block aligned)
    ck = np.cumsum([0] + kv_lens).tolist()
    cq = np.cumsum([0] + q_lens).tolist()
    Hq, Hkv, d, block = 4, 2, 8, 16
    qf = _rand((ck[-1], Hq, d), seed)                  # queries of every position
    k, v = _rand((ck[-1], Hkv, d), seed + 1), _rand((ck[-1], Hkv, d), seed + 2)
    rows = [r for b in range(3) for r in range(ck[b + 1] - q_lens[b], ck[b + 1])]
    return qf, qf[rows], k, v, cq, ck, block


def test_chunked_alpha0_equals_dense_rows_of_the_full_sequence():
    """With every causal block kept, chunked attention of the last q_len queries equals the
    matching rows of brute-force dense causal attention over the whole sequence."""
    qf, q, k, v, cq, ck, block = _chunked_case()
    scale = 1.0 / math.sqrt(q.shape[-1])
    info, _ = O.query_blocks(cq, ck, block)
    qp = O.pool_query_blocks(q, block, cq, ck)
    kp = O.pool_blocks(k, block, ck)
    sc = O.block_scores(qp, kp, cq, block, scale, cu_k=ck)
    keeps = [O.block_keep(s, 0.0, row0=info[b][1]) for b, s in enumerate(sc)]
    out, lse = O.masked_causal_attention(q, k, v, keeps, cq, block, scale, cu_k=ck)
    bo, bl = _brute_attention(qf, k, v, ck, scale)
    rows = [r for b in range(3) for r in range(ck[b + 1] - (cq[b + 1] - cq[b]), ck[b + 1])]
    np.testing.assert_allclose(out, bo[rows], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, bl[:, rows], rtol=0, atol=1e-12)


def test_chunked_query_pool_closed_form():
    """x[t] = absolute position: a query block's mean is the mean of the positions it holds,
    max(P0, I*B) .. min(L, (I+1)*B) - 1."""
    kv_lens, q_lens, block = [70, 33], [30, 33], 16
    ck = np.cumsum([0] + kv_lens).tolist()
    cq = np.cumsum([0] + q_lens).tolist()
    q = np.zeros((cq[-1], 1, 2))
    for b in range(2):
        P0 = kv_lens[b] - q_lens[b]
        for i in range(q_lens[b]):
            q[cq[b] + i] = P0 + i
    p = O.pool_query_blocks(q, block, cq, ck)[0, :, 0]
    expect = []
    for b in range(2):
        P0, L = kv_lens[b] - q_lens[b], kv_lens[b]
        for I in range(P0 // block, (L + block - 1) // block):
            lo, hi = max(P0, I * block), min(L, (I + 1) * block)
            expect.append((lo + hi - 1) / 2.0)
    np.testing.assert_array_equal(p, np.array(expect))


def test_chunked_scores_and_keeps_match_the_full_prefill_on_whole_blocks():
    """A query block that lies wholly inside the chunk pools the same queries as in a full
    prefill, so its pooled row, its scores and its keep set are those of the full prefill."""
    qf, q, k, v, cq, ck, block = _chunked_case(23)
    scale = 1.0 / math.sqrt(q.shape[-1])
    info, _ = O.query_blocks(cq, ck, block)
    sc_c = O.block_scores(O.pool_query_blocks(q, block, cq, ck), O.pool_blocks(k, block, ck),
                          cq, block, scale, cu_k=ck)
    sc_f = O.block_scores(O.pool_blocks(qf, block, ck), O.pool_blocks(k, block, ck), ck,
                          block, scale)
    for b, (P0, I0, nq) in enumerate(info):
        kc = O.block_keep(sc_c[b], 0.3, row0=I0)
        kf = O.block_keep(sc_f[b], 0.3)
        for i in range(nq):
            I = I0 + i
            if I * block >= P0:                       # whole block inside the chunk
                assert np.array_equal(sc_c[b][:, i], sc_f[b][:, I])
                assert np.array_equal(kc[:, i], kf[:, I])


def test_empty_request_contributes_nothing():
    """A request without tokens has no blocks: a batch that holds one gives every other
    request exactly what the batch without it gives."""
    rng = np.random.default_rng(41)
    B, H, d = 16, 2, 8
    lens_with, lens_without = (40, 0, 23), (40, 23)
    T = sum(lens_with)
    q, k, v = (rng.standard_normal((T, H, d)) for _ in range(3))
    outs = []
    for lens in (lens_with, lens_without):
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(int)
        qp = O.pool_blocks(q, B, cu)
        kp = O.pool_blocks(k, B, cu)
        sc = O.block_scores(qp, kp, cu, B, 0.3)
        keeps = [O.block_keep(s, 0.2) for s in sc]
        if len(lens) == 3:
            assert sc[1].shape == (H, 0, 0) and keeps[1].shape == (H, 0, 0)
            assert O.keep_ratio(sc[1]).shape == (H, 0, 0)
        outs.append(O.masked_causal_attention(q, k, v, keeps, cu, B, 0.3)[0])
    assert np.array_equal(outs[0], outs[1])


def test_chunked_request_without_new_queries_has_no_query_block():
    """A request with cached keys but no new queries (q_len = 0, kv_len not a multiple of the
    block) holds no query block: the batch with it gives the other requests exactly what the
    batch without it gives, with the same pooled query rows."""
    block, Hq, Hkv, d = 16, 2, 1, 8
    scale = 1.0 / math.sqrt(d)
    k0, k2, kx = _rand((70, Hkv, d), 51), _rand((33, Hkv, d), 52), _rand((37, Hkv, d), 53)
    v0, v2, vx = _rand((70, Hkv, d), 54), _rand((33, Hkv, d), 55), _rand((37, Hkv, d), 56)
    q = _rand((40, Hq, d), 57)                        # 30 new queries, then 10
    runs = []
    for kv_lens, q_lens, k, v in (([70, 37, 33], [30, 0, 10], np.concatenate([k0, kx, k2]),
                                   np.concatenate([v0, vx, v2])),
                                  ([70, 33], [30, 10], np.concatenate([k0, k2]),
                                   np.concatenate([v0, v2]))):
        ck = np.cumsum([0] + kv_lens).tolist()
        cq = np.cumsum([0] + q_lens).tolist()
        info, _ = O.query_blocks(cq, ck, block)
        qp = O.pool_query_blocks(q, block, cq, ck)
        sc = O.block_scores(qp, O.pool_blocks(k, block, ck), cq, block, scale, cu_k=ck)
        keeps = [O.block_keep(x, 0.2, row0=info[b][1]) for b, x in enumerate(sc)]
        runs.append((qp, *O.masked_causal_attention(q, k, v, keeps, cq, block, scale, cu_k=ck)))
    (qp1, o1, l1), (qp2, o2, l2) = runs
    assert qp1.shape == qp2.shape and np.array_equal(qp1, qp2)
    assert np.isfinite(o1).all()
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
