"""Host-side checks of the seeded input generator (no method arithmetic is involved)."""
import numpy as np
import torch

from block_sparse_long_qk_b200 import synthetic as S


def test_deterministic_and_shapes():
    a = S.make_inputs("tiny", seed=5)
    b = S.make_inputs("tiny", seed=5)
    c = S.make_inputs("tiny", seed=6)
    assert a.q.shape == (2048, 4, 64) and a.k.shape == (2048, 4, 64)
    assert a.q.dtype == torch.bfloat16
    assert torch.equal(a.q, b.q) and torch.equal(a.v, b.v)
    assert not torch.equal(a.q, c.q)
    assert a.cu_seqlens.tolist() == [0, 2048]


def test_e4m3_quantisation_per_head():
    x = torch.randn(300, 3, 16) * torch.tensor([0.01, 1.0, 50.0])[None, :, None]
    codes, scale = S.quantize_e4m3(x)
    assert codes.dtype == torch.float8_e4m3fn and scale.shape == (3,)
    back = codes.to(torch.float32) * scale[None, :, None]
    # absmax maps onto the largest finite e4m3 value, 448
    assert torch.equal(codes.to(torch.float32).abs().amax(dim=(0, 2)),
                       torch.full((3,), 448.0))
    # round-to-nearest: relative error at most half an ulp (2^-4) above the subnormals
    big = (x / scale[None, :, None]).abs() >= 2.0 ** -6
    rel = ((back - x).abs() / x.abs())[big]
    assert rel.max() <= 2.0 ** -4 + 1e-6


def test_paged_layout_round_trip():
    w = S.WORKLOADS["paged"]
    inp = S.make_inputs(w, seqlens=(100, 64, 1))
    P = w.page_size
    cu = inp.cu_seqlens.tolist()
    for b, L in enumerate((100, 64, 1)):
        for t in range(L):
            page = int(inp.page_table[b, t // P])
            assert torch.equal(inp.k_cache[page, t % P], inp.k[cu[b] + t])
            assert torch.equal(inp.v_cache[page, t % P], inp.v[cu[b] + t])
    used = inp.page_table[inp.page_table >= 0].tolist()
    assert sorted(used) == list(range(len(used)))


def test_vertical_stripes_planted():
    w = S.WORKLOADS["llama32k"]
    inp = S.make_inputs(w, seqlens=(4096,))
    k = inp.k.float()
    norms = k.norm(dim=-1).mean(dim=1)
    # 64 planted rows stand out by the 3u shift: norm ~ sqrt(11.3 + 9) = 4.5 against a
    # base norm ~ sqrt(128 / sqrt(128)) = 3.4 (averaged over the 8 KV heads)
    assert int((norms > norms.median() + 0.6).sum()) == 64


def test_chunked_queries_are_the_last_positions():
    w = S.WORKLOADS["chunked"]
    assert len(w.q_lens) == w.batch and all(1 <= n <= min(L, 16384)
                                            for n, L in zip(w.q_lens, w.seqlens))
    small = S.make_inputs(w, seqlens=(300, 700, 5), q_lens=(100, 0, 5))
    assert small.q.shape == (105, w.Hq, w.d) and small.k.shape == (1005, w.Hkv, w.d)
    assert small.cu_q.tolist() == [0, 100, 100, 105]
    assert small.cu_seqlens.tolist() == [0, 300, 1000, 1005]
    # With every position a query, the chunked draw is the plain draw of the same recipe.
    full = S.make_inputs(w, seqlens=(300, 70), q_lens=(300, 70))
    plain = S.make_inputs(S.Workload("chunked", (300, 70), w.Hq, w.Hkv, w.d, w.block,
                                     structure=w.structure, page_size=w.page_size),
                          seed=S.DEFAULT_SEEDS["chunked"])
    for n in ("q", "k", "v", "k_cache", "page_table"):
        assert torch.equal(getattr(full, n), getattr(plain, n)), n
    try:
        S.make_inputs(w, seqlens=(10,), q_lens=(11,))
    except ValueError:
        pass
    else:
        raise AssertionError("q_len > kv_len accepted")
