"""Host-side checks of the parity helpers: the bf16 output-rounding allowance of the attention
tolerance and the stratified row sampler of the full-size comparisons."""
import dataclasses

import numpy as np
import torch

from block_sparse_long_qk_b200 import synthetic as S

from _parity import OracleRun, attn_errors, bf16_half_ulp, stratified_rows


def test_half_ulp_of_bf16_values():
    g = np.array([0.0, 1.0, 1.5, -1.99, 2.0, 3.0, -5.0, 0.3])
    want = np.array([0.0, 2.0 ** -8, 2.0 ** -8, 2.0 ** -8, 2.0 ** -7, 2.0 ** -7, 2.0 ** -6,
                     2.0 ** -10])
    assert np.array_equal(bf16_half_ulp(g), want)


def test_exact_values_rounded_to_bf16_have_no_error():
    """An exact result stored as bf16 passes with zero error beyond its own rounding, even where
    that rounding alone exceeds 1e-2 (magnitudes above 4)."""
    r = np.random.default_rng(0).normal(scale=3.0, size=(64, 2, 16))
    g = torch.from_numpy(r).to(torch.bfloat16)
    raw = np.abs(g.double().numpy() - r).max()
    assert raw > 1e-2
    amax, rel = attn_errors(g, r)
    assert amax == 0.0 and rel < 2.0 ** -8


def test_an_error_beyond_the_rounding_is_caught():
    r = np.random.default_rng(1).normal(scale=0.3, size=(64, 2, 16))
    r[5, 1, 3] = 0.25
    g = torch.from_numpy(r).to(torch.bfloat16)
    g[5, 1, 3] = 0.25 + 0.0125          # bf16-exact; 0.0125 off, half ulp there is 2^-10
    amax, _ = attn_errors(g, r)
    assert amax > 1e-2
    # rows outside the comparison (NaN in the oracle output) are ignored
    r2 = r.copy()
    r2[5] = np.nan
    assert attn_errors(g, r2)[0] <= 2.0 ** -8


def test_stratified_rows_cover_every_head_and_decile():
    w = dataclasses.replace(S.WORKLOADS["paged"], Hq=4, Hkv=2, structure="iid")
    inp = S.make_inputs(w, seed=2, seqlens=(3000, 700, 5000, 130))
    run = OracleRun(inp, 0.5)
    rows = stratified_rows(run, run.keeps, w.Hq, seed=3, per_head=16)
    n = run.qoff[-1]
    assert len(rows) == 16 * w.Hq and len(set(rows)) == len(rows)
    ends = {run.qoff[r + 1] - 1 for r in range(len(run.nq))}
    for h in range(w.Hq):
        mine = [Ig for hh, Ig in rows if hh == h]
        assert n - 1 in mine
        assert ends & set(mine)
        edges = np.linspace(0, n, 11).astype(int)
        dec = {int(np.searchsorted(edges, Ig, side="right")) - 1 for Ig in mine}
        assert dec == set(range(10))
    # a row whose GPU mask differs from the oracle's is left out
    gk = [k.copy() for k in run.keeps]
    gk[-1][0, -1, 0] = ~gk[-1][0, -1, 0]
    rows2 = stratified_rows(run, gk, w.Hq, seed=3, per_head=16)
    assert (0, n - 1) not in rows2 and len(rows2) == len(rows) - 1
