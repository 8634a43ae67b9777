"""The pins catch plausible mistakes: each case plants one in a copy of an oracle function (on
the CPU, in this process only), runs the pin meant to catch it, and requires that pin to fail.
The real oracle is restored after every case; nothing here changes what the oracle computes."""
import inspect
import textwrap

import pytest

import oracle as O
import test_oracle_pins as P

# (oracle function, text in its source, planted mistake, pin that must fail)
MUTANTS = [
    ("masked_causal_attention", "key_pos[None, :] > np.arange(p_lo, p_hi)[:, None]",
     "key_pos[None, :] >= np.arange(p_lo, p_hi)[:, None]",
     P.test_alpha0_keeps_every_causal_block_and_equals_dense_bruteforce),   # diagonal key dropped
    ("masked_causal_attention", "kj = np.asarray(k[kbase + key_pos, h // G]",
     "kj = np.asarray(k[kbase + key_pos, h % k.shape[1]]",
     P.test_gqa_equals_repeated_kv_heads),                                    # wrong KV head
    ("masked_causal_attention", "e = np.exp(s - m)", "e = np.exp(s - m) + 1e-3",
     P.test_alpha0_keeps_every_causal_block_and_equals_dense_bruteforce),   # leaky softmax
    ("masked_causal_attention", "kept = [J for J in range(I + 1) if keeps[b][h, i, J]]",
     "kept = list(range(I + 1))",
     P.test_masked_blocks_contribute_exactly_zero),                           # mask ignored
    ("masked_causal_attention", "vj = vj * float(v_scale[h // G])", "vj = vj",
     P.test_per_head_scale_equals_prescaled_values),                          # V scale dropped
    ("pool_blocks", ".mean(axis=0)", ".sum(axis=0) / block",
     P.test_partial_last_block_mean_closed_form),                             # ragged block mean
    ("block_scores", "full = scale * (qb @ kb.T)", "full = qb @ kb.T",
     P.test_pooled_score_is_mean_of_raw_block_scores),                        # scale dropped
    ("block_scores", "kb = k_pool[h // G, koff[b]:koff[b] + n]",
     "kb = k_pool[h // G, koff[b]:koff[b] + n][::-1]",
     P.test_pooled_score_is_mean_of_raw_block_scores),                        # blocks reversed
    ("block_keep", "keep = p >= alpha * p.max(axis=-1, keepdims=True)",
     "keep = p > alpha * p.max(axis=-1, keepdims=True)",
     lambda: P.test_row_max_always_kept_and_alpha_limits(1.0)),               # tie excluded
    ("block_keep", "keep[:, :, 0] = True", "pass", P.test_threshold_golden_row),   # first not forced
    ("block_keep", "keep[:, np.arange(nq), rows] = True", "pass",
     P.test_threshold_golden_row),                                            # diagonal not forced
    ("pool_query_blocks", "lo, hi = max(P0, I * block), min(L, (I + 1) * block)",
     "lo, hi = I * block, min(L, (I + 1) * block)",
     P.test_chunked_query_pool_closed_form),                                  # prefix in the mean
    ("query_blocks", "I0 = P0 // block", "I0 = (P0 + block - 1) // block",
     P.test_chunked_alpha0_equals_dense_rows_of_the_full_sequence),           # first block lost
    ("query_blocks", "nq = (L + block - 1) // block - I0 if n > 0 else 0",
     "nq = (L + block - 1) // block - I0",
     P.test_chunked_request_without_new_queries_has_no_query_block),         # block of no query
    ("block_scores", "kb = k_pool[h // G, koff[b]:koff[b] + n]",
     "kb = k_pool[h % Hkv, koff[b]:koff[b] + n]",
     P.test_pooled_score_is_mean_of_raw_block_scores),                        # wrong KV head
    ("masked_causal_attention", "k_scale[h // G]", "k_scale[h % Hkv]",
     P.test_per_head_scale_equals_prescaled_values),                          # wrong K scale
    ("masked_causal_attention", "(m + np.log(z))", "(np.log(z))",
     P.test_alpha0_keeps_every_causal_block_and_equals_dense_bruteforce),   # LSE without max
    ("_row_softmax", "e = np.exp(s - m)", "e = np.exp(s)",
     lambda: P.test_row_max_always_kept_and_alpha_limits(0.1)),               # overflowing softmax
    ("block_keep", "keep &= causal[None]", "pass",
     P.test_alpha0_keeps_every_causal_block_and_equals_dense_bruteforce),   # blocks past diagonal
    ("pool_blocks", "hi = min(cu[b + 1], lo + block)", "hi = lo + block",
     P.test_partial_last_block_mean_closed_form),                             # tail past request
    ("request_blocks", "(cu[b + 1] - cu[b] + block - 1) // block", "(cu[b + 1] - cu[b]) // block",
     P.test_partial_last_block_mean_closed_form),                             # ragged block lost
]


@pytest.mark.filterwarnings("ignore::RuntimeWarning")  # a mutant may divide by zero or so
@pytest.mark.parametrize("case", range(len(MUTANTS)))
def test_pin_catches_planted_mistake(case):
    name, old, new, pin = MUTANTS[case]
    original = getattr(O, name)
    src = textwrap.dedent(inspect.getsource(original))
    assert src.count(old) == 1, f"anchor not found once in oracle.{name}"
    scope = dict(vars(O))
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), scope)
    setattr(O, name, scope[name])
    try:
        with pytest.raises(AssertionError):
            pin()
    finally:
        setattr(O, name, original)
    pin()  # and the real oracle passes it again
