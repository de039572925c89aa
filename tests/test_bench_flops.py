"""The FLOP counts behind the bench's headline metric, pinned on CPU.

The metric counts 4 D per unmasked (query, key) pair of the selected blocks.
bench.selected_pairs uses the closed form (min(k, i + 1) blocks per query
block, the diagonal one causal); here the pairs are counted one by one from
the oracle's own block table on the tiny workload, and the dense causal count
is checked against S (S + 1) / 2 per head."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
import gen  # noqa: E402
import oracle  # noqa: E402


def test_selected_pairs_equal_a_token_by_token_count_of_the_oracle_table():
    x = gen.make_inputs("tiny_1k")
    w = x.workload
    kb, qb = oracle.block_pool(x.k, x.q)
    idx, _ = oracle.block_select(qb, kb, w.top_k)
    S, n = w.seq_len, w.n_blocks
    tok_block = np.arange(S) // 64
    for h in range(w.n_kv_heads):
        pairs = 0
        for t in range(S):
            i = t // 64
            sel = idx[0, h, i][idx[0, h, i] >= 0]
            keys = np.arange(t + 1)                       # causal: s <= t
            pairs += int(np.isin(tok_block[keys], sel).sum())
        assert pairs == bench.selected_pairs(w), (h, pairs)
    assert n == S // 64


def test_headline_flops_of_the_two_benchmarked_workloads():
    # 4 D x pairs x batch x query heads; the 8k layer at k = 16 and the 32k
    # workload at k = 16 (the figures the scope table quotes: 6.26e10, 2.62e11)
    w8 = gen.WORKLOADS["llama1b_8k"]
    w32 = gen.WORKLOADS["long_32k"]
    assert abs(bench.algorithmic_flops(w8) - 6.26e10) / 6.26e10 < 5e-3
    assert abs(bench.algorithmic_flops(w32) - 2.62e11) / 2.62e11 < 5e-3


def test_causal_flops_count_every_causal_pair():
    for name in ("tiny_1k", "llama1b_8k", "long_32k"):
        w = gen.WORKLOADS[name]
        S = w.seq_len
        pairs = S * (S + 1) // 2
        assert bench.causal_flops(w) == 4.0 * w.head_dim * pairs * w.batch * w.n_q_heads


def test_full_budget_selection_counts_every_causal_pair():
    # with k >= n every causal block is selected, so the sparse count is the
    # dense one
    w = gen.WORKLOADS["tiny_1k"]

    class Full:
        n_blocks = w.n_blocks
        top_k = w.n_blocks
        head_dim, batch, n_q_heads = w.head_dim, w.batch, w.n_q_heads

    assert bench.algorithmic_flops(Full) == bench.causal_flops(w)
