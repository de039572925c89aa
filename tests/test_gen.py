"""The seeded generator: determinism, planted structure and the score-gap guarantee."""
import numpy as np
import pytest
import torch

import gen
import oracle
from conftest import workload_inputs

BS = 64


def test_same_seed_same_bits_and_shapes():
    a = gen.make_inputs("tiny_1k")
    b = gen.make_inputs("tiny_1k")
    for x, y in ((a.q, b.q), (a.k, b.k), (a.v, b.v)):
        assert x.dtype == torch.bfloat16
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))
    assert tuple(a.q.shape) == (1, 1024, 4, 64)
    assert tuple(a.k.shape) == (1, 1024, 1, 64)


def test_redraw_touches_only_its_row():
    base = gen.make_custom(1, 512, 4, 2, 16, 2, seed=3, n_plant=2)
    red = gen.make_custom(1, 512, 4, 2, 16, 2, seed=3, n_plant=2, redraws=[[0, 1, 5, 1]])
    diff = (base.q != red.q).any(dim=-1)          # [B, S, Hq]
    changed = torch.nonzero(diff)
    assert changed.numel() > 0
    assert set(changed[:, 1].div(BS, rounding_mode="floor").tolist()) == {5}
    assert set(changed[:, 2].tolist()) <= {2, 3}   # heads of KV head 1 (G = 2)
    assert torch.equal(base.k, red.k) and torch.equal(base.v, red.v)


def test_plants_shift_queries_toward_their_blocks():
    x = gen.make_custom(1, 1024, 4, 1, 64, 4, seed=9, n_plant=3, plant_shift=1.5)
    for i in range(4, 16):
        p = x.plants[(0, 0, i)]
        assert len(p) == 3 and all(0 <= j < i for j in p) and len(set(p)) == 3
    assert x.plants[(0, 0, 2)] == (0, 1)


@pytest.mark.slow
@pytest.mark.parametrize("name", list(gen.WORKLOADS))
def test_every_row_has_the_score_gap(name):
    x = workload_inputs(name)
    kbar, qbar = oracle.block_pool(x.k, x.q)
    for topk in x.workload.gap_budgets:
        _, gap = oracle.block_select(qbar, kbar, topk)
        defined = ~np.isnan(gap)
        assert defined.any()
        assert np.all(gap[defined] > 1e-3), (name, topk, float(np.nanmin(gap)))
