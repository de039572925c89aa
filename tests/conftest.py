"""Shared pytest set-up: markers, import path and cached synthetic inputs."""
import functools
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: a CPU test that takes more than a few seconds")


@functools.lru_cache(maxsize=2)
def workload_inputs(name):
    """Generated once per process: the named workload's bf16 inputs (CPU)."""
    import gen
    return gen.make_inputs(name)


@pytest.fixture
def inputs_of():
    return workload_inputs


def oracle_table(x, topk, gpu_idx=None):
    """The oracle's own block table for inputs x (fp64 pooling, then fp64
    selection).  When the GPU's table is given it must be identical (the
    selection is bit-exact), so both sides then work from the same selection
    without the oracle taking any input from the GPU."""
    import numpy as np

    import oracle
    kb, qb = oracle.block_pool(x.k, x.q)
    idx, _ = oracle.block_select(qb, kb, topk)
    if gpu_idx is not None:
        g = gpu_idx.cpu().numpy()
        mism = np.argwhere(g != idx)
        assert mism.size == 0, f"{len(mism)} index mismatches, first {mism[:3].tolist()}"
    return idx


def same_table_rows(rows, gidx, oidx, G):
    """Filter over (b, query head, token) rows: True where the row's query
    block has the same table row on both sides (selections may differ only
    where two scores are within rounding of the boundary)."""
    import numpy as np
    b, h, i = rows[:, 0], rows[:, 1] // G, rows[:, 2] // 64
    return np.all(gidx[b, h, i] == oidx[b, h, i], axis=-1)


def same_reverse_blocks(blocks, gidx, oidx):
    """Filter over (b, KV head, key block j): True where the same query blocks
    select j on both sides (its dK, dV then sum over the same pairs)."""
    import numpy as np
    out = []
    for b, h, j in blocks:
        out.append(np.array_equal((gidx[b, h] == j).any(axis=-1), (oidx[b, h] == j).any(axis=-1)))
    return np.array(out, dtype=bool)
