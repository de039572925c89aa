"""GPU parity of the sparse backward (dQ, dK, dV over the selected pairs)
against the fp64 oracle's explicit formulas, through the C ABI.

Tolerance per tensor: max-abs <= 2e-2 * max(1, max|oracle|) (bf16 inputs and
outputs, fp32 accumulation, P and dS rounded to bf16 for the MMAs), and exact
zeros where the oracle is exactly zero.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_21_b200 as ssa
import gen
import oracle
from conftest import oracle_table, workload_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _tol(ref):
    return 2e-2 * max(1.0, float(np.abs(ref).max()))


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from block_sparse_attention_21_b200 import build
    build.build()
    ssa.lib()


def _run(x, p, do):
    """GPU pool -> select -> forward -> backward; returns tensors on the GPU."""
    q, k, v = (t.to(DEV) for t in (x.q, x.k, x.v))
    st = ssa.SparseStream(p)
    st.forward(q, k, v)
    dq, dk, dv = st.backward(q, k, v, do.to(DEV))
    torch.cuda.synchronize()
    assert ssa.ssa_get_device_error() == 0, hex(ssa.ssa_get_device_error_site())
    return st, dq, dk, dv


def _check_all(x, do, idx, dq, dk, dv):
    B, S, Hq, D = x.q.shape
    Hkv = x.k.shape[2]
    n = S // 64
    rows = oracle.all_rows(B, Hq, S)
    rdq = oracle.sparse_bwd_dq_rows(x.q, x.k, x.v, do, idx, rows)
    gdq = dq.float().cpu().numpy()[rows[:, 0], rows[:, 2], rows[:, 1]]
    assert np.abs(gdq - rdq).max() <= _tol(rdq)
    blocks = oracle.all_rows(B, Hkv, n)
    rdk, rdv = oracle.sparse_bwd_dkv_blocks(x.q, x.k, x.v, do, idx, blocks)
    gdk = dk.float().cpu().numpy().reshape(B, n, 64, Hkv, D).transpose(0, 3, 1, 2, 4).reshape(-1, 64, D)
    gdv = dv.float().cpu().numpy().reshape(B, n, 64, Hkv, D).transpose(0, 3, 1, 2, 4).reshape(-1, 64, D)
    assert np.abs(gdk - rdk).max() <= _tol(rdk)
    assert np.abs(gdv - rdv).max() <= _tol(rdv)
    assert np.all(gdk[rdk == 0.0] == 0.0) and np.all(gdv[rdv == 0.0] == 0.0)


SMALL = [
    # (B, S, Hq, Hkv, D, topk, n_plant)
    (1, 512, 4, 1, 64, 3, 2),
    (2, 320, 8, 2, 64, 2, 0),
    (1, 384, 8, 2, 128, 3, 2),
    (1, 256, 16, 1, 64, 4, 0),     # budget = every causal block
    (1, 512, 4, 2, 128, 1, 0),     # diagonal block only
]


@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "x".join(map(str, s)))
def test_backward_small_every_element(shape):
    B, S, Hq, Hkv, D, topk, npl = shape
    x = gen.make_custom(B, S, Hq, Hkv, D, topk, seed=300 + S + D, n_plant=npl, with_do=True)
    p = ssa.problem(B, S, Hq, Hkv, D, topk)
    st, dq, dk, dv = _run(x, p, x.do)
    _check_all(x, x.do, oracle_table(x, topk, st.block_idx), dq, dk, dv)


def test_backward_zero_gradient_for_unselected_keys():
    # dO = 0 on query block j; a key block no later query block selects then
    # gets dK = dV = 0 exactly
    B, S, Hq, Hkv, D, topk = 1, 1024, 4, 1, 64, 2
    x = gen.make_custom(B, S, Hq, Hkv, D, topk, seed=77, n_plant=1, with_do=True)
    p = ssa.problem(B, S, Hq, Hkv, D, topk)
    kb, qb = oracle.block_pool(x.k, x.q)
    idx, _ = oracle.block_select(qb, kb, topk)
    n = S // 64
    lonely = [j for j in range(n) if not any(j in idx[0, 0, i] for i in range(j + 1, n))]
    assert lonely
    do = x.do.clone()
    for j in lonely:
        do[0, 64 * j:64 * (j + 1)] = 0
    st, dq, dk, dv = _run(x, p, do)
    for j in lonely:
        assert torch.all(dk[0, 64 * j:64 * (j + 1)] == 0) and torch.all(dv[0, 64 * j:64 * (j + 1)] == 0)


def test_backward_training_workload_sampled_and_deterministic():
    x = workload_inputs("train_8k")
    w = x.workload
    p = ssa.problem(w.batch, w.seq_len, w.n_q_heads, w.n_kv_heads, w.head_dim, w.top_k)
    st, dq, dk, dv = _run(x, p, x.do)
    idx = oracle_table(x, w.top_k, st.block_idx)
    q, k, v = (t.to(DEV) for t in (x.q, x.k, x.v))
    dq2, dk2, dv2 = st.backward(q, k, v, x.do.to(DEV))
    torch.cuda.synchronize()
    for a, b in ((dq, dq2), (dk, dk2), (dv, dv2)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), "backward is not deterministic"
    rng = np.random.Generator(np.random.PCG64(5))
    rows = np.stack([rng.integers(0, w.batch, 600), rng.integers(0, w.n_q_heads, 600),
                     rng.integers(0, w.seq_len, 600)], axis=1).astype(np.int64)
    rdq = oracle.sparse_bwd_dq_rows(x.q, x.k, x.v, x.do, idx, rows)
    gdq = dq.float().cpu().numpy()[rows[:, 0], rows[:, 2], rows[:, 1]]
    assert np.abs(gdq - rdq).max() <= _tol(rdq)
    blocks = np.array([[0, 0, 0], [1, 2, 5], [3, 3, 127], [2, 1, 64]], dtype=np.int64)
    rdk, rdv = oracle.sparse_bwd_dkv_blocks(x.q, x.k, x.v, x.do, idx, blocks)
    for r, (b, h, j) in enumerate(blocks):
        gk = dk[b, 64 * j:64 * (j + 1), h].float().cpu().numpy()
        gv = dv[b, 64 * j:64 * (j + 1), h].float().cpu().numpy()
        assert np.abs(gk - rdk[r]).max() <= _tol(rdk[r])
        assert np.abs(gv - rdv[r]).max() <= _tol(rdv[r])
