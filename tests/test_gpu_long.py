"""GPU parity at long sequences, up to the longest supported one (524288
tokens, 8192 query blocks): the selection kernel's shared-memory radix path
(more than 512 query blocks), the pooling and reverse-index kernels at large
n, and sampled forward and backward outputs against the fp64 oracle.

Tolerances as in the other GPU parity tests: indices bit-exact where the
oracle's score gap exceeds 1e-3, outputs max-abs <= 2e-2, LSE <= 1e-3,
gradients <= 2e-2 * max(1, max|oracle|); the backward is bitwise repeatable.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_21_b200 as ssa
import gen
import oracle
from conftest import same_reverse_blocks, same_table_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from block_sparse_attention_21_b200 import build
    build.build()
    ssa.lib()


LONG = [
    # (B, S, Hq, Hkv, D, topk, n_plant)
    (1, 131072, 2, 1, 64, 8, 4),     # 2048 query blocks
    (1, 65536, 4, 2, 128, 8, 4),     # head_dim 128, 1024 query blocks
    (1, 524288, 2, 1, 64, 16, 4),    # the longest supported sequence
]


@pytest.mark.parametrize("shape", LONG, ids=lambda s: "x".join(map(str, s)))
def test_long_sequence_forward_and_backward(shape):
    B, S, Hq, Hkv, D, topk, npl = shape
    n = S // 64
    x = gen.make_custom(B, S, Hq, Hkv, D, topk, seed=900 + n, n_plant=npl, with_do=True)
    p = ssa.problem(B, S, Hq, Hkv, D, topk)
    q, k, v, do = (t.to(DEV) for t in (x.q, x.k, x.v, x.do))
    st = ssa.SparseStream(p)
    st.forward(q, k, v)
    torch.cuda.synchronize()
    assert ssa.ssa_get_device_error() == 0

    # pooling and selection
    okb, oqb = oracle.block_pool(x.k, x.q)
    assert np.abs(st.k_pooled.cpu().numpy() - okb).max() <= 1e-5
    assert np.abs(st.q_pooled.cpu().numpy() - oqb).max() <= 1e-5
    oidx, gap = oracle.block_select(oqb, okb, topk)
    gidx = st.block_idx.cpu().numpy()
    clear = np.isnan(gap) | (gap > 1e-3)
    assert clear.mean() > 0.5
    assert np.array_equal(gidx[clear], oidx[clear])
    # every row is a valid table: ascending, the diagonal last, -1 padding only
    for i in (0, 1, topk - 1, topk, n // 2, n - 1):
        row = gidx[0, 0, i]
        valid = row[row >= 0]
        assert len(valid) == min(topk, i + 1) and valid[-1] == i and np.all(np.diff(valid) > 0)

    # sparse forward on sampled rows (with the whole first and last query blocks)
    rng = np.random.Generator(np.random.PCG64(n))
    rows = [np.stack([np.zeros(300, np.int64), rng.integers(0, Hq, 300), rng.integers(0, S, 300)], axis=1)]
    for blk in (0, n - 1):
        t = np.arange(64 * blk, 64 * blk + 64)
        rows.append(np.stack([np.zeros_like(t), np.zeros_like(t), t], axis=1))
    rows = np.concatenate(rows).astype(np.int64)
    # the oracle works from its own table; rows whose table row differs (a
    # near-tie at the boundary) are left out
    same = same_table_rows(rows, gidx, oidx, Hq // Hkv)
    assert same.mean() > 0.5
    ref = oracle.attn_rows(x.q, x.k, x.v, oidx, rows, want_full=False)
    r = torch.as_tensor(rows, device=DEV)
    go = st.o[r[:, 0], r[:, 2], r[:, 1]].float().cpu().numpy()
    gl = st.lse[r[:, 0], r[:, 1], r[:, 2]].cpu().numpy()
    assert np.abs(go - ref["o_sparse"])[same].max() <= 2e-2
    assert np.abs(gl - ref["lse_sparse"])[same].max() <= 1e-3
    # the forward on the oracle's own table: every sampled row, none left out
    otab = torch.from_numpy(np.ascontiguousarray(oidx, dtype=np.int32)).to(DEV)
    o2, l2 = torch.empty_like(st.o), torch.empty_like(st.lse)
    ssa.ssa_sparse_attn_fwd(p, q, k, v, otab, o2, l2)
    torch.cuda.synchronize()
    assert ssa.ssa_get_device_error() == 0
    go2 = o2[r[:, 0], r[:, 2], r[:, 1]].float().cpu().numpy()
    gl2 = l2[r[:, 0], r[:, 1], r[:, 2]].cpu().numpy()
    assert np.abs(go2 - ref["o_sparse"]).max() <= 2e-2
    assert np.abs(gl2 - ref["lse_sparse"]).max() <= 1e-3

    # sparse backward: repeatable bit for bit, sampled against the oracle
    dq, dk, dv = (t.clone() for t in st.backward(q, k, v, do))
    dq2, dk2, dv2 = st.backward(q, k, v, do)
    torch.cuda.synchronize()
    assert ssa.ssa_get_device_error() == 0
    for a, b_ in ((dq, dq2), (dk, dk2), (dv, dv2)):
        assert torch.equal(a.view(torch.int16), b_.view(torch.int16))
    brows = rows[:200]
    rdq = oracle.sparse_bwd_dq_rows(x.q, x.k, x.v, x.do, oidx, brows)
    gdq = dq[r[:200, 0], r[:200, 2], r[:200, 1]].float().cpu().numpy()
    bsame = same[:200]
    assert np.abs(gdq - rdq)[bsame].max() <= 2e-2 * max(1.0, float(np.abs(rdq).max()))
    # key block 0 is selected by every early query block: the longest reverse
    # list; blocks whose selecting query blocks differ between the two tables
    # are left out
    blocks = np.array([[0, 0, 0], [0, Hkv - 1, n // 3], [0, 0, n - 1], [0, 0, n // 2], [0, 0, 1]],
                      dtype=np.int64)
    blocks = blocks[same_reverse_blocks(blocks, gidx, oidx)]
    assert len(blocks) >= 2
    rdk, rdv = oracle.sparse_bwd_dkv_blocks(x.q, x.k, x.v, x.do, oidx, blocks)
    for m, (b_, h, j) in enumerate(blocks):
        gk = dk[b_, 64 * j:64 * (j + 1), h].float().cpu().numpy()
        gv = dv[b_, 64 * j:64 * (j + 1), h].float().cpu().numpy()
        assert np.abs(gk - rdk[m]).max() <= 2e-2 * max(1.0, float(np.abs(rdk[m]).max()))
        assert np.abs(gv - rdv[m]).max() <= 2e-2 * max(1.0, float(np.abs(rdv[m]).max()))
