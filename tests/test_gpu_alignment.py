"""GPU parity of the alignment objective's backward (ssa_alignment_bwd):
gradients of <dO, h_mode> + alpha (L_sparsity + L_commit) with respect to
q, k, v against the fp64 oracle, every element, for both modes; and the
alpha = 0 case, which must equal the plain sparse backward bit for bit.

Tolerance per tensor: max-abs <= 2e-2 * max(1, max|oracle|)."""
import numpy as np
import pytest
import torch

import block_sparse_attention_21_b200 as ssa
import gen
import oracle
from conftest import oracle_table

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from block_sparse_attention_21_b200 import build
    build.build()
    ssa.lib()


def _tol(ref):
    return 2e-2 * max(1.0, float(np.abs(ref).max()))


def _oracle_grads(x, idx, mode, alpha):
    B, S, Hq, D = x.q.shape
    Hkv = x.k.shape[2]
    n = S // 64
    rows = oracle.all_rows(B, Hq, S)
    r = oracle.attn_rows(x.q, x.k, x.v, idx, rows, want_full=True)
    to = lambda a: a.reshape(B, Hq, S, D).transpose(0, 2, 1, 3)  # noqa: E731
    d_s, d_f = oracle.alignment_output_grads(to(r["o_sparse"]), to(r["o_full"]), x.do, mode, alpha)
    dense = oracle.dense_causal_table(B, Hkv, n)
    blocks = oracle.all_rows(B, Hkv, n)
    out = []
    for d_o, table in ((d_s, idx), (d_f, dense)):
        dq = oracle.sparse_bwd_dq_rows(x.q, x.k, x.v, d_o, table, rows)
        dk, dv = oracle.sparse_bwd_dkv_blocks(x.q, x.k, x.v, d_o, table, blocks)
        out.append((dq, dk, dv))
    return [a + b for a, b in zip(*out)]


SMALL = [
    # (B, S, Hq, Hkv, D, topk, n_plant)
    (1, 512, 4, 1, 64, 3, 2),
    (2, 320, 8, 2, 64, 2, 0),
    (1, 384, 8, 2, 128, 3, 2),
]


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "x".join(map(str, s)))
def test_alignment_backward_every_element(shape, mode):
    B, S, Hq, Hkv, D, topk, npl = shape
    x = gen.make_custom(B, S, Hq, Hkv, D, topk, seed=500 + S + D + mode, n_plant=npl, with_do=True)
    p = ssa.problem(B, S, Hq, Hkv, D, topk)
    q, k, v, do = (t.to(DEV) for t in (x.q, x.k, x.v, x.do))
    st = ssa.SparseStream(p)
    st.alignment(q, k, v)
    alpha = 0.25 * q.numel()   # alignment output gradients c (h_s - h_f) with c = 0.5
    dq, dk, dv = st.alignment_backward(q, k, v, do, mode, alpha)
    torch.cuda.synchronize()
    assert ssa.ssa_get_device_error() == 0, hex(ssa.ssa_get_device_error_site())
    rdq, rdk, rdv = _oracle_grads(x, oracle_table(x, topk, st.block_idx), mode, alpha)
    n = S // 64
    gdq = dq.float().cpu().numpy().transpose(0, 2, 1, 3).reshape(-1, D)
    gdk = dk.float().cpu().numpy().reshape(B, n, 64, Hkv, D).transpose(0, 3, 1, 2, 4).reshape(-1, 64, D)
    gdv = dv.float().cpu().numpy().reshape(B, n, 64, Hkv, D).transpose(0, 3, 1, 2, 4).reshape(-1, 64, D)
    assert np.abs(gdq - rdq).max() <= _tol(rdq)
    assert np.abs(gdk - rdk).max() <= _tol(rdk)
    assert np.abs(gdv - rdv).max() <= _tol(rdv)


def test_alpha_zero_is_the_sparse_backward_bit_for_bit():
    B, S, Hq, Hkv, D, topk = 1, 1024, 8, 2, 64, 4
    x = gen.make_custom(B, S, Hq, Hkv, D, topk, seed=610, n_plant=2, with_do=True)
    p = ssa.problem(B, S, Hq, Hkv, D, topk)
    q, k, v, do = (t.to(DEV) for t in (x.q, x.k, x.v, x.do))
    st = ssa.SparseStream(p)
    st.alignment(q, k, v)
    a = [t.clone() for t in st.alignment_backward(q, k, v, do, 0, 0.0)]
    b = st.backward(q, k, v, do)
    torch.cuda.synchronize()
    for x1, x2 in zip(a, b):
        assert torch.equal(x1.view(torch.int16), x2.view(torch.int16))
