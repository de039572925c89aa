"""GPU check of ssa_sparse_attn_fwd_host, the pipelined host-buffer forward:
its outputs must equal the device-buffer calls (ssa_block_pool,
ssa_block_select, ssa_sparse_attn_fwd) bit for bit, since it runs the same
kernels over chunks of consecutive query blocks (the last chunk may be
shorter).  Its host buffers are also checked against the fp64 oracle on
sampled rows (max-abs 2e-2 for O, 1e-3 for LSE)."""
import numpy as np
import pytest
import torch

import block_sparse_attention_21_b200 as ssa
import gen
import oracle
from conftest import same_table_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from block_sparse_attention_21_b200 import build
    build.build()
    ssa.lib()


@pytest.mark.parametrize("case", [(1, 2048, 8, 2, 64, 6), (2, 1280, 4, 2, 128, 5), (3, 1024, 16, 1, 64, 4),
                                  (1, 8192, 32, 4, 64, 16), (1, 4480, 32, 4, 64, 16), (1, 4096, 16, 2, 128, 8),
                                  (2, 4096, 32, 4, 64, 16)],   # B = 2 in four chunks
                         ids=lambda c: "x".join(map(str, c)))
def test_host_path_equals_device_path(case):
    B, S, Hq, Hkv, D, topk = case
    x = gen.make_custom(B, S, Hq, Hkv, D, topk, seed=1900 + S + D, n_plant=3)
    p = ssa.problem(B, S, Hq, Hkv, D, topk)
    st = ssa.SparseStream(p)
    st.forward(x.q.to(DEV), x.k.to(DEV), x.v.to(DEV))
    hq, hk, hv = (t.contiguous().pin_memory() for t in (x.q, x.k, x.v))
    ho = torch.full(st.o.shape, float("nan"), dtype=torch.bfloat16).pin_memory()
    hl = torch.full(st.lse.shape, float("nan"), dtype=torch.float32).pin_memory()
    st.forward_host(hq, hk, hv, ho, hl)
    torch.cuda.current_stream().synchronize()
    assert ssa.ssa_get_device_error() == 0
    assert torch.equal(ho.view(torch.int16), st.o.cpu().view(torch.int16))
    assert torch.equal(hl, st.lse.cpu())
    # against the oracle: random rows plus every row of the first and last
    # query blocks (batch 0, query head 0), where both tables hold the same row
    n = S // 64
    rng = np.random.Generator(np.random.PCG64(S + D))
    rows = [np.stack([rng.integers(0, B, 400), rng.integers(0, Hq, 400), rng.integers(0, S, 400)], axis=1)]
    for blk in (0, n - 1):
        t = np.arange(64 * blk, 64 * blk + 64)
        rows.append(np.stack([np.zeros_like(t), np.zeros_like(t), t], axis=1))
    rows = np.concatenate(rows).astype(np.int64)
    okb, oqb = oracle.block_pool(x.k, x.q)
    oidx, _ = oracle.block_select(oqb, okb, topk)
    same = same_table_rows(rows, st.block_idx.cpu().numpy(), oidx, Hq // Hkv)
    assert same.mean() > 0.5
    ref = oracle.attn_rows(x.q, x.k, x.v, oidx, rows, want_full=False)
    b_, h_, t_ = rows[:, 0], rows[:, 1], rows[:, 2]
    go = ho.float().numpy()[b_, t_, h_]
    gl = hl.numpy()[b_, h_, t_]
    assert np.abs(go - ref["o_sparse"])[same].max() <= 2e-2
    assert np.abs(gl - ref["lse_sparse"])[same].max() <= 1e-3
