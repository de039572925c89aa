"""The allocation-free backward entry point, for callers that cannot allocate
device memory (they are handed only their input and output buffers, or may
not call an allocator while they serve).  ssa_sparse_attn_bwd_noalloc must
give the results of ssa_sparse_attn_bwd with a caller workspace bit for bit
(the backward is deterministic: no floating-point atomics, fixed reduction
order), on two calls in a row that share the library's fixed scratch.  This file is collected last
so that a run stopping at the first failure has run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_attention_21_b200 as ssa
import gen

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from block_sparse_attention_21_b200 import build
    build.build()
    ssa.lib()


@pytest.mark.parametrize("shape", [(2, 512, 8, 2, 64, 3), (1, 1024, 8, 1, 128, 4)],
                         ids=lambda s: "x".join(map(str, s)))
def test_noalloc_backward_matches_workspace_backward_twice(shape):
    B, S, Hq, Hkv, D, topk = shape
    x = gen.make_custom(B, S, Hq, Hkv, D, topk, seed=900 + S + D, n_plant=2, with_do=True)
    p = ssa.problem(B, S, Hq, Hkv, D, topk)
    q, k, v, do = (t.to(DEV) for t in (x.q, x.k, x.v, x.do))
    st = ssa.SparseStream(p)
    st.forward(q, k, v)
    ref = st.backward(q, k, v, do)
    ref = [t.clone() for t in ref]
    for _ in range(2):
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ssa.ssa_sparse_attn_bwd_noalloc(p, q, k, v, st.o, st.lse, do, st.block_idx, dq, dk, dv)
        torch.cuda.synchronize()
        assert ssa.ssa_get_device_error() == 0
        for got, want in zip((dq, dk, dv), ref):
            assert torch.equal(got, want)


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 4 x 32 x 262144 rows of D_t alone need 128 MiB > the 16 MiB scratch;
    # the size check comes before any launch (the pointers are never used)
    p = ssa.problem(4, 262144, 32, 4, 64, 16)
    assert ssa.ssa_sparse_attn_bwd_workspace(p) > (16 << 20)
    fake = 0x10000
    rc = ssa.lib().ssa_sparse_attn_bwd_noalloc(ctypes.byref(p), *([fake] * 10), None)
    assert rc == 5  # SSA_ERR_WORKSPACE
