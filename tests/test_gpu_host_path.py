"""GPU check of ssa_sparse_attn_fwd_host, the pipelined host-buffer forward:
its outputs must equal the device-buffer calls (ssa_block_pool,
ssa_block_select, ssa_sparse_attn_fwd) bit for bit, since it runs the same
kernels over chunks of consecutive query blocks (the last chunk may be
shorter)."""
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


@pytest.mark.parametrize("case", [(1, 2048, 8, 2, 64, 6), (2, 1280, 4, 2, 128, 5), (3, 1024, 16, 1, 64, 4),
                                  (1, 8192, 32, 4, 64, 16), (1, 4480, 32, 4, 64, 16), (1, 4096, 16, 2, 128, 8)],
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
