"""GPU parity of the early-stop sparse forward (ssa_sparse_attn_fwd_early_stop)
against the fp64 oracle.  The unit that stops is one head's query segment
(query head, query block).  Its stop decision compares a mass ratio with tau,
and its visiting order compares pooled scores; segments where either is
within rounding of flipping (stop margin under 0.05 in log ratio, or two of
the scores it reaches closer than 1e-3) are left out of the exact comparison.
Elsewhere: the blocks visited per segment are equal, outputs max-abs <= 2e-2,
LSE <= 1e-3; and tau = 0 reproduces ssa_sparse_attn_fwd.  The kernel packs two
heads into one 128-row tile, so the cases must include tiles whose two heads
stop at different blocks.  A large top-k with a high tau makes every tile of a
CTA stop while the loader is still several blocks ahead, which must end
without a timed-out wait."""
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


CASES = [
    # (B, S, Hq, Hkv, D, topk, n_plant)
    (1, 1024, 8, 2, 64, 6, 4),
    (1, 768, 4, 2, 128, 5, 3),
    (1, 2048, 16, 2, 64, 8, 6),
    (1, 1536, 8, 2, 128, 6, 4),     # two M-tiles per CTA at head_dim 128
]


@pytest.mark.parametrize("tau", [0.0, 0.02, 0.2])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
def test_early_stop_matches_oracle(case, tau):
    _check(case, tau)


@pytest.mark.parametrize("tau", [0.3, 1.0])
@pytest.mark.parametrize("case", [(1, 4096, 8, 2, 64, 40, 8), (1, 4096, 4, 2, 128, 40, 8),
                                  (1, 4096, 8, 2, 128, 40, 8)],
                         ids=lambda c: "x".join(map(str, c)))
def test_early_stop_well_before_the_last_block(case, tau):
    vis, nsel, apart = _check(case, tau, min_clear=0.5)
    # most segments stop with more than a pipeline's depth of blocks left
    assert np.mean(nsel - vis >= 8) > 0.5
    # and in some tile the two heads stop at different blocks
    assert apart > 0


def _check(case, tau, min_clear=0.6):
    B, S, Hq, Hkv, D, topk, npl = case
    x = gen.make_custom(B, S, Hq, Hkv, D, topk, seed=800 + S + D, n_plant=npl)
    p = ssa.problem(B, S, Hq, Hkv, D, topk)
    q, k, v = (t.to(DEV) for t in (x.q, x.k, x.v))
    st = ssa.SparseStream(p)
    st.forward(q, k, v)
    n, G = S // 64, Hq // Hkv
    o = torch.empty_like(st.o)
    lse = torch.empty_like(st.lse)
    vis = torch.empty(B, Hq, n, dtype=torch.int32, device=DEV)
    ssa.ssa_sparse_attn_fwd_early_stop(p, q, k, v, st.q_pooled, st.k_pooled, st.block_idx, tau, o, lse, vis)
    torch.cuda.synchronize()
    assert ssa.ssa_get_device_error() == 0
    gidx = oracle_table(x, topk, st.block_idx)
    okb, oqb = oracle.block_pool(x.k, x.q)
    ro, rlse, rvis, margin = oracle.early_stop_forward(x.q, x.k, x.v, oqb, okb, gidx, tau)
    gvis = vis.cpu().numpy()                                   # [B, Hq, n]
    nsel = np.repeat((gidx >= 0).sum(axis=-1), G, axis=1)      # [B, Hq, n]
    assert np.all(gvis >= 1) and np.all(gvis <= nsel)
    # segments whose order or stop decision could flip between fp32 and fp64
    clear = margin > 0.05
    for b in range(B):
        for hq in range(Hq):
            h = hq // G
            for i in range(n):
                sel = [j for j in gidx[b, h, i] if 0 <= j < i]
                # only the order of the blocks a segment reaches (and of the
                # next one) can change its result
                sc = np.sort([okb[b, h, j] @ oqb[b, h, i] for j in sel])[::-1][: rvis[b, hq, i] + 1]
                if len(sc) > 1 and np.min(np.abs(np.diff(sc))) < 1e-3:
                    clear[b, hq, i] = False
    assert clear.mean() > min_clear
    assert np.array_equal(gvis[clear], rvis[clear])
    go, gl = o.float().cpu().numpy(), lse.cpu().numpy()
    for b, hq, i in zip(*np.nonzero(clear)):
        rows = slice(64 * i, 64 * i + 64)
        assert np.abs(go[b, rows, hq] - ro[b, rows, hq]).max() <= 2e-2
        assert np.abs(gl[b, hq, rows] - rlse[b, hq, rows]).max() <= 1e-3
    # tiles (head pairs 2p, 2p + 1 of one query block) whose heads stop apart
    pair = clear[:, 0::2] & clear[:, 1::2]
    apart = int(np.sum(pair & (gvis[:, 0::2] != gvis[:, 1::2])))
    if tau == 0.0:
        assert np.array_equal(gvis, nsel)
        assert (o.float() - st.o.float()).abs().max().item() <= 2e-2
    return gvis, nsel, apart
