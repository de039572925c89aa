"""GPU parity of DashAttention's routing (ssa_dash_route) and prior-induced
sparse softmax (ssa_dash_attn_fwd) against the fp64 oracle, through the C ABI.

Routing: the group weights within 2e-4 everywhere; the support bits
bit-exact wherever every head's decision is clear of its threshold by more
than 1e-4 (the GPU finds the threshold in fp32, the oracle in fp64), the
diagonal bit always set and no bit after it.  Attention: outputs max-abs
<= 2e-2, LSE <= 1e-3, every row on small problems (synthetic routings with
set bits at zero weight, bits past the diagonal and cleared diagonal bits),
sampled query blocks at 8k and at the longest supported sequence; end to end
(route then attention) on the rows whose support row is the same on both
sides."""
import numpy as np
import pytest
import torch

import block_sparse_attention_21_b200 as ssa
import gen
import oracle
from conftest import workload_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"
W_TOL, MARGIN, O_TOL, LSE_TOL = 2e-4, 1e-4, 2e-2, 1e-3


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from block_sparse_attention_21_b200 import build
    build.build()
    ssa.lib()


def _gpu_route(p, q, k, alpha, gamma):
    B, S, Hkv, D = p.batch, p.seq_len, p.n_kv_heads, p.head_dim
    n = S // 64
    kb = torch.empty(B, Hkv, n, D, dtype=torch.float32, device=DEV)
    ssa.ssa_block_pool(p, k, None, kb, None)
    w = torch.full((B, Hkv, n, n), float("nan"), dtype=torch.float32, device=DEV)
    mask = torch.full((B, Hkv, n, (n + 31) // 32), -1, dtype=torch.int32, device=DEV)
    ssa.ssa_dash_route(p, q, kb, alpha, gamma, w, mask)
    torch.cuda.synchronize()
    assert ssa.ssa_get_device_error() == 0
    return w.cpu().numpy(), mask.cpu().numpy().view(np.uint32)


def _gpu_attn(p, q, k, v, w, mask, sigma):
    o = torch.full(tuple(q.shape), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((p.batch, p.n_q_heads, p.seq_len), float("nan"), dtype=torch.float32, device=DEV)
    ssa.ssa_dash_attn_fwd(p, q, k, v, w, mask, sigma, o, lse)
    torch.cuda.synchronize()
    assert ssa.ssa_get_device_error() == 0
    return o.float().cpu().numpy(), lse.cpu().numpy()


def _check_route(x, p, alpha, gamma):
    q, k = x.q.to(DEV), x.k.to(DEV)
    gw, gmask = _gpu_route(p, q, k, alpha, gamma)
    okb, _ = oracle.block_pool(x.k, x.q)
    ow, omask, margin = oracle.dash_route(x.q, okb, alpha, gamma)
    assert np.abs(gw - ow).max() <= W_TOL
    n = p.seq_len // 64
    gbits = np.unpackbits(gmask.view(np.uint8), axis=-1, bitorder="little")[..., :n].astype(bool)
    obits = np.unpackbits(omask.view(np.uint8), axis=-1, bitorder="little")[..., :n].astype(bool)
    clear = margin > MARGIN            # inf on and after the diagonal
    assert clear.mean() > 0.9
    assert np.array_equal(gbits[clear], obits[clear])
    i = np.arange(n)
    assert np.all(gbits[..., i, i])
    assert not np.any(gbits & (i[None, :] > i[:, None]))
    # every query block routes to something once it has an earlier chunk
    assert np.all(gbits[..., 1:, :].sum(axis=-1) >= 2)
    return gw, gmask, ow, omask


ROUTE_CASES = [
    # (B, S, Hq, Hkv, D, n_plant)
    (1, 2048, 8, 2, 64, 4),
    (2, 1280, 4, 2, 128, 3),
    (1, 4096, 32, 2, 128, 6),     # 16 query heads per KV head
    (1, 1024, 2, 1, 64, 0),
]


@pytest.mark.parametrize("alpha,gamma", [(1.5, 8.0), (2.0, 4.0), (1.25, 16.0), (1.5, 0.5)])
@pytest.mark.parametrize("case", ROUTE_CASES, ids=lambda c: "x".join(map(str, c)))
def test_route_matches_oracle(case, alpha, gamma):
    B, S, Hq, Hkv, D, npl = case
    x = gen.make_custom(B, S, Hq, Hkv, D, 4, seed=1300 + S + D, n_plant=npl)
    _check_route(x, ssa.problem(B, S, Hq, Hkv, D, 4), alpha, gamma)


ATTN_CASES = [
    # (B, S, Hq, Hkv, D)
    (1, 1024, 8, 2, 64),
    (2, 704, 4, 2, 64),       # 11 blocks: a ragged mask word
    (1, 2112, 2, 1, 64),      # one query-head pair per KV head, 33 blocks
    (1, 1024, 8, 2, 128),
    (1, 1344, 4, 1, 128),
]


@pytest.mark.parametrize("sigma", [0.0, 0.5, 1.0])
@pytest.mark.parametrize("case", ATTN_CASES, ids=lambda c: "x".join(map(str, c)))
def test_attention_on_synthetic_routing_every_row(case, sigma):
    B, S, Hq, Hkv, D = case
    n = S // 64
    x = gen.make_custom(B, S, Hq, Hkv, D, 4, seed=1400 + S + D, n_plant=2)
    r = gen.make_dash_routing(B, Hkv, n, seed=1500 + S, density=0.4)
    p = ssa.problem(B, S, Hq, Hkv, D, 4)
    q, k, v = x.q.to(DEV), x.k.to(DEV), x.v.to(DEV)
    w = torch.from_numpy(r.weights).to(DEV)
    mask = torch.from_numpy(r.mask.view(np.int32)).to(DEV)
    go, gl = _gpu_attn(p, q, k, v, w, mask, sigma)
    ro, rl = oracle.dash_attention(x.q, x.k, x.v, r.mask, r.weights, sigma)
    assert np.abs(go - ro).max() <= O_TOL
    assert np.abs(gl - rl).max() <= LSE_TOL


def _end_to_end(x, p, alpha, gamma, sigma, blocks=None):
    q, k, v = x.q.to(DEV), x.k.to(DEV), x.v.to(DEV)
    gw, gmask, ow, omask = _check_route(x, p, alpha, gamma)
    go, gl = _gpu_attn(p, q, k, v, torch.from_numpy(gw).to(DEV), torch.from_numpy(gmask.view(np.int32)).to(DEV),
                       sigma)
    B, Hkv, n = gmask.shape[0], gmask.shape[1], gmask.shape[2]
    same = np.all(gmask == omask, axis=-1)        # [B, Hkv, n]
    if blocks is None:
        blocks = [(b, h, i) for b in range(B) for h in range(Hkv) for i in range(n)]
    blocks = [t for t in blocks if same[t]]
    assert len(blocks) > 0
    ro, rl = oracle.dash_attention(x.q, x.k, x.v, omask, ow, sigma, blocks=blocks)
    G = p.n_q_heads // Hkv
    for b, h, i in blocks:
        rows, heads = slice(64 * i, 64 * i + 64), slice(h * G, h * G + G)
        assert np.abs(go[b, rows, heads] - ro[b, rows, heads]).max() <= O_TOL
        assert np.abs(gl[b, heads, rows] - rl[b, heads, rows]).max() <= LSE_TOL
    return gmask


@pytest.mark.parametrize("case", [(1, 2048, 8, 2, 64, 4), (1, 1536, 8, 2, 128, 4)],
                         ids=lambda c: "x".join(map(str, c)))
def test_route_then_attention_every_row(case):
    B, S, Hq, Hkv, D, npl = case
    x = gen.make_custom(B, S, Hq, Hkv, D, 4, seed=1600 + S + D, n_plant=npl)
    _end_to_end(x, ssa.problem(B, S, Hq, Hkv, D, 4), 1.5, 8.0, 1.0)


def test_llama_8k_sampled_blocks():
    x = workload_inputs("llama1b_8k")
    w = x.workload
    p = ssa.problem(w.batch, w.seq_len, w.n_q_heads, w.n_kv_heads, w.head_dim, w.top_k)
    blocks = [(0, h, i) for h in range(w.n_kv_heads) for i in (0, 1, 2, 31, 64, 100, 126, 127)]
    gmask = _end_to_end(x, p, 1.5, 8.0, 1.0, blocks)
    # the routing is adaptive: supports differ between query blocks
    counts = np.unpackbits(gmask.view(np.uint8), axis=-1).sum(axis=-1)
    assert counts[..., 16:].min() < counts[..., 16:].max()


def test_longest_supported_sequence_sampled_blocks():
    # 1024 chunks: a full 32-word mask row and the largest routed list
    B, S, Hq, Hkv, D = 1, 65536, 2, 1, 64
    x = gen.make_custom(B, S, Hq, Hkv, D, 4, seed=1700, n_plant=4)
    p = ssa.problem(B, S, Hq, Hkv, D, 4)
    _end_to_end(x, p, 1.5, 2.0, 1.0, [(0, 0, i) for i in (0, 1, 500, 1022, 1023)])


def test_route_class_matches_the_entry_points():
    x = gen.make_custom(1, 1024, 8, 2, 64, 4, seed=1800, n_plant=2)
    p = ssa.problem(1, 1024, 8, 2, 64, 4)
    q, k, v = x.q.to(DEV), x.k.to(DEV), x.v.to(DEV)
    da = ssa.DashAttention(p, alpha=1.5, gamma=8.0, sigma=1.0)
    o, lse = da.forward(q, k, v)
    torch.cuda.synchronize()
    gw, gmask = _gpu_route(p, q, k, 1.5, 8.0)
    go, gl = _gpu_attn(p, q, k, v, torch.from_numpy(gw).to(DEV), torch.from_numpy(gmask.view(np.int32)).to(DEV), 1.0)
    assert np.array_equal(o.float().cpu().numpy(), go) and np.array_equal(lse.cpu().numpy(), gl)
