"""Pins the fp64 oracle to things other than itself.

Each test checks the oracle against a closed form, a brute-force enumeration,
an independent library routine (torch float64 SDPA / autograd), a finite
difference, or an invariant the method fixes.  Chosen so that a dropped term,
a wrong sign or index, or a transposed operand in the oracle fails one of them.
"""
import itertools

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import gen
import oracle

BS = 64


def _rand(shape, seed):
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(shape)


def _tiny(B=1, S=256, Hq=4, Hkv=2, D=8, seed=0):
    q = _rand((B, S, Hq, D), seed)
    k = _rand((B, S, Hkv, D), seed + 1)
    v = _rand((B, S, Hkv, D), seed + 2)
    return q, k, v


def _mask_from_idx(idx, b, h, S, complement=False):
    """Boolean [S, S] attention mask (True = attend) built from a block table."""
    n = S // BS
    blk = np.zeros((n, n), dtype=bool)
    for i in range(n):
        for j in idx[b, h, i]:
            if j >= 0:
                blk[i, j] = True
    tok = np.repeat(np.repeat(blk, BS, axis=0), BS, axis=1)
    causal = np.tril(np.ones((S, S), dtype=bool))
    return (causal & ~tok) if complement else (causal & tok)


def _sdpa_rows(q, k, v, mask_fn):
    """torch float64 SDPA per (b, hq) with an explicit boolean mask -> [B, Hq, S, D]."""
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    out = np.zeros((B, Hq, S, D))
    for b in range(B):
        for hq in range(Hq):
            h = hq // G
            m = torch.from_numpy(mask_fn(b, h))
            qt = torch.from_numpy(q[b, :, hq, :])[None]
            kt = torch.from_numpy(k[b, :, h, :])[None]
            vt = torch.from_numpy(v[b, :, h, :])[None]
            o = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=m[None])
            out[b, hq] = o[0].numpy()
    return out


def _as_bhsd(flat, B, Hq, S, D):
    return flat.reshape(B, Hq, S, D)


# ------------------------------------------------------------------ pooling

def test_pool_is_the_block_mean():
    x = gen.make_inputs("tiny_1k")
    kbar, qbar = oracle.block_pool(x.k, x.q)
    k = oracle.widen(x.k)
    q = oracle.widen(x.q)
    B, S, Hkv, D = k.shape
    G = q.shape[2] // Hkv
    n = S // BS
    ref_k = k.reshape(B, n, BS, Hkv, D).mean(axis=2).transpose(0, 2, 1, 3)
    ref_q = q.reshape(B, n, BS, Hkv, G, D).mean(axis=(2, 4)).transpose(0, 2, 1, 3)
    np.testing.assert_allclose(kbar, ref_k, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(qbar, ref_q, rtol=1e-13, atol=1e-15)


def test_group_pooled_score_equals_mean_of_per_head_scores():
    # linearity: (mean_g qbar_g) . kbar == mean_g (qbar_g . kbar)
    q, k, _ = _tiny(Hq=4, Hkv=1, D=8, seed=7)
    kbar, qbar = oracle.block_pool(k, q)
    per_head = [oracle.block_pool(k, q[:, :, g:g + 1, :])[1] for g in range(4)]
    s_group = np.einsum("bhid,bhjd->bhij", qbar, kbar)
    s_mean = np.mean([np.einsum("bhid,bhjd->bhij", p, kbar) for p in per_head], axis=0)
    np.testing.assert_allclose(s_group, s_mean, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- selection

@pytest.mark.parametrize("topk", [1, 2, 3, 4, 9])
def test_select_matches_brute_force_subsets(topk):
    n, D = 9, 5
    qbar = _rand((1, 2, n, D), 11)
    kbar = _rand((1, 2, n, D), 12)
    idx, gap = oracle.block_select(qbar, kbar, topk)
    for h in range(2):
        for i in range(n):
            m = min(topk - 1, i)
            best, best_sum = None, -np.inf
            for sub in itertools.combinations(range(i), m):
                s = sum(float(qbar[0, h, i] @ kbar[0, h, j]) for j in sub)
                if s > best_sum:
                    best, best_sum = sub, s
            want = sorted(set(best) | {i})
            got = [int(j) for j in idx[0, h, i] if j >= 0]
            assert got == want, (h, i, got, want)
            assert list(idx[0, h, i][len(want):]) == [-1] * (topk - len(want))
            if topk >= 2 and i > topk - 1:
                assert gap[0, h, i] >= 0.0
            else:
                assert np.isnan(gap[0, h, i])


def test_select_tie_goes_to_lower_block_index():
    D = 4
    kbar = np.zeros((1, 1, 5, D))
    kbar[0, 0, :, 0] = [1.0, 2.0, 2.0, 1.0, 0.0]   # blocks 1 and 2 tie, 0 and 3 tie
    qbar = np.zeros((1, 1, 5, D))
    qbar[0, 0, :, 0] = 1.0
    idx, _ = oracle.block_select(qbar, kbar, 3)
    assert list(idx[0, 0, 4]) == [1, 2, 4]
    idx, _ = oracle.block_select(qbar, kbar, 4)
    assert list(idx[0, 0, 4]) == [0, 1, 2, 4]


def test_select_nests_in_k_and_full_budget_takes_every_causal_block():
    x = gen.make_inputs("tiny_1k")
    kbar, qbar = oracle.block_pool(x.k, x.q)
    n = kbar.shape[2]
    prev = None
    for topk in range(1, n + 2):
        idx, _ = oracle.block_select(qbar, kbar, topk)
        sets = [[set(int(j) for j in idx[0, 0, i] if j >= 0) for i in range(n)]]
        for i in range(n):
            assert i in sets[0][i]
            assert len(sets[0][i]) == min(topk, i + 1)
            if prev is not None:
                assert prev[0][i] <= sets[0][i]
        prev = sets
    for i in range(n):
        assert prev[0][i] == set(range(i + 1))


def test_select_finds_exaggerated_plants():
    # wide head dim so that cross-talk between random directions (std ~ shift*sqrt(3/D))
    # stays far below the planted score (~ shift)
    x = gen.make_custom(1, 1024, 4, 2, 512, 4, seed=5, n_plant=3, plant_shift=10.0)
    kbar, qbar = oracle.block_pool(x.k, x.q)
    idx, _ = oracle.block_select(qbar, kbar, 4)
    n = 1024 // BS
    for h in range(2):
        for i in range(4, n):
            got = set(int(j) for j in idx[0, h, i] if j >= 0)
            assert got == set(x.plants[(0, h, i)]) | {i}


# ---------------------------------------------------------------- attention

def test_full_budget_equals_dense_causal_sdpa():
    q, k, v = _tiny(B=2, S=256, Hq=4, Hkv=2, D=16, seed=3)
    out = oracle.sparse_forward_problem(q, k, v, topk=4, want_full=True)
    B, S, Hq, D = q.shape
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)
    kt = torch.from_numpy(k).permute(0, 2, 1, 3).repeat_interleave(2, dim=1)
    vt = torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(2, dim=1)
    ref = F.scaled_dot_product_attention(qt, kt, vt, is_causal=True).numpy()
    np.testing.assert_allclose(_as_bhsd(out["o_sparse"], B, Hq, S, D), ref, atol=1e-12)
    np.testing.assert_allclose(_as_bhsd(out["o_full"], B, Hq, S, D), ref, atol=1e-12)
    assert np.all(out["delta"] == 0.0)
    np.testing.assert_allclose(out["lse_sparse"], out["lse_full"], atol=1e-12)


@pytest.mark.parametrize("topk", [1, 2, 3])
def test_sparse_output_equals_masked_sdpa(topk):
    q, k, v = _tiny(B=1, S=320, Hq=4, Hkv=2, D=16, seed=5)
    out = oracle.sparse_forward_problem(q, k, v, topk=topk, want_full=True)
    B, S, Hq, D = q.shape
    idx = out["idx"]
    ref = _sdpa_rows(q, k, v, lambda b, h: _mask_from_idx(idx, b, h, S))
    np.testing.assert_allclose(_as_bhsd(out["o_sparse"], B, Hq, S, D), ref, atol=1e-12)


def test_lse_matches_logsumexp():
    q, k, v = _tiny(B=1, S=192, Hq=2, Hkv=1, D=8, seed=9)
    out = oracle.sparse_forward_problem(q, k, v, topk=2, want_full=True)
    S = q.shape[1]
    scale = 1.0 / np.sqrt(8)
    idx = out["idx"]
    m = _mask_from_idx(idx, 0, 0, S)
    for r, (b, hq, t) in enumerate(out["rows"]):
        logits = scale * (k[b, :, 0, :] @ q[b, t, hq, :])
        full = torch.logsumexp(torch.from_numpy(logits[: t + 1]), 0).item()
        sp = torch.logsumexp(torch.from_numpy(logits[m[t]]), 0).item()
        assert abs(out["lse_full"][r] - full) < 1e-12
        assert abs(out["lse_sparse"][r] - sp) < 1e-12


def test_rows_are_probability_distributions_over_selected_causal_keys():
    # V = identity rows: O_t[s] is the attention weight P_ts itself.
    B, S, Hq, Hkv, D = 1, 128, 2, 1, 128
    q = _rand((B, S, Hq, D), 21) * 0.3
    k = _rand((B, S, Hkv, D), 22) * 0.3
    v = np.zeros((B, S, Hkv, D))
    v[0, np.arange(S), 0, np.arange(S)] = 1.0
    out = oracle.sparse_forward_problem(q, k, v, topk=1, want_full=True)
    P = out["o_sparse"].reshape(Hq, S, S)
    Pf = out["o_full"].reshape(Hq, S, S)
    scale = 1.0 / np.sqrt(D)
    for hq in range(Hq):
        for t in range(S):
            i = t // BS
            allowed = np.zeros(S, dtype=bool)
            allowed[i * BS:t + 1] = True          # topk=1: the diagonal block only
            assert np.all(P[hq, t][~allowed] == 0.0)
            assert abs(P[hq, t].sum() - 1.0) < 1e-12
            assert np.all(Pf[hq, t][t + 1:] == 0.0)
            assert abs(Pf[hq, t].sum() - 1.0) < 1e-12
            s0 = i * BS
            for s in range(s0 + 1, t + 1):
                want = np.exp(scale * (q[0, t, hq] @ (k[0, s, 0] - k[0, s0, 0])))
                assert abs(P[hq, t, s] / P[hq, t, s0] - want) < 1e-11 * max(1.0, want)


def test_value_ones_gives_ones():
    q, k, v = _tiny(B=1, S=256, Hq=4, Hkv=2, D=8, seed=31)
    v = np.ones_like(v)
    out = oracle.sparse_forward_problem(q, k, v, topk=2, want_full=True)
    np.testing.assert_allclose(out["o_sparse"], 1.0, atol=1e-12)
    np.testing.assert_allclose(out["o_full"], 1.0, atol=1e-12)


# -------------------------------------------------------------- dropped mass

def test_dropped_mass_properties_and_linear_error_identity():
    q, k, v = _tiny(B=1, S=384, Hq=4, Hkv=2, D=16, seed=41)
    B, S, Hq, D = q.shape
    n = S // BS
    prev = None
    for topk in range(1, n + 1):
        out = oracle.sparse_forward_problem(q, k, v, topk=topk, want_full=True)
        d = out["delta"]
        assert np.all(d >= 0.0) and np.all(d <= 1.0)
        np.testing.assert_allclose(d, out["delta_lse"], atol=1e-12)
        t = out["rows"][:, 2]
        assert np.all(d[t // BS < topk] == 0.0)
        if prev is not None:
            assert np.all(d <= prev + 1e-15)
        prev = d
        if topk < n:
            idx = out["idx"]
            o_unsel = _sdpa_rows(q, k, v, lambda b, h: _mask_from_idx(idx, b, h, S, True))
            o_unsel = o_unsel.reshape(-1, D)
            o_sp, o_f = out["o_sparse"], out["o_full"]
            has = d > 0
            lhs = o_f[has]
            rhs = (1 - d[has])[:, None] * o_sp[has] + d[has][:, None] * o_unsel[has]
            np.testing.assert_allclose(lhs, rhs, atol=1e-12)
            vmax = np.abs(v).max()
            assert np.all(np.abs(o_f - o_sp).max(axis=1) <= 2 * d * vmax + 1e-12)
    assert np.all(prev == 0.0)


# ----------------------------------------------------------------- backward

def _loss(q, k, v, do, idx):
    B, S, Hq, D = q.shape
    rows = oracle.all_rows(B, Hq, S)
    o = oracle.attn_rows(q, k, v, idx, rows, want_full=False)["o_sparse"]
    return float(np.sum(o.reshape(B, Hq, S, D).transpose(0, 2, 1, 3) * do))


def _full_bwd(q, k, v, do, idx):
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    n = S // BS
    rows = oracle.all_rows(B, Hq, S)
    dq = oracle.sparse_bwd_dq_rows(q, k, v, do, idx, rows).reshape(B, Hq, S, D).transpose(0, 2, 1, 3)
    blocks = oracle.all_rows(B, Hkv, n)
    dk, dv = oracle.sparse_bwd_dkv_blocks(q, k, v, do, idx, blocks)
    dk = dk.reshape(B, Hkv, n * BS, D).transpose(0, 2, 1, 3)
    dv = dv.reshape(B, Hkv, n * BS, D).transpose(0, 2, 1, 3)
    return dq, dk, dv


def test_backward_matches_central_finite_differences():
    q, k, v = _tiny(B=1, S=256, Hq=4, Hkv=2, D=8, seed=51)
    do = _rand(q.shape, 52)
    kbar, qbar = oracle.block_pool(k, q)
    idx, _ = oracle.block_select(qbar, kbar, 2)   # frozen selection
    grads = _full_bwd(q, k, v, do, idx)
    rng = np.random.Generator(np.random.PCG64(53))
    h = 1e-6
    for name, arr, g in zip("qkv", (q, k, v), grads):
        for _ in range(12):
            pos = tuple(int(rng.integers(0, s)) for s in arr.shape)
            plus, minus = arr.copy(), arr.copy()
            plus[pos] += h
            minus[pos] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = plus, minus
            fd = (_loss(args_p["q"], args_p["k"], args_p["v"], do, idx)
                  - _loss(args_m["q"], args_m["k"], args_m["v"], do, idx)) / (2 * h)
            assert abs(fd - g[pos]) <= 1e-6 * max(1.0, abs(g[pos])), (name, pos, fd, g[pos])


def test_backward_matches_torch_autograd_of_masked_sdpa():
    q, k, v = _tiny(B=1, S=256, Hq=4, Hkv=2, D=8, seed=61)
    do = _rand(q.shape, 62)
    kbar, qbar = oracle.block_pool(k, q)
    idx, _ = oracle.block_select(qbar, kbar, 2)
    dq, dk, dv = _full_bwd(q, k, v, do, idx)
    B, S, Hq, D = q.shape
    G = 2
    qt = torch.from_numpy(q).permute(0, 2, 1, 3).clone().requires_grad_(True)
    kt = torch.from_numpy(k).permute(0, 2, 1, 3).clone().requires_grad_(True)
    vt = torch.from_numpy(v).permute(0, 2, 1, 3).clone().requires_grad_(True)
    mask = torch.stack([torch.from_numpy(_mask_from_idx(idx, 0, hq // G, S)) for hq in range(Hq)])
    o = F.scaled_dot_product_attention(qt, kt.repeat_interleave(G, 1), vt.repeat_interleave(G, 1),
                                       attn_mask=mask[None])
    (o * torch.from_numpy(do).permute(0, 2, 1, 3)).sum().backward()
    np.testing.assert_allclose(dq, qt.grad.permute(0, 2, 1, 3).numpy(), atol=1e-11)
    np.testing.assert_allclose(dk, kt.grad.permute(0, 2, 1, 3).numpy(), atol=1e-11)
    np.testing.assert_allclose(dv, vt.grad.permute(0, 2, 1, 3).numpy(), atol=1e-11)


def test_unselected_block_gets_exactly_zero_gradient():
    q, k, v = _tiny(B=1, S=640, Hq=2, Hkv=1, D=8, seed=71)
    do = _rand(q.shape, 72)
    kbar, qbar = oracle.block_pool(k, q)
    idx, _ = oracle.block_select(qbar, kbar, 2)
    n = 640 // BS
    lonely = [j for j in range(n)
              if not any(j in idx[0, 0, i] for i in range(j + 1, n))]
    assert lonely, "test data should leave some block unselected by later blocks"
    for j in lonely:
        do_j = do.copy()
        do_j[0, j * BS:(j + 1) * BS] = 0.0
        dk, dv = oracle.sparse_bwd_dkv_blocks(q, k, v, do_j, idx, np.array([[0, 0, j]]))
        assert np.all(dk == 0.0) and np.all(dv == 0.0)


# ---------------------------------------------------- alignment objective

def _outputs(q, k, v, idx):
    """Sparse and full outputs [B, S, Hq, D] of every row (fp64)."""
    B, S, Hq, D = q.shape
    rows = oracle.all_rows(B, Hq, S)
    r = oracle.attn_rows(q, k, v, idx, rows, want_full=True)
    to = lambda a: a.reshape(B, Hq, S, D).transpose(0, 2, 1, 3)  # noqa: E731
    return to(r["o_sparse"]), to(r["o_full"])


@pytest.mark.parametrize("mode", [0, 1])
def test_alignment_gradient_matches_finite_differences_with_stop_gradient(mode):
    # J = <G, h_mode> + alpha (mean (h_full - C_s)^2 + mean (h_sparse - C_f)^2),
    # C_s, C_f frozen at the unperturbed outputs (the stop-gradients); the
    # analytic gradient is the oracle's output gradients pushed back through
    # the sparse stream (selected blocks) and the full stream (every causal block)
    q, k, v = _tiny(B=1, S=256, Hq=4, Hkv=2, D=8, seed=81)
    G_ = _rand(q.shape, 82)
    kbar, qbar = oracle.block_pool(k, q)
    idx, _ = oracle.block_select(qbar, kbar, 2)   # frozen selection
    B, S, Hq, D = q.shape
    dense = oracle.dense_causal_table(B, k.shape[2], S // BS)
    o_s0, o_f0 = _outputs(q, k, v, idx)
    alpha = 0.3 * q.size   # alignment terms of the same order as <G, h>
    d_s, d_f = oracle.alignment_output_grads(o_s0, o_f0, G_, mode, alpha)
    gs = _full_bwd(q, k, v, d_s, idx)
    gf = _full_bwd(q, k, v, d_f, dense)
    grads = [a + b for a, b in zip(gs, gf)]

    def J(q_, k_, v_):
        o_s, o_f = _outputs(q_, k_, v_, idx)
        lin = np.sum(G_ * (o_s if mode == 0 else o_f))
        return lin + alpha * (np.mean((o_f - o_s0) ** 2) + np.mean((o_s - o_f0) ** 2))

    rng = np.random.Generator(np.random.PCG64(83 + mode))
    h = 1e-6
    for name, arr, g in zip("qkv", (q, k, v), grads):
        for _ in range(8):
            pos = tuple(int(rng.integers(0, s)) for s in arr.shape)
            plus, minus = arr.copy(), arr.copy()
            plus[pos] += h
            minus[pos] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = plus, minus
            fd = (J(args_p["q"], args_p["k"], args_p["v"]) - J(args_m["q"], args_m["k"], args_m["v"])) / (2 * h)
            assert abs(fd - g[pos]) <= 2e-6 * max(1.0, abs(g[pos])), (name, pos, fd, g[pos])


def test_dense_table_gives_dense_causal_attention():
    q, k, v = _tiny(B=1, S=256, Hq=2, Hkv=1, D=8, seed=91)
    dense = oracle.dense_causal_table(1, 1, 4)
    o_s, o_f = _outputs(q, k, v, dense)
    np.testing.assert_allclose(o_s, o_f, atol=1e-13)
    ref = _sdpa_rows(q, k, v, lambda b, h: np.tril(np.ones((256, 256), dtype=bool)))
    np.testing.assert_allclose(o_s.transpose(0, 2, 1, 3), ref, atol=1e-12)


# ------------------------------------------------------------------ decode

def _decode_case(topk, seed, lengths, capacity=1024, Hq=4, Hkv=2, D=16):
    x = gen.make_decode(len(lengths), capacity, Hq, Hkv, D, topk, seed=seed, n_plant=3,
                        lengths=lengths)
    kbar, _ = oracle.block_pool(x.k)
    return x, kbar


def _row_sdpa(x, b, hq, keep):
    """torch float64 attention of one query row over the cache tokens in keep."""
    k64, v64, q64 = oracle.widen(x.k), oracle.widen(x.v), oracle.widen(x.q)
    G = q64.shape[1] // k64.shape[2]
    h = hq // G
    qt = torch.from_numpy(q64[b, hq])[None, None]
    kt = torch.from_numpy(k64[b, :, h])[None]
    vt = torch.from_numpy(v64[b, :, h])[None]
    m = torch.from_numpy(keep)[None, None]
    return F.scaled_dot_product_attention(qt, kt, vt, attn_mask=m)[0, 0].numpy()


def test_decode_full_budget_equals_dense_causal_row():
    lengths = [1, 64, 65, 700, 1024]
    x, kbar = _decode_case(topk=16, seed=101, lengths=lengths)
    idx, gap, o, lse = oracle.decode_step(x.q, x.k, x.v, kbar, x.lengths, 16)
    for b, L in enumerate(lengths):
        keep = np.arange(1024) < L
        for hq in range(4):
            np.testing.assert_allclose(o[b, hq], _row_sdpa(x, b, hq, keep), atol=1e-12)
        assert np.all(np.isnan(gap[b]))


def test_decode_selection_is_block_select_of_its_pooled_query():
    lengths = [1000, 777, 1024, 513]
    x, kbar = _decode_case(topk=4, seed=102, lengths=lengths)
    idx, gap, _, _ = oracle.decode_step(x.q, x.k, x.v, kbar, x.lengths, 4)
    q64 = oracle.widen(x.q)
    B, Hkv, n, D = kbar.shape
    G = q64.shape[1] // Hkv
    for b, L in enumerate(lengths):
        c = (L - 1) // 64
        qbar = np.zeros_like(kbar)
        for h in range(Hkv):
            qbar[b, h, c] = q64[b, h * G:(h + 1) * G].mean(axis=0)
        ref, rgap = oracle.block_select(qbar, kbar, 4)
        for h in range(Hkv):
            assert np.array_equal(idx[b, h], ref[b, h, c])
            assert gap[b, h] == pytest.approx(rgap[b, h, c], abs=1e-12)
        # brute force: the chosen earlier blocks maximise the summed score
        for h in range(Hkv):
            sc = kbar[b, h, :c] @ q64[b, h * G:(h + 1) * G].mean(axis=0)
            best = max(itertools.combinations(range(c), 3), key=lambda s_: sum(sc[j] for j in s_))
            assert sorted(best) == list(idx[b, h, :3])


def test_decode_attention_is_masked_softmax_over_the_kept_tokens():
    lengths = [1000, 641, 1024]
    x, kbar = _decode_case(topk=3, seed=103, lengths=lengths)
    idx, _, o, lse = oracle.decode_step(x.q, x.k, x.v, kbar, x.lengths, 3)
    k64, q64 = oracle.widen(x.k), oracle.widen(x.q)
    for b, L in enumerate(lengths):
        for hq in range(4):
            h = hq // 2
            keep = np.zeros(1024, dtype=bool)
            for j in idx[b, h]:
                if j >= 0:
                    keep[64 * j:64 * j + 64] = True
            keep &= np.arange(1024) < L
            np.testing.assert_allclose(o[b, hq], _row_sdpa(x, b, hq, keep), atol=1e-12)
            logits = (k64[b, keep, h] @ q64[b, hq]) / 4.0
            np.testing.assert_allclose(lse[b, hq], np.log(np.exp(logits - logits.max()).sum()) + logits.max(),
                                       atol=1e-12)


# -------------------------------------------------------------- early stop

def _early_case(seed):
    q, k, v = _tiny(B=1, S=512, Hq=4, Hkv=1, D=8, seed=seed)
    kbar, qbar = oracle.block_pool(k, q)
    idx, _ = oracle.block_select(qbar, kbar, 5)
    return q, k, v, qbar, kbar, idx


def test_early_stop_with_zero_threshold_is_the_sparse_forward():
    q, k, v, qbar, kbar, idx = _early_case(111)
    o, lse, vis, _ = oracle.early_stop_forward(q, k, v, qbar, kbar, idx, 0.0)
    B, S, Hq, D = q.shape
    r = oracle.attn_rows(q, k, v, idx, oracle.all_rows(B, Hq, S), want_full=False)
    np.testing.assert_allclose(o.transpose(0, 2, 1, 3).reshape(-1, D), r["o_sparse"], atol=1e-12)
    np.testing.assert_allclose(lse.reshape(-1), r["lse_sparse"], atol=1e-12)
    nsel = (idx >= 0).sum(axis=-1)                      # [B, Hkv, n]
    assert np.array_equal(vis, np.repeat(nsel, Hq // k.shape[2], axis=1))


def test_early_stop_with_huge_threshold_keeps_the_diagonal_and_the_best_block():
    q, k, v, qbar, kbar, idx = _early_case(112)
    o, _, vis, _ = oracle.early_stop_forward(q, k, v, qbar, kbar, idx, 1e30)
    B, S, Hq, D = q.shape
    n = S // BS
    keep = np.zeros((n, n), dtype=bool)
    for i in range(n):
        keep[i, i] = True
        earlier = [j for j in idx[0, 0, i] if 0 <= j < i]
        if earlier:
            keep[i, max(earlier, key=lambda j: (kbar[0, 0, j] @ qbar[0, 0, i], -j))] = True
        assert np.all(vis[0, :, i] == (2 if earlier else 1))
    mask = np.repeat(np.repeat(keep, BS, 0), BS, 1) & np.tril(np.ones((S, S), dtype=bool))
    ref = _sdpa_rows(q, k, v, lambda b, h: mask)
    np.testing.assert_allclose(o.transpose(0, 2, 1, 3), ref, atol=1e-12)


def test_early_stop_visits_fewer_blocks_as_the_threshold_grows():
    q, k, v, qbar, kbar, idx = _early_case(113)
    prev = None
    for tau in (0.0, 0.01, 0.05, 0.2, 1.0):
        _, _, vis, _ = oracle.early_stop_forward(q, k, v, qbar, kbar, idx, tau)
        if prev is not None:
            assert np.all(vis <= prev)
        prev = vis
    assert prev.sum() < (idx >= 0).sum() * q.shape[2]


@pytest.mark.parametrize("tau", [0.3, 0.8])
def test_early_stop_matches_a_recomputation_from_prefix_logsumexps(tau):
    """The stop point of each head's query segment from whole-prefix
    logsumexps (one torch.logsumexp over the union of the earlier blocks'
    keys, not a running sum) and the output from masked SDPA over the visited
    blocks.  Heads of one group share the visiting order but stop on their own
    rows only: some pair of heads of the same query block must stop apart."""
    q, k, v = _tiny(B=1, S=1024, Hq=4, Hkv=1, D=8, seed=114)
    kbar, qbar = oracle.block_pool(k, q)
    idx, _ = oracle.block_select(qbar, kbar, 8)
    o, lse, vis, _ = oracle.early_stop_forward(q, k, v, qbar, kbar, idx, tau)
    S, Hq, D = q.shape[1], q.shape[2], q.shape[3]
    n = S // BS
    causal = torch.tril(torch.ones(S, S, dtype=torch.bool))
    logits = [(torch.from_numpy(q[0, :, hq]) @ torch.from_numpy(k[0, :, 0]).T) / np.sqrt(D) for hq in range(Hq)]
    middle = apart = 0
    for i in range(n):
        sel = [int(j) for j in idx[0, 0, i] if 0 <= j < i]
        # descending pooled score, ties to the lower block (lexsort: last key first)
        sc = np.array([kbar[0, 0, j] @ qbar[0, 0, i] for j in sel])
        order = [i] + [sel[x] for x in np.lexsort((np.array(sel), -sc))] if sel else [i]
        rows = slice(BS * i, BS * i + BS)
        for hq in range(Hq):
            nv = len(order)
            for jj in range(1, len(order)):
                keys_b = torch.zeros(S, dtype=torch.bool)
                keys_b[BS * order[jj]:BS * order[jj] + BS] = True
                keys_p = torch.zeros(S, dtype=torch.bool)
                for j in order[:jj]:
                    keys_p[BS * j:BS * j + BS] = True
                ratio = float((torch.logsumexp(logits[hq][rows].masked_fill(~(keys_b & causal[rows]), -np.inf), 1)
                               - torch.logsumexp(logits[hq][rows].masked_fill(~(keys_p & causal[rows]), -np.inf), 1)
                               ).max())
                if ratio < np.log(tau):
                    nv = jj + 1
                    break
            assert vis[0, hq, i] == nv
            middle += 1 < nv < len(order)
            keep = torch.zeros(S, dtype=torch.bool)
            for j in order[:nv]:
                keep[BS * j:BS * j + BS] = True
            m = (keep & causal[rows])[None]
            ref = F.scaled_dot_product_attention(torch.from_numpy(q[0, rows, hq])[None],
                                                 torch.from_numpy(k[0, :, 0])[None],
                                                 torch.from_numpy(v[0, :, 0])[None], attn_mask=m)
            np.testing.assert_allclose(o[0, rows, hq], ref[0].numpy(), atol=1e-12)
            np.testing.assert_allclose(lse[0, hq, rows],
                                       torch.logsumexp(logits[hq][rows].masked_fill(~m[0], -np.inf), 1).numpy(),
                                       atol=1e-12)
        apart += len(set(int(x) for x in vis[0, :, i])) > 1
    assert middle > 0  # some segment stops strictly between its second and last block
    assert apart > 0   # the heads of a group do not stop together


# ------------------------------------------------------------ DashAttention

def _sparsemax_by_sorting(z):
    """Sparsemax (alpha = 2) by the sort-based closed form: the support is the
    largest k with 1 + k z_(k) > z_(1) + ... + z_(k), tau = (that sum - 1) / k."""
    zs = np.sort(z)[::-1]
    cs = np.cumsum(zs)
    k = max(kk for kk in range(1, len(z) + 1) if 1 + kk * zs[kk - 1] > cs[kk - 1])
    tau = (cs[k - 1] - 1) / k
    return np.maximum(z - tau, 0)


def _entmax15_by_quadratic(z):
    """1.5-entmax exactly: with x = z / 2 and support of size k, sum (x_j - tau)^2
    = 1 is a quadratic in tau, tau_k = mean_k - sqrt((1 - ss_k + k mean_k^2) / k);
    the support is the largest k with tau_k <= x_(k)."""
    xs = np.sort(z / 2)[::-1]
    best = None
    for kk in range(1, len(z) + 1):
        mean = xs[:kk].mean()
        ss = (xs[:kk] ** 2).sum()
        delta = (1 - ss + kk * mean ** 2) / kk
        if delta < 0:
            continue
        tau = mean - np.sqrt(delta)
        if tau <= xs[kk - 1]:
            best = tau
    return np.maximum(z / 2 - best, 0) ** 2


def test_entmax_two_is_sparsemax_and_one_point_five_is_the_exact_quadratic():
    rng = np.random.default_rng(120)
    for _ in range(40):
        z = rng.normal(0, rng.uniform(0.3, 4.0), size=rng.integers(2, 40))
        np.testing.assert_allclose(oracle.entmax(z, 2.0)[0], _sparsemax_by_sorting(z), atol=1e-12)
        np.testing.assert_allclose(oracle.entmax(z, 1.5)[0], _entmax15_by_quadratic(z), atol=1e-12)


@pytest.mark.parametrize("alpha", [1.25, 1.5, 1.75, 2.0, 3.0])
def test_entmax_satisfies_its_optimality_conditions(alpha):
    # on the support p_j^(alpha-1) - (alpha-1) z_j is one constant (-tau); off
    # it (alpha-1) z_j <= tau; the p sum to 1; shifting z changes nothing
    rng = np.random.default_rng(121)
    z = rng.normal(0, 2.0, size=(30, 25))
    p, tau = oracle.entmax(z, alpha)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-12)
    x = (alpha - 1) * z
    for r in range(30):
        s = p[r] > 0
        np.testing.assert_allclose(p[r, s] ** (alpha - 1) - x[r, s], -tau[r], atol=1e-9)
        assert np.all(x[r, ~s] <= tau[r] + 1e-9)
    np.testing.assert_allclose(oracle.entmax(z + 3.7, alpha)[0], p, atol=1e-10)


def test_entmax_tends_to_softmax_as_alpha_tends_to_one():
    z = np.random.default_rng(122).normal(0, 1.0, size=(5, 12))
    sm = np.exp(z) / np.exp(z).sum(axis=1, keepdims=True)
    np.testing.assert_allclose(oracle.entmax(z, 1.0005)[0], sm, atol=2e-3)


def _dash_case(seed, S=512, Hq=4, Hkv=2, D=16):
    q, k, v = _tiny(B=1, S=S, Hq=Hq, Hkv=Hkv, D=D, seed=seed)
    kbar, _ = oracle.block_pool(k, q)
    return q, k, v, kbar


def _bit(mask, b, h, i, j):
    return (int(mask[b, h, i, j // 32]) >> (j % 32)) & 1


def test_dash_route_extremes_of_gamma():
    q, k, v, kbar = _dash_case(123)
    B, S, Hq, D = q.shape
    Hkv, n, G = kbar.shape[1], S // BS, Hq // kbar.shape[1]
    # gamma -> 0: every head is uniform over the earlier chunks
    w, mask, _ = oracle.dash_route(q, kbar, 1.5, 1e-9)
    for h in range(Hkv):
        for i in range(n):
            np.testing.assert_allclose(w[0, h, i, :i], 1.0 / max(i, 1), atol=1e-9)
            assert all(_bit(mask, 0, h, i, j) == (j <= i) for j in range(n))
    # gamma -> inf: every head keeps only its best chunk; the group mean counts heads
    w, mask, _ = oracle.dash_route(q, kbar, 1.5, 1e6)
    for h in range(Hkv):
        for i in range(1, n):
            want = np.zeros(n)
            for g in range(G):
                qm = np.array([[float(x) for x in q[0, BS * i + t, h * G + g]] for t in range(BS)]).mean(axis=0)
                want[int(np.argmax([qm @ kbar[0, h, j] for j in range(i)]))] += 1.0 / G
            np.testing.assert_allclose(w[0, h, i], want, atol=1e-9)
            assert all(_bit(mask, 0, h, i, j) == (want[j] > 0 or j == i) for j in range(n))


def _dash_routing_with_oddities(n, Hkv, seed):
    """Random support with set bits at w = 0, bits at and after the diagonal,
    and cleared diagonal bits."""
    rng = np.random.default_rng(seed)
    W = (n + 31) // 32
    w = rng.uniform(0.01, 1.0, size=(1, Hkv, n, n)) * (rng.random((1, Hkv, n, n)) < 0.7)
    mask = np.zeros((1, Hkv, n, W), dtype=np.uint32)
    for h in range(Hkv):
        for i in range(n):
            for j in range(n):
                if rng.random() < 0.5:
                    mask[0, h, i, j // 32] |= np.uint32(1 << (j % 32))
    return w, mask


def test_dash_attention_with_sigma_zero_is_masked_attention_over_the_active_chunks():
    q, k, v, _ = _dash_case(124)
    B, S, Hq, D = q.shape
    Hkv, n, G = k.shape[2], S // BS, Hq // k.shape[2]
    w, mask = _dash_routing_with_oddities(n, Hkv, 125)
    o, lse = oracle.dash_attention(q, k, v, mask, w, 0.0)
    q64, k64 = q.astype(np.float64), k.astype(np.float64)

    def keep(b, h):
        m = np.zeros((S, S), dtype=bool)
        for i in range(n):
            cols = np.zeros(S, dtype=bool)
            for j in range(i):
                if _bit(mask, b, h, i, j) and w[b, h, i, j] > 0:
                    cols[BS * j:BS * j + BS] = True
            cols[BS * i:BS * i + BS] = True
            m[BS * i:BS * i + BS] = cols[None, :]
        return m & np.tril(np.ones((S, S), dtype=bool))

    ref = _sdpa_rows(q, k, v, keep)
    np.testing.assert_allclose(o.transpose(0, 2, 1, 3), ref, atol=1e-12)
    for hq in range(Hq):
        m = torch.from_numpy(keep(0, hq // G))
        lg = torch.from_numpy(q64[0, :, hq] @ k64[0, :, hq // G].T) / np.sqrt(D)
        np.testing.assert_allclose(lse[0, hq], torch.logsumexp(lg.masked_fill(~m, -np.inf), 1).numpy(),
                                   atol=1e-12)


def test_dash_attention_maximises_score_minus_kl_to_the_prior():
    # one-hot values read the attention rows out; each row must maximise
    # F(p) = z.p - KL(p || g) over the simplex on g's support, with g uniform
    # inside a chunk and proportional to w^sigma across chunks
    S, D, sigma = 256, 256, 0.7
    rng = np.random.default_rng(126)
    q = rng.normal(0, 1, (1, S, 1, D)).astype(np.float32)
    k = rng.normal(0, 1, (1, S, 1, D)).astype(np.float32)
    v = np.eye(S, dtype=np.float32)[None, :, None, :]
    n = S // BS
    w, mask = _dash_routing_with_oddities(n, 1, 127)
    o, _ = oracle.dash_attention(q, k, v, mask, w, sigma)
    q64, k64 = q.astype(np.float64), k.astype(np.float64)
    for t in (0, 70, 130, 200, 255):
        i = t // BS
        g = np.zeros(S)
        for j in range(i):
            if _bit(mask, 0, 0, i, j) and w[0, 0, i, j] > 0:
                g[BS * j:BS * j + BS] = w[0, 0, i, j] ** sigma
        g[BS * i:t + 1] = 1.0
        g /= g.sum()
        sup = g > 0
        z = (q64[0, t, 0] @ k64[0, :, 0].T) / np.sqrt(D)
        p = o[0, t, 0]
        assert np.all(p[~sup] == 0) and abs(p.sum() - 1) < 1e-12

        def F(pp):
            return float(z[sup] @ pp[sup] - (pp[sup] * np.log(pp[sup] / g[sup])).sum())
        best = F(p)
        for _ in range(20):
            d = np.zeros(S)
            d[sup] = rng.normal(0, 1, sup.sum())
            d[sup] -= d[sup].mean()
            eps = 0.2 * p[sup].min() / (np.abs(d).max() + 1e-30)
            assert F(p + eps * d) <= best + 1e-12


def test_receptive_field_is_the_guides_figure():
    # The guide's receptive fields (tests/golden/receptive_field.json) at
    # 64-token blocks: k = rf / 64 kept blocks, the diagonal among them.  With
    # one-hot values the sparse output row is the attention row, so its
    # nonzero entries are the keys the query sees: every earlier kept block in
    # full plus the diagonal block up to the query.  A query block with at
    # least k earlier blocks then sees 64 (k - 1) + (t mod 64) + 1 keys, and
    # its last row exactly the receptive field.
    import json
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "receptive_field.json")) as f:
        fx = json.load(f)
    assert fx["block_size"] == BS
    for rf in fx["receptive_fields"]:
        topk = rf // BS
        S = BS * (topk + 1)              # the last block has k earlier blocks to choose from
        q, k, _ = _tiny(1, S, 1, 1, S, seed=rf)
        v = np.eye(S)[None, :, None, :]
        kbar, qbar = oracle.block_pool(k, q)
        idx, _ = oracle.block_select(qbar, kbar, topk)
        n = S // BS
        rows = np.array([[0, 0, t] for t in range(BS * (n - 2), S)], dtype=np.int64)
        p = oracle.attn_rows(q, k, v, idx, rows, want_full=False)["o_sparse"]
        seen = (p > 0).sum(axis=1)
        t = rows[:, 2]
        assert np.array_equal(seen, BS * (topk - 1) + t % BS + 1)
        assert seen.max() == rf
        np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-12)
        # the last block drops exactly one earlier block: the one it did not select
        last = p[-BS:]
        dropped = [j for j in range(n - 1) if j not in idx[0, 0, n - 1]]
        assert len(dropped) == 1
        j = dropped[0]
        assert np.all(last[:, BS * j:BS * j + BS] == 0)
