"""fp64 CPU oracle for the SSA sparse stream -- TEST INFRASTRUCTURE.

Only the tests, the smoke check and the bench's CPU-baseline leg may import
this package.  It shares no code with the CUDA library: the attention
arithmetic lives in ssa_oracle.c (plain C, fp64, pthreads); this module widens
bf16 tensors exactly to fp64, marshals numpy arrays through ctypes, and holds
the alignment objective's elementwise output gradients (fp64 numpy).

Functions (each cites the passage it follows in ssa_oracle.c):
  block_pool      mean of each 64-token key block; GQA-group mean of the queries
  block_select    diagonal + top-(k-1) earlier blocks by pooled score
  attn_rows       sparse output/LSE and, on request, full causal output/LSE and
                  dropped mass (two routes) for a list of query rows
  sparse_bwd_dq_rows / sparse_bwd_dkv_blocks
                  gradient of the sparse output, by the explicit formulas
  dense_causal_table
                  the index table of every causal block (dense attention)
  alignment_output_grads
                  output gradients of the alignment objective (a formula,
                  written here; pinned by finite differences with stop-gradient)
  decode_step     one decoding step: selection for the newest token and its
                  attention (fp64 numpy, small problems)
  early_stop_forward
                  the sparse forward with the early-stop rule, each query
                  segment of one head stopping on its own (fp64 numpy, small
                  problems)
  entmax          alpha-entmax of a vector by its threshold (fp64 bisection)
  dash_route      DashAttention chunk routing: per-head alpha-entmax over the
                  pooled chunk logits, averaged over the GQA group, and the
                  bit-packed support
  dash_attention  DashAttention's prior-induced sparse softmax over the
                  active chunks (fp64 numpy, small problems)
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

import numpy as np

from . import build as _build

BLOCK = 64

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int32)
        lp = ctypes.POINTER(ctypes.c_int64)
        c_int, c_dbl, c_i64 = ctypes.c_int, ctypes.c_double, ctypes.c_int64
        lib.ora_block_pool.argtypes = [c_int] * 6 + [dp, dp, dp, dp, c_int]
        lib.ora_block_select.argtypes = [c_int] * 5 + [dp, dp, ip, dp, c_int]
        lib.ora_attn_rows.argtypes = ([c_int] * 7 + [c_dbl, dp, dp, dp, ip, c_i64, lp, c_int]
                                      + [dp] * 6 + [c_int])
        lib.ora_sparse_bwd_dq_rows.argtypes = ([c_int] * 7 + [c_dbl, dp, dp, dp, dp, ip, c_i64,
                                                              lp, dp, c_int])
        lib.ora_sparse_bwd_dkv_blocks.argtypes = ([c_int] * 7 + [c_dbl, dp, dp, dp, dp, ip,
                                                                 c_i64, lp, dp, dp, c_int])
        for f in (lib.ora_block_pool, lib.ora_block_select, lib.ora_attn_rows,
                  lib.ora_sparse_bwd_dq_rows, lib.ora_sparse_bwd_dkv_blocks):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _ptr(a: Optional[np.ndarray], ctype):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def widen(x) -> np.ndarray:
    """Exact bf16 -> fp64 widening (a torch bf16 tensor, or fp64/fp32 array as is)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            if x.dtype == torch.bfloat16:
                bits = x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
                return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            return x.detach().cpu().numpy().astype(np.float64)
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(x, dtype=np.float64)


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(widen(x), dtype=np.float64)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (rc={rc})")


def block_pool(k, q=None, bs: int = BLOCK, nthreads: Optional[int] = None):
    """K-bar [B,Hkv,n,D] and, if q is given, group-pooled Q-bar [B,Hkv,n,D] (fp64)."""
    k64 = _f64(k)
    B, S, Hkv, D = k64.shape
    q64 = _f64(q) if q is not None else None
    Hq = q64.shape[2] if q64 is not None else Hkv
    n = S // bs
    kbar = np.zeros((B, Hkv, n, D))
    qbar = np.zeros((B, Hkv, n, D)) if q64 is not None else None
    rc = _load().ora_block_pool(B, S, Hq, Hkv, D, bs, _ptr(k64, ctypes.c_double),
                                _ptr(q64, ctypes.c_double), _ptr(kbar, ctypes.c_double),
                                _ptr(qbar, ctypes.c_double), nthreads or default_threads())
    _check(rc, "block_pool")
    return kbar, qbar


def block_select(qbar: np.ndarray, kbar: np.ndarray, topk: int, nthreads: Optional[int] = None):
    """idx [B,Hkv,n,topk] int32 ascending (-1 padded) and gap [B,Hkv,n] (NaN = no boundary)."""
    qbar = np.ascontiguousarray(qbar, dtype=np.float64)
    kbar = np.ascontiguousarray(kbar, dtype=np.float64)
    B, Hkv, n, D = kbar.shape
    idx = np.zeros((B, Hkv, n, topk), dtype=np.int32)
    gap = np.zeros((B, Hkv, n))
    rc = _load().ora_block_select(B, Hkv, n, D, topk, _ptr(qbar, ctypes.c_double),
                                  _ptr(kbar, ctypes.c_double), _ptr(idx, ctypes.c_int32),
                                  _ptr(gap, ctypes.c_double), nthreads or default_threads())
    _check(rc, "block_select")
    return idx, gap


def all_rows(B: int, Hq: int, S: int) -> np.ndarray:
    """Every (b, hq, t) triple, in that nesting order."""
    b, h, t = np.meshgrid(np.arange(B), np.arange(Hq), np.arange(S), indexing="ij")
    return np.stack([b.ravel(), h.ravel(), t.ravel()], axis=1).astype(np.int64)


def attn_rows(q, k, v, idx: np.ndarray, rows: np.ndarray, scale: Optional[float] = None,
              want_full: bool = True, bs: int = BLOCK, nthreads: Optional[int] = None
              ) -> Dict[str, np.ndarray]:
    """Per listed query row: sparse O/LSE and (want_full) full O/LSE and dropped mass."""
    q64, k64, v64 = _f64(q), _f64(k), _f64(v)
    B, S, Hq, D = q64.shape
    Hkv = k64.shape[2]
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    topk = idx.shape[-1]
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
    R = rows.shape[0]
    scale = (1.0 / np.sqrt(D)) if scale is None else float(scale)
    out = {"o_sparse": np.zeros((R, D)), "lse_sparse": np.zeros(R)}
    if want_full:
        out.update(o_full=np.zeros((R, D)), lse_full=np.zeros(R), delta=np.zeros(R),
                   delta_lse=np.zeros(R))
    g = out.get
    rc = _load().ora_attn_rows(
        B, S, Hq, Hkv, D, bs, topk, scale, _ptr(q64, ctypes.c_double), _ptr(k64, ctypes.c_double),
        _ptr(v64, ctypes.c_double), _ptr(idx, ctypes.c_int32), R, _ptr(rows, ctypes.c_int64),
        1 if want_full else 0, _ptr(out["o_sparse"], ctypes.c_double),
        _ptr(out["lse_sparse"], ctypes.c_double), _ptr(g("o_full"), ctypes.c_double),
        _ptr(g("lse_full"), ctypes.c_double), _ptr(g("delta"), ctypes.c_double),
        _ptr(g("delta_lse"), ctypes.c_double), nthreads or default_threads())
    _check(rc, "attn_rows")
    return out


def sparse_bwd_dq_rows(q, k, v, do, idx: np.ndarray, rows: np.ndarray,
                       scale: Optional[float] = None, bs: int = BLOCK,
                       nthreads: Optional[int] = None) -> np.ndarray:
    """dQ [R, D] for the listed (b, hq, t) rows."""
    q64, k64, v64, do64 = _f64(q), _f64(k), _f64(v), _f64(do)
    B, S, Hq, D = q64.shape
    Hkv = k64.shape[2]
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
    scale = (1.0 / np.sqrt(D)) if scale is None else float(scale)
    dq = np.zeros((rows.shape[0], D))
    rc = _load().ora_sparse_bwd_dq_rows(
        B, S, Hq, Hkv, D, bs, idx.shape[-1], scale, _ptr(q64, ctypes.c_double),
        _ptr(k64, ctypes.c_double), _ptr(v64, ctypes.c_double), _ptr(do64, ctypes.c_double),
        _ptr(idx, ctypes.c_int32), rows.shape[0], _ptr(rows, ctypes.c_int64),
        _ptr(dq, ctypes.c_double), nthreads or default_threads())
    _check(rc, "sparse_bwd_dq_rows")
    return dq


def sparse_bwd_dkv_blocks(q, k, v, do, idx: np.ndarray, blocks: np.ndarray,
                          scale: Optional[float] = None, bs: int = BLOCK,
                          nthreads: Optional[int] = None):
    """dK, dV [NB, bs, D] for the listed (b, kvh, key block j) triples."""
    q64, k64, v64, do64 = _f64(q), _f64(k), _f64(v), _f64(do)
    B, S, Hq, D = q64.shape
    Hkv = k64.shape[2]
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    blocks = np.ascontiguousarray(blocks, dtype=np.int64).reshape(-1, 3)
    scale = (1.0 / np.sqrt(D)) if scale is None else float(scale)
    dk = np.zeros((blocks.shape[0], bs, D))
    dv = np.zeros((blocks.shape[0], bs, D))
    rc = _load().ora_sparse_bwd_dkv_blocks(
        B, S, Hq, Hkv, D, bs, idx.shape[-1], scale, _ptr(q64, ctypes.c_double),
        _ptr(k64, ctypes.c_double), _ptr(v64, ctypes.c_double), _ptr(do64, ctypes.c_double),
        _ptr(idx, ctypes.c_int32), blocks.shape[0], _ptr(blocks, ctypes.c_int64),
        _ptr(dk, ctypes.c_double), _ptr(dv, ctypes.c_double), nthreads or default_threads())
    _check(rc, "sparse_bwd_dkv_blocks")
    return dk, dv


def dense_causal_table(B: int, Hkv: int, n: int) -> np.ndarray:
    """Index table [B, Hkv, n, n] that selects every causal block: row i holds
    0..i, then -1.  With it the sparse functions compute dense causal attention."""
    idx = np.full((B, Hkv, n, n), -1, dtype=np.int32)
    for i in range(n):
        idx[:, :, i, :i + 1] = np.arange(i + 1, dtype=np.int32)
    return idx


def alignment_output_grads(o_sparse, o_full, d_o, mode: int, alpha: float):
    """Output gradients of  <d_o, h_mode> + alpha (L_sparsity + L_commit)
    ("Resumen Tecnico: SSA", section 2, "Alineacion Bidireccional").

    The pages do not fix the distance; read as the mean squared error over the
    N elements of h with a stop-gradient (sg) on the target:
        L_sparsity = mean (h_full - sg(h_sparse))^2   (full pulled to sparse)
        L_commit   = mean (h_sparse - sg(h_full))^2   (sparse pulled to full)
    mode 0: d_o is the sparse output's upstream gradient; 1: the full one's.
    Returns (dO_sparse, dO_full) in fp64, shaped like the inputs."""
    o_s, o_f, g = widen(o_sparse), widen(o_full), widen(d_o)
    c = 2.0 * float(alpha) / o_s.size
    d_s = c * (o_s - o_f)          # from L_commit, through h_sparse
    d_f = c * (o_f - o_s)          # from L_sparsity, through h_full
    if mode == 0:
        d_s = d_s + g
    elif mode == 1:
        d_f = d_f + g
    else:
        raise ValueError("mode must be 0 or 1")
    return d_s, d_f


def decode_step(q, k, v, kbar, lengths, topk: int, scale: Optional[float] = None, bs: int = BLOCK):
    """One decoding step of the sparse stream, in fp64 ("SSA: Guida a Sparse
    Sparse Attention per LLM", section "Block-sparse attention e Receptive
    Field", applied to the newest token of each sequence).

    q [B, Hq, D] (token t = lengths[b] - 1), k and v [B, S, Hkv, D] caches,
    kbar [B, Hkv, n, D] mean keys.  Per KV head: the group's mean query scores
    the complete blocks j < c = t // 64; the top k - 1 (ties: lower j) and c are
    kept (every block 0..c when c + 1 <= k); attention over their tokens, keys
    up to t in block c.  Returns idx [B, Hkv, k] (ascending, -1 padded), gap
    [B, Hkv] (k-1-th minus k-th score, NaN when no boundary), o [B, Hq, D] and
    lse [B, Hq]."""
    q64, k64, v64 = widen(q), widen(k), widen(v)
    kbar = np.asarray(kbar, dtype=np.float64)
    B, Hq, D = q64.shape
    Hkv = k64.shape[2]
    G = Hq // Hkv
    scale = (1.0 / np.sqrt(D)) if scale is None else float(scale)
    idx = np.full((B, Hkv, topk), -1, dtype=np.int32)
    gap = np.full((B, Hkv), np.nan)
    o = np.zeros((B, Hq, D))
    lse = np.zeros((B, Hq))
    for b in range(B):
        t = int(lengths[b]) - 1
        c = t // bs
        for h in range(Hkv):
            if c + 1 <= topk:
                sel = list(range(c + 1))
            else:
                qbar = q64[b, h * G:(h + 1) * G].mean(axis=0)
                sc = kbar[b, h, :c] @ qbar
                order = sorted(range(c), key=lambda j: (-sc[j], j))
                gap[b, h] = sc[order[topk - 2]] - sc[order[topk - 1]]
                sel = sorted(order[:topk - 1]) + [c]
            idx[b, h, :len(sel)] = sel
            tok = np.concatenate([np.arange(bs * j, min(bs * j + bs, t + 1)) for j in sel])
            for g in range(G):
                hq = h * G + g
                logits = scale * (k64[b, tok, h] @ q64[b, hq])
                m = logits.max()
                w = np.exp(logits - m)
                lse[b, hq] = m + np.log(w.sum())
                o[b, hq] = (w / w.sum()) @ v64[b, tok, h]
    return idx, gap, o, lse


def early_stop_forward(q, k, v, qbar, kbar, idx: np.ndarray, tau: float,
                       scale: Optional[float] = None, bs: int = BLOCK):
    """The sparse forward with an early stop, in fp64 ("S2O" summary, section 2,
    "Regla de Parada Temprana", applied to the sparse stream; small problems).

    The unit that stops is one query segment of one attention head: query
    head hq, query block i, the 64 tokens of block i (b fixed).  Its blocks are
    visited in the order: i first (the segment's own causal window), then the
    other selected blocks of idx by descending pooled score
    qbar[b,h,i] . kbar[b,h,j] (ties: lower j), h the KV head of hq; this is
    the score the selection ranks by, shared by the heads of the group.  After
    each block after the first, the segment stops if every one of its rows
    gained less than tau times the mass it had in the blocks before it (the
    block itself still counts).  tau = 0 never stops.
    Returns o [B,S,Hq,D], lse [B,Hq,S], visited [B,Hq,n] (blocks each segment
    used) and margin [B,Hq,n]: the smallest |ln(max row ratio) - ln tau| over
    the segment's decisions (inf when tau = 0 or no decision was taken)."""
    q64, k64, v64 = widen(q), widen(k), widen(v)
    qbar = np.asarray(qbar, dtype=np.float64)
    kbar = np.asarray(kbar, dtype=np.float64)
    B, S, Hq, D = q64.shape
    Hkv = k64.shape[2]
    G, n = Hq // Hkv, S // bs
    scale = (1.0 / np.sqrt(D)) if scale is None else float(scale)
    o = np.zeros((B, S, Hq, D))
    lse = np.zeros((B, Hq, S))
    visited = np.zeros((B, Hq, n), dtype=np.int32)
    margin = np.full((B, Hq, n), np.inf)
    tok = np.arange(bs)
    for b in range(B):
        for h in range(Hkv):
            for i in range(n):
                sel = [int(j) for j in idx[b, h, i] if 0 <= j < i]
                sc = {j: float(kbar[b, h, j] @ qbar[b, h, i]) for j in sel}
                order = [i] + sorted(sel, key=lambda j: (-sc[j], j))
                for hq in range(h * G, (h + 1) * G):
                    qrows = q64[b, bs * i + tok, hq]                          # [64, D]
                    # per block: the logits of the segment's rows (causal in block i)
                    lg = []
                    for j in order:
                        l_ = scale * (qrows @ k64[b, bs * j + tok, h].T)      # [64 rows, 64 keys]
                        if j == i:
                            l_ = np.where(tok[None, :] <= tok[:, None], l_, -np.inf)
                        lg.append(l_)
                    blk = np.array([np.logaddexp.reduce(l_, axis=1) for l_ in lg])   # [blocks, 64]
                    nv = len(order)
                    for jj in range(1, len(order)):
                        before = np.logaddexp.reduce(blk[:jj], axis=0)              # [64]
                        lr = float(np.max(blk[jj] - before))                        # ln max row ratio
                        if tau > 0:
                            margin[b, hq, i] = min(margin[b, hq, i], abs(lr - np.log(tau)))
                        if tau > 0 and lr < np.log(tau):
                            nv = jj + 1
                            break
                    visited[b, hq, i] = nv
                    logits = np.concatenate(lg[:nv], axis=1)
                    vals = np.concatenate([v64[b, bs * j + tok, h] for j in order[:nv]], axis=0)
                    m = logits.max(axis=1, keepdims=True)
                    w = np.exp(logits - m)
                    lse[b, hq, bs * i + tok] = m[:, 0] + np.log(w.sum(axis=1))
                    o[b, bs * i + tok, hq] = (w / w.sum(axis=1, keepdims=True)) @ vals
    return o, lse, visited, margin


def sparse_forward_problem(q, k, v, topk: int, rows: Optional[np.ndarray] = None,
                           want_full: bool = False, nthreads: Optional[int] = None):
    """Pool -> select -> attention rows for a whole problem (or a row sample)."""
    kbar, qbar = block_pool(k, q, nthreads=nthreads)
    idx, gap = block_select(qbar, kbar, topk, nthreads=nthreads)
    if rows is None:
        B, S, Hq, _ = tuple(q.shape)
        rows = all_rows(B, Hq, S)
    out = attn_rows(q, k, v, idx, rows, want_full=want_full, nthreads=nthreads)
    out.update(idx=idx, gap=gap, kbar=kbar, qbar=qbar, rows=rows)
    return out


# ------------------------------------------------------------- DashAttention

def entmax(z, alpha: float):
    """alpha-entmax over the last axis, fp64 ("Resumen Tecnico: DashAttention",
    stage 1: the chunk logits become a sparse probability vector whose support
    the scores themselves decide).

    alpha-entmax(z) is the maximiser over the simplex of p.z plus the Tsallis
    alpha-entropy; its solution is p_j = [(alpha - 1) z_j - tau]_+ ^ (1/(alpha - 1))
    with the one threshold tau that makes the p_j sum to 1.  tau is found by
    bisection on [max x - 1, max x - m^(1 - alpha)] (x = (alpha - 1) z, m entries)
    until the bracket stops shrinking; p is then normalised.  1 < alpha.
    Returns (p, tau) with tau of shape z.shape[:-1]."""
    if not alpha > 1.0:
        raise ValueError("alpha-entmax needs alpha > 1")
    x = (alpha - 1.0) * np.asarray(z, dtype=np.float64)
    m = x.shape[-1]
    xmax = x.max(axis=-1, keepdims=True)
    lo = xmax - 1.0
    hi = xmax - float(m) ** (1.0 - alpha)
    inv = 1.0 / (alpha - 1.0)
    for _ in range(2000):
        mid = 0.5 * (lo + hi)
        f = (np.maximum(x - mid, 0.0) ** inv).sum(axis=-1, keepdims=True) - 1.0
        lo_new = np.where(f >= 0.0, mid, lo)
        hi_new = np.where(f >= 0.0, hi, mid)
        if np.array_equal(lo_new, lo) and np.array_equal(hi_new, hi):
            break
        lo, hi = lo_new, hi_new
    tau = 0.5 * (lo + hi)
    p = np.maximum(x - tau, 0.0) ** inv
    p = p / p.sum(axis=-1, keepdims=True)
    return p, tau[..., 0]


def dash_route(q, kbar, alpha: float, gamma: float, scale: Optional[float] = None, bs: int = BLOCK):
    """DashAttention chunk routing, fp64 ("Resumen Tecnico: DashAttention",
    stage 1, with its GQA rule; chunks of 64 tokens summarised by their mean
    key, stage 0 at its zero-initialised summary query).

    Per (b, KV head h, query block i) and query head g of the group: the mean
    query of block i, q_g, scores the complete earlier chunks j < i with
    z_j = gamma * scale * q_g . kbar[b, h, j]; p_g = alpha-entmax(z); the group
    shares w = mean_g p_g.  The diagonal chunk i is not routed (its own
    branch).  Returns
      w      [B, Hkv, n, n] fp64: w[.., i, j] for j < i, 0 elsewhere
      mask   [B, Hkv, n, ceil(n / 32)] uint32: bit j of row i set for j < i
             with w > 0, and bit i (the diagonal) always
      margin [B, Hkv, n, n]: min over g of |x_gj - tau_g| (x = (alpha-1) z),
             how far each support decision is from flipping; inf for j >= i."""
    q64 = widen(q)
    kbar = np.asarray(kbar, dtype=np.float64)
    B, S, Hq, D = q64.shape
    Hkv, n = kbar.shape[1], kbar.shape[2]
    G = Hq // Hkv
    scale = (1.0 / np.sqrt(D)) if scale is None else float(scale)
    W = (n + 31) // 32
    w = np.zeros((B, Hkv, n, n))
    mask = np.zeros((B, Hkv, n, W), dtype=np.uint32)
    margin = np.full((B, Hkv, n, n), np.inf)
    qpool = q64.reshape(B, n, bs, Hq, D).mean(axis=2)          # [B, n, Hq, D]
    for b in range(B):
        for h in range(Hkv):
            for i in range(n):
                if i > 0:
                    qg = qpool[b, i, h * G:(h + 1) * G]            # [G, D]
                    z = gamma * scale * (qg @ kbar[b, h, :i].T)    # [G, i]
                    p, tau = entmax(z, alpha)
                    w[b, h, i, :i] = p.mean(axis=0)
                    margin[b, h, i, :i] = np.abs((alpha - 1.0) * z - tau[:, None]).min(axis=0)
                for j in [jj for jj in range(i) if w[b, h, i, jj] > 0] + [i]:
                    mask[b, h, i, j // 32] |= np.uint32(1 << (j % 32))
    return w, mask, margin


def dash_attention(q, k, v, mask, w, sigma: float, scale: Optional[float] = None, bs: int = BLOCK,
                   blocks=None):
    """DashAttention's prior-induced sparse softmax, fp64 ("Resumen Tecnico:
    DashAttention", stage 2).

    The softmax's uniform reference distribution is replaced by a prior g over
    the keys: g is uniform inside a chunk and proportional to w_j^sigma across
    the active chunks, and 0 elsewhere, so the attention p maximising
    z.p - KL(p || g) is p_s proportional to g_s exp(z_s).  For query t of block
    i the active chunks are the j < i whose mask bit is set and whose w_j is
    finite and > 0, plus the diagonal chunk i with weight 1 (its own branch);
    causal inside i.
    Logits are scale * q_t . k_s + sigma * ln w_j.  Returns o [B, S, Hq, D] and
    lse [B, Hq, S], the natural-log log-sum-exp of the biased logits; with
    `blocks` (rows of (b, KV head, query block)) only those are computed and
    the rest is left 0."""
    q64, k64, v64 = widen(q), widen(k), widen(v)
    w = np.asarray(w, dtype=np.float64)
    mask = np.asarray(mask, dtype=np.uint32)
    B, S, Hq, D = q64.shape
    Hkv = k64.shape[2]
    G, n = Hq // Hkv, S // bs
    scale = (1.0 / np.sqrt(D)) if scale is None else float(scale)
    o = np.zeros((B, S, Hq, D))
    lse = np.zeros((B, Hq, S))
    tok = np.arange(bs)
    if blocks is None:
        blocks = [(b, h, i) for b in range(B) for h in range(Hkv) for i in range(n)]
    for b, h, i in blocks:
        act = [j for j in range(i)
               if (int(mask[b, h, i, j // 32]) >> (j % 32)) & 1 and 0 < w[b, h, i, j] < np.inf]
        keys = np.concatenate([bs * j + tok for j in act] + [bs * i + tok])
        bias = np.concatenate([np.full(bs, sigma * np.log(w[b, h, i, j])) for j in act]
                              + [np.zeros(bs)])
        for hq in range(h * G, (h + 1) * G):
            lg = scale * (q64[b, bs * i + tok, hq] @ k64[b, keys, h].T) + bias[None, :]
            lg[:, -bs:] = np.where(tok[None, :] <= tok[:, None], lg[:, -bs:], -np.inf)
            mx = lg.max(axis=1, keepdims=True)
            e = np.exp(lg - mx)
            lse[b, hq, bs * i + tok] = mx[:, 0] + np.log(e.sum(axis=1))
            o[b, bs * i + tok, hq] = (e / e.sum(axis=1, keepdims=True)) @ v64[b, keys, h]
    return o, lse
