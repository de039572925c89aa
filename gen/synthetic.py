"""Seeded synthetic inputs for the SSA sparse stream (block-sparse causal attention).

This module draws Q, K, V (and an upstream gradient dO) with the shapes of the
workloads the SSA pages describe: a Llama-3.2-1B-like attention layer with
fewer KV heads than query heads ("SSA: Guida a Sparse Sparse Attention per LLM",
sections "Approccio generale" and "Training recipe"), at 8k context and at the
32k continued-training length ("Resumen Tecnico: SSA", section 4).  The pages
evaluate on text datasets with trained weights; neither is available, so these
tensors stand in for that model's post-projection attention inputs.

It holds none of the method's arithmetic: no pooling, no scoring, no
selection, no softmax.  Both the fp64 oracle and the CUDA path consume exactly
the bf16 tensors produced here.

Recipe (one draw in fp64, plants added, one rounding to bf16 at the end):
  * Q, K, V base values are i.i.d. N(0, 1) from numpy PCG64(seed).
  * Planted structure (all configurations except the tiny one): every
    (batch, KV head, key block j) owns a random unit direction u_j; every key
    of block j is shifted by +shift * u_j.  Each query block i draws a set P_i
    of `n_plant` distinct earlier blocks (all of them when i <= n_plant) and
    every query of block i, in all heads of the GQA group, is shifted by
    sum_{j in P_i} u_j.  This concentrates attention mass on P_i.
  * Score-gap plan: the parity contract compares selected block indices bit
    for bit, which is only meaningful when the k-th and (k+1)-th block scores
    are separated.  Rows whose gap was found too small are redrawn: the query
    noise of block i for that KV head's group is replaced by a draw from the
    sub-generator PCG64(SeedSequence([seed, b, kvh, i, attempt])).  The
    attempt number per row is read from a stored plan (JSON) produced by a
    committed script under tests/golden that checks the gap with the oracle.
    No score is computed in this module.
"""
from __future__ import annotations

import dataclasses
import json
import os
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np
import torch

BLOCK = 64

_HERE = os.path.dirname(os.path.abspath(__file__))
DEFAULT_PLAN_PATH = os.path.join(os.path.dirname(_HERE), "tests", "golden", "gap_plan.json")


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, budget and input distribution."""

    name: str
    batch: int
    seq_len: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    top_k: int
    seed: int
    n_plant: int = 0          # planted salient blocks per query block (0 = none)
    plant_shift: float = 1.5  # key shift along u_j
    with_do: bool = False     # also draw an upstream gradient dO ~ N(0, 1)
    top_k_sweep: Tuple[int, ...] = ()  # extra budgets whose score gap is also enforced

    @property
    def n_blocks(self) -> int:
        return self.seq_len // BLOCK

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def gap_budgets(self) -> Tuple[int, ...]:
        ks = {self.top_k, *self.top_k_sweep}
        return tuple(sorted(ks))


# The five workloads.  Names say what each one is.
WORKLOADS: Dict[str, Workload] = {
    # tiny causal problem, i.i.d. N(0,1), RF = 4 blocks * 64 = 256 tokens
    "tiny_1k": Workload("tiny_1k", 1, 1024, 4, 1, 64, 4, seed=1001),
    # Llama-3.2-1B-like attention layer at 8k, RF = 16 * 64 = 1024 tokens
    "llama1b_8k": Workload("llama1b_8k", 1, 8192, 32, 4, 64, 16, seed=1002, n_plant=8),
    # the SSA alignment pass (sparse + counterpart full + dropped mass), batch 2
    "align_8k": Workload("align_8k", 2, 8192, 32, 4, 64, 16, seed=1003, n_plant=8),
    # long-context extrapolation at 32k with a top-k budget sweep
    "long_32k": Workload("long_32k", 1, 32768, 16, 2, 128, 16, seed=1004, n_plant=6,
                         top_k_sweep=(8, 16, 32, 64, 128)),
    # training-shaped sparse stream, forward + backward, batch 4
    "train_8k": Workload("train_8k", 4, 8192, 32, 4, 64, 16, seed=1005, n_plant=8,
                         with_do=True),
}


@dataclasses.dataclass
class SynthInputs:
    workload: Workload
    q: torch.Tensor            # [B, S, Hq, D] bf16, CPU
    k: torch.Tensor            # [B, S, Hkv, D] bf16, CPU
    v: torch.Tensor            # [B, S, Hkv, D] bf16, CPU
    do: Optional[torch.Tensor]  # [B, S, Hq, D] bf16, CPU, or None
    plants: Dict[Tuple[int, int, int], Tuple[int, ...]]  # (b, kvh, i) -> P_i


def load_plan(path: str = DEFAULT_PLAN_PATH) -> Dict[str, List[List[int]]]:
    """Stored redraw plan: {workload name: [[b, kvh, i, attempt], ...]}."""
    if not os.path.exists(path):
        return {}
    with open(path) as f:
        data = json.load(f)
    return {name: entry["redraws"] for name, entry in data.items()}


def _to_bf16(x: np.ndarray) -> torch.Tensor:
    # fp64 -> fp32 (round to nearest even) -> bf16 (round to nearest even)
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


def _sub_generator(seed: int, b: int, kvh: int, i: int, attempt: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, b, kvh, i, attempt])))


def make_custom(batch: int, seq_len: int, n_q_heads: int, n_kv_heads: int, head_dim: int,
                top_k: int, seed: int, n_plant: int = 0, plant_shift: float = 1.5,
                with_do: bool = False, redraws: Sequence[Sequence[int]] = ()) -> SynthInputs:
    """Draw inputs for an arbitrary shape with the recipe of the module docstring."""
    w = Workload("custom", batch, seq_len, n_q_heads, n_kv_heads, head_dim, top_k, seed,
                 n_plant=n_plant, plant_shift=plant_shift, with_do=with_do)
    return _draw(w, redraws)


def make_inputs(name: str, *, redraws: Optional[Sequence[Sequence[int]]] = None,
                plan_path: str = DEFAULT_PLAN_PATH) -> SynthInputs:
    """Inputs of a named workload, with its stored score-gap redraw plan applied."""
    w = WORKLOADS[name]
    if redraws is None:
        redraws = load_plan(plan_path).get(name, [])
    return _draw(w, redraws)


def _draw(w: Workload, redraws: Sequence[Sequence[int]]) -> SynthInputs:
    B, S, Hq, Hkv, D = w.batch, w.seq_len, w.n_q_heads, w.n_kv_heads, w.head_dim
    if S % BLOCK != 0 or Hq % Hkv != 0:
        raise ValueError("seq_len must be a multiple of 64 and n_q_heads of n_kv_heads")
    G, n = Hq // Hkv, S // BLOCK
    rng = np.random.Generator(np.random.PCG64(w.seed))

    q = rng.standard_normal((B, S, Hq, D))
    k = rng.standard_normal((B, S, Hkv, D))
    v = rng.standard_normal((B, S, Hkv, D))

    plants: Dict[Tuple[int, int, int], Tuple[int, ...]] = {}
    q_shift = np.zeros((B, Hkv, n, D))
    if w.n_plant > 0:
        u = rng.standard_normal((B, Hkv, n, D))
        u /= np.linalg.norm(u, axis=-1, keepdims=True)
        for b in range(B):
            for h in range(Hkv):
                for i in range(n):
                    if i <= w.n_plant:
                        pick = tuple(range(i))
                    else:
                        pick = tuple(sorted(int(x) for x in rng.choice(i, size=w.n_plant, replace=False)))
                    plants[(b, h, i)] = pick
                    if pick:
                        q_shift[b, h, i] = u[b, h, list(pick)].sum(axis=0)
        # keys of block j move along their own direction u_j
        k.reshape(B, n, BLOCK, Hkv, D)[...] += w.plant_shift * u.transpose(0, 2, 1, 3)[:, :, None, :, :]
        # queries of block i, all G heads of the group, move along sum of u over P_i
        q.reshape(B, n, BLOCK, Hkv, G, D)[...] += q_shift.transpose(0, 2, 1, 3)[:, :, None, :, None, :]

    do = rng.standard_normal((B, S, Hq, D)) if w.with_do else None

    for entry in redraws:
        b, h, i, attempt = (int(x) for x in entry)
        sub = _sub_generator(w.seed, b, h, i, attempt)
        noise = sub.standard_normal((BLOCK, G, D))
        q[b, i * BLOCK:(i + 1) * BLOCK, h * G:(h + 1) * G, :] = noise + q_shift[b, h, i][None, None, :]

    return SynthInputs(w, _to_bf16(q), _to_bf16(k), _to_bf16(v),
                       _to_bf16(do) if do is not None else None, plants)


@dataclasses.dataclass
class DecodeInputs:
    q: torch.Tensor            # [B, Hq, D] bf16: each sequence's newest token
    k: torch.Tensor            # [B, S, Hkv, D] bf16 cache (S = capacity)
    v: torch.Tensor            # [B, S, Hkv, D] bf16 cache
    lengths: np.ndarray        # [B] int32 cached tokens, the newest included
    top_k: int


def make_decode(batch: int, capacity: int, n_q_heads: int, n_kv_heads: int, head_dim: int,
                top_k: int, seed: int, n_plant: int = 8, plant_shift: float = 1.5,
                lengths: Optional[Sequence[int]] = None) -> DecodeInputs:
    """A KV cache and one new query per sequence, drawn with the recipe of the
    module docstring: N(0, 1) values, every key block shifted by plant_shift
    along its own unit direction u_j, and each sequence's query (all heads of a
    KV head's group) shifted by the sum of u_j over n_plant distinct complete
    blocks before its own.  Lengths default to uniform draws in
    [capacity / 2, capacity]."""
    B, S, Hq, Hkv, D = batch, capacity, n_q_heads, n_kv_heads, head_dim
    if S % BLOCK != 0 or Hq % Hkv != 0:
        raise ValueError("capacity must be a multiple of 64 and n_q_heads of n_kv_heads")
    G, n = Hq // Hkv, S // BLOCK
    rng = np.random.Generator(np.random.PCG64(seed))
    k = rng.standard_normal((B, S, Hkv, D))
    v = rng.standard_normal((B, S, Hkv, D))
    u = rng.standard_normal((B, Hkv, n, D))
    u /= np.linalg.norm(u, axis=-1, keepdims=True)
    k.reshape(B, n, BLOCK, Hkv, D)[...] += plant_shift * u.transpose(0, 2, 1, 3)[:, :, None, :, :]
    if lengths is None:
        lengths = rng.integers(S // 2, S + 1, size=B)
    lengths = np.asarray(lengths, dtype=np.int32)
    q = rng.standard_normal((B, Hq, D))
    for b in range(B):
        c = (int(lengths[b]) - 1) // BLOCK
        for h in range(Hkv):
            m = min(n_plant, c)
            if m > 0:
                pick = rng.choice(c, size=m, replace=False)
                q[b, h * G:(h + 1) * G] += u[b, h, pick].sum(axis=0)
    return DecodeInputs(q=_to_bf16(q), k=_to_bf16(k), v=_to_bf16(v), lengths=lengths, top_k=top_k)


@dataclasses.dataclass
class DashRouting:
    """A synthetic DashAttention routing: group weights and a bit mask."""
    weights: np.ndarray   # [B, Hkv, n, n] float32
    mask: np.ndarray      # [B, Hkv, n, ceil(n / 32)] uint32


def make_dash_routing(batch: int, n_kv_heads: int, n_blocks: int, seed: int, density: float = 0.5,
                      zero_frac: float = 0.3) -> DashRouting:
    """Random routing inputs for the prior-induced softmax, independent of any
    scores: each mask bit is set with probability `density` (bits at and after
    the diagonal and the diagonal bit itself included, so the rule that ignores
    the former and always keeps the diagonal is exercised), and each weight is
    uniform in [0.01, 1) except a `zero_frac` share that is exactly 0 (set bits
    with zero weight must be skipped)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    n = n_blocks
    shape = (batch, n_kv_heads, n, n)
    w = rng.uniform(0.01, 1.0, size=shape) * (rng.random(shape) >= zero_frac)
    bits = rng.random(shape) < density
    words = (n + 31) // 32
    padded = np.zeros((batch, n_kv_heads, n, words * 32), dtype=bool)
    padded[..., :n] = bits
    weights_of_bits = (1 << np.arange(32, dtype=np.uint64)).astype(np.uint64)
    mask = (padded.reshape(batch, n_kv_heads, n, words, 32).astype(np.uint64) * weights_of_bits).sum(axis=-1)
    return DashRouting(weights=w.astype(np.float32), mask=mask.astype(np.uint32))
