"""SSA sparse stream on B200: block-sparse causal attention with top-k KV-block
selection, as hand-written sm_100a kernels behind a C ABI (libssa.so).

The C entry points are re-exported with their own names (argument marshalling
only, see _binding.py).  `SparseStream` strings them together over buffers it
allocates once with torch (device memory and streams are all torch is used for).
"""
from __future__ import annotations

from typing import Optional

import torch

from ._binding import (EXPORTED, LIB_PATH, SsaError, SsaProblem, lib, problem,
                       ssa_alignment_bwd, ssa_alignment_bwd_workspace, ssa_decode_attn,
                       ssa_dash_attn_fwd, ssa_dash_route, ssa_sparse_attn_fwd_host,
                       ssa_sparse_attn_fwd_host_workspace,
                       ssa_decode_attn_workspace, ssa_sparse_attn_fwd_early_stop,
                       ssa_block_pool, ssa_block_select, ssa_debug_exp2_poly, ssa_debug_timeout_probe,
                       ssa_full_attn_fwd_with_mass, ssa_get_device_error,
                       ssa_get_device_error_site, ssa_launch_count,
                       ssa_sparse_attn_bwd, ssa_sparse_attn_bwd_noalloc,
                       ssa_sparse_attn_bwd_workspace,
                       ssa_sparse_attn_fwd, ssa_status_string)

__all__ = ["EXPORTED", "LIB_PATH", "DashAttention", "SsaError", "SsaProblem", "SparseStream", "lib", "problem",
           "ssa_dash_attn_fwd", "ssa_dash_route", "ssa_sparse_attn_fwd_host",
           "ssa_sparse_attn_fwd_host_workspace",
           "ssa_alignment_bwd", "ssa_alignment_bwd_workspace", "ssa_decode_attn",
           "ssa_decode_attn_workspace", "ssa_sparse_attn_fwd_early_stop",
           "ssa_block_pool", "ssa_block_select", "ssa_debug_exp2_poly", "ssa_debug_timeout_probe",
           "ssa_full_attn_fwd_with_mass", "ssa_get_device_error", "ssa_get_device_error_site",
           "ssa_launch_count",
           "ssa_sparse_attn_bwd", "ssa_sparse_attn_bwd_noalloc", "ssa_sparse_attn_bwd_workspace",
           "ssa_sparse_attn_fwd",
           "ssa_status_string"]


class SparseStream:
    """Pre-allocated buffers for one problem shape and the calls of the path.

    forward():   ssa_block_pool -> ssa_block_select -> ssa_sparse_attn_fwd
    alignment(): ssa_block_pool -> ssa_block_select -> ssa_full_attn_fwd_with_mass
    backward():  ssa_sparse_attn_bwd (after forward())
    """

    def __init__(self, p: SsaProblem, device: Optional[torch.device] = None):
        self.p = p
        dev = device or torch.device("cuda", torch.cuda.current_device())
        B, S, Hq, Hkv, D = p.batch, p.seq_len, p.n_q_heads, p.n_kv_heads, p.head_dim
        n = S // p.block_size
        f32, bf16 = torch.float32, torch.bfloat16
        self.k_pooled = torch.empty(B, Hkv, n, D, dtype=f32, device=dev)
        self.q_pooled = torch.empty(B, Hkv, n, D, dtype=f32, device=dev)
        self.block_idx = torch.empty(B, Hkv, n, p.top_k, dtype=torch.int32, device=dev)
        self.o = torch.empty(B, S, Hq, D, dtype=bf16, device=dev)
        self.lse = torch.empty(B, Hq, S, dtype=f32, device=dev)
        self._full = None
        self._grad = None
        self._agrad = None

    def select(self, q, k, stream=None):
        ssa_block_pool(self.p, k, q, self.k_pooled, self.q_pooled, stream)
        ssa_block_select(self.p, self.q_pooled, self.k_pooled, self.block_idx, stream)
        return self.block_idx

    def forward(self, q, k, v, stream=None):
        self.select(q, k, stream)
        ssa_sparse_attn_fwd(self.p, q, k, v, self.block_idx, self.o, self.lse, stream)
        return self.o

    def forward_host(self, q, k, v, o, lse, stream=None):
        """The forward on host tensors (page-locked for overlap): q, k, v in,
        o and lse out, pipelined by (batch, KV head) inside the library."""
        if getattr(self, "_host_ws", None) is None:
            n = ssa_sparse_attn_fwd_host_workspace(self.p)
            self._host_ws = torch.empty(n, dtype=torch.uint8, device=self.o.device)
        ssa_sparse_attn_fwd_host(self.p, q, k, v, o, lse, self._host_ws, self._host_ws.numel(), stream)
        return o

    def alignment(self, q, k, v, stream=None):
        if self._full is None:
            self._full = (torch.empty_like(self.o), torch.empty_like(self.lse),
                          torch.empty_like(self.lse))
        o_full, lse_full, dropped = self._full
        self.select(q, k, stream)
        ssa_full_attn_fwd_with_mass(self.p, q, k, v, self.block_idx, self.o, self.lse, o_full,
                                    lse_full, dropped, stream)
        return self.o, o_full, dropped

    def capture_forward(self, q, k, v) -> "torch.cuda.CUDAGraph":
        """A CUDA graph of forward() over these exact buffers (pool, select and
        sparse attention: three kernel launches); graph.replay() reruns it on
        the current stream.  Refill q, k, v in place to run on new data."""
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self.forward(q, k, v)          # first call sets kernel attributes
        torch.cuda.current_stream().wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            self.forward(q, k, v)
        return graph

    def backward(self, q, k, v, d_o, stream=None):
        if self._grad is None:
            ws = ssa_sparse_attn_bwd_workspace(self.p)
            self._grad = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v),
                          torch.empty(max(ws, 256), dtype=torch.uint8, device=q.device), ws)
        dq, dk, dv, workspace, ws = self._grad
        ssa_sparse_attn_bwd(self.p, q, k, v, self.o, self.lse, d_o, self.block_idx, dq, dk, dv,
                            workspace, workspace.numel(), stream)
        return dq, dk, dv

    def alignment_backward(self, q, k, v, d_o, mode: int = 0, alpha: float = 1.0, stream=None):
        """Gradients with respect to q, k, v of <d_o, h_mode> + alpha * (L_sparsity +
        L_commit) after alignment() ran on the same inputs (mode 0: d_o is the
        gradient of the sparse output, 1: of the full output)."""
        if self._full is None:
            raise RuntimeError("alignment() must run before alignment_backward()")
        if self._agrad is None:
            ws = ssa_alignment_bwd_workspace(self.p)
            self._agrad = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v),
                           torch.empty(max(ws, 256), dtype=torch.uint8, device=q.device))
        dq, dk, dv, workspace = self._agrad
        o_full, lse_full, _ = self._full
        ssa_alignment_bwd(self.p, q, k, v, self.o, self.lse, o_full, lse_full, d_o, mode, alpha,
                          self.block_idx, dq, dk, dv, workspace, workspace.numel(), stream)
        return dq, dk, dv


class DashAttention:
    """DashAttention's forward over buffers allocated once: the chunk summaries
    (ssa_block_pool, keys only), the routing (ssa_dash_route) and the
    prior-induced sparse softmax (ssa_dash_attn_fwd).  alpha: the entmax
    exponent; gamma: the routing temperature; sigma: the prior's strength."""

    def __init__(self, p: SsaProblem, alpha: float = 1.5, gamma: float = 1.0, sigma: float = 1.0,
                 device: Optional[torch.device] = None):
        lib()
        self.p, self.alpha, self.gamma, self.sigma = p, float(alpha), float(gamma), float(sigma)
        dev = device or torch.device("cuda")
        B, S, Hq, Hkv, D = p.batch, p.seq_len, p.n_q_heads, p.n_kv_heads, p.head_dim
        n = S // 64
        self.k_pooled = torch.empty(B, Hkv, n, D, dtype=torch.float32, device=dev)
        self.weights = torch.empty(B, Hkv, n, n, dtype=torch.float32, device=dev)
        self.mask = torch.empty(B, Hkv, n, (n + 31) // 32, dtype=torch.int32, device=dev)
        self.o = torch.empty(B, S, Hq, D, dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(B, Hq, S, dtype=torch.float32, device=dev)

    def route(self, q, k, stream=None):
        ssa_block_pool(self.p, k, None, self.k_pooled, None, stream)
        ssa_dash_route(self.p, q, self.k_pooled, self.alpha, self.gamma, self.weights, self.mask, stream)

    def forward(self, q, k, v, stream=None):
        self.route(q, k, stream)
        ssa_dash_attn_fwd(self.p, q, k, v, self.weights, self.mask, self.sigma, self.o, self.lse, stream)
        return self.o, self.lse
