"""ctypes binding of libssa.so -- argument marshalling only.

Every function here has the name of the C entry point it calls and takes the
same arguments, with torch tensors standing for device pointers.  No step of
the computation happens in Python: each call validates dtypes/devices/shapes,
passes raw pointers and the current CUDA stream, and raises SsaError on a
non-OK status.  If libssa.so is missing the import fails loudly; there is no
fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libssa.so")

SSA_OK = 0
STATUS_NAMES = {0: "SSA_OK", 1: "SSA_ERR_INVALID_ARG", 2: "SSA_ERR_UNSUPPORTED",
                3: "SSA_ERR_CUDA", 4: "SSA_ERR_DEVICE_TIMEOUT", 5: "SSA_ERR_WORKSPACE"}

# every symbol include/ssa.h declares
EXPORTED = ("ssa_block_pool", "ssa_block_select", "ssa_sparse_attn_fwd", "ssa_sparse_attn_fwd_early_stop",
            "ssa_full_attn_fwd_with_mass", "ssa_sparse_attn_bwd_workspace",
            "ssa_sparse_attn_bwd", "ssa_sparse_attn_bwd_noalloc", "ssa_alignment_bwd_workspace",
            "ssa_alignment_bwd", "ssa_decode_attn_workspace", "ssa_decode_attn",
            "ssa_dash_route", "ssa_dash_attn_fwd", "ssa_sparse_attn_fwd_host_workspace",
            "ssa_sparse_attn_fwd_host",
            "ssa_get_device_error",
            "ssa_get_device_error_site",
            "ssa_debug_timeout_probe", "ssa_debug_exp2_poly",
            "ssa_status_string", "ssa_launch_count")


class SsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")
        self.status = status


class SsaProblem(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("seq_len", ctypes.c_int), ("n_q_heads", ctypes.c_int),
                ("n_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("block_size", ctypes.c_int), ("top_k", ctypes.c_int), ("causal", ctypes.c_int),
                ("softmax_scale", ctypes.c_float)]


def problem(batch: int, seq_len: int, n_q_heads: int, n_kv_heads: int, head_dim: int,
            top_k: int, block_size: int = 64, causal: int = 1,
            softmax_scale: float = 0.0) -> SsaProblem:
    return SsaProblem(batch, seq_len, n_q_heads, n_kv_heads, head_dim, block_size, top_k,
                      causal, softmax_scale)


_lib = None


def lib():
    """The loaded libssa.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libssa.so not found at {LIB_PATH}: build it with "
                               "`python -m block_sparse_attention_21_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, P = ctypes.c_void_p, ctypes.POINTER(SsaProblem)
        sigs = {
            "ssa_block_pool": [P, vp, vp, vp, vp, vp],
            "ssa_block_select": [P, vp, vp, vp, vp],
            "ssa_sparse_attn_fwd": [P, vp, vp, vp, vp, vp, vp, vp],
            "ssa_full_attn_fwd_with_mass": [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp],
            "ssa_sparse_attn_bwd": [P] + [vp] * 11 + [ctypes.c_size_t, vp],
            "ssa_sparse_attn_bwd_noalloc": [P] + [vp] * 11,
            "ssa_decode_attn": [P] + [vp] * 9 + [ctypes.c_size_t, vp],
            "ssa_sparse_attn_fwd_early_stop": [P] + [vp] * 6 + [ctypes.c_float] + [vp] * 4,
            "ssa_alignment_bwd": [P] + [vp] * 8 + [ctypes.c_int, ctypes.c_float] + [vp] * 5
                                 + [ctypes.c_size_t, vp],
            "ssa_dash_route": [P, vp, vp, ctypes.c_float, ctypes.c_float, vp, vp, vp],
            "ssa_sparse_attn_fwd_host": [P] + [vp] * 6 + [ctypes.c_size_t, vp],
            "ssa_dash_attn_fwd": [P] + [vp] * 5 + [ctypes.c_float] + [vp] * 3,
            "ssa_get_device_error": [vp],
            "ssa_debug_timeout_probe": [ctypes.c_int, vp],
            "ssa_debug_exp2_poly": [vp, vp, ctypes.c_int, vp],
        }
        for name, args in sigs.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        for name in ("ssa_sparse_attn_bwd_workspace", "ssa_alignment_bwd_workspace",
                     "ssa_decode_attn_workspace", "ssa_sparse_attn_fwd_host_workspace"):
            getattr(L, name).argtypes = [P]
            getattr(L, name).restype = ctypes.c_size_t
        L.ssa_status_string.argtypes = [ctypes.c_int]
        L.ssa_status_string.restype = ctypes.c_char_p
        L.ssa_get_device_error_site.argtypes = []
        L.ssa_get_device_error_site.restype = ctypes.c_uint
        L.ssa_launch_count.argtypes = []
        L.ssa_launch_count.restype = ctypes.c_uint64
        _lib = L
    return _lib


def _ptr(t: Optional[torch.Tensor], dtype=None, name: str = "") -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name}: expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name}: expected {dtype}, got {t.dtype}")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _call(name: str, *args) -> None:
    rc = getattr(lib(), name)(*args)
    if rc != SSA_OK:
        raise SsaError(rc, name)


def _numel_check(t, shape, name):
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")


def _shapes(p: SsaProblem):
    B, S, Hq, Hkv, D = p.batch, p.seq_len, p.n_q_heads, p.n_kv_heads, p.head_dim
    n = S // max(p.block_size, 1)
    return dict(q=(B, S, Hq, D), kv=(B, S, Hkv, D), pooled=(B, Hkv, n, D),
                idx=(B, Hkv, n, p.top_k), lse=(B, Hq, S))


BF16, F32, I32 = torch.bfloat16, torch.float32, torch.int32


def ssa_block_pool(p: SsaProblem, k, q, k_pooled, q_pooled, stream=None) -> None:
    sh = _shapes(p)
    _numel_check(k, sh["kv"], "k")
    _numel_check(k_pooled, sh["pooled"], "k_pooled")
    if q is not None:
        _numel_check(q, sh["q"], "q")
        _numel_check(q_pooled, sh["pooled"], "q_pooled")
    _call("ssa_block_pool", ctypes.byref(p), _ptr(k, BF16, "k"), _ptr(q, BF16, "q"),
          _ptr(k_pooled, F32, "k_pooled"), _ptr(q_pooled, F32, "q_pooled"), _stream(stream))


def ssa_block_select(p: SsaProblem, q_pooled, k_pooled, block_idx, stream=None) -> None:
    sh = _shapes(p)
    _numel_check(q_pooled, sh["pooled"], "q_pooled")
    _numel_check(k_pooled, sh["pooled"], "k_pooled")
    _numel_check(block_idx, sh["idx"], "block_idx")
    _call("ssa_block_select", ctypes.byref(p), _ptr(q_pooled, F32, "q_pooled"),
          _ptr(k_pooled, F32, "k_pooled"), _ptr(block_idx, I32, "block_idx"), _stream(stream))


def ssa_sparse_attn_fwd(p: SsaProblem, q, k, v, block_idx, o, lse, stream=None) -> None:
    sh = _shapes(p)
    for t, s, nm in ((q, "q", "q"), (k, "kv", "k"), (v, "kv", "v"), (block_idx, "idx", "block_idx"),
                     (o, "q", "o"), (lse, "lse", "lse")):
        _numel_check(t, sh[s], nm)
    _call("ssa_sparse_attn_fwd", ctypes.byref(p), _ptr(q, BF16, "q"), _ptr(k, BF16, "k"),
          _ptr(v, BF16, "v"), _ptr(block_idx, I32, "block_idx"), _ptr(o, BF16, "o"),
          _ptr(lse, F32, "lse"), _stream(stream))


def ssa_full_attn_fwd_with_mass(p: SsaProblem, q, k, v, block_idx, o_sparse, lse_sparse, o_full,
                                lse_full, dropped, stream=None) -> None:
    sh = _shapes(p)
    for t, s, nm in ((q, "q", "q"), (k, "kv", "k"), (v, "kv", "v"), (block_idx, "idx", "block_idx"),
                     (o_sparse, "q", "o_sparse"), (lse_sparse, "lse", "lse_sparse"),
                     (o_full, "q", "o_full"), (lse_full, "lse", "lse_full"),
                     (dropped, "lse", "dropped")):
        _numel_check(t, sh[s], nm)
    _call("ssa_full_attn_fwd_with_mass", ctypes.byref(p), _ptr(q, BF16, "q"), _ptr(k, BF16, "k"),
          _ptr(v, BF16, "v"), _ptr(block_idx, I32, "block_idx"), _ptr(o_sparse, BF16, "o_sparse"),
          _ptr(lse_sparse, F32, "lse_sparse"), _ptr(o_full, BF16, "o_full"),
          _ptr(lse_full, F32, "lse_full"), _ptr(dropped, F32, "dropped"), _stream(stream))


def ssa_sparse_attn_bwd_workspace(p: SsaProblem) -> int:
    return int(lib().ssa_sparse_attn_bwd_workspace(ctypes.byref(p)))


def ssa_sparse_attn_bwd(p: SsaProblem, q, k, v, o, lse, d_o, block_idx, dq, dk, dv, workspace,
                        ws_bytes: int, stream=None) -> None:
    sh = _shapes(p)
    for t, s, nm in ((q, "q", "q"), (k, "kv", "k"), (v, "kv", "v"), (o, "q", "o"),
                     (lse, "lse", "lse"), (d_o, "q", "d_o"), (block_idx, "idx", "block_idx"),
                     (dq, "q", "dq"), (dk, "kv", "dk"), (dv, "kv", "dv")):
        _numel_check(t, sh[s], nm)
    _call("ssa_sparse_attn_bwd", ctypes.byref(p), _ptr(q, BF16, "q"), _ptr(k, BF16, "k"),
          _ptr(v, BF16, "v"), _ptr(o, BF16, "o"), _ptr(lse, F32, "lse"), _ptr(d_o, BF16, "d_o"),
          _ptr(block_idx, I32, "block_idx"), _ptr(dq, BF16, "dq"), _ptr(dk, BF16, "dk"),
          _ptr(dv, BF16, "dv"), _ptr(workspace, None, "workspace"), int(ws_bytes),
          _stream(stream))


def ssa_alignment_bwd_workspace(p: SsaProblem) -> int:
    return int(lib().ssa_alignment_bwd_workspace(ctypes.byref(p)))


def ssa_alignment_bwd(p: SsaProblem, q, k, v, o_sparse, lse_sparse, o_full, lse_full, d_o,
                      mode: int, alpha: float, block_idx, dq, dk, dv, workspace, ws_bytes: int,
                      stream=None) -> None:
    """Backward of <d_o, h_mode> + alpha (L_sparsity + L_commit) (mode 0: d_o is
    the sparse output's gradient, 1: the full output's); see include/ssa.h."""
    sh = _shapes(p)
    for t, s, nm in ((q, "q", "q"), (k, "kv", "k"), (v, "kv", "v"), (o_sparse, "q", "o_sparse"),
                     (lse_sparse, "lse", "lse_sparse"), (o_full, "q", "o_full"),
                     (lse_full, "lse", "lse_full"), (d_o, "q", "d_o"),
                     (block_idx, "idx", "block_idx"), (dq, "q", "dq"), (dk, "kv", "dk"),
                     (dv, "kv", "dv")):
        _numel_check(t, sh[s], nm)
    _call("ssa_alignment_bwd", ctypes.byref(p), _ptr(q, BF16, "q"), _ptr(k, BF16, "k"),
          _ptr(v, BF16, "v"), _ptr(o_sparse, BF16, "o_sparse"), _ptr(lse_sparse, F32, "lse_sparse"),
          _ptr(o_full, BF16, "o_full"), _ptr(lse_full, F32, "lse_full"), _ptr(d_o, BF16, "d_o"),
          int(mode), float(alpha), _ptr(block_idx, I32, "block_idx"), _ptr(dq, BF16, "dq"),
          _ptr(dk, BF16, "dk"), _ptr(dv, BF16, "dv"), _ptr(workspace, None, "workspace"),
          int(ws_bytes), _stream(stream))


def ssa_sparse_attn_fwd_early_stop(p: SsaProblem, q, k, v, q_pooled, k_pooled, block_idx, tau: float,
                                   o, lse, visited=None, stream=None) -> None:
    """The sparse forward visiting the diagonal first, then the selected blocks
    by descending pooled score, each head's query segment stopping after the
    first block that adds less than tau of every row's accumulated mass;
    visited is [B, Hq, n]; see include/ssa.h."""
    sh = _shapes(p)
    for t, s, nm in ((q, "q", "q"), (k, "kv", "k"), (v, "kv", "v"), (q_pooled, "pooled", "q_pooled"),
                     (k_pooled, "pooled", "k_pooled"), (block_idx, "idx", "block_idx"), (o, "q", "o"),
                     (lse, "lse", "lse")):
        _numel_check(t, sh[s], nm)
    if visited is not None:
        B, Hkv, n, _ = sh["idx"]
        _numel_check(visited, (B, p.n_q_heads, n), "visited")
    _call("ssa_sparse_attn_fwd_early_stop", ctypes.byref(p), _ptr(q, BF16, "q"), _ptr(k, BF16, "k"),
          _ptr(v, BF16, "v"), _ptr(q_pooled, F32, "q_pooled"), _ptr(k_pooled, F32, "k_pooled"),
          _ptr(block_idx, I32, "block_idx"), float(tau), _ptr(o, BF16, "o"), _ptr(lse, F32, "lse"),
          _ptr(visited, I32, "visited"), _stream(stream))


def _mask_ptr(t, name: str) -> int:
    """Bit masks travel as int32 or uint32 tensors (the same 32 bits)."""
    if t is None or t.dtype not in (I32, getattr(torch, "uint32", I32)):
        raise ValueError(f"{name}: expected an int32 (or uint32) CUDA tensor")
    return _ptr(t, None, name)


def ssa_dash_route(p: SsaProblem, q, k_pooled, alpha: float, gamma: float, weights, mask,
                   stream=None) -> None:
    """DashAttention chunk routing: per-head alpha-entmax over the pooled chunk
    logits, averaged over the GQA group, and the bit-packed support; see
    include/ssa.h."""
    sh = _shapes(p)
    B, Hkv, n, _ = sh["idx"]
    for t, s, nm in ((q, sh["q"], "q"), (k_pooled, sh["pooled"], "k_pooled"), (weights, (B, Hkv, n, n), "weights"),
                     (mask, (B, Hkv, n, (n + 31) // 32), "mask")):
        _numel_check(t, s, nm)
    _call("ssa_dash_route", ctypes.byref(p), _ptr(q, BF16, "q"), _ptr(k_pooled, F32, "k_pooled"), float(alpha),
          float(gamma), _ptr(weights, F32, "weights"), _mask_ptr(mask, "mask"), _stream(stream))


def ssa_dash_attn_fwd(p: SsaProblem, q, k, v, weights, mask, sigma: float, o, lse, stream=None) -> None:
    """DashAttention's prior-induced sparse softmax over the routed chunks and
    the diagonal; see include/ssa.h."""
    sh = _shapes(p)
    B, Hkv, n, _ = sh["idx"]
    for t, s, nm in ((q, sh["q"], "q"), (k, sh["kv"], "k"), (v, sh["kv"], "v"), (weights, (B, Hkv, n, n), "weights"),
                     (mask, (B, Hkv, n, (n + 31) // 32), "mask"), (o, sh["q"], "o"), (lse, sh["lse"], "lse")):
        _numel_check(t, s, nm)
    _call("ssa_dash_attn_fwd", ctypes.byref(p), _ptr(q, BF16, "q"), _ptr(k, BF16, "k"), _ptr(v, BF16, "v"),
          _ptr(weights, F32, "weights"), _mask_ptr(mask, "mask"), float(sigma), _ptr(o, BF16, "o"),
          _ptr(lse, F32, "lse"), _stream(stream))


def _host_ptr(t, dtype, name: str) -> int:
    if t is None or t.is_cuda:
        raise ValueError(f"{name}: expected a host (CPU) tensor, page-locked for overlap")
    if not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name}: expected {dtype}, got {t.dtype}")
    return t.data_ptr()


def ssa_sparse_attn_fwd_host_workspace(p: SsaProblem) -> int:
    return int(lib().ssa_sparse_attn_fwd_host_workspace(ctypes.byref(p)))


def ssa_sparse_attn_fwd_host(p: SsaProblem, q, k, v, o, lse, workspace, ws_bytes: int, stream=None) -> None:
    """Pool, select and the sparse forward on host buffers, pipelined by
    (batch, KV head) so copies in, kernels and copies out overlap; see
    include/ssa.h."""
    sh = _shapes(p)
    for t, s, nm in ((q, sh["q"], "q"), (k, sh["kv"], "k"), (v, sh["kv"], "v"), (o, sh["q"], "o"),
                     (lse, sh["lse"], "lse")):
        _numel_check(t, s, nm)
    _call("ssa_sparse_attn_fwd_host", ctypes.byref(p), _host_ptr(q, BF16, "q"), _host_ptr(k, BF16, "k"),
          _host_ptr(v, BF16, "v"), _host_ptr(o, BF16, "o"), _host_ptr(lse, F32, "lse"),
          _ptr(workspace, None, "workspace"), int(ws_bytes), _stream(stream))


def ssa_decode_attn_workspace(p: SsaProblem) -> int:
    return int(lib().ssa_decode_attn_workspace(ctypes.byref(p)))


def ssa_decode_attn(p: SsaProblem, q, k_cache, v_cache, k_pooled, lengths, o, lse, block_idx,
                    workspace, ws_bytes: int, stream=None) -> None:
    """One decoding step against a KV cache (p.seq_len = cache capacity); see
    include/ssa.h.  block_idx may be None."""
    sh = _shapes(p)
    B, Hq, Hkv, D = p.batch, p.n_q_heads, p.n_kv_heads, p.head_dim
    for t, s, nm in ((q, (B, Hq, D), "q"), (k_cache, sh["kv"], "k_cache"), (v_cache, sh["kv"], "v_cache"),
                     (k_pooled, sh["pooled"], "k_pooled"), (lengths, (B,), "lengths"),
                     (o, (B, Hq, D), "o"), (lse, (B, Hq), "lse")):
        _numel_check(t, s, nm)
    if block_idx is not None:
        _numel_check(block_idx, (B, Hkv, p.top_k), "block_idx")
    _call("ssa_decode_attn", ctypes.byref(p), _ptr(q, BF16, "q"), _ptr(k_cache, BF16, "k_cache"),
          _ptr(v_cache, BF16, "v_cache"), _ptr(k_pooled, F32, "k_pooled"), _ptr(lengths, I32, "lengths"),
          _ptr(o, BF16, "o"), _ptr(lse, F32, "lse"), _ptr(block_idx, I32, "block_idx"),
          _ptr(workspace, None, "workspace"), int(ws_bytes), _stream(stream))


def ssa_sparse_attn_bwd_noalloc(p: SsaProblem, q, k, v, o, lse, d_o, block_idx, dq, dk, dv,
                                stream=None) -> None:
    """ssa_sparse_attn_bwd for callers that cannot allocate: the library's own
    fixed scratch (SSA_NOALLOC_SCRATCH_BYTES per device) replaces the
    workspace; calls that overlap on the GPU race on it."""
    sh = _shapes(p)
    for t, s, nm in ((q, "q", "q"), (k, "kv", "k"), (v, "kv", "v"), (o, "q", "o"),
                     (lse, "lse", "lse"), (d_o, "q", "d_o"), (block_idx, "idx", "block_idx"),
                     (dq, "q", "dq"), (dk, "kv", "dk"), (dv, "kv", "dv")):
        _numel_check(t, sh[s], nm)
    _call("ssa_sparse_attn_bwd_noalloc", ctypes.byref(p), _ptr(q, BF16, "q"), _ptr(k, BF16, "k"),
          _ptr(v, BF16, "v"), _ptr(o, BF16, "o"), _ptr(lse, F32, "lse"), _ptr(d_o, BF16, "d_o"),
          _ptr(block_idx, I32, "block_idx"), _ptr(dq, BF16, "dq"), _ptr(dk, BF16, "dk"),
          _ptr(dv, BF16, "dv"), _stream(stream))


def ssa_get_device_error(stream=None) -> int:
    """Status code (not raised): 0 OK, 4 a bounded device wait ran out."""
    return int(lib().ssa_get_device_error(_stream(stream)))


def ssa_get_device_error_site() -> int:
    return int(lib().ssa_get_device_error_site())


def ssa_debug_timeout_probe(timeout_us: int, stream=None) -> None:
    _call("ssa_debug_timeout_probe", int(timeout_us), _stream(stream))


def ssa_debug_exp2_poly(x: torch.Tensor, y: torch.Tensor, stream=None) -> None:
    """y = 2^x by the forward kernels' FMA-pipe polynomial (fp32 CUDA tensors)."""
    n = x.numel()
    if y.numel() != n:
        raise ValueError("x and y differ in size")
    _call("ssa_debug_exp2_poly", _ptr(x, F32, "x"), _ptr(y, F32, "y"), int(n), _stream(stream))


def ssa_status_string(status: int) -> str:
    return lib().ssa_status_string(int(status)).decode()


def ssa_launch_count() -> int:
    return int(lib().ssa_launch_count())
