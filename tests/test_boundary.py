"""The C ABI boundary, without a GPU: the library loads, exports every symbol
include/ssa.h declares, and rejects bad arguments on the host before launching
anything."""
import ctypes
import os
import re

import pytest

import block_sparse_attention_21_b200 as ssa
from block_sparse_attention_21_b200 import build as ssa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssa.h")

INVALID, UNSUPPORTED, WORKSPACE = 1, 2, 5
FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails first


@pytest.fixture(scope="module")
def lib():
    ssa_build.build()
    return ssa.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ssa_[a-z0-9_]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert sorted(ssa.EXPORTED) == declared_functions()


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code, name in ssa._binding.STATUS_NAMES.items():
        assert ssa.ssa_status_string(code) == name


def _p(**kw):
    base = dict(batch=1, seq_len=1024, n_q_heads=8, n_kv_heads=2, head_dim=64, top_k=4)
    base.update(kw)
    return ssa.problem(**base)


BAD_PROBLEMS = [
    (dict(batch=0), INVALID),               # empty batch
    (dict(seq_len=0), INVALID),             # empty sequence
    (dict(seq_len=1000), INVALID),          # not a multiple of the block
    (dict(n_q_heads=6, n_kv_heads=4), INVALID),
    (dict(top_k=0), INVALID),
    (dict(head_dim=96), UNSUPPORTED),
    (dict(block_size=128), UNSUPPORTED),
    (dict(causal=0), UNSUPPORTED),
    (dict(n_q_heads=2, n_kv_heads=2), UNSUPPORTED),   # G = 1
    (dict(n_q_heads=64, n_kv_heads=2), UNSUPPORTED),  # G = 32
    (dict(seq_len=1048576), UNSUPPORTED),
    (dict(softmax_scale=float("nan")), INVALID),
]


@pytest.mark.parametrize("kw,code", BAD_PROBLEMS)
def test_bad_problem_is_rejected_by_every_entry_point(lib, kw, code):
    p = ctypes.byref(_p(**kw))
    f = FAKE
    assert lib.ssa_block_pool(p, f, f, f, f, None) == code
    assert lib.ssa_block_select(p, f, f, f, None) == code
    assert lib.ssa_sparse_attn_fwd(p, f, f, f, f, f, f, None) == code
    assert lib.ssa_full_attn_fwd_with_mass(p, f, f, f, f, f, f, f, f, f, None) == code
    assert lib.ssa_sparse_attn_bwd(p, f, f, f, f, f, f, f, f, f, f, f, 1 << 30, None) == code
    assert lib.ssa_sparse_attn_bwd_workspace(p) == 0
    assert lib.ssa_alignment_bwd(p, f, f, f, f, f, f, f, f, 0, 1.0, f, f, f, f, f, 1 << 30, None) == code
    assert lib.ssa_alignment_bwd_workspace(p) == 0
    assert lib.ssa_decode_attn(p, f, f, f, f, f, f, f, None, f, 1 << 30, None) == code
    assert lib.ssa_decode_attn_workspace(p) == 0
    assert lib.ssa_sparse_attn_fwd_early_stop(p, f, f, f, f, f, f, 0.1, f, f, None, None) == code
    assert lib.ssa_dash_route(p, f, f, 1.5, 1.0, f, f, None) == code
    assert lib.ssa_dash_attn_fwd(p, f, f, f, f, f, 1.0, f, f, None) == code
    assert lib.ssa_sparse_attn_fwd_host(p, f, f, f, f, f, f, 1 << 30, None) == code
    assert lib.ssa_sparse_attn_fwd_host_workspace(p) == 0


def test_null_problem(lib):
    assert lib.ssa_sparse_attn_fwd(None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None) == INVALID


def test_null_and_misaligned_pointers(lib):
    p = ctypes.byref(_p())
    f = FAKE
    assert lib.ssa_sparse_attn_fwd(p, None, f, f, f, f, f, None) == INVALID
    assert lib.ssa_sparse_attn_fwd(p, f, f, f, f, f + 2, f, None) == INVALID
    assert lib.ssa_block_pool(p, f, f, f, None, None) == INVALID   # q without q_pooled
    assert lib.ssa_block_select(p, f, None, f, None) == INVALID
    assert lib.ssa_full_attn_fwd_with_mass(p, f, f, f, f, f, f, f, f, None, None) == INVALID


def test_backward_workspace_is_checked_before_launch(lib):
    p = ctypes.byref(_p())
    need = lib.ssa_sparse_attn_bwd_workspace(p)
    f = FAKE
    args = [p] + [f] * 10
    assert lib.ssa_sparse_attn_bwd(*args, None, need, None) == WORKSPACE
    if need > 0:
        assert lib.ssa_sparse_attn_bwd(*args, f, need - 1, None) == WORKSPACE
    assert lib.ssa_sparse_attn_bwd(*args, f + 16, need, None) == WORKSPACE   # not 256-aligned


def test_timeout_probe_rejects_bad_limit(lib):
    assert lib.ssa_debug_timeout_probe(0, None) == INVALID


def test_alignment_backward_arguments_are_checked_before_launch(lib):
    p = ctypes.byref(_p())
    f = FAKE
    ws = lib.ssa_alignment_bwd_workspace(p)
    assert ws > lib.ssa_sparse_attn_bwd_workspace(p) > 0
    assert lib.ssa_alignment_bwd(p, f, f, f, f, f, f, f, f, 2, 1.0, f, f, f, f, f, ws, None) == INVALID
    assert lib.ssa_alignment_bwd(p, f, f, f, f, f, f, f, f, 0, float("inf"), f, f, f, f, f, ws, None) == INVALID
    assert lib.ssa_alignment_bwd(p, f, f, f, f, f, f, f, f, 0, 1.0, f, f, f, f, f, ws - 1, None) == WORKSPACE
    assert lib.ssa_alignment_bwd(p, f, f, f, f, f, f, f, f, 0, 1.0, f, f, f, f, None, ws, None) == WORKSPACE
    assert lib.ssa_alignment_bwd(p, f, f, f, f, None, f, f, f, 0, 1.0, f, f, f, f, f, ws, None) == INVALID


def test_decode_arguments_are_checked_before_launch(lib):
    p = ctypes.byref(_p())
    f = FAKE
    # the selection and the partial softmax states stay on chip: no workspace
    assert lib.ssa_decode_attn_workspace(p) == 0
    assert lib.ssa_decode_attn(p, f, f, f, f, None, f, f, None, None, 0, None) == INVALID
    assert lib.ssa_decode_attn(p, f, f, f, f, f, f, f, f + 4, None, 0, None) == INVALID
    assert lib.ssa_decode_attn(p, f, f, f, f, f, f, f + 4, None, None, 0, None) == INVALID


def test_early_stop_arguments_are_checked_before_launch(lib):
    p = ctypes.byref(_p())
    f = FAKE
    assert lib.ssa_sparse_attn_fwd_early_stop(p, f, f, f, f, f, f, -0.1, f, f, None, None) == INVALID
    assert lib.ssa_sparse_attn_fwd_early_stop(p, f, f, f, f, f, f, float("nan"), f, f, None, None) == INVALID
    assert lib.ssa_sparse_attn_fwd_early_stop(p, f, f, f, None, f, f, 0.1, f, f, None, None) == INVALID
    big = ctypes.byref(_p(top_k=257))
    assert lib.ssa_sparse_attn_fwd_early_stop(big, f, f, f, f, f, f, 0.1, f, f, None, None) == UNSUPPORTED


def test_dash_arguments_are_checked_before_launch(lib):
    p = ctypes.byref(_p())
    f = FAKE
    for alpha in (1.0, 0.5, 4.5, float("nan"), float("inf")):
        assert lib.ssa_dash_route(p, f, f, alpha, 1.0, f, f, None) == INVALID
    for gamma in (0.0, -1.0, float("nan"), float("inf")):
        assert lib.ssa_dash_route(p, f, f, 1.5, gamma, f, f, None) == INVALID
    assert lib.ssa_dash_route(p, None, f, 1.5, 1.0, f, f, None) == INVALID
    assert lib.ssa_dash_route(p, f, f, 1.5, 1.0, f, f + 4, None) == INVALID
    for sigma in (-0.1, float("nan"), float("inf")):
        assert lib.ssa_dash_attn_fwd(p, f, f, f, f, f, sigma, f, f, None) == INVALID
    assert lib.ssa_dash_attn_fwd(p, f, f, f, None, f, 1.0, f, f, None) == INVALID
    # more than 1024 chunks: the routed list of a query block no longer fits
    big = ctypes.byref(_p(seq_len=65536 + 64))
    assert lib.ssa_dash_route(big, f, f, 1.5, 1.0, f, f, None) == UNSUPPORTED
    assert lib.ssa_dash_attn_fwd(big, f, f, f, f, f, 1.0, f, f, None) == UNSUPPORTED


def test_host_buffer_forward_checks_pointers_and_workspace_before_any_copy(lib):
    p = ctypes.byref(_p())
    f = FAKE
    need = lib.ssa_sparse_attn_fwd_host_workspace(p)
    assert need > 0
    assert lib.ssa_sparse_attn_fwd_host(p, None, f, f, f, f, f, need, None) == INVALID
    assert lib.ssa_sparse_attn_fwd_host(p, f, f, f, f, None, f, need, None) == INVALID
    assert lib.ssa_sparse_attn_fwd_host(p, f, f, f, f, f, None, need, None) == WORKSPACE
    assert lib.ssa_sparse_attn_fwd_host(p, f, f, f, f, f, f, need - 1, None) == WORKSPACE
    assert lib.ssa_sparse_attn_fwd_host(p, f, f, f, f, f, f + 16, need, None) == WORKSPACE   # not 256-aligned
