"""The FMA-pipe exp2 polynomial the forward kernels use for part of the
softmax exponentials, checked against CUDA's exp2f (through torch.exp2) and
against exact powers of two in fp64."""
import numpy as np
import pytest
import torch

import block_sparse_attention_21_b200 as ssa

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from block_sparse_attention_21_b200 import build
    build.build()
    ssa.lib()


def _poly(x):
    xd = torch.as_tensor(x, dtype=torch.float32, device="cuda")
    y = torch.empty_like(xd)
    ssa.ssa_debug_exp2_poly(xd, y)
    torch.cuda.synchronize()
    return xd, y


def test_relative_error_bound_over_the_softmax_range():
    rng = np.random.Generator(np.random.PCG64(11))
    x = np.concatenate([np.linspace(-125.0, 64.0, 400001), rng.uniform(-30.0, 8.0, 200001),
                        np.arange(-125, 65, dtype=np.float64) + 0.5,
                        np.arange(-125, 65, dtype=np.float64)]).astype(np.float32)
    xd, y = _poly(x)
    exact = np.exp2(x.astype(np.float64))
    rel = np.abs(y.cpu().numpy().astype(np.float64) / exact - 1.0)
    assert rel.max() <= 8e-5, rel.max()
    ref = torch.exp2(xd)  # CUDA exp2f
    rel_cuda = ((y.double() - ref.double()).abs() / ref.double()).max().item()
    assert rel_cuda <= 8e-5


def test_integers_hit_the_exponent_exactly_enough_and_small_inputs_clamp():
    x = np.arange(-125, 65, dtype=np.float32)
    _, y = _poly(x)
    rel = np.abs(y.cpu().numpy().astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= 8e-5
    _, y = _poly(np.array([-126.0, -300.0, -np.inf, -1e30], dtype=np.float32))
    assert torch.allclose(y, torch.full_like(y, 2.0 ** -125), rtol=1e-4, atol=0)


def test_odd_length_and_empty():
    _, y = _poly(np.array([0.0, 1.0, -1.0], dtype=np.float32))
    assert np.allclose(y.cpu().numpy(), [1.0, 2.0, 0.5], rtol=1e-4)
    x = torch.empty(0, device="cuda")
    ssa.ssa_debug_exp2_poly(x, torch.empty_like(x))
