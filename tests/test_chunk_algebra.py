"""The chunk = frame decomposition the kernels use, checked against the fp64
oracle on the CPU (before any kernel runs), including the bf16 rounding
points of the tensor-core path at full frame size."""
import numpy as np
import pytest

import oracle
from chunk_model import chunk_forward
from gated_deltanet_linear_chunkwise_b200 import workloads as W


def rel(x, ref):
    return float(np.abs(x - ref).max() / np.abs(ref).max())


@pytest.mark.parametrize("L,block", [(1, 32), (16, 32), (64, 32), (100, 32), (64, 16), (128, 128)])
@pytest.mark.parametrize("regime", ["lit", "slow"])
def test_chunk_algebra_exact(L, block, regime):
    inp = W.draw(2, 2, 3 * L, 16, 24, frame_len=L, seed=1, regime=regime, dtype="f32", state_std=0.3)
    o, S = chunk_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], inp["S_in"], L, block)
    o_ref, S_ref = oracle.token_recurrence(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], inp["S_in"])
    assert rel(o, o_ref) < 1e-10
    assert rel(S, S_ref) < 1e-10


def test_chunk_algebra_diag_inverse_and_reset():
    inp = W.draw(1, 2, 2 * 96, 16, 16, frame_len=96, seed=2, regime="slow", dtype="f32", state_std=0.3)
    inp["alpha"][0, 40] = 0.0
    o, S = chunk_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], inp["S_in"], 96, 32,
                         diag_inverse=True)
    o_ref, S_ref = oracle.token_recurrence(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], inp["S_in"])
    assert rel(o, o_ref) < 1e-9
    assert rel(S, S_ref) < 1e-9


@pytest.mark.slow
@pytest.mark.parametrize("regime", ["lit", "slow"])
def test_bf16_rounding_budget_full_frame(regime):
    """Two 880-token frames at d = 112 with every tensor-core operand rounded
    to bf16 (fp32/fp64 accumulation): the error (about 5e-3) stays at half
    the 2e-2 bar or below."""
    inp = W.draw(1, 1, 2 * 880, 112, 112, frame_len=880, seed=1001, regime=regime, dtype="bf16", state_std=0.02)
    o, S = chunk_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], inp["S_in"], 880, 128,
                         diag_inverse=True, bf16=True)
    o_ref, S_ref = oracle.token_recurrence(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], inp["S_in"])
    assert rel(o, o_ref) < 1e-2
    assert rel(S, S_ref) < 1e-2
