"""The chunk algorithm of the CUDA path, restated in numpy (tests/emu_chunk.py),
against the token-by-token oracle on the CPU: exact in fp64 on both the fast
(chunk-boundary pivot) and the slow (term-by-term decay) path, for ragged
chunks, fast decays and resets; and within the bf16 tolerance when every
tensor-core operand is rounded to bfloat16 where the kernels round it."""
import numpy as np
import pytest

import emu_chunk as E
import oracle
from gated_delta_rule_gdn2_b200.inputs import make_inputs


def _args(x):
    return [x[n] for n in ("q", "k", "v", "log_alpha", "b", "w")] + [x["S0"]]


@pytest.mark.parametrize("T", [1, 63, 64, 65, 200])
@pytest.mark.parametrize("slow", [False, True])
def test_chunk_algebra_exact(T, slow):
    x = make_inputs(1, T, 2, 64, 64, seed=T, dtype="fp32")
    o, S = oracle.fwd(*_args(x))
    oe, Se = E.chunk_fwd(*_args(x), force_slow=slow)
    np.testing.assert_allclose(oe, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Se, S, rtol=0, atol=1e-12)


def test_chunk_algebra_guard_and_reset():
    x = make_inputs(1, 150, 1, 64, 64, seed=7, dtype="fp32")
    la = x["log_alpha"]
    la[0, 70:76, 0, :4] = -40.0  # one chunk spans e^-240 in four channels: slow path
    o, S = oracle.fwd(*_args(x))
    oe, Se = E.chunk_fwd(*_args(x))
    np.testing.assert_allclose(oe, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Se, S, rtol=0, atol=1e-12)
    la[:] = -800.0
    o, S = oracle.fwd(*_args(x))
    oe, Se = E.chunk_fwd(*_args(x))
    np.testing.assert_allclose(oe, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Se, S, rtol=0, atol=1e-12)


def test_bf16_error_budget():
    x = make_inputs(1, 512, 2, 128, 128, seed=1001, dtype="bf16")
    o, S = oracle.fwd(*_args(x))
    oe, Se = E.chunk_fwd(*_args(x), bf16=True)
    rel = lambda a, b: np.linalg.norm(a - b) / np.linalg.norm(b)
    assert rel(oe, o) < 5e-3 and rel(Se, S) < 5e-3
