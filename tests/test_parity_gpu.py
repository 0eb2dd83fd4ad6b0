"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs, at sizes the oracle finishes in seconds that span several
tiles and a ragged tail, plus the edge cases the method has (empty rows,
Nq != Nk, single rows, MQA, windows, peaked softmax)."""
import numpy as np
import pytest
import torch

import exact_io_aware_89_b200 as fa
from parity_utils import gpu_run, run_case, run_stress_case
from seeded_inputs import make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda(cuda_ok):
    return cuda_ok


# ---------------------------------------------------------------- tiny workload

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_tiny_workload(causal, dtype):
    """B=1, H=2, N=128, d=64, fp32 and bf16, causal and not, fwd + bwd."""
    run_case(1, 128, 128, 2, 2, 64, causal=causal, seed=1001, dtype=dtype)


# ------------------------------------------------- multi-tile with ragged tails

MASKS = [(False, (-1, -1)), (True, (-1, -1)), (True, (70, -1)), (False, (33, 17))]


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal,window", MASKS)
def test_ragged_gqa(d, causal, window):
    """Nq = Nk = 333 (three query tiles, ragged), GQA 4:2, every mask kind."""
    run_case(2, 333, 333, 4, 2, d, causal=causal, window=window, seed=17)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_long_causal_single_head_pair(d):
    """Several CTAs per head and a ragged last key tile."""
    run_case(1, 1100, 1100, 2, 2, d, causal=True, seed=23)


# ------------------------------------------------------------ Nq != Nk, edges

@pytest.mark.parametrize("Nq,Nk,causal,window", [
    (200, 517, True, (-1, -1)),     # bottom-right causal, more keys than queries
    (517, 200, True, (-1, -1)),     # early query rows see no key at all
    (129, 1000, False, (100, 20)),  # band, Nq < Nk
    (1, 300, True, (-1, -1)),       # single query row (decode shape)
    (1, 1, False, (-1, -1)),        # single element
    (300, 1, False, (-1, -1)),      # single key
    (256, 256, False, (0, 0)),      # each row sees exactly its diagonal key
])
@pytest.mark.parametrize("d", [64, 128])
def test_shapes_and_edges(Nq, Nk, causal, window, d):
    run_case(1, Nq, Nk, 2, 1, d, causal=causal, window=window, seed=29)


def test_mqa_many_heads():
    """Hkv = 1 shared by 8 query heads (dK/dV summed over 8 heads)."""
    run_case(1, 300, 300, 8, 1, 128, causal=True, seed=31)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_peaked_softmax(d):
    """Q scaled by 8: rows dominated by a few keys; exercises the running-max
    rescale of O and l.  Outside the N(0,1) regime of the stated tolerances, so
    it is held to twice the error of a bf16 baseline implementation."""
    run_stress_case(1, 400, 400, 2, 2, d, causal=False, seed=37, scale_q=8.0)
    run_stress_case(1, 333, 333, 4, 2, d, causal=True, seed=38, scale_q=8.0)


def test_fp32_path_gqa_window():
    run_case(2, 150, 170, 4, 2, 96, causal=True, window=(40, -1), seed=41, dtype="fp32")


# ------------------------------------------------------------- determinism

def test_backward_is_deterministic():
    """Same inputs -> the same dQ, dK, dV bits on repeated calls."""
    inp = make_inputs(1, 700, 700, 4, 2, 128, seed=43)
    a = gpu_run(inp, 128 ** -0.5, True, (-1, -1))
    b = gpu_run(inp, 128 ** -0.5, True, (-1, -1))
    for n in ("o", "lse", "dq", "dk", "dv"):
        assert np.array_equal(a[n], b[n]), n


@pytest.mark.parametrize("d", [64, 128, 256])
def test_repeated_calls_are_bit_identical(d):
    """Ten forward + backward calls on the same inputs give identical bits: an
    intermittent race in a pipeline (a barrier phase taken too early) shows up
    here as a mismatch even when one call happens to be right."""
    inp = make_inputs(1, 333, 333, 4, 2, d, seed=47, scale_q=8.0)
    first = gpu_run(inp, d ** -0.5, True, (-1, -1))
    for _ in range(9):
        again = gpu_run(inp, d ** -0.5, True, (-1, -1))
        for n in ("o", "lse", "dq", "dk", "dv"):
            assert np.array_equal(first[n], again[n]), n
