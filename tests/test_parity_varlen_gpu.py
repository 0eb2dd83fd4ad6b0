"""GPU parity of fa_fwd_varlen (packed variable-length sequences) against the
fp64 oracle run sequence by sequence.

Lengths straddle the 128-row tiles (1, 127, 128, 129, ...), include empty
sequences, query and key lengths that differ per sequence (causal aligned
bottom-right per sequence), windows, GQA and MQA, every head dim, and rows
that no sequence covers (they must keep what the caller put there: the last
tile of a sequence is stored row by row, never over its neighbour).
"""
import math

import numpy as np
import pytest
import torch

import exact_io_aware_89_b200 as fa
import oracle
from parity_utils import TOL_BF16, compare_lse, o_error
from seeded_inputs import make_inputs

pytestmark = pytest.mark.gpu

SENTINEL_O, SENTINEL_LSE = 3.0, 7.0


@pytest.fixture(autouse=True)
def _need_cuda(cuda_ok):
    return cuda_ok


def check_varlen(lens_q, lens_k, Hq, Hkv, d, causal=False, window=(-1, -1), slack=0, seed=0):
    cu_q = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    total_q, total_k = int(cu_q[-1]) + slack, int(cu_k[-1]) + slack
    inp = make_inputs(1, total_q, total_k, Hq, Hkv, d, seed, with_dout=False)
    q, k, v = (inp[n][0] for n in ("q", "k", "v"))
    dev = torch.device("cuda")
    o = torch.full((total_q, Hq, d), SENTINEL_O, dtype=torch.bfloat16, device=dev)
    lse = torch.full((Hq, total_q), SENTINEL_LSE, dtype=torch.float32, device=dev)
    scale = 1.0 / math.sqrt(d)
    fa.attention_forward_varlen(q.to(dev), k.to(dev), v.to(dev),
                                torch.from_numpy(cu_q).to(dev), torch.from_numpy(cu_k).to(dev),
                                max(lens_q), max(lens_k), scale=scale, causal=causal,
                                window=window, out=o, lse=lse)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status(None) == 0
    o, lse = o.float().cpu().numpy(), lse.cpu().numpy()
    o_ref, lse_ref = oracle.attn_fwd_varlen(q.double().numpy(), k.double().numpy(),
                                            v.double().numpy(), cu_q, cu_k, scale=scale,
                                            causal=causal, window=window)
    what = "varlen q%s k%s Hq%d Hkv%d d%d causal%d win%s" % (lens_q, lens_k, Hq, Hkv, d, causal,
                                                           window)
    covered = int(cu_q[-1])
    err = o_error(o[:covered], o_ref[:covered])
    assert err <= TOL_BF16["o"], "%s: O max err %.3e" % (what, err)
    compare_lse(lse[:, :covered], lse_ref[:, :covered], TOL_BF16["lse"], what)
    assert np.all(o[covered:] == SENTINEL_O) and np.all(lse[:, covered:] == SENTINEL_LSE), \
        "%s: rows outside every sequence were written" % what


def test_lengths_around_the_tile_size_causal():
    lens = [1, 127, 128, 129, 300, 0, 513]
    check_varlen(lens, lens, 4, 2, 128, causal=True, seed=31)


def test_query_and_key_lengths_differ_with_window_d64():
    check_varlen([5, 200, 64, 1], [300, 200, 900, 2], 4, 4, 64, causal=True, window=(100, 0),
                 seed=32)


def test_non_causal_d256_with_uncovered_rows():
    check_varlen([77, 256, 31], [77, 256, 31], 2, 1, 256, slack=50, seed=33)


def test_mqa_window_both_sides():
    check_varlen([640, 33, 257], [700, 33, 300], 8, 1, 128, window=(64, 32), seed=34)


def test_many_short_sequences():
    rng = np.random.default_rng(35)
    lens = rng.integers(1, 200, 40).tolist()
    check_varlen(lens, lens, 4, 1, 128, causal=True, slack=7, seed=35)
