"""GPU parity of fa_fwd_varlen and fa_bwd_varlen (packed variable-length
sequences) against the fp64 oracle run sequence by sequence.

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
from parity_utils import TOL_BF16, ZERO_ABS, compare_lse, o_error, rel_fro
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


def check_varlen_bwd(lens_q, lens_k, Hq, Hkv, d, causal=False, window=(-1, -1), slack=0, seed=0):
    """Forward then backward through the C ABI; dQ, dK, dV of the covered rows
    against the oracle's per-sequence gradients, uncovered rows untouched,
    and the same bits on a second call."""
    cu_q = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    total_q, total_k = int(cu_q[-1]) + slack, int(cu_k[-1]) + slack
    inp = make_inputs(1, total_q, total_k, Hq, Hkv, d, seed)
    q, k, v, do = (inp[n][0] for n in ("q", "k", "v", "do"))
    dev = torch.device("cuda")
    qd, kd, vd, dod = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
    cq, ck = torch.from_numpy(cu_q).to(dev), torch.from_numpy(cu_k).to(dev)
    scale = 1.0 / math.sqrt(d)
    mq, mk = max(lens_q), max(lens_k)
    o, lse = fa.attention_forward_varlen(qd, kd, vd, cq, ck, mq, mk, scale=scale, causal=causal,
                                         window=window)
    grads = []
    for _ in range(2):
        dq = torch.full_like(qd, SENTINEL_O)
        dk = torch.full_like(kd, SENTINEL_O)
        dv = torch.full_like(vd, SENTINEL_O)
        fa.attention_backward_varlen(qd, kd, vd, o, lse, dod, cq, ck, mq, mk, scale=scale,
                                     causal=causal, window=window, dq=dq, dk=dk, dv=dv)
        torch.cuda.synchronize()
        grads.append([t.float().cpu().numpy() for t in (dq, dk, dv)])
    assert fa.fa_get_device_status(None) == 0
    for a, b in zip(grads[0], grads[1]):
        assert np.array_equal(a, b), "backward not deterministic"
    refs = oracle.attn_bwd_varlen(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                  do.double().numpy(), cu_q, cu_k, scale=scale, causal=causal,
                                  window=window)
    what = "varlen bwd q%s k%s Hq%d Hkv%d d%d causal%d win%s" % (lens_q, lens_k, Hq, Hkv, d,
                                                               causal, window)
    covered = (int(cu_q[-1]), int(cu_k[-1]), int(cu_k[-1]))
    for name, g, r, n in zip(("dq", "dk", "dv"), grads[0], refs, covered):
        assert np.all(g[n:] == SENTINEL_O), "%s: %s rows outside every sequence written" % (what, name)
        g, r = g[:n], r[:n]
        if not np.any(r):
            assert float(np.abs(g).max()) <= ZERO_ABS, "%s: %s should be ~0" % (what, name)
            continue
        e = rel_fro(g, r)
        assert e <= TOL_BF16["grad"], "%s: %s rel err %.3e" % (what, name, e)


def test_backward_lengths_around_the_tile_size_causal():
    lens = [1, 127, 128, 129, 300, 0, 513]
    check_varlen_bwd(lens, lens, 4, 2, 128, causal=True, slack=9, seed=41)


def test_backward_query_and_key_lengths_differ_window_d64():
    check_varlen_bwd([5, 200, 64, 1], [300, 200, 900, 2], 4, 4, 64, causal=True, window=(100, 0),
                     seed=42)


def test_backward_non_causal_d256():
    check_varlen_bwd([77, 256, 31], [77, 256, 31], 2, 1, 256, slack=50, seed=43)


def test_backward_mqa_window_both_sides():
    check_varlen_bwd([640, 33, 257], [700, 33, 300], 8, 1, 128, window=(64, 32), seed=44)
