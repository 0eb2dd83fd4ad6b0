"""GPU parity of the split-KV forward (fa_fwd_splitkv: few query rows against
many keys, the keys split across CTAs and merged by their log-sum-exp) against
the fp64 oracle on the same seeded, bf16-rounded inputs.

The cases cover every packing of the query rows (1 to 128 rows per tile, the
rows stored 4, 2 or 1 times in tensor memory), every head dim, ragged key
counts, splits that get no key tile, query tiles past Nq, rows that see no key
at all (Nq > Nk under the bottom-right causal mask), windows on both sides,
and the library's own choice of split count.  Tolerances are those of the
forward pass: O max-abs <= 1e-2, LSE max-abs <= 1e-3.
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


@pytest.fixture(autouse=True)
def _need_cuda(cuda_ok):
    return cuda_ok


def run_splitkv(inp, scale, causal, window, n_splits):
    dev = torch.device("cuda")
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    o, lse = fa.attention_forward_splitkv(q, k, v, scale=scale, causal=causal, window=window,
                                          n_splits=n_splits)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status(None) == 0
    return o.float().cpu().numpy(), lse.cpu().numpy()


def check_case(B, Nq, Nk, Hq, Hkv, d, causal, window, n_splits, seed):
    inp = make_inputs(B, Nq, Nk, Hq, Hkv, d, seed, with_dout=False)
    scale = 1.0 / math.sqrt(d)
    o, lse = run_splitkv(inp, scale, causal, window, n_splits)
    f64 = {n: t.double().numpy() for n, t in inp.items()}
    o_ref, lse_ref = oracle.attn_fwd(f64["q"], f64["k"], f64["v"], scale=scale, causal=causal,
                                     window=window)
    what = "splitkv B%d Nq%d Nk%d Hq%d Hkv%d d%d causal%d win%s splits%d" % (
        B, Nq, Nk, Hq, Hkv, d, causal, window, n_splits)
    err = o_error(o, o_ref)
    assert err <= TOL_BF16["o"], "%s: O max err %.3e" % (what, err)
    compare_lse(lse, lse_ref, TOL_BF16["lse"], what)
    return o, lse


# (B, Nq, Nk, Hq, Hkv, d, causal, window, n_splits)
CASES = [
    (2, 1, 1000, 8, 2, 128, False, (-1, -1), 0),    # ragged Nk, library's split count
    (2, 1, 1000, 8, 2, 128, False, (-1, -1), 1),    # no split: output written by the main kernel
    (2, 1, 1000, 8, 2, 128, False, (-1, -1), 3),
    (1, 1, 700, 4, 4, 64, False, (-1, -1), 16),     # MHA; more splits asked for than its 6 key tiles
    (2, 2, 1500, 16, 1, 64, True, (-1, -1), 5),     # 32 packed rows: 4 copies
    (1, 3, 1200, 16, 1, 256, True, (300, 0), 4),    # 48 rows: 2 copies; window; d 256
    (1, 3, 2000, 32, 1, 128, True, (-1, -1), 0),    # MQA, 96 rows: 1 copy
    (1, 16, 2048, 8, 1, 128, False, (500, 100), 0),  # 128 rows, window on both sides
    (1, 40, 3000, 8, 2, 128, True, (-1, -1), 2),    # 2 query tiles, the last one ragged
    (2, 4, 3, 4, 2, 64, True, (-1, -1), 1),         # Nq > Nk: rows with no visible key
    (1, 1, 5000, 2, 2, 256, False, (-1, -1), 0),    # one packed row, d 256
    (3, 1, 4100, 4, 1, 64, False, (2000, 0), 7),    # window narrower than the keys
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%d_Nq%d_Nk%d_Hq%d_Hkv%d_d%d_c%d_w%d_%d_s%d" % (
    c[0], c[1], c[2], c[3], c[4], c[5], c[6], c[7][0], c[7][1], c[8]))
def test_splitkv_matches_oracle(case):
    B, Nq, Nk, Hq, Hkv, d, causal, window, n_splits = case
    check_case(B, Nq, Nk, Hq, Hkv, d, causal, window, n_splits, seed=hash(case) % 1000)


def test_splitkv_no_visible_key_rows_are_zero():
    """Nq > Nk, causal (bottom-right): the first Nq - Nk rows see no key."""
    o, lse = check_case(1, 6, 2, 4, 2, 128, True, (-1, -1), 1, seed=5)
    assert np.all(np.isneginf(lse[:, :, :4]))
    assert np.all(o[:, :4] == 0.0)


@pytest.mark.parametrize("n_splits", [0, 1, 6])
def test_splitkv_is_deterministic(n_splits):
    inp = make_inputs(2, 2, 3000, 16, 2, 128, 77, with_dout=False)
    a = run_splitkv(inp, 0.088, True, (-1, -1), n_splits)
    b = run_splitkv(inp, 0.088, True, (-1, -1), n_splits)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_splitkv_decode_workload_full():
    """Decoding step of a GQA model: B8, Hq32, Hkv8, one query row, 32768
    cached keys, d128, every row against the oracle."""
    check_case(8, 1, 32768, 32, 8, 128, True, (-1, -1), 0, seed=2001)


def test_splitkv_long_context_single_sequence():
    """One sequence with 131072 cached keys, GQA 32:8 (the keys split about
    18 ways per key/value head), every row against the oracle."""
    check_case(1, 1, 131072, 32, 8, 128, True, (-1, -1), 0, seed=2002)


def test_splitkv_workspace_contents_are_ignored():
    """The per-unit counters live in the caller's workspace: a workspace full of
    arbitrary bytes, reused across calls, and replayed inside a CUDA graph
    gives the same bits every time."""
    B, Nq, Nk, Hq, Hkv, d = 2, 1, 6000, 8, 2, 128
    inp = make_inputs(B, Nq, Nk, Hq, Hkv, d, 91, with_dout=False)
    dev = torch.device("cuda")
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    wsb = fa.fa_fwd_splitkv_workspace_size(B, Nq, Nk, Hq, Hkv, d, 1, -1, -1, 5)
    assert wsb > 0
    ws = torch.full((wsb,), 0xFF, dtype=torch.uint8, device=dev)
    o, lse = fa.attention_forward_splitkv(q, k, v, causal=True, n_splits=5, workspace=ws)
    ref_o, ref_lse = o.clone(), lse.clone()
    for _ in range(3):
        o2, lse2 = fa.attention_forward_splitkv(q, k, v, causal=True, n_splits=5, workspace=ws)
        assert torch.equal(o2, ref_o) and torch.equal(lse2, ref_lse)
    ws.random_(0, 256)
    o3 = torch.empty_like(ref_o)
    lse3 = torch.empty_like(ref_lse)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fa.attention_forward_splitkv(q, k, v, causal=True, n_splits=5, out=o3, lse=lse3, workspace=ws)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            fa.attention_forward_splitkv(q, k, v, causal=True, n_splits=5, out=o3, lse=lse3,
                                         workspace=ws)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(3):
        o3.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(o3, ref_o) and torch.equal(lse3, ref_lse)
    del g
    assert fa.fa_get_device_status(None) == 0
    f64 = {n: t.double().numpy() for n, t in inp.items()}
    o_ref, _ = oracle.attn_fwd(f64["q"], f64["k"], f64["v"], scale=1.0 / math.sqrt(d), causal=True)
    assert o_error(ref_o.float().cpu().numpy(), o_ref) <= TOL_BF16["o"]
