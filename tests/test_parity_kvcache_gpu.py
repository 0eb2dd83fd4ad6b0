"""GPU parity of fa_fwd_kvcache: the new keys/values are appended to the caches
in place (checked bit for bit against the expected caches), then each
sequence's query rows attend to its own cached keys plus the new ones
(checked against the fp64 oracle run per sequence on exactly those keys).

Covers: ragged cache lengths from 0 to the full capacity, speculative steps
(several new rows), no append with given lengths, full caches (no lengths),
appends that overflow the capacity (rows dropped, key count clamped), more
query rows than keys (rows with no visible key), windows, GQA and MQA, every
head dim and the library's own split count.
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


def check_kvcache(B, Nq, Nk, n_new, Hq, Hkv, d, seqlens, causal=True, window=(-1, -1),
                  n_splits=0, seed=0):
    inp = make_inputs(B, Nq, Nk, Hq, Hkv, d, seed, with_dout=False)
    q, kc, vc = inp["q"], inp["k"], inp["v"]
    kn = vn = None
    if n_new:
        new = make_inputs(B, n_new, n_new, Hkv, Hkv, d, seed + 1, with_dout=False)
        kn, vn = new["k"], new["v"]
    # expected caches after the append
    kc_exp, vc_exp = kc.clone(), vc.clone()
    if n_new:
        for b in range(B):
            for t in range(n_new):
                dst = seqlens[b] + t
                if dst < Nk:
                    kc_exp[b, dst] = kn[b, t]
                    vc_exp[b, dst] = vn[b, t]
    dev = torch.device("cuda")
    qd, kcd, vcd = q.to(dev), kc.to(dev), vc.to(dev)
    knd = kn.to(dev) if kn is not None else None
    vnd = vn.to(dev) if vn is not None else None
    sl = torch.tensor(seqlens, dtype=torch.int32, device=dev) if seqlens is not None else None
    scale = 1.0 / math.sqrt(d)
    o, lse = fa.attention_forward_kvcache(qd, kcd, vcd, knd, vnd, sl, scale=scale, causal=causal,
                                          window=window, n_splits=n_splits)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status(None) == 0
    assert torch.equal(kcd.cpu(), kc_exp) and torch.equal(vcd.cpu(), vc_exp), "cache update"
    if sl is not None:
        assert sl.cpu().tolist() == list(seqlens), "cache_seqlens must not be modified"
    o, lse = o.float().cpu().numpy(), lse.cpu().numpy()
    what = "kvcache B%d Nq%d Nk%d new%d Hq%d Hkv%d d%d lens%s win%s" % (
        B, Nq, Nk, n_new, Hq, Hkv, d, seqlens, window)
    for b in range(B):
        L = Nk if seqlens is None else min(Nk, seqlens[b] + n_new)
        if L == 0:
            assert np.all(o[b] == 0.0) and np.all(np.isneginf(lse[b])), what
            continue
        f64 = lambda t: t[b:b + 1].double().numpy()
        o_ref, lse_ref = oracle.attn_fwd(f64(q), f64(kc_exp)[:, :L], f64(vc_exp)[:, :L],
                                         scale=scale, causal=causal, window=window)
        err = o_error(o[b:b + 1], o_ref)
        assert err <= TOL_BF16["o"], "%s batch %d: O max err %.3e" % (what, b, err)
        compare_lse(lse[b:b + 1], lse_ref, TOL_BF16["lse"], "%s batch %d" % (what, b))


def test_ragged_lengths_single_new_token():
    check_kvcache(5, 1, 5000, 1, 8, 2, 128, [0, 1, 2500, 4998, 4999], seed=11)


def test_speculative_step_gqa8_d64():
    check_kvcache(3, 4, 3000, 4, 16, 2, 64, [0, 1500, 2996], n_splits=3, seed=12)


def test_lengths_without_append_window_d256():
    check_kvcache(2, 2, 2000, 0, 4, 1, 256, [700, 1999], window=(200, 0), seed=13)


def test_full_caches_without_lengths():
    check_kvcache(2, 1, 4096, 0, 32, 8, 128, None, seed=14)


def test_append_past_the_capacity_is_dropped():
    check_kvcache(2, 3, 300, 3, 8, 2, 128, [298, 300], n_splits=2, seed=15)


def test_more_query_rows_than_keys():
    check_kvcache(2, 5, 1024, 2, 4, 4, 64, [0, 7], seed=16)


def test_long_ragged_batch_library_split():
    rng = np.random.default_rng(17)
    lens = rng.integers(0, 32768, 8).tolist()
    check_kvcache(8, 1, 32768, 1, 32, 8, 128, lens, seed=17)
