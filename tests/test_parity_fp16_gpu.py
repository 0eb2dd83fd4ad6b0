"""GPU parity of the fp16 entry points against the fp64 oracle on the same
seeded inputs rounded to fp16: the dense forward and backward (every head
dim, ragged tails, GQA, causal and window), packed sequences, the split-KV
decode path and the KV cache.  The bf16 tolerances apply; the O check allows
fp16's own output rounding (|O| * 2^-11)."""
import math

import numpy as np
import pytest
import torch

import exact_io_aware_89_b200 as fa
import oracle
from parity_utils import TOL_BF16, compare_lse, o_error, rel_fro, run_case
from seeded_inputs import make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda(cuda_ok):
    return cuda_ok


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal,window", [(True, (-1, -1)), (False, (33, 17))])
def test_dense_fwd_bwd_fp16(d, causal, window):
    run_case(2, 333, 333, 4, 2, d, causal=causal, window=window, seed=51, dtype="fp16")


def test_dense_fp16_nq_ne_nk():
    run_case(1, 200, 700, 8, 1, 128, causal=True, seed=52, dtype="fp16")


def test_varlen_fwd_bwd_fp16():
    lens_q, lens_k = [130, 1, 257, 64], [300, 5, 257, 64]
    cu_q = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    T, Tk, Hq, Hkv, d = int(cu_q[-1]), int(cu_k[-1]), 4, 2, 128
    inp = make_inputs(1, T, Tk, Hq, Hkv, d, 53, dtype="fp16")
    q, k, v, do = (inp[n][0] for n in ("q", "k", "v", "do"))
    dev = torch.device("cuda")
    qd, kd, vd, dod = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
    cq, ck = torch.from_numpy(cu_q).to(dev), torch.from_numpy(cu_k).to(dev)
    scale = 1.0 / math.sqrt(d)
    o, lse = fa.attention_forward_varlen(qd, kd, vd, cq, ck, max(lens_q), max(lens_k), scale=scale,
                                         causal=True)
    assert o.dtype == torch.float16
    dq, dk, dv = fa.attention_backward_varlen(qd, kd, vd, o, lse, dod, cq, ck, max(lens_q),
                                              max(lens_k), scale=scale, causal=True)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status(None) == 0
    f64 = lambda t: t.double().numpy()
    o_ref, lse_ref = oracle.attn_fwd_varlen(f64(q), f64(k), f64(v), cu_q, cu_k, scale=scale,
                                            causal=True)
    assert o_error(o.float().cpu().numpy(), o_ref, "fp16") <= TOL_BF16["o"]
    compare_lse(lse.cpu().numpy(), lse_ref, TOL_BF16["lse"], "varlen fp16")
    refs = oracle.attn_bwd_varlen(f64(q), f64(k), f64(v), f64(do), cu_q, cu_k, scale=scale,
                                  causal=True)
    for name, g, r in zip(("dq", "dk", "dv"), (dq, dk, dv), refs):
        e = rel_fro(g.float().cpu().numpy(), r)
        assert e <= TOL_BF16["grad"], "varlen fp16 %s rel err %.3e" % (name, e)


@pytest.mark.parametrize("n_splits", [0, 1, 5])
def test_splitkv_fp16(n_splits):
    B, Nq, Nk, Hq, Hkv, d = 2, 2, 3000, 16, 2, 128
    inp = make_inputs(B, Nq, Nk, Hq, Hkv, d, 54, dtype="fp16", with_dout=False)
    dev = torch.device("cuda")
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    o, lse = fa.attention_forward_splitkv(q, k, v, causal=True, n_splits=n_splits)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status(None) == 0
    f64 = {n: t.double().numpy() for n, t in inp.items()}
    o_ref, lse_ref = oracle.attn_fwd(f64["q"], f64["k"], f64["v"], scale=1 / math.sqrt(d),
                                     causal=True)
    assert o_error(o.float().cpu().numpy(), o_ref, "fp16") <= TOL_BF16["o"]
    compare_lse(lse.cpu().numpy(), lse_ref, TOL_BF16["lse"], "splitkv fp16")


def test_kvcache_fp16_append_and_ragged_lengths():
    B, Nq, Nk, Hq, Hkv, d = 3, 1, 2048, 8, 2, 64
    lens = [0, 700, 2047]
    inp = make_inputs(B, Nq, Nk, Hq, Hkv, d, 55, dtype="fp16", with_dout=False)
    new = make_inputs(B, 1, 1, Hkv, Hkv, d, 56, dtype="fp16", with_dout=False)
    dev = torch.device("cuda")
    q, kc, vc = (inp[n].to(dev) for n in ("q", "k", "v"))
    kn, vn = new["k"].to(dev), new["v"].to(dev)
    sl = torch.tensor(lens, dtype=torch.int32, device=dev)
    o, lse = fa.attention_forward_kvcache(q, kc, vc, kn, vn, sl, causal=True)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status(None) == 0
    kc_exp, vc_exp = inp["k"].clone(), inp["v"].clone()
    for b in range(B):
        kc_exp[b, lens[b]] = new["k"][b, 0]
        vc_exp[b, lens[b]] = new["v"][b, 0]
    assert torch.equal(kc.cpu(), kc_exp) and torch.equal(vc.cpu(), vc_exp)
    for b in range(B):
        L = lens[b] + 1
        o_ref, lse_ref = oracle.attn_fwd(inp["q"][b:b + 1].double().numpy(),
                                         kc_exp[b:b + 1, :L].double().numpy(),
                                         vc_exp[b:b + 1, :L].double().numpy(),
                                         scale=1 / math.sqrt(d), causal=True)
        assert o_error(o[b:b + 1].float().cpu().numpy(), o_ref, "fp16") <= TOL_BF16["o"]
        compare_lse(lse[b:b + 1].cpu().numpy(), lse_ref, TOL_BF16["lse"], "kvcache fp16 %d" % b)
