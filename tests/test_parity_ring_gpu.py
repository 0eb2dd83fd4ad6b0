"""Ring (context-parallel) attention on the GPU, against the fp64 oracle.

* fa_lse_merge folding partial results in order equals oracle.merge_partials
  on the same (bf16-rounded) partials; fa_grad_accumulate equals the fp64 sum;
  a part covering some rows of the accumulator changes only those rows.
* The ring of R ranks, emulated on one GPU (each rank's slices in its own
  buffers, the exchange a device copy), run through the library's kernels
  (fa_fwd / fa_bwd per slice pair, the merge and accumulate kernels), equals
  the oracle's attention over the whole sequence within the bf16 tolerances
  of the other parity tests, and gives the same bits on every run.
"""
import math

import numpy as np
import pytest
import torch

import exact_io_aware_89_b200 as fa
import oracle
from exact_io_aware_89_b200 import ring
from parity_utils import TOL_BF16, compare_lse, half_ulp, o_error, rel_fro
from seeded_inputs import make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda(cuda_ok):
    return cuda_ok


@pytest.mark.parametrize("S,d", [(1, 64), (2, 128), (4, 128), (3, 256)])
def test_lse_merge_equals_the_oracle_merge(S, d):
    dev = torch.device("cuda")
    g = torch.Generator().manual_seed(100 + S)
    B, Nq, H = 2, 77, 3
    o_parts = [torch.randn((B, Nq, H, d), generator=g).to(torch.bfloat16) for _ in range(S)]
    lse_parts = [(3.0 * torch.randn((B, H, Nq), generator=g)).float() for _ in range(S)]
    # some rows see no key in some parts (lse = -inf, O = 0); row 0 of head 0 in none
    for s in range(S):
        dead = torch.rand((B, H, Nq), generator=g) < 0.2
        dead[0, 0, 0] = True
        lse_parts[s][dead] = -math.inf
        o_parts[s].permute(0, 2, 1, 3)[dead] = 0
    o_acc = torch.empty((B, Nq, H, d), dtype=torch.float32, device=dev)
    lse_acc = torch.empty((B, H, Nq), dtype=torch.float32, device=dev)
    out = torch.empty((B, Nq, H, d), dtype=torch.bfloat16, device=dev)
    for s in range(S):
        fa.lse_merge(o_acc, lse_acc, o_parts[s].to(dev), lse_parts[s].to(dev), first=(s == 0),
                     out=out if s == S - 1 else None)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.merge_partials([x.double().numpy() for x in o_parts],
                                           [x.double().numpy() for x in lse_parts])
    compare_lse(lse_acc.cpu().numpy(), lse_ref, 1e-5, "merge")
    # fp32 arithmetic on bf16 inputs: relative error a few units of 2^-24
    assert np.abs(o_acc.cpu().numpy() - o_ref).max() <= 1e-5
    assert o_error(out.float().cpu().numpy(), o_ref) <= 1e-5
    assert not out.float()[0, 0, 0].any()


def test_grad_accumulate_sums_in_fp32_and_rounds_once():
    dev = torch.device("cuda")
    g = torch.Generator().manual_seed(7)
    n = 3 * 1000 * 8
    parts = [torch.randn(n, generator=g).to(torch.bfloat16) for _ in range(5)]
    acc = torch.empty(n, dtype=torch.float32, device=dev)
    for s, p in enumerate(parts):
        fa.grad_accumulate(acc, p.to(dev), first=(s == 0))
    out = torch.empty(n, dtype=torch.bfloat16, device=dev)
    fa.grad_accumulate(acc, None, out=out)
    torch.cuda.synchronize()
    ref = sum(p.double().numpy() for p in parts)
    assert np.abs(acc.cpu().numpy() - ref).max() <= 1e-5
    assert (np.abs(out.float().cpu().numpy() - ref) <= half_ulp(ref) + 1e-5).all()


def test_merge_and_accumulate_reach_only_the_given_rows():
    """A part covering rows [row0, row0 + n) of a larger accumulator (B > 1,
    so those rows are not one contiguous range): those rows merge / add as
    the oracle says, every other row keeps its bits."""
    dev = torch.device("cuda")
    g = torch.Generator().manual_seed(11)
    B, Nacc, row0, Nq, H, d = 2, 96, 32, 48, 3, 128
    rows = slice(row0, row0 + Nq)
    o_acc0 = torch.randn((B, Nacc, H, d), generator=g)
    lse_acc0 = torch.randn((B, H, Nacc), generator=g)
    o_part = torch.randn((B, Nq, H, d), generator=g).to(torch.bfloat16)
    lse_part = torch.randn((B, H, Nq), generator=g)
    o_acc, lse_acc = o_acc0.to(dev), lse_acc0.to(dev)
    out = torch.full((B, Nacc, H, d), 7.0, dtype=torch.bfloat16, device=dev)
    fa.lse_merge(o_acc, lse_acc, o_part.to(dev), lse_part.to(dev), first=False, out=out, row0=row0)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.merge_partials([o_acc0[:, rows].double().numpy(), o_part.double().numpy()],
                                           [lse_acc0[:, :, rows].double().numpy(), lse_part.double().numpy()])
    o_acc, lse_acc, out = o_acc.cpu(), lse_acc.cpu(), out.cpu()
    assert np.abs(o_acc[:, rows].numpy() - o_ref).max() <= 1e-5
    compare_lse(lse_acc[:, :, rows].numpy(), lse_ref, 1e-5, "merge rows")
    assert o_error(out[:, rows].float().numpy(), o_ref) <= 1e-5
    keep = torch.ones(Nacc, dtype=torch.bool)
    keep[rows] = False
    assert torch.equal(o_acc[:, keep], o_acc0[:, keep]) and torch.equal(lse_acc[:, :, keep], lse_acc0[:, :, keep])
    assert (out[:, keep].float() == 7.0).all()

    acc0 = torch.randn((B, Nacc, H, d), generator=g)
    part = torch.randn((B, Nq, H, d), generator=g).to(torch.bfloat16)
    for first in (False, True):
        acc = acc0.to(dev)
        fa.grad_accumulate(acc, part.to(dev), first=first, row0=row0)
        torch.cuda.synchronize()
        acc = acc.cpu()
        want = part.float() if first else acc0[:, rows] + part.float()  # one fp32 rounding, as on the GPU
        assert torch.equal(acc[:, rows], want)
        assert torch.equal(acc[:, keep], acc0[:, keep])
    out = torch.full((B, Nacc, H, d), 7.0, dtype=torch.bfloat16, device=dev)
    fa.grad_accumulate(acc0.to(dev), None, out=out, row0=row0)
    torch.cuda.synchronize()
    out = out.cpu()
    assert torch.equal(out[:, row0:], acc0[:, row0:].to(torch.bfloat16))
    assert (out[:, :row0].float() == 7.0).all()


CASES = [
    # (R, B, n per rank, Hq, Hkv, d, causal, layout, dtype)
    (2, 1, 256, 2, 2, 128, True, "contiguous", "bf16"),
    (4, 1, 192, 4, 2, 128, True, "contiguous", "bf16"),
    (3, 2, 128, 2, 1, 64, False, "contiguous", "bf16"),
    (4, 1, 160, 2, 2, 64, True, "contiguous", "bf16"),
    (2, 1, 256, 2, 2, 128, True, "zigzag", "bf16"),
    (4, 2, 192, 4, 2, 128, True, "zigzag", "bf16"),
    (3, 1, 128, 2, 2, 64, True, "zigzag", "bf16"),
    (3, 2, 256, 2, 1, 128, False, "zigzag", "bf16"),
    (2, 1, 256, 2, 2, 64, True, "zigzag", "fp16"),
]


def _rank_rows(x, R, layout):
    """Each rank's rows of the whole-sequence tensor x (dim 1), in its order."""
    n_chunks = R if layout == "contiguous" else 2 * R
    c = x.shape[1] // n_chunks
    return [torch.cat([x[:, i * c:(i + 1) * c] for i in ring.rank_chunks(r, R, layout)], dim=1).contiguous()
            for r in range(R)]


def _whole(xs, R, layout, dim=1):
    """The whole sequence back from the ranks' rows."""
    per = len(ring.rank_chunks(0, R, layout))
    chunks = {}
    for r in range(R):
        parts = torch.chunk(xs[r], per, dim=dim)
        for p, i in enumerate(ring.rank_chunks(r, R, layout)):
            chunks[i] = parts[p]
    return torch.cat([chunks[i] for i in sorted(chunks)], dim=dim)


def _run_ring(R, qs, ks, vs, dos, scale, causal, layout):
    os_, lses = ring.local_ring_forward(qs, ks, vs, scale=scale, causal=causal, layout=layout)
    dq, dk, dv = ring.local_ring_backward(qs, ks, vs, os_, lses, dos, scale=scale, causal=causal, layout=layout)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status(None) == 0
    return (_whole(os_, R, layout), _whole(lses, R, layout, dim=2), _whole(dq, R, layout),
            _whole(dk, R, layout), _whole(dv, R, layout))


@pytest.mark.parametrize("R,B,n,Hq,Hkv,d,causal,layout,dtype", CASES)
def test_emulated_ring_equals_attention_over_the_whole_sequence(R, B, n, Hq, Hkv, d, causal, layout, dtype):
    N = R * n
    inp = make_inputs(B, N, N, Hq, Hkv, d, 5000 + R * 10 + d, dtype=dtype)
    scale = 1.0 / math.sqrt(d)
    dev = torch.device("cuda")
    x = {k_: t.to(dev) for k_, t in inp.items()}
    qs, ks, vs, dos = (_rank_rows(x[name], R, layout) for name in ("q", "k", "v", "do"))
    o, lse, dq, dk, dv = _run_ring(R, qs, ks, vs, dos, scale, causal, layout)
    f64 = {k_: t.double().numpy() for k_, t in inp.items()}
    o_ref, lse_ref = oracle.attn_fwd(f64["q"], f64["k"], f64["v"], scale=scale, causal=causal)
    what = "ring %s R%d B%d N%d Hq%d Hkv%d d%d causal%d %s" % (layout, R, B, N, Hq, Hkv, d, causal, dtype)
    err = o_error(o.float().cpu().numpy(), o_ref, dtype)
    assert err <= TOL_BF16["o"], "%s: O err %.3e" % (what, err)
    compare_lse(lse.cpu().numpy(), lse_ref, TOL_BF16["lse"], what)
    refs = oracle.attn_bwd(f64["q"], f64["k"], f64["v"], f64["do"], scale=scale, causal=causal)
    for name, got, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), refs):
        e = rel_fro(got.float().cpu().numpy(), ref)
        assert e <= TOL_BF16["grad"], "%s: %s rel err %.3e" % (what, name, e)
    # the same bits on a second run
    again = _run_ring(R, qs, ks, vs, dos, scale, causal, layout)
    for a, b_ in zip((o, lse, dq, dk, dv), again):
        assert torch.equal(a, b_)
