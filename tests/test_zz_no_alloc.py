"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory
(allocator-free runtimes that carve their device memory from one arena at
start-up, hosts with a fixed memory budget, code recording into a CUDA graph
without allocating).  It runs fa_bwd's kernels on the library's fixed scratch
array instead of a caller workspace, so its gradients must be fa_bwd's bit for
bit -- any difference would point at the scratch (a wrong offset, a stale
value, a race) -- and, through fa_bwd, match the fp64 oracle.

Collected last on purpose (file name), so that a run stopping at the first
failure has already run every other test; it also passes on its own in a
fresh process (it sets up everything it uses).
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import exact_io_aware_89_b200 as fa
import oracle
from parity_utils import TOL_BF16, rel_fro
from seeded_inputs import make_inputs

pytestmark = pytest.mark.gpu

WORKSPACE_ERR = 4
SCRATCH_BYTES = 16 << 20


def _setup(shape, causal, window, seed):
    B, N, Hq, Hkv, d = shape
    dev = torch.device("cuda")
    inp = make_inputs(B, N, N, Hq, Hkv, d, seed)
    x = {n: inp[n].to(dev) for n in ("q", "k", "v", "do")}
    scale = 1.0 / math.sqrt(d)
    o, lse = fa.attention_forward(x["q"], x["k"], x["v"], scale=scale, causal=causal, window=window)
    return inp, x, o, lse, scale


def _noalloc(x, o, lse, out, shape, scale, causal, window, stream):
    B, N, Hq, Hkv, d = shape
    wl, wr = window
    return fa.fa_bwd_noalloc(x["q"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(), o.data_ptr(),
                             lse.data_ptr(), x["do"].data_ptr(), out[0].data_ptr(), out[1].data_ptr(),
                             out[2].data_ptr(), B, N, N, Hq, Hkv, d, scale, int(causal), wl, wr, stream)


def _check(shape, causal, window, seed, with_oracle):
    inp, x, o, lse, scale = _setup(shape, causal, window, seed)
    ref = fa.attention_backward(x["q"], x["k"], x["v"], o, lse, x["do"], scale=scale, causal=causal,
                                window=window)
    got = [torch.full_like(t, float("nan")) for t in (x["q"], x["k"], x["v"])]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = _noalloc(x, o, lse, got, shape, scale, causal, window, stream)
    assert st == 0, fa.fa_status_string(st)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status(None) == 0
    for name, r, g in zip(("dq", "dk", "dv"), ref, got):
        assert torch.equal(r, g), "%s differs from fa_bwd" % name
    if with_oracle:
        f64 = {n: t.double().numpy() for n, t in inp.items()}
        refs = oracle.attn_bwd(f64["q"], f64["k"], f64["v"], f64["do"], scale=scale, causal=causal,
                               window=window)
        for name, r, g in zip(("dq", "dk", "dv"), refs, got):
            e = rel_fro(g.float().cpu().numpy(), r)
            assert e <= TOL_BF16["grad"], "%s rel err %.3e against the oracle" % (name, e)


@pytest.fixture(autouse=True)
def _need_cuda(cuda_ok):
    return cuda_ok


def test_noalloc_backward_matches_fa_bwd_on_two_calls_in_a_row():
    """Two consecutive calls with different shapes and masks; each gives fa_bwd's
    bits on the same inputs (the second call reuses the scratch the first one
    left behind), and the first also matches the fp64 oracle."""
    _check((2, 333, 4, 2, 128), True, (-1, -1), seed=51, with_oracle=True)
    _check((1, 700, 2, 1, 64), False, (90, 30), seed=52, with_oracle=False)


def test_noalloc_backward_replays_in_a_cuda_graph():
    """One eager call sets up the device, then the call is captured into a CUDA
    graph and replayed twice, with new inputs copied into the captured buffers
    before each replay; every replay gives fa_bwd's bits for its inputs."""
    shape, causal, window = (1, 512, 4, 4, 128), True, (-1, -1)
    B, N, Hq, Hkv, d = shape
    _, x, o, lse, scale = _setup(shape, causal, window, seed=61)
    got = [torch.empty_like(t) for t in (x["q"], x["k"], x["v"])]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        sp = ctypes.c_void_p(s.cuda_stream)
        assert _noalloc(x, o, lse, got, shape, scale, causal, window, sp) == 0
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            assert _noalloc(x, o, lse, got, shape, scale, causal, window, sp) == 0
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    for seed in (62, 63):
        _, x2, o2, lse2, _ = _setup(shape, causal, window, seed)
        for n in x:
            x[n].copy_(x2[n])
        o.copy_(o2)
        lse.copy_(lse2)
        for t in got:
            t.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        ref = fa.attention_backward(x2["q"], x2["k"], x2["v"], o2, lse2, x2["do"], scale=scale,
                                    causal=causal, window=window)
        for name, r, t in zip(("dq", "dk", "dv"), ref, got):
            assert torch.equal(r, t), "replay with seed %d: %s differs from fa_bwd" % (seed, name)
    assert fa.fa_get_device_status(None) == 0
    del g


def test_noalloc_rejects_problems_beyond_its_scratch():
    """A problem whose fa_bwd workspace exceeds the fixed 16 MiB array gets
    FA_ERR_WORKSPACE before anything is launched (the pointers are never used)."""
    fake = 0x10000
    B, Hq, N, d = 1, 1024, 4096, 128
    assert fa.fa_bwd_workspace_size(B, N, Hq, d) > SCRATCH_BYTES
    st = fa.fa_bwd_noalloc(fake, fake, fake, fake, fake, fake, fake, fake, fake, B, N, N, Hq, Hq,
                           d, 0.088, 1, -1, -1, None)
    assert st == WORKSPACE_ERR
