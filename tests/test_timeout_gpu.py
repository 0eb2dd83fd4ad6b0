"""Failure detection on the GPU without a fault: a bounded device-side wait is
made to run out (fa_test_withhold_next_load: the first CTA of the next
forward launch never loads one key/value tile, so the wait for it has nothing
to wait for).  The kernel must give up on its own after its wait limit, report
FA_ERR_TIMEOUT through the device status word, leave the context usable, and
the very next call must be exact again."""
import math
import time

import numpy as np
import pytest
import torch

import exact_io_aware_89_b200 as fa
import oracle
from parity_utils import TOL_BF16, compare_lse, o_error
from seeded_inputs import make_inputs

pytestmark = pytest.mark.gpu

TIMEOUT = 5


@pytest.fixture(autouse=True)
def _need_cuda(cuda_ok):
    return cuda_ok


def test_withheld_load_times_out_and_the_next_call_is_exact():
    # non-causal: the first CTA (the last 256 query rows) walks all 4 key
    # tiles, so it has tiles left after its first two ring stages
    B, N, H, d = 1, 512, 2, 128
    inp = make_inputs(B, N, N, H, H, d, 4242)
    dev = torch.device("cuda")
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    scale = 1.0 / math.sqrt(d)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status(None) == 0

    assert fa.fa_test_withhold_next_load() == 0
    t0 = time.perf_counter()
    fa.attention_forward(q, k, v, scale=scale)
    torch.cuda.synchronize()  # returns: the wait gave up, nothing hangs
    waited = time.perf_counter() - t0
    assert fa.fa_get_device_status(None) == TIMEOUT
    assert waited >= 1.0, "the wait ran out after %.3f s, before its 2 s limit" % waited
    assert fa.fa_get_device_status(None) == 0  # reading the status cleared it

    # the next call (and a backward) on the same context is exact
    o, lse = fa.attention_forward(q, k, v, scale=scale)
    do = inp["do"].to(dev)
    dq, dk, dv = fa.attention_backward(q, k, v, o, lse, do, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status(None) == 0
    f64 = {n: t.double().numpy() for n, t in inp.items()}
    o_ref, lse_ref = oracle.attn_fwd(f64["q"], f64["k"], f64["v"], scale=scale)
    assert o_error(o.float().cpu().numpy(), o_ref) <= TOL_BF16["o"]
    compare_lse(lse.cpu().numpy(), lse_ref, TOL_BF16["lse"], "after timeout")
    refs = oracle.attn_bwd(f64["q"], f64["k"], f64["v"], f64["do"], scale=scale)
    for g, r in zip((dq, dk, dv), refs):
        g = g.float().cpu().numpy()
        assert np.linalg.norm(g - r) / np.linalg.norm(r) <= TOL_BF16["grad"]
