"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory
(code inside a CUDA graph capture or a driver callback, allocator-free
runtimes, hosts with a fixed memory budget).  It must give what fa_bwd gives
while using the library's fixed scratch array instead of a caller workspace.

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
from parity_utils import TOL_BF16, rel_fro
from seeded_inputs import make_inputs

pytestmark = pytest.mark.gpu

WORKSPACE_ERR = 4


def _run(shape, causal, window, seed):
    B, N, Hq, Hkv, d = shape
    dev = torch.device("cuda")
    inp = make_inputs(B, N, N, Hq, Hkv, d, seed)
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    scale = 1.0 / math.sqrt(d)
    o, lse = fa.attention_forward(q, k, v, scale=scale, causal=causal, window=window)
    ref = fa.attention_backward(q, k, v, o, lse, do, scale=scale, causal=causal, window=window)
    got = [torch.empty_like(t) for t in (q, k, v)]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    wl, wr = window
    st = fa.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                           do.data_ptr(), got[0].data_ptr(), got[1].data_ptr(), got[2].data_ptr(),
                           B, N, N, Hq, Hkv, d, scale, int(causal), wl, wr, stream)
    assert st == 0, fa.fa_status_string(st)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status(None) == 0
    for name, r, g in zip(("dq", "dk", "dv"), ref, got):
        r, g = r.float().cpu().numpy(), g.float().cpu().numpy()
        assert rel_fro(g, r) <= TOL_BF16["grad"], name


@pytest.fixture(autouse=True)
def _need_cuda(cuda_ok):
    return cuda_ok


def test_noalloc_backward_matches_fa_bwd_on_two_calls_in_a_row():
    """Two consecutive calls with different shapes and masks; each matches
    fa_bwd on the same inputs (the second call reuses the scratch the first
    one left behind)."""
    _run((2, 333, 4, 2, 128), True, (-1, -1), seed=51)
    _run((1, 700, 2, 1, 64), False, (90, 30), seed=52)


def test_noalloc_rejects_problems_beyond_its_scratch():
    """B * Hq * ceil(Nq/256)*256 rows above the fixed limit -> FA_ERR_WORKSPACE,
    before anything is launched."""
    fake = 0x10000
    B, Hq, N = 1, 1024, 4096  # 4M rows > 2M
    st = fa.fa_bwd_noalloc(fake, fake, fake, fake, fake, fake, fake, fake, fake, B, N, N, Hq, Hq,
                           128, 0.088, 1, -1, -1, None)
    assert st == WORKSPACE_ERR
