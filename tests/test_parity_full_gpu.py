"""GPU parity at the full sizes of the named workloads, on sampled outputs.

The CUDA path runs each workload whole, through the same C ABI calls and
launch configuration bench.py times (fa_fwd, then fa_bwd with its workspace).
The fp64 oracle cannot afford these sizes whole, so it computes selected
outputs one by one: for a few (batch, KV head) pairs -- the query heads of a
GQA group included -- the O/LSE and dQ rows of sampled query rows and the dK/dV
rows of sampled key rows (first and last rows, tile edges, the middle, and
seeded random rows).  Attention of one (batch, KV group) does not depend on the
others, so the oracle is given only that slice of the same seeded inputs.

Tolerances are those of the small-size parity tests (parity_utils): O max-abs
1e-2, LSE max-abs 1e-3, dQ/dK/dV relative Frobenius 2e-2 over the sampled rows.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from parity_utils import TOL_BF16, compare_lse, gpu_run, rel_fro, o_error
from seeded_inputs import config_seed, make_inputs, sweep_seed

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda(cuda_ok):
    return cuda_ok


def sweep(N, d, causal):
    # sequence-length sweep point: hidden 2048 (H = 2048 / d), batch 16384 / N
    return dict(B=16384 // N, N=N, Hq=2048 // d, Hkv=2048 // d, d=d, causal=causal,
                window=(-1, -1), seed=sweep_seed(N, d))


WORKLOADS = {
    "train_B2_H16_N2048_d128_causal":
        dict(B=2, N=2048, Hq=16, Hkv=16, d=128, causal=True, window=(-1, -1), seed=config_seed(2)),
    "gqa_Hq32_Hkv8_N8192_d128_window4096":
        dict(B=1, N=8192, Hq=32, Hkv=8, d=128, causal=True, window=(4096, 0), seed=config_seed(4)),
    "wide_B1_H96_N8192_d128_causal":
        dict(B=1, N=8192, Hq=96, Hkv=96, d=128, causal=True, window=(-1, -1), seed=config_seed(5)),
    "d256_B1_H16_N16384_causal":
        dict(B=1, N=16384, Hq=16, Hkv=16, d=256, causal=True, window=(-1, -1), seed=config_seed(5) + 50),
}
# every point of the sequence-length sweep: N in 512 .. 16k, d in {64, 128},
# causal and non-causal (hidden 2048, B = 16384 / N)
for _N in (512, 1024, 2048, 4096, 8192, 16384):
    for _d in (64, 128):
        for _c in (True, False):
            WORKLOADS["sweep_N%d_d%d_%s" % (_N, _d, "causal" if _c else "noncausal")] = sweep(_N, _d, _c)


def sample_rows(N, rng, extra=4):
    fixed = {0, 1, 63, 64, 127, 128, 255, 256, N // 2, N - 129, N - 2, N - 1}
    rows = sorted(r for r in fixed if 0 <= r < N)
    rand = rng.choice(N, size=min(extra, N), replace=False)
    return sorted(set(rows) | set(int(r) for r in rand))


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_full_size_sampled_rows(name):
    w = WORKLOADS[name]
    B, N, Hq, Hkv, d = w["B"], w["N"], w["Hq"], w["Hkv"], w["d"]
    G = Hq // Hkv
    scale = 1.0 / math.sqrt(d)
    inp = make_inputs(B, N, N, Hq, Hkv, d, w["seed"])
    g = gpu_run(inp, scale, w["causal"], w["window"], backward=True)
    torch.cuda.empty_cache()

    rng = np.random.default_rng(w["seed"])
    qrows = sample_rows(N, rng)
    krows = sample_rows(N, rng)
    # (batch, KV head) pairs: the first and the last
    pairs = sorted({(0, 0), (B - 1, Hkv - 1)})
    for b, hk in pairs:
        hq = list(range(hk * G, (hk + 1) * G))
        sl = {
            "q": inp["q"][b:b + 1, :, hq[0]:hq[-1] + 1].double().numpy(),
            "k": inp["k"][b:b + 1, :, hk:hk + 1].double().numpy(),
            "v": inp["v"][b:b + 1, :, hk:hk + 1].double().numpy(),
            "do": inp["do"][b:b + 1, :, hq[0]:hq[-1] + 1].double().numpy(),
        }
        what = "%s b=%d kv-head=%d" % (name, b, hk)
        kw = dict(scale=scale, causal=w["causal"], window=w["window"])
        o_ref, lse_ref = oracle.attn_fwd_rows(sl["q"], sl["k"], sl["v"], qrows, **kw)
        o_gpu = g["o"][b:b + 1, qrows][:, :, hq[0]:hq[-1] + 1]
        lse_gpu = g["lse"][b:b + 1, hq[0]:hq[-1] + 1][:, :, qrows]
        err_o = o_error(o_gpu, o_ref)
        assert err_o <= TOL_BF16["o"], "%s: O max err %.3e" % (what, err_o)
        compare_lse(lse_gpu, lse_ref, TOL_BF16["lse"], what)

        dq_ref = oracle.attn_dq_rows(sl["q"], sl["k"], sl["v"], sl["do"], qrows, **kw)
        dq_gpu = g["dq"][b:b + 1, qrows][:, :, hq[0]:hq[-1] + 1]
        e = rel_fro(dq_gpu, dq_ref)
        assert e <= TOL_BF16["grad"], "%s: dQ rel err %.3e" % (what, e)

        dk_ref, dv_ref = oracle.attn_dkdv_rows(sl["q"], sl["k"], sl["v"], sl["do"], krows, **kw)
        dk_gpu = g["dk"][b:b + 1, krows][:, :, hk:hk + 1]
        dv_gpu = g["dv"][b:b + 1, krows][:, :, hk:hk + 1]
        for n, gg, rr in (("dK", dk_gpu, dk_ref), ("dV", dv_gpu, dv_ref)):
            e = rel_fro(gg, rr)
            assert e <= TOL_BF16["grad"], "%s: %s rel err %.3e" % (what, n, e)
