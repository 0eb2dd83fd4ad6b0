"""GPU parity of fa_fwd_blocksparse and fa_bwd_blocksparse against the fp64
oracle's block-masked attention and gradients (same seeded inputs, same
128 x 128 block mask).

Random masks per (batch, head) -- so the two 128-row Q tiles of a CTA often
have different key tiles on -- and masks shared across batch and heads
(stride 0), with causal, window and plain masks, GQA, every head dim, ragged
sizes, fp16, an all-zero mask (every row empty) and an all-ones mask (the
dense kernel's result, bit for bit)."""
import math

import numpy as np
import pytest
import torch

import exact_io_aware_89_b200 as fa
import oracle
from parity_utils import TOL_BF16, ZERO_ABS, compare_lse, o_error, rel_fro
from seeded_inputs import make_inputs

pytestmark = pytest.mark.gpu
T = fa.BLOCK_SPARSE_TILE


@pytest.fixture(autouse=True)
def _need_cuda(cuda_ok):
    return cuda_ok


def check_bs(B, Nq, Nk, Hq, Hkv, d, mask, causal=False, window=(-1, -1), seed=0, dtype="bf16"):
    inp = make_inputs(B, Nq, Nk, Hq, Hkv, d, seed, dtype=dtype, with_dout=False)
    dev = torch.device("cuda")
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    scale = 1.0 / math.sqrt(d)
    m = torch.from_numpy(np.ascontiguousarray(mask.astype(np.uint8))).to(dev)
    o, lse = fa.attention_forward_blocksparse(q, k, v, m, scale=scale, causal=causal,
                                              window=window)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status(None) == 0
    f64 = {n: t.double().numpy() for n, t in inp.items()}
    o_ref, lse_ref = oracle.attn_fwd_blockmask(f64["q"], f64["k"], f64["v"], mask, block=T,
                                               scale=scale, causal=causal, window=window)
    what = "blocksparse B%d Nq%d Nk%d Hq%d Hkv%d d%d causal%d win%s %s" % (
        B, Nq, Nk, Hq, Hkv, d, causal, window, dtype)
    err = o_error(o.float().cpu().numpy(), o_ref, dtype)
    assert err <= TOL_BF16["o"], "%s: O max err %.3e" % (what, err)
    compare_lse(lse.cpu().numpy(), lse_ref, TOL_BF16["lse"], what)
    return o, lse


def rand_mask(shape, density, seed):
    return np.random.default_rng(seed).random(shape) < density


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal,window", [(False, (-1, -1)), (True, (-1, -1)), (False, (300, 200))])
def test_random_masks_per_head(d, causal, window):
    B, Nq, Nk, Hq, Hkv = 2, 700, 900, 4, 2
    mask = rand_mask((B, Hq, -(-Nq // T), -(-Nk // T)), 0.5, seed=d + 7 * causal)
    check_bs(B, Nq, Nk, Hq, Hkv, d, mask, causal, window, seed=71)


def test_mask_shared_across_batch_and_heads_fp16():
    B, Nq, Nk, Hq, Hkv, d = 3, 520, 520, 8, 1, 128
    mask = rand_mask((1, 1, 5, 5), 0.6, seed=72)
    mask[0, 0, :, 0] = True
    check_bs(B, Nq, Nk, Hq, Hkv, d, mask, causal=True, seed=73, dtype="fp16")


def test_all_zero_mask_gives_empty_rows():
    B, N, Hq, d = 1, 300, 2, 64
    mask = np.zeros((1, 1, 3, 3), dtype=bool)
    o, lse = check_bs(B, N, N, Hq, Hq, d, mask, seed=74)
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


def test_all_ones_mask_is_the_dense_kernel_bit_for_bit():
    B, N, Hq, Hkv, d = 2, 1000, 4, 2, 128
    inp = make_inputs(B, N, N, Hq, Hkv, d, 75, with_dout=False)
    dev = torch.device("cuda")
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    ones = torch.ones((1, 1, 8, 8), dtype=torch.uint8, device=dev)
    o1, l1 = fa.attention_forward_blocksparse(q, k, v, ones, causal=True)
    o2, l2 = fa.attention_forward(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_local_plus_global_pattern_long():
    """A long sequence with a sliding band of blocks plus the first block
    column (the shape of local + global sparse attention), causal."""
    B, N, Hq, Hkv, d = 1, 4096, 2, 1, 128
    nb = N // T
    mask = np.zeros((1, 1, nb, nb), dtype=bool)
    for i in range(nb):
        mask[0, 0, i, max(0, i - 2):i + 1] = True
        mask[0, 0, i, 0] = True
    check_bs(B, N, N, Hq, Hkv, d, mask, causal=True, seed=76)


def check_bs_bwd(B, Nq, Nk, Hq, Hkv, d, mask, causal=False, window=(-1, -1), seed=0):
    inp = make_inputs(B, Nq, Nk, Hq, Hkv, d, seed)
    dev = torch.device("cuda")
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    scale = 1.0 / math.sqrt(d)
    m = torch.from_numpy(np.ascontiguousarray(mask.astype(np.uint8))).to(dev)
    o, lse = fa.attention_forward_blocksparse(q, k, v, m, scale=scale, causal=causal, window=window)
    g1 = fa.attention_backward_blocksparse(q, k, v, o, lse, do, m, scale=scale, causal=causal,
                                           window=window)
    g2 = fa.attention_backward_blocksparse(q, k, v, o, lse, do, m, scale=scale, causal=causal,
                                           window=window)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status(None) == 0
    for a, b in zip(g1, g2):
        assert torch.equal(a, b), "block-sparse backward not deterministic"
    f64 = {n: t.double().numpy() for n, t in inp.items()}
    refs = oracle.attn_bwd_blockmask(f64["q"], f64["k"], f64["v"], f64["do"], mask, block=T,
                                     scale=scale, causal=causal, window=window)
    what = "blocksparse bwd B%d Nq%d Nk%d Hq%d Hkv%d d%d causal%d win%s" % (
        B, Nq, Nk, Hq, Hkv, d, causal, window)
    for name, g, r in zip(("dq", "dk", "dv"), g1, refs):
        g = g.float().cpu().numpy()
        if not np.any(r):
            assert float(np.abs(g).max()) <= ZERO_ABS, "%s: %s should be ~0" % (what, name)
            continue
        e = rel_fro(g, r)
        assert e <= TOL_BF16["grad"], "%s: %s rel err %.3e" % (what, name, e)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal,window", [(False, (-1, -1)), (True, (-1, -1)), (False, (300, 200))])
def test_backward_random_masks_per_head(d, causal, window):
    B, Nq, Nk, Hq, Hkv = 2, 700, 900, 4, 2
    mask = rand_mask((B, Hq, -(-Nq // T), -(-Nk // T)), 0.5, seed=3 * d + causal)
    check_bs_bwd(B, Nq, Nk, Hq, Hkv, d, mask, causal, window, seed=81)


def test_backward_all_ones_mask_is_the_dense_backward_bit_for_bit():
    B, N, Hq, Hkv, d = 2, 1000, 4, 2, 128
    inp = make_inputs(B, N, N, Hq, Hkv, d, 82)
    dev = torch.device("cuda")
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    ones = torch.ones((1, 1, 8, 8), dtype=torch.uint8, device=dev)
    o, lse = fa.attention_forward(q, k, v, causal=True)
    g1 = fa.attention_backward_blocksparse(q, k, v, o, lse, do, ones, causal=True)
    g2 = fa.attention_backward(q, k, v, o, lse, do, causal=True)
    torch.cuda.synchronize()
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)


def test_backward_fp16_random_mask():
    B, Nq, Nk, Hq, Hkv, d = 1, 520, 700, 4, 2, 64
    mask = rand_mask((B, Hq, -(-Nq // T), -(-Nk // T)), 0.5, seed=91)
    inp = make_inputs(B, Nq, Nk, Hq, Hkv, d, 92, dtype="fp16")
    dev = torch.device("cuda")
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    m = torch.from_numpy(mask.astype(np.uint8)).to(dev)
    o, lse = fa.attention_forward_blocksparse(q, k, v, m, causal=True)
    dq, dk, dv = fa.attention_backward_blocksparse(q, k, v, o, lse, do, m, causal=True)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status(None) == 0 and dq.dtype == torch.float16
    f64 = {n: t.double().numpy() for n, t in inp.items()}
    refs = oracle.attn_bwd_blockmask(f64["q"], f64["k"], f64["v"], f64["do"], mask, block=T,
                                     scale=1 / math.sqrt(d), causal=True)
    for name, g, r in zip(("dq", "dk", "dv"), (dq, dk, dv), refs):
        e = rel_fro(g.float().cpu().numpy(), r)
        assert e <= TOL_BF16["grad"], "blocksparse fp16 %s rel err %.3e" % (name, e)
