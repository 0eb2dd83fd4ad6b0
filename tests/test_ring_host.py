"""Ring (context-parallel) attention on the CPU: the ring schedule with the
fp64 oracle doing each block (tests/ring_oracle_ops.py), checked against the
oracle over the whole sequence; the block masks against brute force; and the
point-to-point exchange through two and three gloo ranks."""
import math
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_89_b200 import ring
from ring_oracle_ops import OracleOps


def _visible(i, j, causal):
    return (not causal) or j <= i


@pytest.mark.parametrize("R", [1, 2, 3, 5])
@pytest.mark.parametrize("causal", [False, True])
def test_block_mode_matches_the_mask_of_the_whole_sequence(R, causal):
    n = 4
    for r in range(R):
        for src in range(R):
            vis = np.array([[_visible(r * n + a, src * n + b, causal) for b in range(n)] for a in range(n)])
            mode = ring.block_mode(r, src, causal)
            if mode == "full":
                assert vis.all()
            elif mode == "causal":
                assert src == r and (vis == np.tril(np.ones((n, n), dtype=bool))).all()
            else:
                assert mode is None and not vis.any()


def _inputs(B, N, Hq, Hkv, d, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, N, Hq, d))
    k = rng.standard_normal((B, N, Hkv, d))
    v = rng.standard_normal((B, N, Hkv, d))
    do = rng.standard_normal((B, N, Hq, d))
    return q, k, v, do


def _split(x, R):
    n = x.shape[1] // R
    return [torch.from_numpy(np.ascontiguousarray(x[:, r * n:(r + 1) * n])) for r in range(R)]


@pytest.mark.parametrize("R,Hq,Hkv,causal", [(1, 2, 2, True), (2, 2, 2, True), (3, 4, 2, True),
                                              (4, 2, 1, False), (3, 2, 2, False)])
def test_local_ring_equals_attention_over_the_whole_sequence(R, Hq, Hkv, causal):
    B, n, d = 2, 5, 8
    N = R * n
    q, k, v, do = _inputs(B, N, Hq, Hkv, d, seed=R * 10 + Hq)
    scale = 1.0 / math.sqrt(d)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, scale=scale, causal=causal)
    g_ref = oracle.attn_bwd(q, k, v, do, scale=scale, causal=causal)
    ops = OracleOps()
    qs, ks, vs, dos = (_split(x, R) for x in (q, k, v, do))
    os_, lses = ring.local_ring_forward(qs, ks, vs, scale=scale, causal=causal, ops=ops)
    o = np.concatenate([x.numpy() for x in os_], axis=1)
    lse = np.concatenate([x.numpy() for x in lses], axis=2)
    np.testing.assert_allclose(o, o_ref, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-12)
    dq, dk, dv = ring.local_ring_backward(qs, ks, vs, os_, lses, dos, scale=scale, causal=causal, ops=ops)
    for got, ref in zip((dq, dk, dv), g_ref):
        np.testing.assert_allclose(np.concatenate([x.numpy() for x in got], axis=1), ref, atol=1e-11)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, causal, q_all, k_all, v_all, do_all, queue):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        n = q_all.shape[1] // world
        sl = lambda x: torch.from_numpy(np.ascontiguousarray(x[:, rank * n:(rank + 1) * n]))
        q, k, v, do = sl(q_all), sl(k_all), sl(v_all), sl(do_all)
        ops = OracleOps()
        o, lse = ring.ring_attention_forward(q, k, v, causal=causal, ops=ops)
        dq, dk, dv = ring.ring_attention_backward(q, k, v, o, lse, do, causal=causal, ops=ops)
        dist.barrier()
        queue.put((rank, o.numpy(), lse.numpy(), dq.numpy(), dk.numpy(), dv.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,causal", [(2, True), (3, True), (2, False)])
def test_gloo_ranks_run_the_ring_exchange(world, causal):
    import torch.multiprocessing as mp
    B, n, Hq, Hkv, d = 1, 4, 2, 1, 8
    q, k, v, do = _inputs(B, world * n, Hq, Hkv, d, seed=77 + world)
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, causal, q, k, v, do, queue))
             for r in range(world)]
    for p in procs:
        p.start()
    out = sorted([queue.get(timeout=180) for _ in range(world)], key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    scale = 1.0 / math.sqrt(d)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, scale=scale, causal=causal)
    g_ref = oracle.attn_bwd(q, k, v, do, scale=scale, causal=causal)
    np.testing.assert_allclose(np.concatenate([x[1] for x in out], axis=1), o_ref, atol=1e-12)
    np.testing.assert_allclose(np.concatenate([x[2] for x in out], axis=2), lse_ref, atol=1e-12)
    for idx, ref in zip((3, 4, 5), g_ref):
        np.testing.assert_allclose(np.concatenate([x[idx] for x in out], axis=1), ref, atol=1e-11)
