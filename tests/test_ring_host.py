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
    """Chunks r and src of an equal split (the contiguous layout's chunks, the
    zig-zag layout's are the same function of the chunk indices)."""
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


def _split(x, R, layout="contiguous"):
    """Each rank's rows, in its row order for the layout (chunks along dim 1)."""
    n_chunks = R if layout == "contiguous" else 2 * R
    c = x.shape[1] // n_chunks
    out = []
    for r in range(R):
        parts = [x[:, i * c:(i + 1) * c] for i in ring.rank_chunks(r, R, layout)]
        out.append(torch.from_numpy(np.ascontiguousarray(np.concatenate(parts, axis=1))))
    return out


def _join(xs, R, layout="contiguous", dim=1):
    """The whole sequence back from the ranks' rows."""
    n_chunks = R if layout == "contiguous" else 2 * R
    per = len(ring.rank_chunks(0, R, layout))
    chunks = [None] * n_chunks
    for r in range(R):
        a = np.asarray(xs[r])
        for p, i in enumerate(ring.rank_chunks(r, R, layout)):
            c = a.shape[dim] // per
            chunks[i] = np.take(a, range(p * c, (p + 1) * c), axis=dim)
    return np.concatenate(chunks, axis=dim)


@pytest.mark.parametrize("layout", ["contiguous", "zigzag"])
@pytest.mark.parametrize("R,Hq,Hkv,causal", [(1, 2, 2, True), (2, 2, 2, True), (3, 4, 2, True),
                                              (4, 2, 1, False), (3, 2, 2, False)])
def test_local_ring_equals_attention_over_the_whole_sequence(R, Hq, Hkv, causal, layout):
    B, n, d = 2, 6, 8
    N = R * n
    q, k, v, do = _inputs(B, N, Hq, Hkv, d, seed=R * 10 + Hq)
    scale = 1.0 / math.sqrt(d)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, scale=scale, causal=causal)
    g_ref = oracle.attn_bwd(q, k, v, do, scale=scale, causal=causal)
    ops = OracleOps()
    qs, ks, vs, dos = (_split(x, R, layout) for x in (q, k, v, do))
    os_, lses = ring.local_ring_forward(qs, ks, vs, scale=scale, causal=causal, ops=ops, layout=layout)
    np.testing.assert_allclose(_join([x.numpy() for x in os_], R, layout), o_ref, atol=1e-12)
    np.testing.assert_allclose(_join([x.numpy() for x in lses], R, layout, dim=2), lse_ref, atol=1e-12)
    dq, dk, dv = ring.local_ring_backward(qs, ks, vs, os_, lses, dos, scale=scale, causal=causal, ops=ops,
                                          layout=layout)
    for got, ref in zip((dq, dk, dv), g_ref):
        np.testing.assert_allclose(_join([x.numpy() for x in got], R, layout), ref, atol=1e-11)


@pytest.mark.parametrize("R", [2, 3, 4, 8])
def test_zigzag_gives_every_rank_the_same_causal_work_at_every_step(R):
    """Visible (query chunk, key chunk) pairs per rank and step, counted in
    units of a causal diagonal pair (half a full one): with the zig-zag layout
    every rank does the same at every step; with contiguous chunks rank 0
    does one diagonal pair in all and rank R - 1 does 2R - 1 times that."""
    def work(layout):
        w = np.zeros((R, R))
        for r in range(R):
            for t in range(R):
                for mode in ring._chunk_pairs(r, R, t, layout, True).values():
                    w[r, t] += 1 if mode == "causal" else 2
        return w
    z = work("zigzag")
    assert (z == z[0, 0]).all() and z[0, 0] == 4
    c = work("contiguous").sum(axis=1)
    assert c[0] == 1 and c[R - 1] == 2 * R - 1


@pytest.mark.parametrize("layout", ["contiguous", "zigzag"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("R", [1, 2, 3, 4, 8])
def test_each_step_is_one_call_covering_exactly_the_visible_pairs(R, causal, layout):
    """Brute force over the rows of a small split: the calls of a step, each a
    rectangle of the rank's rows (causal within it or not), see exactly the
    (query, key) pairs of the whole sequence that are visible, each once."""
    c = 3
    for r in range(R):
        sched = ring._schedule(r, R, layout, causal)
        for t in range(R):
            calls = [x[1:] for x in sched if x[0] == t]
            s = (r - t) % R
            assert len(calls) == (0 if causal and layout == "contiguous" and s > r else 1)
            qpos = [i * c + a for i in ring.rank_chunks(r, R, layout) for a in range(c)]
            kpos = [j * c + b for j in ring.rank_chunks(s, R, layout) for b in range(c)]
            seen = np.zeros((len(qpos), len(kpos)), dtype=int)
            for (i0, i1), (j0, j1), cz in calls:
                for a in range(i0 * c, i1 * c):
                    for b in range(j0 * c, j1 * c):
                        # causal calls are square: bottom-right = top-left
                        if not cz or b - j0 * c <= a - i0 * c:
                            seen[a, b] += 1
            want = np.array([[_visible(qp, kp, causal) for kp in kpos] for qp in qpos], dtype=int)
            assert (seen == want).all(), (r, t)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, causal, q_all, k_all, v_all, do_all, queue, layout="contiguous"):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v, do = (_split(x, world, layout)[rank] for x in (q_all, k_all, v_all, do_all))
        ops = OracleOps()
        o, lse = ring.ring_attention_forward(q, k, v, causal=causal, ops=ops, layout=layout)
        dq, dk, dv = ring.ring_attention_backward(q, k, v, o, lse, do, causal=causal, ops=ops, layout=layout)
        dist.barrier()
        queue.put((rank, o.numpy(), lse.numpy(), dq.numpy(), dk.numpy(), dv.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,causal,layout", [(2, True, "contiguous"), (3, True, "contiguous"),
                                                 (2, False, "contiguous"), (2, True, "zigzag"),
                                                 (3, True, "zigzag")])
def test_gloo_ranks_run_the_ring_exchange(world, causal, layout):
    import torch.multiprocessing as mp
    B, n, Hq, Hkv, d = 1, 4, 2, 1, 8
    q, k, v, do = _inputs(B, world * n, Hq, Hkv, d, seed=77 + world)
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, causal, q, k, v, do, queue, layout))
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
    np.testing.assert_allclose(_join([x[1] for x in out], world, layout), o_ref, atol=1e-12)
    np.testing.assert_allclose(_join([x[2] for x in out], world, layout, dim=2), lse_ref, atol=1e-12)
    for idx, ref in zip((3, 4, 5), g_ref):
        np.testing.assert_allclose(_join([x[idx] for x in out], world, layout), ref, atol=1e-11)
