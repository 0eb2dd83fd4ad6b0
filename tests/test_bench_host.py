"""Host-side logic of bench.py, on the CPU: the FLOP accounting, the roofline
bookkeeping, the ncu-traffic gate, and the multi-process path (two gloo ranks:
max over ranks, weak-scaling throughput, barrier, reference arm on rank 0 only).
"""
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_flop_accounting_matches_the_metric():
    w = bench.WORKLOADS["train"]
    F = bench.fwd_flops(w)
    assert F == 4 * 2 * 16 * 2048 * 2048 * 128 / 2
    alg = bench.kernel_algorithmic(w)
    kernels = {k: v for k, v in alg.items() if k not in bench.SPAN_KINDS}
    tensor = sum(work for kind, (bound, work) in kernels.items() if bound == "tensor")
    assert tensor == pytest.approx(3.5 * F)  # forward + 2.5x for the backward
    assert alg["bwd_prep"][0] == "hbm"
    # the whole backward call carries the backward's work once
    assert alg["bwd_call"] == ("tensor", pytest.approx(2.5 * F))
    assert sum(alg[k][1] for k in bench.STEP_UNITS) == pytest.approx(3.5 * F)


def test_roofline_picks_the_longer_step_unit_and_uses_the_measured_peak():
    w = bench.WORKLOADS["train"]
    F = bench.fwd_flops(w)
    # dQ and dK/dV overlap: their spans add up to more than the backward call
    res = {"trace_ms": {"fwd": 1.0, "bwd_dkdv": 3.0, "bwd_dq": 2.8, "bwd_prep": 0.5,
                        "bwd_call": 3.6},
           "trace_n": {"fwd": 10, "bwd_dkdv": 10, "bwd_dq": 10, "bwd_prep": 10, "bwd_call": 10}}
    peaks = dict(hbm_gbs=6000.0, bf16=1600.0, bf16_sustained=1400.0, source="test")
    dom, per = bench.roofline(w, res, peaks)
    assert dom == "bwd_call"
    assert per["bwd_call"]["achieved"] == pytest.approx(2.5 * F / 0.36e-3 / 1e12, rel=1e-3)
    assert per["bwd_call"]["peak"] == 1400.0
    assert per["bwd_call"]["frac"] == pytest.approx(per["bwd_call"]["achieved"] / 1400.0, abs=1e-4)
    # shares partition the step over its units, the forward and the backward call
    assert per["fwd"]["share"] + per["bwd_call"]["share"] == pytest.approx(1.0, abs=1e-3)
    assert per["bwd_prep"]["unit"] == "GB/s"
    assert "note" in per["bwd_dq"] and "note" in per["bwd_dkdv"]


def test_ncu_traffic_is_reported_only_for_the_profiled_sources():
    _, rows = bench.load_traffic()
    assert rows, "the traffic table lists no capture"
    key = sorted(rows)[0]
    current = (bench.sources_sha256(), rows)
    b, prof = bench.ncu_traffic(*key, table=current)
    assert b > 0 and os.path.exists(os.path.join(ROOT, prof))
    assert bench.ncu_traffic(*key, table=("0" * 64, rows)) == (None, None)
    assert bench.ncu_traffic(*key, table=("", rows)) == (None, None)
    assert bench.ncu_traffic("train", "no_such_kernel", table=current) == (None, None)


def test_traffic_table_names_existing_summaries_and_known_workloads():
    sha, rows = bench.load_traffic()
    assert len(sha) == 64
    n_decode = len(bench.decode_workloads())
    for (wl, kern), t in rows.items():
        if wl.startswith("decode"):
            assert kern == "decode" and 0 <= int(wl[len("decode"):]) < n_decode
        else:
            assert wl in bench.WORKLOADS
        assert t["bytes"] > 0
        assert os.path.exists(os.path.join(ROOT, t["profile"])), t["profile"]


def test_decode_bytes_count_kv_once():
    w = bench.decode_workloads()[0]
    kv = 2 * w["B"] * w["Nk"] * w["Hkv"] * w["d"] * 2
    assert bench.decode_bytes(w) == kv + 2 * w["B"] * w["Nq"] * w["Hq"] * w["d"] * 2 + \
        4 * w["B"] * w["Hq"] * w["Nq"]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r's loop took (r + 1) * 10 ms for 5 steps of 1e12 FLOP each
        t_local = (rank + 1) * 10.0
        tmax = bench.max_over_ranks(t_local, world)
        tf = bench.job_throughput(1e12, 5, t_local, world)
        bench.barrier(world)
        q.put((rank, tmax, tf))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_time_and_job_throughput():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    world, port = 2, _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, tmax, tf in out:
        assert tmax == 20.0                      # the slowest rank's time
        assert tf == pytest.approx(1e12 * 5 * 2 / 20e-3 / 1e12)  # all ranks' work / max time


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    called = []
    monkeypatch.setattr(bench, "oracle_sample", lambda *a, **k: called.append(1) or (1.0, 1, 1.0, 1))

    class A:
        workload, steps, warmup = "train", 3, 3
    bench.run_reference(A(), world=2, rank=1)
    assert called == [] and capsys.readouterr().out == ""


@pytest.mark.parametrize("N,causal,window", [(7, False, (-1, -1)), (7, True, (-1, -1)), (9, True, (3, 0)),
                                              (9, False, (2, 1)), (5, False, (0, 0))])
def test_visible_pairs_counts_the_mask(N, causal, window):
    # brute force over the visibility rule (Nq = Nk: no bottom-right offset)
    wl, wr = window
    wr = 0 if causal else wr
    n = sum(1 for i in range(N) for j in range(N)
            if (wr < 0 or j <= i + wr) and (wl < 0 or j >= i - wl))
    assert bench.visible_pairs(dict(N=N, causal=causal, window=window)) == n


def test_sweep_covers_the_sequence_length_grid():
    ws = bench.sweep_workloads()
    grid = {(w["N"], w["d"], w["causal"]) for w in ws if w["window"] == (-1, -1) and w["d"] in (64, 128)}
    for N in (512, 1024, 2048, 4096, 8192, 16384):
        for d in (64, 128):
            for c in (False, True):
                assert (N, d, c) in grid
    for w in ws:
        if w["name"].startswith("sweep"):
            assert w["B"] * w["N"] == 16384 and w["H"] * w["d"] == 2048


def test_varlen_flops_reduce_to_the_dense_count():
    w = dict(H=16, d=128, causal=True)
    lens = [2048, 2048]
    dense = bench.fwd_flops(dict(B=2, H=16, N=2048, d=128, causal=True))
    # per sequence L (L + 1) / 2 causal pairs: the diagonal counted, as in the dense kernels' work
    assert bench.varlen_fwd_flops(w, lens) == pytest.approx(dense * (2049 / 2048))
    for wl in bench.varlen_workloads():
        l = bench.varlen_lengths(wl)
        assert sum(l) == wl["tokens"] and max(l) <= wl["hi"] and min(l[:-1]) >= wl["lo"]


def test_blocksparse_masks_have_the_stated_structure():
    import numpy as np
    for w in bench.blocksparse_workloads():
        m = bench.blocksparse_mask(w)
        nb = -(-w["N"] // 128)
        assert m.shape[2:] == (nb, nb) and m.dtype == bool
        if w["pattern"] == "local_global":
            assert m[0, 0].diagonal().all() and m[0, 0, :, 0].all() and m[0, 0, 0, :].all()
        else:
            assert abs(m.mean() - w["density"]) < 0.02


def test_decode_bytes_of_ragged_lengths():
    w = [x for x in bench.decode_workloads() if x.get("ragged")][0]
    row = w["Hkv"] * w["d"] * 2
    lens = bench.decode_lengths(w)
    expect = 2 * row * sum(min(w["Nk"], n + 1) for n in lens) + 4 * w["B"] * row \
        + 2 * w["B"] * w["Nq"] * w["Hq"] * w["d"] * 2 + 4 * w["B"] * w["Hq"] * w["Nq"]
    assert bench.decode_bytes(w) == expect


def test_tensor_peak_is_burst_at_full_clock_and_sustained_when_the_clock_drops():
    peaks = dict(hbm_gbs=6000.0, bf16=1662.1, bf16_sustained=1414.8, source="test")
    full = {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []}
    assert bench.tensor_peak(peaks, full) == (1662.1, "burst")
    # the cap reported, the clock still at its maximum: the full-clock figure
    capped = {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"]}
    assert bench.tensor_peak(peaks, capped) == (1662.1, "burst")
    slow = {"sm_mhz": 1400, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"]}
    assert bench.tensor_peak(peaks, slow) == (1414.8, "sustained")
    assert bench.tensor_peak(peaks, {}) == (1414.8, "sustained")
    w = bench.WORKLOADS["wide"]
    F = bench.fwd_flops(w)
    res = {"trace_ms": {"fwd": 16.0, "bwd_call": 50.0}, "trace_n": {"fwd": 10, "bwd_call": 10},
           "clocks": full}
    dom, per = bench.roofline(w, res, peaks)
    assert dom == "bwd_call" and per[dom]["peak"] == 1662.1 and per[dom]["peak_kind"] == "burst"
    assert per[dom]["frac"] == pytest.approx(2.5 * F / 5e-3 / 1e12 / 1662.1, abs=1e-4)


def test_headline_workload_is_the_long_wide_shape():
    import inspect
    src = inspect.getsource(bench.main)
    assert 'default="wide"' in src
    w = bench.WORKLOADS["wide"]
    assert (w["B"], w["H"], w["N"], w["d"], w["causal"]) == (1, 96, 8192, 128, True)
