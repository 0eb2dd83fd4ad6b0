"""CPU-side checks of the C ABI: the library loads, exports every entry point
include/fa.h declares, and rejects bad arguments with the documented status
codes before anything reaches the GPU (no compute call is made here)."""
import ctypes
import os
import re

import pytest

import exact_io_aware_89_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")

FAKE = 0x10000          # 16-byte aligned, never dereferenced on these paths
MISALIGNED = 0x10008


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_expected_entry_points():
    assert declared_functions() == sorted([
        "fa_fwd", "fa_bwd", "fa_bwd_noalloc", "fa_fwd_f32", "fa_bwd_f32", "fa_bwd_workspace_size",
        "fa_fwd_splitkv", "fa_fwd_splitkv_workspace_size", "fa_fwd_kvcache",
        "fa_fwd_kvcache_workspace_size", "fa_fwd_varlen", "fa_bwd_varlen", "fa_fwd_f16",
        "fa_bwd_f16", "fa_fwd_varlen_f16", "fa_bwd_varlen_f16", "fa_fwd_splitkv_f16", "fa_fwd_kvcache_f16",
        "fa_fwd_blocksparse", "fa_fwd_blocksparse_f16", "fa_bwd_blocksparse", "fa_bwd_blocksparse_f16",
        "fa_get_device_status", "fa_status_string", "fa_trace_enable", "fa_trace_read",
        "fa_lse_merge", "fa_lse_merge_f16", "fa_grad_accumulate", "fa_grad_accumulate_f16",
        "fa_test_withhold_next_load"])


def test_kernel_kinds_match_the_header():
    header = open(HEADER).read()
    kinds = re.findall(r"\bFA_KERNEL_([A-Z0-9_]+)\s*=\s*(\d+)", header)
    named = {int(v): n.lower() for n, v in kinds if n != "KINDS"}
    n_kinds = int(dict(kinds)["KINDS"])
    assert [named[i] for i in range(n_kinds)] == list(fa.KERNEL_KINDS)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(fa.library_path())
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert hasattr(fa, name), name


def test_status_strings():
    names = ["FA_OK", "FA_ERR_INVALID_ARG", "FA_ERR_UNSUPPORTED", "FA_ERR_CUDA",
             "FA_ERR_WORKSPACE", "FA_ERR_TIMEOUT"]
    for code, name in enumerate(names):
        assert fa.fa_status_string(code) == name
    assert fa.fa_status_string(99) == "FA_UNKNOWN_STATUS"
    header = open(HEADER).read()
    for code, name in enumerate(names):
        assert re.search(r"\b%s\s*=\s*%d\b" % (name, code), header), name


def test_workspace_size():
    # D and lse2 rows, fp32, rows padded to a multiple of 256
    assert fa.fa_bwd_workspace_size(2, 2048, 16, 128) == 2 * 2 * 16 * 2048 * 4
    assert fa.fa_bwd_workspace_size(1, 1, 1, 64) == 2 * 256 * 4
    assert fa.fa_bwd_workspace_size(1, 257, 3, 64) == 2 * 3 * 512 * 4
    assert fa.fa_bwd_workspace_size(0, 128, 2, 64) == 0
    assert fa.fa_bwd_workspace_size(1, 0, 2, 64) == 0


def _fwd(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Nq=128, Nk=128, Hq=2, Hkv=2, d=64,
             scale=0.125, causal=0, win_l=-1, win_r=-1, stream=None)
    a.update(kw)
    return fa.fa_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Nq"], a["Nk"], a["Hq"],
                     a["Hkv"], a["d"], a["scale"], a["causal"], a["win_l"], a["win_r"], a["stream"])


def _bwd(f32=False, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, dO=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, B=1,
             Nq=128, Nk=128, Hq=2, Hkv=2, d=64, scale=0.125, causal=0, win_l=-1, win_r=-1,
             ws=FAKE, wsb=1 << 20, stream=None)
    a.update(kw)
    fn = fa.fa_bwd_f32 if f32 else fa.fa_bwd
    return fn(a["q"], a["k"], a["v"], a["o"], a["lse"], a["dO"], a["dq"], a["dk"], a["dv"], a["B"],
              a["Nq"], a["Nk"], a["Hq"], a["Hkv"], a["d"], a["scale"], a["causal"], a["win_l"],
              a["win_r"], a["ws"], a["wsb"], a["stream"])


INVALID, UNSUPPORTED, WORKSPACE = 1, 2, 4


@pytest.mark.parametrize("kw", [
    dict(q=0), dict(k=0), dict(v=0), dict(o=0), dict(lse=0),
    dict(q=MISALIGNED), dict(o=MISALIGNED),
    dict(B=0), dict(Nq=0), dict(Nk=-1), dict(Hq=0), dict(Hkv=0),
    dict(Hq=6, Hkv=4),                       # Hq % Hkv != 0
    dict(scale=float("nan")), dict(scale=float("inf")), dict(scale=0.0), dict(scale=-1.0),
])
def test_fwd_rejects_invalid_arguments(kw):
    assert _fwd(**kw) == INVALID


@pytest.mark.parametrize("d", [0, 32, 96, 100, 192, 512])
def test_fwd_rejects_unsupported_head_dim(d):
    assert _fwd(d=d) == UNSUPPORTED


@pytest.mark.parametrize("kw", [dict(dO=0), dict(dq=MISALIGNED), dict(dk=0), dict(dv=0),
                                dict(Hq=3, Hkv=2), dict(B=-2)])
def test_bwd_rejects_invalid_arguments(kw):
    assert _bwd(**kw) == INVALID
    assert _bwd(f32=True, **kw) == INVALID


def test_bwd_rejects_small_or_missing_workspace():
    need = fa.fa_bwd_workspace_size(1, 128, 2, 64)
    assert _bwd(wsb=need - 4) == WORKSPACE
    assert _bwd(ws=0) == WORKSPACE
    assert _bwd(ws=MISALIGNED, wsb=need) == WORKSPACE
    assert _bwd(d=96) == UNSUPPORTED


def test_f32_head_dim_limits():
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE)
    for d in (16, 48, 288):
        assert fa.fa_fwd_f32(a["q"], a["k"], a["v"], a["o"], a["lse"], 1, 8, 8, 1, 1, d, 0.1, 0, -1,
                             -1, None) == UNSUPPORTED


# ------------------------------------------------------------ split-KV forward

def _splitkv(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=2, Nq=1, Nk=1000, Hq=8, Hkv=2, d=128,
             scale=0.125, causal=0, win_l=-1, win_r=-1, n_splits=4, ws=0, wsb=0, stream=None)
    a.update(kw)
    return fa.fa_fwd_splitkv(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Nq"], a["Nk"],
                             a["Hq"], a["Hkv"], a["d"], a["scale"], a["causal"], a["win_l"],
                             a["win_r"], a["n_splits"], a["ws"], a["wsb"], a["stream"])


def test_splitkv_workspace_size():
    # rows of one query tile = queries per tile * group; the partial O rows
    # (fp32, d wide) of every (batch, kv head, query tile, split), then their
    # LSE, then (16-byte aligned) one 8-byte counter per unit
    def expect(units, splits, rows, d):
        n = units * splits * rows
        return (n * d * 4 + n * 4 + 15) // 16 * 16 + 8 * units
    ws = fa.fa_fwd_splitkv_workspace_size
    assert ws(2, 1, 1000, 8, 2, 128, 0, -1, -1, 4) == expect(2 * 2, 4, 4, 128)
    # group 4: 32 queries per tile, 40 queries -> 2 tiles of 128 packed rows
    assert ws(1, 40, 4096, 8, 2, 64, 1, -1, -1, 3) == expect(1 * 2 * 2, 3, 128, 64)
    # MQA with 32 query heads: up to 4 queries per tile, here both of the 2
    assert ws(3, 2, 512, 32, 1, 256, 0, 100, 0, 2) == expect(3 * 1 * 1, 2, 64, 256)
    assert ws(2, 1, 1000, 8, 2, 128, 0, -1, -1, 1) == 0          # no split, no workspace
    assert ws(1, 1, 1000, 256, 1, 128, 0, -1, -1, 4) == 0        # group > 128: unsupported
    assert ws(1, 1, 1000, 8, 2, 96, 0, -1, -1, 4) == 0           # head dim
    assert ws(1, 1, 1000, 6, 4, 128, 0, -1, -1, 4) == 0          # Hq % Hkv
    assert ws(1, 1, 1000, 8, 2, 128, 0, -1, -1, 5000) == 0       # too many splits


@pytest.mark.parametrize("kw", [
    dict(q=0), dict(k=MISALIGNED), dict(o=0), dict(lse=MISALIGNED), dict(B=0), dict(Nk=0),
    dict(Hq=6, Hkv=4), dict(scale=float("nan")), dict(n_splits=5000),
])
def test_splitkv_rejects_invalid_arguments(kw):
    assert _splitkv(**kw) == INVALID


def test_splitkv_rejects_unsupported_and_missing_workspace():
    assert _splitkv(d=96) == UNSUPPORTED
    assert _splitkv(Hq=256, Hkv=1) == UNSUPPORTED
    need = fa.fa_fwd_splitkv_workspace_size(2, 1, 1000, 8, 2, 128, 0, -1, -1, 4)
    assert need > 0
    assert _splitkv(ws=0, wsb=need) == WORKSPACE
    assert _splitkv(ws=FAKE, wsb=need - 4) == WORKSPACE
    assert _splitkv(ws=MISALIGNED, wsb=need) == WORKSPACE


def _kvcache(**kw):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, kn=FAKE, vn=FAKE, sl=FAKE, o=FAKE, lse=FAKE, B=2, Nq=1,
             Nk=1000, n_new=1, Hq=8, Hkv=2, d=128, scale=0.125, causal=1, win_l=-1, win_r=-1,
             n_splits=4, ws=FAKE, wsb=1 << 20, stream=None)
    a.update(kw)
    return fa.fa_fwd_kvcache(a["q"], a["kc"], a["vc"], a["kn"], a["vn"], a["sl"], a["o"], a["lse"],
                             a["B"], a["Nq"], a["Nk"], a["n_new"], a["Hq"], a["Hkv"], a["d"],
                             a["scale"], a["causal"], a["win_l"], a["win_r"], a["n_splits"], a["ws"],
                             a["wsb"], a["stream"])


@pytest.mark.parametrize("kw", [
    dict(q=0), dict(kc=0), dict(vc=MISALIGNED), dict(o=0), dict(lse=0), dict(B=0), dict(Nk=0),
    dict(n_new=-1), dict(kn=0), dict(vn=MISALIGNED), dict(sl=0), dict(sl=FAKE + 2),
    dict(Hq=6, Hkv=4), dict(scale=float("inf")), dict(n_splits=5000),
])
def test_kvcache_rejects_invalid_arguments(kw):
    assert _kvcache(**kw) == INVALID


def test_kvcache_rejects_unsupported_and_missing_workspace():
    assert _kvcache(d=96) == UNSUPPORTED
    assert _kvcache(Hq=512, Hkv=2) == UNSUPPORTED
    assert _kvcache(ws=0) == WORKSPACE
    assert _kvcache(wsb=16) == WORKSPACE


def _varlen(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, cq=FAKE, ck=FAKE, B=3, mq=100, mk=120, tq=200,
             tk=250, Hq=4, Hkv=2, d=128, scale=0.125, causal=1, win_l=-1, win_r=-1, stream=None)
    a.update(kw)
    return fa.fa_fwd_varlen(a["q"], a["k"], a["v"], a["o"], a["lse"], a["cq"], a["ck"], a["B"],
                            a["mq"], a["mk"], a["tq"], a["tk"], a["Hq"], a["Hkv"], a["d"], a["scale"],
                            a["causal"], a["win_l"], a["win_r"], a["stream"])


@pytest.mark.parametrize("kw", [
    dict(q=0), dict(k=MISALIGNED), dict(o=0), dict(lse=MISALIGNED), dict(cq=0), dict(ck=0),
    dict(cq=FAKE + 2), dict(B=0), dict(mq=0), dict(mk=0), dict(mq=201), dict(mk=251), dict(tq=0),
    dict(Hq=3), dict(scale=float("nan")),
])
def test_varlen_rejects_invalid_arguments(kw):
    assert _varlen(**kw) == INVALID


def test_varlen_rejects_unsupported_head_dim():
    assert _varlen(d=96) == UNSUPPORTED


def _bwd_varlen(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, dO=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, cq=FAKE,
             ck=FAKE, B=3, mq=100, mk=120, tq=200, tk=250, Hq=4, Hkv=2, d=128, scale=0.125, causal=1,
             win_l=-1, win_r=-1, ws=FAKE, wsb=1 << 20, stream=None)
    a.update(kw)
    return fa.fa_bwd_varlen(a["q"], a["k"], a["v"], a["o"], a["lse"], a["dO"], a["dq"], a["dk"],
                            a["dv"], a["cq"], a["ck"], a["B"], a["mq"], a["mk"], a["tq"], a["tk"],
                            a["Hq"], a["Hkv"], a["d"], a["scale"], a["causal"], a["win_l"],
                            a["win_r"], a["ws"], a["wsb"], a["stream"])


@pytest.mark.parametrize("kw", [
    dict(dO=0), dict(dq=MISALIGNED), dict(dk=0), dict(dv=0), dict(cq=0), dict(ck=FAKE + 1),
    dict(B=0), dict(mq=0), dict(mk=251), dict(Hq=3), dict(scale=0.0),
])
def test_bwd_varlen_rejects_invalid_arguments(kw):
    assert _bwd_varlen(**kw) == INVALID


def test_bwd_varlen_workspace_and_head_dim():
    need = fa.fa_bwd_workspace_size(3, 100, 4, 128)   # per sequence, padded to the longest
    assert _bwd_varlen(wsb=need - 4) == WORKSPACE
    assert _bwd_varlen(ws=0) == WORKSPACE
    assert _bwd_varlen(d=96) == UNSUPPORTED


def test_fp16_entry_points_check_arguments_like_bf16():
    assert fa.fa_fwd_f16(0, FAKE, FAKE, FAKE, FAKE, 1, 128, 128, 2, 2, 64, 0.125, 0, -1, -1,
                         None) == INVALID
    assert fa.fa_fwd_f16(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 128, 128, 2, 2, 96, 0.125, 0, -1, -1,
                         None) == UNSUPPORTED
    assert fa.fa_bwd_f16(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 128, 128, 2, 2,
                         64, 0.125, 0, -1, -1, 0, 0, None) == WORKSPACE


def test_blocksparse_rejects_invalid_arguments():
    def call(**kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, m=FAKE, sb=0, sh=0, B=1, Nq=256, Nk=256,
                 Hq=2, Hkv=2, d=128, scale=0.1, causal=0, wl=-1, wr=-1)
        a.update(kw)
        return fa.fa_fwd_blocksparse(a["q"], a["k"], a["v"], a["o"], a["lse"], a["m"], a["sb"],
                                     a["sh"], a["B"], a["Nq"], a["Nk"], a["Hq"], a["Hkv"], a["d"],
                                     a["scale"], a["causal"], a["wl"], a["wr"], None)
    assert call(m=0) == INVALID
    assert call(sb=-1) == INVALID
    assert call(q=MISALIGNED) == INVALID
    assert call(Hq=3) == INVALID
    assert call(d=96) == UNSUPPORTED


def test_ring_combining_calls_reject_invalid_arguments_before_launching():
    ok = dict(o_acc=FAKE, lse_acc=FAKE, o_part=FAKE, lse_part=FAKE, o_out=None, B=1, Nq=8, H=2, d=64, Nq_acc=8,
              row0=0, first=1)

    def merge(**kw):
        a = dict(ok, **kw)
        return fa.fa_lse_merge(a["o_acc"], a["lse_acc"], a["o_part"], a["lse_part"], a["o_out"], a["B"],
                               a["Nq"], a["H"], a["d"], a["Nq_acc"], a["row0"], a["first"], None)
    for kw in (dict(o_acc=0), dict(lse_part=FAKE + 4), dict(o_out=FAKE + 8), dict(B=0), dict(Nq=0), dict(H=-1),
               dict(Nq_acc=7), dict(row0=-1), dict(Nq_acc=16, row0=9)):
        assert merge(**kw) == INVALID, kw
    assert merge(d=96) == UNSUPPORTED
    assert merge(d=96, Nq_acc=16, row0=8) == UNSUPPORTED         # rows in range, head size not
    assert fa.fa_lse_merge_f16(FAKE, FAKE, FAKE, FAKE, None, 1, 8, 2, 100, 8, 0, 0, None) == UNSUPPORTED
    okg = dict(acc=FAKE, part=FAKE, out=None, B=1, rows_acc=1, row0=0, rows=1, row_elems=16, first=0)

    def acc(**kw):
        a = dict(okg, **kw)
        return fa.fa_grad_accumulate(a["acc"], a["part"], a["out"], a["B"], a["rows_acc"], a["row0"], a["rows"],
                                     a["row_elems"], a["first"], None)
    for kw in (dict(row_elems=12),                 # not a multiple of 8
               dict(row_elems=0), dict(part=None),  # nothing to do
               dict(acc=FAKE + 4),                  # misaligned
               dict(B=0), dict(B=65536), dict(rows=0), dict(rows_acc=2, rows=3),
               dict(rows_acc=4, row0=2, rows=3), dict(row0=-1)):
        assert acc(**kw) == INVALID, kw
    assert fa.fa_grad_accumulate_f16(0, FAKE, None, 1, 1, 0, 1, 16, 0, None) == INVALID
