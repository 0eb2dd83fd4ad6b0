"""fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY: imported by tests/, by ``__graft_entry__.smoke()`` and
by the CPU-baseline leg of ``bench.py``; never by the product package.  It
shares no code with the CUDA library.

Every function takes numpy arrays in the library's layout -- Q/O/dO
``[B, Nq, Hq, d]``, K/V ``[B, Nk, Hkv, d]``, LSE ``[B, Hq, Nq]`` -- converts
them to fp64 and calls the plain C implementation in ``attn_oracle.c``
(row-by-row definition, two-pass softmax; see that file's header for the
passages each step follows and the readings taken where the pages are silent).
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        i = ctypes.c_int
        lib.oracle_attn_fwd.argtypes = [dp, dp, dp, dp, dp, i, i, i, i, i, i,
                                        ctypes.c_double, i, i, i, i]
        lib.oracle_attn_fwd_blockwise.argtypes = [dp, dp, dp, dp, dp, i, i, i, i, i, i,
                                                  ctypes.c_double, i, i, i, i, i]
        lib.oracle_attn_bwd.argtypes = [dp, dp, dp, dp, dp, dp, dp, i, i, i, i, i, i,
                                        ctypes.c_double, i, i, i, i]
        ip = ctypes.POINTER(ctypes.c_int)
        lib.oracle_attn_fwd_rows.argtypes = [dp, dp, dp, dp, dp, i, i, i, i, i, i,
                                             ctypes.c_double, i, i, i, ip, i, i]
        lib.oracle_attn_dq_rows.argtypes = [dp, dp, dp, dp, dp, i, i, i, i, i, i,
                                            ctypes.c_double, i, i, i, ip, i, i]
        lib.oracle_attn_dkdv_rows.argtypes = [dp, dp, dp, dp, dp, dp, i, i, i, i, i, i,
                                              ctypes.c_double, i, i, i, ip, i, i]
        for f in (lib.oracle_attn_fwd, lib.oracle_attn_fwd_blockwise, lib.oracle_attn_bwd,
                  lib.oracle_attn_fwd_rows, lib.oracle_attn_dq_rows, lib.oracle_attn_dkdv_rows):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _dims(q, k, v):
    if q.ndim != 4 or k.ndim != 4 or v.ndim != 4:
        raise ValueError("expected 4-D [B, N, H, d] arrays")
    B, Nq, Hq, d = q.shape
    Bk, Nk, Hkv, dk = k.shape
    if v.shape != k.shape or Bk != B or dk != d:
        raise ValueError("shape mismatch between q, k and v")
    return B, Nq, Nk, Hq, Hkv, d


def _window(causal, window):
    wl, wr = window if window is not None else (-1, -1)
    return int(bool(causal)), int(wl), int(wr)


def attn_fwd(q, k, v, scale=None, causal=False, window=(-1, -1), nthreads=None):
    """Return (O [B,Nq,Hq,d], LSE [B,Hq,Nq]) in fp64 by the two-pass definition."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Nq, Nk, Hq, Hkv, d = _dims(q, k, v)
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    c, wl, wr = _window(causal, window)
    o = np.empty((B, Nq, Hq, d), np.float64)
    lse = np.empty((B, Hq, Nq), np.float64)
    rc = _load().oracle_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                 B, Nq, Nk, Hq, Hkv, d, scale, c, wl, wr,
                                 nthreads or default_threads())
    if rc != 0:
        raise RuntimeError("oracle_attn_fwd failed (%d)" % rc)
    return o, lse


def attn_fwd_blockwise(q, k, v, block_n, scale=None, causal=False, window=(-1, -1),
                       nthreads=None):
    """Return (O, LSE) by the online-softmax recurrence over key blocks of block_n."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Nq, Nk, Hq, Hkv, d = _dims(q, k, v)
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    c, wl, wr = _window(causal, window)
    o = np.empty((B, Nq, Hq, d), np.float64)
    lse = np.empty((B, Hq, Nq), np.float64)
    rc = _load().oracle_attn_fwd_blockwise(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                           B, Nq, Nk, Hq, Hkv, d, scale, c, wl, wr,
                                           int(block_n), nthreads or default_threads())
    if rc != 0:
        raise RuntimeError("oracle_attn_fwd_blockwise failed (%d)" % rc)
    return o, lse


def attn_bwd(q, k, v, dout, scale=None, causal=False, window=(-1, -1), nthreads=None):
    """Return (dQ, dK, dV) in fp64: gradients of sum(dout * O) by the explicit formulas."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, Nq, Nk, Hq, Hkv, d = _dims(q, k, v)
    if dout.shape != q.shape:
        raise ValueError("dout must have q's shape")
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    c, wl, wr = _window(causal, window)
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    dv = np.empty_like(v)
    rc = _load().oracle_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq),
                                 _ptr(dk), _ptr(dv), B, Nq, Nk, Hq, Hkv, d, scale,
                                 c, wl, wr, nthreads or default_threads())
    if rc != 0:
        raise RuntimeError("oracle_attn_bwd failed (%d)" % rc)
    return dq, dk, dv


def attn_fwd_varlen(q, k, v, cu_q, cu_k, scale=None, causal=False, window=(-1, -1), nthreads=None):
    """Packed variable-length sequences: q [total_q, Hq, d], k/v [total_k, Hkv,
    d], offsets cu_q / cu_k of B + 1 entries.  Each sequence is the plain
    attention of its own rows (attn_fwd with one batch), masks aligned to its
    own lengths.  Returns O [total_q, Hq, d] (zero on rows no sequence covers)
    and LSE [Hq, total_q] (-inf there)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    total_q, Hq, d = q.shape
    o = np.zeros_like(q)
    lse = np.full((Hq, total_q), -np.inf)
    for b in range(len(cu_q) - 1):
        q0, q1, k0, k1 = int(cu_q[b]), int(cu_q[b + 1]), int(cu_k[b]), int(cu_k[b + 1])
        if q1 <= q0:
            continue
        if k1 <= k0:  # no keys at all: every row is empty
            continue
        ob, lb = attn_fwd(q[None, q0:q1], k[None, k0:k1], v[None, k0:k1], scale=scale,
                          causal=causal, window=window, nthreads=nthreads)
        o[q0:q1] = ob[0]
        lse[:, q0:q1] = lb[0]
    return o, lse


def attn_bwd_varlen(q, k, v, dout, cu_q, cu_k, scale=None, causal=False, window=(-1, -1),
                    nthreads=None):
    """Gradients for packed sequences (layouts of attn_fwd_varlen): each
    sequence's own attn_bwd; rows no sequence covers get zero."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b in range(len(cu_q) - 1):
        q0, q1, k0, k1 = int(cu_q[b]), int(cu_q[b + 1]), int(cu_k[b]), int(cu_k[b + 1])
        if q1 <= q0 or k1 <= k0:
            continue
        g = attn_bwd(q[None, q0:q1], k[None, k0:k1], v[None, k0:k1], dout[None, q0:q1],
                     scale=scale, causal=causal, window=window, nthreads=nthreads)
        dq[q0:q1], dk[k0:k1], dv[k0:k1] = g[0][0], g[1][0], g[2][0]
    return dq, dk, dv


def attn_fwd_blockmask(q, k, v, block_mask, block=128, scale=None, causal=False,
                       window=(-1, -1)):
    """Block-sparse attention (abeam.tech FlashAttention summary, the
    block-sparse extension): the definition of attn_fwd with key j also
    hidden from query i when block_mask[b, h, i // block, j // block] is
    zero.  q [B,Nq,Hq,d], k/v [B,Nk,Hkv,d]; block_mask broadcastable to
    [B, Hq, ceil(Nq/block), ceil(Nk/block)].  Plain numpy in fp64, every
    (b, h) materialising its Nq x Nk scores -- for small problems only.
    Rows that see no key: O = 0, LSE = -inf."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Nq, Nk, Hq, Hkv, d = _dims(q, k, v)
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    G = Hq // Hkv
    nqb, nkb = -(-Nq // block), -(-Nk // block)
    bm = np.broadcast_to(np.asarray(block_mask) != 0, (B, Hq, nqb, nkb))
    i = np.arange(Nq)[:, None]
    j = np.arange(Nk)[None, :]
    delta = Nk - Nq
    wl, wr = window if window is not None else (-1, -1)
    wr = 0 if causal else wr
    vis = np.ones((Nq, Nk), dtype=bool)
    if wr >= 0:
        vis &= j <= i + delta + wr
    if wl >= 0:
        vis &= j >= i + delta - wl
    o = np.zeros((B, Nq, Hq, d))
    lse = np.full((B, Hq, Nq), -np.inf)
    for b in range(B):
        for h in range(Hq):
            hk = h // G
            blk = np.repeat(np.repeat(bm[b, h], block, axis=0), block, axis=1)[:Nq, :Nk]
            m = vis & blk
            s = scale * (q[b, :, h, :] @ k[b, :, hk, :].T)
            s = np.where(m, s, -np.inf)
            mx = s.max(axis=1)
            live = np.isfinite(mx)
            p = np.where(m, np.exp(s - np.where(live, mx, 0.0)[:, None]), 0.0)
            l = p.sum(axis=1)
            o[b, live, h, :] = (p[live] @ v[b, :, hk, :]) / l[live, None]
            lse[b, h, live] = mx[live] + np.log(l[live])
    return o, lse


def attn_bwd_blockmask(q, k, v, dout, block_mask, block=128, scale=None, causal=False,
                       window=(-1, -1)):
    """Gradients of sum(dout * O) for attn_fwd_blockmask's O: the backward
    formulas of attn_bwd (D = rowsum(dO * O), dS = P (dP - D), dQ = scale dS K,
    dK = scale dS^T Q, dV = P^T dO, summed over a key/value head's query
    heads) with P zero wherever the block mask or the causal / window masks
    hide a key.  Plain numpy in fp64, for small problems."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, Nq, Nk, Hq, Hkv, d = _dims(q, k, v)
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    G = Hq // Hkv
    nqb, nkb = -(-Nq // block), -(-Nk // block)
    bm = np.broadcast_to(np.asarray(block_mask) != 0, (B, Hq, nqb, nkb))
    i = np.arange(Nq)[:, None]
    j = np.arange(Nk)[None, :]
    delta = Nk - Nq
    wl, wr = window if window is not None else (-1, -1)
    wr = 0 if causal else wr
    vis = np.ones((Nq, Nk), dtype=bool)
    if wr >= 0:
        vis &= j <= i + delta + wr
    if wl >= 0:
        vis &= j >= i + delta - wl
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            hk = h // G
            blk = np.repeat(np.repeat(bm[b, h], block, axis=0), block, axis=1)[:Nq, :Nk]
            m = vis & blk
            s = np.where(m, scale * (q[b, :, h, :] @ k[b, :, hk, :].T), -np.inf)
            mx = s.max(axis=1)
            live = np.isfinite(mx)
            e = np.where(m, np.exp(s - np.where(live, mx, 0.0)[:, None]), 0.0)
            l = e.sum(axis=1)
            p = np.where(live[:, None], e / np.where(live, l, 1.0)[:, None], 0.0)
            o = p @ v[b, :, hk, :]
            do = dout[b, :, h, :]
            Drow = (do * o).sum(axis=1)
            dp = do @ v[b, :, hk, :].T
            ds = p * (dp - Drow[:, None])
            dq[b, :, h, :] = scale * (ds @ k[b, :, hk, :])
            dk[b, :, hk, :] += scale * (ds.T @ q[b, :, h, :])
            dv[b, :, hk, :] += p.T @ do
    return dq, dk, dv


def merge_partials(o_parts, lse_parts):
    """Merge attention results computed over disjoint key subsets.

    o_parts[s] [B, Nq, Hq, d] and lse_parts[s] [B, Hq, Nq] are the outputs of
    attention restricted to the s-th subset (O normalised over that subset,
    LSE its natural log-sum-exp; -inf and O = 0 for a subset with no visible
    key).  The blockwise softmax rule (abeam.tech FlashAttention summary,
    "computing softmax blockwise correctly"), applied to whole subsets:
    with l_s = exp(lse_s) the subset's row sum relative to a common
    reference, the full row sum is sum_s l_s and the full output the l_s
    weighted mean of the O_s.  In log form, relative to m = max_s lse_s:
        lse = m + ln sum_s exp(lse_s - m),   O = sum_s exp(lse_s - lse) O_s.
    Rows with every lse_s = -inf give lse = -inf and O = 0.  fp64 numpy."""
    lse_parts = [np.asarray(x, dtype=np.float64) for x in lse_parts]
    o_parts = [np.asarray(x, dtype=np.float64) for x in o_parts]
    if not lse_parts or len(lse_parts) != len(o_parts):
        raise ValueError("need matching, non-empty lists of partial results")
    ls = np.stack(lse_parts)                       # [S, B, Hq, Nq]
    m = ls.max(axis=0)
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    with np.errstate(invalid="ignore"):
        w = np.where(np.isneginf(ls), 0.0, np.exp(ls - m_safe))
    total = w.sum(axis=0)
    lse = np.where(finite, m_safe + np.log(np.where(finite, total, 1.0)), -np.inf)
    wn = np.where(finite, w / np.where(finite, total, 1.0), 0.0)   # [S, B, Hq, Nq]
    o = np.zeros_like(o_parts[0])
    for s, op in enumerate(o_parts):
        o += np.transpose(wn[s], (0, 2, 1))[..., None] * op     # weights as [B, Nq, Hq, 1]
    return o, lse


def attn_bwd_given_stats(q, k, v, dout, o, lse, scale=None, causal=False, window=(-1, -1)):
    """The share of one key set in the gradients of sum(dout * O), where O
    [B,Nq,Hq,d] and LSE [B,Hq,Nq] are the forward results of the full rows
    (over a key set that contains k/v): the backward formulas of attn_bwd
    with P taken from the given LSE and D from the given O (abeam.tech
    FlashAttention summary, "backward uses recomputation": P is recomputed
    from the saved statistics),
        P = exp(scale q.k - LSE), D = rowsum(dout * O), dS = P (dP - D),
        dQ_share = scale dS K, dK = scale dS^T Q, dV = P^T dout,
    dK / dV summed over a key/value head's query heads.  The causal / window
    masks apply within this set as in attn_fwd (bottom-right aligned).  Over
    a partition of the keys the dQ shares add up to dQ, and each set's dK / dV
    are the rows of the full dK / dV.  Plain numpy in fp64, small problems."""
    q, k, v, dout, o = _f64(q), _f64(k), _f64(v), _f64(dout), _f64(o)
    lse = np.asarray(lse, dtype=np.float64)
    B, Nq, Nk, Hq, Hkv, d = _dims(q, k, v)
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    G = Hq // Hkv
    i = np.arange(Nq)[:, None]
    j = np.arange(Nk)[None, :]
    delta = Nk - Nq
    wl, wr = window if window is not None else (-1, -1)
    wr = 0 if causal else wr
    vis = np.ones((Nq, Nk), dtype=bool)
    if wr >= 0:
        vis &= j <= i + delta + wr
    if wl >= 0:
        vis &= j >= i + delta - wl
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            hk = h // G
            s = scale * (q[b, :, h, :] @ k[b, :, hk, :].T)
            L = lse[b, h, :]
            live = np.isfinite(L)[:, None]
            p = np.where(vis & live, np.exp(np.where(vis & live, s - np.where(live, L[:, None], 0.0), -np.inf)), 0.0)
            do = dout[b, :, h, :]
            Drow = (do * o[b, :, h, :]).sum(axis=1)
            dp = do @ v[b, :, hk, :].T
            ds = p * (dp - Drow[:, None])
            dq[b, :, h, :] = scale * (ds @ k[b, :, hk, :])
            dk[b, :, hk, :] += scale * (ds.T @ q[b, :, h, :])
            dv[b, :, hk, :] += p.T @ do
    return dq, dk, dv


def _rows(rows):
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).ravel())
    return r, r.ctypes.data_as(ctypes.POINTER(ctypes.c_int))


def attn_fwd_rows(q, k, v, rows, scale=None, causal=False, window=(-1, -1), nthreads=None):
    """(O, LSE) for the listed absolute query rows only: O [B, n, Hq, d], LSE [B, Hq, n].
    Each row is computed exactly as attn_fwd computes it."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Nq, Nk, Hq, Hkv, d = _dims(q, k, v)
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    c, wl, wr = _window(causal, window)
    r, rp = _rows(rows)
    o = np.empty((B, len(r), Hq, d), np.float64)
    lse = np.empty((B, Hq, len(r)), np.float64)
    rc = _load().oracle_attn_fwd_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Nq, Nk,
                                      Hq, Hkv, d, scale, c, wl, wr, rp, len(r),
                                      nthreads or default_threads())
    if rc != 0:
        raise RuntimeError("oracle_attn_fwd_rows failed (%d)" % rc)
    return o, lse


def attn_dq_rows(q, k, v, dout, rows, scale=None, causal=False, window=(-1, -1), nthreads=None):
    """dQ for the listed absolute query rows only: [B, n, Hq, d]."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, Nq, Nk, Hq, Hkv, d = _dims(q, k, v)
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    c, wl, wr = _window(causal, window)
    r, rp = _rows(rows)
    dq = np.empty((B, len(r), Hq, d), np.float64)
    rc = _load().oracle_attn_dq_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), B, Nq, Nk,
                                     Hq, Hkv, d, scale, c, wl, wr, rp, len(r),
                                     nthreads or default_threads())
    if rc != 0:
        raise RuntimeError("oracle_attn_dq_rows failed (%d)" % rc)
    return dq


def attn_dkdv_rows(q, k, v, dout, rows, scale=None, causal=False, window=(-1, -1),
                   nthreads=None):
    """(dK, dV) for the listed absolute key rows only: each [B, n, Hkv, d]."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, Nq, Nk, Hq, Hkv, d = _dims(q, k, v)
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    c, wl, wr = _window(causal, window)
    r, rp = _rows(rows)
    dk = np.empty((B, len(r), Hkv, d), np.float64)
    dv = np.empty((B, len(r), Hkv, d), np.float64)
    rc = _load().oracle_attn_dkdv_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dk), _ptr(dv),
                                       B, Nq, Nk, Hq, Hkv, d, scale, c, wl, wr, rp, len(r),
                                       nthreads or default_threads())
    if rc != 0:
        raise RuntimeError("oracle_attn_dkdv_rows failed (%d)" % rc)
    return dk, dv


def fwd_flops(B, Nq, Nk, Hq, d, causal):
    """Forward FLOP count of the metric: 4*B*Hq*Nq*Nk*d, halved when causal."""
    f = 4.0 * B * Hq * Nq * Nk * d
    return f / 2 if causal else f
