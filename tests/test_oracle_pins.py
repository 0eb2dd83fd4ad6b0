"""Pins for the fp64 oracle: things the pages and the mathematics fix, checked
against the oracle so that it is not trusted on its own word.

Each test names the fact it uses.  Together they are chosen so that a plausible
slip in the oracle (a dropped rescale, a wrong sign, a transposed operand, the
wrong GQA head, an off-by-one in the mask, a misplaced scale) fails at least
one of them.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def _eval(x):
    return eval(str(x), {"__builtins__": {}}, {"log": math.log, "inf": math.inf})


def _arr(nested):
    return np.vectorize(_eval, otypes=[np.float64])(np.array(nested, dtype=object))


def _rand(shape, rng):
    return rng.standard_normal(shape)


def n_visible(i, Nq, Nk, causal, wl, wr):
    """Count of visible keys for query i under the stated reading (inclusive
    window bounds, bottom-right alignment, negative = unbounded)."""
    delta = Nk - Nq
    wr = 0 if causal else wr
    lo = 0 if wl < 0 else max(0, i + delta - wl)
    hi = Nk - 1 if wr < 0 else min(Nk - 1, i + delta + wr)
    return max(0, hi - lo + 1), lo, hi


# ---------------------------------------------------------------- golden cases

with open(os.path.join(HERE, "golden", "closed_form_cases.json")) as f:
    GOLDEN = json.load(f)["cases"]


@pytest.mark.parametrize("case", GOLDEN, ids=[c["name"] for c in GOLDEN])
def test_golden_closed_form(case):
    """Hand-derived exact values (tests/golden/closed_form_cases.json)."""
    q, k, v = _arr(case["q"]), _arr(case["k"]), _arr(case["v"])
    scale = _eval(case["scale"])
    wl, wr = case["window"]
    o, lse = oracle.attn_fwd(q, k, v, scale=scale, causal=case["causal"], window=(wl, wr),
                             nthreads=2)
    np.testing.assert_allclose(o, _arr(case["o"]), rtol=1e-13, atol=1e-13)
    exp_lse = _arr(case["lse"])
    assert np.array_equal(np.isinf(lse), np.isinf(exp_lse))
    fin = np.isfinite(exp_lse)
    np.testing.assert_allclose(lse[fin], exp_lse[fin], rtol=1e-13, atol=1e-13)
    if "dq" in case:
        dq, dk, dv = oracle.attn_bwd(q, k, v, _arr(case["do"]), scale=scale,
                                     causal=case["causal"], window=(wl, wr), nthreads=1)
        np.testing.assert_allclose(dq, _arr(case["dq"]), rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(dk, _arr(case["dk"]), rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(dv, _arr(case["dv"]), rtol=1e-13, atol=1e-13)


# ------------------------------------------------------------ closed forms

MASKS = [(False, -1, -1), (True, -1, -1), (True, 5, -1), (False, 3, 2), (False, -1, 4)]


@pytest.mark.parametrize("causal,wl,wr", MASKS)
@pytest.mark.parametrize("Nq,Nk", [(9, 9), (5, 12), (12, 5)])
def test_identical_keys_give_mean_of_visible_values(causal, wl, wr, Nq, Nk):
    """All keys equal -> P uniform over the visible keys: O_i is the mean of the
    visible V rows and LSE_i = s_i + ln(n_visible_i).  Also pins the exact mask
    reading through n_visible."""
    rng = np.random.default_rng(1)
    d, Hq, Hkv = 4, 4, 2
    q = _rand((1, Nq, Hq, d), rng)
    kvec = _rand((d,), rng)
    k = np.broadcast_to(kvec, (1, Nk, Hkv, d)).copy()
    v = _rand((1, Nk, Hkv, d), rng)
    scale = 0.7
    o, lse = oracle.attn_fwd(q, k, v, scale=scale, causal=causal, window=(wl, wr), nthreads=3)
    for h in range(Hq):
        hk = h // (Hq // Hkv)
        for i in range(Nq):
            n, lo, hi = n_visible(i, Nq, Nk, causal, wl, wr)
            if n == 0:
                assert np.all(o[0, i, h] == 0) and lse[0, h, i] == -np.inf
                continue
            np.testing.assert_allclose(o[0, i, h], v[0, lo:hi + 1, hk].mean(axis=0),
                                       rtol=1e-12, atol=1e-12)
            s = scale * q[0, i, h] @ kvec
            assert abs(lse[0, h, i] - (s + math.log(n))) < 1e-12


def test_dominant_score_selects_its_value_row():
    """One key's scaled score exceeds all others by Delta ->
    |O_i - V_j*| <= (n-1) e^-Delta max|V| (per element)."""
    rng = np.random.default_rng(2)
    Nk, d = 16, 8
    q = np.zeros((1, 1, 1, d)); q[0, 0, 0, 0] = 1.0
    k = 0.1 * _rand((1, Nk, 1, d), rng)
    k[0, :, 0, 0] = rng.uniform(-1, 1, Nk)
    jstar = 11
    delta = 12.0
    k[0, jstar, 0, 0] = k[0, :, 0, 0].max() + delta
    v = _rand((1, Nk, 1, d), rng)
    o, _ = oracle.attn_fwd(q, k, v, scale=1.0, nthreads=1)
    bound = (Nk - 1) * math.exp(-delta) * np.abs(v).max()
    assert np.abs(o[0, 0, 0] - v[0, jstar, 0]).max() <= bound


def test_causal_row_zero_is_v0():
    """Causal, Nq == Nk: row 0 sees only key 0, so O_0 = V_0 and LSE_0 = S_00."""
    rng = np.random.default_rng(3)
    q, k, v = (_rand((2, 7, 3, 5), rng) for _ in range(3))
    o, lse = oracle.attn_fwd(q, k, v, scale=0.3, causal=True, nthreads=2)
    np.testing.assert_array_equal(o[:, 0], v[:, 0])
    np.testing.assert_allclose(lse[:, :, 0], 0.3 * np.einsum("bhc,bhc->bh", q[:, 0], k[:, 0]),
                               rtol=1e-14, atol=1e-14)


def test_two_keys_reduce_to_logistic():
    """With two visible keys softmax is the logistic function:
    O = v0 + (v1 - v0) * sigmoid(s1 - s0), LSE = s0 + log1p(exp(s1 - s0))."""
    rng = np.random.default_rng(4)
    q = _rand((1, 6, 2, 3), rng)
    k = _rand((1, 2, 2, 3), rng)
    v = _rand((1, 2, 2, 3), rng)
    o, lse = oracle.attn_fwd(q, k, v, scale=1.3, nthreads=1)
    for h in range(2):
        s0 = 1.3 * q[0, :, h] @ k[0, 0, h]
        s1 = 1.3 * q[0, :, h] @ k[0, 1, h]
        sig = 1.0 / (1.0 + np.exp(-(s1 - s0)))
        exp_o = v[0, 0, h] + (v[0, 1, h] - v[0, 0, h]) * sig[:, None]
        np.testing.assert_allclose(o[0, :, h], exp_o, rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(lse[0, h], s0 + np.log1p(np.exp(s1 - s0)), rtol=1e-13)


# -------------------------------------------------- recurrence == definition

@pytest.mark.parametrize("block", [1, 3, 16, 40])
@pytest.mark.parametrize("causal,wl,wr", MASKS)
def test_online_recurrence_equals_two_pass(block, causal, wl, wr):
    """The blockwise online softmax (running max/sum and O rescaled by
    exp(m_old - m_new)) equals the two-pass softmax to rounding."""
    rng = np.random.default_rng(5)
    q = 3.0 * _rand((1, 23, 4, 8), rng)   # peaked rows exercise the rescale
    k = _rand((1, 40, 2, 8), rng)
    v = _rand((1, 40, 2, 8), rng)
    o1, l1 = oracle.attn_fwd(q, k, v, scale=0.5, causal=causal, window=(wl, wr), nthreads=2)
    o2, l2 = oracle.attn_fwd_blockwise(q, k, v, block, scale=0.5, causal=causal,
                                       window=(wl, wr), nthreads=2)
    np.testing.assert_allclose(o2, o1, rtol=1e-13, atol=1e-13)
    assert np.array_equal(np.isinf(l1), np.isinf(l2))
    fin = np.isfinite(l1)
    np.testing.assert_allclose(l2[fin], l1[fin], rtol=1e-13, atol=1e-13)


# ------------------------------------------------------- finite differences

def _loss(q, k, v, do, **kw):
    o, _ = oracle.attn_fwd(q, k, v, nthreads=1, **kw)
    return float(np.sum(do * o))


@pytest.mark.parametrize("shape,causal,wl,wr", [
    ((1, 6, 2, 2, 4), False, -1, -1),
    ((1, 7, 2, 1, 3), True, -1, -1),   # GQA 2:1, causal
    ((2, 5, 4, 2, 3), True, 2, -1),    # window + GQA
    ((1, 4, 1, 1, 5), False, 1, 1),    # band
])
def test_gradients_match_central_differences(shape, causal, wl, wr):
    """Analytic dQ, dK, dV equal central differences of L = sum(dO * O)
    (h = 1e-6) on tiny fp64 inputs; pins the backward formulas, the scale in
    dQ/dK and the GQA reduction of dK/dV."""
    B, N, Hq, Hkv, d = shape
    rng = np.random.default_rng(6)
    q = _rand((B, N, Hq, d), rng)
    k = _rand((B, N + 1, Hkv, d), rng)   # Nq != Nk as well
    v = _rand((B, N + 1, Hkv, d), rng)
    do = _rand((B, N, Hq, d), rng)
    kw = dict(scale=0.8, causal=causal, window=(wl, wr))
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, nthreads=2, **kw)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = x.copy(); xp[idx] += h
            xm = x.copy(); xm[idx] -= h
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            lp = _loss(args["q"], args["k"], args["v"], do, **kw)
            args[name] = xm
            lm = _loss(args["q"], args["k"], args["v"], do, **kw)
            num[idx] = (lp - lm) / (2 * h)
        err = np.abs(num - g).max() / max(1e-12, np.abs(g).max())
        assert err < 1e-6, (name, err)


# --------------------------------------------------------------- invariants

def _rand_qkv(rng, B=1, Nq=17, Nk=17, Hq=2, Hkv=2, d=6):
    return (_rand((B, Nq, Hq, d), rng), _rand((B, Nk, Hkv, d), rng),
            _rand((B, Nk, Hkv, d), rng), _rand((B, Nq, Hq, d), rng))


@pytest.mark.parametrize("causal", [False, True])
def test_gradient_sums(causal):
    """Rows of P sum to 1 -> sum_j dV_j = sum_i dO_i; rows of dS sum to 0 ->
    sum_j dK_j = 0 (per head, MHA, every row has a visible key)."""
    rng = np.random.default_rng(7)
    q, k, v, do = _rand_qkv(rng)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, scale=0.4, causal=causal, nthreads=2)
    np.testing.assert_allclose(dv.sum(axis=1), do.sum(axis=1), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-12)


def test_key_shift_invariance():
    """Adding u to every key leaves O unchanged and shifts LSE_i by scale*q_i.u."""
    rng = np.random.default_rng(8)
    q, k, v, _ = _rand_qkv(rng)
    u = 5.0 * _rand((6,), rng)
    o1, l1 = oracle.attn_fwd(q, k, v, scale=0.5, causal=True, nthreads=2)
    o2, l2 = oracle.attn_fwd(q, k + u, v, scale=0.5, causal=True, nthreads=2)
    np.testing.assert_allclose(o2, o1, rtol=1e-11, atol=1e-11)
    shift = 0.5 * np.einsum("bihc,c->bhi", q, u)
    np.testing.assert_allclose(l2, l1 + shift, rtol=1e-11, atol=1e-11)


def test_permutation_invariance_non_causal():
    """Permuting keys and values together leaves O and LSE unchanged (no mask)."""
    rng = np.random.default_rng(9)
    q, k, v, _ = _rand_qkv(rng)
    perm = rng.permutation(k.shape[1])
    o1, l1 = oracle.attn_fwd(q, k, v, nthreads=2)
    o2, l2 = oracle.attn_fwd(q, k[:, perm], v[:, perm], nthreads=2)
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(l2, l1, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("causal,wl", [(False, -1), (True, 4)])
def test_gqa_equals_mha_with_repeated_kv(causal, wl):
    """GQA (Hq = 4, Hkv = 2) equals MHA with each KV head repeated for its group
    (contiguous groups), and GQA dK/dV are the group sums of the MHA ones."""
    rng = np.random.default_rng(10)
    q, k, v, do = _rand_qkv(rng, Hq=4, Hkv=2)
    kr, vr = np.repeat(k, 2, axis=2), np.repeat(v, 2, axis=2)
    kw = dict(scale=0.6, causal=causal, window=(wl, -1), nthreads=2)
    o1, l1 = oracle.attn_fwd(q, k, v, **kw)
    o2, l2 = oracle.attn_fwd(q, kr, vr, **kw)
    np.testing.assert_allclose(o1, o2, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=1e-13, atol=1e-13)
    dq1, dk1, dv1 = oracle.attn_bwd(q, k, v, do, **kw)
    dq2, dk2, dv2 = oracle.attn_bwd(q, kr, vr, do, **kw)
    np.testing.assert_allclose(dq1, dq2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dk1, dk2.reshape(1, 17, 2, 2, 6).sum(axis=3), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dv1, dv2.reshape(1, 17, 2, 2, 6).sum(axis=3), rtol=1e-12, atol=1e-12)


def test_output_is_convex_combination_of_values():
    """O_i is a convex combination of V rows: min_j V_jc <= O_ic <= max_j V_jc."""
    rng = np.random.default_rng(11)
    q, k, v, _ = _rand_qkv(rng)
    q *= 4
    o, _ = oracle.attn_fwd(q, k, v, causal=False, nthreads=2)
    assert np.all(o <= v.max(axis=1, keepdims=True) + 1e-12)
    assert np.all(o >= v.min(axis=1, keepdims=True) - 1e-12)


def test_thread_count_does_not_change_results():
    """The oracle is reproducible: 1 and 5 threads give identical bits."""
    rng = np.random.default_rng(12)
    q, k, v, do = _rand_qkv(rng, Hq=4, Hkv=2)
    a = oracle.attn_bwd(q, k, v, do, causal=True, nthreads=1)
    b = oracle.attn_bwd(q, k, v, do, causal=True, nthreads=5)
    for x, y in zip(a, b):
        # dK/dV sums are re-associated across thread slices: equal to rounding
        np.testing.assert_allclose(x, y, rtol=1e-13, atol=1e-13)
    o1, _ = oracle.attn_fwd(q, k, v, nthreads=1)
    o2, _ = oracle.attn_fwd(q, k, v, nthreads=5)
    np.testing.assert_array_equal(o1, o2)


# ------------------------------------------------------- selected-row oracle

@pytest.mark.parametrize("causal,wl,wr", [(False, -1, -1), (True, -1, -1), (True, 3, -1)])
def test_selected_rows_equal_full_functions(causal, wl, wr):
    """The row-subset oracle (used to check large problems on a sample) returns
    exactly the rows of the full functions, which the tests above pin."""
    rng = np.random.default_rng(13)
    q, k, v, do = (_rand(s, rng) for s in [(2, 11, 4, 5), (2, 14, 2, 5), (2, 14, 2, 5), (2, 11, 4, 5)])
    kw = dict(scale=0.7, causal=causal, window=(wl, wr))
    o, lse = oracle.attn_fwd(q, k, v, nthreads=3, **kw)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, nthreads=1, **kw)
    rows = [0, 3, 10, 4]
    o_r, lse_r = oracle.attn_fwd_rows(q, k, v, rows, nthreads=2, **kw)
    np.testing.assert_array_equal(o_r, o[:, rows])
    np.testing.assert_array_equal(lse_r, lse[:, :, rows])
    np.testing.assert_array_equal(oracle.attn_dq_rows(q, k, v, do, rows, nthreads=2, **kw), dq[:, rows])
    krows = [13, 0, 7]
    dk_r, dv_r = oracle.attn_dkdv_rows(q, k, v, do, krows, nthreads=3, **kw)
    np.testing.assert_allclose(dk_r, dk[:, krows], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(dv_r, dv[:, krows], rtol=1e-13, atol=1e-13)


# ------------------------------------------------- merging partial results

def _subset_result(q, k, v, idx, scale):
    """Attention restricted to the keys in idx (non-causal); an empty subset
    gives O = 0 and LSE = -inf."""
    B, Nq, Hq, d = q.shape
    if len(idx) == 0:
        return np.zeros((B, Nq, Hq, d)), np.full((B, Hq, Nq), -np.inf)
    return oracle.attn_fwd(q, k[:, idx], v[:, idx], scale=scale)


@pytest.mark.parametrize("n_parts", [1, 2, 4, 7])
def test_merge_of_key_subsets_equals_attention_over_all_keys(n_parts):
    """Splitting the keys into disjoint subsets (contiguous or scattered, one
    possibly empty), attending over each and merging gives attention over all
    keys: the merge is pinned to the two-pass definition."""
    rng = np.random.default_rng(40 + n_parts)
    B, Nq, Nk, Hq, Hkv, d = 2, 5, 23, 4, 2, 8
    q = rng.standard_normal((B, Nq, Hq, d))
    k = rng.standard_normal((B, Nk, Hkv, d))
    v = rng.standard_normal((B, Nk, Hkv, d))
    scale = 0.7
    labels = rng.integers(0, n_parts, Nk)
    if n_parts > 2:
        labels[labels == n_parts - 1] = 0          # the last subset is empty
    parts = [_subset_result(q, k, v, np.flatnonzero(labels == s), scale) for s in range(n_parts)]
    o, lse = oracle.merge_partials([p[0] for p in parts], [p[1] for p in parts])
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, scale=scale)
    assert np.abs(o - o_ref).max() < 1e-12
    assert np.abs(lse - lse_ref).max() < 1e-12


def test_merge_of_contiguous_splits_is_order_free():
    rng = np.random.default_rng(7)
    q = rng.standard_normal((1, 3, 2, 4))
    k = rng.standard_normal((1, 40, 2, 4))
    v = rng.standard_normal((1, 40, 2, 4))
    cuts = [0, 9, 10, 31, 40]
    parts = [_subset_result(q, k, v, np.arange(a, b), 0.5) for a, b in zip(cuts, cuts[1:])]
    o1, l1 = oracle.merge_partials([p[0] for p in parts], [p[1] for p in parts])
    o2, l2 = oracle.merge_partials([p[0] for p in parts[::-1]], [p[1] for p in parts[::-1]])
    assert np.abs(o1 - o2).max() < 1e-14 and np.abs(l1 - l2).max() < 1e-14


def test_merge_rows_without_keys():
    """A row whose every subset is empty stays empty (LSE -inf, O 0); a row
    with one non-empty subset gets exactly that subset's result."""
    o_a = np.ones((1, 2, 1, 3))
    o_b = np.full((1, 2, 1, 3), 2.0)
    lse_a = np.array([[[-np.inf, 0.25]]])
    lse_b = np.array([[[-np.inf, -np.inf]]])
    o_b[:, 1] = 0.0
    o_a[:, 0] = 0.0
    o, lse = oracle.merge_partials([o_a, o_b], [lse_a, lse_b])
    assert np.isneginf(lse[0, 0, 0]) and np.all(o[0, 0] == 0.0)
    assert lse[0, 0, 1] == 0.25 and np.all(o[0, 1] == 1.0)


# ------------------------------------------------------- packed sequences

def test_varlen_of_equal_lengths_is_the_batched_attention():
    rng = np.random.default_rng(23)
    B, N, Hq, Hkv, d = 3, 9, 4, 2, 8
    q = rng.standard_normal((B, N, Hq, d))
    k = rng.standard_normal((B, N, Hkv, d))
    v = rng.standard_normal((B, N, Hkv, d))
    cu = np.arange(B + 1) * N
    o, lse = oracle.attn_fwd_varlen(q.reshape(B * N, Hq, d), k.reshape(B * N, Hkv, d),
                                    v.reshape(B * N, Hkv, d), cu, cu, causal=True)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, causal=True)
    assert np.abs(o - o_ref.reshape(B * N, Hq, d)).max() < 1e-14
    assert np.abs(lse - np.transpose(lse_ref, (1, 0, 2)).reshape(Hq, B * N)).max() < 1e-14


def test_varlen_sequences_do_not_see_each_other():
    """Changing the keys of one sequence changes no other sequence's output;
    rows outside every sequence stay empty."""
    rng = np.random.default_rng(24)
    cu_q = np.array([0, 3, 3, 10])
    cu_k = np.array([0, 5, 9, 12])
    q = rng.standard_normal((12, 2, 4))
    k = rng.standard_normal((12, 1, 4))
    v = rng.standard_normal((12, 1, 4))
    o1, l1 = oracle.attn_fwd_varlen(q, k, v, cu_q, cu_k)
    k2, v2 = k.copy(), v.copy()
    k2[0:5] += 1.0
    v2[0:5] -= 2.0
    o2, l2 = oracle.attn_fwd_varlen(q, k2, v2, cu_q, cu_k)
    assert np.array_equal(o1[3:10], o2[3:10]) and np.array_equal(l1[:, 3:10], l2[:, 3:10])
    assert not np.allclose(o1[0:3], o2[0:3])
    assert np.all(o1[10:] == 0.0) and np.all(np.isneginf(l1[:, 10:]))


def test_varlen_gradients_of_equal_lengths_are_the_batched_gradients():
    rng = np.random.default_rng(25)
    B, N, Hq, Hkv, d = 2, 7, 2, 1, 4
    q = rng.standard_normal((B, N, Hq, d))
    k = rng.standard_normal((B, N, Hkv, d))
    v = rng.standard_normal((B, N, Hkv, d))
    do = rng.standard_normal((B, N, Hq, d))
    cu = np.arange(B + 1) * N
    g = oracle.attn_bwd_varlen(q.reshape(B * N, Hq, d), k.reshape(B * N, Hkv, d),
                               v.reshape(B * N, Hkv, d), do.reshape(B * N, Hq, d), cu, cu,
                               causal=True, window=(3, -1))
    ref = oracle.attn_bwd(q, k, v, do, causal=True, window=(3, -1))
    for a, r in zip(g, ref):
        assert np.abs(a - r.reshape(a.shape)).max() < 1e-14


# ------------------------------------------------------------ block-sparse

@pytest.mark.parametrize("causal,window", [(False, (-1, -1)), (True, (-1, -1)), (False, (5, 3))])
def test_blockmask_all_ones_is_the_dense_attention(causal, window):
    rng = np.random.default_rng(60)
    q = rng.standard_normal((2, 13, 4, 6))
    k = rng.standard_normal((2, 17, 2, 6))
    v = rng.standard_normal((2, 17, 2, 6))
    o, lse = oracle.attn_fwd_blockmask(q, k, v, np.ones((1, 1, 4, 5)), block=4, causal=causal,
                                       window=window)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, causal=causal, window=window)
    assert np.abs(o - o_ref).max() < 1e-12
    fin = np.isfinite(lse_ref)
    assert np.array_equal(fin, np.isfinite(lse)) and np.abs(lse[fin] - lse_ref[fin]).max() < 1e-12


def test_blockmask_key_blocks_off_equals_dropping_those_keys():
    """Non-causal: a key block off for every query block is the attention over
    the remaining keys (the C oracle on the sliced keys)."""
    rng = np.random.default_rng(61)
    q = rng.standard_normal((1, 10, 2, 5))
    k = rng.standard_normal((1, 22, 1, 5))
    v = rng.standard_normal((1, 22, 1, 5))
    bm = np.ones((1, 1, 3, 6))
    bm[..., 1] = 0
    bm[..., 4] = 0
    o, lse = oracle.attn_fwd_blockmask(q, k, v, bm, block=4)
    keep = np.r_[0:4, 8:16, 20:22]
    o_ref, lse_ref = oracle.attn_fwd(q, k[:, keep], v[:, keep])
    assert np.abs(o - o_ref).max() < 1e-12 and np.abs(lse - lse_ref).max() < 1e-12


def test_blockmask_query_block_off_gives_empty_rows_and_heads_differ():
    rng = np.random.default_rng(62)
    q = rng.standard_normal((1, 8, 2, 3))
    k = rng.standard_normal((1, 8, 2, 3))
    v = rng.standard_normal((1, 8, 2, 3))
    bm = np.ones((1, 2, 2, 2))
    bm[0, 1, 0, :] = 0          # head 1: rows 0-3 see nothing
    o, lse = oracle.attn_fwd_blockmask(q, k, v, bm, block=4)
    assert np.all(o[0, :4, 1] == 0) and np.all(np.isneginf(lse[0, 1, :4]))
    o_ref, _ = oracle.attn_fwd(q, k, v)
    assert np.abs(o[0, :, 0] - o_ref[0, :, 0]).max() < 1e-12
    assert np.abs(o[0, 4:, 1] - o_ref[0, 4:, 1]).max() < 1e-12


@pytest.mark.parametrize("causal,window", [(False, (-1, -1)), (True, (-1, -1)), (True, (4, -1))])
def test_blockmask_gradients_all_ones_are_the_dense_gradients(causal, window):
    rng = np.random.default_rng(63)
    q = rng.standard_normal((1, 11, 4, 5))
    k = rng.standard_normal((1, 14, 2, 5))
    v = rng.standard_normal((1, 14, 2, 5))
    do = rng.standard_normal((1, 11, 4, 5))
    g = oracle.attn_bwd_blockmask(q, k, v, do, np.ones((1, 1, 3, 4)), block=4, causal=causal,
                                  window=window)
    ref = oracle.attn_bwd(q, k, v, do, causal=causal, window=window)
    for a, r in zip(g, ref):
        assert np.abs(a - r).max() < 1e-11


def test_blockmask_gradients_with_key_blocks_off_are_those_of_the_remaining_keys():
    rng = np.random.default_rng(64)
    q = rng.standard_normal((1, 9, 2, 4))
    k = rng.standard_normal((1, 16, 1, 4))
    v = rng.standard_normal((1, 16, 1, 4))
    do = rng.standard_normal((1, 9, 2, 4))
    bm = np.ones((1, 1, 3, 4))
    bm[..., 2] = 0
    dq, dk, dv = oracle.attn_bwd_blockmask(q, k, v, do, bm, block=4)
    keep = np.r_[0:8, 12:16]
    rq, rk, rv = oracle.attn_bwd(q, k[:, keep], v[:, keep], do)
    assert np.abs(dq - rq).max() < 1e-11
    assert np.abs(dk[:, keep] - rk).max() < 1e-11 and np.abs(dv[:, keep] - rv).max() < 1e-11
    assert np.all(dk[:, 8:12] == 0) and np.all(dv[:, 8:12] == 0)


# ---------------------------------------------------------------- a key set's share of the gradients

@pytest.mark.parametrize("causal,window", [(False, (-1, -1)), (True, (-1, -1)), (False, (3, 2))])
def test_share_of_the_whole_key_set_is_the_gradient(causal, window):
    """With every key in the set, the share is attn_bwd's gradient (the
    given O and LSE are then the set's own)."""
    rng = np.random.default_rng(11)
    B, N, Hq, Hkv, d = 1, 10, 4, 2, 6
    q, k, v, do = (rng.standard_normal(s) for s in ((B, N, Hq, d), (B, N, Hkv, d), (B, N, Hkv, d), (B, N, Hq, d)))
    o, lse = oracle.attn_fwd(q, k, v, causal=causal, window=window)
    for got, ref in zip(oracle.attn_bwd_given_stats(q, k, v, do, o, lse, causal=causal, window=window),
                        oracle.attn_bwd(q, k, v, do, causal=causal, window=window)):
        np.testing.assert_allclose(got, ref, atol=1e-12)


def test_shares_over_scattered_key_sets_add_up_to_the_gradients():
    """Non-causal attention over keys split into scattered sets (every third
    key): the dQ shares sum to dQ, and each set's dK / dV are the full
    gradients' rows of its keys."""
    rng = np.random.default_rng(12)
    B, N, Hq, Hkv, d = 2, 12, 2, 1, 5
    q, k, v, do = (rng.standard_normal(s) for s in ((B, N, Hq, d), (B, N, Hkv, d), (B, N, Hkv, d), (B, N, Hq, d)))
    o, lse = oracle.attn_fwd(q, k, v)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do)
    sdq = np.zeros_like(dq)
    for m in range(3):
        idx = np.arange(m, N, 3)
        a, b_, c = oracle.attn_bwd_given_stats(q, k[:, idx], v[:, idx], do, o, lse)
        sdq += a
        np.testing.assert_allclose(b_, dk[:, idx], atol=1e-12)
        np.testing.assert_allclose(c, dv[:, idx], atol=1e-12)
    np.testing.assert_allclose(sdq, dq, atol=1e-12)


@pytest.mark.parametrize("R", [2, 3, 4])
def test_shares_over_causal_ring_blocks_add_up_to_the_gradients(R):
    """Split a causal sequence into R equal slices: slice pairs above the
    diagonal are hidden, the diagonal pairs are causal, the rest are seen
    whole.  attn_bwd_given_stats on each visible pair, with the full rows' O
    and LSE, sums to attn_bwd (dQ over the key slices, dK / dV over the query
    slices)."""
    rng = np.random.default_rng(20 + R)
    B, n, Hq, Hkv, d = 2, 4, 4, 2, 8
    N = R * n
    q, k, v, do = (rng.standard_normal(s) for s in ((B, N, Hq, d), (B, N, Hkv, d), (B, N, Hkv, d), (B, N, Hq, d)))
    o, lse = oracle.attn_fwd(q, k, v, causal=True)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, causal=True)
    sdq, sdk, sdv = np.zeros_like(dq), np.zeros_like(dk), np.zeros_like(dv)
    for r in range(R):
        qs = slice(r * n, (r + 1) * n)
        for s in range(r + 1):
            ks = slice(s * n, (s + 1) * n)
            a, b_, c = oracle.attn_bwd_given_stats(q[:, qs], k[:, ks], v[:, ks], do[:, qs], o[:, qs],
                                                   lse[:, :, qs], causal=(s == r))
            sdq[:, qs] += a
            sdk[:, ks] += b_
            sdv[:, ks] += c
    np.testing.assert_allclose(sdq, dq, atol=1e-12)
    np.testing.assert_allclose(sdk, dk, atol=1e-12)
    np.testing.assert_allclose(sdv, dv, atol=1e-12)


def test_share_of_a_set_no_row_sees_is_zero():
    """Rows with LSE = -inf (they see no key) contribute nothing."""
    rng = np.random.default_rng(5)
    q, k, v, do, o = (rng.standard_normal((1, 4, 1, 4)) for _ in range(5))
    lse = np.full((1, 1, 4), -np.inf)
    for g in oracle.attn_bwd_given_stats(q, k, v, do, o, lse):
        assert not np.any(g)
