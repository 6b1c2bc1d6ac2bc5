"""Pins for the CPU oracle: each oracle step is checked against something other
than itself - closed forms, brute force over tiny inputs, library routines on
special cases, invariants, and a worked example derived by hand.

Sources restated (no page prints a worked example):
  * axolotl docs, integrations.expert_parallel.args, ExpertParallelArgs
    (expert_parallel_token_capacity, expert_parallel_dispatch_chunks,
    expert_parallel_size, expert_parallel_backend = torch all_to_all_single);
  * LightLLM PR 1687 (top-k with norm_topk_prob, psum layout, silu_and_mul,
    decode reduce into a dense output).
"""
import itertools
import math
import struct
from fractions import Fraction

import numpy as np
import pytest

import oracle

F32_EPS = 2.0 ** -23


def ulp32(v: float) -> float:
    """Spacing of fp32 numbers at |v| (normal range)."""
    if v == 0.0:
        return 2.0 ** -149
    e = math.frexp(abs(v))[1]  # v = m * 2^e, m in [0.5, 1)
    return 2.0 ** max(e - 24, -149)


def f32(v: float) -> float:
    return struct.unpack("<f", struct.pack("<f", v))[0]


# ----------------------------------------------------------------- exp_det

def test_exp_det_exact_points():
    assert oracle.exp_det(0.0) == 1.0
    assert oracle.exp_det(-0.0) == 1.0
    assert oracle.exp_det(-87.5) == 0.0
    assert oracle.exp_det(-1000.0) == 0.0
    # e^{-87} is a normal fp32 number
    assert oracle.exp_det(-87.0) > 1.17549435e-38


def test_exp_det_against_closed_form_dense_sweep():
    # fp64 exp is accurate to < 1 fp64 ulp, i.e. exact at fp32 resolution.
    rng = np.random.default_rng(0)
    pts = np.concatenate([np.linspace(-87.0, 0.0, 40001, dtype=np.float32),
                          -rng.exponential(3.0, 20000).astype(np.float32),
                          -rng.uniform(0, 1e-3, 2000).astype(np.float32)])
    pts = pts[pts >= -87.0]
    worst = 0.0
    for r in pts:
        got = oracle.exp_det(float(r))
        ref = math.exp(float(r))
        err = abs(got - ref) / ulp32(ref)
        worst = max(worst, err)
    assert worst <= 2.0, worst


def test_exp_det_powers_of_two():
    ln2 = math.log(2.0)
    for n in range(0, 126):
        r = f32(-n * ln2)
        got = oracle.exp_det(r)
        ref = math.exp(r)
        assert abs(got - ref) <= 2 * ulp32(ref)
        # and close to 2^-n itself (the residual r + n ln2 is below an fp32 ulp of r)
        assert abs(got / 2.0 ** -n - 1.0) < 1e-5


# ----------------------------------------------------------------- top-k routing

def _topk_by_sort(l, k):
    order = sorted(range(len(l)), key=lambda e: (-l[e], e))
    return order[:k]


def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(1)
    for E in (3, 4, 6):
        for k in range(1, min(E, 3) + 1):
            T = 40
            logits = rng.integers(-2, 3, size=(T, E)).astype(np.float32)  # many ties
            idx, w, counts, st = oracle.route_topk(logits, None, k)
            assert st == oracle.ORC_OK
            for t in range(T):
                l = [float(v) for v in logits[t]]
                # brute force: the chosen set is the only k-subset whose every
                # member ranks before every non-member (value desc, index asc)
                winners = []
                for S in itertools.combinations(range(E), k):
                    rest = [b for b in range(E) if b not in S]
                    if all(l[a] > l[b] or (l[a] == l[b] and a < b) for a in S for b in rest):
                        winners.append(set(S))
                assert len(winners) == 1
                assert set(idx[t].tolist()) == winners[0]
                # slot order is rank order
                assert idx[t].tolist() == _topk_by_sort(l, k)
            np.testing.assert_array_equal(counts, np.bincount(idx.ravel(), minlength=E))


def test_topk_weights_closed_form():
    rng = np.random.default_rng(2)
    T, E, k = 300, 64, 8
    logits = (rng.standard_normal((T, E)) * 3).astype(np.float32)
    idx, w, counts, st = oracle.route_topk(logits, None, k)
    assert st == oracle.ORC_OK
    for t in range(T):
        sel = [float(logits[t, e]) for e in idx[t]]
        m = sel[0]
        z = [math.exp(v - m) for v in sel]
        s = sum(z)
        for j in range(k):
            ref = z[j] / s
            assert abs(float(w[t, j]) - ref) <= (k + 4) * ulp32(ref), (t, j)
        # renormalised weights sum to one within k ulp
        assert abs(float(np.sum(w[t].astype(np.float64))) - 1.0) <= k * F32_EPS
        # full softmax restricted to the top k and renormalised gives the same weights
        full = np.exp(logits[t].astype(np.float64) - logits[t].max())
        p = full / full.sum()
        np.testing.assert_allclose(w[t], p[idx[t]] / p[idx[t]].sum(), rtol=(k + 4) * F32_EPS)


def test_topk_all_equal_logits():
    for k in (1, 2, 3, 5, 8):
        logits = np.full((7, 16), 0.25, np.float32)
        idx, w, counts, st = oracle.route_topk(logits, None, k)
        assert (idx == np.arange(k, dtype=np.int32)).all()
        # e_j = 1 exactly, S = k exactly, IEEE division
        assert (w == np.float32(1.0) / np.float32(k)).all()


def test_topk_k1_weight_is_one():
    rng = np.random.default_rng(3)
    logits = rng.standard_normal((50, 10)).astype(np.float32)
    idx, w, _, _ = oracle.route_topk(logits, None, 1)
    assert (w == 1.0).all()
    assert (idx[:, 0] == logits.argmax(axis=1)).all()


def test_topk_signed_zero_ties_and_bias():
    logits = np.array([[-0.0, 0.0, -1.0, -2.0]], np.float32)
    idx, w, _, _ = oracle.route_topk(logits, None, 2)
    assert idx[0].tolist() == [0, 1]          # -0 == +0: lower index first
    assert (w[0] == np.float32(0.5)).all()
    bias = np.array([0.0, 0.0, 5.0, 0.0], np.float32)
    idx, w, _, _ = oracle.route_topk(logits, bias, 2)
    assert idx[0].tolist() == [2, 0]
    # weights use the biased logits: exp(0 - 4) / (1 + exp(-4))
    assert abs(float(w[0, 1]) - math.exp(-4.0) / (1 + math.exp(-4.0))) <= 4 * ulp32(0.018)


def test_topk_rejects_nonfinite():
    logits = np.zeros((3, 4), np.float32)
    logits[1, 2] = np.nan
    *_, st = oracle.route_topk(logits, None, 2)
    assert st == oracle.ORC_ERR_NONFINITE
    logits[1, 2] = np.inf
    *_, st = oracle.route_topk(logits, None, 2)
    assert st == oracle.ORC_ERR_NONFINITE


# ----------------------------------------------------------------- routing variants

def _ranks_before(va, a, vb, b):
    return va > vb or (va == vb and a < b)


def _group_scores_f32(l, n_group, mode):
    """A group's best value, or the fp32 sum of its two best (mode 1)."""
    gs = l.shape[0] // n_group
    out = []
    for g in range(n_group):
        v = sorted((float(x) for x in l[g * gs:(g + 1) * gs]), reverse=True)
        out.append(np.float32(v[0]) if mode == 0 else np.float32(np.float32(v[0]) + np.float32(v[1])))
    return out


@pytest.mark.parametrize("mode", [0, 1])
def test_grouped_topk_reduces_to_plain(mode):
    rng = np.random.default_rng(21)
    logits = rng.standard_normal((40, 12)).astype(np.float32)
    ref_idx, ref_w, ref_c, _ = oracle.route_topk(logits, None, 3)
    for n_group, topk_group in ((1, 1), (4, 4), (6, 6)):
        idx, w, c, st = oracle.route_topk(logits, None, 3, n_group=n_group, topk_group=topk_group,
                                          group_score=mode)
        assert st == oracle.ORC_OK
        np.testing.assert_array_equal(idx, ref_idx)
        np.testing.assert_array_equal(w.view(np.uint32), ref_w.view(np.uint32))
        np.testing.assert_array_equal(c, ref_c)


@pytest.mark.parametrize("mode", [0, 1])
def test_grouped_topk_brute_force_with_ties(mode):
    """Characterisation on tiny inputs with many ties: every kept group outranks
    every dropped one (score desc, lower group first), every chosen expert lies in
    a kept group and outranks every unchosen expert of the kept groups, and the
    slots are in rank order."""
    rng = np.random.default_rng(5 + mode)
    E, n_group = 8, 4
    gs = E // n_group
    for trial in range(60):
        logits = rng.integers(-3, 4, size=(6, E)).astype(np.float32) * np.float32(0.5)
        topk_group = 1 + trial % 3
        k = 1 + trial % (topk_group * gs)
        idx, w, counts, st = oracle.route_topk(logits, None, k, n_group=n_group,
                                               topk_group=topk_group, group_score=mode)
        assert st == oracle.ORC_OK
        for t in range(logits.shape[0]):
            l = logits[t]
            sc = _group_scores_f32(l, n_group, mode)
            # the kept groups: the topk_group best by (score desc, index asc), by exhaustion
            best_set = None
            for G in itertools.combinations(range(n_group), topk_group):
                ok = all(_ranks_before(sc[g], g, sc[h], h)
                         for g in G for h in range(n_group) if h not in G)
                if ok:
                    assert best_set is None
                    best_set = set(G)
            allowed = [e for e in range(E) if e // gs in best_set]
            chosen = [int(e) for e in idx[t]]
            assert len(set(chosen)) == k and all(e in allowed for e in chosen)
            for e in chosen:
                for f in allowed:
                    if f not in chosen:
                        assert _ranks_before(l[e], e, l[f], f)
            for a, b in zip(chosen, chosen[1:]):
                assert _ranks_before(l[a], a, l[b], b)
            # weights: renormalised softmax over the chosen biased logits
            ref = np.exp(np.array([float(l[e]) for e in chosen]) - float(l[chosen[0]]))
            np.testing.assert_allclose(w[t], ref / ref.sum(), rtol=1e-6)
        assert int(counts.sum()) == k * logits.shape[0]


def test_grouped_topk_rejects_bad_arguments():
    logits = np.zeros((2, 8), np.float32)
    for kw in (dict(n_group=3, topk_group=1),            # E not divisible
               dict(n_group=4, topk_group=0),            # no group kept
               dict(n_group=4, topk_group=5),            # more than there are
               dict(n_group=8, topk_group=1, group_score=1)):   # one-expert groups, sum of two
        *_, st = oracle.route_topk(logits, None, 1, **kw)
        assert st == oracle.ORC_ERR_ARG
    *_, st = oracle.route_topk(logits, None, 3, n_group=4, topk_group=1)   # k > 1 group of 2
    assert st == oracle.ORC_ERR_ARG


def test_bias_select_only():
    rng = np.random.default_rng(8)
    logits = rng.standard_normal((50, 16)).astype(np.float32)
    bias = (2.0 * rng.standard_normal(16)).astype(np.float32)
    # zero bias: the same as plain routing, bit for bit
    z = np.zeros(16, np.float32)
    a = oracle.route_topk(logits, z, 4, bias_select_only=True)
    b = oracle.route_topk(logits, None, 4)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1].view(np.uint32), b[1].view(np.uint32))
    # with a bias: the experts are the biased choice, the weights the softmax of
    # the unbiased logits of those experts (closed form in double)
    idx, w, _, st = oracle.route_topk(logits, bias, 4, bias_select_only=True)
    assert st == oracle.ORC_OK
    ref_idx, ref_w_biased, _, _ = oracle.route_topk(logits, bias, 4)
    np.testing.assert_array_equal(idx, ref_idx)
    for t in range(logits.shape[0]):
        v = np.array([float(logits[t, e]) for e in idx[t]])
        ref = np.exp(v - v.max())
        np.testing.assert_allclose(w[t], ref / ref.sum(), rtol=1e-6)
        assert abs(float(w[t].sum()) - 1.0) <= 4 * 2.0 ** -23
    assert not np.array_equal(w, ref_w_biased)   # the bias does change the weights otherwise
    # combined with grouping: the chosen experts are those of grouped routing on the
    # biased logits
    g = oracle.route_topk(logits, bias, 4, n_group=4, topk_group=2, group_score=1,
                          bias_select_only=True)
    g_ref = oracle.route_topk(logits, bias, 4, n_group=4, topk_group=2, group_score=1)
    np.testing.assert_array_equal(g[0], g_ref[0])


# ----------------------------------------------------------------- capacity clip

def _brute_force_keep(assigns, C):
    """assigns: list of (w, t).  Every C-subset; keep the max exact weight sum,
    ties to the lexicographically smallest sorted token list (the higher token
    is dropped first among equal weights)."""
    n = len(assigns)
    if C < 0 or n <= C:
        return set(range(n))
    best = None
    for S in itertools.combinations(range(n), C):
        tot = sum(Fraction(assigns[i][0]) for i in S)
        toks = sorted(assigns[i][1] for i in S)
        key = (-tot, toks)
        if best is None or key < best[0]:
            best = (key, set(S))
    return best[1]


def test_capacity_clip_brute_force():
    rng = np.random.default_rng(4)
    for trial in range(30):
        T = int(rng.integers(1, 9))
        E = int(rng.integers(2, 5))
        k = int(rng.integers(1, min(E, 3) + 1))
        logits = rng.integers(-1, 2, size=(T, E)).astype(np.float32)  # ties in weights
        idx, w, counts, _ = oracle.route_topk(logits, None, k)
        for C in range(0, T + 1):
            keep, kept = oracle.capacity_clip(idx, w, E, C)
            for e in range(E):
                pairs = [(t, j) for t in range(T) for j in range(k) if idx[t, j] == e]
                assigns = [(float(w[t, j]), t) for t, j in pairs]
                want = _brute_force_keep(assigns, C)
                got = {i for i, (t, j) in enumerate(pairs) if keep[t, j]}
                assert got == want, (trial, C, e)
                assert kept[e] == len(want) <= C
        keep, kept = oracle.capacity_clip(idx, w, E, -1)
        assert keep.all() and (kept == counts).all()


def test_capacity_clip_special_cases():
    rng = np.random.default_rng(5)
    logits = rng.standard_normal((64, 8)).astype(np.float32)
    idx, w, counts, _ = oracle.route_topk(logits, None, 2)
    keep, kept = oracle.capacity_clip(idx, w, 8, 64)     # C >= T: nothing dropped
    assert keep.all() and (kept == counts).all()
    keep, kept = oracle.capacity_clip(idx, w, 8, 0)      # C = 0: everything dropped
    assert not keep.any() and (kept == 0).all()
    # all-equal logits: every token picks experts 0..k-1 with equal weight,
    # so the kept tokens are exactly 0..C-1
    idx, w, _, _ = oracle.route_topk(np.zeros((20, 6), np.float32), None, 2)
    keep, kept = oracle.capacity_clip(idx, w, 6, 7)
    assert keep[:7].all() and not keep[7:].any()
    assert kept.tolist() == [7, 7, 0, 0, 0, 0]


# ----------------------------------------------------------------- dispatch layout

def _check_layout(idx, keep, E, ep, tb, tc, lay):
    k = idx.shape[1]
    pairs = sorted((int(idx[t, j]), t, j) for t in range(tb, tb + tc) for j in range(k)
                   if keep[t, j])
    N = len(pairs)
    assert lay["N"] == N
    assert lay["recv_token"].tolist() == [t for _, t, _ in pairs]
    assert lay["recv_slot"].tolist() == [j for _, _, j in pairs]
    hist = np.bincount(np.array([e for e, _, _ in pairs], dtype=np.int64), minlength=E)
    assert lay["expert_offsets"].tolist() == [0] + np.cumsum(hist).tolist()
    epr = E // ep
    assert lay["rank_offsets"].tolist() == [lay["expert_offsets"][d * epr] for d in range(ep + 1)]
    # pos and recv are mutual inverses; dropped slots are -1
    for i in range(tc):
        for j in range(k):
            p = lay["pos"][i, j]
            if keep[tb + i, j]:
                assert lay["recv_token"][p] == tb + i and lay["recv_slot"][p] == j
            else:
                assert p == -1
    # send splits: brute-force count, sums to N, and column sums are the
    # per-rank receive counts
    tpr = tc // ep
    want = np.zeros((ep, ep), np.int64)
    for e, t, j in pairs:
        want[(t - tb) // tpr, e // epr] += 1
    np.testing.assert_array_equal(lay["send_splits"], want)
    assert lay["send_splits"].sum() == N
    np.testing.assert_array_equal(lay["send_splits"].sum(axis=0), np.diff(lay["rank_offsets"]))


def test_dispatch_layout_against_sort_and_invariants():
    rng = np.random.default_rng(6)
    for (T, E, k, ep, C, nch) in [(16, 4, 2, 2, -1, 1), (48, 8, 3, 4, 5, 1),
                                  (66, 12, 2, 3, 9, 2), (30, 6, 1, 1, 2, 3),
                                  (8, 6, 3, 2, 0, 1)]:
        logits = rng.standard_normal((T, E)).astype(np.float32)
        idx, w, _, _ = oracle.route_topk(logits, None, k)
        keep, kept = oracle.capacity_clip(idx, w, E, C)
        tc = T // nch
        total = 0
        for c in range(nch):
            lay = oracle.dispatch_layout(idx, keep, E, ep, c * tc, tc)
            _check_layout(idx, keep, E, ep, c * tc, tc, lay)
            total += lay["N"]
        assert total == int(kept.sum()) == int(keep.sum())


def test_dispatch_layout_rejects_bad_topology():
    idx = np.zeros((6, 1), np.int32)
    keep = np.ones((6, 1), np.uint8)
    with pytest.raises(ValueError):
        oracle.dispatch_layout(idx, keep, 5, 2)       # E % EP != 0
    with pytest.raises(ValueError):
        oracle.dispatch_layout(idx, keep, 4, 4)       # tokens % EP != 0


# ----------------------------------------------------------------- permute

def test_permute_is_row_gather():
    rng = np.random.default_rng(7)
    x = rng.integers(0, 65535, size=(10, 6)).astype(np.uint16)
    rt = np.array([3, 3, 0, 9, 1], np.int32)
    np.testing.assert_array_equal(oracle.permute(x, rt), x[rt])
    xf = rng.standard_normal((10, 5)).astype(np.float32)
    np.testing.assert_array_equal(oracle.permute(xf, rt), xf[rt])


# ----------------------------------------------------------------- bf16 rounding

def test_bf16_rounding_single_step():
    b = oracle.bf16_bits_from_double
    assert b(1.0) == 0x3F80
    assert b(-2.0) == 0xC000
    assert b(1.0 + 2 ** -8) == 0x3F80              # tie -> even
    assert b(1.0 + 3 * 2 ** -8) == 0x3F82          # tie -> even (upwards)
    # one rounding from fp64: a double-rounding through fp32 would give 0x3F80
    assert b(1.0 + 2 ** -8 + 2 ** -30) == 0x3F81
    assert b(1e39) == 0x7F80 and b(-1e39) == 0xFF80
    assert b(0.0) == 0 and b(-0.0) == 0x8000


# ----------------------------------------------------------------- FFN

def _silu(a):
    return a / (1.0 + math.exp(-a))


def test_ffn_closed_form_with_selection_matrices():
    # gate row i picks x[a(i)], up row i picks x[b(i)], down row o picks h[c(o)]:
    # y_o = silu(x[a(c(o))]) * x[b(c(o))] exactly (fp32 inputs, no rounding of h).
    rng = np.random.default_rng(8)
    H, I = 12, 5
    a = rng.integers(0, H, I)
    bb = rng.integers(0, H, I)
    c = rng.integers(0, I, H)
    w13 = np.zeros((2 * I, H), np.float32)
    w2 = np.zeros((H, I), np.float32)
    for i in range(I):
        w13[i, a[i]] = 1.0
        w13[I + i, bb[i]] = 1.0
    for o in range(H):
        w2[o, c[o]] = 1.0
    x = rng.standard_normal(H).astype(np.float32)
    h, y, ye = oracle.ffn_row(x, w13, w2, round_h=False)
    for o in range(H):
        i = c[o]
        ref = _silu(float(x[a[i]])) * float(x[bb[i]])
        assert abs(ye[o] - ref) <= 1e-15 * max(1.0, abs(ref))
    for i in range(I):
        assert h[i] == np.float32(_silu(float(x[a[i]])) * float(x[bb[i]]))


def test_ffn_matches_numpy_dense():
    rng = np.random.default_rng(9)
    H, I = 24, 10
    x = rng.standard_normal(H).astype(np.float32)
    w13 = (rng.standard_normal((2 * I, H)) / math.sqrt(H)).astype(np.float32)
    w2 = (rng.standard_normal((H, I)) / math.sqrt(H)).astype(np.float32)
    h, y, ye = oracle.ffn_row(x, w13, w2, round_h=False)
    g = w13[:I].astype(np.float64) @ x.astype(np.float64)
    u = w13[I:].astype(np.float64) @ x.astype(np.float64)
    hh = g / (1.0 + np.exp(-g)) * u
    np.testing.assert_allclose(ye, w2.astype(np.float64) @ hh, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(y, (w2.astype(np.float64) @ hh).astype(np.float32), rtol=1e-6)
    # a dropped term (gate and up swapped) would fail this
    hs = u / (1.0 + np.exp(-u)) * g
    assert not np.allclose(ye, w2.astype(np.float64) @ hs, rtol=1e-6)


def test_ffn_bf16_storage_rounds_h():
    rng = np.random.default_rng(10)
    H, I = 16, 8
    import torch
    xf = torch.from_numpy(rng.standard_normal(H).astype(np.float32)).bfloat16()
    w13f = torch.from_numpy((rng.standard_normal((2 * I, H)) / 4).astype(np.float32)).bfloat16()
    w2f = torch.from_numpy((rng.standard_normal((H, I)) / 4).astype(np.float32)).bfloat16()
    u16 = lambda t: t.view(torch.int16).numpy().view(np.uint16).copy()
    h, y, ye = oracle.ffn_row(u16(xf), u16(w13f), u16(w2f), round_h=True)
    g = w13f[:I].double() @ xf.double()
    u = w13f[I:].double() @ xf.double()
    hh = (g / (1 + torch.exp(-g)) * u)
    hb = torch.from_numpy(h.view(np.int16).copy()).view(torch.bfloat16).double()
    # h is hh rounded once to bf16 (half an ulp: 2^-9 relative)
    assert ((hb - hh).abs() <= hh.abs() * 2.0 ** -8 + 1e-30).all()
    np.testing.assert_allclose(ye, (w2f.double() @ hb).numpy(), rtol=1e-12, atol=1e-14)


# ----------------------------------------------------------------- combine + whole layer

def test_combine_special_cases():
    rng = np.random.default_rng(11)
    T, H, k = 6, 4, 2
    y = rng.standard_normal((T * k, H)).astype(np.float32)
    pos = np.arange(T * k, dtype=np.int32).reshape(T, k)
    w = np.full((T, k), 0.5, np.float32)
    out = oracle.combine(y, pos, w, T)
    np.testing.assert_allclose(out, 0.5 * (y[0::2] + y[1::2]), rtol=1e-6)
    pos[2, :] = -1                     # a token with every slot dropped
    out = oracle.combine(y, pos, w, T)
    assert (out[2] == 0).all()
    # k = 1 with weight 1: combine is the identity on its row
    out = oracle.combine(y[:T], np.arange(T, dtype=np.int32).reshape(T, 1),
                         np.ones((T, 1), np.float32), T)
    np.testing.assert_array_equal(out, y[:T])


def _bit_coded_rows(N, H, k):
    """Receive rows whose every entry is a distinct power of two per (row, slot):
    y[p, c] = (c + 1) * 2^(-k*p) and slot weights w_j = 2^-(j+1), so the term
    w_j * y[p] = (c + 1) * 2^-(j + 1 + k*p) lands on its own bit and an exact
    fp64 sum tells which (slot, row) pairs were added."""
    y = np.empty((N, H), np.float64)
    for p in range(N):
        y[p] = np.arange(1, H + 1) * 2.0 ** (-k * p)
    return y


def _decode_bits(v, k, N):
    """Inverse of the coding above for column 0 (c + 1 = 1): the set of (slot, row)
    pairs whose term is present in v (exact fp64)."""
    pairs = set()
    for j in range(k):
        for p in range(N):
            if math.ldexp(1.0, -(j + 1 + k * p)) <= v and \
                    int(math.ldexp(v, j + 1 + k * p)) & 1:
                pairs.add((j, p))
    return pairs


@pytest.mark.parametrize("tok_begin", [0, 4])
def test_combine_exact_sums_exactly_the_kept_slots(tok_begin):
    """Decode form of the combine (LightLLM PR 1687: the decode path reduces expert
    outputs straight into a dense output).  With bit-coded rows and power-of-two
    weights every (slot, row) term of a token's sum sits on its own bit, so the
    exact fp64 output names the rows and slots that were added: it must be exactly
    {(j, pos[i, j]) : pos[i, j] >= 0} for token tok_begin + i, read with the weights
    of that absolute token row.  A dropped term, a wrong slot weight, pos read
    against the wrong base or the chunk written to the wrong rows changes the bits."""
    k, H, tc, T = 2, 3, 4, 8
    rng = np.random.default_rng(41)
    N = 7
    y = _bit_coded_rows(N, H, k)
    # pos: a permutation of the rows over the chunk's slots, some slots dropped
    slots = rng.permutation(tc * k)[:N]
    pos = np.full(tc * k, -1, np.int32)
    pos[slots] = np.arange(N, dtype=np.int32)
    pos = pos.reshape(tc, k)
    w = np.zeros((T, k), np.float32)
    for j in range(k):
        w[tok_begin:tok_begin + tc, j] = 2.0 ** -(j + 1)
    w[:tok_begin] = 7.0               # other chunks' weights must not be read
    w[tok_begin + tc:] = 7.0
    out = np.full((T, H), -1.0, np.float64)
    oracle.combine_exact(y, pos, w, T, np.float64, tok_begin, out)
    for i in range(tc):
        want = {(j, int(pos[i, j])) for j in range(k) if pos[i, j] >= 0}
        got = _decode_bits(out[tok_begin + i, 0], k, N)
        assert got == want, (i, got, want)
        for c in range(H):              # column c is column 0 times (c + 1), exactly
            assert out[tok_begin + i, c] == (c + 1) * out[tok_begin + i, 0]
    # rows outside the chunk are untouched
    assert (np.delete(out, range(tok_begin, tok_begin + tc), axis=0) == -1.0).all()


def test_combine_exact_adds_the_shared_rows_by_chunk_row():
    """The shared expert's rows are indexed by chunk-relative row: row i belongs to
    token tok_begin + i, on bits far below every routed term."""
    k, H, tc, T, tb = 2, 2, 3, 6, 3
    y = _bit_coded_rows(4, H, k)
    pos = np.array([[0, -1], [-1, -1], [1, 2]], np.int32)
    w = np.zeros((T, k), np.float32)
    w[tb:, 0], w[tb:, 1] = 0.5, 0.25
    ys = np.array([[(i + 1) * 2.0 ** -40] * H for i in range(tc)])
    out = np.zeros((T, H), np.float64)
    oracle.combine_exact(y, pos, w, T, np.float64, tb, out, y_shared=ys)
    expect = [0.5 * y[0, 0] + 1 * 2.0 ** -40, 2 * 2.0 ** -40, 0.5 * y[1, 0] + 0.25 * y[2, 0] + 3 * 2.0 ** -40]
    assert out[tb:, 0].tolist() == expect
    assert (out[:tb] == 0).all()


def test_combine_exact_rounds_once_and_matches_the_stored_form_at_k1():
    """With one slot of weight 1 the decode form's single rounding of w * y_exact is
    the rounding of y_exact, which is what the stored form combines: the two give
    the same bits (fp32 and bf16).  And a token with every slot dropped gets 0."""
    rng = np.random.default_rng(42)
    N, H, T = 5, 6, 6
    ye = rng.standard_normal((N, H)) * 3
    pos = np.array([[0], [1], [-1], [2], [3], [4]], np.int32)
    w = np.ones((T, 1), np.float32)
    for dt, rnd in ((np.float32, lambda a: a.astype(np.float32)),
                    (np.uint16, lambda a: np.array([[oracle.bf16_bits_from_double(v) for v in r] for r in a],
                                                   np.uint16))):
        a = oracle.combine_exact(ye, pos, w, T, dt)
        b = oracle.combine(rnd(ye), pos, w, T)
        np.testing.assert_array_equal(a, b)
        assert (a[2] == 0).all()


@pytest.mark.parametrize("capacity,n_chunks", [(-1, 1), (5, 2), (0, 2)])
def test_decode_layer_equals_dense_sum_of_unrounded_rows(capacity, n_chunks):
    """The decode-form layer against a per-token dense loop in numpy that keeps y
    unrounded (h rounded to storage, as the CUDA path stores it): out_t =
    fp32(sum over kept j of w_j * W2[e_j] h_j), over two chunks with drops."""
    rng = np.random.default_rng(43)
    T, H, E, k, I = 24, 16, 6, 2, 12
    logits = rng.standard_normal((T, E)).astype(np.float32)
    x = rng.standard_normal((T, H)).astype(np.float32)
    w13 = (rng.standard_normal((E, 2 * I, H)) / 4).astype(np.float32)
    w2 = (rng.standard_normal((E, H, I)) / 4).astype(np.float32)
    res = oracle.moe_layer(logits, None, x, w13, w2, k, 2, capacity, n_chunks, reduce_dense=True)
    idx, w, keep = res["topk_idx"], res["topk_w"], res["keep"]
    ref = np.zeros((T, H))
    for t in range(T):
        for j in range(k):
            if not keep[t, j]:
                continue
            e = idx[t, j]
            xv = x[t].astype(np.float64)
            g = w13[e, :I].astype(np.float64) @ xv
            u = w13[e, I:].astype(np.float64) @ xv
            hh = (g / (1 + np.exp(-g)) * u).astype(np.float32).astype(np.float64)
            ref[t] += float(w[t, j]) * (w2[e].astype(np.float64) @ hh)
    np.testing.assert_allclose(res["out"], ref.astype(np.float32), rtol=2e-7, atol=1e-12)
    if capacity == 0:
        assert (res["out"] == 0).all()


def _dense_reference(logits, bias, x, w13, w2, k, capacity):
    """Per-token dense loop in numpy: out_t = sum_{kept j} w_j * FFN_{e_j}(x_t)."""
    idx, w, _, _ = oracle.route_topk(logits, bias, k)
    keep, _ = oracle.capacity_clip(idx, w, logits.shape[1], capacity)
    T, H = x.shape
    I = w13.shape[1] // 2
    out = np.zeros((T, H))
    for t in range(T):
        for j in range(k):
            if not keep[t, j]:
                continue
            e = idx[t, j]
            xv = x[t].astype(np.float64)
            g = w13[e, :I].astype(np.float64) @ xv
            u = w13[e, I:].astype(np.float64) @ xv
            hh = (g / (1 + np.exp(-g)) * u).astype(np.float32).astype(np.float64)
            out[t] += float(w[t, j]) * (w2[e].astype(np.float64) @ hh).astype(np.float32)
    return out


@pytest.mark.parametrize("capacity,n_chunks,ep", [(-1, 1, 2), (6, 1, 4), (6, 2, 2), (0, 1, 1)])
def test_whole_layer_equals_per_token_sum(capacity, n_chunks, ep):
    rng = np.random.default_rng(12)
    T, H, E, k, I = 32, 16, 8, 2, 12
    logits = rng.standard_normal((T, E)).astype(np.float32)
    x = rng.standard_normal((T, H)).astype(np.float32)
    w13 = (rng.standard_normal((E, 2 * I, H)) / 4).astype(np.float32)
    w2 = (rng.standard_normal((E, H, I)) / 4).astype(np.float32)
    res = oracle.moe_layer(logits, None, x, w13, w2, k, ep, capacity, n_chunks)
    ref = _dense_reference(logits, None, x, w13, w2, k, capacity)
    np.testing.assert_allclose(res["out"], ref, rtol=1e-5, atol=1e-6)
    if capacity == 0:
        assert (res["out"] == 0).all()


def test_chunking_changes_nothing():
    # axolotl: dispatch chunks only change the overlap, not the result
    rng = np.random.default_rng(13)
    T, H, E, k, I = 24, 8, 6, 2, 8
    logits = rng.standard_normal((T, E)).astype(np.float32)
    x = rng.standard_normal((T, H)).astype(np.float32)
    w13 = (rng.standard_normal((E, 2 * I, H)) / 3).astype(np.float32)
    w2 = (rng.standard_normal((E, H, I)) / 3).astype(np.float32)
    a = oracle.moe_layer(logits, None, x, w13, w2, k, 2, 5, 1)["out"]
    b = oracle.moe_layer(logits, None, x, w13, w2, k, 2, 5, 3)["out"]
    np.testing.assert_array_equal(a, b)


# ----------------------------------------------------------------- shared expert

def _shared_case(rng, T=24, H=16, E=6, k=2, I=12, Is=10):
    logits = rng.standard_normal((T, E)).astype(np.float32)
    x = rng.standard_normal((T, H)).astype(np.float32)
    w13 = (rng.standard_normal((E, 2 * I, H)) / 4).astype(np.float32)
    w2 = (rng.standard_normal((E, H, I)) / 4).astype(np.float32)
    w13s = (rng.standard_normal((2 * Is, H)) / 4).astype(np.float32)
    w2s = (rng.standard_normal((H, Is)) / 4).astype(np.float32)
    return logits, x, w13, w2, w13s, w2s


@pytest.mark.parametrize("reduce_dense", [False, True])
def test_shared_expert_zero_weights_change_nothing(reduce_dense):
    logits, x, w13, w2, w13s, w2s = _shared_case(np.random.default_rng(31))
    a = oracle.moe_layer(logits, None, x, w13, w2, 2, 2, reduce_dense=reduce_dense)["out"]
    b = oracle.moe_layer(logits, None, x, w13, w2, 2, 2, reduce_dense=reduce_dense,
                         w13_shared=np.zeros_like(w13s), w2_shared=np.zeros_like(w2s))["out"]
    np.testing.assert_array_equal(a, b)


def test_shared_expert_alone_when_every_assignment_is_dropped():
    logits, x, w13, w2, w13s, w2s = _shared_case(np.random.default_rng(32))
    res = oracle.moe_layer(logits, None, x, w13, w2, 2, 2, capacity=0,
                           w13_shared=w13s, w2_shared=w2s, n_chunks=2)
    ys = np.concatenate([c["y_shared"] for c in res["chunks"]])
    np.testing.assert_array_equal(res["out"], ys)
    # and ys is the dense SwiGLU of every row (closed form in double)
    Is = w2s.shape[1]
    g = x.astype(np.float64) @ w13s[:Is].T.astype(np.float64)
    u = x.astype(np.float64) @ w13s[Is:].T.astype(np.float64)
    ref = ((g / (1 + np.exp(-g))) * u).astype(np.float32).astype(np.float64) @ w2s.T.astype(np.float64)
    np.testing.assert_allclose(ys, ref, rtol=1e-5, atol=1e-6)


def test_shared_expert_equal_to_the_routed_one_doubles_it():
    # all-equal logits and k = 1 route every token to expert 0 with w = 1; with the
    # shared expert's weights equal to expert 0's, out = round(y + y) = 2 y exactly
    logits, x, w13, w2, _, _ = _shared_case(np.random.default_rng(33))
    logits[:] = 0.5
    res = oracle.moe_layer(logits, None, x, w13, w2, 1, 2, w13_shared=w13[0], w2_shared=w2[0])
    assert (res["topk_idx"] == 0).all() and (res["topk_w"] == 1.0).all()
    ys = res["chunks"][0]["y_shared"]
    np.testing.assert_array_equal(res["out"], 2 * ys)


def test_worked_example_by_hand():
    """T=4, E=4, k=2, EP=2, C=2, derived by hand from the definitions.

    logits: t0 [1,1,0,0] -> experts (0,1); t1 [0,2,2,0] -> (1,2);
            t2 [3,3,0,0] -> (0,1);         t3 [0,5,0,5] -> (1,3);
    every selected pair is tied, so every weight is exactly 1/2.
    Expert 1 holds t0..t3 (4 > C=2): equal weights, so the higher tokens t2
    (slot 1) and t3 (slot 0) are dropped.  Receive order by (expert, token):
      e0: t0 s0, t2 s0 | e1: t0 s1, t1 s0 | e2: t1 s1 | e3: t3 s1.
    Source ranks: t0,t1 -> 0; t2,t3 -> 1.  Destination: e0,e1 -> 0; e2,e3 -> 1.
    FFN (same for every expert): gate row [1,0], up row [0,1], down [[1],[2]],
    so y = [h, 2h] with h = silu(x0) * x1.
    """
    logits = np.array([[1, 1, 0, 0], [0, 2, 2, 0], [3, 3, 0, 0], [0, 5, 0, 5]], np.float32)
    idx, w, counts, _ = oracle.route_topk(logits, None, 2)
    assert idx.tolist() == [[0, 1], [1, 2], [0, 1], [1, 3]]
    assert (w == 0.5).all()
    assert counts.tolist() == [2, 4, 1, 1]
    keep, kept = oracle.capacity_clip(idx, w, 4, 2)
    assert keep.tolist() == [[1, 1], [1, 1], [1, 0], [0, 1]]
    assert kept.tolist() == [2, 2, 1, 1]
    lay = oracle.dispatch_layout(idx, keep, 4, 2)
    assert lay["N"] == 6
    assert lay["recv_token"].tolist() == [0, 2, 0, 1, 1, 3]
    assert lay["recv_slot"].tolist() == [0, 0, 1, 0, 1, 1]
    assert lay["expert_offsets"].tolist() == [0, 2, 4, 5, 6]
    assert lay["rank_offsets"].tolist() == [0, 4, 6]
    assert lay["pos"].tolist() == [[0, 2], [3, 4], [1, -1], [-1, 5]]
    assert lay["send_splits"].tolist() == [[3, 1], [1, 1]]

    x = np.array([[1, 2], [1, 1], [2, 1], [-1, 3]], np.float32)
    w13 = np.tile(np.array([[1, 0], [0, 1]], np.float32), (4, 1, 1))
    w2 = np.tile(np.array([[1], [2]], np.float32), (4, 1, 1))
    res = oracle.moe_layer(logits, None, x, w13, w2, 2, 2, 2)
    s1 = 1 / (1 + math.exp(-1.0))            # silu(1)
    s2 = 2 / (1 + math.exp(-2.0))            # silu(2)
    sm1 = -1 / (1 + math.exp(1.0))           # silu(-1)
    want = np.array([[2 * s1, 4 * s1],       # both slots kept: 0.5 + 0.5
                     [s1, 2 * s1],
                     [0.5 * s2, s2],         # one slot kept
                     [0.5 * 3 * sm1, 3 * sm1]])
    np.testing.assert_allclose(res["out"], want, rtol=2e-7)
