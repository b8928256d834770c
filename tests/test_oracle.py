"""Pins of the CPU oracle against what the RouteRelay page and mathematics fix.

Page: "RouteRelay: Event-Triggered Cross-Layer Route Reuse for Efficient
Dynamic Sparse Attention" (arXiv 2609.07306), cited as RouteRelay §x.
Each test names the fact it pins and would fail on a plausible slip in the
oracle (dropped term, wrong sign/index, transposed operand, wrong tie order,
wrong counting rule).
"""
import math
import os
import subprocess

import numpy as np
import pytest

import oracle
from oracle import Params

HERE = os.path.dirname(os.path.abspath(__file__))


def rownorm(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


# --------------------------------------------------------------- Eq. 1 --
def test_scores_match_float64_matmul_and_are_not_transposed():
    rng = np.random.default_rng(1)
    q = rng.standard_normal((7, 13)).astype(np.float32)
    k = rng.standard_normal((11, 13)).astype(np.float32)
    S = oracle.scores(q, k)
    ref = q.astype(np.float64) @ k.astype(np.float64).T
    assert S.shape == (7, 11)
    np.testing.assert_allclose(S, ref, rtol=1e-12, atol=1e-12)
    # no 1/sqrt(d) scaling (the scaling of Eq. 3 belongs to attention)
    e = np.eye(13, dtype=np.float32)
    assert np.array_equal(oracle.scores(e[:3] * 2, e[:3]), np.diag([2.0, 2.0, 2.0]))


def test_valid_count_causal():
    assert [oracle.valid_count(i, 5, True) for i in range(7)] == [1, 2, 3, 4, 5, 5, 5]
    assert [oracle.valid_count(i, 5, False) for i in range(3)] == [5, 5, 5]


# --------------------------------------------------------------- Eq. 2 --
def _rank_by_counting(s):
    """Independent definition: rank_j = #{j' : s_j' > s_j or (s_j' == s_j and j' < j)}."""
    n = len(s)
    rank = np.empty(n, dtype=np.int64)
    for j in range(n):
        rank[j] = sum(1 for jj in range(n) if s[jj] > s[j] or (s[jj] == s[j] and jj < j))
    order = np.empty(n, dtype=np.int64)
    order[rank] = np.arange(n)
    return order


@pytest.mark.parametrize("trial", range(40))
def test_route_row_equals_brute_force_ranks(trial):
    rng = np.random.default_rng(100 + trial)
    n = int(rng.integers(1, 17))
    if trial % 2:
        s = rng.integers(-3, 4, size=n).astype(np.float64)  # many exact ties
    else:
        s = rng.standard_normal(n)
    order = _rank_by_counting(s)
    for k in range(1, n + 2):
        for m in (0, 1, 3, n):
            route, near, alpha = oracle.route_row(s, n, k, m)
            nr = min(k, n)
            nm = min(m, n - nr)
            assert list(route[:nr]) == list(order[:nr])
            assert all(x == -1 for x in route[nr:])
            assert list(near[:nm]) == list(order[nr:nr + nm])
            assert all(x == -1 for x in near[nm:])
            assert alpha == min(s[j] for j in order[:nr])


def test_route_row_closed_forms():
    s = np.array([0.5, -1.0, 2.0, 0.25])
    route, near, alpha = oracle.route_row(s, 4, 4, 2)
    assert list(route) == [2, 0, 3, 1] and list(near) == [-1, -1]
    assert alpha == s.min()
    # causal prefix: only the first n_valid entries are candidates
    route, near, alpha = oracle.route_row(np.array([1.0, 9.0, 8.0]), 1, 2, 1)
    assert list(route) == [0, -1] and list(near) == [-1] and alpha == 1.0
    # equal scores: ascending index wins
    route, near, _ = oracle.route_row(np.array([1.0, 1.0, 1.0, 0.0]), 4, 2, 1)
    assert list(route) == [0, 1] and list(near) == [2]


# ------------------------------------------------------------ Philox ----
def test_philox_matches_torch_engine():
    """Cross-check against torch's own Philox4x32-10 engine (an independent
    implementation of Salmon et al., SC'11) compiled on the host."""
    import torch
    inc = os.path.join(os.path.dirname(torch.__file__), "include")
    src = os.path.join(HERE, "_philox_torch_check.cpp")
    exe = os.path.join(HERE, "..", "_build", "philox_torch_check")
    os.makedirs(os.path.dirname(exe), exist_ok=True)
    subprocess.check_call(["g++", "-std=c++17", "-O1", "-I" + inc, "-o", exe, src])
    rng = np.random.default_rng(7)
    cases = [(0, 0, 0, 0, 0, 0), (0xFFFFFFFF,) * 6]
    cases += [tuple(int(x) for x in rng.integers(0, 2**32, size=6)) for _ in range(30)]
    inp = "\n".join(" ".join(str(v) for v in c) for c in cases) + "\n"
    out = subprocess.run([exe], input=inp, capture_output=True, text=True, check=True).stdout.split("\n")
    for c, line in zip(cases, out):
        want = [int(x, 16) for x in line.split()]
        got = oracle.philox4x32_10(c[:4], c[4:])
        assert list(got) == want, (c, got, want)


# ------------------------------------------------- random sentinels -----
def test_random_sentinels_distinct_in_pool_and_fill():
    rng = np.random.default_rng(3)
    for trial in range(300):
        n = int(rng.integers(1, 80))
        n_ex = int(rng.integers(0, min(n, 30) + 1))
        excl = rng.choice(n, size=n_ex, replace=False).astype(np.int32)
        excl = np.concatenate([excl, np.full(int(rng.integers(0, 3)), -1, np.int32)])
        r = int(rng.integers(1, 20))
        out, draws = oracle.random_sentinels(trial, trial % 5, trial % 97, trial % 31, n, excl, r, 64 * 40)
        pool = sorted(set(range(n)) - set(int(x) for x in excl if x >= 0))
        got = [int(x) for x in out if x >= 0]
        assert len(set(got)) == len(got)
        assert set(got) <= set(pool)
        assert len(got) == min(r, len(pool))
        assert all(x == -1 for x in out[len(got):])
        if len(pool) <= r:
            assert got == pool and draws == 0


def test_random_sentinels_first_draw_is_multiply_shift_of_philox_word0():
    seed, bh, row, layer, n = 0x1234_5678_9ABC_DEF0, 3, 17, 5, 1000
    w = oracle.philox4x32_10([bh, row, layer, 0], [seed & 0xFFFFFFFF, seed >> 32])
    out, _ = oracle.random_sentinels(seed, bh, row, layer, n, [], 1, 64)
    assert out[0] == (int(w[0]) * n) >> 32


def test_random_sentinels_uniform_chi2():
    """Uniform over the residual pool (RouteRelay §3.1 item 2, §3.4)."""
    n, r = 40, 4
    excl = np.arange(0, 40, 4, dtype=np.int32)  # 10 excluded
    pool = sorted(set(range(n)) - set(excl.tolist()))
    counts = {j: 0 for j in pool}
    trials = 6000
    for t in range(trials):
        out, _ = oracle.random_sentinels(11, t % 7, t // 7, 2, n, excl, r, 64 * 24)
        for j in out:
            counts[int(j)] += 1
    obs = np.array([counts[j] for j in pool], dtype=np.float64)
    exp = trials * r / len(pool)
    chi2 = float(((obs - exp) ** 2 / exp).sum())
    # 29 degrees of freedom: the 99.9% quantile is 58.3
    assert chi2 < 58.3, chi2


def test_random_sentinels_miss_probability_eq10():
    """RouteRelay §3.4 Eq. 10: with u challengers in a residual pool of size
    N and r draws without replacement, P(miss all) = C(N-u, r)/C(N, r)."""
    n_valid, u, r = 60, 5, 6
    excl = np.arange(0, 12, dtype=np.int32)  # pool = 12..59, N = 48
    Np = n_valid - len(excl)
    challengers = set(range(30, 30 + u))
    p = math.comb(Np - u, r) / math.comb(Np, r)
    assert p <= (1 - u / Np) ** r  # the page's bound
    trials = 8000
    miss = 0
    for t in range(trials):
        out, _ = oracle.random_sentinels(99, 1, t, 3, n_valid, excl, r, 64 * 30)
        if not (set(int(x) for x in out) & challengers):
            miss += 1
    sd = math.sqrt(p * (1 - p) / trials)
    assert abs(miss / trials - p) < 3.3 * sd, (miss / trials, p)


# ---------------------------------------------------------- layers ------
def _layer_inputs(seed, bh, n, d, scale=1.0):
    rng = np.random.default_rng(seed)
    q = rownorm(rng.standard_normal((bh, n, d))).astype(np.float32)
    k = rownorm(rng.standard_normal((bh, n, d))).astype(np.float32)
    return q, k


@pytest.mark.parametrize("causal", [False, True])
def test_anchor_rows_are_full_routes_with_sentinels(causal):
    p = Params(nq=40, nk=40, d=16, k=5, m=4, r=3, causal=causal, seed=5)
    q, k = _layer_inputs(0, 1, 40, 16)
    led = oracle.HeadLedger.empty(p)
    flags, beta, ref, pairs, st = oracle.head_layer(p, 0, 0, True, q[0], k[0], led)
    assert st == 0 and ref == 40 and flags.all()
    S = q[0].astype(np.float64) @ k[0].astype(np.float64).T
    nv = [oracle.valid_count(i, 40, causal) for i in range(40)]
    assert pairs == sum(nv)
    for i in range(40):
        order = _rank_by_counting(S[i, : nv[i]])
        nr = min(5, nv[i]); nm = min(4, nv[i] - nr)
        assert list(led.ids[i, :nr]) == list(order[:nr])
        assert list(led.ids[i, 5:5 + nm]) == list(order[nr:nr + nm])
        assert led.alpha[i] == S[i, order[nr - 1]]
        rand = [int(x) for x in led.ids[i, 9:] if x >= 0]
        assert set(rand).isdisjoint(set(order[: nr + nm].tolist()))
        assert len(rand) == min(3, nv[i] - nr - nm)
        assert led.anchor_layer[i] == 0


def test_zero_drift_relay_keeps_every_route():
    """Same Q, K at the relay layer, distinct scores: alpha is the rank-k
    score and beta is at most the rank-(k+1) score, so Eq. 8 holds strictly
    for every row and no row refreshes."""
    p = Params(nq=64, nk=96, d=32, k=8, m=6, r=4, seed=1)
    q, k = _layer_inputs(2, 1, 96, 32)
    q = q[:, :64]
    led = oracle.HeadLedger.empty(p)
    oracle.head_layer(p, 0, 0, True, q[0], k[0], led)
    before = led.copy()
    flags, beta, ref, pairs, st = oracle.head_layer(p, 0, 1, False, q[0], k[0], led)
    assert st == 0 and ref == 0 and not flags.any()
    assert np.array_equal(led.ids, before.ids)
    assert np.array_equal(led.alpha, before.alpha)
    assert np.array_equal(led.anchor_layer, before.anchor_layer)
    assert pairs == 64 * p.c


def test_lemma1_bounded_perturbation_keeps_routes_and_raises_no_flag():
    """RouteRelay §3.3 Lemma 1: max_j |S^l - S^a| <= eps and Delta > 2 eps
    imply R^l = R^a; the relay test then also passes (alpha^l >= alpha^a -
    eps > max_{j not in R} S^a + eps >= beta^l)."""
    p = Params(nq=48, nk=64, d=24, k=6, m=5, r=4, seed=2)
    rng = np.random.default_rng(4)
    q, k = _layer_inputs(5, 1, 64, 24)
    q0 = q[0, :48].astype(np.float32)
    k0 = k[0]
    S_a = q0.astype(np.float64) @ k0.astype(np.float64).T
    srt = -np.sort(-S_a, axis=1)
    delta = srt[:, p.k - 1] - srt[:, p.k]  # Eq. 9 anchor margin
    kmax = np.linalg.norm(k0.astype(np.float64), axis=1).max()
    eps = 0.4 * delta
    d = rng.standard_normal(q0.shape)
    d = d / np.linalg.norm(d, axis=1, keepdims=True) * (eps / kmax)[:, None]
    q1 = (q0.astype(np.float64) + d).astype(np.float32)
    S_l = q1.astype(np.float64) @ k0.astype(np.float64).T
    assert (np.abs(S_l - S_a).max(axis=1) <= 0.45 * delta).all()
    led = oracle.HeadLedger.empty(p)
    oracle.head_layer(p, 0, 0, True, q0, k0, led)
    anchor_routes = led.ids[:, : p.k].copy()
    flags, beta, ref, pairs, st = oracle.head_layer(p, 0, 1, False, q1, k0, led)
    assert not flags.any() and ref == 0
    exact = oracle.exact_topk(p, q1, k0)
    for i in range(48):
        assert set(exact[i].tolist()) == set(anchor_routes[i].tolist())


def test_stability_condition_and_refresh_semantics():
    """Eq. 8 with a guard margin: rows with alpha > beta + gamma keep their
    ids bit for bit; the others are rebuilt as full routes at this layer."""
    for gamma in (0.0, 0.05):
        p = Params(nq=80, nk=80, d=16, k=6, m=6, r=4, causal=True, gamma=gamma, seed=9)
        rng = np.random.default_rng(6)
        q0, k0 = _layer_inputs(7, 1, 80, 16)
        q1 = rownorm(q0[0] + 0.3 * rng.standard_normal(q0[0].shape)).astype(np.float32)
        k1 = rownorm(k0[0] + 0.3 * rng.standard_normal(k0[0].shape)).astype(np.float32)
        led = oracle.HeadLedger.empty(p)
        oracle.head_layer(p, 0, 0, True, q0[0], k0[0], led)
        before = led.copy()
        flags, beta, ref, pairs, st = oracle.head_layer(p, 0, 3, False, q1, k1, led)
        S = q1.astype(np.float64) @ k1.astype(np.float64).T
        n_cand = 0
        for i in range(80):
            nv = oracle.valid_count(i, 80, True)
            ids = before.ids[i]
            r_ids = [j for j in ids[: p.k] if j >= 0]
            c_ids = [j for j in ids[p.k:] if j >= 0]
            n_cand += len(r_ids) + len(c_ids)
            a = min(S[i, j] for j in r_ids)
            b = max((S[i, j] for j in c_ids), default=-np.inf)
            assert beta[i] == b
            if a > b + gamma:
                assert flags[i] == 0
                assert np.array_equal(led.ids[i], before.ids[i])
                assert led.alpha[i] == a and led.anchor_layer[i] == 0
            else:
                assert flags[i] == 1 and led.anchor_layer[i] == 3
                route, near, alpha = oracle.route_row(S[i, :nv], nv, p.k, p.m)
                assert list(led.ids[i, : p.k]) == list(route)
                assert list(led.ids[i, p.k:p.k + p.m]) == list(near)
                excl = np.concatenate([route, near])
                rand, _ = oracle.random_sentinels(p.seed, 0, i, 3, nv, excl, p.r, 64 * p.c)
                assert list(led.ids[i, p.k + p.m:]) == list(rand)
                assert led.alpha[i] == alpha
        assert ref == int(flags.sum())
        assert pairs == n_cand + sum(oracle.valid_count(i, 80, True) for i in range(80) if flags[i])
        if gamma > 0:
            assert flags.sum() > 0


def test_rows_with_at_most_k_valid_chunks_never_refresh():
    p = Params(nq=10, nk=10, d=8, k=4, m=2, r=2, causal=True, seed=0)
    q0, k0 = _layer_inputs(8, 1, 10, 8)
    q1, k1 = _layer_inputs(9, 1, 10, 8)
    led = oracle.HeadLedger.empty(p)
    oracle.head_layer(p, 0, 0, True, q0[0], k0[0], led)
    flags, beta, *_ = oracle.head_layer(p, 0, 1, False, q1[0], k1[0], led)
    assert not flags[:4].any()
    assert np.isneginf(beta[:4]).all()


# --------------------------------------------------- counting rules -----
def _read_golden(name):
    rows = []
    with open(os.path.join(HERE, "golden", name)) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                rows.append(line.split())
    return rows


def test_counting_rule_reproduces_table3():
    """RouteRelay §5.2 Table 3: with one anchor at layer 0 of 24, the printed
    rerouted fraction f and the counting rule (anchor rows count as
    rerouted and cost n; relay rows cost c plus n when refreshed) must give
    the printed score-pair fraction, within the tables' rounding."""
    n, L = 256, 24

    def pairs(f, c, rule):
        s_rho = L * f - 1.0  # relay-layer sum of refreshed fractions
        if rule == "page":
            return oracle.pair_fraction_from_counts(L, n, n, c, [s_rho * n] + [0.0] * (L - 2))
        if rule == "no_candidates":
            return (1 + s_rho) / L
        if rule == "anchor_not_rerouted":
            return (1 + (L - 1) * c / n + L * f) / L
        raise ValueError(rule)

    def matches(f_pct, c, p_pct, rule):
        fs = np.linspace(f_pct - 0.05, f_pct + 0.05, 201) / 100
        vals = np.array([pairs(f, c, rule) for f in fs]) * 100
        return bool(((vals >= p_pct - 0.05) & (vals <= p_pct + 0.05)).any())

    rows = _read_golden("table3_sentinel_ablation.txt")
    assert len(rows) == 4
    for label, k, m, r, f_pct, p_pct in rows:
        c = int(k) + int(m) + int(r)
        assert matches(float(f_pct), c, float(p_pct), "page"), label
    # the readings that were rejected do not reproduce the table
    assert not all(matches(float(f), int(k) + int(m) + int(r), float(pp), "no_candidates")
                   for _, k, m, r, f, pp in rows)
    assert not all(matches(float(f), int(k) + int(m) + int(r), float(pp), "anchor_not_rerouted")
                   for _, k, m, r, f, pp in rows)


def test_rerouted_rows_count_anchor_layers_table2():
    """RouteRelay §5.1 Table 2: refreshing every row at every fourth of 32
    layers is 25.0% rerouted rows; routing every layer is 100.0%."""
    p = Params(nq=6, nk=6, d=4, k=2, m=1, r=1, seed=0)
    rng = np.random.default_rng(0)
    for label, layers, H, pct in _read_golden("table2_fixed_stride.txt"):
        layers, H = int(layers), int(H)
        rt = oracle.Router(p, bh=1, anchor_interval=H)
        for l in range(layers):
            q = rng.standard_normal((1, 6, 4)).astype(np.float32)
            k = rng.standard_normal((1, 6, 4)).astype(np.float32)
            # "fixed stride": every non-anchor layer reuses without testing
            anchor = oracle.is_anchor(l, H)
            if anchor:
                rt.step(l, q, k, recall=False)
            else:
                rt.stats.append(oracle.LayerStats(l, False, 0, 0))
        s = rt.summary()
        assert abs(100 * s["rerouted_fraction"] - float(pct)) < 0.05, label


def test_router_counters_follow_counting_rule():
    p = Params(nq=32, nk=32, d=8, k=4, m=3, r=2, causal=True, seed=3)
    rng = np.random.default_rng(1)
    rt = oracle.Router(p, bh=2, anchor_interval=4)
    x_q = rownorm(rng.standard_normal((2, 32, 8)))
    x_k = rownorm(rng.standard_normal((2, 32, 8)))
    for l in range(6):
        before = [led.copy() for led in rt.ledgers]
        res, st = rt.step(l, x_q.astype(np.float32), x_k.astype(np.float32))
        nv = np.array([oracle.valid_count(i, 32, True) for i in range(32)])
        if st.anchor:
            assert st.refreshed == 64 and st.pairs == 2 * nv.sum()
        else:
            cand = sum(int((b.ids >= 0).sum()) for b in before)
            fl = [r[0] for r in res]
            assert st.refreshed == sum(int(f.sum()) for f in fl)
            assert st.pairs == cand + sum(int(nv[f.astype(bool)].sum()) for f in fl)
        x_q = rownorm(x_q + 0.2 * rng.standard_normal(x_q.shape))
        x_k = rownorm(x_k + 0.2 * rng.standard_normal(x_k.shape))


def test_sharded_heads_equal_unsharded():
    """Heads are independent and the random key carries the global head
    index, so running heads in two shards reproduces the joint run."""
    p = Params(nq=24, nk=24, d=8, k=3, m=3, r=3, seed=12)
    rng = np.random.default_rng(2)
    qs = [rng.standard_normal((4, 24, 8)).astype(np.float32) for _ in range(3)]
    ks = [rng.standard_normal((4, 24, 8)).astype(np.float32) for _ in range(3)]
    full = oracle.Router(p, bh=4, anchor_interval=2)
    a = oracle.Router(p, bh=2, anchor_interval=2, bh_offset=0)
    b = oracle.Router(p, bh=2, anchor_interval=2, bh_offset=2)
    for l in range(3):
        full.step(l, qs[l], ks[l], recall=False)
        a.step(l, qs[l][:2], ks[l][:2], recall=False)
        b.step(l, qs[l][2:], ks[l][2:], recall=False)
    for h in range(4):
        part = a.ledgers[h] if h < 2 else b.ledgers[h - 2]
        assert np.array_equal(full.ledgers[h].ids, part.ids)
        assert np.array_equal(full.ledgers[h].alpha, part.alpha)


def test_recall_is_one_when_every_layer_is_an_anchor():
    p = Params(nq=16, nk=16, d=8, k=3, m=2, r=2, seed=0)
    rng = np.random.default_rng(5)
    rt = oracle.Router(p, bh=1, anchor_interval=1)
    for l in range(4):
        rt.step(l, rng.standard_normal((1, 16, 8)).astype(np.float32),
                rng.standard_normal((1, 16, 8)).astype(np.float32))
    s = rt.summary()
    assert s["recall"] == 1.0 and s["rerouted_fraction"] == 1.0 and s["pair_fraction"] == 1.0


# ---- per-row guard margins and lifetime bound (RouteRelay §3.2 Eq. 8 gamma_i;
# "Forced anchors ... bound the lifetime of stale random sentinels") ----------

def _drifting_layers(bh, n, d, layers, sigma, seed):
    rng = np.random.default_rng(seed)
    q = rownorm(rng.standard_normal((bh, n, d)))
    k = rownorm(rng.standard_normal((bh, n, d)))
    out = []
    for _ in range(layers):
        out.append((q.astype(np.float32), k.astype(np.float32)))
        q = rownorm(q + sigma * rng.standard_normal(q.shape))
        k = rownorm(k + sigma * rng.standard_normal(k.shape))
    return out


def _run(p, bh, layers_qk, H, gamma_rows=None):
    rt = oracle.Router(p, bh=bh, anchor_interval=H, gamma_rows=gamma_rows)
    hist = []
    for l, (q, k) in enumerate(layers_qk):
        res, _ = rt.step(l, q, k, recall=False)
        hist.append(([led.copy() for led in rt.ledgers], [r[0].copy() for r in res], [r[1].copy() for r in res]))
    return hist


def test_gamma_rows_equal_to_the_scalar_reproduce_the_scalar_run():
    p = Params(nq=40, nk=40, d=8, k=4, m=3, r=2, causal=True, gamma=0.02, seed=4)
    lq = _drifting_layers(2, 40, 8, 7, 0.15, 21)
    a = _run(p, 2, lq, 8)
    b = _run(p, 2, lq, 8, gamma_rows=np.full((2, 40), 0.02))
    for (la, fa, _), (lb, fb, _) in zip(a, b):
        for h in range(2):
            assert np.array_equal(la[h].ids, lb[h].ids)
            assert np.array_equal(la[h].alpha, lb[h].alpha)
            assert np.array_equal(fa[h], fb[h])


def test_mixed_gamma_rows_follow_the_uniform_run_of_each_row():
    """Rows are independent (own ledger, own random key), so a run with a
    per-row margin equals, row by row, the run whose margin is that row's for
    every row."""
    p0 = Params(nq=48, nk=48, d=8, k=4, m=3, r=3, causal=False, gamma=0.0, seed=9)
    big = 1e9
    lq = _drifting_layers(2, 48, 8, 8, 0.1, 33)
    g = np.where(np.random.default_rng(5).random((2, 48)) < 0.5, 0.0, big)
    mixed = _run(p0, 2, lq, 8, gamma_rows=g)
    zero = _run(p0, 2, lq, 8)
    huge = _run(Params(**{**p0.__dict__, "gamma": big}), 2, lq, 8)
    assert sum(int(f.sum()) for f in zero[3][1]) < 2 * 48   # margin 0 keeps some rows
    for l in range(8):
        for h in range(2):
            for i in range(48):
                ref = huge if g[h, i] > 0 else zero
                assert np.array_equal(mixed[l][0][h].ids[i], ref[l][0][h].ids[i]), (l, h, i)
                assert mixed[l][0][h].alpha[i] == ref[l][0][h].alpha[i]
                assert mixed[l][1][h][i] == ref[l][1][h][i]
            # a huge margin refreshes every relay row
            if l % 8:
                assert all(mixed[l][1][h][i] == 1 for i in range(48) if g[h, i] > 0)


def test_max_age_one_routes_every_layer_exactly():
    p = Params(nq=32, nk=32, d=8, k=4, m=2, r=2, causal=True, seed=6, max_age=1)
    lq = _drifting_layers(1, 32, 8, 6, 0.02, 8)
    rt = oracle.Router(p, bh=1, anchor_interval=100)
    for l, (q, k) in enumerate(lq):
        res, st = rt.step(l, q, k)
        assert st.refreshed == 32
        assert all(int(f) == 1 for f in res[0][0])
    s = rt.summary()
    assert s["recall"] == 1.0 and s["rerouted_fraction"] == 1.0


def test_max_age_bounds_every_rows_ledger_age_and_leaves_younger_rows_to_the_test():
    A = 3
    p = Params(nq=40, nk=40, d=8, k=4, m=3, r=2, causal=False, seed=2, max_age=A)
    lq = _drifting_layers(1, 40, 8, 10, 0.03, 44)   # low drift: many stable rows
    rt = oracle.Router(p, bh=1, anchor_interval=100)
    forced_seen = 0
    for l, (q, k) in enumerate(lq):
        before = rt.ledgers[0].copy()
        res, _ = rt.step(l, q, k, recall=False)
        flags, beta = res[0][0], res[0][1]
        after = rt.ledgers[0]
        assert np.all(l - after.anchor_layer < A)        # no row reused A or more layers after it was built
        if l == 0:
            continue
        S = oracle.scores(q[0], k[0])
        for i in range(40):
            a = min(S[i, j] for j in before.ids[i, : p.k] if j >= 0)
            test_refresh = not (a > beta[i] + p.gamma)
            if l - before.anchor_layer[i] >= A:
                assert flags[i] == 1
                forced_seen += int(not test_refresh)
            else:
                assert flags[i] == int(test_refresh)
    assert forced_seen > 0   # the bound actually forced some otherwise stable rows


# ---- hysteresis: minimum reuse horizon (RouteRelay §3.2 "Hysteresis") --------

def test_min_reuse_keeps_rebuilt_rows_for_the_horizon_and_tests_the_rest():
    h = 2
    p = Params(nq=32, nk=32, d=8, k=4, m=2, r=2, causal=True, seed=8, min_reuse=h)
    lq = _drifting_layers(1, 32, 8, 9, 0.6, 61)   # high drift: the test refreshes most rows
    rt = oracle.Router(p, bh=1, anchor_interval=100)
    kept_by_horizon = 0
    for l, (q, k) in enumerate(lq):
        before = rt.ledgers[0].copy()
        res, _ = rt.step(l, q, k, recall=False)
        if l == 0:
            continue
        flags, beta = res[0][0], res[0][1]
        S = oracle.scores(q[0], k[0])
        for i in range(32):
            age = l - before.anchor_layer[i]
            a = min(S[i, j] for j in before.ids[i, : p.k] if j >= 0)
            test_refresh = not (a > beta[i] + p.gamma)
            if age <= h:
                assert flags[i] == 0 and np.array_equal(rt.ledgers[0].ids[i], before.ids[i])
                kept_by_horizon += int(test_refresh)
            else:
                assert flags[i] == int(test_refresh)
    assert kept_by_horizon > 0


def test_min_reuse_beyond_the_run_never_refreshes_and_the_bound_takes_precedence():
    lq = _drifting_layers(1, 24, 8, 6, 0.6, 62)
    p = Params(nq=24, nk=24, d=8, k=3, m=2, r=2, seed=1, min_reuse=10)
    rt = oracle.Router(p, bh=1, anchor_interval=100)
    rt.step(0, *lq[0], recall=False)
    anchor_ids = rt.ledgers[0].ids.copy()
    for l in range(1, 6):
        res, st = rt.step(l, *lq[l], recall=False)
        assert st.refreshed == 0
    assert np.array_equal(rt.ledgers[0].ids, anchor_ids)
    # a lifetime bound shorter than the horizon still forces the refresh
    p2 = Params(nq=24, nk=24, d=8, k=3, m=2, r=2, seed=1, min_reuse=10, max_age=2)
    rt2 = oracle.Router(p2, bh=1, anchor_interval=100)
    for l in range(6):
        res, st = rt2.step(l, *lq[l], recall=False)
        assert np.all(l - rt2.ledgers[0].anchor_layer < 2)


# ---- hysteresis: elevated guard margin after a refresh (RouteRelay §3.2
# "Hysteresis": a refreshed row "may use a larger guard margin until its
# anchor margin recovers").  Reading: a row rebuilt at a relay layer is marked;
# a marked row's test uses max(gamma_i, gamma_h); its first pass clears the
# mark; a row built at an anchor layer is unmarked. ------------------------

def _alpha_beta(S, ids_row, k):
    r = [S[j] for j in ids_row[:k] if j >= 0]
    s = [S[j] for j in ids_row[k:] if j >= 0]
    return min(r), (max(s) if s else -np.inf)


def test_elevated_margin_applies_to_refreshed_rows_until_they_pass():
    G = 0.1
    p = Params(nq=40, nk=40, d=8, k=4, m=3, r=2, causal=False, seed=12, gamma_h=G)
    lq = _drifting_layers(1, 40, 8, 12, 0.12, 71)
    rt = oracle.Router(p, bh=1, anchor_interval=6)
    flipped = recovered = stayed = 0
    for l, (q, k) in enumerate(lq):
        before = rt.ledgers[0].copy()
        res, _ = rt.step(l, q, k, recall=False)
        flags = res[0][0]
        after = rt.ledgers[0]
        if oracle.is_anchor(l, 6):
            assert np.all(after.elevated == 0) and np.all(flags == 1)
            continue
        S = oracle.scores(q[0], k[0])
        for i in range(40):
            a, b = _alpha_beta(S[i], before.ids[i], p.k)
            margin = G if before.elevated[i] else 0.0
            expect = int(not (a > b + margin))
            assert flags[i] == expect, (l, i)
            assert after.elevated[i] == expect, (l, i)   # refreshed: marked; passed: cleared
            if before.elevated[i]:
                flipped += int(expect == 1 and a > b)   # the larger margin decided this one
                recovered += int(expect == 0)
            stayed += int(expect == 0 and not before.elevated[i])
    assert flipped > 0 and recovered > 0 and stayed > 0


def test_elevated_margin_off_is_the_plain_test_and_gamma_rows_below_it_are_raised():
    lq = _drifting_layers(2, 32, 8, 8, 0.12, 72)
    base = Params(nq=32, nk=32, d=8, k=4, m=2, r=2, causal=True, seed=3)
    a = _run(base, 2, lq, 5)
    b = _run(Params(**{**base.__dict__, "gamma_h": 0.0}), 2, lq, 5)
    for (la, fa, _), (lb, fb, _) in zip(a, b):
        for h in range(2):
            assert np.array_equal(la[h].ids, lb[h].ids) and np.array_equal(fa[h], fb[h])
            assert not lb[h].elevated.any()
    # a per-row margin above gamma_h is not lowered by the mark: with gamma_h
    # below every gamma_i the run equals the run without the mark
    g = np.full((2, 32), 0.05)
    c = _run(Params(**{**base.__dict__, "gamma_h": 0.01}), 2, lq, 5, gamma_rows=g)
    d = _run(base, 2, lq, 5, gamma_rows=g)
    for (lc, fc, _), (ld, fd, _) in zip(c, d):
        for h in range(2):
            assert np.array_equal(lc[h].ids, ld[h].ids) and np.array_equal(fc[h], fd[h])


def test_elevated_margin_with_the_reuse_horizon_keeps_the_mark_until_tested():
    G, hz = 0.1, 1
    p = Params(nq=32, nk=32, d=8, k=4, m=2, r=2, causal=False, seed=5, gamma_h=G, min_reuse=hz)
    lq = _drifting_layers(1, 32, 8, 10, 0.2, 73)
    rt = oracle.Router(p, bh=1, anchor_interval=100)
    kept_marked = 0
    for l, (q, k) in enumerate(lq):
        before = rt.ledgers[0].copy()
        res, _ = rt.step(l, q, k, recall=False)
        if l == 0:
            continue
        flags, after = res[0][0], rt.ledgers[0]
        S = oracle.scores(q[0], k[0])
        for i in range(32):
            if l - before.anchor_layer[i] <= hz:   # inside the horizon: no test, mark unchanged
                assert flags[i] == 0 and after.elevated[i] == before.elevated[i]
                kept_marked += int(before.elevated[i])
            else:
                a, b = _alpha_beta(S[i], before.ids[i], p.k)
                expect = int(not (a > b + (G if before.elevated[i] else 0.0)))
                assert flags[i] == expect and after.elevated[i] == expect
    assert kept_marked > 0


# ---- mandatory global sentinels (RouteRelay §3.1 item 3: sink and recent) ----

@pytest.mark.parametrize("causal", [True, False])
def test_global_sentinels_are_the_sink_and_recent_chunks_outside_the_route(causal):
    gs, gr = 2, 3
    p = Params(nq=40, nk=40, d=8, k=4, m=3, r=3, causal=causal, seed=5, g_sink=gs, g_recent=gr)
    rng = np.random.default_rng(17)
    q = rownorm(rng.standard_normal((40, 8))).astype(np.float32)
    k = rownorm(rng.standard_normal((40, 8))).astype(np.float32)
    led = oracle.HeadLedger.empty(p)
    oracle.head_layer(p, 0, 0, True, q, k, led)
    base = oracle.HeadLedger.empty(Params(**{**p.__dict__, "g_sink": 0, "g_recent": 0}))
    oracle.head_layer(Params(**{**p.__dict__, "g_sink": 0, "g_recent": 0}), 0, 0, True, q, k, base)
    for i in range(40):
        nv = oracle.valid_count(i, 40, causal)
        row = led.ids[i]
        sel = [int(x) for x in row[: p.k + p.m] if x >= 0]
        assert np.array_equal(row[: p.k + p.m], base.ids[i, : p.k + p.m])   # route / near-miss unchanged
        want = []
        for j in list(range(gs)) + list(range(i - gr + 1, i + 1)):
            if 0 <= j < nv and j not in sel and j not in want:
                want.append(j)
        glob = [int(x) for x in row[p.k + p.m + p.r:]]
        assert glob == want + [-1] * (gs + gr - len(want)), i
        rand = [int(x) for x in row[p.k + p.m: p.k + p.m + p.r] if x >= 0]
        pool = [j for j in range(nv) if j not in sel and j not in want]
        assert len(set(rand)) == len(rand) and all(j in pool for j in rand)
        assert len(rand) == min(p.r, len(pool))
        if len(pool) <= p.r:
            assert rand == pool                                            # the whole pool, ascending


def test_global_sentinels_take_part_in_beta():
    """At a relay layer beta is the maximum over every sentinel, globals
    included (Eq. 7 over C_i, which holds near-miss, random and global
    candidates)."""
    p = Params(nq=32, nk=32, d=8, k=3, m=2, r=2, causal=True, seed=3, g_sink=2, g_recent=2)
    lq = _drifting_layers(1, 32, 8, 3, 0.3, 71)
    led = oracle.HeadLedger.empty(p)
    oracle.head_layer(p, 0, 0, True, lq[0][0][0], lq[0][1][0], led)
    before = led.copy()
    flags, beta, _, _, _ = oracle.head_layer(p, 0, 1, False, lq[1][0][0], lq[1][1][0], led)
    S = oracle.scores(lq[1][0][0], lq[1][1][0])
    n_glob_max = 0
    for i in range(32):
        sent = [int(j) for j in before.ids[i, p.k:] if j >= 0]
        if sent:
            assert beta[i] == max(S[i, j] for j in sent)
        glob = [int(j) for j in before.ids[i, p.k + p.m + p.r:] if j >= 0]
        if glob and sent and max(S[i, j] for j in glob) == beta[i]:
            n_glob_max += 1
    assert n_glob_max > 0   # some rows' beta comes from a global candidate


# ---- properties of the routing on random small problems (hypothesis) ---------
from hypothesis import assume, given, settings, strategies as st  # noqa: E402


def _min_gap(S, nv):
    """Smallest gap between distinct-rank scores of each row's valid prefix."""
    g = np.inf
    for i in range(S.shape[0]):
        s = np.sort(S[i, : nv[i]])
        if s.size > 1:
            g = min(g, float(np.min(np.diff(s))))
    return g


@settings(max_examples=40, deadline=None)
@given(seed=st.integers(0, 2**31 - 1), causal=st.booleans(), scale_exp=st.integers(-2, 3),
       nq=st.integers(2, 20), nk=st.integers(2, 20), k=st.integers(1, 4), m=st.integers(0, 4),
       r=st.integers(0, 4))
def test_a_positive_key_scale_and_a_common_key_shift_keep_every_decision(seed, causal, scale_exp, nq, nk,
                                                                         k, m, r):
    """k_j -> 2^e k_j + c scales every score of row i by 2^e and adds q_i . c:
    each row's order, its alpha - beta sign (gamma = 0) and therefore the
    whole ledger (random draws depend only on the excluded set) and every
    refresh flag stay the same, over an anchor and a relay layer."""
    assume(k <= nk)
    rng = np.random.default_rng(seed)
    d = 6
    p = Params(nq=nq, nk=nk, d=d, k=k, m=m, r=r, causal=causal, seed=seed)
    layers = [(rng.standard_normal((nq, d)).astype(np.float32), rng.standard_normal((nk, d)).astype(np.float32))
              for _ in range(2)]
    a = np.float32(2.0 ** scale_exp)
    c = rng.standard_normal(d).astype(np.float32)
    nv = [oracle.valid_count(i, nk, causal) for i in range(nq)]
    for q, kk in layers:   # no near-ties that fp32 rounding of the shift could flip
        for kx in (kk, a * kk + c):
            assume(_min_gap(oracle.scores(q, kx), nv) > 1e-4)
    A, B = oracle.HeadLedger.empty(p), oracle.HeadLedger.empty(p)
    for layer, (q, kk) in enumerate(layers):
        fa, ba, ra, _, _ = oracle.head_layer(p, 0, layer, layer == 0, q, kk, A)
        fb, bb, rb, _, _ = oracle.head_layer(p, 0, layer, layer == 0, q, a * kk + c, B)
        if layer > 0:   # the relay margins must not sit at the decision boundary either
            r_ids = [[j for j in A.ids[i, :k] if j >= 0] for i in range(nq)]
            S = oracle.scores(q, kk)
            margin = [min(S[i, j] for j in r_ids[i]) - ba[i] for i in range(nq) if r_ids[i]]
            assume(all(abs(x) > 1e-4 or not np.isfinite(x) for x in margin))
        assert np.array_equal(fa, fb) and ra == rb
        assert np.array_equal(A.ids, B.ids) and np.array_equal(A.anchor_layer, B.anchor_layer)


@settings(max_examples=40, deadline=None)
@given(seed=st.integers(0, 2**31 - 1), nq=st.integers(1, 16), nk=st.integers(2, 24), k=st.integers(1, 5),
       m=st.integers(0, 5))
def test_permuting_queries_and_keys_permutes_routes_and_near_misses(seed, nq, nk, k, m):
    """Non-causal anchor: relabelling the key chunks by a permutation P and
    reordering the query rows maps each row's route and near-miss ids
    through P (distinct scores: no tie to break) and keeps alpha."""
    assume(k <= nk)
    rng = np.random.default_rng(seed)
    d = 5
    q = rng.standard_normal((nq, d)).astype(np.float32)
    kk = rng.standard_normal((nk, d)).astype(np.float32)
    assume(_min_gap(oracle.scores(q, kk), [nk] * nq) > 1e-6)
    P = rng.permutation(nk)             # new key index of old key j is P[j]
    R = rng.permutation(nq)             # new row r holds old row R[r]
    kp = np.empty_like(kk)
    kp[P] = kk
    p = Params(nq=nq, nk=nk, d=d, k=k, m=m, r=0, seed=seed)
    A, B = oracle.HeadLedger.empty(p), oracle.HeadLedger.empty(p)
    oracle.head_layer(p, 0, 0, True, q, kk, A)
    oracle.head_layer(p, 0, 0, True, q[R], kp, B)
    w = k + m
    mapped = np.where(A.ids[:, :w] >= 0, P[np.maximum(A.ids[:, :w], 0)], -1)
    assert np.array_equal(B.ids[:, :w], mapped[R])
    assert np.array_equal(B.alpha, A.alpha[R])
