"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.  Bit-exact ids and flags outside the tie margin, alpha
within it (see rr_parity)."""
import numpy as np
import pytest
import torch

import oracle
import rr_workloads as W
from rr_parity import Report, compare_head, config_of, layer_stepped, params_of

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def rr():
    import cross_layer_route_b200 as rr
    torch.cuda.set_device(0)
    return rr


def _check(rep: Report, max_tie_frac=0.05):
    """No mismatch outside the tie margin, every tie row valid, and the tie
    rows a small share (at 4096 chunks the gap between neighbouring ranks is
    ~1e-4, so a 1e-5 margin catches a few percent of rows)."""
    assert not rep.mismatches, rep.mismatches[:10]
    assert rep.compared > 0
    assert rep.ties <= max(2, max_tie_frac * rep.rows), (rep.ties, rep.rows)
    print(f"rows={rep.rows} compared={rep.compared} tie_route={rep.tie_route} "
          f"tie_flag={rep.tie_flag} tie_identical={rep.tie_identical}")


def _workload(name, bh, n, d, dtype, k, m, r, causal, layers=1, H=4, sigma=0.03, seed=0, nk=None):
    return W.Workload(name, bh, n, d, dtype, layers, sigma, H, k, m, r, causal, seed)


ANCHOR_SHAPES = [
    # name, bh, n, d, dtype, k, m, r, causal
    ("pr1", 1, 128, 64, "f32", 12, 12, 4, False),
    ("ragged_causal", 3, 200, 64, "f32", 12, 12, 8, True),
    ("ragged_small", 2, 77, 8, "f32", 5, 7, 9, False),
    ("bf16_d128", 2, 300, 128, "bf16", 32, 32, 16, True),
    ("n_le_k", 2, 5, 16, "f32", 5, 3, 2, False),
    ("n_le_k_plus_m", 2, 20, 16, "f32", 12, 12, 4, False),
    ("pool_le_r", 2, 30, 16, "bf16", 12, 12, 8, True),
    ("max_ksel", 1, 300, 64, "f32", 64, 64, 128, False),
    ("no_sentinels", 2, 100, 32, "f32", 10, 0, 0, True),
    ("only_random", 2, 100, 32, "bf16", 10, 0, 30, False),
    ("d256", 1, 96, 256, "f32", 8, 8, 8, True),
    ("seed_big", 2, 150, 64, "f32", 12, 12, 12, True),
    # fp32 on the CUDA cores at d = 64 (k + m above the selection kernel's 64)
    ("f32_d64_cuda_cores", 2, 300, 64, "f32", 48, 24, 8, True),
    # shapes of the tensor-core path (bf16, d in {64, 128}, k + m <= 64, r <= 32;
    # fp32 at d = 64 with the three-way bf16 split)
    ("split_d64_causal", 3, 1000, 64, "f32", 12, 12, 8, True),
    ("split_exact_tile", 2, 256, 64, "f32", 40, 24, 32, False),
    ("split_k1_r0", 2, 129, 64, "f32", 1, 0, 0, True),
    ("split_wide_rows", 1, 4700, 64, "f32", 12, 12, 8, False),
    ("tc_d64", 3, 1000, 64, "bf16", 12, 12, 8, True),
    ("tc_d128_noncausal", 2, 300, 128, "bf16", 32, 32, 16, False),
    ("tc_small_n", 3, 70, 128, "bf16", 32, 32, 16, True),
    ("tc_exact_tile", 2, 256, 64, "bf16", 40, 24, 32, False),
    ("tc_k1_r0", 2, 129, 128, "bf16", 1, 0, 0, True),
    # rows longer than the finalize kernel's 4096-chunk membership bitmap
    ("tc_wide_rows", 1, 4700, 64, "bf16", 12, 12, 8, False),
]


@pytest.mark.parametrize("shape", ANCHOR_SHAPES, ids=[s[0] for s in ANCHOR_SHAPES])
def test_anchor_full_route_matches_oracle(rr, shape):
    name, bh, n, d, dt, k, m, r, causal = shape
    seed = 0xDEADBEEF12345 if name == "seed_big" else 3
    w = _workload(name, bh, n, d, dt, k, m, r, causal, layers=1, seed=seed)
    led = rr.RouteLedger(config_of(w, rr), DEV)
    rep, per_layer = layer_stepped(w, rr, led, 1, range(bh), DEV)
    _check(rep)
    cnt = per_layer[0][3]
    nv = sum(oracle.valid_count(i, n, causal) for i in range(n))
    assert int(cnt[rr.CNT_ROWS]) == bh * n and int(cnt[rr.CNT_PAIRS]) == bh * nv
    assert int(cnt[rr.CNT_ERROR]) == 0 and int(cnt[rr.CNT_LAYERS]) == 1


STEPPED = [
    (W.PR1, None),
    (W.C2.with_(bh=4, layers=12), None),
    (W.C3.with_(bh=2, layers=10), None),
    (W.C4.with_(bh=1, layers=10), None),
    (W.C5.with_(bh=1, n=1024, layers=18), None),
    (W.low_drift(W.C2).with_(bh=4, layers=12), "stable"),
    (W.low_drift(W.C5).with_(bh=1, n=768, layers=18), "stable"),
]


@pytest.mark.parametrize("case", STEPPED, ids=[c[0].name for c in STEPPED])
def test_layer_stepped_parity(rr, case):
    w, kind = case
    led = rr.RouteLedger(config_of(w, rr), DEV)
    rep, per_layer = layer_stepped(w, rr, led, w.layers, range(w.bh), DEV)
    _check(rep)
    for l, anchor, lr, cnt in per_layer:
        assert int(cnt[rr.CNT_LAST_LAYER]) == l and int(cnt[rr.CNT_ERROR]) == 0
        assert int(cnt[rr.CNT_ROWS]) == lr.refreshed_gpu
        assert abs(lr.refreshed_gpu - lr.refreshed_oracle) <= lr.tie_flag
        if lr.tie_flag == 0:
            assert int(cnt[rr.CNT_PAIRS]) == lr.pairs_oracle
    if kind == "stable":
        relay = [lr for l, a, lr, _ in per_layer if not a]
        assert sum(lr.refreshed_gpu for lr in relay) < 0.9 * sum(lr.rows for lr in relay)


FULL = [
    (W.C2.with_(layers=3), [0, 77, 127]),
    (W.C3.with_(layers=3), [0, 127]),
    (W.C4.with_(layers=2), [0, 63]),
    (W.C5.with_(layers=2), [0, 255]),
]


@pytest.mark.parametrize("case", FULL, ids=[c[0].name for c in FULL])
def test_full_size_sampled_heads(rr, case):
    """Full-size workloads in the launch configuration the benchmark uses;
    the oracle checks sampled heads (heads are independent and the random
    draws are keyed per head, so a sampled head is an exact check)."""
    w, heads = case
    led = rr.RouteLedger(config_of(w, rr), DEV)
    rep, per_layer = layer_stepped(w, rr, led, w.layers, heads, DEV, stream_device=DEV)
    _check(rep)
    for l, anchor, lr, cnt in per_layer:
        assert int(cnt[rr.CNT_ERROR]) == 0


def _drive(rr, w, led, layers, device=DEV):
    st = W.LayerStream(w, "cpu")
    xs = []
    for l in range(layers):
        _, _, qs, ks = st.next()
        xs.append((qs.to(device), ks.to(device)))
    for l, (q, k) in enumerate(xs):
        led.layer(q, k, l)
    return xs


def test_zero_drift_relay_keeps_routes(rr):
    w = W.C2.with_(bh=8, layers=1)
    led = rr.RouteLedger(config_of(w, rr), DEV)
    (q, k), = _drive(rr, w, led, 1)
    before = led.read()
    for l in (1, 2, 3):
        led.relay_layer(q, k, l)
    after = led.read()
    # ties aside (none expected at fp32 with random data), no row refreshes
    assert int(after["counters"][rr.CNT_ROWS]) == 0
    assert torch.equal(before["ids"], after["ids"])
    assert int(after["counters"][rr.CNT_PAIRS]) == 8 * 256 * w.c


def test_deterministic_and_graph_replay_equal_eager(rr):
    w = W.C3.with_(bh=6, layers=9, anchor_interval=4)
    st = W.LayerStream(w, "cpu")
    xs = []
    for l in range(w.layers):
        _, _, qs, ks = st.next()
        xs.append((qs.to(DEV), ks.to(DEV)))
    eager = rr.RouteLedger(config_of(w, rr), DEV)
    for l, (q, k) in enumerate(xs):
        eager.layer(q, k, l)
    a = eager.read()
    again = rr.RouteLedger(config_of(w, rr), DEV)
    for l, (q, k) in enumerate(xs):
        again.layer(q, k, l)
    b = again.read()
    assert torch.equal(a["ids"], b["ids"]) and torch.equal(a["alpha"], b["alpha"])
    graphed = rr.RouteLedger(config_of(w, rr), DEV)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):   # warm-up (first call sets kernel attributes)
        for l, (q, k) in enumerate(xs):
            graphed.layer(q, k, l)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for l, (q, k) in enumerate(xs):
            graphed.layer(q, k, l)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    c = graphed.read()
    assert torch.equal(a["ids"], c["ids"]) and torch.equal(a["alpha"], c["alpha"])
    assert torch.equal(a["anchor_layer"], c["anchor_layer"]) and torch.equal(a["flags"], c["flags"])


def test_head_shards_reproduce_the_joint_ledger(rr):
    w = W.C3.with_(bh=4, layers=5, anchor_interval=3)
    st = W.LayerStream(w, "cpu")
    full = rr.RouteLedger(config_of(w, rr), DEV)
    parts = [rr.RouteLedger(config_of(w, rr, bh=2, bh_offset=2 * s), DEV) for s in range(2)]
    for l in range(w.layers):
        _, _, qs, ks = st.next()
        q, k = qs.to(DEV), ks.to(DEV)
        full.layer(q, k, l)
        for s, p in enumerate(parts):
            p.layer(q[2 * s:2 * s + 2].contiguous(), k[2 * s:2 * s + 2].contiguous(), l)
    a = full.read()
    b = [p.read() for p in parts]
    assert torch.equal(a["ids"], torch.cat([x["ids"] for x in b]))
    assert torch.equal(a["alpha"], torch.cat([x["alpha"] for x in b]))


def test_out_of_range_ledger_id_sets_error_word(rr):
    w = W.C2.with_(bh=2, layers=1)
    led = rr.RouteLedger(config_of(w, rr), DEV)
    (q, k), = _drive(rr, w, led, 1)
    dv = led.device_view()
    dv["ids"][1, 7, 0] = w.n + 5      # an id no row may hold
    torch.cuda.synchronize()
    led.relay_layer(q, k, 1)
    with pytest.raises(rr.RRError) as e:
        led.read()
    assert e.value.status == rr.RR_EDEVICE
    out = led.read(check=False)
    assert int(out["counters"][rr.CNT_ERROR]) & 1


def test_layer_order_is_enforced(rr):
    w = W.C2.with_(bh=1, layers=1)
    led = rr.RouteLedger(config_of(w, rr), DEV)
    (q, k), = _drive(rr, w, led, 1)
    led.relay_layer(q, k, 3)
    for bad in (3, 2):
        with pytest.raises(rr.RRError) as e:
            led.relay_layer(q, k, bad)
        assert e.value.status == rr.RR_ESTATE
    led.full_route(q, k, 0)   # an anchor starts a new sequence at any layer
    led.relay_layer(q, k, 1)
    assert int(led.read()["counters"][rr.CNT_LAST_LAYER]) == 1


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("bf16", 64), ("f32", 64), ("f32", 32)])
def test_equal_scores_pick_lowest_chunks(rr, dtype, d):
    """All keys equal -> every score of a row ties: the route is the k lowest
    valid chunks and the near-miss the next m (ties go to the smaller index).
    On the tensor-core path this is the case the three-pass certificate
    rejects, so it also exercises the exact one-pass retry."""
    bh, n, k, m, r = 2, 300, 8, 6, 4
    cfg = rr.Config(bh=bh, nq=n, nk=n, d=d, k=k, m_near=m, r_rand=r, dtype=dtype, causal=True)
    g = torch.Generator().manual_seed(5)
    q = torch.randn((bh, n, d), generator=g)
    kk = torch.randn((bh, 1, d), generator=g).expand(bh, n, d).contiguous()
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    led = rr.RouteLedger(cfg, DEV)
    led.full_route(q.to(td).to(DEV), kk.to(td).to(DEV), 0)
    out = led.read()
    ids = out["ids"]
    for i in (0, 3, 7, 13, 14, 50, 299):
        nv = i + 1
        nr = min(k, nv)
        nm = min(m, nv - nr)
        assert ids[0, i, :nr].tolist() == list(range(nr))
        assert ids[0, i, k:k + nm].tolist() == list(range(nr, nr + nm))
        rand = [x for x in ids[0, i, k + m:].tolist() if x >= 0]
        assert len(rand) == min(r, nv - nr - nm) and all(nr + nm <= x < nv for x in rand)
    if d in (64, 128):   # tensor-core paths: every row overflows its slots and is redone
        assert int(out["counters"][rr.CNT_RETRY_TOTAL]) > 0


def test_retry_lists_longer_than_the_retry_grid(rr):
    """Equal keys again, with 640 heads: the retry launch has one CTA per head
    (about four per SM over all heads), and each head's 172 overflowing rows
    (the rows with more than 128 valid chunks) take six tiles of 32, so every
    retry CTA strides over several tiles.  Checked on every row of every
    head, after the anchor layer and after a relay layer (equal scores:
    alpha = beta, every row challenged and rebuilt)."""
    bh, n, d, k, m, r = 640, 300, 64, 8, 6, 4
    cfg = rr.Config(bh=bh, nq=n, nk=n, d=d, k=k, m_near=m, r_rand=r, dtype="bf16", causal=True)
    g = torch.Generator().manual_seed(11)
    q = torch.randn((bh, n, d), generator=g).to(torch.bfloat16).to(DEV)
    kk = torch.randn((bh, 1, d), generator=g).expand(bh, n, d).contiguous().to(torch.bfloat16).to(DEV)
    led = rr.RouteLedger(cfg, DEV)
    nv = np.arange(1, n + 1)
    nr = np.minimum(k, nv)
    nm = np.minimum(m, nv - nr)
    want = np.full((n, k + m), -1, dtype=np.int64)
    for i in range(n):
        want[i, :nr[i]] = np.arange(nr[i])
        want[i, k:k + nm[i]] = np.arange(nr[i], nr[i] + nm[i])
    for layer, call in ((0, led.full_route), (1, led.relay_layer)):
        call(q, kk, layer)
        out = led.read()
        ids = out["ids"].numpy().astype(np.int64)
        assert np.array_equal(ids[:, :, :k + m], np.broadcast_to(want, (bh, n, k + m))), layer
        rand = ids[:, :, k + m:]
        lo = (nr + nm)[None, :, None]
        ok = (rand == -1) | ((rand >= lo) & (rand < nv[None, :, None]))
        assert ok.all(), layer
        assert int(out["counters"][rr.CNT_RETRY_TOTAL]) >= (layer + 1) * bh * (n - 128)


def test_retry_path_is_rare_on_the_full_size_workload(rr):
    """On the bf16 workload the three-pass certificate should hold for nearly
    every row (the retry path is a safety net, not the common case)."""
    w = W.C5.with_(bh=16, layers=1)
    led = rr.RouteLedger(config_of(w, rr), DEV)
    _drive(rr, w, led, 1)
    c = led.read()["counters"]
    assert int(c[rr.CNT_RETRY_TOTAL]) <= 0.005 * w.bh * w.n, int(c[rr.CNT_RETRY_TOTAL])


GUARD = [
    (W.low_drift(W.C5).with_(bh=2, n=384, layers=10), "bf16_tensor_cores"),
    (W.low_drift(W.C3).with_(bh=2, layers=8), "f32_split_tensor_cores"),
    (W.low_drift(W.C3).with_(bh=2, d=32, layers=8), "f32_cuda_cores"),
]


@pytest.mark.parametrize("case", GUARD, ids=[c[1] for c in GUARD])
def test_per_row_margins_and_lifetime_bound(rr, case):
    """Relay with per-row guard margins gamma_i (Eq. 8) and a per-row
    lifetime bound, layer by layer against the oracle given the same margins
    and bound; afterwards no row's ledger is max_age or more layers old."""
    w, _ = case
    max_age = 3
    led = rr.RouteLedger(config_of(w, rr), DEV)
    g = torch.where(torch.rand(w.bh, w.n, generator=torch.Generator().manual_seed(7)) < 0.5,
                    torch.tensor(0.0), torch.tensor(0.05)).float()
    led.set_guard(g.reshape(-1).contiguous().to(DEV), max_age=max_age)
    rep, per_layer = layer_stepped(w, rr, led, w.layers, range(w.bh), DEV, gamma_rows=g.numpy(),
                                   max_age=max_age)
    _check(rep)
    last = led.read()
    assert int((w.layers - 1 - last["anchor_layer"]).max()) < max_age
    relay = [lr for l, a, lr, _ in per_layer if not a]
    assert sum(lr.refreshed_gpu for lr in relay) < sum(lr.rows for lr in relay)   # some rows were kept


HYST = [
    (W.C5.with_(bh=2, n=256, layers=8), "bf16_tensor_cores"),
    (W.C3.with_(bh=2, n=256, layers=8), "f32_split_tensor_cores"),
    (W.C3.with_(bh=2, n=256, d=32, layers=8), "f32_cuda_cores"),
]


@pytest.mark.parametrize("case", HYST, ids=[c[1] for c in HYST])
def test_hysteresis_horizon(rr, case):
    """Relay with a one-layer minimum reuse horizon (RouteRelay §3.2,
    Hysteresis) under the workload's high drift, layer by layer against the
    oracle given the same horizon: rows rebuilt at the previous layer are
    kept, the others follow the test."""
    w, _ = case
    led = rr.RouteLedger(config_of(w, rr), DEV)
    led.set_hysteresis(1)
    rep, per_layer = layer_stepped(w, rr, led, w.layers, range(w.bh), DEV, min_reuse=1)
    _check(rep)
    relay = [lr for l, a, lr, _ in per_layer if not a]
    # under this drift the test refreshes nearly every row, so the horizon
    # keeps about every other layer's rows
    assert sum(lr.refreshed_gpu for lr in relay) < 0.75 * sum(lr.rows for lr in relay)


GLOBALS = [
    (W.C5.with_(bh=2, n=384, layers=5), "bf16_tensor_cores"),
    (W.C3.with_(bh=2, n=256, layers=5), "f32_split_tensor_cores"),
    (W.C3.with_(bh=2, n=256, d=32, layers=5), "f32_cuda_cores"),
]


@pytest.mark.parametrize("case", GLOBALS, ids=[c[1] for c in GLOBALS])
def test_global_sentinels_layer_by_layer(rr, case):
    """Mandatory global sentinels (RouteRelay §3.1 item 3: 2 sink and 3
    recent chunks per row) on anchor and relay layers, against the oracle."""
    w, _ = case
    led = rr.RouteLedger(config_of(w, rr, g_sink=2, g_recent=3), DEV)
    rep, per_layer = layer_stepped(w, rr, led, w.layers, range(w.bh), DEV, g_sink=2, g_recent=3)
    _check(rep)


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64), ("f32", 32)])
def test_global_sentinels_on_equal_scores_match_the_oracle(rr, dtype, d):
    """All scores of a row tie, so route, near-miss and globals are fixed by
    the index order and the random draws by the exclusion set: every id must
    equal the oracle's.  On the tensor-core path these rows take the retry
    kernel."""
    bh, n, k, m, r, gs, gr = 1, 200, 8, 6, 4, 2, 3
    cfg = rr.Config(bh=bh, nq=n, nk=n, d=d, k=k, m_near=m, r_rand=r, dtype=dtype, causal=True,
                    g_sink=gs, g_recent=gr, seed=11)
    g = torch.Generator().manual_seed(6)
    q = torch.randn((bh, n, d), generator=g)
    kk = torch.randn((bh, 1, d), generator=g).expand(bh, n, d).contiguous()
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    led = rr.RouteLedger(cfg, DEV)
    led.full_route(q.to(td).to(DEV), kk.to(td).to(DEV), 0)
    out = led.read()
    p = oracle.Params(nq=n, nk=n, d=d, k=k, m=m, r=r, causal=True, seed=11, g_sink=gs, g_recent=gr)
    ol = oracle.HeadLedger.empty(p)
    oracle.head_layer(p, 0, 0, True, q.to(td).float()[0].numpy(), kk.to(td).float()[0].numpy(), ol)
    assert np.array_equal(out["ids"][0].numpy(), ol.ids)


HYST_MARGIN = [
    (W.low_drift(W.C5).with_(bh=2, n=384, layers=10), "bf16_tensor_cores"),
    (W.low_drift(W.C3).with_(bh=2, n=256, layers=10), "f32_split_tensor_cores"),
    (W.low_drift(W.C3).with_(bh=2, n=256, d=32, layers=10), "f32_cuda_cores"),
]


@pytest.mark.parametrize("case", HYST_MARGIN, ids=[c[1] for c in HYST_MARGIN])
def test_hysteresis_margin_marks_and_recovery(rr, case):
    """The larger guard margin after a refresh (RouteRelay §3.2,
    Hysteresis): rows rebuilt at a relay layer carry the mark (flags bit 1)
    and test with max(gamma_i, gamma_h) until they first pass.  Layer by
    layer against the oracle given the same margin: flags, marks, ids and
    alpha."""
    w, _ = case
    G = 0.01
    led = rr.RouteLedger(config_of(w, rr), DEV)
    led.set_hysteresis_margin(G)
    rep, per_layer = layer_stepped(w, rr, led, w.layers, range(w.bh), DEV, gamma_h=G)
    _check(rep)
    flags = led.read()["flags"]
    assert int(((flags >> 1) & 1).sum()) > 0                  # some rows carry the mark
    relay = [lr for l, a, lr, _ in per_layer if not a]
    assert sum(lr.refreshed_gpu for lr in relay) < sum(lr.rows for lr in relay)   # some rows were kept


def test_a_wait_that_runs_out_sets_the_error_bit_and_the_rows_are_redone(rr):
    """Every wait in the tensor-core kernels is bounded.  With the epilogue's
    accumulator waits cut to a few hundred cycles, a wait runs out while the
    selection kernel's copies and MMAs are in flight: the CTA drains its
    copies, waits for its last MMA, frees its TMEM and sets bit 1 of the
    error word; its rows go to the exact one-pass path, so the ledger still
    matches the oracle.  A ledger with the default budget is unaffected."""
    w = W.C5.with_(bh=2, n=384, layers=3)
    led = rr.RouteLedger(config_of(w, rr), DEV)
    rr.rr_ledger_set_wait_budget(led.handle, 300)
    rep, per_layer = layer_stepped(w, rr, led, w.layers, range(w.bh), DEV, check=False)
    _check(rep)
    err = [int(cnt[rr.CNT_ERROR]) for _, _, _, cnt in per_layer]
    assert all(e & 2 for e in err), err
    assert int(per_layer[-1][3][rr.CNT_RETRY_TOTAL]) > 0
    fresh = rr.RouteLedger(config_of(w, rr), DEV)
    rep2, per_layer2 = layer_stepped(w, rr, fresh, w.layers, range(w.bh), DEV)
    _check(rep2)
    assert all(int(cnt[rr.CNT_ERROR]) == 0 for _, _, _, cnt in per_layer2)


def test_split_fp32_scores_stay_within_the_split_error_bound(rr):
    """fp32 rows run on the tensor cores as six bf16 products of a three-way
    split (hi + mid + lo = x exactly); the dropped products add at most
    2^-23 |q||k| per score and the fp32 accumulation of 24 MMA steps a few
    2^-24 |q||k| more.  alpha (the k-th best score of every row, §3.2 Eq. 6)
    is checked against the fp64 k-th score on every row of a causal anchor:
    the worst error must stay below 2^-19 of the row's scale, 50 times inside
    the 1e-5 tie margin and about 2000 times below a bf16 rounding of the
    inputs."""
    w = W.C4.with_(bh=2, layers=1)
    cfg = config_of(w, rr)
    led = rr.RouteLedger(cfg, DEV)
    st = W.LayerStream(w, "cpu")
    qf, kf, qs, ks = st.next()
    led.full_route(qs.to(DEV), ks.to(DEV), 0)
    alpha = led.read()["alpha"].numpy().astype(np.float64)
    worst = 0.0
    for h in range(w.bh):
        q = qf[h].double().numpy()
        k = kf[h].double().numpy()
        S = q @ k.T
        scale = np.linalg.norm(q, axis=1) * np.linalg.norm(k, axis=1).max()
        for i in range(w.n):
            nv = i + 1
            if nv < w.k:
                continue
            kth = np.sort(S[i, :nv])[::-1][w.k - 1]
            worst = max(worst, abs(alpha[h, i] - kth) / scale[i])
    assert worst <= 2.0 ** -19, worst
    print(f"worst alpha error / row scale: {worst:.3e}")
