"""Parity of the sparse attention over a route (rr_sparse_attention,
include/rr_attention.h) with the oracle (oracle/attention.py).

Page: "RouteRelay: Event-Triggered Cross-Layer Route Reuse for Efficient
Dynamic Sparse Attention" (arXiv 2609.07306), §2.1 (chunks expanded into
token indices, online softmax) and §2.2 Eq. 3.

Tolerance, derived from the kernel's arithmetic: q, k, v are bf16, so every
product q_d k_d is exact in fp32 and the fp32 sums of DH terms carry a
relative error near DH * 2^-24; the softmax runs in fp32.  The one coarse
step is the rounding of the weights P to bf16 before the P.V product
(relative error <= 2^-8 each), while the normaliser sums the fp32 weights.
Hence, per output element, |o_gpu - o| <= 2^-8 * sum_s p_s |v_s| plus the
fp32 terms, where p is the exact softmax: the oracle evaluated on |v|
gives that weighted mean.  The bound asserted is (2^-8 + 2^-12) * that
mean + 1e-6.

The file is named so that pytest collects it after the routing tests.
"""
import numpy as np
import pytest
import torch

import oracle
import rr_workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
EPS_P = 2.0 ** -8 + 2.0 ** -12


@pytest.fixture(scope="module")
def rr():
    import cross_layer_route_b200 as rr
    torch.cuda.set_device(0)
    return rr


def _np(x):
    return x.float().cpu().numpy()


def _check(out, q, k, v, route, chunk, causal, width):
    qn, kn, vn = _np(q), _np(k), _np(v)
    rn = route[:, :, :width].numpy()
    ref = oracle.sparse_attention(qn, kn, vn, rn, chunk, causal)
    bound = EPS_P * oracle.sparse_attention(qn, kn, np.abs(vn), rn, chunk, causal) + 1e-6
    got = out.cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    bad = err > bound
    assert not bad.any(), (f"{int(bad.sum())} elements outside the bound; worst at "
                           f"{np.unravel_index(np.argmax(err - bound), err.shape)}: err {err.max():.3g}")
    return float((err / bound).max())


def _run(rr, q, k, v, route, chunk, causal, width=None):
    out = rr.sparse_attention(q.to(DEV), k.to(DEV), v.to(DEV), route.to(DEV), chunk, causal=causal,
                              width=width)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("dh,chunk,causal", [(128, 64, True), (128, 64, False), (64, 64, True),
                                             (64, 32, False), (128, 16, True), (64, 16, False),
                                             (128, 128, True), (64, 128, False), (128, 32, True)])
def test_matches_the_oracle_on_random_routes(rr, dh, chunk, causal):
    bh, n_chunks, width, stride = 3, 12, 6, 9
    q, k, v = W.attention_tokens(bh, n_chunks * chunk, dh, seed=dh + chunk)
    route = W.random_routes(bh, n_chunks, n_chunks, width, causal, seed=chunk, stride=stride, pad=0.2)
    out = _run(rr, q, k, v, route, chunk, causal, width)
    _check(out, q, k, v, route, chunk, causal, width)
    assert torch.isfinite(out).all()


def test_edge_routes(rr):
    # ids past the key chunks, below -1, past the query chunk under causal,
    # a repeated id, an all-padding row, and fewer key chunks than query chunks
    chunk, dh, nq_chunks, nk_chunks = 64, 128, 6, 4
    q, _, _ = W.attention_tokens(2, nq_chunks * chunk, dh, seed=1)
    _, k, v = W.attention_tokens(2, nk_chunks * chunk, dh, seed=2)
    rows = [[0, 1, 2, 3], [1, 9, -1, -5], [1, 1, 0, -1], [-1, -1, -1, -1], [3, 2, 4, 5], [5, 0, 2, 2]]
    route = torch.tensor([rows, rows[::-1]], dtype=torch.int32)
    for causal in (False, True):
        out = _run(rr, q, k, v, route, chunk, causal)
        _check(out, q, k, v, route, chunk, causal, 4)
    # an all-padding row, and width 0, give zero rows
    assert torch.count_nonzero(out[0, 3 * chunk:4 * chunk]) == 0
    out0 = _run(rr, q, k, v, route, chunk, True, width=0)
    assert torch.count_nonzero(out0) == 0


def test_nothing_to_do(rr):
    q = torch.empty((0, 128, 64), dtype=torch.bfloat16, device=DEV)
    route = torch.empty((0, 2, 4), dtype=torch.int32, device=DEV)
    out = rr.sparse_attention(q, q, q, route, 64)
    assert out.shape == (0, 128, 64)
    q1 = torch.empty((2, 0, 64), dtype=torch.bfloat16, device=DEV)
    k1 = torch.zeros((2, 128, 64), dtype=torch.bfloat16, device=DEV)
    out1 = rr.sparse_attention(q1, k1, k1, torch.empty((2, 0, 4), dtype=torch.int32, device=DEV), 64)
    assert out1.shape == (2, 0, 64)


def test_ledger_routes_feed_the_attention(rr):
    """The composition of §2.1: route with the ledger, then attend over the
    ledger's routes in place.  The in-place call must equal the call on a
    copy of the routes (same kernel, same ids), and both must match the
    oracle's attention over the oracle's own routes wherever the two
    routers chose the same set (all rows outside the tie margin)."""
    from rr_parity import config_of, params_of
    w = W.C5.with_(bh=2, n=256, layers=1)
    chunk, dh = 64, 128
    cfg = config_of(w, rr)
    led = rr.RouteLedger(cfg, DEV)
    qf, kf, qs, ks = W.LayerStream(w, "cpu").next()
    led.layer(qs.to(DEV), ks.to(DEV), 0)
    q, k, v = W.attention_tokens(w.bh, w.n * chunk, dh, seed=3)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    in_place = led.sparse_attention(qd, kd, vd, chunk)
    ids = led.read()["ids"]
    copy = rr.sparse_attention(qd, kd, vd, ids[:, :, :w.k].contiguous().to(DEV), chunk, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(in_place, copy)

    p = params_of(w)
    o_routes = np.full((w.bh, w.n, w.k), -1, dtype=np.int32)
    for h in range(w.bh):
        hl = oracle.HeadLedger.empty(p)
        oracle.head_layer(p, h, 0, True, qf[h].numpy(), kf[h].numpy(), hl)
        o_routes[h] = hl.ids[:, :w.k]
    same = np.array([[set(o_routes[h, i]) == set(ids[h, i, :w.k].tolist()) for i in range(w.n)]
                     for h in range(w.bh)])
    assert same.mean() >= 0.99
    qn, kn, vn = _np(q), _np(k), _np(v)
    ref = oracle.sparse_attention(qn, kn, vn, o_routes, chunk, True)
    bound = EPS_P * oracle.sparse_attention(qn, kn, np.abs(vn), o_routes, chunk, True) + 1e-6
    got = in_place.cpu().numpy()
    for h in range(w.bh):
        for i in np.nonzero(same[h])[0]:
            rows = slice(i * chunk, (i + 1) * chunk)
            assert (np.abs(got[h, rows] - ref[h, rows]) <= bound[h, rows]).all(), (h, i)


def test_full_size_sampled(rr):
    """Four heads of the largest workload at token level (4096 chunks of 64
    tokens per head, dh 128, route width 32, causal), one launch; the oracle
    checks 40 query chunks per head, the first and last among them."""
    a = W.ATTN_C5
    q, k, v = W.attention_tokens(a.bh, a.tokens, a.dh, seed=a.seed)
    route = W.random_routes(a.bh, a.n_chunks, a.n_chunks, a.k, a.causal, seed=a.seed, stride=a.k + 48)
    out = _run(rr, q, k, v, route, a.chunk, a.causal, a.k).cpu()
    assert torch.isfinite(out).all()
    qn, kn, vn = _np(q), _np(k), _np(v)
    rn = route[:, :, :a.k].numpy()
    rng = np.random.default_rng(11)
    for h in range(a.bh):
        sample = np.unique(np.concatenate([[0, 1, 31, 32, a.n_chunks - 1], rng.integers(0, a.n_chunks, 35)]))
        for i in sample:
            ref = oracle.sparse_attention_rows(qn, kn, vn, rn, a.chunk, a.causal, h, i)
            bound = EPS_P * oracle.sparse_attention_rows(qn, kn, np.abs(vn), rn, a.chunk, a.causal, h, i) + 1e-6
            got = out[h, i * a.chunk:(i + 1) * a.chunk].numpy()
            assert (np.abs(got - ref) <= bound).all(), (h, int(i))
