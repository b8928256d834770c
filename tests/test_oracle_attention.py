"""Pins of the sparse-attention oracle (oracle/attention.py) against what the
RouteRelay page and mathematics fix.

Page: "RouteRelay: Event-Triggered Cross-Layer Route Reuse for Efficient
Dynamic Sparse Attention" (arXiv 2609.07306): §2.1 (selected chunks expanded
into token indices for a sparse online-softmax kernel), §2.2 Eq. 3
(o_i = softmax(q_i K_R^T / sqrt(d)) V_R).

The pins: a full route reduces to dense (causal) attention, computed by
torch's own scaled_dot_product_attention; zero queries give the plain mean
of the expanded, visible value rows (closed form, with the token sets built
here by explicit loops); constant values come back unchanged; a lone
visible key returns its value row.  The last tests plant mistakes in the
oracle (strict causal rule, no 1/sqrt(d), wrong chunk expansion) and check
that a pin catches each one.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as A


def _inputs(rng, bh, n_tok, dh):
    return tuple(rng.standard_normal((bh, n_tok, dh)) for _ in range(3))


def _sdpa(q, k, v, causal):
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(torch.float64)
    return torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), is_causal=causal).numpy()


def _full_routes(rng, bh, n_chunks, causal, width):
    """Every valid chunk of each query chunk, shuffled, with -1 padding mixed in."""
    route = np.full((bh, n_chunks, width), -1, dtype=np.int32)
    for h in range(bh):
        for i in range(n_chunks):
            ids = np.arange(i + 1 if causal else n_chunks)
            rng.shuffle(ids)
            slots = np.sort(rng.choice(width, size=ids.size, replace=False))
            route[h, i, slots] = ids
    return route


def _random_routes(rng, bh, n_chunks, causal, width):
    """Up to `width` distinct valid chunks per query chunk, -1 padded at the end."""
    route = np.full((bh, n_chunks, width), -1, dtype=np.int32)
    for h in range(bh):
        for i in range(n_chunks):
            n_valid = i + 1 if causal else n_chunks
            ids = rng.choice(n_valid, size=min(width, n_valid), replace=False)
            route[h, i, :ids.size] = ids
    return route


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("chunk,dh", [(4, 8), (16, 32), (1, 5)])
def test_full_route_is_dense_attention(causal, chunk, dh):
    # Eq. 3 with R = every valid chunk is ordinary (causal) attention
    rng = np.random.default_rng(10 + chunk)
    n_chunks = 6
    q, k, v = _inputs(rng, 3, n_chunks * chunk, dh)
    route = _full_routes(rng, 3, n_chunks, causal, width=n_chunks + 3)
    got = oracle.sparse_attention(q, k, v, route, chunk, causal)
    np.testing.assert_allclose(got, _sdpa(q, k, v, causal), rtol=1e-12, atol=1e-12)


def _token_set(route_row, chunk, nk_chunks, t, causal):
    out = []
    for j in route_row:
        j = int(j)
        if j < 0 or j >= nk_chunks:
            continue
        for s in range(j * chunk, j * chunk + chunk):
            if not causal or s <= t:
                out.append(s)
    return out


@pytest.mark.parametrize("causal", [False, True])
def test_zero_queries_average_the_visible_expanded_tokens(causal):
    # q = 0: every logit is 0, softmax is uniform over the visible expanded
    # tokens; with V = I the output row is that uniform distribution.
    rng = np.random.default_rng(3)
    chunk, n_chunks, width = 4, 8, 3
    n_tok = chunk * n_chunks
    q = np.zeros((2, n_tok, n_tok))
    k = rng.standard_normal((2, n_tok, n_tok))
    v = np.broadcast_to(np.eye(n_tok), (2, n_tok, n_tok)).copy()
    route = np.empty((2, n_chunks, width), dtype=np.int32)
    for h in range(2):                       # distinct ids per row, like a ledger route
        for i in range(n_chunks):
            ids = rng.choice(n_chunks, size=width, replace=False)
            route[h, i] = np.where(rng.random(width) < 0.25, -1, ids)
    got = oracle.sparse_attention(q, k, v, route, chunk, causal)
    for h in range(2):
        for t in range(n_tok):
            T = _token_set(route[h, t // chunk], chunk, n_chunks, t, causal)
            want = np.zeros(n_tok)
            if T:
                want[T] = 1.0 / len(T)
            np.testing.assert_allclose(got[h, t], want, rtol=0, atol=1e-15)


def test_constant_values_and_empty_rows():
    rng = np.random.default_rng(4)
    chunk, n_chunks, dh = 8, 5, 16
    q, k, _ = _inputs(rng, 1, chunk * n_chunks, dh)
    v = np.broadcast_to(rng.standard_normal(dh), (1, chunk * n_chunks, dh)).copy()
    route = np.array([[[2, -1], [-1, -1], [0, 1], [4, 3], [7, -1]]], dtype=np.int32)  # 7: out of range
    got = oracle.sparse_attention(q, k, v, route, chunk, causal=False)
    for i in range(n_chunks):
        rows = got[0, i * chunk:(i + 1) * chunk]
        if i in (1, 4):                       # nothing to attend: zero rows
            assert np.all(rows == 0)
        else:                                 # weights sum to one
            np.testing.assert_allclose(rows, np.broadcast_to(v[0, 0], rows.shape), rtol=1e-13, atol=1e-13)


def test_lone_visible_key_returns_its_value_row():
    # causal, route = own chunk only: the first token of each chunk sees itself alone
    rng = np.random.default_rng(5)
    chunk, n_chunks, dh = 4, 6, 8
    q, k, v = _inputs(rng, 2, chunk * n_chunks, dh)
    route = np.broadcast_to(np.arange(n_chunks, dtype=np.int32)[None, :, None], (2, n_chunks, 1)).copy()
    got = oracle.sparse_attention(q, k, v, route, chunk, causal=True)
    first = np.arange(n_chunks) * chunk
    np.testing.assert_array_equal(got[:, first], v[:, first])


def test_route_order_padding_and_scale_invariances():
    rng = np.random.default_rng(6)
    chunk, n_chunks, dh = 4, 8, 16
    q, k, v = _inputs(rng, 1, chunk * n_chunks, dh)
    route = np.stack([rng.choice(n_chunks, size=3, replace=False) for _ in range(n_chunks)])[None].astype(np.int32)
    base = oracle.sparse_attention(q, k, v, route, chunk, causal=False)
    shuffled = route[:, :, ::-1].copy()
    padded = np.concatenate([np.full((1, n_chunks, 2), -1, np.int32), route], axis=2)
    np.testing.assert_allclose(oracle.sparse_attention(q, k, v, shuffled, chunk, False), base, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(oracle.sparse_attention(q, k, v, padded, chunk, False), base, rtol=1e-12, atol=1e-13)
    # an explicit scale s equals the default scale applied to q * s * sqrt(dh)
    s = 0.37
    np.testing.assert_allclose(oracle.sparse_attention(q, k, v, route, chunk, False, scale=s),
                               oracle.sparse_attention(q * s * math.sqrt(dh), k, v, route, chunk, False),
                               rtol=1e-12, atol=1e-13)


def test_sampled_rows_match_the_whole_problem():
    rng = np.random.default_rng(7)
    chunk, n_chunks, dh = 8, 6, 16
    q, k, v = _inputs(rng, 2, chunk * n_chunks, dh)
    route = _random_routes(rng, 2, n_chunks, True, width=4)
    whole = oracle.sparse_attention(q, k, v, route, chunk, causal=True)
    for h in range(2):
        for i in range(n_chunks):
            part = oracle.sparse_attention_rows(q, k, v, route, chunk, True, h, i)
            np.testing.assert_array_equal(part, whole[h, i * chunk:(i + 1) * chunk])


# ---- planted mistakes: each must break a pin ------------------------------
def _dense_pin_holds(causal=True):
    rng = np.random.default_rng(8)
    chunk, n_chunks, dh = 4, 5, 8
    q, k, v = _inputs(rng, 1, chunk * n_chunks, dh)
    route = _full_routes(rng, 1, n_chunks, causal, width=n_chunks)
    return np.allclose(oracle.sparse_attention(q, k, v, route, chunk, causal), _sdpa(q, k, v, causal),
                       rtol=1e-9, atol=1e-9)


def test_planted_mistakes_are_caught(monkeypatch):
    assert _dense_pin_holds()
    with monkeypatch.context() as m:          # strict causal rule (s < t)
        m.setattr(A, "_visible", lambda keys, tok, causal: keys[None, :] < tok[:, None] if causal
                  else np.ones((tok.size, keys.size), dtype=bool))
        assert not _dense_pin_holds()
    with monkeypatch.context() as m:          # Eq. 3 without 1/sqrt(d)
        m.setattr(A, "_scale", lambda dh, scale: 1.0)
        assert not _dense_pin_holds()
    with monkeypatch.context() as m:          # chunk j expanded from token j instead of j*chunk
        m.setattr(A, "expand_route", lambda row, chunk, nk: np.concatenate(
            [np.arange(j, j + chunk) for j in (int(x) for x in row) if 0 <= j < nk] or [np.zeros(0, np.int64)]))
        assert not _dense_pin_holds(causal=False) or not _dense_pin_holds(causal=True)


# ---- properties Eq. 3 must have, on random small problems --------------------
from hypothesis import given, settings, strategies as st  # noqa: E402


@st.composite
def _problem(draw):
    chunk = draw(st.sampled_from([1, 2, 4]))
    n_chunks = draw(st.integers(1, 5))
    dh = draw(st.integers(1, 6))
    width = draw(st.integers(0, 6))
    causal = draw(st.booleans())
    seed = draw(st.integers(0, 2**31 - 1))
    rng = np.random.default_rng(seed)
    n_tok = chunk * n_chunks
    q, k, v = (rng.standard_normal((1, n_tok, dh)) for _ in range(3))
    route = rng.integers(-2, n_chunks + 2, size=(1, n_chunks, width)).astype(np.int32)
    return q, k, v, route, chunk, causal, rng


@settings(max_examples=60, deadline=None)
@given(_problem())
def test_a_common_key_shift_leaves_every_softmax_unchanged(p):
    # k_s -> k_s + c adds q_t . c / sqrt(d) to every logit of query t
    q, k, v, route, chunk, causal, rng = p
    c = rng.standard_normal(k.shape[2])
    a = oracle.sparse_attention(q, k, v, route, chunk, causal)
    b = oracle.sparse_attention(q, k + c, v, route, chunk, causal)
    np.testing.assert_allclose(b, a, rtol=1e-9, atol=1e-9)


@settings(max_examples=60, deadline=None)
@given(_problem())
def test_outputs_are_affine_in_the_values(p):
    # o(a v + b) = a o(v) + b on rows that see at least one key (weights sum to 1)
    q, k, v, route, chunk, causal, rng = p
    alpha, beta = rng.standard_normal(), rng.standard_normal(v.shape[2])
    o = oracle.sparse_attention(q, k, v, route, chunk, causal)
    seen = oracle.sparse_attention(q, k, np.ones_like(v), route, chunk, causal)[0, :, 0] != 0
    o2 = oracle.sparse_attention(q, k, alpha * v + beta, route, chunk, causal)
    np.testing.assert_allclose(o2[0, seen], alpha * o[0, seen] + beta, rtol=1e-9, atol=1e-9)
    assert np.all(o2[0, ~seen] == 0) and np.all(o[0, ~seen] == 0)


@settings(max_examples=60, deadline=None)
@given(_problem())
def test_route_order_and_padding_are_irrelevant(p):
    q, k, v, route, chunk, causal, rng = p
    a = oracle.sparse_attention(q, k, v, route, chunk, causal)
    perm = route[:, :, rng.permutation(route.shape[2])]
    padded = np.concatenate([perm, np.full((1, route.shape[1], 2), -1, np.int32)], axis=2)
    np.testing.assert_allclose(oracle.sparse_attention(q, k, v, padded, chunk, causal), a, rtol=1e-9, atol=1e-12)
