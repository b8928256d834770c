"""CPU oracle of the sparse attention that consumes a route -- TEST
INFRASTRUCTURE ONLY (the tests, the smoke check and the benchmark's CPU leg
may call it; the product package never imports it).

Source: "RouteRelay: Event-Triggered Cross-Layer Route Reuse for Efficient
Dynamic Sparse Attention" (arXiv 2609.07306):
  §2.1, after Eq. 2: the chunks a query row selects are expanded into token
      indices and handed to a sparse online-softmax attention kernel;
  §2.2 Eq. 3: o_i = softmax(q_i K_R^T / sqrt(d)) V_R over the reused route R;
  §4.3: the router leaves token expansion and causal masking to the
      attention backend unchanged.

Readings (the page leaves these open):
  * A chunk is `chunk` consecutive tokens: chunk j covers tokens
    j*chunk .. j*chunk + chunk - 1, for queries and keys alike.
  * Causal masking is the token-level rule: key token s is visible to query
    token t iff s <= t.  (The router's chunk rule j <= i is its coarse form.)
  * Only the route (the first `width` ids of a ledger row) is attended;
    sentinels are routing metadata, not attention targets.
  * The 1/sqrt(d) of Eq. 3 uses d = the token head dimension.
  * Ids that are -1 (padding) or outside [0, number of key chunks) are
    skipped.  Each remaining entry contributes its tokens once per
    occurrence (a ledger route never repeats an id).
  * A query token with no visible key gets a zero output row (Eq. 3 is
    undefined on an empty set).

Everything is computed in fp64 from the inputs as given (bf16 inputs are
widened exactly), one query chunk at a time: gather the expanded key list,
score, mask, softmax with the row maximum subtracted, weight the values.
"""
from __future__ import annotations

import math

import numpy as np


def expand_route(route_row, chunk: int, nk_chunks: int) -> np.ndarray:
    """Token indices of the chunks listed in one route row, in route order
    (§2.1: selected chunks expanded into token indices)."""
    toks = [np.arange(j * chunk, (j + 1) * chunk, dtype=np.int64)
            for j in (int(x) for x in route_row) if 0 <= j < nk_chunks]
    return np.concatenate(toks) if toks else np.zeros(0, dtype=np.int64)


def _chunk_rows(q_rows, k_rows, v_rows, keys, tok, causal: bool, sc: float):
    """Eq. 3 for the query tokens `tok` (their rows q_rows) against the key
    and value rows k_rows, v_rows gathered from the expanded route; `keys`
    holds those rows' token positions (for the causal rule)."""
    out = np.zeros(q_rows.shape, dtype=np.float64)
    if keys.size == 0:
        return out
    logits = (q_rows @ k_rows.T) * sc                             # [len(tok), len(keys)]
    visible = _visible(keys, tok, causal)
    logits = np.where(visible, logits, -np.inf)
    has_any = visible.any(axis=1)
    mx = np.where(has_any, logits.max(axis=1), 0.0)
    w = np.where(visible, np.exp(logits - mx[:, None]), 0.0)      # softmax numerators
    den = w.sum(axis=1)
    o = w @ v_rows
    out[has_any] = o[has_any] / den[has_any, None]
    return out


def _visible(keys, tok, causal: bool) -> np.ndarray:
    """[len(tok), len(keys)] mask: key token s is visible to query token t
    iff s <= t when causal, always otherwise."""
    if causal:
        return keys[None, :] <= tok[:, None]
    return np.ones((tok.size, keys.size), dtype=bool)


def _scale(dh: int, scale) -> float:
    return 1.0 / math.sqrt(dh) if scale is None else float(scale)


def sparse_attention_head(q, k, v, route, chunk: int, causal: bool, scale: float | None = None):
    """Eq. 3 for one head.  q [nq_tok, dh], k and v [nk_tok, dh], route
    [nq_tok // chunk, width] chunk ids.  Returns o [nq_tok, dh] in fp64."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    route = np.asarray(route)
    nq_tok, dh = q.shape
    nk_tok = k.shape[0]
    assert nq_tok % chunk == 0 and nk_tok % chunk == 0 and v.shape == k.shape
    assert route.shape[0] == nq_tok // chunk
    sc = _scale(dh, scale)
    out = np.zeros((nq_tok, dh), dtype=np.float64)
    for i in range(nq_tok // chunk):
        tok = np.arange(i * chunk, (i + 1) * chunk)
        keys = expand_route(route[i], chunk, nk_tok // chunk)
        out[tok] = _chunk_rows(q[tok], k[keys], v[keys], keys, tok, causal, sc)
    return out


def sparse_attention(q, k, v, route, chunk: int, causal: bool, scale: float | None = None):
    """Eq. 3 for every head: q [bh, nq_tok, dh], k, v [bh, nk_tok, dh],
    route [bh, nq_tok // chunk, width].  Returns [bh, nq_tok, dh] fp64."""
    q = np.asarray(q)
    out = np.zeros(q.shape, dtype=np.float64)
    for h in range(q.shape[0]):
        out[h] = sparse_attention_head(q[h], k[h], v[h], route[h], chunk, causal, scale)
    return out


def sparse_attention_rows(q, k, v, route, chunk: int, causal: bool, head: int, q_chunk: int,
                          scale: float | None = None):
    """Eq. 3 for the `chunk` query tokens of query chunk `q_chunk` of head
    `head` only (a sampled check on a large problem).  Same conventions as
    sparse_attention; k and v are gathered for this chunk's route only."""
    i = int(q_chunk)
    tok = np.arange(i * chunk, (i + 1) * chunk)
    keys = expand_route(np.asarray(route[head, i]), chunk, k.shape[1] // chunk)
    qq = np.asarray(q[head, i * chunk:(i + 1) * chunk], dtype=np.float64)
    kk = np.asarray(k[head, keys], dtype=np.float64)
    vv = np.asarray(v[head, keys], dtype=np.float64)
    return _chunk_rows(qq, kk, vv, keys, tok, causal, _scale(q.shape[2], scale))
