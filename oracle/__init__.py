"""CPU oracle of the RouteRelay routing path -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product package never imports it and the
two share no code.  The arithmetic lives in ``rr_oracle.c`` (plain C, fp64);
this module only marshals numpy arrays through ctypes and keeps the
multi-head, multi-layer bookkeeping of the evaluation loop.

Source: "RouteRelay: Event-Triggered Cross-Layer Route Reuse for Efficient
Dynamic Sparse Attention" (arXiv 2609.07306), abbreviated RouteRelay:
§2.1 Eq. 1-2 (scores, TopK), §3.1 Eq. 4 (ledger, sentinel classes),
§3.2 Eq. 5-8 (relay test and refresh), §3.2 "Forced anchors" (anchor every
H layers), §4.1 (ledger dataflow), §5.1-5.2 (recall, rerouted rows, score
pairs).

The submodule ``oracle.attention`` (plain NumPy, fp64) is the oracle of the
downstream consumer of a route: token expansion and the sparse attention of
§2.2 Eq. 3.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rr_oracle.c")
_LIB_PATH = os.path.join(_HERE, "librr_oracle.so")
_lib = None
_lib_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile rr_oracle.c into librr_oracle.so (gcc, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fno-fast-math",
                               "-ffp-contract=off", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Params(ctypes.Structure):
    _fields_ = [("nq", ctypes.c_int32), ("nk", ctypes.c_int32), ("d", ctypes.c_int32),
                ("k", ctypes.c_int32), ("m", ctypes.c_int32), ("r", ctypes.c_int32),
                ("causal", ctypes.c_int32), ("max_draws", ctypes.c_int32),
                ("gamma", ctypes.c_double), ("seed", ctypes.c_uint64),
                ("max_age", ctypes.c_int32), ("min_reuse", ctypes.c_int32),
                ("g_sink", ctypes.c_int32), ("g_recent", ctypes.c_int32), ("gamma_h", ctypes.c_double)]


def lib():
    global _lib
    with _lib_lock:
        if _lib is None:
            _lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            i32 = ctypes.c_int32
            _lib.rro_scores.argtypes = [P, P, i32, i32, i32, P]
            _lib.rro_valid_count.argtypes = [i32, i32, i32]
            _lib.rro_valid_count.restype = i32
            _lib.rro_route_row.argtypes = [P, i32, i32, i32, P, P, P]
            _lib.rro_route_row.restype = i32
            _lib.rro_philox4x32_10.argtypes = [P, P, P]
            _lib.rro_random_sentinels.argtypes = [ctypes.c_uint64, i32, i32, i32, i32, P, i32, i32, i32, P]
            _lib.rro_random_sentinels.restype = i32
            _lib.rro_head_layer.argtypes = [ctypes.POINTER(_Params), i32, i32, i32, P, P, P, P, P, P, P, P, P, P]
            _lib.rro_head_layer.restype = i32
            _lib.rro_exact_topk.argtypes = [ctypes.POINTER(_Params), P, P, P]
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


@dataclass
class Params:
    """Problem statement of one routed head (RouteRelay §2.1, §3.1, §3.2)."""
    nq: int
    nk: int
    d: int
    k: int
    m: int
    r: int
    causal: bool = False
    gamma: float = 0.0
    seed: int = 0
    max_draws: int | None = None  # default 64 * (k + m + r)
    max_age: int = 0              # per-row lifetime bound (0: off)
    min_reuse: int = 0            # hysteresis: layers a rebuilt row is reused without the test
    g_sink: int = 0               # mandatory global sentinels: sink chunks 0..g_sink-1
    g_recent: int = 0             # ... and the row's recent chunks i-g_recent+1..i
    gamma_h: float = 0.0          # hysteresis: larger guard margin of a refreshed row (0: off)

    @property
    def c(self) -> int:
        return self.k + self.m + self.r + self.g_sink + self.g_recent

    def _c(self) -> _Params:
        md = self.max_draws if self.max_draws is not None else 64 * self.c
        return _Params(self.nq, self.nk, self.d, self.k, self.m, self.r, int(bool(self.causal)), md,
                       float(self.gamma), int(self.seed) & 0xFFFFFFFFFFFFFFFF, int(self.max_age),
                       int(self.min_reuse), int(self.g_sink), int(self.g_recent), float(self.gamma_h))


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def scores(q, k) -> np.ndarray:
    """S = Qc Kc^T in fp64 (RouteRelay Eq. 1). q [nq,d], k [nk,d]."""
    q = _f32(q); k = _f32(k)
    S = np.empty((q.shape[0], k.shape[0]), dtype=np.float64)
    lib().rro_scores(_ptr(q), _ptr(k), q.shape[0], k.shape[0], q.shape[1], _ptr(S))
    return S


def valid_count(i: int, nk: int, causal: bool) -> int:
    return int(lib().rro_valid_count(i, nk, int(bool(causal))))


def route_row(s_row, n_valid: int, k: int, m: int):
    """Top-k route and m near-miss ids of one row, plus alpha (Eq. 2, §3.1)."""
    s = np.ascontiguousarray(np.asarray(s_row, dtype=np.float64))
    route = np.empty(max(k, 1), dtype=np.int32)
    near = np.empty(max(m, 1), dtype=np.int32)
    alpha = ctypes.c_double()
    lib().rro_route_row(_ptr(s), n_valid, k, m, _ptr(route), _ptr(near), ctypes.byref(alpha))
    return route[:k].copy(), near[:m].copy(), alpha.value


def philox4x32_10(ctr, key) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(ctr, dtype=np.uint32))
    kk = np.ascontiguousarray(np.asarray(key, dtype=np.uint32))
    out = np.empty(4, dtype=np.uint32)
    lib().rro_philox4x32_10(_ptr(c), _ptr(kk), _ptr(out))
    return out


def random_sentinels(seed: int, bh: int, row: int, layer: int, n_valid: int, excl, r: int,
                     max_draws: int):
    """Random sentinels of one row (§3.1 item 2, §3.4). Returns (ids, draws)."""
    e = np.ascontiguousarray(np.asarray(excl, dtype=np.int32))
    if e.size == 0:
        e = np.full(1, -1, dtype=np.int32)
    out = np.empty(max(r, 1), dtype=np.int32)
    t = lib().rro_random_sentinels(int(seed) & 0xFFFFFFFFFFFFFFFF, bh, row, layer, n_valid,
                                   _ptr(e), e.size, r, max_draws, _ptr(out))
    return out[:r].copy(), int(t)


def exact_topk(p: Params, q, k) -> np.ndarray:
    """Exact per-layer top-k (the 'route every layer' reference, §5.1)."""
    q = _f32(q); k = _f32(k)
    out = np.empty((p.nq, p.k), dtype=np.int32)
    cp = p._c()
    lib().rro_exact_topk(ctypes.byref(cp), _ptr(q), _ptr(k), _ptr(out))
    return out


@dataclass
class HeadLedger:
    """Ledger of one head: ids [nq, c] (route | near-miss | random), alpha,
    anchor layer (RouteRelay Eq. 4, §4.1), and the per-row mark of the
    elevated guard margin (1 = the row's next test uses gamma_h)."""
    ids: np.ndarray
    alpha: np.ndarray
    anchor_layer: np.ndarray
    elevated: np.ndarray = None

    def __post_init__(self):
        if self.elevated is None:
            self.elevated = np.zeros(self.ids.shape[0], dtype=np.uint8)

    @staticmethod
    def empty(p: Params) -> "HeadLedger":
        return HeadLedger(np.full((p.nq, p.c), -1, dtype=np.int32),
                          np.zeros(p.nq, dtype=np.float64),
                          np.full(p.nq, -1, dtype=np.int32))

    def copy(self) -> "HeadLedger":
        return HeadLedger(self.ids.copy(), self.alpha.copy(), self.anchor_layer.copy(), self.elevated.copy())


def head_layer(p: Params, bh: int, layer: int, anchor: bool, q, k, led: HeadLedger, gamma_rows=None):
    """One layer of one head, in place on ``led``.  gamma_rows: per-row
    guard margins [nq] (RouteRelay Eq. 8 gamma_i), or None for p.gamma on
    every row.  Returns (flags, beta, refreshed_rows, score_pairs, status)."""
    q = _f32(q); k = _f32(k)
    g = None
    if gamma_rows is not None:
        g = np.ascontiguousarray(np.asarray(gamma_rows, dtype=np.float64))
        assert g.shape == (p.nq,)
    assert q.shape == (p.nq, p.d) and k.shape == (p.nk, p.d)
    flags = np.zeros(p.nq, dtype=np.uint8)
    beta = np.empty(p.nq, dtype=np.float64)
    counts = np.zeros(2, dtype=np.int64)
    cp = p._c()
    st = lib().rro_head_layer(ctypes.byref(cp), bh, layer, int(bool(anchor)), _ptr(q), _ptr(k),
                              _ptr(led.ids), _ptr(led.alpha), _ptr(led.anchor_layer),
                              _ptr(flags), _ptr(beta), _ptr(counts), _ptr(g) if g is not None else None,
                              _ptr(led.elevated))
    return flags, beta, int(counts[0]), int(counts[1]), int(st)


def is_anchor(layer: int, anchor_interval: int) -> bool:
    """Forced anchors every H layers (RouteRelay §3.2), layer 0 included."""
    return layer == 0 or (anchor_interval > 0 and layer % anchor_interval == 0)


@dataclass
class LayerStats:
    layer: int
    anchor: bool
    refreshed: int
    pairs: int
    recall_hits: int = 0
    recall_total: int = 0


@dataclass
class Router:
    """Multi-head, multi-layer oracle run (the evaluation loop of RouteRelay
    §5.1: anchor or relay at each layer, recall against exact per-layer
    top-k).  Heads run in a thread pool (each head is independent)."""
    p: Params
    bh: int
    anchor_interval: int
    bh_offset: int = 0
    threads: int = 1
    gamma_rows: object = None   # [bh, nq] per-row guard margins, or None
    ledgers: list = field(default_factory=list)
    stats: list = field(default_factory=list)

    def __post_init__(self):
        self.ledgers = [HeadLedger.empty(self.p) for _ in range(self.bh)]

    def _map(self, fn, items):
        if self.threads <= 1:
            return [fn(x) for x in items]
        with ThreadPoolExecutor(self.threads) as ex:
            return list(ex.map(fn, items))

    def step(self, layer: int, q, k, heads=None, recall: bool = True, anchor: bool | None = None):
        """q, k: [BH, N, d] float32 arrays (all heads) for this layer."""
        if anchor is None:
            anchor = is_anchor(layer, self.anchor_interval)
        heads = list(range(self.bh)) if heads is None else list(heads)

        def one(h):
            g = None if self.gamma_rows is None else self.gamma_rows[h]
            flags, beta, ref, pairs, st = head_layer(self.p, self.bh_offset + h, layer, anchor,
                                                      q[h], k[h], self.ledgers[h], gamma_rows=g)
            hits = tot = 0
            if recall:
                ex = exact_topk(self.p, q[h], k[h])
                used = self.ledgers[h].ids[:, : self.p.k]
                for i in range(self.p.nq):
                    e = set(int(x) for x in ex[i] if x >= 0)
                    u = set(int(x) for x in used[i] if x >= 0)
                    hits += len(e & u)
                    tot += len(e)
            return flags, beta, ref, pairs, st, hits, tot

        res = self._map(one, heads)
        st = LayerStats(layer, anchor, sum(r[2] for r in res), sum(r[3] for r in res),
                        sum(r[5] for r in res), sum(r[6] for r in res))
        self.stats.append(st)
        return res, st

    def summary(self) -> dict:
        return summarize(self.stats, self.p, len(self.ledgers))


def summarize(stats, p: Params, bh: int) -> dict:
    """Recall (pooled over rows, mean over layers), rerouted-row fraction and
    score-pair fraction relative to full per-layer routing (§5.1-5.2)."""
    full_pairs_per_layer = bh * sum(valid_count(i, p.nk, p.causal) for i in range(p.nq))
    L = len(stats)
    rec = [s.recall_hits / s.recall_total for s in stats if s.recall_total]
    return {
        "layers": L,
        "recall": float(np.mean(rec)) if rec else float("nan"),
        "rerouted_fraction": sum(s.refreshed for s in stats) / (L * bh * p.nq) if L else float("nan"),
        "pair_fraction": sum(s.pairs for s in stats) / (L * full_pairs_per_layer) if L else float("nan"),
    }


def pair_fraction_from_counts(n_layers: int, rows: int, n_valid_per_row: int, c: int,
                              refreshed_per_relay_layer) -> float:
    """Counting rule on its own: layer 0 is an anchor (every row costs
    n_valid), each later layer costs c per row plus n_valid per refreshed
    row; the result is relative to n_layers full routings."""
    total = rows * n_valid_per_row
    for ref in refreshed_per_relay_layer:
        total += rows * c + ref * n_valid_per_row
    return total / (n_layers * rows * n_valid_per_row)


from .attention import expand_route, sparse_attention, sparse_attention_head, sparse_attention_rows  # noqa: E402,F401
