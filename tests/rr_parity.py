"""Parity helpers: compare the CUDA path's ledger with the CPU oracle, layer by
layer, on the same seeded inputs.

Tie margin: the oracle ranks in fp64, the kernels in fp32.  A row whose
decision rests on a score gap below TIE_REL x scale (scale = |q_i| x max_j
|k_j|, about 1 for the row-normalised workloads) may legitimately come out
either way; such rows are counted and reported, not compared bit for bit.
The gaps that decide a row are: the rank-k / rank-(k+1) gap (route set), the
rank-(k+m) / rank-(k+m+1) gap (near-miss set, hence the random pool), and at
a relay layer alpha - beta - gamma (the refresh decision).  Everything else
must match: ids bit for bit, order up to equal scores, alpha within the
margin, flags, anchor layers and counters.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

import oracle

TIE_REL = 1e-5


def params_of(w, bh_offset: int = 0, max_age: int = 0, min_reuse: int = 0, g_sink: int = 0,
              g_recent: int = 0, gamma_h: float = 0.0) -> oracle.Params:
    return oracle.Params(nq=w.n, nk=w.n, d=w.d, k=w.k, m=w.m, r=w.r, causal=w.causal,
                         gamma=w.gamma, seed=w.seed, max_age=max_age, min_reuse=min_reuse,
                         g_sink=g_sink, g_recent=g_recent, gamma_h=gamma_h)


def config_of(w, rr, bh: int | None = None, bh_offset: int = 0, g_sink: int = 0, g_recent: int = 0):
    return rr.Config(bh=w.bh if bh is None else bh, nq=w.n, nk=w.n, d=w.d, k=w.k, m_near=w.m,
                     r_rand=w.r, dtype=w.dtype, anchor_interval=w.anchor_interval, causal=w.causal,
                     gamma=w.gamma, seed=w.seed, bh_offset=bh_offset, g_sink=g_sink, g_recent=g_recent)


@dataclass
class Report:
    rows: int = 0
    compared: int = 0
    tie_route: int = 0
    tie_flag: int = 0
    tie_identical: int = 0
    refreshed_gpu: int = 0
    refreshed_oracle: int = 0
    pairs_oracle: int = 0
    mismatches: list = field(default_factory=list)

    def add(self, o: "Report"):
        for f in ("rows", "compared", "tie_route", "tie_flag", "tie_identical", "refreshed_gpu", "refreshed_oracle",
                  "pairs_oracle"):
            setattr(self, f, getattr(self, f) + getattr(o, f))
        self.mismatches += o.mismatches

    @property
    def ties(self) -> int:
        return self.tie_route + self.tie_flag


def _sorted_valid(s_row: np.ndarray, nv: int):
    idx = np.arange(nv)
    order = np.lexsort((idx, -s_row[:nv]))
    return order, s_row[:nv][order]


def compare_head(p: oracle.Params, gh: int, layer: int, anchor: bool, q: np.ndarray, k: np.ndarray,
                 prev_ids, prev_alpha, prev_anchor, gpu_ids, gpu_alpha, gpu_anchor, gpu_flags,
                 max_report: int = 10, gamma_rows=None, prev_flags=None) -> Report:
    """Runs the oracle on one head from the GPU's previous ledger and checks
    the GPU's ledger after the same layer.  gamma_rows: this head's per-row
    guard margins (None: p.gamma).  Flags: bit 0 (refresh) is compared with
    the oracle's flag, bit 1 (the hysteresis mark, p.gamma_h > 0) with the
    oracle's mark after the layer; the oracle starts from the GPU's previous
    marks (prev_flags bit 1)."""
    gpu_mark = (np.asarray(gpu_flags) >> 1) & 1
    gpu_flags = np.asarray(gpu_flags) & 1
    rep = Report(rows=p.nq)
    S = oracle.scores(q, k)
    scale = np.linalg.norm(q.astype(np.float64), axis=1) * np.linalg.norm(k.astype(np.float64), axis=1).max()
    tol = TIE_REL * np.maximum(scale, 1e-30)
    if anchor:
        led = oracle.HeadLedger.empty(p)
    else:
        led = oracle.HeadLedger(prev_ids.astype(np.int32).copy(), prev_alpha.astype(np.float64).copy(),
                                prev_anchor.astype(np.int32).copy())
        if prev_flags is not None:
            led.elevated = ((np.asarray(prev_flags) >> 1) & 1).astype(np.uint8)
    prev_mark = None if anchor else led.elevated.copy()
    flags_o, beta_o, ref_o, pairs_o, st = oracle.head_layer(p, gh, layer, anchor, q, k, led,
                                                             gamma_rows=gamma_rows)
    assert st == 0
    rep.refreshed_oracle = ref_o
    rep.pairs_oracle = pairs_o
    rep.refreshed_gpu = int(gpu_flags.sum())

    def bad(i, what):
        if len(rep.mismatches) < max_report:
            rep.mismatches.append((gh, layer, i, what))
        else:
            rep.mismatches.append(None)

    def valid_full_row(i, nv, srt):
        """A fully routed row whose ranking sits inside the tie margin: check
        that the GPU's choice is one of the correct ones."""
        g = gpu_ids[i]
        nr = min(p.k, nv)
        nm = min(p.m, nv - nr)
        route = [int(x) for x in g[: p.k] if x >= 0]
        near = [int(x) for x in g[p.k:p.k + p.m] if x >= 0]
        rand = [int(x) for x in g[p.k + p.m:p.k + p.m + p.r] if x >= 0]
        glob = [int(x) for x in g[p.k + p.m + p.r:]]
        want = []
        for t, j in enumerate(list(range(p.g_sink)) + list(range(i - p.g_recent + 1, i + 1))):
            if 0 <= j < nv and not (t >= p.g_sink and j < p.g_sink) and j not in route + near:
                want.append(j)
        if glob != want + [-1] * (p.g_sink + p.g_recent - len(want)):
            return "global sentinels"
        allids = route + near + rand + want
        if len(route) != nr or len(near) != nm or len(set(allids)) != len(allids):
            return "wrong counts or repeated ids"
        if any(x < 0 or x >= nv for x in allids):
            return "id outside the valid range"
        if any(S[i, j] < srt[nr - 1] - tol[i] for j in route):
            return "route member below the k-th score"
        if nm and any(S[i, j] < srt[nr + nm - 1] - tol[i] or S[i, j] > srt[nr - 1] + tol[i] for j in near):
            return "near-miss member outside its rank band"
        if len(rand) != min(p.r, nv - nr - nm - len(want)):
            return "wrong random count"
        if abs(float(gpu_alpha[i]) - srt[nr - 1]) > tol[i]:
            return "alpha"
        if int(gpu_anchor[i]) != layer or int(gpu_flags[i]) != 1:
            return "anchor layer / flag"
        return None

    for i in range(p.nq):
        nv = oracle.valid_count(i, p.nk, p.causal)
        if not anchor:
            r_ids = [j for j in prev_ids[i, : p.k] if j >= 0]
            a = min(S[i, j] for j in r_ids) if r_ids else np.inf
            g_i = p.gamma if gamma_rows is None else float(gamma_rows[i])
            if p.gamma_h > 0 and prev_mark[i] and p.gamma_h > g_i:
                g_i = p.gamma_h
            age = layer - int(prev_anchor[i])
            forced = (p.max_age > 0 and age >= p.max_age) or (p.min_reuse > 0 and age <= p.min_reuse)
            if not forced and np.isfinite(beta_o[i]) and abs(a - beta_o[i] - g_i) < tol[i]:
                rep.tie_flag += 1
                if int(gpu_flags[i]):
                    why = valid_full_row(i, nv, _sorted_valid(S[i], nv)[1])
                    if why:
                        bad(i, "tie row refreshed invalidly: " + why)
                elif not np.array_equal(gpu_ids[i], prev_ids[i]):
                    bad(i, "tie row kept its route but changed ids")
                continue
            if int(gpu_flags[i]) != int(flags_o[i]):
                bad(i, f"flag gpu={int(gpu_flags[i])} oracle={int(flags_o[i])} alpha={a} beta={beta_o[i]}")
                continue
            if not flags_o[i]:
                rep.compared += 1
                if int(gpu_mark[i]) != int(led.elevated[i]):
                    bad(i, f"hysteresis mark of a kept row gpu={int(gpu_mark[i])} oracle={int(led.elevated[i])}")
                if not np.array_equal(gpu_ids[i], prev_ids[i]):
                    bad(i, "stable row changed its ids")
                if abs(float(gpu_alpha[i]) - a) > tol[i]:
                    bad(i, f"stable alpha gpu={gpu_alpha[i]} oracle={a}")
                if int(gpu_anchor[i]) != int(prev_anchor[i]):
                    bad(i, "stable row changed its anchor layer")
                continue
        # fully routed row (anchor, or refreshed at relay)
        order, srt = _sorted_valid(S[i], nv)
        nr = min(p.k, nv)
        nm = min(p.m, nv - nr)
        tie = (nr < nv and srt[nr - 1] - srt[nr] < tol[i]) or \
              (nr + nm < nv and nm > 0 and srt[nr + nm - 1] - srt[nr + nm] < tol[i])
        if tie:
            rep.tie_route += 1
            why = valid_full_row(i, nv, srt)
            if why:
                bad(i, "tie row invalid: " + why)
            elif np.array_equal(gpu_ids[i], led.ids[i]):
                rep.tie_identical += 1
            continue
        rep.compared += 1
        g = gpu_ids[i]
        o = led.ids[i]
        if set(g[:nr].tolist()) != set(o[:nr].tolist()) or any(x != -1 for x in g[nr:p.k]):
            bad(i, f"route gpu={g[:p.k].tolist()} oracle={o[:p.k].tolist()}")
            continue
        if set(g[p.k:p.k + nm].tolist()) != set(o[p.k:p.k + nm].tolist()) \
                or any(x != -1 for x in g[p.k + nm:p.k + p.m]):
            bad(i, f"near-miss gpu={g[p.k:p.k + p.m].tolist()} oracle={o[p.k:p.k + p.m].tolist()}")
            continue
        pos = list(range(nr)) + [p.k + t for t in range(nm)]
        for rank, slot in enumerate(pos):
            if abs(S[i, g[slot]] - srt[rank]) > tol[i]:
                bad(i, f"order at slot {slot}: gpu id {g[slot]} score {S[i, g[slot]]} vs {srt[rank]}")
                break
        if not np.array_equal(g[p.k + p.m:], o[p.k + p.m:]):
            bad(i, f"random gpu={g[p.k + p.m:].tolist()} oracle={o[p.k + p.m:].tolist()}")
        if abs(float(gpu_alpha[i]) - srt[nr - 1]) > tol[i]:
            bad(i, f"alpha gpu={gpu_alpha[i]} oracle={srt[nr - 1]}")
        if int(gpu_anchor[i]) != layer:
            bad(i, f"anchor layer gpu={gpu_anchor[i]} expected {layer}")
        if int(gpu_flags[i]) != 1:
            bad(i, "fully routed row without flag")
        if int(gpu_mark[i]) != int(led.elevated[i]):
            bad(i, f"hysteresis mark of a rebuilt row gpu={int(gpu_mark[i])} oracle={int(led.elevated[i])}")
    return rep


def layer_stepped(w, rr, led, layers, heads, device, stream_device="cpu", report_every=None,
                  gamma_rows=None, max_age: int = 0, min_reuse: int = 0, g_sink: int = 0,
                  g_recent: int = 0, gamma_h: float = 0.0, check: bool = True):
    """Runs `layers` layers of workload w through the CUDA ledger `led` and
    compares every layer of the listed heads with the oracle started from
    the GPU's own previous ledger.  gamma_rows ([bh, nq] array) and max_age
    must match what the ledger was given with set_guard.  Returns (total
    report, per-layer list)."""
    import rr_workloads
    st = rr_workloads.LayerStream(w, stream_device)
    p = params_of(w, max_age=max_age, min_reuse=min_reuse, g_sink=g_sink, g_recent=g_recent,
                  gamma_h=gamma_h)
    total = Report()
    per_layer = []
    prev = None
    for l in range(layers):
        qf, kf, qs, ks = st.next()
        qd = qs.to(device).contiguous()
        kd = ks.to(device).contiguous()
        anchor = oracle.is_anchor(l, w.anchor_interval)
        led.layer(qd, kd, l)
        after = led.read(check=check)
        layer_rep = Report()
        qn = qf.cpu().numpy()
        kn = kf.cpu().numpy()
        for h in heads:
            pi = prev["ids"][h].numpy() if prev is not None else None
            pa = prev["alpha"][h].numpy() if prev is not None else None
            pl = prev["anchor_layer"][h].numpy() if prev is not None else None
            pf = prev["flags"][h].numpy() if prev is not None else None
            r = compare_head(p, h, l, anchor, qn[h], kn[h], pi, pa, pl, after["ids"][h].numpy(),
                             after["alpha"][h].numpy(), after["anchor_layer"][h].numpy(),
                             after["flags"][h].numpy(),
                             gamma_rows=None if gamma_rows is None else np.asarray(gamma_rows[h]),
                             prev_flags=pf)
            layer_rep.add(r)
        per_layer.append((l, anchor, layer_rep, after["counters"].clone()))
        total.add(layer_rep)
        prev = after
        del qd, kd
    return total, per_layer
