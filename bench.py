#!/usr/bin/env python
"""Benchmark of the B200 RouteRelay router.

One step = one full routing pass of the workload through every layer: an
anchor (full routing of every row) at layer 0 and every H layers, relay
(rescore -> compact -> refresh of the flagged rows) at the others, on
synthetic drifting chunk representations already resident in HBM.

Default workload: BH = 256 batch x head units, 4096 query and key chunks
per head (256K tokens at 64-token chunks), d = 128 bf16, causal, 32 layers,
anchor every 16, top-32 with 32 near-miss and 16 random sentinels, drift
sigma 0.03.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload NAME] [--attention]

Prints one JSON line (rank 0).  With N > 1 (launched by torchrun) every
rank routes its own BH units (heads are independent: no collective on the
data path) and the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import rr_workloads as W  # noqa: E402

METRIC = "routed rows/s per layer & score-pairs/s; % of tensor/HBM roofline; recall"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    d = dict(PEAKS_FALLBACK)
    d["source"] = "fallback"
    return d


# ---------------------------------------------------------------- clocks ----
class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while running."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.Q, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        srt = sorted(sm)
        loaded = [x for x in srt if x >= 0.5 * srt[-1]] or srt
        return {"sm_mhz": loaded[len(loaded) // 2], "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def smi_id(device) -> str:
    """nvidia-smi id of a torch device (its UUID; CUDA_VISIBLE_DEVICES may
    renumber devices, nvidia-smi does not)."""
    try:
        u = str(torch.cuda.get_device_properties(device).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        idx = torch.device(device).index or 0
        if vis:
            return vis.split(",")[idx]
        return str(idx)


# ------------------------------------------------------------- workload -----
def make_inputs(w, device, seed):
    st = W.LayerStream(w, device, seed=seed)
    qs, ks = [], []
    for _ in range(w.layers):
        _, _, q, k = st.next()
        qs.append(q.contiguous())
        ks.append(k.contiguous())
    del st
    return qs, ks


def code_sha256(path: str) -> str:
    """sha256 of a C/CUDA source's code: comments removed, each line stripped
    of surrounding blanks, blank lines dropped (a comment-only edit keeps it)."""
    import hashlib
    import re
    text = open(path, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = [re.sub(r"//.*$", "", ln).strip() for ln in text.splitlines()]
    return hashlib.sha256("\n".join(ln for ln in lines if ln).encode()).hexdigest()


def profiled_traffic_per_row(kernel_file: str, summary_glob: str):
    """DRAM bytes per routed row from a committed ncu summary, or None when
    the kernel source's code changed since the counters were taken."""
    import glob
    src = os.path.join(ROOT, "cross_layer_route_b200", "csrc", kernel_file)
    if not os.path.exists(src):
        return None
    sha = code_sha256(src)
    for path in glob.glob(os.path.join(ROOT, "profiles", summary_glob)):
        vals = {}
        for line in open(path):
            if ":" in line and line.split(":")[0] in ("traffic_bytes_per_row", "code_sha256"):
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
        if vals.get("code_sha256") == sha and "traffic_bytes_per_row" in vals:
            return float(vals["traffic_bytes_per_row"])
    return None


def uses_tensor_cores(w) -> bool:
    """Which full-routing kernel the library runs for this workload: the
    selection kernel on the tensor cores for bf16 with d in {64, 128} and for
    fp32 with d = 64 (three-way bf16 split), when k + m <= 64 and r <= 32;
    the CUDA-core kernel otherwise."""
    return ((w.dtype == "bf16" and w.d in (64, 128)) or (w.dtype == "f32" and w.d == 64)) \
        and w.k + w.m <= 64 and w.r <= 32


def uses_split(w) -> bool:
    """fp32 on the tensor cores: Qc, Kc split into three bf16 parts each."""
    return uses_tensor_cores(w) and w.dtype == "f32"


def shard_offset(rank: int, w) -> int:
    """Global index of this rank's first BH unit: every rank routes its own
    w.bh units (weak scaling) and keys its random draws by the global index."""
    return rank * w.bh


def max_over_ranks(x: float, world: int, device=None) -> float:
    """The slowest rank's value (step times are compared across ranks)."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def layer_kinds(rows_per_layer: int, anchor_ms: float, n_anchor: int, relay_ms: float, n_relay: int) -> dict:
    """Anchor and relay layers apart (this rank): layers timed, mean time per
    layer, and rows per second through that kind of layer."""
    out = {}
    for name, ms, n in (("anchor", anchor_ms, n_anchor), ("relay", relay_ms, n_relay)):
        if n > 0 and ms > 0:
            out[name] = {"layers": n, "ms_per_layer": round(ms / n, 4),
                         "rows_per_s": rows_per_layer * n / (ms * 1e-3)}
    return out


def sum_over_ranks(xs, world: int, device=None) -> list:
    """Element-wise sum of per-rank counts (refreshed rows, score pairs): the
    one collective of the sharded path, on the host side of the step."""
    if world <= 1:
        return [float(x) for x in xs]
    t = torch.tensor([float(x) for x in xs], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return [float(x) for x in t.tolist()]


def launches_per_step(w, n_anchor: int, n_relay: int, oneshot: bool) -> int:
    """Our kernels launched by one step.  Tensor-core path: anchor = select,
    finish, retry (CUDA cores, usually an empty list), counters (4); one-shot
    relay = select, finish, exact rescoring, retry, counters (5); staged
    relay = rescore, compact, select, finish, retry, counters (6); fp32
    split: one more per routing call (the key split).
    CUDA-core path: anchor = route, counters (2); relay = rescore, compact,
    route, counters (4)."""
    if uses_tensor_cores(w):
        x = 1 if uses_split(w) else 0
        return (4 + x) * n_anchor + ((5 if oneshot else 6) + x) * n_relay
    return 2 * n_anchor + 4 * n_relay


def graph_mode(args, w) -> bool:
    """Whether the timed step is replayed from a CUDA graph: always with
    --graph on, never with --graph off, and by default for the workloads of
    fewer than 2^19 rows per layer, whose layers take microseconds to tens of
    microseconds and would otherwise time the launch path."""
    if args.graph == "auto":
        return w.bh * w.n < (1 << 19)
    return args.graph == "on"


def full_pairs_per_layer(w) -> int:
    if not w.causal:
        return w.bh * w.n * w.n
    return w.bh * w.n * (w.n + 1) // 2


# ---------------------------------------------------------------- ours ------
def run_ours(args, w, rank, world, device):
    import cross_layer_route_b200 as rr

    torch.cuda.set_device(device)
    cfg = rr.Config(bh=w.bh, nq=w.n, nk=w.n, d=w.d, k=w.k, m_near=w.m, r_rand=w.r, dtype=w.dtype,
                    anchor_interval=w.anchor_interval, causal=w.causal, gamma=w.gamma, seed=w.seed,
                    bh_offset=shard_offset(rank, w))
    qs, ks = make_inputs(w, device, seed=w.seed * 1009 + rank)
    led = rr.RouteLedger(cfg, device)
    stream = torch.cuda.current_stream(device)
    L = w.layers
    anchors = [l for l in range(L) if led.is_anchor(l)]
    relays = [l for l in range(L) if not led.is_anchor(l)]

    # On the tensor-core path a relay layer is one C-ABI call (rr_relay_layer:
    # every row routed, the relay test taken from the kept scores); the
    # three-stage form (rescore -> compact -> refresh) is timed with --relay
    # staged, and is what the CUDA-core path runs.
    oneshot = uses_tensor_cores(w) and args.relay == "oneshot"

    # events on the launching stream: each layer's span, and in the staged
    # form the boundaries between its three stages
    def make_events(n):
        return [torch.cuda.Event(enable_timing=True) for _ in range(n)]

    def step(ev=None):
        for l in range(L):
            if ev is not None:
                ev["start"][l].record(stream)
            if led.is_anchor(l):
                led.full_route(qs[l], ks[l], l)
            elif oneshot:
                led.relay_layer(qs[l], ks[l], l)
            else:
                led.relay_rescore(qs[l], ks[l], l)
                if ev is not None:
                    ev["compact"][l].record(stream)
                led.relay_compact(l)
                if ev is not None:
                    ev["refresh"][l].record(stream)
                led.relay_refresh(qs[l], ks[l], l)
            if ev is not None:
                ev["end"][l].record(stream)

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(device)

    # CUDA-graph mode: one whole step (every layer's launches) captured once
    # and replayed K times; the per-layer split then comes from one eager
    # step with events after the timed region
    use_graph = graph_mode(args, w)
    for _ in range(args.warmup):
        step()
    barrier()
    graph = None
    if use_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        graph.replay()
        barrier()
    c0 = led.read()["counters"].clone()
    K = args.steps
    K_ev = 1 if use_graph else K
    evs = [{n: make_events(L) for n in ("start", "compact", "refresh", "end")} for _ in range(K_ev)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(smi_id(device) if args.smi_index is None else args.smi_index) as clk:
        barrier()
        t_start.record(stream)
        for s in range(K):
            if graph is not None:
                graph.replay()
            else:
                step(evs[s])
        t_end.record(stream)
        barrier()
    ms_total = t_start.elapsed_time(t_end)
    c1 = led.read()["counters"].clone()
    if graph is not None:
        step(evs[0])
        barrier()
        del graph

    anchor_layer_ms = relay_layer_ms = rescore_ms = compact_ms = refresh_ms = 0.0
    for s in range(K_ev):
        for l in range(L):
            span = evs[s]["start"][l].elapsed_time(evs[s]["end"][l])
            if l in anchors:
                anchor_layer_ms += span
            else:
                relay_layer_ms += span
                if not oneshot:
                    rescore_ms += evs[s]["start"][l].elapsed_time(evs[s]["compact"][l])
                    compact_ms += evs[s]["compact"][l].elapsed_time(evs[s]["refresh"][l])
                    refresh_ms += evs[s]["refresh"][l].elapsed_time(evs[s]["end"][l])
    n_rescore = 0 if oneshot else K_ev * len(relays)
    # the full-routing stage: anchor layers, and the relay layers' routing
    # (one-shot: the whole relay call; staged: the refresh launches)
    route_ms = anchor_layer_ms + (relay_layer_ms if oneshot else refresh_ms)
    n_route = K_ev * L

    ms_step = max_over_ranks(ms_total / K, world, device)

    rows_per_step = w.bh * w.n * L
    d_cnt = (c1 - c0).tolist()
    pairs_per_step = d_cnt[rr.CNT_PAIRS_TOTAL] / K
    full_pairs_per_step = d_cnt[rr.CNT_FULL_PAIRS_TOTAL] / K
    refreshed_per_step = d_cnt[rr.CNT_ROWS_TOTAL] / K
    # all ranks' counts (every rank takes this step, in the same place)
    pairs_all, refreshed_all, retry_all = sum_over_ranks(
        [pairs_per_step, refreshed_per_step, d_cnt[rr.CNT_RETRY_TOTAL] / K], world, device)
    relay_rows = w.bh * w.n * len(relays) * world
    rho = (refreshed_all - w.bh * w.n * len(anchors) * world) / relay_rows if relay_rows else 0.0

    peaks = load_peaks()
    esz = 2 if w.dtype == "bf16" else 4
    # dominant kernel: full routing (anchor + refresh).  Algorithmic work =
    # one multiply-add per (row, valid key, dim) -> 2*d flops per score pair.
    route_flops = 2.0 * w.d * full_pairs_per_step * K_ev
    route_tflops = route_flops / (route_ms * 1e-3) / 1e12
    if uses_split(w):
        # six bf16 products per fp32 product: the arithmetic's own peak is the
        # bf16 dense peak / 6
        peak = float(peaks["bf16_tflops_sustained"]) / 6.0
        roofline = {"kernel": "full routing, fp32 split in three bf16 parts: split_keys_kernel + "
                              "route_select_kernel + route_finish_kernel (+ exact rescoring at relay layers)",
                    "bound": "tensor",
                    "peak_source": f"{peaks['source']} bf16 dense, sustained, / 6 (six bf16 MMAs per fp32 product)"}
    elif uses_tensor_cores(w):
        peak = float(peaks["bf16_tflops_sustained"])
        what = ("route_select_kernel (tcgen05, query tile in TMEM, two-pass selection) + route_finish_kernel"
                " + exact fallbacks; anchor and relay layers (relay test taken from the kept scores)"
                if oneshot else
                "route_select_kernel + route_finish_kernel + exact fallback; anchor layers and refresh launches")
        roofline = {"kernel": "full routing: " + what, "bound": "tensor",
                    "peak_source": f"{peaks['source']} bf16 dense, sustained (timed inside a long step)"}
    else:
        peak = 148 * 128 * 2 * float(peaks.get("sm_max_mhz", 1965.0)) * 1e6 / 1e12
        roofline = {"kernel": "route_rows (CUDA cores; anchor + refresh)", "bound": "alu",
                    "peak_source": "148 SMs x 128 fp32 lanes x 2 flop x max SM clock"}
    traffic = None
    if uses_tensor_cores(w) and not uses_split(w):
        # DRAM bytes per routed row of the two kernels of a routing call, from
        # the committed ncu summaries of the 64-head case (traffic grows with
        # the rows routed), while their source is unchanged
        parts = [profiled_traffic_per_row("rr_select_tc.cu", g)
                 for g in ("route_select_kernel__*.md", "route_finish_kernel__*.md")]
        per_row = sum(parts) if all(x is not None for x in parts) else None
        if per_row is not None and n_route:
            rows_routed = (w.bh * w.n * L) if oneshot else refreshed_per_step
            traffic = round(per_row * rows_routed * K_ev / n_route)   # bytes per launch
    roofline.update({"achieved": round(route_tflops, 3), "peak": round(peak, 1), "unit": "TFLOP/s",
                     "frac": round(route_tflops / peak, 4), "traffic": traffic,
                     "avg_launch_ms": round(route_ms / max(n_route, 1), 4),
                     "launches": n_route})
    kernels = {}
    if not oneshot and rescore_ms > 0:
        # staged relay: rescoring (bytes it must move per row: q (d*e) + its
        # head's keys once (N*d*e/N) + ids (4c) + alpha/flag writes (5))
        rescore_bytes = w.bh * w.n * (2 * w.d * esz + 4 * w.c + 5) * n_rescore
        rescore_gbs = rescore_bytes / (rescore_ms * 1e-3) / 1e9
        rescore = {"bound": "hbm", "achieved_gbs": round(rescore_gbs, 1), "peak_gbs": peaks["hbm_gbs"],
                   "frac": round(rescore_gbs / peaks["hbm_gbs"], 4),
                   "avg_launch_ms": round(rescore_ms / max(n_rescore, 1), 4)}
        if uses_tensor_cores(w) and not uses_split(w):
            # dense tiles: every valid pair of the row block is scored (2*d flops per pair)
            dense_tflops = 2.0 * w.d * full_pairs_per_layer(w) * n_rescore / (rescore_ms * 1e-3) / 1e12
            rescore = {"kernel": "relay_rescore_tc_kernel (tcgen05 dense tiles)", "bound": "tensor",
                       "achieved": round(dense_tflops, 2), "unit": "TFLOP/s (dense tile work)",
                       "peak": float(peaks["bf16_tflops_sustained"]),
                       "frac": round(dense_tflops / float(peaks["bf16_tflops_sustained"]), 4),
                       "hbm_gbs": round(rescore_gbs, 1),
                       "avg_launch_ms": round(rescore_ms / max(n_rescore, 1), 4)}
        kernels["rescore"] = rescore
        kernels["compact"] = {"avg_launch_ms": round(compact_ms / max(n_rescore, 1), 4)}
        kernels["refresh"] = {"avg_launch_ms": round(refresh_ms / max(n_rescore, 1), 4)}

    result = {
        "metric": METRIC, "value": rows_per_step * world / (ms_step * 1e-3), "unit": "rows/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic",
        "config": workload_config(w, world),
        "score_pairs_per_s": pairs_all / (ms_step * 1e-3),
        "pair_fraction": pairs_all / (full_pairs_per_layer(w) * L * world),
        "rho_relay": rho,
        "layer_kinds": layer_kinds(w.bh * w.n, anchor_layer_ms, K_ev * len(anchors), relay_layer_ms,
                                   K_ev * len(relays)),
        "timing": ("CUDA graph of the whole step, replayed K times; layer_kinds and roofline from one "
                   "eager step with per-layer events after the timed region" if use_graph else
                   "eager launches; per-layer events on the launching stream"),
        "retry_rows_per_step": retry_all,
        "relay": "one-shot (rr_relay_layer)" if oneshot else "staged (rescore, compact, refresh)",
        "roofline": roofline,
        "kernels": kernels,
        "gpu_launches": K * launches_per_step(w, len(anchors), len(relays), oneshot),
        "clocks": clk.summary(),
        "peaks_source": peaks["source"],
    }
    return result, (led, qs, ks, cfg)


def measure_e2e(args, w, state, device):
    """Same metric through the public API with the inputs in pinned host
    memory: each step copies every layer's Qc, Kc host->device (copy stream,
    double-buffered) and reads the ledger back device->host at its end."""
    import cross_layer_route_b200 as rr
    led, qs, ks, cfg = state
    L = w.layers
    hq = [q.cpu().pin_memory() for q in qs]
    hk = [k.cpu().pin_memory() for k in ks]
    bq = [torch.empty_like(qs[0]) for _ in range(2)]
    bk = [torch.empty_like(ks[0]) for _ in range(2)]
    comp = torch.cuda.current_stream(device)
    copy = torch.cuda.Stream(device)
    out_ids = torch.empty((cfg.bh, cfg.nq, cfg.c), dtype=torch.int32, pin_memory=True)
    out_alpha = torch.empty((cfg.bh, cfg.nq), dtype=torch.float32, pin_memory=True)
    out_cnt = torch.empty((rr.NUM_COUNTERS,), dtype=torch.int64, pin_memory=True)
    view = rr.rr_ledger_view(out_ids.data_ptr(), out_alpha.data_ptr(), None, None, out_cnt.data_ptr())
    done = [torch.cuda.Event() for _ in range(2)]
    ready = [torch.cuda.Event() for _ in range(2)]

    def step():
        for l in range(L):
            b = l & 1
            copy.wait_event(done[b])
            with torch.cuda.stream(copy):
                bq[b].copy_(hq[l], non_blocking=True)
                bk[b].copy_(hk[l], non_blocking=True)
                ready[b].record(copy)
            comp.wait_event(ready[b])
            led.layer(bq[b], bk[b], l, stream=comp)
            done[b].record(comp)
        rr.rr_ledger_read(led.handle, view, comp.cuda_stream)

    for b in range(2):
        done[b].record(comp)
    step()
    torch.cuda.synchronize(device)
    K = max(1, min(args.steps, 3))
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(comp)
    for _ in range(K):
        step()
    t1.record(comp)
    torch.cuda.synchronize(device)
    ms = t0.elapsed_time(t1) / K
    h2d = sum(q.numel() * q.element_size() + k.numel() * k.element_size() for q, k in zip(qs, ks))
    d2h = out_ids.numel() * 4 + out_alpha.numel() * 4 + out_cnt.numel() * 8
    return {"value": w.bh * w.n * L / (ms * 1e-3), "unit": "rows/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms, "steps": K}


def measure_recall(w, state, device):
    """Recall of the relayed routes against exact per-layer top-k (a second
    ledger that fully routes every layer), pooled over rows, mean over
    layers."""
    import cross_layer_route_b200 as rr
    led, qs, ks, cfg = state
    exact_cfg = rr.Config(**{**cfg.__dict__, "anchor_interval": 1})
    ex = rr.RouteLedger(exact_cfg, device)
    dv, ev = led.device_view(), ex.device_view()
    rec = []
    for l in range(w.layers):
        led.layer(qs[l], ks[l], l)
        ex.layer(qs[l], ks[l], l)
        hits = tot = 0
        for h0 in range(0, w.bh, 16):
            used = dv["ids"][h0:h0 + 16, :, : w.k]
            exact = ev["ids"][h0:h0 + 16, :, : w.k]
            m = (used[..., :, None] == exact[..., None, :]) & (exact[..., None, :] >= 0)
            hits += int(m.any(-2).sum())
            tot += int((exact >= 0).sum())
        rec.append(hits / tot)
    del ex
    return sum(rec) / len(rec), min(rec)


def visible_pairs(route: torch.Tensor, nk_chunks: int, chunk: int, causal: bool) -> int:
    """(query token, key token) pairs the attention over `route` ([bh,
    nq_chunks, width] key-chunk ids) evaluates: a usable off-diagonal chunk
    gives chunk^2 pairs, the causal diagonal chunk chunk (chunk + 1) / 2;
    -1, out-of-range ids and (causal) ids past the query chunk give none."""
    ids = route.long()
    i_idx = torch.arange(ids.shape[1])[None, :, None]
    usable = (ids >= 0) & (ids < nk_chunks)
    if causal:
        full = usable & (ids < i_idx)
        diag = usable & (ids == i_idx)
    else:
        full = usable
        diag = torch.zeros_like(usable)
    return int(full.sum()) * chunk * chunk + int(diag.sum()) * chunk * (chunk + 1) // 2


def measure_attention(args, w, state, device):
    """The consumer of the routes (opt-in, outside the timed step): sparse
    attention over the ledger's current routes for the first heads of the
    ledger, at token level (chunks of W.ATTN_C5.chunk tokens, head dim
    W.ATTN_C5.dh, seeded N(0, 1) bf16 q, k, v).  Useful work = 4 * dh flops
    per visible (query token, key token) pair: q.k and p.v."""
    import cross_layer_route_b200 as rr
    led, qs, ks, cfg = state
    a = W.ATTN_C5
    heads = min(a.bh, w.bh)
    q, k, v = (x.to(device) for x in W.attention_tokens(heads, w.n * a.chunk, a.dh, seed=a.seed))
    route = led.device_view()["ids"][:heads]               # [heads, n, c], first k ids read
    out = torch.empty((heads, w.n * a.chunk, a.dh), dtype=torch.float32, device=device)
    pairs = visible_pairs(route[:, :, :w.k].cpu(), w.n, a.chunk, w.causal)
    stream = torch.cuda.current_stream(device)

    def call():
        rr.sparse_attention(q, k, v, route, a.chunk, causal=w.causal, width=w.k, out=out, stream=stream)

    for _ in range(3):
        call()
    torch.cuda.synchronize(device)
    n = 10
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(n):
        call()
    t1.record(stream)
    torch.cuda.synchronize(device)
    ms = t0.elapsed_time(t1) / n
    peaks = load_peaks()
    tflops = 4.0 * a.dh * pairs / (ms * 1e-3) / 1e12
    return {"kernel": "sparse_attention_kernel (bf16 mma.sync, online softmax)",
            "workload": f"attn_bh{heads}_n{w.n}_c{a.chunk}_dh{a.dh}_bf16" + ("_causal" if w.causal else ""),
            "routes": "the ledger's routes after the last layer", "bound": "tensor",
            "avg_launch_ms": round(ms, 4), "tokens_per_s": heads * w.n * a.chunk / (ms * 1e-3),
            "achieved": round(tflops, 2), "unit": "TFLOP/s", "peak": float(peaks["bf16_tflops"]),
            "frac": round(tflops / float(peaks["bf16_tflops"]), 4),
            "peak_source": f"{peaks['source']} bf16 dense, burst (timed alone)",
            "visible_pairs": pairs, "launches": n}


RECALL_KIND = ("GPU vs GPU: the relayed ledger's routes against a second GPU ledger that fully routes "
               "every layer (anchor interval 1), all rows, mean over layers; full routing itself is "
               "checked against the oracle (parity tests; oracle_sample on sampled heads)")

SMALL_WORKLOADS = (W.PR1, W.C2, W.C3, W.C4)


def per_workload(args, device, oracle_leg: bool) -> dict:
    """The four smaller workloads, one GPU each in turn, each timed the same
    way as the headline one (a CUDA graph of the whole step for the
    CUDA-core path), with recall and, when the CPU leg runs, the oracle
    sample."""
    keys = ("value", "unit", "ms_per_step", "steps", "score_pairs_per_s", "pair_fraction", "rho_relay",
            "layer_kinds", "retry_rows_per_step", "roofline", "gpu_launches", "timing", "dtype", "config",
            "clocks")
    out = {}
    for w in SMALL_WORKLOADS:
        sub = argparse.Namespace(**{**vars(args), "steps": max(args.steps, 20), "relay": "oneshot"})
        res, state = run_ours(sub, w, 0, 1, device)
        entry = {k: res[k] for k in keys}
        r_mean, r_min = measure_recall(w, state, device)
        entry.update({"recall": r_mean, "recall_min_layer": r_min, "recall_kind": RECALL_KIND})
        if oracle_leg:
            entry["cpu_baseline"] = cpu_baseline(w, state[1], state[2])
            entry["oracle_sample"] = oracle_sample(w, state)
        out[w.name] = entry
        del state
        torch.cuda.empty_cache()
    return out


# ------------------------------------------------------- CPU baseline ------
def cpu_baseline(w, qs, ks, threads=None, layers=2):
    """The oracle as it stands, on a bounded sample: `threads` heads (one per
    thread) through `layers` layers (anchor then relay)."""
    import numpy as np

    import oracle
    ncpu = os.cpu_count() or 1
    T = max(1, min(threads or ncpu, 16, w.bh))
    p = oracle.Params(nq=w.n, nk=w.n, d=w.d, k=w.k, m=w.m, r=w.r, causal=w.causal, gamma=w.gamma,
                      seed=w.seed)
    rt = oracle.Router(p, bh=T, anchor_interval=w.anchor_interval, threads=T)
    xs = [(qs[l][:T].float().cpu().numpy(), ks[l][:T].float().cpu().numpy()) for l in range(layers)]
    t0 = time.perf_counter()
    for l in range(layers):
        rt.step(l, xs[l][0], xs[l][1], recall=False)
    dt = time.perf_counter() - t0
    rows = T * w.n * layers
    return {"value": rows / dt, "unit": "rows/s", "cores": T, "kind": "oracle",
            "sample": f"{T} heads x {layers} layers (anchor, relay) of {w.name}, one head per thread, "
                      f"{dt:.1f} s wall on {ncpu} host cores",
            "cpu_model": cpu_model()}


def oracle_sample(w, state, heads=None, layers=(0, 1)):
    """Tie-margin and mismatch counts at the bench's own size: after the
    timed region, layers 0 (anchor) and 1 (relay) go through the GPU ledger
    once more, and on the sampled heads each is compared with the oracle
    started from the GPU's previous ledger (the parity tests' comparison:
    ids, order, alpha, flags and anchor layers row by row; rows whose
    deciding score gap is below 1e-5 x scale are counted as ties and only
    checked for validity).  Also the oracle's recall of the relayed routes
    at the relay layer against its own exact top-k on those heads."""
    import numpy as np

    import oracle
    tests_dir = os.path.join(ROOT, "tests")
    if tests_dir not in sys.path:
        sys.path.insert(0, tests_dir)
    import rr_parity

    led, qs, ks, cfg = state
    heads = sorted({0, w.bh - 1}) if heads is None else list(heads)
    p = rr_parity.params_of(w)
    rep = rr_parity.Report()
    hits = tot = 0
    prev = None
    t0 = time.perf_counter()
    for l in layers:
        led.layer(qs[l], ks[l], l)
        dv = led.device_view()
        after = {n: dv[n][heads].cpu().numpy() for n in ("ids", "alpha", "anchor_layer", "flags")}
        anchor = oracle.is_anchor(l, w.anchor_interval)
        for j, h in enumerate(heads):
            q = qs[l][h].float().cpu().numpy()
            k = ks[l][h].float().cpu().numpy()
            pv = (lambda n: None) if prev is None else (lambda n: prev[n][j])
            rep.add(rr_parity.compare_head(p, cfg.bh_offset + h, l, anchor, q, k, pv("ids"), pv("alpha"),
                                           pv("anchor_layer"), after["ids"][j], after["alpha"][j],
                                           after["anchor_layer"][j], after["flags"][j],
                                           prev_flags=pv("flags")))
            if not anchor:
                exact = oracle.exact_topk(p, q, k)
                used = after["ids"][j][:, :w.k]
                valid = exact >= 0
                hits += int(((used[:, :, None] == exact[:, None, :]).any(1) & valid).sum())
                tot += int(valid.sum())
        prev = after
    dt = time.perf_counter() - t0
    mism = [m for m in rep.mismatches if m is not None]
    return {"heads": heads, "layers": list(layers), "rows": rep.rows, "compared": rep.compared,
            "ties": rep.ties, "tie_route": rep.tie_route, "tie_flag": rep.tie_flag,
            "tie_identical": rep.tie_identical, "mismatches": len(rep.mismatches),
            "first_mismatches": [list(map(str, m)) for m in mism[:3]],
            "oracle_recall_relay_layer": (hits / tot) if tot else None,
            "seconds": round(dt, 1)}


def cpu_model() -> str:
    """The host CPU's model name (Linux /proc/cpuinfo), or "unknown"."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def workload_config(w, world: int) -> dict:
    """The bench line's config block (both arms)."""
    esz = 2 if w.dtype == "bf16" else 4
    return {"workload": w.name, "bh_per_gpu": w.bh, "n_chunks": w.n, "d": w.d,
            "layers": w.layers, "anchor_interval": w.anchor_interval, "k": w.k, "near_miss": w.m,
            "random": w.r, "causal": w.causal, "drift_sigma": w.sigma,
            "l2": f"no flush: inputs {2 * w.layers * w.bh * w.n * w.d * esz / 2**30:.1f} GiB per step exceed L2",
            "parallelism": f"bh-sharded x{world}, no collective"}


def run_reference(args, w):
    """The oracle timed as a benchmark arm on this workload (rank 0 only)."""
    import numpy as np
    st = W.LayerStream(w.with_(bh=min(w.bh, 16)), "cpu")
    qs, ks = [], []
    for _ in range(2):
        _, _, q, k = st.next()
        qs.append(q)
        ks.append(k)
    ncpu = os.cpu_count() or 1
    T = max(1, min(ncpu, 16, w.bh))
    for _ in range(args.warmup):
        cpu_baseline(w, qs, ks, threads=T, layers=1)
    vals = []
    t_all = time.perf_counter()
    for _ in range(args.steps):
        vals.append(cpu_baseline(w, qs, ks, threads=T, layers=2))
    ms_step = (time.perf_counter() - t_all) / args.steps * 1e3
    v = sum(x["value"] for x in vals) / len(vals)
    cb = dict(vals[-1])
    cb["value"] = v
    return {"metric": METRIC, "value": v, "unit": "rows/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": workload_config(w, args.gpus),
            "cpu_baseline": cb,
            "e2e": {"value": v, "unit": "rows/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def free_port() -> int:
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def launcher_command(argv, n: int, port: int) -> list:
    """The command that runs this script as n ranks on one node (one rank
    per GPU), with the same arguments."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
            "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__)] + list(argv)


def resolve_world(args, env=None, device_count=None):
    """How this process runs --gpus N: ("run", world) to go on in this process
    as one of `world` ranks, ("launch", n) to start n ranks through the
    launcher, or ("fail", message).  A launcher's WORLD_SIZE must equal
    --gpus; without a launcher, --gpus N > 1 starts N ranks (never a silent
    single rank), and needs N visible GPUs.  The reference arm's work is rank
    0's alone, so it runs in place."""
    env = os.environ if env is None else env
    if "WORLD_SIZE" in env:
        world = int(env["WORLD_SIZE"])
        if world != args.gpus:
            return ("fail", f"--gpus {args.gpus} but the launcher started {world} ranks")
        return ("run", world)
    if args.gpus <= 1 or args.impl == "reference":
        return ("run", 1)
    n_dev = torch.cuda.device_count() if device_count is None else device_count
    if n_dev < args.gpus:
        return ("fail", f"--gpus {args.gpus} needs {args.gpus} visible GPUs, found {n_dev}")
    return ("launch", args.gpus)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=W.C5.name, choices=sorted(W.BY_NAME))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-recall", action="store_true")
    ap.add_argument("--attention", action="store_true",
                    help="also time the sparse attention over the ledger's routes (not part of the step)")
    ap.add_argument("--relay", default="oneshot", choices=["oneshot", "staged"],
                    help="tensor-core path: time relay layers as one rr_relay_layer call or as its three stages")
    ap.add_argument("--graph", default="auto", choices=["auto", "on", "off"],
                    help="replay the timed step from a CUDA graph (auto: for the CUDA-core workloads)")
    ap.add_argument("--per-workload", default="auto", choices=["auto", "on", "off"],
                    help="also measure the four smaller workloads (auto: on for the default run on one GPU)")
    ap.add_argument("--no-oracle-sample", action="store_true",
                    help="skip the tie/mismatch count against the oracle on sampled heads")
    ap.add_argument("--smi-index", type=int, default=None)
    ap.add_argument("--low-drift", action="store_true",
                    help="the supplementary low-drift variant of the workload (sigma / sqrt(d) per element)")
    ap.add_argument("--bh", type=int, default=None, help="override BH (profiling a smaller case)")
    ap.add_argument("--layers", type=int, default=None, help="override the layer count")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    w = W.BY_NAME[args.workload]
    if args.low_drift:
        w = W.low_drift(w)
    if args.bh is not None:
        w = w.with_(bh=args.bh, name=f"{w.name}@bh{args.bh}")
    if args.layers is not None:
        w = w.with_(layers=args.layers, name=f"{w.name}@L{args.layers}")

    if args.gpus < 1:
        ap.error("--gpus must be at least 1")
    how, val = resolve_world(args)
    if how == "fail":
        print(f"bench.py: {val}", file=sys.stderr, flush=True)
        return 2
    if how == "launch":
        return subprocess.call(launcher_command(sys.argv[1:], val, free_port()))
    world = val
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, w)), flush=True)
        return 0

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    result, state = run_ours(args, w, rank, world, device)
    if not args.no_recall:
        r_mean, r_min = measure_recall(w, state, device)
        result["recall"] = r_mean
        result["recall_min_layer"] = r_min
        result["recall_kind"] = RECALL_KIND
    if args.attention and rank == 0:
        result["kernels"]["attention"] = measure_attention(args, w, state, device)
    if not args.no_e2e:
        e2e = measure_e2e(args, w, state, device)
        if world > 1:
            e2e["ms_per_step"] = max_over_ranks(e2e["ms_per_step"], world, device)
            e2e["value"] = w.bh * w.n * w.layers * world / (e2e["ms_per_step"] * 1e-3)
        result["e2e"] = e2e
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(w, state[1], state[2])
        one = cpu_baseline(w, state[1], state[2], threads=1)
        result["cpu_baseline"]["single_thread"] = {"value": one["value"], "unit": one["unit"],
                                                   "sample": one["sample"]}
        if not args.no_oracle_sample:
            result["oracle_sample"] = oracle_sample(w, state)
    del state
    if world == 1 and (args.per_workload == "on" or (
            args.per_workload == "auto" and args.workload == W.C5.name and args.bh is None
            and args.layers is None and not args.low_drift)):
        torch.cuda.empty_cache()
        result["per_workload"] = per_workload(args, device, oracle_leg=not args.no_cpu_baseline
                                              and not args.no_oracle_sample)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
