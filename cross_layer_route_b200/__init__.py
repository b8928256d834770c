"""B200-native RouteRelay router: Python binding of librr.so (include/rr.h).

Method: "RouteRelay: Event-Triggered Cross-Layer Route Reuse for Efficient
Dynamic Sparse Attention" (arXiv 2609.07306).  Anchor layers fully route
every query chunk (S = Qc Kc^T, top-k, §2.1 Eq. 1-2); intermediate layers
rescore each row's ledger candidates, test alpha > beta + gamma (§3.2 Eq.
5-8) and fully re-route only the rows that fail (§4.1-4.2).  The routes feed
a sparse attention over their chunks' tokens (§2.1, Eq. 3; sparse_attention,
RouteLedger.sparse_attention).

This module only marshals arguments: every step of the routing path runs in
the CUDA kernels of librr.so.  There is no CPU fallback; importing it without
the built library raises.  PyTorch supplies device memory and streams.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librr.so")

RR_OK, RR_EINVAL, RR_ESTATE, RR_ENOMEM, RR_ECUDA, RR_EDEVICE, RR_ECAPACITY = range(7)
RR_F32, RR_BF16 = 0, 1
CNT_ROWS, CNT_PAIRS, CNT_ERROR, CNT_ROWS_TOTAL, CNT_PAIRS_TOTAL, CNT_LAYERS, CNT_LAST_LAYER, \
    CNT_DRAW_CAP, CNT_FULL_PAIRS, CNT_FULL_PAIRS_TOTAL, CNT_RETRY_TOTAL = range(11)
NUM_COUNTERS = 16


class rr_config(ctypes.Structure):
    _fields_ = [("bh", ctypes.c_int32), ("nq", ctypes.c_int32), ("nk", ctypes.c_int32),
                ("d", ctypes.c_int32), ("dtype", ctypes.c_int32), ("k", ctypes.c_int32),
                ("m_near", ctypes.c_int32), ("r_rand", ctypes.c_int32),
                ("anchor_interval", ctypes.c_int32), ("causal", ctypes.c_int32),
                ("gamma", ctypes.c_float), ("bh_offset", ctypes.c_int32), ("seed", ctypes.c_uint64),
                ("g_sink", ctypes.c_int32), ("g_recent", ctypes.c_int32)]


class rr_ledger_view(ctypes.Structure):
    _fields_ = [("ids", ctypes.c_void_p), ("alpha", ctypes.c_void_p),
                ("anchor_layer", ctypes.c_void_p), ("flags", ctypes.c_void_p),
                ("counters", ctypes.c_void_p)]


class rr_attn_config(ctypes.Structure):
    _fields_ = [("bh", ctypes.c_int32), ("nq_tokens", ctypes.c_int32), ("nk_tokens", ctypes.c_int32),
                ("dh", ctypes.c_int32), ("chunk", ctypes.c_int32), ("width", ctypes.c_int32),
                ("route_stride", ctypes.c_int32), ("causal", ctypes.c_int32), ("scale", ctypes.c_float)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"librr.so is not built ({LIB_PATH}); run python cross_layer_route_b200/build.py")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    lib.rr_ledger_workspace_bytes.argtypes = [ctypes.POINTER(rr_config)]
    lib.rr_ledger_workspace_bytes.restype = ctypes.c_size_t
    lib.rr_ledger_create.argtypes = [ctypes.POINTER(rr_config), P, ctypes.c_size_t, ctypes.POINTER(P)]
    lib.rr_ledger_create.restype = ctypes.c_int
    lib.rr_ledger_destroy.argtypes = [P]
    lib.rr_ledger_destroy.restype = ctypes.c_int
    for name in ("rr_full_route", "rr_relay_layer", "rr_relay_rescore", "rr_relay_refresh"):
        f = getattr(lib, name)
        f.argtypes = [P, P, P, ctypes.c_int32, P]
        f.restype = ctypes.c_int
    lib.rr_relay_compact.argtypes = [P, ctypes.c_int32, P]
    lib.rr_relay_compact.restype = ctypes.c_int
    lib.rr_ledger_read.argtypes = [P, ctypes.POINTER(rr_ledger_view), P]
    lib.rr_ledger_read.restype = ctypes.c_int
    lib.rr_ledger_device_view.argtypes = [P, ctypes.POINTER(rr_ledger_view)]
    lib.rr_ledger_device_view.restype = ctypes.c_int
    lib.rr_ledger_set_guard.argtypes = [P, P, ctypes.c_int32]
    lib.rr_ledger_set_guard.restype = ctypes.c_int
    lib.rr_ledger_set_hysteresis.argtypes = [P, ctypes.c_int32]
    lib.rr_ledger_set_hysteresis.restype = ctypes.c_int
    lib.rr_ledger_set_wait_budget.argtypes = [P, ctypes.c_int64]
    lib.rr_ledger_set_wait_budget.restype = ctypes.c_int
    lib.rr_ledger_set_hysteresis_margin.argtypes = [P, ctypes.c_float]
    lib.rr_ledger_set_hysteresis_margin.restype = ctypes.c_int
    lib.rr_route_layer_static.argtypes = [ctypes.POINTER(rr_config), P, P, ctypes.c_int32, P, P, P, P, P, P]
    lib.rr_route_layer_static.restype = ctypes.c_int
    lib.rr_sparse_attention.argtypes = [ctypes.POINTER(rr_attn_config), P, P, P, P, P, P]
    lib.rr_sparse_attention.restype = ctypes.c_int
    lib.rr_status_string.argtypes = [ctypes.c_int]
    lib.rr_status_string.restype = ctypes.c_char_p
    return lib


_lib = _load()


class RRError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {rr_status_string(status)}")


def _check(status: int, what: str):
    if status != RR_OK:
        raise RRError(status, what)


# ---- the C ABI, name for name ---------------------------------------------
def rr_status_string(status: int) -> str:
    return _lib.rr_status_string(status).decode()


def rr_ledger_workspace_bytes(cfg: rr_config) -> int:
    return int(_lib.rr_ledger_workspace_bytes(ctypes.byref(cfg)))


def rr_ledger_create(cfg: rr_config, d_workspace: int, nbytes: int) -> ctypes.c_void_p:
    out = ctypes.c_void_p()
    _check(_lib.rr_ledger_create(ctypes.byref(cfg), ctypes.c_void_p(d_workspace), nbytes,
                                 ctypes.byref(out)), "rr_ledger_create")
    return out


def rr_ledger_destroy(handle) -> None:
    _check(_lib.rr_ledger_destroy(handle), "rr_ledger_destroy")


def rr_full_route(handle, d_qc: int, d_kc: int, layer: int, stream: int) -> None:
    _check(_lib.rr_full_route(handle, ctypes.c_void_p(d_qc), ctypes.c_void_p(d_kc), layer,
                              ctypes.c_void_p(stream)), "rr_full_route")


def rr_relay_layer(handle, d_qc: int, d_kc: int, layer: int, stream: int) -> None:
    _check(_lib.rr_relay_layer(handle, ctypes.c_void_p(d_qc), ctypes.c_void_p(d_kc), layer,
                               ctypes.c_void_p(stream)), "rr_relay_layer")


def rr_relay_rescore(handle, d_qc: int, d_kc: int, layer: int, stream: int) -> None:
    _check(_lib.rr_relay_rescore(handle, ctypes.c_void_p(d_qc), ctypes.c_void_p(d_kc), layer,
                                 ctypes.c_void_p(stream)), "rr_relay_rescore")


def rr_relay_compact(handle, layer: int, stream: int) -> None:
    _check(_lib.rr_relay_compact(handle, layer, ctypes.c_void_p(stream)), "rr_relay_compact")


def rr_relay_refresh(handle, d_qc: int, d_kc: int, layer: int, stream: int) -> None:
    _check(_lib.rr_relay_refresh(handle, ctypes.c_void_p(d_qc), ctypes.c_void_p(d_kc), layer,
                                 ctypes.c_void_p(stream)), "rr_relay_refresh")


def rr_ledger_read(handle, view: rr_ledger_view, stream: int) -> None:
    _check(_lib.rr_ledger_read(handle, ctypes.byref(view), ctypes.c_void_p(stream)), "rr_ledger_read")


def rr_ledger_device_view(handle) -> rr_ledger_view:
    v = rr_ledger_view()
    _check(_lib.rr_ledger_device_view(handle, ctypes.byref(v)), "rr_ledger_device_view")
    return v


def rr_ledger_set_guard(handle, d_gamma_rows: int, max_age: int) -> None:
    _check(_lib.rr_ledger_set_guard(handle, ctypes.c_void_p(d_gamma_rows), max_age), "rr_ledger_set_guard")


def rr_ledger_set_hysteresis(handle, min_reuse: int) -> None:
    _check(_lib.rr_ledger_set_hysteresis(handle, min_reuse), "rr_ledger_set_hysteresis")


def rr_ledger_set_hysteresis_margin(handle, gamma_h: float) -> None:
    _check(_lib.rr_ledger_set_hysteresis_margin(handle, float(gamma_h)), "rr_ledger_set_hysteresis_margin")


def rr_ledger_set_wait_budget(handle, cycles: int) -> None:
    """Test hook (include/rr.h): the budget of the selection kernel's
    epilogue waits, in SM cycles (0: the default, about a second)."""
    _check(_lib.rr_ledger_set_wait_budget(handle, int(cycles)), "rr_ledger_set_wait_budget")


def rr_route_layer_static(cfg: rr_config, d_qc: int, d_kc: int, layer: int, d_ids: int, d_alpha: int,
                          d_anchor_layer: int, d_flags: int, d_counters: int, stream: int) -> None:
    """One layer on caller-held ledger arrays with no workspace and no
    allocation, for callers that cannot allocate device memory (their host
    framework owns every allocation).  See rr_route_layer_static in
    include/rr.h for its fixed capacity and its shared static scratch."""
    _check(_lib.rr_route_layer_static(ctypes.byref(cfg), ctypes.c_void_p(d_qc), ctypes.c_void_p(d_kc), layer,
                                      ctypes.c_void_p(d_ids), ctypes.c_void_p(d_alpha),
                                      ctypes.c_void_p(d_anchor_layer), ctypes.c_void_p(d_flags),
                                      ctypes.c_void_p(d_counters), ctypes.c_void_p(stream)),
           "rr_route_layer_static")


def rr_sparse_attention(cfg: rr_attn_config, d_q: int, d_k: int, d_v: int, d_route: int, d_out: int,
                        stream: int) -> None:
    """Sparse attention over a route (include/rr_attention.h)."""
    _check(_lib.rr_sparse_attention(ctypes.byref(cfg), ctypes.c_void_p(d_q), ctypes.c_void_p(d_k),
                                    ctypes.c_void_p(d_v), ctypes.c_void_p(d_route), ctypes.c_void_p(d_out),
                                    ctypes.c_void_p(stream)), "rr_sparse_attention")


# ---- convenience wrapper over torch memory --------------------------------
@dataclass
class Config:
    """Problem statement of one ledger (see rr_config in include/rr.h)."""
    bh: int
    nq: int
    nk: int
    d: int
    k: int
    m_near: int
    r_rand: int
    dtype: str = "f32"          # "f32" | "bf16"
    anchor_interval: int = 0
    causal: bool = False
    gamma: float = 0.0
    seed: int = 0
    bh_offset: int = 0
    g_sink: int = 0             # mandatory global sentinels: sink chunks
    g_recent: int = 0           # ... and recent chunks per row

    @property
    def c(self) -> int:
        return self.k + self.m_near + self.r_rand + self.g_sink + self.g_recent

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def to_c(self) -> rr_config:
        return rr_config(self.bh, self.nq, self.nk, self.d, RR_BF16 if self.dtype == "bf16" else RR_F32,
                         self.k, self.m_near, self.r_rand, self.anchor_interval, int(bool(self.causal)),
                         float(self.gamma), self.bh_offset, int(self.seed) & 0xFFFFFFFFFFFFFFFF,
                         self.g_sink, self.g_recent)


def _stream_handle(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def sparse_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, route: torch.Tensor, chunk: int,
                     causal: bool = False, width: int | None = None, scale: float | None = None,
                     out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Attention of every query token over the tokens of its chunk's route
    (RouteRelay §2.1, Eq. 3).  q [bh, nq_tokens, dh], k and v [bh, nk_tokens,
    dh]: contiguous bf16 on one CUDA device; route: contiguous int32 [bh,
    nq_tokens // chunk, stride] of key-chunk ids, of which the first `width`
    (default: all) are read.  Returns (or fills) fp32 [bh, nq_tokens, dh]."""
    bh, nq_tok, dh = q.shape
    nk_tok = k.shape[1]
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or t.dim() != 3 \
                or t.shape[0] != bh or t.shape[2] != dh or t.device != q.device:
            raise ValueError(f"{name}: expected contiguous bf16 [bh, tokens, {dh}] on {q.device}, "
                             f"got {t.dtype} {tuple(t.shape)} on {t.device}")
    if tuple(v.shape) != tuple(k.shape):
        raise ValueError(f"v {tuple(v.shape)} must match k {tuple(k.shape)}")
    if route.dtype != torch.int32 or not route.is_contiguous() or route.device != q.device or route.dim() != 3 \
            or route.shape[0] != bh or route.shape[1] * chunk != nq_tok:
        raise ValueError(f"route: expected contiguous int32 [{bh}, {nq_tok // max(chunk, 1)}, stride] on "
                         f"{q.device}, got {route.dtype} {tuple(route.shape)} on {route.device}")
    stride = route.shape[2]
    width = stride if width is None else int(width)
    if out is None:
        out = torch.empty((bh, nq_tok, dh), dtype=torch.float32, device=q.device)
    elif out.dtype != torch.float32 or not out.is_contiguous() or tuple(out.shape) != (bh, nq_tok, dh) \
            or out.device != q.device:
        raise ValueError("out: expected contiguous float32 [bh, nq_tokens, dh] on the inputs' device")
    cfg = rr_attn_config(bh, nq_tok, nk_tok, dh, chunk, width, max(stride, 1), int(bool(causal)),
                         0.0 if scale is None else float(scale))
    rr_sparse_attention(cfg, q.data_ptr(), k.data_ptr(), v.data_ptr(), route.data_ptr(), out.data_ptr(),
                        _stream_handle(stream))
    return out


class RouteLedger:
    """One ledger (RouteRelay Eq. 4) in a torch-allocated device workspace."""

    def __init__(self, cfg: Config, device=None):
        self.cfg = cfg
        self._c = cfg.to_c()
        dev = torch.device(device if device is not None else "cuda")
        if dev.type == "cuda" and dev.index is None:
            dev = torch.device("cuda", torch.cuda.current_device())
        self.device = dev
        nbytes = rr_ledger_workspace_bytes(self._c)
        if nbytes == 0:
            raise RRError(RR_EINVAL, "rr_ledger_workspace_bytes (invalid config)")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        self.handle = rr_ledger_create(self._c, self.workspace.data_ptr(), nbytes)

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and _lib is not None:
            _lib.rr_ledger_destroy(h)
            self.handle = None

    def _args(self, qc: torch.Tensor, kc: torch.Tensor):
        c = self.cfg
        for name, t, n in (("qc", qc, c.nq), ("kc", kc, c.nk)):
            if t.device != self.device or t.dtype != c.torch_dtype or not t.is_contiguous() \
                    or tuple(t.shape) != (c.bh, n, c.d):
                raise ValueError(f"{name}: expected contiguous {c.torch_dtype} [{c.bh}, {n}, {c.d}] on "
                                 f"{self.device}, got {t.dtype} {tuple(t.shape)} on {t.device}")
        return qc.data_ptr(), kc.data_ptr()

    def full_route(self, qc, kc, layer: int, stream=None):
        q, k = self._args(qc, kc)
        rr_full_route(self.handle, q, k, layer, _stream_handle(stream))

    def relay_layer(self, qc, kc, layer: int, stream=None):
        q, k = self._args(qc, kc)
        rr_relay_layer(self.handle, q, k, layer, _stream_handle(stream))

    def relay_rescore(self, qc, kc, layer: int, stream=None):
        q, k = self._args(qc, kc)
        rr_relay_rescore(self.handle, q, k, layer, _stream_handle(stream))

    def relay_compact(self, layer: int, stream=None):
        rr_relay_compact(self.handle, layer, _stream_handle(stream))

    def relay_refresh(self, qc, kc, layer: int, stream=None):
        q, k = self._args(qc, kc)
        rr_relay_refresh(self.handle, q, k, layer, _stream_handle(stream))

    def is_anchor(self, layer: int) -> bool:
        H = self.cfg.anchor_interval
        return layer == 0 or (H > 0 and layer % H == 0)

    def read(self, device="cpu", stream=None, check: bool = True) -> dict:
        """Copies the ledger out (ids [bh, nq, c], alpha, anchor_layer, flags,
        counters), synchronises the stream and raises on a device error."""
        c = self.cfg
        pin = torch.device(device).type == "cpu"
        mk = lambda shape, dt: torch.empty(shape, dtype=dt, device=device, pin_memory=pin)
        out = {"ids": mk((c.bh, c.nq, c.c), torch.int32), "alpha": mk((c.bh, c.nq), torch.float32),
               "anchor_layer": mk((c.bh, c.nq), torch.int32), "flags": mk((c.bh, c.nq), torch.uint8),
               "counters": mk((NUM_COUNTERS,), torch.int64)}
        v = rr_ledger_view(out["ids"].data_ptr(), out["alpha"].data_ptr(), out["anchor_layer"].data_ptr(),
                           out["flags"].data_ptr(), out["counters"].data_ptr())
        rr_ledger_read(self.handle, v, _stream_handle(stream))
        torch.cuda.synchronize(self.device)
        if check and int(out["counters"][CNT_ERROR]) != 0:
            raise RRError(RR_EDEVICE, f"device error word {int(out['counters'][CNT_ERROR]):#x}")
        return out

    def set_guard(self, gamma_rows=None, max_age: int = 0) -> None:
        """Per-row relay trigger: gamma_rows, a float32 device tensor of bh*nq
        guard margins (or None for cfg.gamma on every row), and the per-row
        lifetime bound max_age (0: off).  The tensor is kept referenced."""
        ptr = 0
        if gamma_rows is not None:
            c = self.cfg
            assert gamma_rows.dtype == torch.float32 and gamma_rows.is_contiguous()
            assert gamma_rows.numel() == c.bh * c.nq and gamma_rows.device == self.workspace.device
            ptr = gamma_rows.data_ptr()
        rr_ledger_set_guard(self.handle, ptr, int(max_age))
        self._gamma_rows = gamma_rows

    def set_hysteresis(self, min_reuse: int) -> None:
        """Minimum reuse horizon after a row is rebuilt (0: off)."""
        rr_ledger_set_hysteresis(self.handle, int(min_reuse))

    def set_hysteresis_margin(self, gamma_h: float) -> None:
        """Larger guard margin of a row rebuilt at a relay layer, until its
        test first passes (0: off; the mark is bit 1 of the flags)."""
        rr_ledger_set_hysteresis_margin(self.handle, float(gamma_h))

    def device_view(self) -> dict:
        """Zero-copy torch views of the ledger inside the workspace."""
        v = rr_ledger_device_view(self.handle)
        c = self.cfg
        base = self.workspace.data_ptr()
        ws = self.workspace

        def view(ptr, nbytes, dt, shape):
            off = ptr - base
            return ws[off:off + nbytes].view(dt).view(shape)

        rows = c.bh * c.nq
        return {"ids": view(v.ids, rows * c.c * 4, torch.int32, (c.bh, c.nq, c.c)),
                "alpha": view(v.alpha, rows * 4, torch.float32, (c.bh, c.nq)),
                "anchor_layer": view(v.anchor_layer, rows * 4, torch.int32, (c.bh, c.nq)),
                "flags": view(v.flags, rows, torch.uint8, (c.bh, c.nq)),
                "counters": view(v.counters, NUM_COUNTERS * 8, torch.int64, (NUM_COUNTERS,))}

    def sparse_attention(self, q, k, v, chunk: int, out=None, stream=None) -> torch.Tensor:
        """Attention over the ledger's current routes (the first k ids of each
        row, read in place): q [bh, nq * chunk, dh], k and v [bh, nk * chunk,
        dh] bf16 token tensors of the same layer, with the ledger's causal rule
        applied at token level."""
        c = self.cfg
        if q.shape[0] != c.bh or q.shape[1] != c.nq * chunk or k.shape[1] != c.nk * chunk:
            raise ValueError(f"q/k: expected [{c.bh}, {c.nq * chunk}, dh] / [{c.bh}, {c.nk * chunk}, dh], "
                             f"got {tuple(q.shape)} / {tuple(k.shape)}")
        ids = self.device_view()["ids"]
        return sparse_attention(q, k, v, ids, chunk, causal=c.causal, width=c.k, out=out, stream=stream)

    def layer(self, qc, kc, layer: int, stream=None):
        """Layer l of a sequence: an anchor at l == 0, else rr_relay_layer
        (which itself turns forced-anchor layers into full routing)."""
        if layer == 0:
            self.full_route(qc, kc, layer, stream)
        else:
            self.relay_layer(qc, kc, layer, stream)
