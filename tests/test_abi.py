"""Host-side checks of the C ABI (include/rr.h): the library loads, exports
every declared entry point, lays out the workspace as documented and rejects
bad arguments before touching a device.  No GPU needed: none of these calls
reaches the CUDA runtime."""
import ctypes
import os
import re

import pytest

import cross_layer_route_b200 as rr

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE_WS = 0x7F00_0000_0000      # never dereferenced by these tests
FAKE_Q = 0x7F10_0000_0000


def header_functions():
    names = set()
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(rr_[a-z_0-9]+)\s*\(", src))
    return names


def test_library_is_built_for_sm100a_and_exports_every_declared_symbol():
    lib = ctypes.CDLL(rr.LIB_PATH)
    names = header_functions()
    assert {"rr_ledger_create", "rr_full_route", "rr_relay_layer", "rr_ledger_read"} <= names
    for n in sorted(names):
        assert hasattr(lib, n), n


def cfg(**kw):
    base = dict(bh=2, nq=64, nk=64, d=64, k=8, m_near=8, r_rand=4, dtype="f32", anchor_interval=4)
    base.update(kw)
    return rr.Config(**base)


def test_workspace_layout_and_ledger_size():
    # RouteRelay §4.4: a 32-bit index ledger with nq = 1024 and c = 64 holds 256 KB
    c = cfg(bh=1, nq=1024, nk=1024, k=32, m_near=16, r_rand=16)
    nbytes = rr.rr_ledger_workspace_bytes(c.to_c())
    h = rr.rr_ledger_create(c.to_c(), FAKE_WS, nbytes)
    v = rr.rr_ledger_device_view(h)
    assert v.ids == FAKE_WS
    assert v.alpha - v.ids == 1024 * 64 * 4 == 256 * 1024
    assert v.anchor_layer - v.alpha >= 1024 * 4 and v.flags - v.anchor_layer >= 1024 * 4
    assert v.counters % 256 == 0 and nbytes >= (v.counters - v.ids) + 64
    rr.rr_ledger_destroy(h)


@pytest.mark.parametrize("bad", [
    dict(k=0), dict(k=65, nk=64), dict(d=12), dict(d=264), dict(d=0), dict(m_near=-1),
    dict(k=100, m_near=29), dict(r_rand=129), dict(bh=0), dict(nq=0), dict(nk=0),
    dict(gamma=-0.1), dict(gamma=float("nan")), dict(gamma=float("inf")), dict(anchor_interval=-1),
])
def test_invalid_configs_are_rejected(bad):
    c = cfg(**bad)
    assert rr.rr_ledger_workspace_bytes(c.to_c()) == 0
    with pytest.raises(rr.RRError) as e:
        rr.rr_ledger_create(c.to_c(), FAKE_WS, 1 << 30)
    assert e.value.status == rr.RR_EINVAL


def test_limits_at_the_edge_are_accepted():
    for c in (cfg(k=64, nk=64, m_near=64, r_rand=128, d=256), cfg(d=8, k=1, m_near=0, r_rand=0)):
        nbytes = rr.rr_ledger_workspace_bytes(c.to_c())
        assert nbytes > 0
        rr.rr_ledger_destroy(rr.rr_ledger_create(c.to_c(), FAKE_WS, nbytes))


def test_create_argument_errors():
    c = cfg()
    nbytes = rr.rr_ledger_workspace_bytes(c.to_c())
    with pytest.raises(rr.RRError) as e:
        rr.rr_ledger_create(c.to_c(), 0, nbytes)
    assert e.value.status == rr.RR_EINVAL
    with pytest.raises(rr.RRError) as e:
        rr.rr_ledger_create(c.to_c(), FAKE_WS + 16, nbytes)   # not 256-byte aligned
    assert e.value.status == rr.RR_EINVAL
    with pytest.raises(rr.RRError) as e:
        rr.rr_ledger_create(c.to_c(), FAKE_WS, nbytes - 1)
    assert e.value.status == rr.RR_ENOMEM
    lib = ctypes.CDLL(rr.LIB_PATH)
    lib.rr_ledger_create.restype = ctypes.c_int
    assert lib.rr_ledger_create(None, None, ctypes.c_size_t(0), None) == rr.RR_EINVAL


def test_call_order_and_pointer_errors_before_any_device_work():
    c = cfg()
    nbytes = rr.rr_ledger_workspace_bytes(c.to_c())
    h = rr.rr_ledger_create(c.to_c(), FAKE_WS, nbytes)
    with pytest.raises(rr.RRError) as e:             # relay before any anchor
        rr.rr_relay_layer(h, FAKE_Q, FAKE_Q, 1, 0)
    assert e.value.status == rr.RR_ESTATE
    for q, k, layer in ((0, FAKE_Q, 0), (FAKE_Q, 0, 0), (FAKE_Q + 4, FAKE_Q, 0), (FAKE_Q, FAKE_Q, -1)):
        with pytest.raises(rr.RRError) as e:
            rr.rr_full_route(h, q, k, layer, 0)
        assert e.value.status == rr.RR_EINVAL
        with pytest.raises(rr.RRError) as e:
            rr.rr_relay_layer(h, q, k, layer, 0)
        assert e.value.status == rr.RR_EINVAL
    with pytest.raises(rr.RRError):
        rr.rr_ledger_read(None, rr.rr_ledger_view(), 0)
    rr.rr_ledger_destroy(h)
    rr.rr_ledger_destroy(None)


def test_status_strings():
    for s in range(6):
        assert rr.rr_status_string(s).startswith("RR_")
    assert rr.rr_status_string(99) == "RR_UNKNOWN"


def test_trigger_setters_validate_their_arguments_without_a_cuda_call():
    import ctypes
    import cross_layer_route_b200 as rr
    lib = rr._lib
    assert lib.rr_ledger_set_guard(None, None, 0) == rr.RR_EINVAL
    cfg = rr.Config(bh=2, nq=8, nk=8, d=16, k=2, m_near=1, r_rand=1).to_c()
    nbytes = lib.rr_ledger_workspace_bytes(ctypes.byref(cfg))
    buf = ctypes.create_string_buffer(nbytes + 256)
    base = (ctypes.addressof(buf) + 255) // 256 * 256   # host memory: create never touches it
    h = ctypes.c_void_p()
    assert lib.rr_ledger_create(ctypes.byref(cfg), ctypes.c_void_p(base), nbytes, ctypes.byref(h)) == rr.RR_OK
    try:
        assert lib.rr_ledger_set_guard(h, None, -1) == rr.RR_EINVAL
        assert lib.rr_ledger_set_guard(h, None, 0) == rr.RR_OK
        assert lib.rr_ledger_set_guard(h, ctypes.c_void_p(base), 4) == rr.RR_OK
        assert lib.rr_ledger_set_hysteresis(h, -1) == rr.RR_EINVAL
        assert lib.rr_ledger_set_hysteresis(h, 1) == rr.RR_OK
        assert lib.rr_ledger_set_hysteresis(None, 1) == rr.RR_EINVAL
        for bad in (-0.1, float("nan"), float("inf")):
            assert lib.rr_ledger_set_hysteresis_margin(h, bad) == rr.RR_EINVAL
        assert lib.rr_ledger_set_hysteresis_margin(h, 0.0) == rr.RR_OK
        assert lib.rr_ledger_set_hysteresis_margin(h, 0.05) == rr.RR_OK
        assert lib.rr_ledger_set_hysteresis_margin(None, 0.05) == rr.RR_EINVAL
        assert lib.rr_ledger_set_wait_budget(h, -1) == rr.RR_EINVAL
        assert lib.rr_ledger_set_wait_budget(h, 0) == rr.RR_OK
        assert lib.rr_ledger_set_wait_budget(None, 0) == rr.RR_EINVAL
    finally:
        lib.rr_ledger_destroy(h)


# ---- rr_sparse_attention (include/rr_attention.h) --------------------------
def attn_cfg(**kw):
    base = dict(bh=2, nq_tokens=256, nk_tokens=256, dh=128, chunk=64, width=4, route_stride=8, causal=1,
                scale=0.0)
    base.update(kw)
    return rr.rr_attn_config(*(base[f] for f, _ in rr.rr_attn_config._fields_))


@pytest.mark.parametrize("bad", [
    dict(dh=96), dict(dh=0), dict(chunk=48), dict(chunk=256), dict(nq_tokens=100), dict(nk_tokens=65),
    dict(width=-1), dict(width=1025, route_stride=2048), dict(route_stride=3), dict(route_stride=0, width=0),
    dict(bh=-1), dict(nq_tokens=-64), dict(scale=-1.0), dict(scale=float("nan")), dict(scale=float("inf")),
])
def test_attention_rejects_bad_shapes_without_a_cuda_call(bad):
    with pytest.raises(rr.RRError) as e:
        rr.rr_sparse_attention(attn_cfg(**bad), FAKE_Q, FAKE_Q, FAKE_Q, FAKE_Q, FAKE_Q, 0)
    assert e.value.status == rr.RR_EINVAL


def test_attention_rejects_null_and_misaligned_pointers():
    c = attn_cfg()
    for args in ((0, FAKE_Q, FAKE_Q, FAKE_Q, FAKE_Q), (FAKE_Q + 8, FAKE_Q, FAKE_Q, FAKE_Q, FAKE_Q),
                 (FAKE_Q, 0, FAKE_Q, FAKE_Q, FAKE_Q), (FAKE_Q, FAKE_Q, FAKE_Q + 2, FAKE_Q, FAKE_Q),
                 (FAKE_Q, FAKE_Q, FAKE_Q, 0, FAKE_Q), (FAKE_Q, FAKE_Q, FAKE_Q, FAKE_Q + 2, FAKE_Q),
                 (FAKE_Q, FAKE_Q, FAKE_Q, FAKE_Q, FAKE_Q + 4)):
        with pytest.raises(rr.RRError) as e:
            rr.rr_sparse_attention(c, *args, 0)
        assert e.value.status == rr.RR_EINVAL


def test_attention_with_nothing_to_do_returns_at_once():
    # no query token: nothing is launched, so even fake pointers are fine
    rr.rr_sparse_attention(attn_cfg(bh=0), FAKE_Q, FAKE_Q, FAKE_Q, FAKE_Q, FAKE_Q, 0)
    rr.rr_sparse_attention(attn_cfg(nq_tokens=0), FAKE_Q, FAKE_Q, FAKE_Q, FAKE_Q, FAKE_Q, 0)


def test_attention_binding_checks_tensors_before_the_library():
    import torch
    q = torch.zeros((1, 64, 64), dtype=torch.bfloat16)          # host tensors: rejected, nothing launched
    route = torch.zeros((1, 1, 4), dtype=torch.int32)
    with pytest.raises(ValueError):
        rr.sparse_attention(q, q, q, route, 64)
    with pytest.raises(ValueError):
        rr.sparse_attention(q.float(), q, q, route, 64)
    with pytest.raises(ValueError):
        rr.sparse_attention(q, q, q, route.long(), 64)
