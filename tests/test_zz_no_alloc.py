"""The allocation-free entry point, rr_route_layer_static, against the regular
ledger entry points.

rr_route_layer_static serves callers that cannot allocate device memory
(their host framework owns every allocation): they pass only inputs and the
ledger arrays, and the call's scratch lives in a fixed array inside librr.so.
Here it must reproduce, layer after layer, what rr_full_route and
rr_relay_layer write into a workspace-backed ledger from the same inputs.
For bf16 the kernels compute the same scores and are deterministic, so
ids, flags, anchor layers and counters must be identical and alpha equal
(the parity tests' margin, 1e-5, is the bound asserted; exact equality is
expected).  An fp32 ledger routes on the tensor cores with the three-way
bf16 split while this entry point, which has no room for the selection
buffers, routes fp32 on the CUDA cores: the two round differently, so the
fp32 case checks the entry point against the oracle layer by layer instead
(the parity tests' comparison, ties counted).

The file is named so that pytest collects it last; it also runs alone.
"""
import pytest
import torch

import rr_workloads as W
from rr_parity import Report, compare_head, config_of, params_of

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def rr():
    import cross_layer_route_b200 as rr
    torch.cuda.set_device(0)
    return rr


def _static_arrays(rr, cfg):
    rows = cfg.bh * cfg.nq
    return {"ids": torch.full((cfg.bh, cfg.nq, cfg.c), -1, dtype=torch.int32, device=DEV),
            "alpha": torch.zeros(rows, dtype=torch.float32, device=DEV),
            "anchor_layer": torch.zeros(rows, dtype=torch.int32, device=DEV),
            "flags": torch.zeros(rows, dtype=torch.uint8, device=DEV),
            "counters": torch.zeros(rr.NUM_COUNTERS, dtype=torch.int64, device=DEV)}


def _call_static(rr, cfg, q, k, layer, a):
    rr.rr_route_layer_static(cfg.to_c(), q.data_ptr(), k.data_ptr(), layer, a["ids"].data_ptr(),
                             a["alpha"].data_ptr(), a["anchor_layer"].data_ptr(), a["flags"].data_ptr(),
                             a["counters"].data_ptr(), torch.cuda.current_stream().cuda_stream)


def test_static_entry_point_matches_the_oracle_on_fp32(rr):
    w = W.C3.with_(bh=4, layers=4, anchor_interval=8)
    cfg = config_of(w, rr)
    arrs = _static_arrays(rr, cfg)
    st = W.LayerStream(w, "cpu")
    p = params_of(w)
    total = Report()
    prev = None
    for layer in range(w.layers):
        qf, kf, qs, ks = st.next()
        _call_static(rr, cfg, qs.to(DEV), ks.to(DEV), layer, arrs)
        torch.cuda.synchronize()
        got = {"ids": arrs["ids"].cpu().numpy(),
               "alpha": arrs["alpha"].cpu().view(cfg.bh, cfg.nq).numpy(),
               "anchor_layer": arrs["anchor_layer"].cpu().view(cfg.bh, cfg.nq).numpy(),
               "flags": arrs["flags"].cpu().view(cfg.bh, cfg.nq).numpy()}
        anchor = layer == 0 or layer % w.anchor_interval == 0
        for h in range(w.bh):
            pv = (lambda n: None) if prev is None else (lambda n: prev[n][h])
            total.add(compare_head(p, h, layer, anchor, qf[h].numpy(), kf[h].numpy(), pv("ids"),
                                   pv("alpha"), pv("anchor_layer"), got["ids"][h], got["alpha"][h],
                                   got["anchor_layer"][h], got["flags"][h], prev_flags=pv("flags")))
        cnt = arrs["counters"].cpu()
        assert int(cnt[rr.CNT_ERROR]) == 0 and int(cnt[rr.CNT_LAST_LAYER]) == layer
        prev = got
    assert not total.mismatches, total.mismatches[:5]
    assert total.ties <= max(2, 0.05 * total.rows), (total.ties, total.rows)


@pytest.mark.parametrize("w", [W.C5.with_(bh=2, n=640, layers=4, anchor_interval=16)], ids=["bf16_causal"])
def test_static_entry_point_matches_ledger_entry_points(rr, w):
    cfg = config_of(w, rr)
    led = rr.RouteLedger(cfg, DEV)
    arrs = _static_arrays(rr, cfg)
    st = W.LayerStream(w, "cpu")
    for layer in range(w.layers):
        _, _, qs, ks = st.next()
        q, k = qs.to(DEV), ks.to(DEV)
        led.layer(q, k, layer)
        _call_static(rr, cfg, q, k, layer, arrs)
        ref = led.read()
        torch.cuda.synchronize()
        got = {n: t.cpu() for n, t in arrs.items()}
        assert torch.equal(got["ids"], ref["ids"]), layer
        assert torch.equal(got["flags"].view(cfg.bh, cfg.nq), ref["flags"]), layer
        assert torch.equal(got["anchor_layer"].view(cfg.bh, cfg.nq), ref["anchor_layer"]), layer
        assert torch.allclose(got["alpha"].view(cfg.bh, cfg.nq), ref["alpha"], rtol=0, atol=1e-5), layer
        assert torch.equal(got["counters"], ref["counters"]), layer
        if layer > 0:
            # relay layers are the ones that use the static scratch
            assert int(got["counters"][rr.CNT_LAST_LAYER]) == layer
    # two relay calls in a row ran (layers 1..3); some rows were refreshed
    assert int(arrs["counters"][rr.CNT_ROWS_TOTAL]) > cfg.bh * cfg.nq


def test_static_entry_point_rejects_problems_beyond_its_capacity(rr):
    cfg = rr.Config(bh=300, nq=4096, nk=4096, d=64, k=8, m_near=8, r_rand=8)   # 1.2M rows > 2^20
    dummy = torch.zeros(16, dtype=torch.int64, device=DEV)
    p = dummy.data_ptr()
    with pytest.raises(rr.RRError) as e:
        rr.rr_route_layer_static(cfg.to_c(), p, p, 1, p, p, p, p, p, 0)
    assert e.value.status == rr.RR_ECAPACITY
    cfg = rr.Config(bh=5000, nq=8, nk=8, d=64, k=4, m_near=2, r_rand=1)         # more heads than 4096
    with pytest.raises(rr.RRError) as e:
        rr.rr_route_layer_static(cfg.to_c(), p, p, 1, p, p, p, p, p, 0)
    assert e.value.status == rr.RR_ECAPACITY


@pytest.mark.parametrize("w", [W.C3.with_(bh=4, layers=6, anchor_interval=3),
                               W.C5.with_(bh=2, n=640, layers=6, anchor_interval=3)],
                         ids=["f32_causal", "bf16_causal"])
def test_static_entry_point_allocates_nothing(rr, w):
    """The entry point's defining property: once a device is set up (the
    first anchor and relay calls also load the kernels), further anchor and
    relay layers change neither torch's reserved pool nor the device's free
    memory as the driver reports it."""
    cfg = config_of(w, rr)
    arrs = _static_arrays(rr, cfg)
    st = W.LayerStream(w, "cpu")
    xs = []
    for _ in range(w.layers):
        _, _, qs, ks = st.next()
        xs.append((qs.to(DEV), ks.to(DEV)))
    for layer in (0, 1):   # set-up calls: an anchor and a relay layer
        _call_static(rr, cfg, xs[layer][0], xs[layer][1], layer, arrs)
    torch.cuda.synchronize()
    reserved0 = torch.cuda.memory_reserved(DEV)
    free0, _ = torch.cuda.mem_get_info(DEV)
    for layer in range(2, w.layers):   # layer 3 is a forced anchor, the others relay layers
        _call_static(rr, cfg, xs[layer][0], xs[layer][1], layer, arrs)
    torch.cuda.synchronize()
    assert torch.cuda.memory_reserved(DEV) == reserved0
    free1, _ = torch.cuda.mem_get_info(DEV)
    assert free1 == free0, (free0, free1)
    assert int(arrs["counters"][rr.CNT_LAST_LAYER].item()) == w.layers - 1
    assert int(arrs["counters"][rr.CNT_ERROR].item()) == 0
