"""Host-side arithmetic of bench.py, checked without a GPU: the visible-pair
count behind the attention roofline, the clock-record summary that decides
whether a run is kept, the lookup of a profiled traffic figure by source
hash, and the config block both arms print."""
import hashlib

import pytest

import bench
import oracle
import rr_workloads as W


@pytest.mark.parametrize("causal", [False, True])
def test_visible_pairs_match_brute_force(causal):
    n, chunk, width = 10, 4, 5
    route = W.random_routes(2, n, n, width, causal, seed=9, pad=0.3)
    route[0, 3, 0] = n + 2            # out of range: no pairs
    route[1, 2, 1] = 7                # past the query chunk: none under causal
    brute = 0
    for h in range(2):
        for i in range(n):
            toks = oracle.expand_route(route[h, i].numpy(), chunk, n)
            for t in range(i * chunk, (i + 1) * chunk):
                brute += int((toks <= t).sum()) if causal else toks.size
    assert bench.visible_pairs(route, n, chunk, causal) == brute


def test_clock_summary_reads_reasons_and_the_loaded_median():
    c = bench.ClockSampler(0)
    row = "0, {sm}, 1965, 700.0, 0x0, {hw}, Not Active, Not Active, {pc}"
    c.lines = [row.format(sm=345, hw="Not Active", pc="Not Active")] + \
              [row.format(sm=s, hw="Not Active", pc="Active" if s == 1900 else "Not Active")
               for s in (1965, 1965, 1900, 1965)] + ["garbage", "0, N/A, 1965"]
    s = c.summary()
    assert s["sm_mhz"] == 1965 and s["sm_max_mhz"] == 1965 and s["samples"] == 5
    assert s["reasons"] == ["sw_power_cap"]
    c.lines = [row.format(sm=1965, hw="Active", pc="Not Active")]
    assert c.summary()["reasons"] == ["hw_slowdown"]
    c.lines = []
    assert c.summary()["reasons"] == ["unsampled"]


def test_profiled_traffic_needs_the_profiled_source(tmp_path, monkeypatch):
    (tmp_path / "cross_layer_route_b200" / "csrc").mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    src = tmp_path / "cross_layer_route_b200" / "csrc" / "k.cu"
    src.write_text("int k(int x) {  // v1\n    return x + 1;\n}\n")
    sha = hashlib.sha256(b"int k(int x) {\nreturn x + 1;\n}").hexdigest()
    assert bench.code_sha256(str(src)) == sha
    (tmp_path / "profiles" / "k__case.md").write_text(f"x\ntraffic_bytes_per_row: 1234\ncode_sha256: {sha}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic_per_row("k.cu", "k__*.md") == 1234.0
    # comments and blank lines only: the same code, the counters still hold
    src.write_text("/* the kernel */\nint k(int x) {  // v1, reworded\n\n    return x + 1;\n}\n")
    assert bench.profiled_traffic_per_row("k.cu", "k__*.md") == 1234.0
    src.write_text("int k(int x) {\n    return x + 2;\n}\n")   # the code changed: the counters are stale
    assert bench.profiled_traffic_per_row("k.cu", "k__*.md") is None


def test_config_block_and_shards():
    cfg = bench.workload_config(W.C5, 4)
    assert cfg["workload"] == W.C5.name and cfg["bh_per_gpu"] == 256 and cfg["parallelism"].endswith("no collective")
    assert "16.0 GiB" in cfg["l2"]
    assert [bench.shard_offset(r, W.C5) for r in range(3)] == [0, 256, 512]
    assert bench.full_pairs_per_layer(W.C5) == 256 * 4096 * 4097 // 2
    assert bench.full_pairs_per_layer(W.C2) == 128 * 256 * 256


def test_layer_kinds_split():
    k = bench.layer_kinds(1000, anchor_ms=8.0, n_anchor=4, relay_ms=30.0, n_relay=10)
    assert k["anchor"] == {"layers": 4, "ms_per_layer": 2.0, "rows_per_s": 1000 * 4 / 8e-3}
    assert k["relay"]["ms_per_layer"] == 3.0 and k["relay"]["rows_per_s"] == pytest.approx(1000 / 3e-3)
    assert bench.layer_kinds(1000, 5.0, 2, 0.0, 0) == {"anchor": {"layers": 2, "ms_per_layer": 2.5,
                                                                  "rows_per_s": 1000 * 2 / 5e-3}}


def test_cpu_baseline_runs_the_oracle_on_a_bounded_sample():
    st = W.LayerStream(W.PR1, "cpu")
    qs, ks = [], []
    for _ in range(2):
        _, _, q, k = st.next()
        qs.append(q)
        ks.append(k)
    cb = bench.cpu_baseline(W.PR1, qs, ks, threads=1, layers=2)
    assert cb["kind"] == "oracle" and cb["unit"] == "rows/s" and cb["cores"] == 1 and cb["value"] > 0
    assert "1 heads x 2 layers" in cb["sample"] and isinstance(cb["cpu_model"], str)


def _args(gpus, impl="ours"):
    import argparse
    return argparse.Namespace(gpus=gpus, impl=impl)


def test_gpus_n_without_a_launcher_starts_n_ranks_or_fails():
    # N > 1 and no launcher: start N ranks when N GPUs are visible, else fail
    assert bench.resolve_world(_args(2), env={}, device_count=8) == ("launch", 2)
    how, why = bench.resolve_world(_args(2), env={}, device_count=1)
    assert how == "fail" and "--gpus 2" in why
    assert bench.resolve_world(_args(1), env={}, device_count=0) == ("run", 1)
    # under a launcher the rank count must be --gpus
    assert bench.resolve_world(_args(4), env={"WORLD_SIZE": "4"}) == ("run", 4)
    assert bench.resolve_world(_args(4), env={"WORLD_SIZE": "2"})[0] == "fail"
    assert bench.resolve_world(_args(1), env={"WORLD_SIZE": "2"})[0] == "fail"
    # the reference arm is rank 0's work: it runs in place and reports --gpus
    assert bench.resolve_world(_args(8, "reference"), env={}, device_count=0) == ("run", 1)
    cmd = bench.launcher_command(["--gpus", "2", "--steps", "3"], 2, 29555)
    assert cmd[1:3] == ["-m", "torch.distributed.run"] and "--nproc-per-node=2" in cmd
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1" and cmd[cmd.index("--master-port") + 1] == "29555"
    assert cmd[-4:] == ["--gpus", "2", "--steps", "3"] and cmd[-5].endswith("bench.py")


def test_bench_gpus_2_never_runs_a_single_rank_silently():
    """The script itself, as the driver would start it without torchrun: on a
    host with fewer than two GPUs it must exit non-zero and print no result
    line (a one-rank line labelled n_gpus 1 is what this guards against)."""
    import subprocess
    import sys
    env = {k: v for k, v in __import__("os").environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    env["CUDA_VISIBLE_DEVICES"] = ""
    p = subprocess.run([sys.executable, bench.__file__, "--gpus", "2", "--steps", "1"], env=env,
                       capture_output=True, text=True, timeout=300)
    assert p.returncode != 0
    assert '"metric"' not in p.stdout and "--gpus 2" in p.stderr


def test_graph_mode_default_follows_the_step_length():
    import argparse
    a = argparse.Namespace(graph="auto")
    assert bench.graph_mode(a, W.C2) and bench.graph_mode(a, W.PR1) and not bench.graph_mode(a, W.C5)
    assert bench.graph_mode(argparse.Namespace(graph="on"), W.C5)
    assert not bench.graph_mode(argparse.Namespace(graph="off"), W.C2)


def test_kernel_path_and_launch_count_per_workload():
    assert bench.uses_tensor_cores(W.C5) and not bench.uses_split(W.C5)
    for w in (W.PR1, W.C2, W.C3, W.C4):
        assert bench.uses_tensor_cores(w) and bench.uses_split(w)
    assert not bench.uses_tensor_cores(W.C2.with_(d=32))
    assert not bench.uses_tensor_cores(W.C2.with_(k=48, m=24))
    # C5: 2 anchors x 4 + 30 one-shot relays x 5; C2 (split): 4 x 5 + 28 x 6
    assert bench.launches_per_step(W.C5, 2, 30, True) == 2 * 4 + 30 * 5
    assert bench.launches_per_step(W.C2, 4, 28, True) == 4 * 5 + 28 * 6
    assert bench.launches_per_step(W.C2.with_(d=32), 4, 28, True) == 4 * 2 + 28 * 4
