"""bench.py's host-side bookkeeping on the CPU: the DRAM traffic recorded under
profiles/ is reported only while the measured kernels' sources are unchanged,
and the whole-job aggregate is the slowest rank's time over all ranks' tokens."""
import json

import bench


def test_recorded_traffic_follows_the_kernel_sources(tmp_path, monkeypatch):
    h = bench.kernel_source_hash()
    assert len(h) == 16 and h == bench.kernel_source_hash()  # deterministic
    assert bench.kernel_source_hash(bench.WGRAD_SOURCES) != h  # other kernels, other hash
    prof = tmp_path / "profiles"
    prof.mkdir()
    rec = {"wl": {"expert_gate_up": {"dram_bytes_per_launch": 123, "source_hash": h},
                  "expert_down": {"dram_bytes_per_launch": 456, "source_hash": "0" * 16}}}
    (prof / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # the sources are read from the package, the record from the patched root: link them
    real = bench.kernel_source_hash
    monkeypatch.setattr(bench, "kernel_source_hash", lambda files=bench.GEMM_SOURCES: h)
    assert bench.recorded_traffic("wl", "expert_gate_up") == 123
    assert bench.recorded_traffic("wl", "expert_down") is None       # stale record
    assert bench.recorded_traffic("wl", "missing") is None
    assert bench.recorded_traffic("other", "expert_gate_up") is None
    monkeypatch.setattr(bench, "kernel_source_hash", real)


def test_committed_traffic_record_is_consistent():
    """The committed record is self-consistent, and the bench reports it only
    while the forward GEMMs' sources hash to what it was taken on (after a
    kernel change and before a new capture, traffic is null)."""
    with open(bench.os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    e = rec["mixtral_8x"]["expert_gate_up"]
    assert e["dram_bytes_per_launch"] == e["read"] + e["write"]
    assert e["dram_bytes_per_launch"] >= e["algorithmic_bytes"] * 0.5
    got = bench.recorded_traffic("mixtral_8x", "expert_gate_up")
    if e["source_hash"] == bench.kernel_source_hash():
        assert got == e["dram_bytes_per_launch"]
    else:
        assert got is None


def test_aggregate_single_rank():
    ms_total, ms_step, value = bench.aggregate(100.0, 1, 8192, 20, "cpu")
    assert ms_total == 100.0 and ms_step == 5.0
    assert abs(value - 8192 / 5e-3) < 1e-6


def test_cpu_baseline_batches_each_expert_on_all_threads():
    """The oracle baseline on the tiny fp32 layer: every sampled row goes to the
    oracle once, all host threads are used, the value is positive, and the
    single-thread figure is the slower one."""
    import oracle
    from workloads import WORKLOADS
    r = bench.cpu_baseline(WORKLOADS["tiny_fp32"], seconds=1.0)
    assert r["kind"] == "oracle" and r["cores"] == oracle.num_threads()
    assert r["value"] > 0 and r["single_thread"]["value"] > 0
    if r["cores"] > 1:
        assert r["value"] > r["single_thread"]["value"]
    assert "1024 expert rows over 8 experts" in r["sample"]


def test_sample_tokens_respects_the_expert_budget():
    """The CPU sample stops adding tokens that need experts beyond the host
    weight budget (1.5 G elements), and otherwise follows the random order."""
    import numpy as np
    from workloads import WORKLOADS
    wl = WORKLOADS["decode_e256"]  # 3 * 7168 * 2048 elements per expert: 34 experts fit
    rng = np.random.default_rng(0)
    ids = np.stack([rng.permutation(wl.E)[:wl.K] for _ in range(wl.T)])
    kept = np.ones_like(ids, dtype=bool)
    toks, experts = bench._sample_tokens(wl, ids, kept, np.arange(wl.T), rows_target=1e9)
    assert len(experts) <= 34 and len(toks) >= 1
    assert set(experts) == {int(e) for t in toks for e in ids[t]}


def test_extra_config_workloads():
    w = bench.config_workload("mixtral_8x+shared")
    assert w.F_shared == w.F == 14336 and w.T == 8192
    assert bench.config_workload("fine_skewed").E == 64
