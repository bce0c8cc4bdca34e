"""bench.py on a machine without a GPU: the reference arm's JSON line, the byte and
operation counts behind the roofline, and the guard that ties committed ncu
traffic figures to the kernel sources they were taken on."""
import json

import bench


def test_reference_arm_json_line(capsys):
    assert bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "3",
                       "--warmup", "1"]) == 0
    line = capsys.readouterr().out.strip().splitlines()[-1]
    r = json.loads(line)
    assert r["impl"] == "reference" and r["metric"] == bench.METRIC
    assert r["unit"] == "TOPS" and r["value"] > 0 and r["higher_is_better"] is True
    assert r["n_gpus"] == 1 and r["steps"] == 3 and r["warmup"] == 3  # warm-up raised to 3
    assert r["config"]["workload"] == "tiny"
    cb = r["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == r["value"]
    assert r["e2e"] == {"value": r["value"], "unit": "TOPS", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_gemm_counts():
    M, N, K, ko = 16, 4096, 4096, 64
    # weights (codes + scales + outlier columns) + activations + output
    assert bench.gemm_bytes("w8", M, N, K, ko) == (N * K + 4 * N + 2 * N * ko + M * K + 4 * M
                                                   + 2 * M * ko + 2 * M * N)
    assert bench.gemm_bytes("w4", M, N, K, ko) - bench.gemm_bytes("w8", M, N, K, ko) == \
        N * K // 2 + 4 * N * K // 128 - N * K
    assert bench.gemm_ops(M, N, K, ko, False) == 2 * M * N * K
    assert bench.gemm_ops(M, N, K, ko, True) == 2 * M * N * (K + ko)


def test_code_only_strips_comments_not_strings():
    src = 'int a; // one\n/* two\nthree */ const char *s = "x // y /* z */";\n\n  int b;'
    out = bench._code_only(src)
    assert "one" not in out and "two" not in out and "three" not in out
    assert '"x // y /* z */"' in out and out.splitlines()[-1] == "  int b;"


def test_traffic_is_tied_to_each_kernel_kinds_sources(tmp_path, monkeypatch):
    kinds = ("gemm_w8", "gemm_w4", "quantize")
    rec = {"source_hashes": {k: bench.kernel_source_hash(k) for k in kinds},
           "workloads": {"llama7b-decode": {k: {"bytes_per_launch": 1000.0 + i}
                                            for i, k in enumerate(kinds)}}}
    p = tmp_path / "traffic.json"
    p.write_text(json.dumps(rec))
    # figures taken on the current sources of a kind are returned
    for i, k in enumerate(kinds):
        assert bench.load_traffic(k, "llama7b-decode", str(p)) == 1000.0 + i
    assert bench.load_traffic("gemm_unknown", "llama7b-decode", str(p)) is None
    assert bench.load_traffic("gemm_w8", "llama7b-prefill", str(p)) is None
    # a change to one kind's sources voids that kind's figure only
    real = bench.kernel_source_hash
    monkeypatch.setattr(bench, "kernel_source_hash",
                        lambda kind=None: "0" * 16 if kind == "gemm_w4" else real(kind))
    assert bench.load_traffic("gemm_w4", "llama7b-decode", str(p)) is None
    assert bench.load_traffic("gemm_w8", "llama7b-decode", str(p)) == 1000.0


def test_committed_traffic_matches_its_recorded_sources():
    """Each committed figure is reported only while its kind's sources are unchanged."""
    with open(bench.os.path.join(bench.ROOT, "profiles", "dram_traffic.json")) as f:
        rec = json.load(f)
    for w, kinds in rec["workloads"].items():
        for k, v in kinds.items():
            if k not in bench.KERNEL_SOURCES:
                continue
            fresh = rec["source_hashes"].get(k) == bench.kernel_source_hash(k)
            assert bench.load_traffic(k, w) == (v["bytes_per_launch"] if fresh else None)


def _bench_cmd(*extra, env=None):
    import os
    import subprocess
    import sys
    e = dict(os.environ)
    e.pop("WORLD_SIZE", None)
    e.pop("RANK", None)
    e.update(env or {})
    return subprocess.run([sys.executable, bench.os.path.join(bench.ROOT, "bench.py"), *extra],
                          capture_output=True, text=True, env=e, timeout=600)


def test_gpus_flag_starts_one_process_per_gpu():
    """--gpus 2 without a launcher runs two ranks (rank 0 prints n_gpus 2), it does not
    silently run one."""
    p = _bench_cmd("--impl", "reference", "--gpus", "2", "--workload", "tiny", "--steps", "1",
                   "--warmup", "3")
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    assert json.loads(lines[0])["n_gpus"] == 2


def test_gpus_flag_must_match_the_launcher():
    p = _bench_cmd("--impl", "reference", "--gpus", "2", "--workload", "tiny",
                   env={"WORLD_SIZE": "1", "RANK": "0"})
    assert p.returncode == 2 and "--gpus 2" in p.stderr


def test_workload_modes_and_bytes_of_the_fp16_scale_format():
    _, cases = bench.workload_cases("llama7b-decode")
    assert {m for _, ms in cases for m in ms} == {"w8", "w4", "w4b"}
    _, cases = bench.workload_cases("llama7b-prefill", modes="w4b")
    assert all(ms == ("w4b",) for _, ms in cases)
    M, N, K, ko = 16, 4096, 4096, 64
    # reading-B weights carry no per-row scale s_w
    assert bench.gemm_bytes("w4", M, N, K, ko) - bench.gemm_bytes("w4b", M, N, K, ko) == 4 * N
