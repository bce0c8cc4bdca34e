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


def test_traffic_is_tied_to_each_kernel_kinds_sources(monkeypatch):
    # the committed figures were taken on the current sources of the measured kinds
    for w in ("llama7b-decode", "llama7b-prefill"):
        for k in ("gemm_w8", "gemm_w4", "quantize"):
            assert bench.load_traffic(k, w) > 0, (k, w)
    assert bench.load_traffic("gemm_unknown", "llama7b-decode") is None
    # a change to one kind's sources voids that kind's figure only
    real = bench.kernel_source_hash
    monkeypatch.setattr(bench, "kernel_source_hash",
                        lambda kind=None: "0" * 16 if kind == "gemm_w4" else real(kind))
    assert bench.load_traffic("gemm_w4", "llama7b-decode") is None
    assert bench.load_traffic("gemm_w8", "llama7b-decode") > 0
