"""The reference arm of bench.py (the CPU oracle timed on a bounded sample)
runs without a GPU: its JSON line carries the keys the benchmark contract
asks for, on the same metric and workload as the CUDA arm."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "1"],
                         cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [line for line in out.stdout.splitlines() if line.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["N"] == 4096 and d["config"]["B"] == 2 and d["config"]["H"] == 12


def test_attention_source_follows_the_dispatch_rule_and_the_traffic_records():
    """bench.py names the attention kernel whose DRAM traffic record it
    reports with the library's dispatch rule (tcgen05 from 45 % of the block
    map selected, bf16, head size 64): the saturated N=2048 workload takes the
    tcgen05 kernel, the others the warp-level one, and every recorded
    attention traffic entry belongs to the kernel that runs its workload."""
    sys.path.insert(0, ROOT)
    import bench
    from resolution_block_sparse_b200.workloads import WORKLOADS
    want = {1: "mra_attn.cu", 2: "mra_attn.cu", 3: "mra_attn_tc.cu", 4: "mra_attn.cu", 5: "mra_attn.cu"}
    for i, src in want.items():
        assert bench.attention_source(WORKLOADS[i]) == src, i
        assert bench.attention_source(WORKLOADS[i], "mma") == "mra_attn.cu"
    assert bench.attention_source(WORKLOADS[4], "tc") == "mra_attn_tc.cu"
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    for key, entry in rec.items():
        if key.startswith("_") or "attention" not in entry:
            continue
        assert entry["attention"]["source"] == bench.attention_source(WORKLOADS[int(key)]), key


def test_cuda_arm_line_from_a_stubbed_run(monkeypatch, capsys):
    """The CUDA arm's JSON line, assembled on the CPU from a stubbed device
    run of the N=4096 workload: every key the benchmark contract asks for,
    the attention phase as the roofline kernel with the recorded DRAM
    traffic, and the throughput computed from the stubbed step time."""
    sys.path.insert(0, ROOT)
    import bench

    def fake_run(args, w, world, rank, local):
        return {"ms": 0.0625, "e2e_ms": 1.0, "eager_ms": 0.19, "h2d": 37748736, "d2h": 12582912,
                "phases": {"pool": (1, 0.0124), "lowres_select": (1, 0.0214), "attention": (1, 0.0359)},
                "status": 0, "launches_per_step": 3,
                "clocks": {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 4}}

    monkeypatch.setattr(bench, "run_cuda", fake_run)
    monkeypatch.delenv("MRA_ATTN_IMPL", raising=False)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--no-cpu-baseline"])
    bench.main()
    lines = [line for line in capsys.readouterr().out.splitlines() if line.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches",
                "clocks"):
        assert key in d, key
    assert abs(d["value"] - 2 * 4096 / 0.0625e-3) < 1e-3 * d["value"]
    assert d["roofline"]["kernel"] == "attention" and d["roofline"]["bound"] == "hbm"
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        recorded = json.load(f)["4"]["attention"]["dram_bytes_per_launch"]
    assert d["roofline"]["traffic"] == recorded
    assert d["gpu_launches"] == 3 * d["steps"]
    assert d["e2e"]["h2d_bytes_per_step"] == 37748736
