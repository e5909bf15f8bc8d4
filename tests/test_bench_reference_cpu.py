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
