"""bench.py's contract on the host: the reference arm's JSON line (the oracle on a bounded
sample, run here with a one-second sample) and the algorithmic work formulas."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0",
                          "--cpu-seconds", "1"], cwd=ROOT, capture_output=True, text=True, timeout=600, check=True)
    lines = [l for l in out.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "config",
                "cpu_baseline", "e2e"):
        assert key in j, key
    assert j["impl"] == "reference" and j["value"] > 0
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["cores"] >= 1
    assert j["cpu_baseline"]["value"] == j["value"]
    assert j["e2e"]["h2d_bytes_per_step"] == 0 and j["e2e"]["d2h_bytes_per_step"] == 0
    assert j["e2e"]["unit"] == j["unit"]


def test_prefill_flops_closed_forms():
    sys.path.insert(0, ROOT)
    import bench
    d = bench.D
    # one token, no memory: one visible key per (layer, head), 4 d flops
    assert bench.prefill_flops(1, 1, 1, 0) == 4 * d
    # T tokens causal over themselves plus M memory rows: T M + T (T + 1) / 2 pairs
    assert bench.prefill_flops(2, 3, 4, 5) == 4 * d * 2 * 3 * (4 * 5 + 10)


def test_gpus_flag_spawns_its_own_ranks():
    # --gpus 2 without a launcher starts two local ranks itself (torch.distributed.run on
    # 127.0.0.1); on the host the reference arm's ranks meet over gloo and rank 0 alone
    # prints the line
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1",
                          "--warmup", "0", "--cpu-seconds", "0.5"], cwd=ROOT, capture_output=True, text=True,
                         timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["n_gpus"] == 2 and j["value"] > 0


def test_gpus_flag_must_match_the_launcher():
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1",
                          "--warmup", "0", "--cpu-seconds", "0.5"], cwd=ROOT, capture_output=True, text=True,
                         timeout=300, env=env)
    assert out.returncode == 2 and "--gpus 2" in out.stderr
