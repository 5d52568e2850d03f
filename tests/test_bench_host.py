"""bench.py's host-side pieces that need no GPU: the reference arm (the oracle on the host cores) and the
traffic lookup in profiles/."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_runs_the_requested_steps():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "4",
                          "--warmup", "3"], cwd=ROOT, capture_output=True, text=True, timeout=300, check=True)
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["steps"] == 4 and line["warmup"] == 3
    assert line["value"] > 0 and line["unit"] == "tok/s" and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["config"]["workload"] == "tiny"


def test_reference_arm_other_ranks_stay_silent():
    env = dict(os.environ, RANK="1")
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "2",
                          "--warmup", "3"], cwd=ROOT, capture_output=True, text=True, timeout=300, check=True,
                         env=env)
    assert out.stdout.strip() == ""


def test_profile_traffic_matches_source_hash():
    sys.path.insert(0, ROOT)
    import bench
    # the prefill capture's kernel source is unchanged since the capture; an unknown kernel has none
    assert bench.profile_traffic("gemm_gateup") is None or bench.profile_traffic("gemm_gateup") > 0
    assert bench.profile_traffic("no_such_kernel") is None
