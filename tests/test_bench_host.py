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


def test_kernel_source_sections_exist():
    """Every kernel the bench hashes for its ncu traffic lines has its section markers in its source: a
    renamed marker would otherwise turn the traffic silently null."""
    sys.path.insert(0, ROOT)
    import bench
    for kernel, (src, start, end) in bench._KERNEL_SOURCE.items():
        h = bench.kernel_source_hash(kernel)
        assert h is not None and len(h) == 16, kernel
        if start is not None:
            text = open(os.path.join(ROOT, "bit_expert_ffn_gemv_b200", "csrc", src)).read()
            i = text.find(start)
            assert i >= 0 and text.find(end, i + 1) > i, kernel
    # the gate/up and down kernels share one section; the router's is another
    assert bench.kernel_source_hash("gemm_gateup") == bench.kernel_source_hash("gemm_down")
    assert bench.kernel_source_hash("gemm_gateup") != bench.kernel_source_hash("router_gemm")
    # a committed capture is used only for its own workload size, and only while its section is unchanged
    assert bench.profile_traffic("gemm_gateup", 8192) in (None, 677046272)
    assert bench.profile_traffic("gemm_down", 8192) in (None, 548585984)
    assert bench.profile_traffic("gemm_gateup", 64) is None
