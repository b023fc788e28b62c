"""The committed ncu summaries describe the kernels as they stand.

`bench.py` fills the roofline line's `traffic` from the summaries' traffic
lines only when their kernel-source hash matches the current sources; these
checks keep the summaries and the sources together, and the commands that made
them runnable from committed files.
"""
import os
import re
import subprocess

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROFILES = os.path.join(ROOT, "profiles")


def _summaries():
    return {f: open(os.path.join(PROFILES, f)).read() for f in sorted(os.listdir(PROFILES)) if f.endswith(".md")}


def test_traffic_lines_match_current_kernel_sources():
    sha = bench.kernel_source_sha()
    for k in ("gemm_wi_geglu", "gemm_wo2_res_ln", "gemm_wo_res_ln", "attn_global", "attn_local"):
        v = bench.recorded_traffic(k, "throughput")
        assert v is not None, f"no traffic line for {k} at kernel sources {sha}"
        assert 1000.0 < v < 8000.0, (k, v)


def test_launch_list_names_current_kernel_sources():
    txt = _summaries()["launches_forward_throughput_1024rows.md"]
    assert f"Kernel sources `{bench.kernel_source_sha()}`" in txt


def test_profile_commands_run_committed_files():
    try:
        tracked = set(subprocess.run(["git", "ls-files"], cwd=ROOT, capture_output=True, text=True).stdout.split())
    except OSError:
        tracked = set()
    if not tracked:  # a copy of the tree without its git metadata: the files must at least exist
        tracked = {f for f in os.listdir(ROOT) if f.endswith(".py")}
    for name, txt in _summaries().items():
        blocks = re.findall(r"```\n(.*?)```", txt, re.S)
        assert blocks, f"{name}: no command given"
        for b in blocks:
            assert "_work" not in b, name
            for script in re.findall(r"python\s+(\S+\.py)", b):
                assert script in tracked, (name, script)
            for line in b.splitlines():
                if line.startswith("ncu "):
                    assert "--clock-control none" in line, (name, line)
