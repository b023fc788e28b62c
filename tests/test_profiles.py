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


def test_traffic_lines_are_well_formed():
    """Every traffic line names a timed kernel, a workload, a plausible DRAM figure per token and a
    16-digit source hash; bench.py uses a line only while that hash is the kernel's current one
    (`kernel_source_sha(kernel)`), so a kernel changed since its capture reports traffic null."""
    seen = set()
    for name, txt in _summaries().items():
        for m in re.finditer(r"traffic\s+kernel=(\S+)\s+workload=(\S+)\s+dram_bytes_per_token=([0-9.eE+-]+)"
                             r"\s+source_sha=(\S+)", txt):
            k, wl, v, sha = m.group(1), m.group(2), float(m.group(3)), m.group(4)
            assert wl in ("throughput", "long", "router"), (name, wl)
            assert 500.0 < v < 8000.0, (name, k, v)
            assert re.fullmatch(r"[0-9a-f]{16}", sha), (name, sha)
            seen.add(k)
    assert {"gemm_wi_geglu", "gemm_wo2_res_ln", "attn_global", "attn_local"} <= seen


def test_per_kernel_source_hash_follows_its_file(tmp_path, monkeypatch):
    """A kernel's hash covers its own source file and the shared headers only."""
    a = bench.kernel_source_sha("attn_local")
    assert a != bench.kernel_source_sha("gemm_wi_geglu")
    assert bench.kernel_source_sha("gemm_wo_res_ln") == bench.kernel_source_sha("gemm_wi_geglu")
    assert bench.kernel_source_sha("embed_ln") == bench.kernel_source_sha("scorer")


def test_launch_lists_name_a_kernel_source_hash():
    for name, txt in _summaries().items():
        if name.startswith("launches_"):
            assert re.search(r"Kernel sources `[0-9a-f]{16}`", txt), name


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
