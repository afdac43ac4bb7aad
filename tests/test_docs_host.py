"""The profiler summaries stay runnable: every bench.py command quoted in
profiles/ parses with bench.py's own argument parser, runs no working file, and
every ncu command there leaves the GPU clocks alone.  CPU only."""
import glob
import os
import re
import shlex

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROFILES = sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md")))


def _commands(path):
    """Shell commands of the fenced blocks, continuation lines joined."""
    text = open(path, encoding="utf-8").read()
    out = []
    for block in re.findall(r"```\n(.*?)```", text, flags=re.S):
        out += [c.strip() for c in block.replace("\\\n", " ").split("\n") if c.strip()]
    return out


@pytest.mark.parametrize("path", PROFILES, ids=[os.path.basename(p) for p in PROFILES])
def test_profile_commands_parse_and_keep_clocks(path):
    import bench
    cmds = _commands(path)
    assert cmds, f"{path} gives no command"
    n_bench = 0
    for cmd in cmds:
        for part in cmd.split("&&"):
            words = shlex.split(part)
            if "ncu" in words and "-i" not in words:  # "-i" reads a saved report, no GPU
                assert "--clock-control" in words and words[words.index("--clock-control") + 1] == "none", part
            if "bench.py" in words:
                bench.build_arg_parser().parse_args(words[words.index("bench.py") + 1:])
                n_bench += 1
            for w in words:
                assert "_work" not in w, f"{path} runs a working file: {w}"
    assert n_bench > 0


def _check_command(cmd):
    import bench
    n_bench = 0
    for part in cmd.split("&&"):
        words = shlex.split(part)
        if "ncu" in words and "-i" not in words:
            assert "--clock-control" in words and words[words.index("--clock-control") + 1] == "none", part
        if "bench.py" in words:
            bench.build_arg_parser().parse_args(words[words.index("bench.py") + 1:])
            n_bench += 1
        for w in words:
            assert "_work" not in w, f"runs a working file: {w}"
    return n_bench


def test_attention_traffic_records_are_complete():
    """Each DRAM-traffic record bench.py may scale names its workload, block size,
    capture length, byte counts (read + write = the per-launch figure), the
    kernel-source hash it belongs to and a runnable capture command; bench.py
    matches records by (workload, block, hash)."""
    import json
    recs = json.load(open(os.path.join(ROOT, "profiles", "attention_traffic.json")))["records"]
    assert recs
    keys = set()
    for r in recs:
        assert r["dram_bytes_read"] + r["dram_bytes_write"] == r["dram_bytes_per_launch_at_capture"]
        assert r["captured_N"] > 0 and r["block"] in (64, 128, 512)
        assert re.fullmatch(r"[0-9a-f]{16}", r["kernel_source_sha256_16"])
        assert _check_command(r["command"]) == 2  # the plain run, then the same command under ncu
        keys.add((r["workload"], r["block"], r["kernel_source_sha256_16"]))
    assert len(keys) == len(recs)
