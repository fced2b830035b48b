"""The committed profile summaries stay reproducible and safe to re-run: every command they
give runs committed files only, every ncu command leaves the GPU clocks alone, and the
DRAM-traffic table names kernel sources that exist."""

import glob
import json
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROFILES = sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md")))


def logical_lines(text):
    """Lines with shell continuations (a trailing backslash) joined."""
    out, cur = [], ""
    for line in text.splitlines():
        if line.rstrip().endswith("\\"):
            cur += line.rstrip()[:-1] + " "
        else:
            out.append(cur + line)
            cur = ""
    if cur:
        out.append(cur)
    return out


def test_there_are_profile_summaries():
    assert len(PROFILES) >= 5


def test_summaries_name_no_scratch_paths():
    for path in PROFILES:
        text = open(path).read()
        assert "_work/" not in text, path
        assert "gpurun" not in text, path


def test_every_ncu_command_leaves_clocks_alone():
    n = 0
    for path in PROFILES:
        for line in logical_lines(open(path).read()):
            if re.search(r"(^\s*|&&\s*)ncu\s+-", line):   # a command, not prose about ncu
                n += 1
                assert "--clock-control none" in line, (path, line)
    assert n >= 5


def test_commands_run_committed_scripts():
    for path in PROFILES:
        for line in logical_lines(open(path).read()):
            for script in re.findall(r"python3?\s+([\w./-]+\.py)", line):
                assert os.path.exists(os.path.join(ROOT, script)), (path, script)


def test_traffic_table_sources_exist():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        entries = json.load(f)["entries"]
    assert entries
    for e in entries:
        assert e["leg"] in ("prefill", "decode")
        assert e["bytes"] > 0
        for name in e["sources"]:
            assert os.path.exists(os.path.join(ROOT, "kv_cache_decode_attn_b200", "csrc", name)), name
