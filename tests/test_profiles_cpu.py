"""The profile summaries stay reproducible from committed files: every command they give runs
bench.py with flags its parser accepts, every ncu command keeps the clocks unlocked, and nothing
names an uncommitted working file. (Parsing only; nothing is run.)"""
import glob
import os
import re
import shlex

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROFILES = sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md")))


def _commands(path):
    """Shell commands inside the file's fenced blocks, continuation lines joined."""
    text = open(path).read()
    cmds = []
    for block in re.findall(r"```[a-z]*\n(.*?)```", text, flags=re.S):
        joined = re.sub(r"\\\n\s*", " ", block)
        for line in joined.splitlines():
            for part in re.split(r"&&|\|\|", line):
                part = part.strip()
                if part:
                    cmds.append(part)
    return cmds


def _bench_args(cmd):
    """The argument list of `python bench.py ...` inside cmd (also when ncu wraps it)."""
    toks = shlex.split(cmd.split(">")[0])
    for i in range(len(toks) - 1):
        if toks[i] == "python" and toks[i + 1] == "bench.py":
            return toks[i + 2:]
    return None


def test_profiles_exist():
    assert len(PROFILES) >= 8


@pytest.mark.parametrize("path", PROFILES, ids=[os.path.basename(p) for p in PROFILES])
def test_profile_commands_use_committed_bench_flags(path, monkeypatch):
    import sys

    import bench

    text = open(path).read()
    assert "_work" not in text, "a profile names an uncommitted working file"
    cmds = _commands(path)
    for c in cmds:
        if c.startswith("ncu"):
            assert "--clock-control none" in c, c
            assert "python bench.py" in c, c
    bench_cmds = [a for a in (_bench_args(c) for c in cmds) if a is not None]
    assert bench_cmds, f"{os.path.basename(path)} gives no bench.py command"
    for args in bench_cmds:
        monkeypatch.setattr(sys, "argv", ["bench.py", *args])
        try:
            bench.parse()
        except SystemExit as e:  # argparse rejects an unknown flag or a bad choice
            pytest.fail(f"{os.path.basename(path)}: bench.py {' '.join(args)} is not accepted ({e})")
