"""The committed ncu summaries stay reproducible: every command they give
runs committed files with flags the harness accepts, and each names the
kernel it measured."""

import glob
import os
import re
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROFILES = sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md")))


def _bench_flags():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--help"],
                         capture_output=True, text=True, check=True).stdout
    return set(re.findall(r"(--[a-z][a-z0-9-]*)", out))


def _commands(text):
    """Lines of the fenced blocks, with backslash continuations joined."""
    cmds = []
    for block in re.findall(r"```\n(.*?)```", text, flags=re.S):
        cmds += [c.strip() for c in block.replace("\\\n", " ").splitlines() if c.strip()]
    return cmds


def test_there_are_profiles():
    assert len(PROFILES) >= 6


def test_profile_commands_use_known_bench_flags_and_committed_files():
    flags = _bench_flags()
    for path in PROFILES:
        text = open(path, encoding="utf-8").read()
        assert "_work" not in text, path
        cmds = _commands(text)
        assert cmds, f"{path}: no command"
        for cmd in cmds:
            if "bench.py" not in cmd:
                continue
            bench_args = cmd[cmd.index("bench.py"):]
            for flag in re.findall(r"(--[a-z][a-z0-9-]*)", bench_args):
                if flag in ("--clock-control", "--metrics", "--set", "--csv", "--log-file",
                            "--section"):
                    continue  # ncu's own, when it precedes the bench command
                assert flag in flags, f"{os.path.basename(path)}: unknown bench flag {flag}"


def test_ncu_commands_keep_clock_control_off():
    for path in PROFILES:
        for cmd in _commands(open(path, encoding="utf-8").read()):
            if cmd.startswith("ncu "):
                assert "--clock-control none" in cmd, f"{os.path.basename(path)}: {cmd}"
