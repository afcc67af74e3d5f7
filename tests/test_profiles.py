"""The ncu summaries under profiles/: each names its kernel and workload, gives the command that
made it (ncu with unlocked clocks, on one kernel and at most three launches for a full capture),
and that command runs committed files only."""
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROFILES = os.path.join(ROOT, "profiles")
FILES = sorted(f for f in os.listdir(PROFILES) if f.endswith(".md"))


def _commands(text):
    return [b for b in re.findall(r"```\n(.*?)```", text, re.S) if "ncu" in b]


def test_profiles_exist():
    assert any(f.startswith("launches_") for f in FILES)
    assert any(f.startswith("gemm_transform_") for f in FILES)


@pytest.mark.parametrize("name", FILES)
def test_profile_command(name):
    text = open(os.path.join(PROFILES, name)).read()
    cmds = _commands(text)
    assert cmds, f"{name}: no ncu command"
    for cmd in cmds:
        ncu = cmd[cmd.index("ncu"):]
        assert "--clock-control none" in ncu
        if "--set full" in ncu or "--section" in ncu:
            assert re.search(r"-k \"?regex:", ncu), "a full capture names its kernel"
            c = re.search(r"-c (\d+)", ncu)
            assert c and int(c.group(1)) <= 3, "a full capture takes at most three launches"
        # the command runs committed files only: the benchmark from the repository root
        assert "_work" not in cmd
        assert re.search(r"python bench\.py", cmd)
        # the plain run exits 0 before ncu starts (same command, `&&`)
        assert "&&" in cmd
    assert "Reading:" in text or "| kernel |" in text
