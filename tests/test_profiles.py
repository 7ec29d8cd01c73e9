"""The ncu summaries under profiles/: each gives the full command that made it,
every such command leaves the GPU clocks alone (--clock-control none), a
full-set capture names one kernel (-k) and at most three launches (-c), and the
program it profiles is a committed file of this repository, run on a workload
it defines."""
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SUMMARIES = sorted(glob.glob(os.path.join(ROOT, "profiles", "*.txt")))


def ncu_commands(path):
    """The ncu command lines of a summary's header, continuation lines joined."""
    cmds, cur = [], None
    for line in open(path):
        if not line.startswith("#"):
            break
        body = line[1:].strip()
        if cur is not None:
            cur += " " + body.rstrip("\\").strip()
            if not body.endswith("\\"):
                cmds.append(cur)
                cur = None
        elif body.startswith("ncu ") and "--" in body and ("-o " in body or "--log-file" in body or "--csv" in body):
            cur = body.rstrip("\\").strip()
            if not body.endswith("\\"):
                cmds.append(cur)
                cur = None
    return cmds


def test_there_are_summaries():
    assert SUMMARIES


@pytest.mark.parametrize("path", SUMMARIES, ids=os.path.basename)
def test_summary_states_a_safe_command(path):
    cmds = ncu_commands(path)
    assert cmds, "no ncu command in the header"
    for cmd in cmds:
        assert "--clock-control none" in cmd, cmd
        if "--set full" in cmd:
            assert re.search(r"\s-k\s", cmd), cmd
            c = re.search(r"\s-c\s+(\d+)", cmd)
            assert c and 1 <= int(c.group(1)) <= 3, cmd
        prog = re.search(r"\spython\s+(\S+\.py)", cmd)
        assert prog, cmd
        assert os.path.exists(os.path.join(ROOT, prog.group(1))), cmd
        assert "_work" not in cmd.split(), cmd
        wl = re.search(r"--workload\s+(\S+)", cmd)
        if wl:
            import synth

            assert wl.group(1) in synth.ALL_WORKLOADS, cmd
