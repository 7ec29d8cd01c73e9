"""The C ABI from plain C: tests/abi_consumer.c includes include/vggt_attn.h
as C99 (gcc, warnings as errors; the CUDA runtime header it includes uses
anonymous unions, so not -pedantic), links against the in-tree
libvggt_attn.so with every declared entry point resolved, and runs the
header's host-side rules (status strings, pooled token counts, argument
checks, empty problems) without a GPU."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB_DIR = os.path.join(ROOT, "feed_forward_view_b200")
CUDA_INC = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs a C compiler")
def test_plain_c_program_builds_links_and_passes_host_checks(tmp_path):
    lib = os.path.join(LIB_DIR, "libvggt_attn.so")
    assert os.path.exists(lib), "build the library first (feed_forward_view_b200/build.py)"
    exe = str(tmp_path / "abi_consumer")
    cc = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
          "-I", CUDA_INC, os.path.join(ROOT, "tests", "abi_consumer.c"), lib, f"-Wl,-rpath,{LIB_DIR}", "-o", exe]
    res = subprocess.run(cc, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0 and run.stdout.strip() == "ok", run.stdout + run.stderr


def test_plain_c_program_takes_every_declared_entry_point():
    import re

    from test_abi_host import declared_functions

    src = open(os.path.join(ROOT, "tests", "abi_consumer.c")).read()
    table = set(re.findall(r"\(vggt_fn\)&(vggt_\w+)", src))
    assert table == declared_functions()
