"""The C ABI from a plain C99 program (tests/c_consumer/abi_consumer.c): the
headers compile as C with strict warnings, the program links against the
in-tree libtsp.so, and its checks of the plan, map, schedules, sizes and error
reporting pass.  No GPU needed."""

import os
import shutil
import subprocess

import pytest

import folded_tensor_sequence_map_b200.tsp as TT

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_c_program_builds_and_passes(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler on this host")
    libdir = os.path.dirname(TT.LIB_PATH)
    exe = tmp_path / "abi_consumer"
    cmd = [cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c_consumer", "abi_consumer.c"), "-o", str(exe), "-L", libdir, "-ltsp",
           "-Wl,-rpath," + libdir]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)
