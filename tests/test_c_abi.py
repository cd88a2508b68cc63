"""The C ABI from C: tests/c/abi_host.c is compiled with gcc against
include/nattn.h, linked with libnattn.so and run (host-side entry points
only, so no GPU is needed)."""

import os
import shutil
import subprocess

import pytest

from tests._util import ensure_built

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_links_and_checks_host_entry_points(tmp_path):
    lib = ensure_built()
    libdir = os.path.dirname(lib)
    exe = tmp_path / "abi_host"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror",
                    "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_host.c"),
                    "-L", libdir, "-lnattn", "-Wl,-rpath," + libdir, "-o", str(exe)],
                   check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "ok"
