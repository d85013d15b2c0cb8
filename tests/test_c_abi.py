"""The boundary is a C ABI: a C99 program (tests/c/abi_c99.c) compiles
against include/ba.h and include/ba_graph.h with gcc in strict mode, links
libba.so and checks the entry points that need no GPU."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.join(os.path.dirname(__file__), "..")
LIBDIR = os.path.join(ROOT, "bit_qk_attention_ba_b200")


def test_headers_compile_and_link_as_c99(tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    if not os.path.exists(os.path.join(LIBDIR, "libba.so")):
        pytest.skip("libba.so not built")
    exe = str(tmp_path / "abi_c99")
    libdir = os.path.abspath(LIBDIR)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c", "abi_c99.c"),
           "-L", libdir, "-lba", "-Wl,-rpath," + libdir, "-o", exe]
    build = subprocess.run(cmd, capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stderr
    assert run.stdout.strip() == "ok"
