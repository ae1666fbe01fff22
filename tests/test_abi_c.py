"""The C ABI from C: tests/abi_check.c includes include/wall.h as plain C99,
takes the address of every entry point (so the link resolves each one
against libwall.so) and calls the host-side checks, which answer without a
GPU."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "channel_decay_softmax_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_compiles_as_c_and_links(tmp_path):
    from channel_decay_softmax_b200 import build
    build.build()
    exe = tmp_path / "abi_check"
    cc = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
          os.path.join(ROOT, "tests", "abi_check.c"), "-L", PKG, "-lwall",
          "-Wl,-rpath," + PKG, "-o", str(exe)]
    res = subprocess.run(cc, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr[-4000:]
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    # the C caller names every entry point the header declares
    from tests.test_abi import _declared
    names = _declared()
    src = open(os.path.join(ROOT, "tests", "abi_check.c")).read()
    missing = [n for n in names if f"(any_fn){n}," not in src and f"(any_fn){n}\n" not in src]
    assert not missing, missing
    assert f"abi_check: ok ({len(names)} entry points)" in run.stdout
