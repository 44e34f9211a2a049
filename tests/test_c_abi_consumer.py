"""The C ABI from plain C: tests/c_abi/consumer.c includes include/wukong.h, is compiled with
gcc against the built libwukong.so, and calls the entry points that need no GPU (status
strings, argument checks that return before any device call)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_plain_c_consumer(tmp_path):
    from recsys_feature_interaction_b200 import build

    lib = build.build()
    exe = str(tmp_path / "consumer")
    libdir = os.path.dirname(lib)
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                        os.path.join(ROOT, "tests", "c_abi", "consumer.c"), "-o", exe, "-L", libdir, "-lwukong",
                        "-Wl,-rpath," + libdir], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0 and "c abi consumer: ok" in run.stdout, run.stdout + run.stderr
