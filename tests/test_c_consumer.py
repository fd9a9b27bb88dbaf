"""The boundary is a C ABI: a C99 program compiles against include/fg.h
(strict warnings as errors), links libfg.so and calls the entry points that
need no GPU."""
import os
import shutil
import subprocess

import pytest

from ragged_paged_kv_b200 import fg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c99_consumer_builds_and_runs(tmp_path):
    fg.lib()  # the library is built
    exe = tmp_path / "consumer"
    libdir = os.path.dirname(fg.LIB_PATH)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "consumer.c"), "-L", libdir, "-lfg", f"-Wl,-rpath,{libdir}",
           "-o", str(exe)]
    out = subprocess.run(cmd, capture_output=True, text=True)
    assert out.returncode == 0, out.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stderr
    assert run.stdout.strip() == "ok"
