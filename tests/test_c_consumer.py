"""The C ABI from C: tests/c_consumer.c includes include/pa.h, links libpa.so and calls the
host-side entry points (CPU only: no GPU call is made)."""
import os
import shutil
import subprocess

import pytest

from paged_kv_cache_327_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_links_and_runs(tmp_path):
    lib = build.build()
    exe = tmp_path / "c_consumer"
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_consumer.c"), "-o", str(exe), "-L", os.path.dirname(lib),
                    "-l:libpa.so", f"-Wl,-rpath,{os.path.dirname(lib)}"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
