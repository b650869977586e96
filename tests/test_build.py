"""Concurrent builds of libpa.so (CPU only): every GPU rank of a multi-GPU run calls build(),
so two builders may meet a missing or stale library at the same moment.  They must take turns:
one compiles, the other finds the fresh library under the lock, and the result loads."""
import ctypes
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_SCRIPT = """
import sys, time
sys.path.insert(0, {root!r})
from paged_kv_cache_327_b200 import build
t = time.time()
build.build(lib={lib!r})
print(round(time.time() - t, 1))
"""


def test_two_concurrent_builders_produce_a_loadable_library(tmp_path):
    lib = str(tmp_path / "libpa.so")
    code = _SCRIPT.format(root=ROOT, lib=lib)
    procs = [subprocess.Popen([sys.executable, "-c", code], stdout=subprocess.PIPE, stderr=subprocess.PIPE,
                              text=True) for _ in range(2)]
    outs = [p.communicate(timeout=900) for p in procs]
    for p, (out, err) in zip(procs, outs):
        assert p.returncode == 0, err
    assert os.path.exists(lib)
    # no temporary file is left behind, and the library is whole: it loads and answers
    assert not [f for f in os.listdir(tmp_path) if f.endswith(".tmp")]
    assert ctypes.CDLL(lib).pa_version() == 101
