"""Compile the fp64 CPU oracle (``pa_oracle.c``) into ``libpa_oracle.so``.

Test infrastructure: the oracle is only loaded by the tests, by the package's
``smoke()`` check and by the bench's CPU-baseline / reference arm.
"""
import fcntl
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "pa_oracle.c")
LIB = os.path.join(HERE, "libpa_oracle.so")


def build(src: str = SRC, out: str = LIB, extra_flags=()) -> str:
    """Build the oracle library with gcc (plain C11, -O2, POSIX threads).

    Concurrent builders take turns under a file lock beside the output and write through a
    temporary file of their own, so a process never loads a half-written library."""
    def fresh():
        return os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src) and not extra_flags

    if fresh():
        return out
    with open(out + ".lock", "w") as lock:
        fcntl.flock(lock, fcntl.LOCK_EX)
        if fresh():
            return out
        tmp = f"{out}.{os.getpid()}.tmp"
        cmd = ["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-pthread", "-D_GNU_SOURCE",
               *extra_flags, src, "-o", tmp, "-lm"]
        try:
            subprocess.run(cmd, check=True)
            os.replace(tmp, out)
        finally:
            if os.path.exists(tmp):
                os.unlink(tmp)
    return out


if __name__ == "__main__":
    print(build())
