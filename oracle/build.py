"""Build the CPU oracle (plain C) into a shared library next to its source.

Test infrastructure: the library built here is loaded only by the tests, the
smoke check and the benchmark's CPU-baseline leg.

    python oracle/build.py            # -> oracle/libhyb_oracle.so
    build(mutant=3, out=...)          # a variant with one planted mistake
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "hyb_oracle.c")
DEFAULT_OUT = os.path.join(HERE, "libhyb_oracle.so")


def build(mutant: int = 0, out: str = DEFAULT_OUT, force: bool = False) -> str:
    """Compile hyb_oracle.c with gcc; returns the path of the .so."""
    deps = [SRC, os.path.join(HERE, "hyb_oracle.h")]
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= max(os.path.getmtime(d) for d in deps)):
        return out
    cmd = ["gcc", "-O2", "-std=c99", "-Wall", "-Wextra", "-fPIC", "-shared",
           f"-DORACLE_MUTANT={int(mutant)}", SRC, "-o", out + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
