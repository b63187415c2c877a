"""Compile the float64 CPU oracle (test infrastructure) into a shared library.

Only the test suite, the smoke check and the bench's CPU-baseline leg load the
result; building it is part of building the checker, not the product.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(HERE, "lightning_oracle.c")
LIBRARY = os.path.join(HERE, "liblightning_oracle.so")


def build(force: bool = False) -> str:
    """Compile lightning_oracle.c with OpenMP; return the library path."""
    if (not force and os.path.exists(LIBRARY)
            and os.path.getmtime(LIBRARY) >= os.path.getmtime(SOURCE)):
        return LIBRARY
    tmp = LIBRARY + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-o", tmp, SOURCE, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIBRARY)
    return LIBRARY


if __name__ == "__main__":
    print(build(force=True))
