"""Build step for the fp64 CPU oracle (test infrastructure only).

Compiles oracle.c into liboracle.so beside it with plain gcc: -O2, OpenMP
over tokens, no fast-math and no floating-point contraction, so every
multiply and add rounds exactly as written in the source.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(HERE, "oracle.c")
LIBRARY = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if (not force and os.path.exists(LIBRARY)
            and os.path.getmtime(LIBRARY) >= os.path.getmtime(SOURCE)):
        return LIBRARY
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-fno-fast-math", "-Wall", "-Wextra",
           SOURCE, "-o", LIBRARY + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(LIBRARY + ".tmp", LIBRARY)
    return LIBRARY


def build_variant(source_text: str, out_path: str) -> str:
    """Compile a modified copy of the oracle source (used by the tests that
    plant a mistake in the oracle to show the pins catch it)."""
    src = out_path + ".c"
    with open(src, "w") as f:
        f.write(source_text)
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-fno-fast-math", src, "-o", out_path, "-lm"]
    subprocess.run(cmd, check=True)
    return out_path


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
