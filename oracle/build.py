"""Build the CPU oracle (test infrastructure) into oracle/liboracle.so.

Plain gcc, IEEE binary32 arithmetic: no fused multiply-add contraction and no
fast-math, so that each float operation in the oracle is one correctly
rounded operation.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "fp4_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

FLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-ffp-contract=off",
         "-fno-fast-math", "-fexcess-precision=standard", "-Wall", "-Wextra"]


def compile_to(src: str, out: str) -> str:
    """Compile an oracle source file with the oracle's flags."""
    subprocess.run(["gcc", *FLAGS, "-o", out, src, "-lm"], check=True)
    return out


def build(force: bool = False) -> str:
    # The mutation test points this at a deliberately broken copy of the
    # oracle, compiled by compile_to, to check that the pins catch it.
    override = os.environ.get("FP4_ORACLE_LIB")
    if override:
        return override
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    return compile_to(SRC, LIB)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
