"""Compile the oracle's plain-C float64 Oja loop (test infrastructure)."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))


def build(force: bool = False) -> str:
    src = os.path.join(HERE, "oja_ref.c")
    out = os.path.join(HERE, "_oja_ref.so")
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    tmp = out + ".tmp"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC",
                           "-o", tmp, src, "-lm"])
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force=True))
