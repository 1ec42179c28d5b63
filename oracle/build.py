"""Build the float64 CPU oracle (test infrastructure; never part of the product path).

``python oracle/build.py`` compiles ``ssd_oracle.c`` into ``libssd_oracle.so`` next to it.
``build(mutation=k)`` compiles a deliberately broken variant ``libssd_oracle_mut<k>.so``
that only the pin tests use, to show that each planted mistake fails a pin.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "ssd_oracle.c")


def lib_path(mutation: int = 0) -> str:
    name = "libssd_oracle.so" if mutation == 0 else f"libssd_oracle_mut{mutation}.so"
    return os.path.join(HERE, name)


def build(mutation: int = 0, force: bool = False) -> str:
    out = lib_path(mutation)
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(SRC):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c99", "-Wall",
           f"-DORACLE_MUTATION={mutation}", SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
