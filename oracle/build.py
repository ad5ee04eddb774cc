"""Compile the C oracle into oracle/liboracle.so (test infrastructure; see oracle/__init__.py).

`mutant` builds a variant with one planted mistake (a -DORACLE_MUTANT_* macro) into a separate
file, so that tests can show the oracle's pins catch it. Only tests use mutants.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "pkv_oracle.c")


def lib_path(mutant: str | None = None) -> str:
    name = "liboracle.so" if not mutant else f"liboracle_{mutant.lower()}.so"
    return os.path.join(HERE, name)


def build(mutant: str | None = None, force: bool = False) -> str:
    out = lib_path(mutant)
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(SRC):
        return out
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-Wall", "-Wextra", SRC, "-o", out + ".tmp", "-lm"]
    if mutant:
        cmd.insert(1, f"-DORACLE_MUTANT_{mutant}")
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(force=True))
