"""Build the CPU oracle shared libraries (TEST INFRASTRUCTURE).

Compiles oracle/qsa_oracle.c twice with gcc: libqsa_oracle.so accumulates in
fp64, libqsa_oracle_f32.so in fp32 (used only to cross-check the first).
-ffp-contract=off keeps the fixed rounding points free of fused multiply-adds.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "qsa_oracle.c")
VARIANTS = {
    "libqsa_oracle.so": [],
    "libqsa_oracle_f32.so": ["-DQSA_ORACLE_ACC_F32"],
}


def lib_path(name="libqsa_oracle.so"):
    return os.path.join(HERE, name)


def build(force=False, verbose=False):
    for name, extra in VARIANTS.items():
        out = lib_path(name)
        if (not force and os.path.exists(out)
                and os.path.getmtime(out) >= max(os.path.getmtime(SRC),
                                                 os.path.getmtime(os.path.join(HERE, "qsa_oracle.h")))):
            continue
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-shared", "-fPIC", "-Wall", "-Wextra", *extra, SRC, "-o", out, "-lm"]
        if verbose:
            print(" ".join(cmd))
        subprocess.run(cmd, check=True)


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
