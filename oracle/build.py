"""Compile the CPU oracle (plain C, fp64, OpenMP) into oracle/libkv4_oracle.so.

Test infrastructure: only the tests, the smoke check and the benchmark's
CPU-baseline leg load the result.

Flags: -O3 with AVX2-class code (x86-64-v3, which every current server CPU
runs; the library is built once and may run on another host), and
-ffp-contract=off so that no a*b+c is fused: every fp64 operation of the
oracle rounds as written.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "kv4_oracle.c")
LIB = os.path.join(HERE, "libkv4_oracle.so")
FLAGS = ["-O3", "-march=x86-64-v3", "-ffp-contract=off", "-std=c11", "-fopenmp", "-fPIC"]


def build(force: bool = False) -> str:
    hdr = os.path.join(HERE, "kv4_oracle.h")
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= max(os.path.getmtime(SRC), os.path.getmtime(hdr),
                                             os.path.getmtime(os.path.abspath(__file__)))):
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = ["gcc"] + FLAGS + ["-shared", "-Wall", "-Wextra", "-o", tmp, SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
