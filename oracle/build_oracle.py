"""Build the C++ oracle (oracle/dsa_oracle.cpp) into oracle/libdsa_oracle.so with
the host's g++: plain -O2, no fast-math, no architecture-specific flags.

    python -m oracle.build_oracle

Test infrastructure only (see oracle/dsa_oracle.cpp)."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "dsa_oracle.cpp")
LIB = os.path.join(HERE, "libdsa_oracle.so")
CXX = os.environ.get("CXX", "g++")


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + ".%d.tmp" % os.getpid()
        cmd = [CXX, "-O2", "-std=c++17", "-Wall", "-shared", "-fPIC", "-pthread", SRC, "-o", tmp]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("oracle build failed:\n" + r.stderr)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
