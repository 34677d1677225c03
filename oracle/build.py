"""Compile the CPU oracle (plain C) into ``oracle/libcsa2_oracle.so``.

Test infrastructure only.  ``-ffp-contract=off`` keeps the compiler from fusing
the score's separate multiplies and adds; the explicit ``fmaf`` calls of the
indexer-K projection stay fused either way.  The vectorised build
(``-mavx2 -mfma``) is used only on CPUs that report both features.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csa2_oracle.c")


def _cpu_has(*flags):
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("flags"):
                    have = set(line.split(":", 1)[1].split())
                    return all(fl in have for fl in flags)
    except OSError:
        pass
    return False


def lib_path():
    name = "libcsa2_oracle_v3.so" if _cpu_has("avx2", "fma") else "libcsa2_oracle.so"
    return os.path.join(HERE, name)


def build(force=False):
    out = lib_path()
    if not force and os.path.exists(out) and os.path.getmtime(out) >= max(
            os.path.getmtime(SRC), os.path.getmtime(os.path.join(HERE, "csa2_oracle.h"))):
        return out
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
           "-Wall", "-Wextra", "-Wno-unused-parameter"]
    if out.endswith("_v3.so"):
        cmd += ["-mavx2", "-mfma"]
    cmd += ["-o", out + ".tmp", SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(force=True))
