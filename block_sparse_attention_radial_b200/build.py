"""Build libbsa.so in-tree with nvcc for sm_100a.

    python -m block_sparse_attention_radial_b200.build [--verbose]
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SOURCES = [os.path.join(HERE, "csrc", name)
           for name in ("libbsa.cu", "module.cu", "host_pipeline.cu")]
OUTPUT = os.path.join(HERE, "libbsa.so")
GENCODE = "arch=compute_100a,code=sm_100a"


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def build(verbose: bool = False, output: str = OUTPUT) -> str:
    cmd = [nvcc_path(), "-gencode", GENCODE, "-lineinfo", "-O3", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-I", os.path.join(ROOT, "include"),
           "-o", output + ".tmp"] + SOURCES
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(output + ".tmp", output)
    return output


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv))
