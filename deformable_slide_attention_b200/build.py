"""Build libdsa3d.so in-tree with nvcc for sm_100a (B200).

    python -m deformable_slide_attention_b200.build [--debug] [--verbose]

``--debug`` adds the device-side checks (DSA3D_DEBUG) that record failures for
``dsa3d_check_device``; ``--verbose`` prints ptxas register/spill/shared-memory use.
"""
from __future__ import annotations

import argparse
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libdsa3d.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    # the attention's translation unit, and the DWConv3D term's
    return [os.path.join(CSRC, "dsa3d.cu"), os.path.join(CSRC, "dsa3d_conv.cu")]


def _stale(out):
    if not os.path.exists(out):
        return True
    deps = glob.glob(os.path.join(CSRC, "*")) + glob.glob(os.path.join(INCLUDE, "*.h")) + [__file__]
    return os.path.getmtime(out) < max(os.path.getmtime(p) for p in deps)


def build(debug: bool = False, verbose: bool = False, force: bool = False, out: str = LIB) -> str:
    if not force and not _stale(out):
        return out
    cmd = [NVCC, *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
           "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC, "-o", out + ".tmp", *sources()]
    if debug:
        cmd.insert(1, "-DDSA3D_DEBUG")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--debug", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--force", action="store_true")
    args = ap.parse_args(argv)
    print(build(args.debug, args.verbose, args.force or args.debug or args.verbose))


if __name__ == "__main__":
    sys.exit(main())
