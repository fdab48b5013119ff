"""Build the in-tree shared libraries for sm_100a with nvcc.

  libdc.so        the serving library (C ABI declared in include/dc.h)
  libdc_synth.so  the device twin of the seeded input generator (test/bench inputs only)

Usage: python -m tenant_mixed_precision_b200.build [--force]
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

LIBS = {
    "libdc.so": {
        "sources": ["dc_host.cpp", "dc_prinmix.cpp", "dc_kernels.cu", "dc_pager.cu", "dc_svd.cu"],
        "headers": ["dc_layout.h", "dc_pack.h", "dc_internal.h", "dc_tma.h", "dc_umma.h", "dc_devstate.h", "dc_lru.h", "dc_btsched.h"],
        "link": ["-lcudart"],
    },
    "libdc_synth.so": {
        "sources": ["synth/synth_gen.cu"],
        "headers": [],
        "link": ["-lcudart"],
    },
}


def _newer(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return False
    t = os.path.getmtime(target)
    return all(os.path.getmtime(d) <= t for d in deps)


def build(force: bool = False, verbose: bool = False) -> list[str]:
    out = []
    for name, spec in LIBS.items():
        target = os.path.join(HERE, name)
        srcs = [os.path.join(CSRC, s) for s in spec["sources"]]
        deps = srcs + [os.path.join(CSRC, h) for h in spec["headers"]] + [os.path.join(INCLUDE, "dc.h"), __file__]
        if not force and _newer(target, deps):
            out.append(target)
            continue
        objs = []
        for src in srcs:
            obj = os.path.join(HERE, "_build", os.path.basename(src) + ".o")
            os.makedirs(os.path.dirname(obj), exist_ok=True)
            cmd = [NVCC, "-std=c++17", "-O3", "-lineinfo", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC, *ARCH,
                   "-c", src, "-o", obj]
            if src.endswith(".cu") and verbose:
                cmd[1:1] = ["-Xptxas", "-v"]
            r = subprocess.run(cmd, capture_output=True, text=True)
            if r.returncode != 0:
                raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
            if verbose and r.stderr:
                sys.stderr.write(r.stderr)
            objs.append(obj)
        cmd = [NVCC, "-shared", *ARCH, "-o", target, *objs, *spec["link"]]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed for {name}:\n{r.stdout}\n{r.stderr}")
        out.append(target)
    return out


if __name__ == "__main__":
    for p in build(force="--force" in sys.argv, verbose="-v" in sys.argv):
        print(p)
