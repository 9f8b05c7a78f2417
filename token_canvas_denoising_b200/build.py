"""Builds libdgcanvas.so in-tree with nvcc for sm_100a.

    python -m token_canvas_denoising_b200.build [--force] [-v]

Each .cu under csrc/ is compiled to an object and the objects are linked into
a shared library next to this file. An object is rebuilt unless the hash
recorded beside it equals the hash of its source, every header and the
compiler command (file times are not trusted: a copied tree can carry
objects newer than their sources); the library is relinked whenever an object
was rebuilt or the recorded hash of the object set differs. The CUDA runtime
is linked statically.
"""
import argparse
import glob
import hashlib
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libdgcanvas.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2",
              "-Xptxas", "-O3", "--expt-relaxed-constexpr"]


def nvcc():
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found")
    return path


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h")))


def _digest(paths, extra):
    h = hashlib.sha256()
    for p in paths:
        with open(p, "rb") as f:
            h.update(os.path.relpath(p, ROOT).encode() + b"\0" + f.read())
    h.update(" ".join(os.path.relpath(x, ROOT) if os.path.isabs(x) else x for x in extra).encode())
    return h.hexdigest()


def _recorded(path):
    try:
        with open(path) as f:
            return f.read().strip()
    except OSError:
        return None


def build(force=False, verbose=False, jobs=None):
    os.makedirs(BUILD, exist_ok=True)
    hdrs = headers()
    objs, cmds, stamps = [], [], []
    for src in sources():
        obj = os.path.join(BUILD, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        cmd = [nvcc(), *ARCH, *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj]
        digest = _digest([src] + hdrs, cmd[1:])
        if force or not os.path.exists(obj) or _recorded(obj + ".sha256") != digest:
            cmds.append(cmd)
            stamps.append((obj + ".sha256", digest))
    procs = []
    for cmd in cmds:
        if verbose:
            print(" ".join(cmd), flush=True)
        procs.append((cmd, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)))
    failed = []
    for cmd, p in procs:
        out, _ = p.communicate()
        text = out.decode(errors="replace")
        if p.returncode != 0:
            failed.append((cmd[-3], text))
        elif verbose and text.strip():
            print(text)
    if failed:
        msg = "\n".join(f"--- {src}\n{txt}" for src, txt in failed)
        raise RuntimeError("nvcc failed:\n" + msg)
    for path, digest in stamps:
        with open(path, "w") as f:
            f.write(digest + "\n")
    link = [nvcc(), *ARCH, "-shared", "-o", LIB, *objs, "-cudart", "static"]
    lib_digest = _digest(objs, link[1:])
    if cmds or force or not os.path.exists(LIB) or _recorded(LIB + ".sha256") != lib_digest:
        if verbose:
            print(" ".join(link), flush=True)
        r = subprocess.run(link, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)
        if r.returncode != 0:
            raise RuntimeError("link failed:\n" + r.stdout.decode(errors="replace"))
        with open(LIB + ".sha256", "w") as f:
            f.write(lib_digest + "\n")
    return LIB


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))


if __name__ == "__main__":
    sys.exit(main())
