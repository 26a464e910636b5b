"""Build libtpconv.so (sm_100a) in-tree.

Steps: compile and run the table generator (host C++), compile every CUDA source
for sm_100a in parallel, link the shared library next to this file.  Re-running only
rebuilds what changed.  Usage: ``python -m equivariant_gnn_tensor_dst_b200.build``.
"""

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libtpconv.so")
# (source, unit defines): the streaming kernels are instantiated once per unit so
# that their many (l_in, l_sh, l_out) specialisations compile in parallel.
_PARTS = {"STATE": 1, "SRC": 2, "RECV": 3, "FWD": 4, "GRADW": 5}


def _units():
    units = [("k_misc.cu", {}), ("k_gemm_tc.cu", {}), ("launch.cu", {}), ("api.cu", {}), ("k_order.cu", {})]
    for kp in (8, 16):
        for mode in (0, 1):   # generic and fast variants of the receiver backward
            units.append(("k_recv_edge.cu", {"TPC_UNIT_KP": kp, "TPC_UNIT_MODE": mode}))
        for mode in (0, 1):
            for part in ("STATE", "SRC"):
                units.append(("k_uvw.cu", {"TPC_UNIT_KP": kp, "TPC_UNIT_MODE": mode, "TPC_UNIT_PART": _PARTS[part]}))
            for part in ("FWD", "GRADW", "SRC"):
                units.append(("k_uvu.cu", {"TPC_UNIT_KP": kp, "TPC_UNIT_MODE": mode, "TPC_UNIT_PART": _PARTS[part]}))
        units.append(("k_uvu.cu", {"TPC_UNIT_KP": kp, "TPC_UNIT_MODE": 0, "TPC_UNIT_PART": _PARTS["RECV"]}))
        # tangents of the receiver backward without (1) and with (2) an A_dot term
        for mode in (1, 2):
            units.append(("k_uvw_dbl.cu", {"TPC_UNIT_KP": kp, "TPC_UNIT_MODE": mode}))
            units.append(("k_uvu_dbl.cu", {"TPC_UNIT_KP": kp, "TPC_UNIT_MODE": mode}))
    return units


def _includes(path, dirs, seen=None):
    """Every local header a source includes, transitively (quoted includes only)."""
    seen = set() if seen is None else seen
    try:
        text = open(path).read()
    except OSError:
        return seen
    for line in text.splitlines():
        line = line.strip()
        if not line.startswith("#include \""):
            continue
        name = line.split('"')[1]
        for d in [os.path.dirname(path)] + dirs:
            cand = os.path.normpath(os.path.join(d, name))
            if os.path.exists(cand):
                if cand not in seen:
                    seen.add(cand)
                    _includes(cand, dirs, seen)
                break
    return seen


ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc():
    cand = os.environ.get("NVCC") or shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    return cand


def _mtime(p):
    return os.path.getmtime(p) if os.path.exists(p) else -1.0


def _run(cmd):
    r = subprocess.run(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)
    if r.returncode != 0:
        raise RuntimeError("command failed: " + " ".join(cmd) + "\n" + r.stdout)
    return r.stdout


def build(verbose=False, jobs=None, extra_flags=()):
    os.makedirs(BUILD, exist_ok=True)
    gen_src = os.path.join(CSRC, "gen_tables.cpp")
    gen_bin = os.path.join(BUILD, "gen_tables")
    tables = os.path.join(BUILD, "tables.inc")
    if _mtime(gen_bin) < _mtime(gen_src):
        _run(["g++", "-O2", "-std=c++17", "-o", gen_bin, gen_src])
    if _mtime(tables) < _mtime(gen_bin):
        _run([gen_bin, tables])
    inc_dirs = [BUILD, CSRC, os.path.join(ROOT, "include")]
    flags = ARCH + ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
                    "-Xcompiler", "-fPIC", "-I", BUILD, "-I", CSRC, "-I", os.path.join(ROOT, "include")]
    flags += list(extra_flags)
    objs = []
    todo = []
    for s, defs in _units():
        src = os.path.join(CSRC, s)
        tag = "_".join(f"{v}" for v in defs.values())
        obj = os.path.join(BUILD, s + (("." + tag) if tag else "") + ".o")
        objs.append(obj)
        deps = _includes(src, inc_dirs)
        if _mtime(obj) < max([_mtime(src)] + [_mtime(h) for h in deps]):
            dflags = [f"-D{k}={v}" for k, v in defs.items()]
            todo.append([_nvcc(), "-c", src, "-o", obj] + flags + dflags)
    # longest compiles (the tangent receiver units) first
    todo.sort(key=lambda c: 0 if "_dbl.cu" in c[2] else 1)
    if todo:
        with cf.ThreadPoolExecutor(max_workers=jobs or min(os.cpu_count() or 8, len(todo))) as ex:
            for out in ex.map(_run, todo):
                if verbose and out.strip():
                    print(out)
    if todo or _mtime(LIB) < max(_mtime(o) for o in objs):
        _run([_nvcc(), "-shared", "-o", LIB] + objs + ARCH + ["-cudart", "static"])
    return LIB


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv))
