"""Builds the CUDA library (liblsq.so) in-tree for sm_100a with nvcc.

    python -m layer_streamed_qlora_nf4_b200.build [--force] [--ptxas]
    python -m layer_streamed_qlora_nf4_b200.build --define LSQ_GEMM_KTL --out /tmp/liblsq_ktl.so

Every translation unit under csrc/ is compiled with
``-gencode arch=compute_100a,code=sm_100a -O3 -lineinfo`` and linked into one
shared library next to this file (the CUDA runtime is linked statically, so the
library loads with or without torch).  Rebuilds only when a source is newer.

``--define NAME`` (repeatable) compiles a diagnostic variant: LSQ_GEMM_STAMPS
(per-CTA phase stamps of the fused GEMM) or LSQ_GEMM_KTL (its per-k-tile timeline
of every role).  A variant needs ``--out``: it is built from its own object folder
into that path and never replaces the library above.
"""
import concurrent.futures as cf
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "liblsq.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2",
                "-I", INCLUDE, "-I", CSRC, "--expt-relaxed-constexpr"]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(INCLUDE, "*.h")))


def _newest(paths):
    return max((os.path.getmtime(p) for p in paths), default=0.0)


def _compile(src, extra, build_dir=BUILD):
    obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
    hdr_t = _newest(_headers())
    if os.path.exists(obj) and os.path.getmtime(obj) >= max(os.path.getmtime(src), hdr_t):
        return obj, ""
    cmd = [NVCC] + FLAGS + extra + ["-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed for %s:\n%s\n%s" % (src, " ".join(cmd), r.stderr))
    return obj, r.stderr


def build(force=False, verbose=False, ptxas_info=False, defines=(), out=None):
    if defines and not out:
        raise ValueError("a diagnostic variant (defines) needs its own output path")
    lib = os.path.abspath(out) if out else LIB
    build_dir = BUILD if not defines else BUILD + "_" + "_".join(sorted(defines)).lower()
    os.makedirs(build_dir, exist_ok=True)
    srcs = _sources()
    if force:
        for o in glob.glob(os.path.join(build_dir, "*.o")):
            os.remove(o)
    extra = (["-Xptxas", "-v"] if ptxas_info else []) + ["-D" + d for d in defines]
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 4)) as ex:
        results = list(ex.map(lambda s: _compile(s, extra, build_dir), srcs))
    objs = [o for o, _ in results]
    if verbose:
        for _, log in results:
            if log:
                sys.stderr.write(log)
    if force or not os.path.exists(lib) or os.path.getmtime(lib) < _newest(objs):
        cmd = [NVCC] + ARCH + ["-shared", "-o", lib] + objs + ["-lcuda", "-ldl"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("link failed:\n%s\n%s" % (" ".join(cmd), r.stderr))
    return lib


if __name__ == "__main__":
    argv = sys.argv[1:]
    defs = [argv[i + 1] for i, a in enumerate(argv[:-1]) if a == "--define"]
    outs = [argv[i + 1] for i, a in enumerate(argv[:-1]) if a == "--out"]
    print(build(force="--force" in argv, verbose=True, ptxas_info="--ptxas" in argv,
                defines=defs, out=outs[-1] if outs else None))
