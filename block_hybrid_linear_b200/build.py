"""Build ``libbha.so`` (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m block_hybrid_linear_b200.build [--force] [--ptxas-verbose]

The CUDA runtime is linked statically and the driver's tensor-map encoder is
fetched at run time, so the library loads on a machine without a GPU driver
(its compute calls then report BHA_ERR_CUDA).
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libbha.so")
SOURCES = ["bha_api.cu", "k_f32.cu", "k_step.cu", "k_state.cu", "k_prefix.cu", "k_reuse.cu",
           "bha_noalloc.cu"]
HEADERS = ["bha_internal.h", "bha_ptx.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc():
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(INCLUDE, "bha.h"))
    return any(os.path.getmtime(p) > t for p in deps)


def build(force=False, verbose_ptxas=False):
    """Compile every CUDA source into libbha.so (skipped when up to date)."""
    if not force and not _stale():
        return LIB
    objs = []
    build_dir = os.path.join(HERE, "_build")
    os.makedirs(build_dir, exist_ok=True)
    flags = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
                    "--expt-relaxed-constexpr", "-I" + INCLUDE, "-I" + CSRC]
    if verbose_ptxas:
        flags += ["-Xptxas", "-v"]
    procs = []
    for src in SOURCES:
        obj = os.path.join(build_dir, src.replace(".cu", ".o"))
        objs.append(obj)
        cmd = [_nvcc()] + flags + ["-c", os.path.join(CSRC, src), "-o", obj]
        procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE,
                                            stderr=subprocess.STDOUT)))
    failed = []
    for src, p in procs:
        out, _ = p.communicate()
        if out and (p.returncode != 0 or verbose_ptxas):
            sys.stderr.write(out.decode(errors="replace"))
        if p.returncode != 0:
            failed.append(src)
    if failed:
        raise RuntimeError("nvcc failed for: " + ", ".join(failed))
    tmp = LIB + ".tmp%d" % os.getpid()
    subprocess.run([_nvcc()] + ARCH + ["-shared", "-o", tmp] + objs, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose_ptxas="--ptxas-verbose" in sys.argv)
    print(LIB)
