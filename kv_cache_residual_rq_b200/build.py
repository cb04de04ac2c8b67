"""Build librq.so (the CUDA library) in-tree for sm_100a.

    python -m kv_cache_residual_rq_b200.build [--force]

nvcc compiles every .cu under csrc/ for compute_100a/sm_100a (one process
per file, in parallel) and links them into kv_cache_residual_rq_b200/librq.so
with the CUDA runtime linked statically, so the library loads without a CUDA
toolkit on the path.
"""
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "librq.so")
# the same library with every computed index checked before its access
# (-DRQ_BOUNDS_CHECK; a failed check raises a status bit, nothing traps)
LIB_BOUNDS = os.path.join(HERE, "librq_bounds.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2,-Wall",
    "-Xptxas", "-v",
    "--expt-relaxed-constexpr",
    "-diag-suppress=177",
    "-cudart", "static",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib=LIB):
    if not os.path.exists(lib):
        return True
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) \
        + glob.glob(os.path.join(INCLUDE, "*.h"))
    return max(os.path.getmtime(d) for d in deps) > os.path.getmtime(lib)


def _nvcc():
    nvcc = os.environ.get("NVCC", "nvcc")
    if os.path.exists("/usr/local/cuda/bin/nvcc") and nvcc == "nvcc":
        nvcc = "/usr/local/cuda/bin/nvcc"
    return nvcc


def build(force=False, verbose=False, bounds=False):
    """Compile every translation unit for sm_100a in parallel (one nvcc per
    .cu file), then link them into librq.so (bounds: librq_bounds.so, built
    with -DRQ_BOUNDS_CHECK)."""
    import tempfile
    from concurrent.futures import ThreadPoolExecutor
    lib = LIB_BOUNDS if bounds else LIB
    extra_flags = ("-DRQ_BOUNDS_CHECK",) if bounds else ()
    if not force and not _stale(lib):
        return lib
    nvcc = _nvcc()
    flags = [*NVCC_FLAGS, *extra_flags, "-I", INCLUDE, "-I", CSRC]
    with tempfile.TemporaryDirectory(prefix="rq_build_") as tmp:
        def compile_one(src):
            obj = os.path.join(tmp, os.path.basename(src) + ".o")
            r = subprocess.run([nvcc, *flags, "-c", "-o", obj, src], capture_output=True,
                               text=True)
            return src, obj, r
        srcs = sources()
        with ThreadPoolExecutor(max(1, min(len(srcs), os.cpu_count() or 1))) as ex:
            results = list(ex.map(compile_one, srcs))
        for src, _, r in results:
            if r.returncode != 0:
                sys.stderr.write(r.stdout + r.stderr)
                raise RuntimeError(f"nvcc failed on {os.path.basename(src)}")
            if verbose:
                sys.stderr.write(r.stderr)
        r = subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-cudart",
                            "static", "-shared", "-o", lib + ".tmp",
                            *[obj for _, obj, _ in results]],
                           capture_output=True, text=True)
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError("nvcc failed linking " + os.path.basename(lib))
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                bounds="--bounds" in sys.argv))
