"""Build libsha_decode.so (the C-ABI CUDA library) in-tree for sm_100a.

    python head_sparse_decode_b200/build.py [--force] [--verbose]
    python head_sparse_decode_b200/build.py --define KNOB=VALUE [...] --output PATH

The second form builds the library with non-default build-time knobs (for
example SHA_MHA_TENSOR_CORES=0) at another path; the binding loads it when
SHA_DECODE_LIBRARY names that path.
"""
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIBRARY = os.path.join(PKG, "libsha_decode.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "--expt-relaxed-constexpr",
    "-Xcompiler", "-fPIC,-O2,-Wall",
]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + [os.path.join(INCLUDE, "sha_decode.h")])


def build(force: bool = False, verbose: bool = False, defines=(), output=None,
          sources=None) -> str:
    """Compile the library unless it is newer than every source file.

    defines: extra -D settings (the kernels' build-time tuning knobs);
    output:  another path for the library (builds with non-default knobs);
    sources: the .cu files of csrc/ to compile (default all of them)."""
    library = output or LIBRARY
    if not force and os.path.exists(library):
        newest = max(os.path.getmtime(p) for p in _sources())
        if os.path.getmtime(library) >= newest:
            return library
    # each .cu is its own translation unit (its kernels are launched from it),
    # so the objects compile side by side and link without relocatable device code
    cmd = [NVCC, *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, *[f"-D{d}" for d in defines]]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")) if sources is None
                     else [os.path.join(CSRC, name) for name in sources])
    objects = [f"{library}.{os.path.basename(src)}.o" for src in sources]
    procs = [subprocess.Popen(cmd + ["-c", "-o", obj, src]) for src, obj in zip(sources, objects)]
    failed = [src for src, proc in zip(sources, procs) if proc.wait() != 0]
    try:
        if failed:
            raise subprocess.CalledProcessError(1, failed)
        subprocess.run([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared",
                        "-o", library + ".tmp", *objects], check=True)
    finally:
        for obj in objects:
            if os.path.exists(obj):
                os.remove(obj)
    os.replace(library + ".tmp", library)
    return library


# The decode library with test hooks (a pipeline wait limit the tests can
# lower, see sha_test_set_wait_limit); only the tests load it.
TEST_HOOKS_LIBRARY = os.path.join(PKG, "libsha_decode_test_hooks.so")


def build_test_hooks(force: bool = False) -> str:
    return build(force=force, defines=("SHA_TEST_HOOKS=1",), output=TEST_HOOKS_LIBRARY)


if __name__ == "__main__":
    import argparse
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--define", action="append", default=[])
    ap.add_argument("--output")
    a = ap.parse_args()
    if a.define or a.output:
        print(build(force=True, verbose=a.verbose, defines=a.define, output=a.output))
    else:
        print(build(force=a.force, verbose=a.verbose))
        print(build_test_hooks(force=a.force))
