"""Build libpa.so (all CUDA kernels for sm_100a plus the host pool) in-tree.

    python paged_kv_cache_452_b200/build.py [--verbose] [--force]

(run by path: importing the package loads libpa.so, which may not exist yet
or may predate the sources)

nvcc compiles each source to an object under _build/ and links them into
paged_kv_cache_452_b200/libpa.so (static CUDA runtime, no libcuda link: the
driver's tensor-map encoder is fetched at run time).
"""
import concurrent.futures as cf
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libpa.so")
SOURCES = ["api.cu", "cache_write.cu", "decode_tc.cu", "attn_simt.cu", "prefill_tc.cu", "prefill_umma.cu", "decode_noalloc.cu", "block_copy.cu", "pool.cpp"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def _flags(verbose):
    f = ARCH + ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2,-Wall",
                "-I", INCLUDE, "-I", CSRC, "--expt-relaxed-constexpr"]
    if verbose:
        f += ["-Xptxas", "-v"]
    return f


def _stale(obj, src):
    if not os.path.exists(obj):
        return True
    deps = [src] + [os.path.join(CSRC, h) for h in os.listdir(CSRC) if h.endswith((".h", ".cuh"))]
    deps.append(os.path.join(INCLUDE, "pa.h"))
    return any(os.path.getmtime(d) > os.path.getmtime(obj) for d in deps)


def _compile(src, verbose, force):
    obj = os.path.join(BUILD, os.path.splitext(src)[0] + ".o")
    path = os.path.join(CSRC, src)
    if not force and not _stale(obj, path):
        return obj, ""
    cmd = [NVCC] + _flags(verbose) + ["-x", "cu" if src.endswith(".cu") else "c++", "-c", path, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    return obj, r.stdout + r.stderr


def build(verbose: bool = False, force: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        results = list(ex.map(lambda s: _compile(s, verbose, force), SOURCES))
    logs = "".join(r[1] for r in results)
    if verbose and logs:
        print(logs)
    objs = [r[0] for r in results]
    if force or not os.path.exists(LIB) or any(os.path.getmtime(o) > os.path.getmtime(LIB) for o in objs):
        cmd = [NVCC] + ARCH + ["-shared", "-o", LIB + ".tmp"] + objs + ["-cudart", "static"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv, force="--force" in sys.argv))
