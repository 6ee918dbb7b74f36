"""Build libiq.so in-tree (nvcc, sm_100a).  Usage: python -m rotated_bit_kv_iq_b200.build [-v]"""

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libiq.so")
CUDA_SOURCES = ["iq_api.cu", "iq_encode.cu", "iq_decode.cu", "iq_export.cu", "iq_noalloc.cu", "iq_deferred.cu",
                # decode kernels, one unit per (K bits, V bits) pair
                "iq_decode_k2v2.cu", "iq_decode_k3v2.cu", "iq_decode_k3v3.cu", "iq_decode_k4v2.cu",
                "iq_decode_k4v3.cu", "iq_decode_k4v4.cu"]
HOST_SOURCES = ["iq_host.cpp"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc():
    for cand in [os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"]:
        if cand and (os.path.isfile(cand) or cand == "nvcc"):
            return cand
    return "nvcc"


def _newest_source_mtime():
    paths = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    paths.append(os.path.join(HERE, "..", "include", "iq.h"))
    paths.append(os.path.abspath(__file__))
    return max(os.path.getmtime(p) for p in paths if os.path.exists(p))


def build(verbose=False, force=False):
    """Compile every source into libiq.so unless it is newer than all sources."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= _newest_source_mtime():
        return LIB
    nvcc = _nvcc()
    bdir = os.path.join(HERE, "_build")
    os.makedirs(bdir, exist_ok=True)
    common = ["-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-I", CSRC, "-I", os.path.join(HERE, "..", "include")]
    jobs = []
    for src in CUDA_SOURCES:
        obj = os.path.join(bdir, src + ".o")
        cmd = [nvcc, *ARCH, "-lineinfo", *common, "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            cmd += ["-Xptxas", "-v"]
        jobs.append((cmd, obj))
    for src in HOST_SOURCES:
        obj = os.path.join(bdir, src + ".o")
        # host PRNG: IEEE double arithmetic without contraction (bit-reproducible parameters)
        cmd = [nvcc, *common, "-Wno-deprecated-gpu-targets", "-Xcompiler", "-ffp-contract=off", "-x", "c++", "-c",
               os.path.join(CSRC, src), "-o", obj]
        jobs.append((cmd, obj))
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        for f in [ex.submit(subprocess.run, cmd, check=True) for cmd, _ in jobs]:
            f.result()
    objs = [obj for _, obj in jobs]
    tmp = LIB + ".tmp"
    subprocess.run([nvcc, *ARCH, "-shared", "-o", tmp, *objs, "-lcudart"], check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, force=True))
