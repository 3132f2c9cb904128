"""Build liboq.so (C ABI in include/oq.h) in-tree for sm_100a with nvcc.

Sources: csrc/oq_host.cpp (handles, table builders, launches), csrc/k1_rotquant.cu (fused
rotate + norm + quantize on the CUDA cores), csrc/k1_tc.cu (the same with the block transform
on the tensor cores, bf16 rows), csrc/k2_decode.cu (code -> fp16 prepass), csrc/k2_linear.cu
(tcgen05 GEMM; it decodes 4-bit activation codes itself), csrc/k3_fused.cu (the one-call step
as one persistent kernel).  Objects are compiled
in parallel into calibration_free_bit_b200/_build/ and linked into
calibration_free_bit_b200/liboq.so; the CUDA runtime is linked statically, the driver API is
reached through cudaGetDriverEntryPoint, so the library loads on a machine without a GPU.
"""
import concurrent.futures as cf
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "liboq.so")
INCLUDE = os.path.join(ROOT, "include")
SOURCES = ["oq_host.cpp", "k1_rotquant.cu", "k1_tc.cu", "k2_decode.cu", "k2_linear.cu",
           "k3_fused.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O3",
                "-I" + INCLUDE, "-I" + CSRC]


def _inputs():
    files = [os.path.join(CSRC, s) for s in SOURCES]
    files += [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    files += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
    files.append(os.path.abspath(__file__))
    return files


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in _inputs())


def _compile(src: str) -> str:
    obj = os.path.join(BUILD, os.path.splitext(src)[0] + ".o")
    cmd = ["nvcc"] + FLAGS + ["-c", os.path.join(CSRC, src), "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    return obj


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not needs_build():
        return LIB
    os.makedirs(BUILD, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        objs = list(ex.map(_compile, SOURCES))
    tmp = LIB + ".tmp"
    cmd = ["nvcc"] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + objs
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    if verbose:
        print(f"built {LIB}")
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
