"""Build libetp.so in-tree for sm_100a (nvcc cross-compiles; no GPU needed).

    python -m equivariant_mlip_tensor_edge_b200.build [--force]

Object files go to <repo>/_build/; the shared library lands next to this file so that it
travels with the source tree. Rebuilds only when a source is newer than the library.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libetp.so")
SOURCES = ["etp_abi.cu", "etp_graph.cu", "etp_conv.cu", "etp_fwd_tc.cu", "etp_bwd_tc.cu", "etp_noalloc.cu", "etp_dw.cu", "etp_fwd_cx.cu", "etp_ladder_full.cu", "etp_product.cu", "etp_general.cu", "etp_general_tc.cu"]
HEADERS = [os.path.join(ROOT, "include", "etp.h"), os.path.join(CSRC, "etp_internal.h"),
           os.path.join(CSRC, "generated", "etp_paths.h"), os.path.join(CSRC, "etp_device.h"), os.path.join(CSRC, "etp_tc_common.h")]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
         "-Xcompiler", "-fPIC", "-I" + os.path.join(ROOT, "include"), "-I" + CSRC]


def _stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, s) for s in SOURCES] + HEADERS + [os.path.abspath(__file__)]
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src):
    obj = os.path.join(BUILD, src.replace(".cu", ".o"))
    log = os.path.join(BUILD, src.replace(".cu", ".log"))
    cmd = [NVCC, *FLAGS, "-Xptxas", "-v", "-c", os.path.join(CSRC, src), "-o", obj]
    with open(log, "w") as f:
        rc = subprocess.call(cmd, stdout=f, stderr=subprocess.STDOUT)
    if rc != 0:
        raise RuntimeError(f"nvcc failed for {src}; see {log}:\n" + open(log).read()[-4000:])
    return obj


def build(force=False):
    if not force and not _stale():
        return LIB
    os.makedirs(BUILD, exist_ok=True)
    with ThreadPoolExecutor(len(SOURCES)) as ex:
        objs = list(ex.map(_compile, SOURCES))
    tmp = LIB + ".tmp"
    rc = subprocess.call([NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", *objs, "-o", tmp,
                          "-lcudart"])
    if rc != 0:
        raise RuntimeError("link of libetp.so failed")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
