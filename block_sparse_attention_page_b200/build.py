"""Build liblserve.so in place (nvcc, sm_100a only).

    python block_sparse_attention_page_b200/build.py [--force] [--verbose]

(run by path: importing the package loads the library this script builds)

Objects go to block_sparse_attention_page_b200/_build/; the shared library is
written next to this file so that it travels with the source tree.
"""
from __future__ import annotations

import concurrent.futures
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
SOURCES = ["api.cu", "page_stats.cu", "page_select.cu", "decode_attn.cu", "decode_append.cu",
           "prefill.cu", "prefill_to_pages.cu", "select_noalloc.cu",
           "quantize_kv.cu", "seq_shard.cu"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def lib_path() -> str:
    return os.path.join(HERE, "liblserve.so")


def _deps():
    return [os.path.join(CSRC, s) for s in SOURCES] + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(CSRC, "*.h")) + [os.path.join(ROOT, "include", "lserve.h")]


def build(force: bool = False, verbose: bool = False) -> str:
    out = lib_path()
    newest = max(os.path.getmtime(p) for p in _deps())
    if not force and os.path.exists(out) and os.path.getmtime(out) >= newest:
        return out
    bdir = os.path.join(HERE, "_build")
    os.makedirs(bdir, exist_ok=True)
    extra = []
    if verbose:
        extra += ["-Xptxas", "-v"]

    def compile_one(src):
        obj = os.path.join(bdir, src.replace(".cu", ".o"))
        cmd = [NVCC] + FLAGS + extra + ["-c", os.path.join(CSRC, src), "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stderr}")
        return obj, r.stderr

    with concurrent.futures.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        results = list(ex.map(compile_one, SOURCES))
    if verbose:
        for _, err in results:
            sys.stderr.write(err)
    tmp = out + ".tmp"
    cmd = [NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-o", tmp] + \
        [o for o, _ in results]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stderr}")
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
