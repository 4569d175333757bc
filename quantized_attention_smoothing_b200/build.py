"""Build libsage.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m quantized_attention_smoothing_b200.build [--force]

Each CUDA translation unit is compiled separately (in parallel) with
``-gencode arch=compute_100a,code=sm_100a -lineinfo -O3 -Xptxas -v``; the
ptxas register / spill report of every kernel goes to ``_build/ptxas.log``.
Only the ``sage_*`` C symbols are exported (linker version script).
"""
import os
import re
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libsage.so")
HEADER = os.path.join(ROOT, "include", "sage.h")

# per-TU extra flags: the quantisation kernels must not contract a*b+c into
# FMAs (their outputs are compared bit for bit)
SOURCES = {
    "quant.cu": ["-fmad=false"],
    "attn_fwd.cu": [],
    "attn_mx.cu": [],
    "decode.cu": [],
    "sage_api.cu": [],
    "probe.cu": [],
}
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ARCH + ["-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-Xptxas", "-v",
                 "-I", os.path.join(ROOT, "include")]


def _nvcc():
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.isabs(c) and os.path.exists(c) or not os.path.isabs(c)):
            return c
    return "nvcc"


def _deps():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [HEADER]
    return max(os.path.getmtime(f) for f in files)


def _compile(src, extra):
    obj = os.path.join(BUILD, src.replace(".cu", ".o"))
    cmd = [_nvcc()] + COMMON + extra + ["-c", os.path.join(CSRC, src), "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    return src, obj, r.returncode, r.stdout + r.stderr


def spills(log_text):
    """(kernel, spill stores, spill loads) for every kernel with spills."""
    out = []
    cur = None
    for line in log_text.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            cur = m.group(1)
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m and cur and (int(m.group(1)) or int(m.group(2))):
            out.append((cur, int(m.group(1)), int(m.group(2))))
    return out


def build(force=False, verbose=False):
    os.makedirs(BUILD, exist_ok=True)
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= _deps():
        return LIB
    with ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        results = list(ex.map(lambda kv: _compile(*kv), SOURCES.items()))
    log = []
    for src, obj, rc, text in results:
        log.append("==== %s\n%s" % (src, text))
        if rc != 0:
            sys.stderr.write(text)
            raise RuntimeError("nvcc failed on %s" % src)
    with open(os.path.join(BUILD, "ptxas.log"), "w") as f:
        f.write("\n".join(log))
    vs = os.path.join(BUILD, "exports.map")
    with open(vs, "w") as f:
        f.write("{ global: sage_*; local: *; };\n")
    tmp = LIB + ".tmp.%d" % os.getpid()
    cmd = [_nvcc()] + ARCH + ["-shared", "-o", tmp] + [r[1] for r in results] + \
        ["-Xlinker", "--version-script=" + vs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("link failed")
    os.replace(tmp, LIB)
    if verbose:
        for k, st, ld in spills("\n".join(log)):
            print("SPILL %s: %d B stores, %d B loads" % (k, st, ld))
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
