"""Build libfs4.so (the sm_100a kernels and the C ABI of include/fs4.h) in-tree with nvcc."""
from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIBDIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIBDIR, "libfs4.so")
SOURCES = ["kernels.cu", "gemm.cu", "momentum.cu", "api.cu", "noalloc.cu"]
NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-O3",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return "nvcc"


def build(verbose: bool = False, ptxas_info: bool = False) -> str:
    """Compile every CUDA source for sm_100a and link libfs4.so; returns its path."""
    os.makedirs(LIBDIR, exist_ok=True)
    inc = ["-I", os.path.join(ROOT, "include"), "-I", CSRC]
    extra = ["-Xptxas", "-v"] if ptxas_info else []

    def compile_one(src: str) -> str:
        obj = os.path.join(LIBDIR, src.replace(".cu", ".o"))
        cmd = [nvcc(), *NVCC_FLAGS, *extra, *inc, "-c", os.path.join(CSRC, src), "-o", obj]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{res.stderr}")
        if verbose or ptxas_info:
            sys.stderr.write(res.stderr)
        return obj

    with ThreadPoolExecutor(len(SOURCES)) as ex:
        objs = list(ex.map(compile_one, SOURCES))
    cmd = [nvcc(), "-shared", "-gencode", "arch=compute_100a,code=sm_100a", *objs, "-o", LIB]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"link failed:\n{res.stderr}")
    return LIB


def source_digest() -> str:
    """Short hash of every file under csrc/ (ties a stored resource report to its sources)."""
    import hashlib
    h = hashlib.sha256()
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cuh", ".h")):
            with open(os.path.join(CSRC, name), "rb") as f:
                h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


_OPT_TAGS = ((1, "H16r"), (2, "4/6"), (16, "BF16"), (32, "wide-K"))
_EPI = {"0": "Plain", "1": "GramX", "2": "GramA", "3": "Update"}


def _kernel_name(demangled: str) -> str:
    """A short readable kernel name: no namespaces or argument list; GEMM variants as
    nvfp4_gemm_kernel<Epilogue> plus their option tags."""
    import re
    n = demangled.replace("fs4::(anonymous namespace)::", "").replace("fs4::", "")
    n = re.sub(r"^void ", "", n)
    n = n[:n.rfind("(")] if n.endswith(")") else n
    n = re.sub(r"\(Epi\)(\d)", lambda m: _EPI[m.group(1)], n)
    m = re.match(r"nvfp4_gemm_kernel<(\w+), (\d+)u>$", n)
    if m:
        o = int(m.group(2))
        tags = [t for b, t in _OPT_TAGS if o & b] or ["plain"]
        n = f"nvfp4_gemm_kernel<{m.group(1)}> {'+'.join(tags)}"
    return n


def ptxas_table() -> str:
    """Build with -Xptxas -v and return a markdown table of every kernel's registers,
    spills, stack, static shared memory and barriers, sorted by name."""
    import contextlib
    import io
    import re
    err = io.StringIO()
    with contextlib.redirect_stderr(err):
        build(ptxas_info=True)
    rows, cur = [], None
    for ln in err.getvalue().splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", ln)
        if m:
            cur = {"mangled": m.group(1)}
            rows.append(cur)
            continue
        if cur is None:
            continue
        m = re.search(r"(\d+) bytes stack frame, (\d+) bytes spill stores, (\d+) bytes spill loads", ln)
        if m:
            cur["stack"], cur["st"], cur["ld"] = map(int, m.groups())
        m = re.search(r"Used (\d+) registers(?:, used (\d+) barriers)?(?:, (\d+) bytes smem)?", ln)
        if m:
            cur["regs"], cur["bars"], cur["smem"] = int(m.group(1)), int(m.group(2) or 0), int(m.group(3) or 0)
    demangled = subprocess.run(["c++filt"], input="\n".join(r["mangled"] for r in rows),
                               capture_output=True, text=True, check=True).stdout.splitlines()
    for r, d in zip(rows, demangled):
        r["name"] = _kernel_name(d)
    rows.sort(key=lambda r: r["name"])
    out = ["| kernel | registers | spill stores / loads (B) | stack (B) | static smem (B) | barriers |",
           "|---|---|---|---|---|---|"]
    for r in rows:
        out.append(f"| `{r['name']}` | {r['regs']} | {r['st']} / {r['ld']} | {r['stack']} | {r['smem']} | "
                   f"{r['bars']} |")
    out.append("")
    out.append(f"{len(rows)} kernels; CUDA source digest {source_digest()}")
    return "\n".join(out)


if __name__ == "__main__":
    if "--ptxas-table" in sys.argv:
        print(ptxas_table())
    else:
        print(build(verbose="-v" in sys.argv, ptxas_info="--ptxas" in sys.argv))
