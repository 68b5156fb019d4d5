"""Build step for libselscan (sm_100a) and the seeded-input generator.

``build()`` compiles ``csrc/selscan.cu`` with nvcc for sm_100a only into
``libselscan.so`` next to this file (in-tree, so it travels with the source
tree), and ``gen/ssgen.c`` with gcc.  Rebuilds only when a source is newer
than the library, unless ``force``.
"""
import concurrent.futures
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libselscan.so")

BUILD_DIR = os.path.join(HERE, "_build")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC",
]

# (input type, output type, name part) x state bucket: one translation unit each.
DTYPE_PAIRS = [("float", "float", "f32_f32"), ("__nv_bfloat16", "__nv_bfloat16", "bf16_bf16"),
               ("__nv_bfloat16", "float", "bf16_f32")]
STATE_BUCKETS = [4, 8, 16, 32, 64]
BWD_STATE_BUCKETS = [4, 8, 16, 32, 64]  # the backward holds 4 states per lane


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _sources():
    return (glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
            glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h")))


def _compile_jobs(verbose: bool):
    base = [_nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, "-c"]
    if verbose:
        base += ["-Xptxas", "-v"]
    jobs = [(base + [os.path.join(CSRC, "selscan.cu"), "-o",
                     os.path.join(BUILD_DIR, "selscan.o")], "selscan"),
            (base + [os.path.join(CSRC, "ss_noalloc.cu"), "-o",
                     os.path.join(BUILD_DIR, "ss_noalloc.o")], "ss_noalloc")]
    for tin, tout, tag in DTYPE_PAIRS:
        for n in BWD_STATE_BUCKETS:
            name = f"bwd_{tag}_n{n}"
            jobs.append((base + [f"-DSS_INST_TIN={tin}", f"-DSS_INST_TOUT={tout}",
                                 f"-DSS_INST_NMAX={n}", f"-DSS_INST_NAME={name}",
                                 os.path.join(CSRC, "ss_bwd_inst.cu"), "-o",
                                 os.path.join(BUILD_DIR, name + ".o")], name))
    for tin, tout, tag in DTYPE_PAIRS:
        for n in STATE_BUCKETS:
            name = f"launch_{tag}_n{n}"
            jobs.append((base + [f"-DSS_INST_TIN={tin}", f"-DSS_INST_TOUT={tout}",
                                 f"-DSS_INST_NMAX={n}", f"-DSS_INST_NAME={name}",
                                 os.path.join(CSRC, "ss_fwd_inst.cu"), "-o",
                                 os.path.join(BUILD_DIR, name + ".o")], name))
    return jobs


def build_selscan(force: bool = False, verbose: bool = False, jobs: int = 0) -> str:
    newest = max(os.path.getmtime(s) for s in _sources())
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= newest:
        return LIB
    os.makedirs(BUILD_DIR, exist_ok=True)
    todo = _compile_jobs(verbose)
    workers = jobs or min(len(todo), os.cpu_count() or 4)

    def run(job):
        cmd, name = job
        r = subprocess.run(cmd, capture_output=True, text=True)
        return name, r

    failed = []
    with concurrent.futures.ThreadPoolExecutor(workers) as ex:
        for name, r in ex.map(run, todo):
            if verbose or r.returncode != 0:
                sys.stderr.write(r.stdout + r.stderr)
            if r.returncode != 0:
                failed.append(name)
    if failed:
        raise RuntimeError("nvcc failed for: " + ", ".join(failed))
    objs = [cmd[cmd.index("-o") + 1] for cmd, _ in todo]
    subprocess.run([_nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", *objs,
                    "-o", LIB + ".tmp"], check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


def build(force: bool = False, verbose: bool = False) -> None:
    from . import gen
    gen.build(force=force)
    build_selscan(force=force, verbose=verbose)


if __name__ == "__main__":
    sys.path.insert(0, ROOT)
    from selective_state_space_41_b200 import build as _b
    _b.build(force=True, verbose="-v" in sys.argv)
    print(LIB)
