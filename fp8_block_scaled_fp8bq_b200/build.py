"""Build libfp8bq.so (the C-ABI library) in-tree with nvcc for sm_100a.

Every .cu file under csrc/ is compiled separately (in parallel) with
``-gencode arch=compute_100a,code=sm_100a -lineinfo -O3``, IEEE-exact float
settings (no fast math: division and denormals as IEEE-754 requires), and
linked into fp8_block_scaled_fp8bq_b200/libfp8bq.so against the static CUDA
runtime.  ``-Xptxas -v`` output (registers, spills, shared memory) goes to
_build/ptxas.log.
"""
import concurrent.futures as cf
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libfp8bq.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-ftz=false", "-prec-div=true", "-prec-sqrt=true",
                "-fmad=true", "-Xcompiler", "-fPIC,-fvisibility=hidden", "-Xptxas", "-v",
                "-I" + os.path.join(ROOT, "include"), "--expt-relaxed-constexpr"]


# Kernels that split registers between warpgroups with setmaxnreg: the launch
# register count ptxas reports must equal the count the split assumes.
SETMAXNREG_KERNELS = {"gemm_promote_kernel": 168, "decode_kernel": 168, "gemm_pair_kernel": 168,
                      "gemm_native_kernel": 168, "prefill_attn_kernel": 168}


def _check_registers(log_text):
    import re
    current = None
    for line in log_text.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            current = m.group(1)
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and current:
            for name, want in SETMAXNREG_KERNELS.items():
                if name in current and int(m.group(1)) != want:
                    raise RuntimeError("%s: ptxas used %s registers, the setmaxnreg split assumes %d"
                                       % (name, m.group(1), want))


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        [os.path.join(ROOT, "include", "fp8bq.h"), os.path.abspath(__file__)]


def _stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in _deps())


def _compile(src):
    obj = os.path.join(BUILD, os.path.basename(src) + ".o")
    r = subprocess.run([NVCC, *FLAGS, "-c", src, "-o", obj], capture_output=True, text=True)
    return src, obj, r


def build(force=False, verbose=False):
    """Compile libfp8bq.so if missing or stale; return its path."""
    if not force and not _stale():
        return LIB
    os.makedirs(BUILD, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 4)) as ex:
        results = list(ex.map(_compile, _sources()))
    log = []
    objs = []
    for src, obj, r in results:
        log.append("== %s\n%s%s" % (os.path.basename(src), r.stdout, r.stderr))
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError("nvcc failed on %s" % src)
        objs.append(obj)
    with open(os.path.join(BUILD, "ptxas.log"), "w") as f:
        f.write("\n".join(log))
    _check_registers("\n".join(log))
    tmp = LIB + ".tmp%d" % os.getpid()
    r = subprocess.run([NVCC, *ARCH, "-shared", "-Xcompiler", "-fPIC", *objs, "-o", tmp,
                        "-cudart", "static"], capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("link of libfp8bq.so failed")
    os.replace(tmp, LIB)
    if verbose:
        print("\n".join(log))
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
