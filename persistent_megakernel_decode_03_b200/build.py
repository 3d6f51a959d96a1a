"""Builds libmk.so (the C-ABI library with the sm_100a megakernel) in place."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmk.so")
SOURCES = ["api.cu", "megakernel.cu", "graph.cpp", "noalloc.cu"]
HEADERS = ["mk_internal.h", "graph.h", "megakernel.h"]


def nvcc_cmd(ptxas_verbose: bool = False):
    cmd = ["nvcc", "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
           "-maxrregcount=200",
           "-Xcompiler", "-fPIC", "-shared", "-I", os.path.join(HERE, "..", "include")]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES] + ["-o", LIB]
    return cmd


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(HERE, "..", "include", "mk.h"))
    return any(os.path.getmtime(d) > t for d in deps)


MIN_LAUNCH_REGS = 168   # kMinLaunchRegs in csrc/mk_internal.h (setmaxnreg budget)


def build(verbose: bool = False, ptxas_verbose: bool = False) -> str:
    cmd = nvcc_cmd(True)
    if verbose:
        print(" ".join(cmd))
    out = subprocess.run(cmd, capture_output=True, text=True)
    log = out.stdout + out.stderr
    if out.returncode != 0:
        errs = [ln for ln in log.splitlines() if "ptxas info" not in ln and "bytes stack frame" not in ln]
        raise RuntimeError("nvcc failed:\n" + "\n".join(errs[-60:]))
    if ptxas_verbose:
        print(log)
    # The megakernel re-splits its registers between warpgroups at run time
    # (setmaxnreg); that split is only valid if every instantiation launches with
    # at least MIN_LAUNCH_REGS registers per thread.
    import re
    cur = None
    for line in log.splitlines():
        m = re.search(r"Compiling entry function '(\S+)'", line)
        if m:
            cur = m.group(1)
        m = re.search(r"Used (\d+) registers", line)
        # (megakernel<HPG, DPL, MM, WIDE> splits unless MM and DPL == 2: mangled "...ELi2ELb1E...")
        splits = cur is not None and "megakernel" in cur and "ELi2ELb1E" not in cur
        if m and splits and int(m.group(1)) < MIN_LAUNCH_REGS:
            os.remove(LIB)
            raise RuntimeError(f"{cur} launches with {m.group(1)} registers per thread; the "
                               f"warpgroup register split needs at least {MIN_LAUNCH_REGS}")
    return LIB


if __name__ == "__main__":
    build(verbose=True, ptxas_verbose="-v" in sys.argv)
