"""The promoted (FP8_BLOCK128) GEMMs move registers between warpgroups with
setmaxnreg: warpgroup 0 decreases to PROMOTE_CTRL_REGS and the two epilogue
warpgroups increase to PROMOTE_EPI_REGS.  An increase waits until the block
has the registers free, so the split is only safe when the kernel launches
with PROMOTE_LAUNCH_REGS per thread; if ptxas allocated fewer at launch the
epilogue warpgroups would wait forever.  This compiles the device code (no
GPU needed) and checks ptxas's launch allocation of every promoted kernel, the
split's arithmetic, and that the 256-wide promoted bodies do not spill."""
import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "mixture_experts_topk_b200", "csrc")


def constant(name):
    src = open(os.path.join(CSRC, "gemm.cuh")).read()
    m = re.search(r"constexpr int %s = (\d+);" % name, src)
    assert m, name
    return int(m.group(1))


@pytest.fixture(scope="module")
def ptxas_report(tmp_path_factory):
    nvcc = os.environ.get("NVCC", "nvcc")
    if shutil.which(nvcc) is None:
        pytest.skip("nvcc not found")
    out = tmp_path_factory.mktemp("cubin") / "moe_api.cubin"
    r = subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "--cubin", "-O3", "-std=c++17",
                        "-Xptxas=-v", "-I", os.path.join(ROOT, "include"), os.path.join(CSRC, "moe_api.cu"),
                        "-o", str(out)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-2000:]
    kernels = {}
    for block in re.split(r"ptxas info\s+: Compiling entry function '", r.stderr)[1:]:
        mangled = block.split("'")[0]
        name = subprocess.run(["c++filt", mangled], capture_output=True, text=True).stdout.strip() or mangled
        regs = re.search(r"Used (\d+) registers", block)
        spill = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", block)
        kernels[name.split("(")[0]] = (int(regs.group(1)), int(spill.group(1)), int(spill.group(2)))
    return kernels


def promoted(kernels):
    return {n: v for n, v in kernels.items()
            if re.search(r"grouped_gemm_kernel<\d+, 1, true,", n) or "down_gemm_poly_kernel" in n}


def test_split_fits_the_launch_allocation():
    launch, ctrl, epi = (constant("PROMOTE_LAUNCH_REGS"), constant("PROMOTE_CTRL_REGS"),
                         constant("PROMOTE_EPI_REGS"))
    threads = 384   # warpgroup 0 + two epilogue warpgroups
    assert launch == (65536 // threads) // 8 * 8
    assert 128 * ctrl + 256 * epi <= threads * launch
    # each sub-partition holds one warp of each warpgroup
    assert 32 * (ctrl + 2 * epi) <= 16384
    assert ctrl % 8 == 0 and epi % 8 == 0 and 24 <= ctrl <= 256 and 24 <= epi <= 256


def test_promoted_kernels_launch_with_the_split_budget(ptxas_report):
    kernels = promoted(ptxas_report)
    assert len(kernels) >= 3, sorted(ptxas_report)
    launch = constant("PROMOTE_LAUNCH_REGS")
    for name, (regs, _, _) in kernels.items():
        assert regs == launch, (name, regs)


def test_wide_promoted_bodies_do_not_spill(ptxas_report):
    wide = {n: v for n, v in promoted(ptxas_report).items() if ", true, 256," in n}
    assert wide
    for name, (_, stores, loads) in wide.items():
        assert stores == 0 and loads == 0, (name, stores, loads)
