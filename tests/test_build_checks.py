"""The build's launch-register check (CPU; nvcc cross-compiles for sm_100a).

The warp-specialised kernels regroup registers with setmaxnreg: some
warpgroups grow, the others shrink, and the shares add up to the registers
the block was launched with. If ptxas gave a kernel fewer registers per
thread than its split assumes, the growing warpgroups would wait forever on
the GPU. The build reads ptxas's report and refuses such a library; these
tests check that the report parser finds a mismatch and that the kernels as
they stand pass.
"""
import os
import shutil
import subprocess
from concurrent.futures import ThreadPoolExecutor

import pytest

from segment_causal_masked_b200 import build as B

REPORT = """\
ptxas info    : Compiling entry function '_ZN3sca15attn_fwd_kernelILb0EEEv14CUtensorMap_stS1_' for 'sm_100a'
ptxas info    : Function properties for _ZN3sca15attn_fwd_kernelILb0EEEv14CUtensorMap_stS1_
    16 bytes stack frame, 20 bytes spill stores, 96 bytes spill loads
ptxas info    : Used {fwd} registers, used 1 barriers, 16 bytes cumulative stack size
ptxas info    : Compiling entry function '_ZN3sca15attn_fwd_kernelILb1EEEv14CUtensorMap_stS1_' for 'sm_100a'
ptxas info    : Used 128 registers, used 1 barriers
ptxas info    : Compiling entry function '_ZN3sca13bwd_dq_kernelE14CUtensorMap_stS0_' for 'sm_100a'
ptxas info    : Used 168 registers, used 1 barriers
ptxas info    : Compiling entry function '_ZN3sca15bwd_dkdv_kernelE14CUtensorMap_stS0_' for 'sm_100a'
ptxas info    : Used 168 registers, used 1 barriers
ptxas info    : Compiling entry function '_ZN3sca12merge_kernelENS_8AttnArgsE' for 'sm_100a'
ptxas info    : Used 40 registers, used 0 barriers
"""


def test_parser_reads_every_entry():
    regs = B.kernel_registers(REPORT.format(fwd=168))
    assert sorted(regs.values()) == [40, 128, 168, 168, 168]
    B.check_launch_registers(REPORT.format(fwd=168))


@pytest.mark.parametrize("fwd", [160, 176])
def test_mismatched_registers_are_refused(fwd):
    with pytest.raises(RuntimeError, match="attn_fwd_kernelILb0E"):
        B.check_launch_registers(REPORT.format(fwd=fwd))


def test_missing_kernel_is_refused():
    with pytest.raises(RuntimeError, match="bwd_dkdv_kernel"):
        B.check_launch_registers(REPORT.format(fwd=168).split("_ZN3sca15bwd_dkdv")[0])


@pytest.mark.skipif(shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"),
                    reason="needs nvcc")
def test_current_kernels_get_the_registers_their_splits_need(tmp_path):
    def compile_one(src):
        cmd = [B.nvcc(), *B.ARCH, "-O3", "-std=c++17", "-Xptxas", "-v", "-I", B.INCLUDE,
               "-I", B.CSRC, "-DSCA_BUILD", "-c", os.path.join(B.CSRC, src),
               "-o", str(tmp_path / (src + ".o"))]
        p = subprocess.run(cmd, capture_output=True, text=True)
        assert p.returncode == 0, p.stderr[-2000:]
        return p.stdout + p.stderr

    with ThreadPoolExecutor(2) as ex:
        log = "".join(ex.map(compile_one, ["sca_kernels.cu", "sca_bwd.cu"]))
    B.check_launch_registers(log)
