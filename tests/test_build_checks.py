"""Build-level checks on the CPU: the launch-register check (nvcc
cross-compiles for sm_100a) and a plain C program calling the library.

The warp-specialised kernels regroup registers with setmaxnreg: some
warpgroups grow, the others shrink, and the shares add up to the registers
the block was launched with. If ptxas gave a kernel fewer registers per
thread than its split assumes, the growing warpgroups would wait forever on
the GPU. The build reads ptxas's report and refuses such a library; these
tests check that the report parser finds a mismatch and that the kernels as
they stand pass. The last test compiles tests/c/abi_host_only.c with gcc
against include/sca.h and libsca.so alone and runs its host-side calls.
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


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_plain_c_caller_of_the_abi(tmp_path):
    """tests/c/abi_host_only.c uses nothing but include/sca.h and libsca.so:
    it builds the 480p long session's metadata, reads counts and schedule,
    and checks two refused layouts. A is the hand-worked closed form
    12,090 (12 x 12,218 + 12,250) + 128 x 12,218 + 128 x 12,250; the tile
    counts must equal what the Python binding reads from the same library."""
    from segment_causal_masked_b200 import sca
    from segment_causal_masked_b200 import workloads as W

    exe = tmp_path / "abi_host_only"
    lib_dir = os.path.dirname(sca.LIB_PATH)
    src = os.path.join(os.path.dirname(os.path.abspath(__file__)), "c", "abi_host_only.c")
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", B.INCLUDE, src,
                         "-L", lib_dir, "-lsca", f"-Wl,-rpath,{lib_dir}", "-o", str(exe)],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    lines = dict(line.split(" ", 1) for line in run.stdout.strip().splitlines())

    counts = [int(x) for x in lines["counts"].split()]
    assert counts[0] == 12_090 * (12 * 12_218 + 12_250) + 128 * 12_218 + 128 * 12_250
    c = sca.build_for(W.session_480p_long()).counts()
    assert counts == [c["unmasked_pairs"], c["n_queries"], c["n_cache_keys"], c["n_q_tiles"],
                      c["n_kv_tiles"], c["nnz"], c["n_full"], c["n_partial"]]
    assert counts[1:5] == [12_346, 148_152, 97, 1158 + 97]
    assert lines["schedule"].split() == [str(c["nnz"]), "0", str(sca.TILE_FULL)]

    for key in ("bad_segment", "bad_window"):
        code, message = lines[key].split(" ", 1)
        assert int(code) == sca.ERR_INVALID_ARG and message, key
    assert "num_frames" in lines["bad_segment"] and "[24, 32)" in lines["bad_window"]


def test_binding_constants_match_the_header():
    """The Python binding restates some of sca.h's constants; read them back
    from the header so the two cannot drift apart."""
    import re

    from segment_causal_masked_b200 import sca

    text = open(os.path.join(B.INCLUDE, "sca.h")).read()
    enums = {m.group(1): int(m.group(2)) for m in re.finditer(r"\b(SCA_\w+)\s*=\s*(-?\d+)", text)}
    defines = {m.group(1): m.group(2) for m in re.finditer(r"#define\s+(SCA_\w+)\s+(.+)", text)}
    pairs = {
        "SCA_OK": sca.OK, "SCA_ERR_INVALID_ARG": sca.ERR_INVALID_ARG,
        "SCA_ERR_UNSUPPORTED": sca.ERR_UNSUPPORTED, "SCA_ERR_MISALIGNED": sca.ERR_MISALIGNED,
        "SCA_ERR_CAPACITY": sca.ERR_CAPACITY, "SCA_ERR_CUDA": sca.ERR_CUDA,
        "SCA_ERR_DEVICE_TIMEOUT": sca.ERR_DEVICE_TIMEOUT, "SCA_ERR_MISMATCH": sca.ERR_MISMATCH,
        "SCA_TEXTQ_OWN_TAIL": sca.TEXTQ_OWN_TAIL, "SCA_TEXTQ_FULL_SEGMENT": sca.TEXTQ_FULL_SEGMENT,
        "SCA_TILE_EMPTY": sca.TILE_EMPTY, "SCA_TILE_PARTIAL": sca.TILE_PARTIAL,
        "SCA_TILE_FULL": sca.TILE_FULL, "SCA_CAM_ALL": sca.CAM_ALL,
        "SCA_CAM_OWN_FRAME": sca.CAM_OWN_FRAME, "SCA_CAM_UP_TO_FRAME": sca.CAM_UP_TO_FRAME,
    }
    for name, value in pairs.items():
        assert enums[name] == value, name
    assert int(defines["SCA_HEAD_DIM"]) == sca.HEAD_DIM
    assert int(defines["SCA_TILE"]) == sca.TILE
    assert int(defines["SCA_MAX_ACTIONS"]) == sca.MAX_ACTIONS
    assert int(defines["SCA_MAX_CAMERA_TOKENS"]) == sca.MAX_CAMERA_TOKENS
    m = re.match(r"\((\d+)ull\s*<<\s*(\d+)\)", defines["SCA_STATIC_WORKSPACE_BYTES"].strip())
    assert m and int(m.group(1)) << int(m.group(2)) == sca.STATIC_WORKSPACE_BYTES


def test_binding_signatures_match_the_header_prototypes():
    """Every exported prototype in sca.h has a ctypes signature in the binding
    with the same number of arguments."""
    import re

    from segment_causal_masked_b200 import sca

    text = open(os.path.join(B.INCLUDE, "sca.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    protos = {m.group(1): m.group(2) for m in
              re.finditer(r"SCA_API\s+[\w\s\*]+?\b(sca_\w+)\s*\(([^)]*)\)\s*;", text, flags=re.S)}
    assert len(protos) >= 25
    for name, args in protos.items():
        n = 0 if args.strip() in ("", "void") else args.count(",") + 1
        assert name in sca._SIGS, name
        assert len(sca._SIGS[name]) == n, (name, n, len(sca._SIGS[name]))
    assert set(protos) == set(sca.EXPORTED)
