"""Host-side checks of the build script: the register-count gate on the
kernels whose warpgroups re-split their registers with setmaxnreg."""
import pytest

from long_context_fp8_b200 import build

LOG = """ptxas info    : 0 bytes gmem
ptxas info    : Compiling entry function '_ZN3dsa44_GLOBAL__N__23299cfa_11_index_tc_cu_559ba1b617fill_upper_kernelEPflll' for 'sm_100a'
ptxas info    : Function properties for _ZN3dsa44_GLOBAL__N__23299cfa_11_index_tc_cu_559ba1b617fill_upper_kernelEPflll
    0 bytes stack frame, 0 bytes spill stores, 0 bytes spill loads
ptxas info    : Used 26 registers, used 0 barriers
ptxas info    : Compiling entry function '_ZN3dsa44_GLOBAL__N__23299cfa_11_index_tc_cu_559ba1b615index_tc_kernelE14CUtensorMap_stS1_S1_NS0_9IdxTcArgsE' for 'sm_100a'
ptxas info    : Function properties for _ZN3dsa44_GLOBAL__N__23299cfa_11_index_tc_cu_559ba1b615index_tc_kernelE14CUtensorMap_stS1_S1_NS0_9IdxTcArgsE
    0 bytes stack frame, 8 bytes spill stores, 8 bytes spill loads
ptxas info    : Used {regs} registers, used 1 barriers, 32 bytes smem
ptxas info    : Compiling entry function '_ZN3dsa45_GLOBAL__N__f0520456_12_decode_tc_cu_6038446a22decode_index_tc_kernelILi64EEEv14CUtensorMap_stS2_NS0_9DecTcArgsE' for 'sm_100a'
ptxas info    : Used 158 registers, used 1 barriers
"""


def test_kernel_name_of_mangled_nested_names():
    assert build.kernel_name("_ZN3dsa44_GLOBAL__N__23299cfa_11_index_tc_cu_559ba1b615index_tc_kernelE14CUtensorMap_st"
                             ) == "index_tc_kernel"
    assert build.kernel_name("_ZN3dsa45_GLOBAL__N__f0520456_12_decode_tc_cu_6038446a22decode_index_tc_kernelILi64EEEv"
                             ) == "decode_index_tc_kernel"
    assert build.kernel_name("plain_c_kernel") == "plain_c_kernel"


def test_register_gate_accepts_the_exact_count():
    found = build.check_registers(LOG.format(regs=168), "index_tc.cu")
    assert [(build.kernel_name(n), r, s) for n, r, s in found] == [
        ("fill_upper_kernel", 26, 0), ("index_tc_kernel", 168, 8), ("decode_index_tc_kernel", 158, 0)]


def test_register_gate_rejects_another_count():
    with pytest.raises(RuntimeError, match="index_tc_kernel built with 160 registers"):
        build.check_registers(LOG.format(regs=160), "index_tc.cu")
