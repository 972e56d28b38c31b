"""CPU checks of the checked build (-DGDR_CHECK): it compiles for sm_100a,
loads, exports every symbol the headers declare, and says it is the checked
build; the normal library says it is not and refuses the bounds self-test on
the host."""
import ctypes
import os

from gated_delta_rule_90_b200 import binding, build

from test_abi import declared_functions


def checked_lib():
    if not os.path.exists(binding.CHECKED_LIB_PATH):
        build.build(checked=True)
    return ctypes.CDLL(binding.CHECKED_LIB_PATH)


def test_checked_library_exports_every_declared_symbol():
    L = checked_lib()
    for n in declared_functions():
        assert hasattr(L, n), n
    L.gdr_checked_build.restype = ctypes.c_int
    assert L.gdr_checked_build() == 1


def test_normal_library_is_not_checked():
    assert binding.checked_build() is False
    # refused before any CUDA call (a null stream; no device needed)
    assert binding.lib().gdr_selftest_bounds(None) == binding.GDR_ERR_UNSUPPORTED


def test_bounds_status_string():
    assert binding.status_string(binding.GDR_ERR_BOUNDS).startswith("GDR_ERR_BOUNDS")
