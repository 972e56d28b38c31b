"""CPU checks of the C-ABI library: it loads, exports every declared symbol,
and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest
import torch

from gated_delta_rule_90_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
           if f.endswith(".h")]


def declared_functions():
    names = []
    for h in HEADERS:
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s*(gdr_[a-z0-9_]+)\s*\(",
                            src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("gdr_fwd", "gdr_decode_step", "gdr_status_string", "gdr_fwd_workspace_size",
              "gdr_device_status", "gdr_selftest_wait_timeout"):
        assert n in names


def test_library_exports_every_declared_symbol():
    L = binding.lib()
    for n in declared_functions():
        assert hasattr(L, n), n


def test_status_strings():
    for s in range(6):
        assert binding.status_string(s).startswith("GDR_")
    assert "UNKNOWN" in binding.status_string(99)


# Fake, aligned, never-dereferenced device addresses: every call below is
# rejected by host-side validation before any launch.  On a machine with a GPU
# these tests are skipped so a validation bug can never launch on them.
nogpu = pytest.mark.skipif(torch.cuda.is_available(), reason="host-validation tests use fake pointers")
P = ctypes.c_void_p(0x10000)


def fwd(**kw):
    a = dict(q=P, k=P, v=P, g=P, beta=P, S0=None, out=P, S_final=None, B=1, T=64, H=1, dk=64,
             dv=64, chunk=64, cu=None, n_seq=0, dtype=0, gate=0, path=0, ws=None, wsb=0,
             stream=None)
    a.update(kw)
    return binding.lib().gdr_fwd(a["q"], a["k"], a["v"], a["g"], a["beta"], a["S0"], a["out"],
                                 a["S_final"], a["B"], a["T"], a["H"], a["dk"], a["dv"], a["chunk"],
                                 a["cu"], a["n_seq"], a["dtype"], a["gate"], a["path"], a["ws"],
                                 a["wsb"], a["stream"])


@nogpu
@pytest.mark.parametrize("kw,expect", [
    (dict(q=None), 1), (dict(out=None), 1), (dict(beta=None), 1),
    (dict(B=0), 1), (dict(H=0), 1), (dict(T=-1), 1), (dict(chunk=48), 1), (dict(chunk=0), 1),
    (dict(dtype=7), 1), (dict(gate=3), 1), (dict(path=9), 1),
    (dict(q=ctypes.c_void_p(0x10004)), 1), (dict(S_final=ctypes.c_void_p(0x10008)), 1),
    (dict(cu=P, B=2, n_seq=2), 1), (dict(cu=P, B=1, n_seq=0), 1),
    (dict(dk=256, dv=64), 2), (dict(dk=24), 2), (dict(chunk=256), 1),
    (dict(chunk=128, path=2, dtype=1, dk=128, dv=128), 2),
    (dict(path=2, dtype=0), 2), (dict(path=2, dtype=1, dk=64, dv=64), 2),
])
def test_fwd_rejects_on_host(kw, expect):
    assert fwd(**kw) == expect


@nogpu
@pytest.mark.parametrize("kw,expect", [
    (dict(S=None), 1), (dict(N=0), 1), (dict(dk=96), 2), (dict(dv=48), 2), (dict(dtype=5), 1),
    (dict(q=ctypes.c_void_p(0x10002)), 1),
])
def test_decode_rejects_on_host(kw, expect):
    a = dict(q=P, k=P, v=P, g=P, beta=P, S=P, out=P, N=2, H=2, dk=128, dv=128, dtype=1, gate=0)
    a.update(kw)
    st = binding.lib().gdr_decode_step(a["q"], a["k"], a["v"], a["g"], a["beta"], a["S"], a["out"],
                                       a["N"], a["H"], a["dk"], a["dv"], a["dtype"], a["gate"], None)
    assert st == expect


def test_workspace_size_is_zero_for_simt_and_rejected_args():
    assert binding.fwd_workspace_size(1, 256, 2, 64, 64, 64, 0, False, 0, 0, "auto") == 0
    assert binding.fwd_workspace_size(0, 256, 2, 64, 64, 64, 0, False, 0, 0, "auto") == 0


def test_selftest_rejects_bad_limit():
    assert binding.lib().gdr_selftest_wait_timeout(0, None) == binding.GDR_ERR_INVALID


def product(**kw):
    a = dict(q=P, k=P, v=P, g=P, beta=P, S0=None, out=P, SF=P, B=2, T=64, H=2, nh=2, dk=128,
             dv=128, chunk=64, cu=None, n_seq=2, dtype=1, gate=0, path=0, ws=P, ws_bytes=16)
    a.update(kw)
    return binding.lib().gdr_fwd_product(
        a["q"], a["k"], a["v"], a["g"], a["beta"], a["S0"], a["out"], a["SF"], a["B"], a["T"],
        a["H"], a["nh"], a["dk"], a["dv"], a["chunk"], a["cu"], a["n_seq"], a["dtype"], a["gate"],
        a["path"], a["ws"], a["ws_bytes"], None)


@nogpu
@pytest.mark.parametrize("kw,expect", [
    (dict(nh=0), 1), (dict(dk=72), 2), (dict(dv=136), 2), (dict(q=ctypes.c_void_p(0x10004)), 1),
    (dict(cu=P, B=2), 1), (dict(dtype=7), 1), (dict(ws=None, ws_bytes=0), 1), (dict(ws_bytes=16), 1),
    (dict(k=None), 1),
])
def test_product_rejects_on_host(kw, expect):
    assert product(**kw) == expect


def test_gdn2_workspace_only_on_the_tensor_core_path():
    assert binding.fwd_gdn2_workspace_size(2, 256, 4, 128, 128, 64, 2, False, 1, 1, "auto") > 0
    # the scalar decay takes the tensor-core path too (broadcast in the kernel)
    assert binding.fwd_gdn2_workspace_size(2, 256, 4, 128, 128, 64, 2, False, 1, 0, "auto") > 0
    assert binding.fwd_gdn2_workspace_size(2, 256, 4, 128, 128, 64, 2, False, 0, 0, "auto") == 0
    assert binding.fwd_gdn2_workspace_size(2, 256, 4, 128, 128, 64, 2, False, 1, 1, "simt") == 0
    assert binding.fwd_gdn2_workspace_size(2, 256, 4, 128, 128, 64, 2, False, 1, 1, "auto") == \
        binding.fwd_workspace_size(2, 256, 4, 128, 128, 64, 2, False, 1, 1, "auto")


def test_product_workspace_holds_the_virtual_sequence():
    """The product workspace covers q~, g~ and o~ for n_h T virtual steps plus
    the gated delta rule's own workspace for them."""
    lib = binding.lib()
    B, T, H, nh, d = 2, 300, 4, 3, 128
    inner = binding.fwd_workspace_size(B, T * nh, H, d, d, 64, B, False, 1, 0, "auto")
    ws = binding.fwd_product_workspace_size(B, T, H, nh, d, d, 64, B, False, 1, 0, "auto")
    assert inner > 0 and ws >= inner + 2 * B * T * nh * H * d * 2 + B * T * nh * H * 4
    assert binding.fwd_product_workspace_size(B, T, H, 0, d, d, 64, B, False, 1, 0, "auto") == 0
    assert lib.gdr_fwd_product_workspace_size is not None


@nogpu
@pytest.mark.parametrize("kw,expect", [
    (dict(b=None), 1), (dict(dk=72), 2), (dict(chunk=48), 1),
    (dict(chunk=128, dtype=1, dk=128, dv=128, path=2), 2),
    (dict(w=ctypes.c_void_p(0x10008)), 1), (dict(cu=P, B=2), 1), (dict(gate=3), 1),
    (dict(path=2), 2), (dict(dtype=1, dk=128, dv=128, path=2), 1), (dict(path=7), 1),
])
def test_gdn2_fwd_rejects_on_host(kw, expect):
    a = dict(q=P, k=P, v=P, g=P, b=P, w=P, S0=None, out=P, SF=P, B=2, T=64, H=2, dk=64, dv=64,
             chunk=64, cu=None, n_seq=2, dtype=0, gate=1, path=0, ws=None, ws_bytes=0)
    a.update(kw)
    st = binding.lib().gdr_fwd_gdn2(a["q"], a["k"], a["v"], a["g"], a["b"], a["w"], a["S0"],
                                    a["out"], a["SF"], a["B"], a["T"], a["H"], a["dk"], a["dv"],
                                    a["chunk"], a["cu"], a["n_seq"], a["dtype"], a["gate"],
                                    a["path"], a["ws"], a["ws_bytes"], None)
    assert st == expect


@nogpu
@pytest.mark.parametrize("kw,expect", [(dict(w=None), 1), (dict(dk=96), 2), (dict(N=0), 1)])
def test_gdn2_decode_rejects_on_host(kw, expect):
    a = dict(q=P, k=P, v=P, g=P, b=P, w=P, S=P, out=P, N=2, H=2, dk=128, dv=128, dtype=1, gate=1)
    a.update(kw)
    st = binding.lib().gdr_decode_step_gdn2(a["q"], a["k"], a["v"], a["g"], a["b"], a["w"],
                                            a["S"], a["out"], a["N"], a["H"], a["dk"], a["dv"],
                                            a["dtype"], a["gate"], None)
    assert st == expect


@nogpu
@pytest.mark.parametrize("kw,expect", [
    (dict(n=0), 1), (dict(dk=12), 2), (dict(dv=136), 2), (dict(gamma=None), 1),
    (dict(ws=None, ws_bytes=0), 1), (dict(q=ctypes.c_void_p(0x10006)), 1), (dict(gate=4), 1),
])
def test_frame_rejects_on_host(kw, expect):
    a = dict(q=P, k=P, v=P, g=P, gamma=P, S0=None, out=P, SF=P, B=1, T=64, H=2, dk=64, dv=64, n=16,
             dtype=0, gate=1, ws=P, ws_bytes=16)
    a.update(kw)
    st = binding.lib().gdr_fwd_frame(a["q"], a["k"], a["v"], a["g"], a["gamma"], a["S0"], a["out"],
                                     a["SF"], a["B"], a["T"], a["H"], a["dk"], a["dv"], a["n"],
                                     a["dtype"], a["gate"], a["ws"], a["ws_bytes"], None)
    assert st == expect


def test_frame_workspace_size():
    B, T, H, d, n = 1, 1000, 3, 128, 256
    F = -(-T // n)
    assert binding.fwd_frame_workspace_size(B, T, H, d, d, n) >= 3 * B * F * H * d * d * 4
    assert binding.fwd_frame_workspace_size(B, T, H, 12, d, n) == 0


def test_gram_spread_limit_is_clamped_and_restored():
    """gdr_set_gram_spread_limit returns the previous limit, clamps into
    [0, 80] and ignores NaN (host state only; no launch)."""
    prev = binding.set_gram_spread_limit(60.0)
    try:
        assert binding.set_gram_spread_limit(1000.0) == 60.0
        assert binding.set_gram_spread_limit(-5.0) == 80.0
        assert binding.set_gram_spread_limit(float("nan")) == 0.0
        assert binding.set_gram_spread_limit(60.0) == 0.0
    finally:
        binding.set_gram_spread_limit(prev)
