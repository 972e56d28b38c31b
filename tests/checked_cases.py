"""Small calls of every entry point and kernel family, shared by the checked-
build test: run once through the normal library (in the test process) and once
through the checked library (in a child process with GDR_LIBRARY set), the
outputs compared bit for bit.  Each call is followed by gdr_device_status,
which must be GDR_OK (no guard fired, no wait expired)."""
import sys

import numpy as np
import torch

from gated_delta_rule_90_b200 import binding, inputs


def _up(x, dtype, dev):
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return (t.to(torch.bfloat16) if dtype == "bf16" else t).to(dev)


def _np(t):
    return t.float().cpu().numpy() if t.dtype == torch.bfloat16 else t.cpu().numpy()


def _ok(name):
    st = binding.device_status()
    assert st == binding.GDR_OK, (name, binding.status_string(st))


def run_cases(dev) -> dict:
    res = {}

    def prefill(name, cfg, path, cu=None):
        inp = inputs.prefill_inputs(cfg)
        c = None if cu is None else torch.tensor(cu, dtype=torch.int32, device=dev)
        S0 = inp.S0
        if cu is not None:
            S0 = np.random.default_rng(3).standard_normal(
                (len(cu) - 1, cfg.H, cfg.d_v, cfg.d_k)).astype(np.float32) * 0.1
        out, SF = binding.gdr_fwd(_up(inp.q, cfg.dtype, dev), _up(inp.k, cfg.dtype, dev),
                                  _up(inp.v, cfg.dtype, dev), _up(inp.g, "f32", dev),
                                  _up(inp.beta, "f32", dev),
                                  None if S0 is None else _up(S0, "f32", dev), chunk=cfg.chunk,
                                  cu_seqlens=c, path=path)
        _ok(name)
        res[name + ".out"], res[name + ".S"] = _np(out), _np(SF)

    P = inputs.PREFILL
    prefill("tc_scalar", P["gdn_prefill"].replace(B=2, T=200, H=2), "tc")
    prefill("tc_channel", P["kda_prefill"].replace(B=1, T=130, H=2, s0_var=0.01), "tc")
    prefill("tc_c16", P["gdn_prefill_c16"].replace(B=1, T=100, H=2), "tc")
    prefill("tc_varlen", P["gdn_prefill"].replace(B=1, T=200, H=2), "tc", cu=[0, 37, 37, 200])
    prefill("simt_fp32", P["tiny_fp32"], "simt")
    prefill("simt_varlen", P["tiny_fp32"].replace(T=150), "simt", cu=[0, 50, 150])

    pc = P["gdp_prefill"].replace(B=1, T=100, H=2)
    pi = inputs.product_inputs(pc)
    out, SF = binding.gdr_fwd_product(*(_up(x, "bf16", dev) for x in (pi.q, pi.k, pi.v)),
                                      _up(pi.g, "f32", dev), _up(pi.beta, "f32", dev),
                                      _up(pi.S0, "f32", dev))
    _ok("product")
    res["product.out"], res["product.S"] = _np(out), _np(SF)

    gc = P["gdn2_prefill"].replace(B=1, T=150, H=2)
    gi = inputs.gdn2_inputs(gc)
    for path in ("tc", "simt"):
        out, SF = binding.gdr_fwd_gdn2(*(_up(x, "bf16", dev) for x in (gi.q, gi.k, gi.v)),
                                       *(_up(x, "f32", dev) for x in (gi.g, gi.b, gi.w)),
                                       path=path)
        _ok("gdn2_" + path)
        res["gdn2_%s.out" % path], res["gdn2_%s.S" % path] = _np(out), _np(SF)

    for fname, fcfg in (("frame_tc", inputs.FRAME["frame_prefill"].replace(T=300, H=2, n=128)),
                        ("frame_fp32", inputs.FRAME["frame_prefill"].replace(
                            T=130, H=2, d_k=32, d_v=48, n=50, dtype="f32"))):
        fi = inputs.frame_inputs(fcfg)
        out, SF = binding.gdr_fwd_frame(*(_up(x, fcfg.dtype, dev) for x in (fi.q, fi.k, fi.v)),
                                        _up(fi.g, "f32", dev), _up(fi.gamma, "f32", dev), fcfg.n)
        _ok(fname)
        res[fname + ".out"], res[fname + ".S"] = _np(out), _np(SF)

    for dname in ("decode", "kda_decode"):
        dcfg = inputs.DECODE[dname].replace(N=4, H=4)
        S = torch.from_numpy(inputs.decode_state(dcfg)).to(dev)
        tok = inputs.decode_token(dcfg, 0)
        out = binding.gdr_decode_step(_up(tok.q, "bf16", dev), _up(tok.k, "bf16", dev),
                                      _up(tok.v, "bf16", dev), _up(tok.g, "f32", dev),
                                      _up(tok.beta, "f32", dev), S)
        _ok(dname)
        res[dname + ".out"], res[dname + ".S"] = _np(out), _np(S)
    return res


if __name__ == "__main__":
    # child process: GDR_LIBRARY names the checked build
    assert binding.checked_build(), binding.library_path()
    dev = torch.device("cuda:0")
    assert binding.selftest_bounds() == binding.GDR_OK
    assert binding.device_status() == binding.GDR_ERR_BOUNDS  # the guard fired, nothing touched
    assert binding.device_status() == binding.GDR_OK          # and the word was cleared
    np.savez(sys.argv[1], **run_cases(dev))
    print("checked cases ok")
