"""GPU parity of Gated DeltaProduct ("Linear Attention, Visualized", section
"Gated Delta Product (GDP)") through ``gdr_fwd_product`` against the fp64
substep oracle, on the same seeded, dtype-rounded inputs.  Tolerance as for the
gated delta rule: max relative Frobenius error per (sequence, head) of O and
S_final, <= 1e-4 with fp32 inputs and <= 1e-2 with bf16 inputs."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_90_b200 import binding, inputs
from helpers import prefill_out_rel, state_rel, to_dev, to_np

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 1e-2}


def cfg_of(**kw):
    return inputs.PREFILL["gdp_prefill"].replace(**kw)


def run_gpu(inp, dev, path):
    c = inp.cfg
    q, k, v = (to_dev(x, c.dtype, dev) for x in (inp.q, inp.k, inp.v))
    g, b = to_dev(inp.g, "f32", dev), to_dev(inp.beta, "f32", dev)
    S0 = to_dev(inp.S0, "f32", dev)
    cu = None if inp.cu_seqlens is None else torch.from_numpy(inp.cu_seqlens).to(dev)
    out, SF = binding.gdr_fwd_product(q, k, v, g, b, S0, chunk=c.chunk, cu_seqlens=cu, path=path)
    torch.cuda.synchronize()
    assert binding.device_status() == binding.GDR_OK
    return to_np(out), to_np(SF)


def check(inp, dev, path):
    O, SF = run_gpu(inp, dev, path)
    Or, SFr = oracle.product_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.S0, inp.cu_seqlens)
    eo, es = prefill_out_rel(O, Or, inp.cu_seqlens), state_rel(SF, SFr)
    tol = TOL[inp.cfg.dtype]
    assert eo <= tol and es <= tol, (eo, es)


@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("n_h", [1, 2, 3])
def test_gdp_simt_fp32(cuda_device, gate, n_h):
    cfg = cfg_of(B=2, T=77, H=2, d_k=64, d_v=48, dtype="f32", gate=gate, chunk=32, n_h=n_h,
                 gate_scale=0.1 if gate == "scalar" else 0.05)
    check(inputs.product_inputs(cfg, seed=501), cuda_device, "simt")


@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("n_h", [2, 3, 4, 8])
def test_gdp_tc_bf16(cuda_device, gate, n_h):
    """The tensor-core path writes the kept rows itself: staged and stored by
    TMA when n_h divides the chunk (2 and 4 by fixed strides, 8 by the general
    loop), plain stores otherwise (3) and on a sequence's last, partial chunk."""
    cfg = cfg_of(B=2, T=150, H=3, gate=gate, n_h=n_h,
                 gate_scale=0.1 if gate == "scalar" else 0.05)
    check(inputs.product_inputs(cfg, seed=502), cuda_device, "tc")


@pytest.mark.parametrize("path", ["simt", "tc"])
def test_gdp_varlen_with_empty_and_unit_sequences(cuda_device, path):
    cfg = cfg_of(B=1, T=300, H=2, n_h=2)
    inp = inputs.product_inputs(cfg, seed=503)
    inp.cu_seqlens = np.array([0, 0, 1, 40, 97, 97, 300], dtype=np.int32)
    inp.S0 = np.random.default_rng(7).standard_normal((6, 2, 128, 128)).astype(np.float32) * 0.1
    check(inp, cuda_device, path)


def test_gdp_zero_tokens_copies_state(cuda_device):
    inp = inputs.product_inputs(cfg_of(B=2, T=0, H=2, d_k=64, d_v=64, dtype="f32"), seed=504)
    O, SF = run_gpu(inp, cuda_device, "simt")
    assert O.size == 0 and np.array_equal(SF, inp.S0.astype(np.float64))


def test_gdp_prefill_full_size_sampled(cuda_device):
    """The full Gated DeltaProduct workload (B=4, H=16, T=2048, n_h=2) as the
    benchmark launches it; the oracle checks 2 heads of every sequence."""
    inp = inputs.product_inputs(inputs.PREFILL["gdp_prefill"])
    O, SF = run_gpu(inp, cuda_device, "auto")
    heads = [0, 11]
    Or, SFr = oracle.product_fwd(inp.q[:, :, heads], inp.k[:, :, :, heads], inp.v[:, :, :, heads],
                                 inp.g[:, :, heads], inp.beta[:, :, :, heads], inp.S0[:, heads])
    assert np.isfinite(O).all() and np.isfinite(SF).all()
    eo, es = prefill_out_rel(O[:, :, heads], Or), state_rel(SF[:, heads], SFr)
    assert eo <= 1e-2 and es <= 1e-2, (eo, es)


@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("n_h", [2, 3])
def test_gdp_tc_bf16_chunk16(cuda_device, gate, n_h):
    """Gated DeltaProduct with 16-step chunks of the virtual sequence on the
    tensor cores (four chunks per 64-step tile)."""
    cfg = cfg_of(B=2, T=150, H=3, gate=gate, n_h=n_h, chunk=16,
                 gate_scale=0.1 if gate == "scalar" else 0.05)
    check(inputs.product_inputs(cfg, seed=505), cuda_device, "tc")
