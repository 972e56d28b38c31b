"""Host-side logic, on the CPU: the seeded input generators (each workload's
recipe), the benchmark's accounting of algorithmic work against the figures
derived from the chunk algorithm, and the kernel-id table of the binding."""
import re

import numpy as np
import pytest
import torch

import bench
from gated_delta_rule_90_b200 import binding, inputs

ROOT = __import__("os").path.dirname(__import__("os").path.dirname(__file__))


# ------------------------------------------------------------------ generators
def test_bf16_rounding_matches_torch():
    """round_to(·, "bf16") is round-to-nearest-even on the bit pattern, the
    same rounding torch applies, across 60 decades and both signs."""
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(200000) * 10.0 ** rng.uniform(-30, 30, 200000)).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    got = inputs.round_to(x, "bf16")
    assert np.array_equal(got, ref)
    assert np.all((got.view(np.uint32) & 0xFFFF) == 0)


def test_bf16_ties_go_to_even():
    x = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8)], dtype=np.float32)
    assert list(inputs.round_to(x, "bf16")) == [1.0, np.float32(1 + 2 ** -6), -1.0]


def small(name):
    cfg = inputs.PREFILL[name]
    if cfg.n_seq:
        return cfg.replace(T=200, H=2, d_k=32, d_v=16, n_seq=4, len_lo=20, len_hi=80)
    return cfg.replace(B=2, T=70, H=2, d_k=32, d_v=16)


def draw(cfg, seed):
    if cfg.n_h > 1:
        return inputs.product_inputs(cfg, seed=seed)
    if cfg.variant == "gdn2":
        return inputs.gdn2_inputs(cfg, seed=seed)
    return inputs.prefill_inputs(cfg, seed=seed)


@pytest.mark.parametrize("name", list(inputs.PREFILL))
def test_prefill_generators(name):
    """Shapes, value ranges and determinism of every prefill workload's recipe:
    unit-norm queries and keys (before rounding), values rounded to the
    workload's dtype, negative log-decays, step sizes and gates in (0, 1)."""
    cfg = small(name)
    a, b, c = draw(cfg, 11), draw(cfg, 11), draw(cfg, 12)
    for f in ("q", "k", "v", "g"):
        assert np.array_equal(getattr(a, f), getattr(b, f)), f
    assert not np.array_equal(a.k, c.k)
    B, T, H, dk, dv = cfg.B, cfg.T, cfg.H, cfg.d_k, cfg.d_v
    nh = cfg.n_h
    assert a.q.shape == (B, T, H, dk)
    assert a.k.shape == ((B, T, nh, H, dk) if nh > 1 else (B, T, H, dk))
    assert a.v.shape == ((B, T, nh, H, dv) if nh > 1 else (B, T, H, dv))
    assert a.g.shape == ((B, T, H, dk) if cfg.gate == "channel" else (B, T, H))
    assert np.all(a.g < 0)
    tol = 1e-2 if cfg.dtype == "bf16" else 1e-5
    for x in (a.q, a.k):
        assert np.max(np.abs(np.linalg.norm(x.astype(np.float64), axis=-1) - 1)) < tol
    if cfg.dtype == "bf16":
        for x in (a.q, a.k, a.v):
            assert np.all((x.view(np.uint32) & 0xFFFF) == 0)
    if cfg.variant == "gdn2":
        for x in (a.b, a.w):
            assert np.all((x > 0) & (x < 1))
    else:
        assert np.all((a.beta > 0) & (a.beta < 1))
    if cfg.n_seq:
        lens = np.diff(a.cu_seqlens)
        assert a.cu_seqlens[0] == 0 and lens.sum() == T and len(lens) == cfg.n_seq
        assert lens.min() >= cfg.len_lo and lens.max() <= cfg.len_hi
    if cfg.s0_var > 0:
        n_seq = cfg.n_seq or B
        assert a.S0.shape == (n_seq, H, dv, dk)


def test_varlen_lengths_recipe():
    """The 16-sequence packed workload: 15 lengths uniform in [1024, 7168], the
    16th takes the remainder to 65,536 and lies in range too."""
    cfg = inputs.PREFILL["varlen_prefill"]
    for seed in range(20):
        lens = inputs.varlen_lengths(np.random.default_rng(seed), cfg.n_seq, cfg.T, cfg.len_lo,
                                     cfg.len_hi)
        assert len(lens) == 16 and lens.sum() == 65536
        assert lens.min() >= 1024 and lens.max() <= 7168


@pytest.mark.parametrize("name", list(inputs.DECODE))
def test_decode_tokens_are_deterministic_per_step(name):
    cfg = inputs.DECODE[name].replace(N=3, H=2)
    t0, t0b, t1 = inputs.decode_token(cfg, 0), inputs.decode_token(cfg, 0), inputs.decode_token(cfg, 1)
    assert np.array_equal(t0.k, t0b.k) and not np.array_equal(t0.k, t1.k)
    assert t0.g.shape == ((3, 2, cfg.d_k) if cfg.gate == "channel" else (3, 2))
    S = inputs.decode_state(cfg)
    assert S.shape == (3, 2, cfg.d_v, cfg.d_k) and S.dtype == np.float32


def test_frame_generator():
    cfg = inputs.FRAME["frame_prefill"].replace(T=300, H=2, n=64)
    a = inputs.frame_inputs(cfg, seed=3)
    assert a.g.shape == (1, cfg.frames, 2, cfg.d_k) and cfg.frames == 5
    assert np.all(a.gamma > 0) and a.gamma.shape == (1, 300, 2)


# ------------------------------------------------------------------ accounting
def test_prefill_flops_per_token_head():
    """2C(3 d_k + 2 d_v) + 6 d_k d_v: the eight chunk GEMMs counted dense."""
    assert bench.prefill_flops_per_token_head(64, 128, 128) == 180224
    assert bench.prefill_flops_per_token_head(64, 64, 64) == 65536
    assert bench.prefill_flops_split(64, 128, 128) == (65536, 114688)
    for C in (16, 32, 64, 128):
        wy, st = bench.prefill_flops_split(C, 128, 128)
        assert wy + st == bench.prefill_flops_per_token_head(C, 128, 128)


def test_prefill_min_bytes():
    """One read of q, k, v, g, beta and one write of out per token-head (1,032 B
    for bf16 with a scalar gate, 1,540 B with a per-channel gate), plus the
    states read and written once."""
    gdn = inputs.PREFILL["gdn_prefill"]
    th = gdn.B * gdn.T * gdn.H
    st = gdn.B * gdn.H * 128 * 128 * 4
    assert bench.prefill_min_bytes(gdn, gdn.B) == th * 1032 + 2 * st
    assert bench.prefill_min_bytes(gdn.replace(s0_var=0.0), gdn.B) == th * 1032 + st
    kda = inputs.PREFILL["kda_prefill"]
    th = kda.B * kda.T * kda.H
    assert bench.prefill_min_bytes(kda, kda.B) == th * 1540 + kda.B * kda.H * 128 * 128 * 4
    for name in ("gdn_prefill", "kda_prefill", "gdp_prefill", "gdn2_prefill"):
        cfg = inputs.PREFILL[name]
        parts = sum(bench.prefill_kernel_min_bytes(cfg, cfg.B, k) for k in ("tc_wy", "tc_state"))
        assert parts == bench.prefill_min_bytes(cfg, cfg.B)


def test_decode_bytes():
    """2 x 512 MiB of state plus 8,192 x 1,032 B of token I/O per step."""
    assert bench.decode_bytes(inputs.DECODE["decode"]) == 1_082_195_968
    assert bench.decode_bytes(inputs.DECODE["kda_decode"]) == 2 * 2 ** 29 + 8192 * 1540


def test_frame_flops():
    dk = dv = 128
    n = 1024
    per = 2 * dk * (dk + dv) + 2 * dk * dv + (dk ** 3 / 3 + 2 * dv * dk * dk) / n
    assert bench.frame_flops_per_token_head(dk, dv, n) == pytest.approx(per)


def test_ncu_traffic_is_tied_to_the_sources(monkeypatch):
    """A recorded traffic figure is reported only while the kernel sources
    still hash to the digest it was taken on."""
    assert bench.ncu_traffic("tc_wy", "no_such_workload") is None
    for key, (_, _, val) in bench.NCU_TRAFFIC.items():
        assert bench.ncu_traffic(*key) in (None, val), key  # current, or null once stale
    files, _, val = bench.NCU_TRAFFIC[("decode", "decode")]
    monkeypatch.setitem(bench.NCU_TRAFFIC, ("decode", "decode"), (files, "0" * 16, val))
    assert bench.ncu_traffic("decode", "decode") is None


@pytest.mark.parametrize("name", list(inputs.PREFILL) + list(inputs.DECODE) + list(inputs.FRAME))
def test_workload_config_names_the_workload(name):
    cfg, conf = bench.workload_config(name)
    assert conf["workload"] == name and "H" in conf and "d_k" in conf and "d_v" in conf


# ------------------------------------------------------------------ binding
def test_kernel_ids_match_the_header():
    """binding.KERNELS carries every GDR_K_* id of include/gdr.h, same values."""
    hdr = open(__import__("os").path.join(ROOT, "include", "gdr.h")).read()
    ids = {m.group(1).lower(): int(m.group(2))
           for m in re.finditer(r"GDR_K_([A-Z0-9_]+)\s*=\s*(\d+)", hdr) if m.group(1) != "COUNT"}
    assert sorted(ids.values()) == sorted(binding.KERNELS.values())
    assert len(ids) == len(binding.KERNELS)


def test_binding_rejects_host_tensors_before_any_launch():
    """Host tensors never reach the library: their addresses would be device
    faults in the kernels."""
    q = torch.zeros(1, 4, 2, 16)
    with pytest.raises(ValueError, match="CUDA"):
        binding.gdr_fwd(q, q, q, torch.zeros(1, 4, 2), torch.zeros(1, 4, 2))
    with pytest.raises(ValueError, match="CUDA"):
        binding.gdr_decode_step(q[0], q[0], q[0], torch.zeros(4, 2), torch.zeros(4, 2),
                                torch.zeros(4, 2, 16, 16))


def test_binding_checks_device_dtype_and_size():
    """The tensor checks the binding applies before a call (shown on the CPU
    device): a narrower dtype, a too-small tensor or another device is refused."""
    dev = torch.device("cpu")
    ok = ("g", torch.zeros(6, dtype=torch.float32), torch.float32, 6)
    binding._check(dev, ok, ("absent", None, torch.float32, 10))
    with pytest.raises(TypeError):
        binding._check(dev, ("g", torch.zeros(6, dtype=torch.bfloat16), torch.float32, 6))
    with pytest.raises(ValueError, match="elements"):
        binding._check(dev, ("beta", torch.zeros(5), torch.float32, 6))
    with pytest.raises(ValueError, match="expected"):
        binding._check(dev, ("S0", torch.zeros(6, device="meta"), torch.float32, 6))
    with pytest.raises(TypeError):
        binding._check(dev, ("k", [0.0] * 6, None, 6))


# ------------------------------------------------------------------ binding device rules
def test_binding_calls_run_with_the_tensors_device_current(monkeypatch):
    """libgdr launches on the current CUDA device, so the binding makes the
    tensors' device current around every call (a mocked device guard records
    which device it was given)."""
    import contextlib

    from gated_delta_rule_90_b200 import binding

    seen = []

    @contextlib.contextmanager
    def fake_device(d):
        seen.append(torch.device(d))
        yield

    monkeypatch.setattr(binding.torch.cuda, "device", fake_device)
    assert binding._call_on(torch.device("cuda", 3), lambda: 17) == 17
    assert seen == [torch.device("cuda", 3)]


def test_binding_rejects_a_stream_of_another_device():
    from gated_delta_rule_90_b200 import binding

    class FakeStream:
        device = torch.device("cuda", 1)
        cuda_stream = 1234

    with pytest.raises(ValueError):
        binding._stream(FakeStream(), torch.device("cuda", 0))
    assert binding._stream(FakeStream(), torch.device("cuda", 1)).value == 1234
    assert binding._stream(5678, torch.device("cuda", 0)).value == 5678  # raw handle: unchecked


def test_binding_rejects_a_workspace_on_another_device():
    from gated_delta_rule_90_b200 import binding

    ws = torch.empty(16, dtype=torch.uint8)  # host memory
    with pytest.raises(ValueError):
        binding._check(torch.device("cuda", 0), ("workspace", ws, None, 0))
    binding._check(torch.device("cpu"), ("workspace", ws, None, 0))
