"""Benchmark of the gated delta rule forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one gdr_fwd over the workload's whole batch (prefill workloads) or
one gdr_decode_step over all sequences (decode).  Inputs are seeded synthetic
data of the workload's shapes and distributions (gated_delta_rule_90_b200.inputs),
resident in HBM before the timed region.  Prints ONE JSON line on rank 0.

Multi-GPU (launched by torch.distributed.run): the (sequence, head) units of
the method are independent, so every rank runs its own copy of the workload
(weak scaling) with no collective on the data path; only the timing is reduced
(max over ranks).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gated_delta_rule_90_b200 import binding, inputs  # noqa: E402

METRIC = "gated-delta-rule fwd tokens/s; % roofline (TC TFLOP/s prefill, HBM GB/s decode)"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
SM_COUNT = 148
# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) from
# one ncu capture (summaries under profiles/), valid only for the kernel sources
# it was taken on: keyed by (kernel, workload), with the first 16 hex digits of
# the sha256 of those sources in order.
_TC_SRC = ('csrc/fwd_tc.cu', 'csrc/sm100.cuh', 'csrc/common.cuh')
_DEC_SRC = ('csrc/decode.cu', 'csrc/common.cuh')
_FR_SRC = ('csrc/frame.cu', 'csrc/sm100.cuh', 'csrc/tmap.cuh', 'csrc/common.cuh')
NCU_TRAFFIC = {
    ("tc_wy", "gdn_prefill"): (_TC_SRC, "90c504ae376e1600", 206.136064e6 + 253.452032e6),
    ("tc_state", "gdn_prefill"): (_TC_SRC, "90c504ae376e1600", 308.366336e6 + 52.554752e6),
    ("tc_wy", "kda_prefill"): (_TC_SRC, "90c504ae376e1600", 681.240832e6 + 565.438464e6),
    ("decode", "decode"): (_DEC_SRC, "67d72f2db8183636", 543.343360e6 + 481.382144e6),
    ("decode", "kda_decode"): (_DEC_SRC, "67d72f2db8183636", 547.481088e6 + 481.806848e6),
    ("frame_chain", "frame_prefill"): (_FR_SRC, "d7a96b3509fa7060", 33.724160e6 + 0.0),
    ("frame_solve", "frame_prefill"): (_FR_SRC, "d7a96b3509fa7060", 16.797184e6 + 0.0),
}


def ncu_traffic(kernel, workload):
    """Measured traffic of `kernel` on `workload` if its sources are unchanged
    since the capture, else None."""
    import hashlib
    ent = NCU_TRAFFIC.get((kernel, workload))
    if ent is None:
        return None
    h = hashlib.sha256()
    try:
        for f in ent[0]:
            with open(os.path.join(ROOT, "gated_delta_rule_90_b200", f), "rb") as fh:
                h.update(fh.read())
    except OSError:
        return None
    return ent[2] if h.hexdigest()[:16] == ent[1] else None


L2_FLUSH_BYTES = 256 << 20


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------- algorithmic work
def prefill_flops_per_token_head(C, dk, dv):
    """The 8 chunk GEMMs counted dense: K K^T, Q K^T (2 C d_k each), T V (2 C d_v),
    T K<- (2 C d_k), A Z (2 C d_v), W<- S^T, Q<- S^T, Z^T K-> (2 d_k d_v each)."""
    return 2 * C * (3 * dk + 2 * dv) + 6 * dk * dv


def prefill_flops_split(C, dk, dv):
    """(WY-transform share, state-pass share) of the flops per token-head."""
    wy = 2 * C * dk * 2 + 2 * C * dv + 2 * C * dk
    return wy, prefill_flops_per_token_head(C, dk, dv) - wy


def prefill_min_bytes(cfg, n_seq):
    """One read of q, k, v, g, beta, S0 and one write of out and S_final (k, v
    and beta once per substep when a token has n_h > 1 substeps)."""
    e = 2 if cfg.dtype == "bf16" else 4
    th = cfg.B * cfg.T * cfg.H
    nh = cfg.n_h
    gates = 4 * (cfg.d_k + cfg.d_v) if cfg.variant == "gdn2" else 4 * nh  # b, w or beta
    per = ((cfg.d_k + nh * (cfg.d_k + cfg.d_v)) * e + cfg.d_v * e + gates
           + (4 * cfg.d_k if cfg.gate == "channel" else 4))
    states = n_seq * cfg.H * cfg.d_k * cfg.d_v * 4 * ((1 if cfg.s0_var > 0 else 0) + 1)
    return th * per + states


def prefill_kernel_min_bytes(cfg, n_seq, kernel):
    """A prefill kernel's share of prefill_min_bytes: the WY pass reads the
    token inputs (q, k, v, g and beta or the GDN-2 gates) once; the state pass
    reads S0 and writes out and S_final once."""
    e = 2 if cfg.dtype == "bf16" else 4
    th = cfg.B * cfg.T * cfg.H
    states = n_seq * cfg.H * cfg.d_k * cfg.d_v * 4 * ((1 if cfg.s0_var > 0 else 0) + 1)
    out = th * cfg.d_v * e
    total = prefill_min_bytes(cfg, n_seq)
    return total - out - states if kernel == "tc_wy" else out + states


def decode_bytes(cfg):
    e = 2 if cfg.dtype == "bf16" else 4
    heads = cfg.N * cfg.H
    gb = 4 * cfg.d_k if cfg.gate == "channel" else 4
    return 2 * heads * cfg.d_k * cfg.d_v * 4 + heads * ((2 * cfg.d_k + 2 * cfg.d_v) * e + gb + 4)


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.proc = None
        self.gpu = gpu_index
        self.path = os.path.join("/tmp", f"gdr_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        busy = [s for s in sm if mx and s > 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(busy) if busy else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------- helpers
def dev_tensor(x, dtype, device):
    if x is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
    return t.to(device)


def max_over_ranks(x, world):
    if world <= 1:
        return x
    t = torch.tensor([x], dtype=torch.float64,
                     device="cuda" if torch.distributed.get_backend() == "nccl" else "cpu")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def aggregate(tokens_per_rank, ms_per_step, world):
    """Whole-job throughput of a weak-scaling run: every rank processed
    tokens_per_rank tokens per step; the job's step time is the slowest rank's.
    Returns (tokens/s over all ranks, max ms per step)."""
    ms = max_over_ranks(ms_per_step, world)
    return tokens_per_rank * world / (ms * 1e-3), ms


# ----------------------------------------------------------------- prefill
class PrefillRun:
    def __init__(self, cfg, device, seed, path):
        self.cfg = cfg
        self.device = device
        self.gdn2 = cfg.variant == "gdn2"
        gen = (inputs.gdn2_inputs if self.gdn2 else
               inputs.product_inputs if cfg.n_h > 1 else inputs.prefill_inputs)
        self.inp = gen(cfg, seed=seed)
        inp = self.inp
        self.n_seq = inp.n_seq
        self.q, self.k, self.v = (dev_tensor(x, cfg.dtype, device) for x in (inp.q, inp.k, inp.v))
        self.g = dev_tensor(inp.g, "f32", device)
        # Gated DeltaNet-2 passes its (erase, write) gates where the others pass beta
        self.beta = ((dev_tensor(inp.b, "f32", device), dev_tensor(inp.w, "f32", device))
                     if self.gdn2 else dev_tensor(inp.beta, "f32", device))
        self.S0 = dev_tensor(inp.S0, "f32", device)
        self.cu = None if inp.cu_seqlens is None else torch.from_numpy(inp.cu_seqlens).to(device)
        self.path = path
        self.out = torch.empty((cfg.B, cfg.T, cfg.H, cfg.d_v), dtype=self.q.dtype, device=device)
        self.SF = torch.empty((self.n_seq, cfg.H, cfg.d_v, cfg.d_k), dtype=torch.float32,
                              device=device)
        self.ws = torch.empty(max(self.ws_bytes(cfg.B, self.n_seq), 256), dtype=torch.uint8,
                              device=device)

    def ws_bytes(self, B, n_seq):
        cfg, path = self.cfg, self.path
        gate = 1 if cfg.gate == "channel" else 0
        dt = 1 if cfg.dtype == "bf16" else 0
        varlen = self.cu is not None
        if self.gdn2:
            return binding.fwd_gdn2_workspace_size(B, cfg.T, cfg.H, cfg.d_k, cfg.d_v, cfg.chunk,
                                                   n_seq, varlen, dt, gate, path)
        if cfg.n_h > 1:
            return binding.fwd_product_workspace_size(B, cfg.T, cfg.H, cfg.n_h, cfg.d_k, cfg.d_v,
                                                      cfg.chunk, n_seq, varlen, dt, gate, path)
        return binding.fwd_workspace_size(B, cfg.T, cfg.H, cfg.d_k, cfg.d_v, cfg.chunk, n_seq,
                                          varlen, dt, gate, path)

    def call(self, q, k, v, g, b, S0, cu, out=None, S_final=None, ws=None, stream=None):
        ws = self.ws if ws is None else ws
        if self.gdn2:
            return binding.gdr_fwd_gdn2(q, k, v, g, b[0], b[1], S0, chunk=self.cfg.chunk,
                                        cu_seqlens=cu, out=out, S_final=S_final, path=self.path,
                                        workspace=ws, stream=stream)
        fn = binding.gdr_fwd_product if self.cfg.n_h > 1 else binding.gdr_fwd
        return fn(q, k, v, g, b, S0, chunk=self.cfg.chunk, cu_seqlens=cu, out=out,
                  S_final=S_final, path=self.path, workspace=ws, stream=stream)

    def step(self):
        self.call(self.q, self.k, self.v, self.g, self.beta, self.S0, self.cu, self.out, self.SF)

    def tokens(self):
        return self.cfg.B * self.cfg.T

    def e2e(self, steps):
        """Same step through the C-ABI with pinned HOST buffers: H2D of every
        input, the call, D2H of out and S_final, all inside the timed region.
        A batch of B > 1 sequences goes as B per-sequence calls alternating
        over two streams, so that one sequence's inputs cross PCIe while the
        previous one computes and the one before that copies its outputs back
        (the link carries both directions at once); a packed batch is one call."""
        cfg, inp, dev = self.cfg, self.inp, self.device

        def host(x, dtype):
            if x is None:
                return None
            t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
            if dtype == "bf16":
                t = t.to(torch.bfloat16)
            return t.pin_memory()

        hq, hk, hv = (host(x, cfg.dtype) for x in (inp.q, inp.k, inp.v))
        hg, hS0 = host(inp.g, "f32"), host(inp.S0, "f32")
        hb = (host(inp.b, "f32"), host(inp.w, "f32")) if self.gdn2 else host(inp.beta, "f32")
        hcu = None if inp.cu_seqlens is None else torch.from_numpy(inp.cu_seqlens).pin_memory()
        hout = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        hSF = torch.empty(self.SF.shape, dtype=torch.float32).pin_memory()
        hbs = hb if isinstance(hb, tuple) else (hb,)
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hg, *hbs, hS0, hcu)
                  if t is not None)
        d2h = hout.numel() * hout.element_size() + hSF.numel() * hSF.element_size()
        st = torch.cuda.current_stream()
        pieces = cfg.B if hcu is None and cfg.B > 1 else 1
        if pieces > 1:
            streams = [torch.cuda.Stream(device=dev) for _ in range(2)]
            wsp = [torch.empty(max(self.ws_bytes(1, 1), 256), dtype=torch.uint8, device=dev)
                   for _ in range(2)]

            def sl(t, i):
                return None if t is None else t[i:i + 1]

            def one():
                start = torch.cuda.Event()
                start.record(st)
                for s_ in streams:
                    s_.wait_event(start)
                for i in range(pieces):
                    s_ = streams[i % 2]
                    with torch.cuda.stream(s_):
                        q, k, v, g = (sl(x, i).to(dev, non_blocking=True) for x in (hq, hk, hv, hg))
                        b = (tuple(sl(x, i).to(dev, non_blocking=True) for x in hb)
                             if isinstance(hb, tuple) else sl(hb, i).to(dev, non_blocking=True))
                        S0 = None if hS0 is None else sl(hS0, i).to(dev, non_blocking=True)
                        out, SF = self.call(q, k, v, g, b, S0, None, ws=wsp[i % 2], stream=s_)
                        hout[i:i + 1].copy_(out, non_blocking=True)
                        hSF[i:i + 1].copy_(SF, non_blocking=True)
                for s_ in streams:
                    done = torch.cuda.Event()
                    done.record(s_)
                    st.wait_event(done)
        else:
            def one():
                q = hq.to(dev, non_blocking=True)
                k = hk.to(dev, non_blocking=True)
                v = hv.to(dev, non_blocking=True)
                g = hg.to(dev, non_blocking=True)
                b = (tuple(x.to(dev, non_blocking=True) for x in hb) if isinstance(hb, tuple)
                     else hb.to(dev, non_blocking=True))
                S0 = None if hS0 is None else hS0.to(dev, non_blocking=True)
                cu = None if hcu is None else hcu.to(dev, non_blocking=True)
                out, SF = self.call(q, k, v, g, b, S0, cu)
                hout.copy_(out, non_blocking=True)
                hSF.copy_(SF, non_blocking=True)

        one()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        for _ in range(steps):
            one()
        e1.record(st)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / steps
        # the host copies against the device-resident step's results (same kernels, same inputs)
        self.e2e_matches = bool(torch.equal(hout.to(dev), self.out) and torch.equal(hSF.to(dev), self.SF))
        self.e2e_pieces = pieces
        return ms, h2d, d2h


# ----------------------------------------------------------------- frame update
class FrameRun:
    """The implicit frame-level update over a batch of frames."""

    def __init__(self, cfg, device, seed):
        self.cfg = cfg
        self.device = device
        self.inp = inp = inputs.frame_inputs(cfg, seed=seed)
        self.q, self.k, self.v = (dev_tensor(x, cfg.dtype, device) for x in (inp.q, inp.k, inp.v))
        self.g, self.gamma = dev_tensor(inp.g, "f32", device), dev_tensor(inp.gamma, "f32", device)
        self.S0 = dev_tensor(inp.S0, "f32", device)
        self.out = torch.empty((cfg.B, cfg.T, cfg.H, cfg.d_v), dtype=self.q.dtype, device=device)
        self.SF = torch.empty((cfg.B, cfg.H, cfg.d_v, cfg.d_k), dtype=torch.float32, device=device)
        ws = binding.fwd_frame_workspace_size(cfg.B, cfg.T, cfg.H, cfg.d_k, cfg.d_v, cfg.n)
        self.ws = torch.empty(max(ws, 256), dtype=torch.uint8, device=device)
        self.n_seq = cfg.B

    def step(self):
        binding.gdr_fwd_frame(self.q, self.k, self.v, self.g, self.gamma, self.cfg.n, self.S0,
                              out=self.out, S_final=self.SF, workspace=self.ws)

    def tokens(self):
        return self.cfg.B * self.cfg.T


def frame_flops_per_token_head(dk, dv, n):
    """The method's own count: G_t and C_t (2 d_k (d_k + d_v) per token), the
    output (2 d_k d_v per token), and per frame a Cholesky of I + G_t
    (d_k^3 / 3) and the two triangular solves for the d_v rows of S_t
    (2 d_v d_k^2), spread over the frame's n tokens.  The kernels form the
    whole inverse instead (2 d_k^3 flops by the sweep) and multiply by it
    (2 d_v d_k^2); the extra work is not counted."""
    per_frame = dk ** 3 / 3 + 2 * dv * dk * dk
    return 2 * dk * (dk + dv) + 2 * dk * dv + per_frame / n


# ----------------------------------------------------------------- decode
class DecodeRun:
    """The decode workload: fresh tokens every step (drawn on the device from a
    seeded generator before the timed region), state updated in place."""

    def __init__(self, cfg, device, seed, n_steps):
        self.cfg = cfg
        self.device = device
        self.S = torch.from_numpy(inputs.decode_state(cfg, seed=seed)).to(device)
        gen = torch.Generator(device=device)
        gen.manual_seed(seed)
        N, H, dk, dv = cfg.N, cfg.H, cfg.d_k, cfg.d_v
        tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32

        def unit(shape):
            x = torch.randn(shape, generator=gen, device=device)
            return (x / x.norm(dim=-1, keepdim=True)).to(tdt)

        P = self.pool = max(1, n_steps)
        self.q = unit((P, N, H, dk))
        self.k = unit((P, N, H, dk))
        self.v = torch.randn((P, N, H, dv), generator=gen, device=device).to(tdt)
        self.b = torch.sigmoid(torch.randn((P, N, H), generator=gen, device=device))
        gshape = (P, N, H, dk) if cfg.gate == "channel" else (P, N, H)
        self.g = -torch.nn.functional.softplus(torch.randn(gshape, generator=gen, device=device)) * cfg.gate_scale
        self.out = torch.empty((N, H, dv), dtype=tdt, device=device)
        self.i = 0

    def step(self):
        j = self.i % self.pool
        self.i += 1
        binding.gdr_decode_step(self.q[j], self.k[j], self.v[j], self.g[j], self.b[j], self.S,
                                out=self.out)

    def tokens(self):
        return self.cfg.N


# ----------------------------------------------------------------- CPU oracle
def oracle_prefill_sample(cfg, seed, budget_s):
    """Time the fp64 oracle on a bounded sample of the workload: the first h
    heads of every sequence, h chosen so the run takes about budget_s seconds.
    Returns (equivalent tokens/s, cores, description)."""
    import oracle  # CPU baseline leg only

    product, gdn2 = cfg.n_h > 1, cfg.variant == "gdn2"
    gen = inputs.gdn2_inputs if gdn2 else inputs.product_inputs if product else inputs.prefill_inputs
    inp = gen(cfg, seed=seed)
    cores = 1 if (product or gdn2) else oracle.default_threads()

    def run(h):
        sl = lambda x: None if x is None else np.ascontiguousarray(x[:, :, :h])
        sl3 = lambda x: np.ascontiguousarray(x[:, :, :, :h])  # [B, T, n_h, H, ...]
        S0 = None if inp.S0 is None else np.ascontiguousarray(inp.S0[:, :h])
        t = time.perf_counter()
        if gdn2:
            oracle.gdn2_fwd(sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.g), sl(inp.b), sl(inp.w), S0,
                            inp.cu_seqlens)
        elif product:
            oracle.product_fwd(sl(inp.q), sl3(inp.k), sl3(inp.v), sl(inp.g), sl3(inp.beta), S0,
                               inp.cu_seqlens)
        else:
            oracle.recurrence_fwd(sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.g), sl(inp.beta),
                                  S0=S0, cu_seqlens=inp.cu_seqlens, threads=cores)
        return time.perf_counter() - t

    t1 = run(1)
    per_head = t1  # one head of every sequence
    h = int(max(1, min(cfg.H, budget_s / max(per_head, 1e-6))))
    if h > 1:
        dt = run(h)
    else:
        dt = t1
    token_heads = cfg.B * cfg.T * h
    return (token_heads / cfg.H) / dt, cores, (f"{h} of {cfg.H} heads x all {cfg.B * cfg.T} "
                                               f"tokens ({token_heads} token-heads, {dt:.2f} s)"), dt


def oracle_frame_sample(cfg, seed, budget_s):
    """The frame-update oracle on the first h heads (single-threaded)."""
    import oracle

    inp = inputs.frame_inputs(cfg, seed=seed)

    def run(h):
        sl = lambda x: np.ascontiguousarray(x[:, :, :h])
        S0 = None if inp.S0 is None else np.ascontiguousarray(inp.S0[:, :h])
        t = time.perf_counter()
        oracle.frame_fwd(sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.g), sl(inp.gamma), cfg.n, S0)
        return time.perf_counter() - t

    t1 = run(1)
    h = int(max(1, min(cfg.H, budget_s / max(t1, 1e-6))))
    dt = run(h) if h > 1 else t1
    return (cfg.B * cfg.T * h / cfg.H) / dt, 1, (f"{h} of {cfg.H} heads x all {cfg.B * cfg.T} "
                                                 f"tokens ({dt:.2f} s)"), dt


def oracle_decode_sample(cfg, seed, budget_s):
    import oracle

    S = inputs.decode_state(cfg, seed=seed).astype(np.float64)
    t0 = time.perf_counter()
    steps = 0
    while time.perf_counter() - t0 < budget_s and steps < cfg.steps:
        tok = inputs.decode_token(cfg, steps, seed=seed)
        t = time.perf_counter()
        _, S = oracle.recurrence_decode_step(tok.q, tok.k, tok.v, tok.g, tok.beta, S)
        steps += 1
        if steps == 1:
            t_compute = time.perf_counter() - t
        else:
            t_compute += time.perf_counter() - t
    return cfg.N * steps / t_compute, 1, f"{steps} full decode steps ({cfg.N}x{cfg.H} heads)", t_compute


# ----------------------------------------------------------------- main
def workload_config(name):
    if name in inputs.PREFILL:
        c = inputs.PREFILL[name]
        return c, {"workload": name, "B": c.B, "T": c.T, "H": c.H, "d_k": c.d_k, "d_v": c.d_v,
                   "chunk": c.chunk, "gate": c.gate, "dtype_io": c.dtype,
                   **({"n_seq": c.n_seq} if c.n_seq else {}),
                   **({"n_h": c.n_h} if c.n_h > 1 else {}),
                   **({"variant": c.variant} if c.variant else {})}
    if name in inputs.FRAME:
        c = inputs.FRAME[name]
        return c, {"workload": name, "B": c.B, "T": c.T, "H": c.H, "d_k": c.d_k, "d_v": c.d_v,
                   "frame_tokens": c.n, "frames": c.frames, "gate": c.gate, "dtype_io": c.dtype}
    c = inputs.DECODE[name]
    return c, {"workload": name, "N": c.N, "H": c.H, "d_k": c.d_k, "d_v": c.d_v, "gate": c.gate,
               "dtype_io": c.dtype, "steps_per_sequence": c.steps}


L2_NOTE_FLUSHED = (f"flushed between steps ({L2_FLUSH_BYTES >> 20} MiB write, then a "
                   f"{L2_FLUSH_BYTES >> 20} MiB read of another buffer, outside the per-step "
                   "CUDA-event intervals)")
L2_NOTE_DECODE = "no flush: the 512 MiB state is larger than L2 and is streamed every step"


def full_config(name, path, world):
    """The workload's config as both arms print it: its shapes plus the L2
    treatment, the kernel path and the replica count."""
    cfg, conf = workload_config(name)
    is_decode = isinstance(cfg, inputs.DecodeConfig)
    conf["l2"] = L2_NOTE_DECODE if is_decode else L2_NOTE_FLUSHED
    if not is_decode and not isinstance(cfg, inputs.FrameConfig):
        conf["path"] = path
    conf["parallelism"] = f"replicas x{world}"
    return cfg, conf


class L2Flush:
    """Leaves L2 cold and clean between steps: writes one buffer larger than L2,
    then reads a second one, so the dirty lines of the write are written back
    before the next timed interval starts instead of inside it."""

    def __init__(self, device):
        self.w = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
        self.r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
        self.acc = torch.empty((), dtype=torch.float32, device=device)

    def zero_(self):
        self.w.zero_()
        torch.sum(self.r, dim=0, out=self.acc)


def time_steps(run, steps, flush):
    """Per-step CUDA-event times (ms) on the launching stream; L2 flushed
    between steps (outside the timed intervals) when `flush` is given."""
    st = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for a, b in evs:
        if flush is not None:
            flush.zero_()
        a.record(st)
        run.step()
        b.record(st)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def run_reference(args, rank, world):
    """Reference arm: the fp64 CPU oracle, timed as it stands on the host cores."""
    if rank != 0:
        return
    cfg, conf = full_config(args.workload, args.path, world)
    budget = max(0.5, args.ref_budget_s / max(1, args.steps + args.warmup))
    vals = []
    if isinstance(cfg, inputs.DecodeConfig):
        for i in range(args.warmup + args.steps):
            v, cores, sample, _ = oracle_decode_sample(cfg, inputs.BASE_SEED + cfg.seed_index,
                                                       budget)
            if i >= args.warmup:
                vals.append(v)
    elif isinstance(cfg, inputs.FrameConfig):
        for i in range(args.warmup + args.steps):
            v, cores, sample, _ = oracle_frame_sample(cfg, inputs.BASE_SEED + cfg.seed_index,
                                                      budget)
            if i >= args.warmup:
                vals.append(v)
    else:
        for i in range(args.warmup + args.steps):
            v, cores, sample, _ = oracle_prefill_sample(cfg, inputs.BASE_SEED + cfg.seed_index,
                                                        budget)
            if i >= args.warmup:
                vals.append(v)
    value = statistics.median(vals)
    tok = cfg.N if isinstance(cfg, inputs.DecodeConfig) else cfg.B * cfg.T
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * tok / value, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": conf,
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def measure(args, name, device, rank, world, peaks, peak_kind, path, steps, warmup,
            with_cpu, with_e2e, sampler=None):
    cfg, conf = full_config(name, path, world)
    seed = (inputs.BASE_SEED + cfg.seed_index) * 1000 + rank
    is_decode = isinstance(cfg, inputs.DecodeConfig)
    is_frame = isinstance(cfg, inputs.FrameConfig)
    run = (DecodeRun(cfg, device, seed, steps + warmup) if is_decode
           else FrameRun(cfg, device, seed) if is_frame
           else PrefillRun(cfg, device, seed, path))
    flush = None if is_decode else L2Flush(device)
    for _ in range(warmup):
        if flush is not None:
            flush.zero_()
        run.step()
    torch.cuda.synchronize()
    binding.profile_read()  # reset counters
    binding.profile_enable(True)
    if sampler:
        sampler.start()
    barrier(world)
    torch.cuda.synchronize()
    w0 = time.perf_counter()
    times = time_steps(run, steps, flush)
    torch.cuda.synchronize()
    barrier(world)
    wall = time.perf_counter() - w0
    clocks = sampler.stop() if sampler else None
    binding.profile_enable(False)
    prof = binding.profile_read()
    assert binding.device_status() == binding.GDR_OK
    value, ms = aggregate(run.tokens(), sum(times) / len(times), world)
    tokens_all = run.tokens() * world
    kernels = {k: {"launches": n, "avg_ms": (t / n if n else 0.0)} for k, (n, t) in prof.items()
               if n}
    launches = sum(n for n, _ in prof.values())

    # roofline of the dominant kernel
    dom = max(kernels.items(), key=lambda kv: kv[1]["avg_ms"] * kv[1]["launches"])[0]
    dom_ms = kernels[dom]["avg_ms"]
    if is_decode:
        B_ = decode_bytes(cfg)
        ach = B_ / (dom_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "kernel": dom, "achieved": ach, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": ach / peaks["hbm_gbs"], "traffic": ncu_traffic(dom, name),
                "peak_source": peak_kind + " hbm_gbs", "algorithmic_bytes_per_launch": B_,
                "frac_of_8TBps_spec": ach / 8000.0}
    elif is_frame:
        # the dominant pass against its own roof: for bf16 d = 128 the token
        # contractions (Gram, output) and the chain run on the tensor cores (the
        # chain's flops counted once, though its bf16 split executes three
        # products); the factorisation, and every pass of the fp32 path, is
        # fp32 CUDA-core work
        th = cfg.B * cfg.T * cfg.H
        fh = cfg.B * cfg.frames * cfg.H
        dk, dv = cfg.d_k, cfg.d_v
        tc_path = cfg.dtype == "bf16" and dk == 128 and dv == 128
        pflops = {"frame_gram": 2 * dk * (dk + dv) * th, "frame_out": 2 * dk * dv * th,
                  "frame_solve": dk ** 3 / 3 * fh,
                  "frame_chain": 2 * dv * dk * dk * fh}
        flops = pflops.get(dom, 0)
        on_tc = tc_path and dom in ("frame_gram", "frame_out", "frame_chain")
        alu_peak = SM_COUNT * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
        peak = peaks["bf16_tflops"] if on_tc else alu_peak
        ach = flops / (dom_ms * 1e-3) / 1e12
        roof = {"bound": "tensor" if on_tc else "alu", "kernel": dom, "achieved": ach,
                "peak": peak, "unit": "TFLOP/s", "frac": ach / peak, "traffic": ncu_traffic(dom, name),
                "peak_source": (peak_kind + " bf16_tflops (burst)") if on_tc else
                "fp32 FMA: 148 SMs x 128 lanes x 2 flop x max SM clock",
                "algorithmic_flops_per_launch": flops,
                "step": {"tflops": frame_flops_per_token_head(dk, dv, cfg.n) * th / (ms * 1e-3) / 1e12}}
    else:
        th = cfg.B * cfg.T * cfg.H * cfg.n_h  # virtual steps when a token has substeps
        f_all = prefill_flops_per_token_head(cfg.chunk, cfg.d_k, cfg.d_v)
        wy, st_ = prefill_flops_split(cfg.chunk, cfg.d_k, cfg.d_v)
        share = {"fwd_simt": f_all, "gdn2_simt": f_all, "tc_wy": wy, "tc_state": st_}.get(dom, 0)
        flops = share * th
        if dom in ("fwd_simt", "gdn2_simt"):
            peak = SM_COUNT * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
            ach = flops / (dom_ms * 1e-3) / 1e12
            roof = {"bound": "alu", "kernel": dom, "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                    "frac": ach / peak, "traffic": None,
                    "peak_source": "fp32 FMA: 148 SMs x 128 lanes x 2 flop x max SM clock",
                    "algorithmic_flops_per_launch": flops}
        else:
            # Both roofs of the kernel's share of the step's algorithmic work: its
            # share of the chunk GEMM flops, and its share of the minimum bytes
            # (the WY pass reads the inputs once, the state pass reads S0 and
            # writes out and S_final once).  The binding roof is the one that
            # takes longer at the measured peaks.
            sh_bytes = prefill_kernel_min_bytes(cfg, run.n_seq, dom)
            t_tc = flops / (peaks["bf16_tflops"] * 1e12)
            t_hbm = sh_bytes / (peaks["hbm_gbs"] * 1e9)
            sec = dom_ms * 1e-3
            tc = {"achieved": flops / sec / 1e12, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                  "frac": flops / sec / 1e12 / peaks["bf16_tflops"],
                  "algorithmic_flops_per_launch": flops,
                  "peak_source": peak_kind + " bf16_tflops (burst)"}
            hb = {"achieved": sh_bytes / sec / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                  "frac": sh_bytes / sec / 1e9 / peaks["hbm_gbs"],
                  "algorithmic_bytes_per_launch": sh_bytes,
                  "peak_source": peak_kind + " hbm_gbs"}
            top = hb if t_hbm > t_tc else tc
            roof = {"bound": "hbm" if t_hbm > t_tc else "tensor", "kernel": dom,
                    "achieved": top["achieved"], "peak": top["peak"], "unit": top["unit"],
                    "frac": top["frac"], "traffic": ncu_traffic(dom, name),
                    "peak_source": top["peak_source"], "tensor_view": tc, "hbm_view": hb}
        min_bytes = prefill_min_bytes(cfg, run.n_seq)
        roof["step"] = {"tflops": f_all * th / (ms * 1e-3) / 1e12,
                        "tc_frac": f_all * th / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                        "hbm_gbs_min_bytes": min_bytes / (ms * 1e-3) / 1e9,
                        "hbm_frac": min_bytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                        "flops_per_step": f_all * th, "min_bytes_per_step": min_bytes}
        # the whole step against the bf16 tensor-core peak (the end-to-end
        # fraction the prefill target is stated in), next to the dominant
        # kernel's own fraction above
        roof["frac_is"] = f"dominant kernel {dom}: {roof['bound']} roof of its algorithmic share"
        roof["step_tc_frac"] = roof["step"]["tc_frac"]
        roof["step_hbm_frac"] = roof["step"]["hbm_frac"]
        roof["step_tflops"] = roof["step"]["tflops"]
    res = {"value": value, "ms_per_step": ms, "wall_s_incl_flush": wall, "roofline": roof,
           "kernels": kernels, "gpu_launches": launches, "clocks": clocks, "config": conf,
           "cfg": cfg, "run": run}
    if with_e2e and not is_decode and not is_frame:
        e_ms, h2d, d2h = run.e2e(max(1, min(steps, 5)))
        e_ms = max_over_ranks(e_ms, world)
        res["e2e"] = {"value": tokens_all / (e_ms * 1e-3), "unit": "tokens/s",
                      "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms,
                      "calls_per_step": run.e2e_pieces, "streams": 2 if run.e2e_pieces > 1 else 1,
                      "matches_device_path": run.e2e_matches}
    if with_cpu and rank == 0 and world == 1:
        if is_decode:
            v, cores, sample, _ = oracle_decode_sample(cfg, seed, 10.0)
        elif is_frame:
            v, cores, sample, _ = oracle_frame_sample(cfg, seed, 10.0)
        else:
            v, cores, sample, _ = oracle_prefill_sample(cfg, seed, 10.0)
        res["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                               "sample": sample}
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="gdn_prefill",
                    choices=list(inputs.PREFILL) + list(inputs.DECODE) + list(inputs.FRAME))
    ap.add_argument("--path", default="auto", choices=["auto", "simt", "tc"])
    ap.add_argument("--extra", default=("kda_prefill,varlen_prefill,gdp_prefill,gdn2_prefill,"
                                        "frame_prefill,gdn_prefill_c16,kda_prefill_c16,"
                                        "gdn_prefill_c128,decode,kda_decode"),
                    help="comma-separated workloads measured after the main one ('' for none)")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--ref-budget-s", type=float, default=90.0)
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
            return
        device = torch.device("cuda", local)
        torch.cuda.set_device(device)
        binding.lib()
        peaks, peak_kind = load_peaks()
        sampler = ClockSampler(local) if rank == 0 else None
        main_res = measure(args, args.workload, device, rank, world, peaks, peak_kind, args.path,
                           args.steps, args.warmup, not args.no_cpu, not args.no_e2e, sampler)
        extra = {}
        for name in [x for x in args.extra.split(",") if x and x != args.workload]:
            steps = 200 if name in inputs.DECODE else 20
            r = measure(args, name, device, rank, world, peaks, peak_kind, args.path, steps, 3,
                        False, False, None)
            # compact, so that the line's tail holds every extra workload
            rf = r["roofline"]
            extra[name] = {"ms_per_step": round(r["ms_per_step"], 5),
                           "tokens_per_s": round(r["value"], 1), "steps": steps,
                           "roofline": {"kernel": rf["kernel"], "bound": rf["bound"],
                                        "frac": round(rf["frac"], 4),
                                        **({"step_tc_frac": round(rf["step_tc_frac"], 4)}
                                           if "step_tc_frac" in rf else {})},
                           "kernel_ms": {k: round(v["avg_ms"], 5) for k, v in r["kernels"].items()}}
            del r
            torch.cuda.empty_cache()
        if rank == 0:
            cfg = main_res["cfg"]
            line = {"metric": METRIC, "value": main_res["value"], "unit": "tokens/s",
                    "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                    "ms_per_step": main_res["ms_per_step"], "higher_is_better": True,
                    "scaling": "weak", "vs_baseline": None,
                    "dtype": "bf16" if getattr(cfg, "dtype", "bf16") == "bf16" else "f32",
                    "data": "synthetic (seeded; shapes and distributions of the workload)",
                    "config": main_res["config"],
                    "roofline": main_res["roofline"], "e2e": main_res.get("e2e"),
                    "gpu_launches": main_res["gpu_launches"], "clocks": main_res["clocks"],
                    "kernels": main_res["kernels"], "cpu_baseline": main_res.get("cpu_baseline"),
                    "extra": extra}
            print(json.dumps(line), flush=True)
    finally:
        if world > 1 and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
