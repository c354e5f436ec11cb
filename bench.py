#!/usr/bin/env python
"""Benchmark of the Falcon fast-weight forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl falcon|reference]

One step = one chunk-parallel forward pass (falcon_fwd_chunk: prep, chunk-local
solve and state propagation, fused in one kernel) of Falcon-1 over the
workload B8 H16 T4096 d128, chunk 64, bf16 q/k/v, fp32 state (synthetic seeded
inputs resident in HBM; 549.5 MB per step, larger than the 126 MB L2, so no
flush is needed between steps). The same run also times the single-token
decode step (256 sequences x 32 heads, 128x128 fp32 state, 1000 repeated
steps) and reports its HBM GB/s, and the fp32 recurrent form on its small
workload.

Multi-GPU (torchrun, one rank per GPU): every rank runs its own independent
batch (weak scaling, no collective on the data path); the timed region is
bracketed by barriers and the max over ranks is taken.

--impl reference times the fp64 CPU oracle (the only reference this method
has) on a bounded sample of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Falcon-1 chunk fwd tokens/s & % roofline (B8 H16 T4K d128); decode GB/s"
FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS = 6650.0, 1590.0
CHUNK_KERNEL_SOURCES = ["chunk_ws.cu", "tc_common.cuh", "common.cuh"]


# ----------------------------------------------------------------------------- helpers

def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def kernel_source_hash(files):
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, "delta_rule_linear_falcon_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, files):
    """DRAM bytes per launch from a committed ncu capture, if the kernel source is unchanged."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(kernel)
    if not rec or rec.get("source_sha256_16") != kernel_source_hash(files):
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self.ok = False
        self._stop = threading.Event()
        self._th = None
        try:
            import pynvml as N
            N.nvmlInit()
            self.N = N
            h = None
            try:
                import torch
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
                h = N.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
            except Exception:
                h = N.nvmlDeviceGetHandleByIndex(device_index)
            self.h = h
            self.max_mhz = N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML missing: report no clocks rather than guess
            self.err = repr(e)

    def _run(self):
        N = self.N
        while not self._stop.is_set():
            try:
                self.samples.append(N.nvmlDeviceGetClockInfo(self.h, N.NVML_CLOCK_SM))
                try:
                    r = N.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except Exception:
                    r = N.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        self._stop.clear()
        if self.ok:
            self._th = threading.Thread(target=self._run, daemon=True)
            self._th.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._th:
            self._th.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "NVML unavailable"}
        busy = [s for s in self.samples]
        return {"sm_mhz": statistics.median(busy) if busy else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(busy),
                "source": "NVML, sampled every 2 ms during the timed regions"}


# ----------------------------------------------------------------------------- workload sizes

def chunk_algorithmic_bytes(B, H, T, dk, dv, io_bytes=2):
    """Bytes the forward pass must move at minimum: read q, k, v, alpha, eta once,
    write o, the final state and the continuation key once."""
    n = B * H * T
    return (n * (2 * dk + dv) * io_bytes + n * 2 * 4 + n * dv * io_bytes
            + B * H * dv * dk * 4 + B * H * dk * io_bytes)


def chunk_algorithmic_flops(B, H, T, dk, dv, window=1):
    """Recurrent-form FLOPs: (3 + 4w) dk dv per token-head (7 dk dv for Falcon-1)."""
    return (3 + 4 * window) * dk * dv * B * H * T


def decode_algorithmic_bytes(N, H, dk, dv, io_bytes=2):
    nh = N * H
    return (nh * dv * dk * 4 * 2          # state read + write
            + nh * (2 * dk + dv) * io_bytes  # q, k, v
            + nh * dk * io_bytes * 2       # k_prev read + write
            + nh * 2 * 4                   # alpha, eta
            + nh * dv * io_bytes)          # o


# ----------------------------------------------------------------------------- distributed

class Dist:
    """One process per GPU (torchrun env). NCCL on GPUs; gloo for CPU tests.
    Only the timing reduction and barriers cross ranks: no data-path collective."""

    def __init__(self, backend: str = "nccl"):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.backend = backend
        self.pg = None
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            kw = {}
            if backend == "nccl":
                import torch
                torch.cuda.set_device(self.local)
                kw["device_id"] = torch.device("cuda", self.local)
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
            self.pg = dist

    def barrier(self):
        if self.pg:
            if self.backend == "nccl":
                import torch
                self.pg.barrier(device_ids=[self.local])
                torch.cuda.synchronize()
            else:
                self.pg.barrier()

    def max(self, x: float) -> float:
        if not self.pg:
            return x
        import torch
        dev = "cuda" if self.backend == "nccl" else "cpu"
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()
            self.pg = None


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own independent batch (weak scaling)."""
    return base_seed + 1000 * rank


def weak_scaling_value(units_per_rank: float, world: int, max_ms: float) -> float:
    """Whole-job throughput: units processed by all ranks / slowest rank's time."""
    return units_per_rank * world / (max_ms * 1e-3)


# ----------------------------------------------------------------------------- GPU arms

def bench_chunk(args, D: Dist, clk):
    import torch
    from delta_rule_linear_falcon_b200 import falcon as F
    from delta_rule_linear_falcon_b200 import inputs as I

    s = I.make_seq(I.RULE_1, args.batch, 16, args.seq_len, 128, 128, seed=rank_seed(1, D.rank), io_dtype="bf16",
                   normalise_qk=True, alpha_mu=4.0, chunk=64)
    B, H, T, dk, dv = s.shape
    dev = torch.device("cuda", D.local)
    hq, hk, hv = (torch.from_numpy(x).to(torch.bfloat16).pin_memory() for x in (s.q, s.k, s.v))
    ha, he = (torch.from_numpy(x).pin_memory() for x in (s.alpha, s.eta))
    q, k, v, a, e = (x.to(dev) for x in (hq, hk, hv, ha, he))
    o = torch.empty((B, H, T, dv), dtype=torch.bfloat16, device=dev)
    S = torch.empty((B, H, dv, dk), dtype=torch.float32, device=dev)
    kl = torch.empty((B, H, dk), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    # the two-pass path's tiles (every block's solved T_f, T'), allocated once like the outputs
    need = F.falcon_workspace_size(F.make_args(q, k, v, a, e, rule=1, eps=s.eps, chunk=64, o=o, S_out=S,
                                               k_last=kl))
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)

    def step():
        F.falcon_fwd_chunk(q, k, v, a, e, rule=1, eps=s.eps, chunk=64, o=o, S_out=S, k_last=kl,
                           workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    D.barrier()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with clk:
        t0.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
    D.barrier()
    total_ms = D.max(t0.elapsed_time(t1))
    kern_ms = statistics.mean(a_.elapsed_time(b_) for a_, b_ in ev)
    assert F.falcon_check_device_errors(stream) == F.FALCON_OK
    assert torch.isfinite(o.float()).all().item()

    # End to end through the same C-ABI call from pinned host buffers. Every step uploads its
    # inputs and downloads its outputs (o and the final state), as a serving loop would: the
    # upload of step i+1 (copy stream), the kernel of step i (compute stream) and the download
    # of step i-1 (second copy stream) overlap, with two device buffer sets and events between
    # the streams. The timed region runs from before the first upload to after the last download.
    ho = [torch.empty((B, H, T, dv), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    hS = [torch.empty((B, H, dv, dk), dtype=torch.float32).pin_memory() for _ in range(2)]
    ins = [(q, k, v, a, e), tuple(torch.empty_like(x) for x in (q, k, v, a, e))]
    outs = [(o, S, kl), tuple(torch.empty_like(x) for x in (o, S, kl))]
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_run(n):
        ready = [torch.cuda.Event() for _ in range(2)]      # inputs of a buffer set uploaded
        used = [torch.cuda.Event() for _ in range(2)]       # kernel done with a buffer set
        fetched = [torch.cuda.Event() for _ in range(2)]    # outputs of a buffer set downloaded
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)

        def upload(i):
            b = i % 2
            # the buffer set is free once the kernel of step i-2 is done with it
            up.wait_event(used[b] if i >= 2 else start)
            with torch.cuda.stream(up):
                for dst, src in zip(ins[b], (hq, hk, hv, ha, he)):
                    dst.copy_(src, non_blocking=True)
            ready[b].record(up)

        upload(0)
        for i in range(n):
            b = i % 2
            if i + 1 < n:
                upload(i + 1)
            stream.wait_event(ready[b])
            if i >= 2:
                stream.wait_event(fetched[b])               # outputs of step i-2 are on the host
            qq, kk, vv, aa, ee = ins[b]
            oo, SS, kk_last = outs[b]
            F.falcon_fwd_chunk(qq, kk, vv, aa, ee, rule=1, eps=s.eps, chunk=64, o=oo, S_out=SS,
                               k_last=kk_last, workspace=ws, stream=stream)
            used[b].record(stream)
            down.wait_event(used[b])
            with torch.cuda.stream(down):
                ho[b].copy_(oo, non_blocking=True)
                hS[b].copy_(SS, non_blocking=True)
            fetched[b].record(down)
        stream.wait_stream(down)
        end.record(stream)
        return start, end

    for _ in range(max(1, min(args.warmup, 3))):
        e2e_run(2)
    torch.cuda.synchronize()
    D.barrier()
    n_e2e = max(2, min(args.steps, 20))
    with clk:
        e0, e1 = e2e_run(n_e2e)
        torch.cuda.synchronize()
    D.barrier()
    e2e_ms = D.max(e0.elapsed_time(e1)) / n_e2e
    # the last download is the output of the same inputs as the device-resident run
    assert torch.equal(ho[(n_e2e - 1) % 2], o.cpu())
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, ha, he))
    d2h = ho[0].numel() * ho[0].element_size() + hS[0].numel() * hS[0].element_size()
    return dict(s=s, total_ms=total_ms, kern_ms=kern_ms, e2e_ms=e2e_ms, h2d=h2d, d2h=d2h,
                launches=2 if need else 1, workspace_bytes=need)


def bench_decode(args, D: Dist, clk):
    import torch
    from delta_rule_linear_falcon_b200 import falcon as F
    from delta_rule_linear_falcon_b200 import inputs as I

    d = I.workload_decode(N=args.decode_seqs, seed=rank_seed(4, D.rank))
    dev = torch.device("cuda", D.local)
    S = torch.from_numpy(d.S).to(dev)
    kp = torch.from_numpy(d.k_prev).to(torch.bfloat16).to(dev)
    P = d.q.shape[0]
    toks = [tuple(torch.from_numpy(x[p]).to(dt).to(dev) for x, dt in
                  ((d.q, torch.bfloat16), (d.k, torch.bfloat16), (d.v, torch.bfloat16),
                   (d.alpha, torch.float32), (d.eta, torch.float32))) for p in range(P)]
    N, H, dv, dk = S.shape
    o = torch.empty((N, H, dv), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    for i in range(max(args.warmup, 3)):
        F.falcon_decode_step(S, kp, *toks[i % P], rule=1, eps=d.eps, o=o, stream=stream)
    torch.cuda.synchronize()
    D.barrier()
    n = args.decode_steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with clk:
        t0.record(stream)
        for i in range(n):
            F.falcon_decode_step(S, kp, *toks[i % P], rule=1, eps=d.eps, o=o, stream=stream)
        t1.record(stream)
        torch.cuda.synchronize()
    D.barrier()
    ms = D.max(t0.elapsed_time(t1)) / n
    assert F.falcon_check_device_errors(stream) == F.FALCON_OK
    assert torch.isfinite(S).all().item()
    return dict(N=N, H=H, dk=dk, dv=dv, ms=ms, steps=n)


def bench_recurrent(args, D: Dist):
    import torch
    from delta_rule_linear_falcon_b200 import falcon as F
    from delta_rule_linear_falcon_b200 import inputs as I

    s = I.workload_recurrent_small()
    dev = torch.device("cuda", D.local)
    q, k, v, a, e = (torch.from_numpy(x).to(dev) for x in (s.q, s.k, s.v, s.alpha, s.eta))
    stream = torch.cuda.current_stream(dev)
    run = lambda: F.falcon_fwd_recurrent(q, k, v, a, e, rule=1, eps=s.eps, stream=stream)
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(20):
        run()
    t1.record(stream)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / 20
    B, H, T, dk, dv = s.shape
    out = {"workload": s.name, "ms_per_call": round(ms, 4),
           "tokens_per_s": round(B * T / (ms * 1e-3), 1), "note": "latency bound, parity workload"}
    # The per-column rules (Falcon-2 / 2A) run on the recurrent kernel only: one head per CTA walks
    # its tokens one by one, so a full-width problem shows that path's own rate.
    per_col = {}
    for rule, name in ((5, "falcon2"), (6, "falcon2a")):
        s2 = I.make_seq(rule, 1, 16, 4096, 128, 128, seed=11, io_dtype="bf16")
        q2, k2, v2 = (torch.from_numpy(x).to(torch.bfloat16).to(dev) for x in (s2.q, s2.k, s2.v))
        a2, e2 = (torch.from_numpy(x).to(dev) for x in (s2.alpha, s2.eta))
        n_out = torch.empty((1, 16, 128), dtype=torch.float32, device=dev)
        run2 = lambda: F.falcon_fwd_recurrent(q2, k2, v2, a2, e2, rule=rule, eps=s2.eps, n_out=n_out,
                                              stream=stream)
        for _ in range(2):
            run2()
        torch.cuda.synchronize()
        t0.record(stream)
        for _ in range(3):
            run2()
        t1.record(stream)
        torch.cuda.synchronize()
        ms2 = t0.elapsed_time(t1) / 3
        per_col[f"{name}_recurrent_bf16_B1H16T4096d128"] = {
            "ms_per_call": round(ms2, 3), "tokens_per_s": round(4096 / (ms2 * 1e-3), 1),
            "note": "recurrent kernel (the only path of the per-column rules), latency bound"}
    out["per_column_rules"] = per_col
    return out


def bench_backward(args, D: Dist):
    """Backward pass of the recurrent form (rank 0, CUDA events): Falcon-1, bf16 inputs, B1 H16 T1024
    d128, with an initial state, a cached key and an upstream gradient of the final state. Latency
    bound (one CTA walks each head's steps three times: checkpoints, recompute, reverse)."""
    import numpy as np
    import torch
    from delta_rule_linear_falcon_b200 import falcon as F
    from delta_rule_linear_falcon_b200 import inputs as I

    B, H, T, d = 1, 16, 1024, 128
    s = I.make_seq(1, B, H, T, d, d, seed=7, io_dtype="bf16", with_state=True, with_kprev=True)
    dev = torch.device("cuda", D.local)
    stream = torch.cuda.current_stream(dev)
    bf = lambda x: torch.from_numpy(x).to(torch.bfloat16).to(dev)
    f32 = lambda x: torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(dev)
    q, k, v, kp = bf(s.q), bf(s.k), bf(s.v), bf(s.k_prev)
    a, e, S0 = f32(s.alpha), f32(s.eta), f32(s.S0)
    dO = f32(I.normal(8, 8, B * H * T * d).reshape(B, H, T, d))
    dST = f32(I.normal(8, 9, B * H * d * d).reshape(B, H, d, d))
    args_ = F.make_args(q, k, v, a, e, rule=1, eps=s.eps, S0=S0, k_prev=kp)
    ws = torch.empty(F.falcon_bwd_workspace_size(args_), dtype=torch.uint8, device=dev)
    run = lambda: F.falcon_bwd_recurrent(q, k, v, a, e, dO, rule=1, eps=s.eps, S0=S0, k_prev=kp, dS_T=dST,
                                         workspace=ws, stream=stream)
    for _ in range(2):
        run()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(3):
        run()
    t1.record(stream)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / 3
    return {"workload": f"falcon1_bwd_recurrent_bf16_B{B}H{H}T{T}d{d}", "ms_per_call": round(ms, 3),
            "tokens_per_s": round(B * T / (ms * 1e-3), 1), "workspace_bytes": int(ws.numel()),
            "note": "latency bound: one CTA per 8 value rows of a head, forward to checkpoints, then "
                    "recompute and reverse per segment"}


def bench_more_chunk(args, D: Dist):
    """Secondary chunk workloads (rank 0, device-resident inputs, CUDA events): Falcon-3 and
    Falcon-3A (w = 4, B4 H16 T8192 d128), Falcon-1A on B1 H16 T32768 d128, and the benchmark
    workload with the same-step flag."""
    import torch
    from delta_rule_linear_falcon_b200 import falcon as F
    from delta_rule_linear_falcon_b200 import inputs as I

    dev = torch.device("cuda", D.local)
    stream = torch.cuda.current_stream(dev)
    hbm, tf, _ = peaks()
    out = {}

    def timed(s, rule, label):
        q, k, v = (torch.from_numpy(x).to(torch.bfloat16).to(dev) for x in (s.q, s.k, s.v))
        a, e = (torch.from_numpy(x).to(dev) for x in (s.alpha, s.eta))
        B, H, T, dk, dv = s.shape
        o = torch.empty_like(v)
        S = torch.empty((B, H, dv, dk), dtype=torch.float32, device=dev)
        kl = torch.empty((B, H, dk), dtype=torch.bfloat16, device=dev)
        need = F.falcon_workspace_size(F.make_args(q, k, v, a, e, rule=rule, eps=s.eps, window=s.window,
                                                   chunk=64, o=o, S_out=S, k_last=kl))
        ws = torch.empty(need, dtype=torch.uint8, device=dev) if need else None
        run = lambda: F.falcon_fwd_chunk(q, k, v, a, e, rule=rule, eps=s.eps, window=s.window, chunk=64,
                                         o=o, S_out=S, k_last=kl, workspace=ws, stream=stream)
        for _ in range(2):
            run()
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n = 5
        t0.record(stream)
        for _ in range(n):
            run()
        t1.record(stream)
        torch.cuda.synchronize()
        assert F.falcon_check_device_errors(stream) == F.FALCON_OK
        ms = t0.elapsed_time(t1) / n
        nbytes = chunk_algorithmic_bytes(B, H, T, dk, dv)
        flops = chunk_algorithmic_flops(B, H, T, dk, dv, window=s.window)
        gbs = nbytes / (ms * 1e-3) / 1e9
        # roofline time = max(bytes / HBM peak, recurrent-form FLOPs / bf16 peak)
        t_roof = max(nbytes / (hbm * 1e9), flops / (tf * 1e12))
        out[label] = {"workload": label, "ms_per_launch": round(ms, 4),
                      "tokens_per_s": round(B * T / (ms * 1e-3), 1), "gbs_algorithmic": round(gbs, 1),
                      "tflops_algorithmic": round(flops / (ms * 1e-3) / 1e12, 2),
                      "t_roofline_us": round(t_roof * 1e6, 2),
                      "roofline_bound": "hbm" if nbytes / (hbm * 1e9) >= flops / (tf * 1e12) else "tensor",
                      "roofline_frac": round(t_roof / (ms * 1e-3), 4), "launches": n,
                      # the sequence split of the inner-product rule: state pass, scan, chunk kernel;
                      # the two-pass path of the regression rules: solve pass, chain kernel
                      "kernels_per_call": (2 if rule & 1 else 3) if need else 1, "workspace_bytes": need}
        del q, k, v, a, e, o, S, kl, ws

    s3 = I.workload_chunk_f3()
    timed(s3, 3, "falcon3_w4_chunk_bf16_B4H16T8192d128")
    timed(s3, 4, "falcon3a_w4_chunk_bf16_B4H16T8192d128")
    del s3
    s2 = I.workload_chunk_f1a_long()
    timed(s2, 2, "falcon1a_chunk_bf16_B1H16T32768d128")
    del s2
    s1 = I.workload_chunk_f1(B=args.batch, T=args.seq_len)
    timed(s1, 1 | F.FALCON_SAME_STEP, f"falcon1_same_step_chunk_bf16_B{args.batch}H16T{args.seq_len}d128")
    return out


# ----------------------------------------------------------------------------- CPU oracle

_SAMPLE_CACHE = {}


def _oracle_sample_inputs(heads: int, T: int):
    from delta_rule_linear_falcon_b200 import inputs as I
    key = (heads, T)
    if key not in _SAMPLE_CACHE:
        _SAMPLE_CACHE[key] = I.make_seq(I.RULE_1, 1, heads, T, 128, 128, seed=1, io_dtype="bf16",
                                        normalise_qk=True, alpha_mu=4.0)
    return _SAMPLE_CACHE[key]


def cpu_oracle_sample(heads: int, T: int = 4096, threads=None):
    """Time the fp64 oracle (recurrent form, OpenMP over heads) on `heads` heads of the
    chunk workload (b = 0, h = 0..heads-1, all T tokens). Returns (tokens/s, seconds, cores)."""
    import oracle
    from delta_rule_linear_falcon_b200 import inputs as I
    s = _oracle_sample_inputs(heads, T)
    cores = threads or os.cpu_count() or 1
    t = time.perf_counter()
    oracle.recurrent(I.RULE_1, s.q, s.k, s.v, s.alpha, s.eta, s.eps, threads=cores)
    dt = time.perf_counter() - t
    # tokens of the workload are (b, t) positions carrying 16 heads each
    return heads * T / 16.0 / dt, dt, min(cores, heads)


def host_cpu():
    """(logical cores, CPU model name) of this host."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return os.cpu_count() or 1, model


def oracle_heads(cores: int) -> int:
    """Heads per oracle pass: at least one per core (OpenMP spreads heads over threads), a
    multiple of the core count, at most the 128 heads of the workload."""
    return max(1, min(128, cores * max(1, 16 // cores)))


def _oracle_rate(heads: int, threads: int, min_seconds: float):
    total_t, total_tok, passes, used = 0.0, 0.0, 0, 1
    while total_t < min_seconds:
        tps, dt, used = cpu_oracle_sample(heads, threads=threads)
        total_t += dt
        total_tok += tps * dt
        passes += 1
    return total_tok / total_t, total_t, passes, used


def cpu_baseline(min_seconds: float = 10.0):
    """The oracle as it stands on the host cores, on 1 core and on all cores: repeated passes
    over a subset of the 128 heads of the B8 H16 T4096 d128 workload (at least one head per
    thread) until at least `min_seconds` of work each."""
    nproc, model = host_cpu()
    heads = oracle_heads(nproc)
    v_all, t_all, p_all, used = _oracle_rate(heads, nproc, min_seconds)
    v_one, t_one, p_one, _ = _oracle_rate(1, 1, min_seconds / 2)
    return {"value": round(v_all, 1), "unit": "tokens/s", "cores": used, "kind": "oracle",
            "nproc": nproc, "cpu_model": model,
            "one_core": {"value": round(v_one, 1), "unit": "tokens/s", "cores": 1,
                         "sample": f"{p_one} passes x 1 head x 4096 tokens ({t_one:.1f} s)"},
            "all_cores": {"value": round(v_all, 1), "unit": "tokens/s", "cores": used,
                          "sample": f"{p_all} passes x {heads} heads x 4096 tokens ({t_all:.1f} s)"},
            "sample": f"{p_all} passes x {heads} of 128 heads x 4096 tokens of the B8 H16 T4096 d128 "
                      f"workload, fp64 recurrent oracle, OpenMP over heads on {used} threads "
                      f"({t_all:.1f} s); tokens are (b, t) positions of 16 heads each"}


# ----------------------------------------------------------------------------- main

def run_reference(args):
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    cores, model = host_cpu()
    heads = oracle_heads(cores)
    vals = []
    for _ in range(args.warmup):
        cpu_oracle_sample(heads, threads=cores)
    for _ in range(args.steps):
        tps, dt, used = cpu_oracle_sample(heads, threads=cores)
        vals.append((tps, dt, used))
    tps = statistics.median(v[0] for v in vals)
    ms = statistics.median(v[1] for v in vals) * 1e3
    used = vals[0][2]
    sample = (f"{heads} of 128 heads x 4096 tokens of the B8 H16 T4096 d128 workload per step, "
              f"fp64 recurrent oracle, OpenMP over heads on {used} of {cores} cores ({model})")
    line = {"impl": "reference", "metric": METRIC, "value": round(tps, 1), "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": base_config(args),
            "cpu_baseline": {"value": round(tps, 1), "unit": "tokens/s", "cores": used, "kind": "oracle",
                             "nproc": cores, "cpu_model": model, "sample": sample},
            "e2e": {"value": round(tps, 1), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def base_config(args):
    B, T = args.batch, getattr(args, "seq_len", 4096)
    nbytes = chunk_algorithmic_bytes(B, 16, T, 128, 128)
    return {"workload": f"falcon1_chunk_bf16_B{B}H16T{T}d128_chunk64", "rule": "falcon1",
            "B": B, "H": 16, "T": T, "dk": 128, "dv": 128, "chunk": 64,
            "global_batch": B * args.gpus, "seq_len": T,
            "parallelism": f"dp{args.gpus} (independent sequences per rank, no collective)",
            "l2": f"inputs larger than L2 ({nbytes / 1e6:.1f} MB per step vs 126 MB), no flush"}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["falcon", "reference"], default="falcon")
    ap.add_argument("--batch", type=int, default=8,
                    help="batch of the chunk workload (8 = the benchmark; smaller only for profiler captures)")
    ap.add_argument("--seq-len", type=int, default=4096,
                    help="tokens per sequence of the chunk workload (4096 = the benchmark; shorter "
                         "only for profiler captures: same kernel configuration, fewer blocks)")
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--decode-seqs", type=int, default=256,
                    help="sequences of the decode workload (256 = the benchmark)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)

    import torch
    from delta_rule_linear_falcon_b200 import falcon as F
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    F.lib()  # fails loudly if the library is missing
    D = Dist("nccl")
    torch.cuda.set_device(D.local)
    clk = ClockSampler(D.local)

    ch = bench_chunk(args, D, clk)
    dec = bench_decode(args, D, clk)
    rec = bench_recurrent(args, D) if D.rank == 0 else None
    more = bench_more_chunk(args, D) if D.rank == 0 else None
    bwd = bench_backward(args, D) if D.rank == 0 else None

    s = ch["s"]
    B, H, T, dk, dv = s.shape
    hbm, tf, src = peaks()
    tokens = B * T * D.world
    ms = ch["total_ms"] / args.steps
    value = weak_scaling_value(B * T, D.world, ms)
    nbytes = chunk_algorithmic_bytes(B, H, T, dk, dv)
    flops = chunk_algorithmic_flops(B, H, T, dk, dv)
    achieved = nbytes / (ch["kern_ms"] * 1e-3) / 1e9
    t_roof = max(nbytes / (hbm * 1e9), flops / (tf * 1e12))
    two_pass = ch["launches"] == 2
    traffic = recorded_traffic("chunk_two_pass" if two_pass else "chunk_ws_kernel", CHUNK_KERNEL_SOURCES)
    kname = "chunk_local_kernel + chunk_ws_kernel (one call)" if two_pass else "chunk_ws_kernel"
    dbytes = decode_algorithmic_bytes(dec["N"], dec["H"], dec["dk"], dec["dv"])
    dgbs = dbytes / (dec["ms"] * 1e-3) / 1e9

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": D.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": base_config(args),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                     "frac": round(achieved / hbm, 4), "traffic": traffic,
                     "peak_source": f"{src} (MEASURED_PEAKS.json hbm_gbs)" if src == "measured" else src,
                     "algorithmic_bytes_per_launch": nbytes, "kernel": kname,
                     "kernel_ms": round(ch["kern_ms"], 4), "launches_per_step": ch["launches"],
                     "workspace_bytes": ch["workspace_bytes"]},
        "roofline_flops_and_bytes": {"flops": flops, "bytes": nbytes, "t_roofline_us": round(t_roof * 1e6, 2),
                                "frac": round(t_roof / (ch["kern_ms"] * 1e-3), 4),
                                "tflops": round(flops / (ch["kern_ms"] * 1e-3) / 1e12, 2),
                                "definition": "max(FLOPs/bf16 peak, bytes/HBM peak) / kernel time, "
                                              "FLOPs = recurrent-form count 7 dk dv per token-head"},
        "e2e": {"value": round(tokens / (ch["e2e_ms"] * 1e-3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": ch["h2d"], "d2h_bytes_per_step": ch["d2h"],
                "ms_per_step": round(ch["e2e_ms"], 3)},
        "clocks": clk.summary(),
        "gpu_launches": args.steps * ch["launches"],
        "decode": {"workload": f"falcon1_decode_N{dec['N']}H{dec['H']}d{dec['dk']}", "value": round(dgbs, 1),
                   "unit": "GB/s", "ms_per_step": round(dec["ms"], 4), "steps": dec["steps"],
                   "gpu_launches": dec["steps"],
                   "roofline": {"bound": "hbm", "achieved": round(dgbs, 1), "peak": hbm, "unit": "GB/s",
                                "frac": round(dgbs / hbm, 4),
                                "traffic": recorded_traffic("decode_kernel", ["decode.cu", "common.cuh"]),
                                "algorithmic_bytes_per_launch": dbytes}},
    }
    if rec is not None:
        line["recurrent"] = rec
    if more is not None:
        line["more_chunk"] = more
    if bwd is not None:
        line["backward"] = bwd
    if D.rank == 0 and D.world == 1:
        line["cpu_baseline"] = cpu_baseline(min_seconds=10.0)
    if D.rank == 0:
        print(json.dumps(line), flush=True)
    D.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
