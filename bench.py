#!/usr/bin/env python
"""Benchmark of the KDA prefill hot path on B200 (one JSON line on rank 0).

A step is one pass of the whole hot path over one batch of synthetic input.  For the default
workload (one 131072-token sequence, 32 value heads, dk = dv = 128, bf16 q/k/v, fp32 gates and
state, cut into 16 segments of 8192) a step is the context-parallel prefill:
  1. kda_segment_summarize_and_scan with q: every segment in parallel builds its transition M_i,
     its contribution U_i and each token's two local readouts, then the exclusive affine scan
     gives incoming / outgoing / final states;
  2. kda_context_parallel_apply: every output row from its readouts and its segment's incoming
     state.
Other workloads (``--workload``), and the default one with ``--straight`` (the straight pass
over the whole sequence), time one kda_chunk_fwd call over the whole batch; their state pool
carries over from step to step (each step resumes from the previous final states,
as a split prefill would), so the timed work never includes a pool restore.

Besides the contract's keys the line carries ``roofline`` (the dominant launch's algorithmic
bytes over its device time, against the measured HBM bandwidth), ``step_roofline`` (the whole
step's algorithmic bytes and FLOPs: GB/s, TFLOP/s, and the fraction of the roofline taken as
the slower of bytes at HBM bandwidth and FLOPs at the dense bf16 peak) and ``breakdown_ms``.

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same workload (the
oracle is the only reference implementation there is).  Under torchrun every rank runs its
own replica of the workload (weak scaling, no data-path collective); timings are device
times, max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import kda_workloads as W  # noqa: E402

METRIC = "KDA prefill tokens/s (H=32,dk=dv=128,bf16) and % of roofline on 1 B200"
DECODE_METRIC = "KDA decode tokens/s (one token per sequence, dk=dv=128) and % of roofline on 1 B200"
DEFAULT_WORKLOAD = "long_T131072_H32_cp16"


# ------------------------------------------------------------------------------------------
# algorithmic traffic and work (per launch), see the design notes for the derivation
# ------------------------------------------------------------------------------------------

def io_bytes_per_token_head(qkv_bytes=2, out_bytes=2, dk=128, dv=128, group=1):
    # q and k are read once per key head; for Hv = Hk each value head reads its own q, k
    return (2 * dk * qkv_bytes) / group + dv * qkv_bytes + dk * 4 + 4 + dv * out_bytes


def chunk_fwd_bytes(w, num_seqs, dk=128, dv=128):
    th = w.total_tokens * w.num_v_heads
    group = w.num_v_heads // w.num_k_heads
    qkv = 2 if w.q.dtype == torch.bfloat16 else 4
    ob = 2 if w.output_dtype == torch.bfloat16 else 4
    return th * io_bytes_per_token_head(qkv, ob, dk, dv, group) + num_seqs * w.num_v_heads * 2 * dk * dv * 4


def decode_bytes(w):
    """One token per (sequence, head): the state block read and written once, plus the token's
    q, k, v, gate, beta and output."""
    group = w.num_v_heads // w.num_k_heads
    qkv = 2 if w.q.dtype == torch.bfloat16 else 4
    ob = 2 if w.output_dtype == torch.bfloat16 else 4
    th = w.batch * w.num_v_heads
    return th * (io_bytes_per_token_head(qkv, ob, w.dk, w.dv, group) + 2 * w.dk * w.dv * 4)


def segment_build_bytes(w, N, dk=128, dv=128):
    """The method's own bytes of the segment build plus the scan over N pieces: q, k, v, gate and
    beta in (the straight pass's reads), M and U out; the scan reads M and U and writes the
    incoming and outgoing states.  The per-token readouts the build also writes are this
    design's intermediate (the apply reads them back), not the method's, and are counted apart
    (``segment_build_intermediate_bytes``)."""
    th = w.total_tokens * w.num_v_heads
    group = w.num_v_heads // w.num_k_heads
    reads = th * ((2 * dk * 2) / group + dv * 2 + dk * 4 + 4)
    summaries = N * w.num_v_heads * (dk * dk + dk * dv) * 4
    scan = summaries + N * w.num_v_heads * dk * dv * 4 * 2
    return reads + summaries + scan


def segment_build_intermediate_bytes(w, dv=128):
    """The build's two bf16 readouts per token-head (written here, read back by the apply)."""
    return w.total_tokens * w.num_v_heads * 2 * dv * 2


def apply_bytes(w, N, dv=128):
    """Readouts and incoming states in, outputs out."""
    th = w.total_tokens * w.num_v_heads
    ob = 2 if w.output_dtype == torch.bfloat16 else 4
    return th * (2 * dv * 2 + dv * ob) + N * w.num_v_heads * dv * dv * 4


def step_roofline(w, ms_step, segments, pk, dk=128, dv=128, sm_mhz=None):
    """The whole step against the roofline as the slower of its algorithmic bytes at the HBM
    bandwidth and its algorithmic FLOPs at the dense bf16 tensor peak.  Bytes: the straight
    prefill's (q, k, v, gate, beta, outputs, the state read and written per chain), plus, for the
    context-parallel step, twice the segments' M, U and incoming tensors."""
    if segments:
        nbytes = chunk_fwd_bytes(w, 1, dk, dv) + 2 * segments * w.num_v_heads * 3 * dk * dv * 4
    else:
        nbytes = chunk_fwd_bytes(w, w.batch, dk, dv)
    flops = chunk_fwd_flops(w, dk=dk, dv=dv)
    t_hbm = nbytes / (pk["hbm_gbs"] * 1e9) * 1e3
    t_tensor = flops / (pk["bf16_tflops"] * 1e12) * 1e3
    res = {"bound": "hbm" if t_hbm >= t_tensor else "tensor", "algorithmic_bytes": nbytes,
           "algorithmic_flops": flops, "gbs": nbytes / (ms_step / 1e3) / 1e9,
           "tflops": flops / (ms_step / 1e3) / 1e12, "roofline_ms": max(t_hbm, t_tensor),
           "hbm_ms": t_hbm, "tensor_ms": t_tensor, "frac": max(t_hbm, t_tensor) / ms_step,
           "peak_source": pk["source"]}
    # beside it, not part of it: the special-function floor of the gates, three transcendental
    # operations per token, head and key channel (softplus's exp and log, the decay's exp) at 16
    # per clock per SM
    if sm_mhz and torch.cuda.is_available():
        sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
        sfu_ops = 3.0 * w.total_tokens * w.num_v_heads * dk
        res["sfu_ms"] = sfu_ops / (16.0 * sms * sm_mhz * 1e6) * 1e3
    return res


def chunk_fwd_flops(w, C=64, dk=128, dv=128):
    # 6 d^2 (W S, (Q o Gamma) S, K'^T Delta) + 5 C d (A, P, W, U, P Delta) + C^2/3 (inverse)
    th = w.total_tokens * w.num_v_heads
    return th * (2 * 3 * dk * dv + 2 * 2.5 * C * dk + C * C / 3)


# ------------------------------------------------------------------------------------------
# helpers
# ------------------------------------------------------------------------------------------

def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# the sources each recorded kernel is built from (its DRAM traffic holds while they are unchanged)
KERNEL_SOURCES = {
    "fused_chunk_kernel<build,readout> + affine_scan_kernel": [
        "kda_fused.cu", "kda_simt.cu", "kda_api.cu", "kda_sm100.cuh", "kda_common.cuh", "kda_internal.h"],
    "fused_chunk_kernel<prefill>": ["kda_fused.cu", "kda_api.cu", "kda_sm100.cuh", "kda_common.cuh",
                                    "kda_internal.h"],
    "decode_kernel": ["kda_decode.cu", "kda_api.cu", "kda_common.cuh", "kda_internal.h"],
}


def kernel_source_hash(kernel=None):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "kimi_delta_attention_23_b200", "csrc")
    names = KERNEL_SOURCES.get(kernel) or sorted(os.listdir(csrc))
    for name in sorted(names):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel):
    """DRAM bytes per launch from a committed ncu summary, only if the kernel is unchanged."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel)
    if not e or e.get("source_hash") != kernel_source_hash(kernel):
        return None
    return float(e["dram_bytes_per_launch"])


class ClockSampler:
    """SM clock and throttle reasons sampled during the timed region.

    Polls NVML from a background thread every few milliseconds (the timed region can be far
    shorter than nvidia-smi's sampling interval); falls back to nvidia-smi if NVML is absent."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, device_index=0, period_s=0.005):
        self.device_index, self.period = device_index, period_s
        self.samples, self.thread, self.stop_flag, self.nvml = [], None, False, None

    def _handle(self):
        import pynvml
        pynvml.nvmlInit()
        pr = torch.cuda.get_device_properties(self.device_index)
        bus = "%08X:%02X:%02X.0" % (int(pr.pci_domain_id), int(pr.pci_bus_id), int(pr.pci_device_id))
        try:
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.device_index)

    def _run(self):
        nv, hnd = self.nvml
        while not self.stop_flag:
            try:
                sm = nv.nvmlDeviceGetClockInfo(hnd, nv.NVML_CLOCK_SM)
                mx = nv.nvmlDeviceGetMaxClockInfo(hnd, nv.NVML_CLOCK_SM)
                get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    nv.nvmlDeviceGetCurrentClocksThrottleReasons
                rs = get_reasons(hnd)
                pw = nv.nvmlDeviceGetPowerUsage(hnd) / 1000.0
                self.samples.append((sm, mx, rs, pw))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        import threading
        try:
            self.nvml = self._handle()
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
            time.sleep(0.02)  # the first samples land before the timed work starts
        except Exception:
            self.nvml = None
        return self

    def __exit__(self, *exc):
        self.stop_flag = True
        if self.thread is not None:
            self.thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock samples (NVML unavailable)"]}
        sm = [s[0] for s in self.samples]
        reasons = sorted({n for s in self.samples for n, bit in self.REASONS.items() if s[2] & bit})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(s[1] for s in self.samples),
                "power_w_max": max(s[3] for s in self.samples), "samples": len(self.samples), "reasons": reasons,
                "source": "nvml"}


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def rank_seed(workload, rank):
    """Seed of a rank's own replica: rank 0 uses the workload's seed, others a distinct one."""
    return None if rank == 0 else 1000 * rank + W.WORKLOADS.index(workload)


def max_over_ranks(value, pg, device="cpu"):
    """The slowest rank's time (every rank takes part; the result is the same everywhere)."""
    if pg is None:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def whole_job_throughput(units_per_rank, world, ms_per_step):
    """Units all ranks processed per second, timed by the slowest rank (weak scaling)."""
    return units_per_rank * world / (ms_per_step / 1e3)


# ------------------------------------------------------------------------------------------
# CPU oracle timing (reference arm and cpu_baseline)
# ------------------------------------------------------------------------------------------

def oracle_time_sample(w, n_tokens):
    """Run the oracle over the first n_tokens of every (sequence, head) chain's token range."""
    import oracle
    cu = w.cu_seqlens.cpu().tolist()
    # take a prefix of the packed batch, cutting sequence boundaries where they fall
    n = min(n_tokens, w.total_tokens)
    cu_s = [c for c in cu if c < n] + [n]
    B = len(cu_s) - 1
    cpu = lambda t: t.detach().cpu()  # noqa: E731
    # only the slots the sampled sequences name (the oracle touches no other slot)
    idx = cpu(w.state_indices)[:B].long()
    pool = cpu(w.state_pool)[idx]
    t0 = time.perf_counter()
    oracle.kda_forward(cpu(w.q)[:n], cpu(w.k)[:n], cpu(w.v)[:n], cpu(w.raw_gate)[:n], cpu(w.beta_logits)[:n],
                       cpu(w.a_log), cpu(w.dt_bias), torch.tensor(cu_s, dtype=torch.int32),
                       pool, torch.arange(B, dtype=torch.int32), gate_mode=w.gate_mode, beta_mode=w.beta_mode,
                       state_layout=w.state_layout, gate_lower_bound=w.gate_lower_bound)
    return time.perf_counter() - t0, n


def calibrate_oracle(w, target_s):
    n = 256
    while True:
        dt, n_done = oracle_time_sample(w, n)
        if dt >= target_s / 4 or n_done >= w.total_tokens:
            scale = target_s / max(dt, 1e-6)
            return max(1, min(w.total_tokens, int(n_done * scale)))
        n *= 4


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    w = W.make(args.workload, device="cpu")
    n = calibrate_oracle(w, target_s=args.ref_step_seconds)
    for _ in range(args.warmup):
        oracle_time_sample(w, n)
    times = [oracle_time_sample(w, n)[0] for _ in range(args.steps)]
    total = sum(times)
    value = n * args.steps / total
    line = {"impl": "reference", "metric": DECODE_METRIC if w.notes.get("decode") else METRIC, "value": value,
            "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": args.workload, "tokens_per_step": n,
                                            "num_v_heads": w.num_v_heads, "dk": w.dk, "dv": w.dv},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": f"first {n} tokens of the workload, all {w.num_v_heads} heads, per step"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------------------
# GPU arm
# ------------------------------------------------------------------------------------------

class Step:
    """One pass of the hot path on device-resident inputs; records per-call CUDA events."""

    def __init__(self, w, stream, public=False, straight=False):
        import kimi_delta_attention_23_b200 as kda
        self.kda, self.w, self.stream, self.public = kda, w, stream, public
        dev = w.q.device
        # straight: a segmented workload run as one kda_chunk_fwd call over the whole sequence
        self.cp = w.seg_offsets is not None and not straight
        self.decode = bool(w.notes.get("decode"))
        T, Hv, dv, dk = w.total_tokens, w.num_v_heads, w.dv, w.dk
        self.out = torch.empty((T, Hv, dv), dtype=w.output_dtype, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        if self.cp:
            N = w.seg_offsets.numel() - 1
            st = (dk, dv) if w.state_layout == "K_FIRST" else (dv, dk)
            self.N = N
            # single-sequence workload whose state sits in pool slot 0 (a view: it follows the pool)
            self.init = w.state_pool[0]
            self.M = torch.empty((N, Hv, dk, dk), device=dev)
            self.U = torch.empty((N, Hv, *st), device=dev)
            self.inc = torch.empty((N, Hv, *st), device=dev)
            self.outg = torch.empty((N, Hv, *st), device=dev)
            self.fin = torch.empty((Hv, *st), device=dev)
            # the library builds every segment as `pieces` chunk-aligned pieces (more chains than
            # SMs' worth of segments); the step below makes the same calls as the prefill entry
            self.pieces = kda.kda_context_parallel_pieces(T, N, Hv)
            P = N * self.pieces
            self.P = P
            if public:
                self.ws = torch.empty(max(kda.kda_context_parallel_workspace_preferred(T, N, Hv, dv), 1),
                                      dtype=torch.uint8, device=dev)
            else:
                # head-major readouts, as the prefill entry keeps them in its workspace
                self.rm = torch.empty((Hv, T, dv), dtype=torch.bfloat16, device=dev)
                self.ru = torch.empty((Hv, T, dv), dtype=torch.bfloat16, device=dev)
                if self.pieces > 1:
                    self.poffs = torch.empty(P + 1, dtype=torch.int32, device=dev)
                    self.pM = torch.empty((P, Hv, dk, dk), device=dev)
                    self.pU = torch.empty((P, Hv, *st), device=dev)
                    self.pIn = torch.empty((P + 1, Hv, *st), device=dev)  # slot p + 1: outgoing of piece p
        self.pool = None if self.cp else w.state_pool.clone()
        if self.decode:
            self.ws = torch.empty(0, dtype=torch.uint8, device=dev)
        elif not self.cp:
            # the prefill's optional workspace: with it, a batch of few or uneven sequences may
            # take the split route (decided on the device by the library's planner)
            Hk = w.k.shape[1]
            need = kda.kda_workspace_size(T, w.batch, Hk, Hv, dk, dv) if w.q.dtype == torch.bfloat16 else 0
            self.ws = torch.empty(need, dtype=torch.uint8, device=dev)
        self.events = []

    def kw(self):
        w = self.w
        return dict(gate_mode=w.gate_mode, beta_mode=w.beta_mode, state_layout=w.state_layout,
                    gate_lower_bound=w.gate_lower_bound, device_status=self.status, stream=self.stream)

    def launches(self):
        if self.decode:
            return 1
        if not self.cp:
            # split route: planner, plain kernel (gated), build, pool scan, apply; else one kernel
            return 5 if self.ws.numel() > 0 else 1
        # (piece boundaries,) segment build with readouts, scan, (composition,) apply
        return 5 if self.pieces > 1 else 3

    def __call__(self, record=False):
        w, kda = self.w, self.kda
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)] if record else None
        if ev:
            ev[0].record(self.stream)
        if self.cp and self.public:
            kda.kda_context_parallel_prefill(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias,
                                             w.seg_offsets, self.init, self.out, final_state=self.fin, M=self.M,
                                             U=self.U, incoming=self.inc, outgoing=self.outg, workspace=self.ws,
                                             **self.kw())
            for e in (ev or [])[1:]:
                e.record(self.stream)
        elif self.cp and self.pieces > 1:
            kda.kda_context_parallel_piece_offsets(w.seg_offsets, self.pieces, out=self.poffs, stream=self.stream)
            kda.kda_segment_summarize_and_scan(w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias,
                                               self.poffs, self.init, M=self.pM, U=self.pU, incoming=self.pIn[:-1],
                                               outgoing=self.pIn[1:], final_state=self.fin, q=w.q,
                                               readout_m=self.rm, readout_u=self.ru, readout_layout="head_major",
                                               **self.kw())
            if ev:
                ev[1].record(self.stream)
            kda.kda_segment_compose(self.pM, self.pU, self.pIn, self.fin, self.pieces, M=self.M, U=self.U,
                                    incoming=self.inc, outgoing=self.outg, state_layout=w.state_layout,
                                    stream=self.stream)
            if ev:
                ev[2].record(self.stream)
            kda.kda_context_parallel_apply(self.rm, self.ru, self.pIn[:-1], self.poffs, self.out,
                                           readout_layout="head_major", state_layout=w.state_layout,
                                           device_status=self.status, stream=self.stream)
        elif self.cp:
            kda.kda_segment_summarize_and_scan(w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias,
                                               w.seg_offsets, self.init, M=self.M, U=self.U, incoming=self.inc,
                                               outgoing=self.outg, final_state=self.fin, q=w.q, readout_m=self.rm,
                                               readout_u=self.ru, readout_layout="head_major", **self.kw())
            if ev:
                ev[1].record(self.stream)
                ev[2].record(self.stream)
            kda.kda_context_parallel_apply(self.rm, self.ru, self.inc, w.seg_offsets, self.out,
                                           readout_layout="head_major", state_layout=w.state_layout,
                                           device_status=self.status, stream=self.stream)
        elif self.decode:
            if ev:
                ev[1].record(self.stream)
                ev[2].record(self.stream)
            kda.kda_decode(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias, self.pool,
                           w.state_indices, self.out, **self.kw())
        else:
            if ev:
                ev[1].record(self.stream)
                ev[2].record(self.stream)
            kda.kda_chunk_fwd(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias, w.cu_seqlens,
                              self.pool, w.state_indices, self.out, workspace=self.ws, **self.kw())
        if ev:
            ev[3].record(self.stream)
            self.events.append(ev)


def run_ours(args):
    rank, world, local_rank = dist_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
        pg = dist
    from kimi_delta_attention_23_b200 import build as kbuild
    kbuild.build()
    w = W.make(args.workload, device=dev, seed=rank_seed(args.workload, rank))
    stream = torch.cuda.current_stream(dev)
    step = Step(w, stream, straight=args.straight)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if int(step.status.item()) != 0:
        raise RuntimeError(f"device status {int(step.status.item())} during warm-up")

    def barrier():
        if pg is not None:
            pg.barrier()

    # timed region: K steps, events per API call plus the bracketing pair
    step.events.clear()
    barrier()
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clocks:
        start.record(stream)
        for _ in range(args.steps):
            step(record=True)
        stop.record(stream)
        torch.cuda.synchronize()
    barrier()
    ms_total = start.elapsed_time(stop)
    seg_ms = [e[0].elapsed_time(e[1]) for e in step.events]
    comp_ms = [e[1].elapsed_time(e[2]) for e in step.events]
    pass_ms = [e[2].elapsed_time(e[3]) for e in step.events]
    ms_total = max_over_ranks(ms_total, pg, dev)
    ms_step = ms_total / args.steps
    tokens = w.total_tokens
    value = whole_job_throughput(tokens, world, ms_step)

    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(w, args, stream, pg)

    if rank != 0:
        if pg is not None:
            pg.destroy_process_group()
        return 0
    pk = peaks()
    ms_pass = statistics.mean(pass_ms)
    ms_seg = statistics.mean(seg_ms) if step.cp else 0.0
    if step.cp:
        # dominant launch: the segment build with readouts over the pieces (its call also runs the
        # short scan; the piece boundaries are computed first, in a negligible launch)
        dom, bytes_dom, ms_dom = "fused_chunk_kernel<build,readout> + affine_scan_kernel", \
            segment_build_bytes(w, step.P), ms_seg
        breakdown = {"segment_build_and_scan": ms_seg, "compose_pieces": statistics.mean(comp_ms),
                     "context_parallel_apply": ms_pass}
    elif step.decode:
        dom, bytes_dom, ms_dom = "decode_kernel", decode_bytes(w), ms_pass
        breakdown = {"decode": ms_pass}
    else:
        dom = "fused_chunk_kernel<prefill>" if step.ws.numel() == 0 else \
            "kda_chunk_fwd (planner; pieces: build with readouts, pool scan, apply; or the prefill kernel)"
        bytes_dom, ms_dom = chunk_fwd_bytes(w, w.batch), ms_pass
        breakdown = {"chunk_fwd": ms_pass}
    achieved = bytes_dom / (ms_dom / 1e3) / 1e9
    roof = {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / pk["hbm_gbs"], "traffic": recorded_traffic(dom),
            "algorithmic_bytes_per_launch": bytes_dom, "ms_per_launch": ms_dom,
            "peak_source": pk["source"]}
    if step.cp:
        # the readouts: written by this launch and read back by the apply; not the method's bytes
        roof["intermediate_bytes_per_launch"] = segment_build_intermediate_bytes(w)
    line = {"metric": DECODE_METRIC if step.decode else METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if w.q.dtype == torch.bfloat16 else "f32", "data": "synthetic",
            "config": {"workload": args.workload, "tokens": tokens, "num_v_heads": w.num_v_heads,
                       "num_k_heads": w.num_k_heads, "dk": w.dk, "dv": w.dv, "batch": w.batch,
                       "segments": step.N if step.cp else None,
                       "pass": "context_parallel" if step.cp else ("decode" if step.decode else "straight"),
                       "pieces_per_segment": step.pieces if step.cp else None, "gate_mode": w.gate_mode,
                       "state_layout": w.state_layout, "parallelism": f"dp{world}" if world > 1 else "single",
                       "l2": "inputs larger than L2 (%.2f GB read per step), no flush" % (
                           (segment_build_bytes(w, step.P) if step.cp else
                            decode_bytes(w) if step.decode else chunk_fwd_bytes(w, w.batch)) / 1e9)},
            "breakdown_ms": breakdown,
            "roofline": roof, "gpu_launches": step.launches() * args.steps, "clocks": clocks.summary()}
    if not step.decode:
        line["step_roofline"] = step_roofline(w, ms_step, step.N if step.cp else 0, pk,
                                              sm_mhz=line["clocks"].get("sm_mhz") or line["clocks"].get("sm_max_mhz"))
    if e2e is not None:
        line["e2e"] = e2e
    if world == 1 and not args.no_workloads and args.workload == DEFAULT_WORKLOAD and not args.straight:
        # the other headline and reported workloads, timed in the same run (the same protocol:
        # W untimed steps, K timed ones bracketed by CUDA events on the launching stream, clocks
        # sampled during them); the straight pass reuses this workload's inputs
        del step
        line["workloads"] = extra_workloads(w, args, stream, pk, dev)
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args)
    print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()
    return 0


EXTRA_WORKLOADS = (("long_T131072_H32_cp16 --straight", None), ("varlen8_H32_vfirst", "varlen8_H32_vfirst"),
                   ("batch64_T2048_H16_safe", "batch64_T2048_H16_safe"), ("single_T4096_H16", "single_T4096_H16"))


def time_workload(w, args, stream, pk, straight=False):
    """One workload's step timed like the main one: its ms per step, tokens/s and the fraction of
    its roofline (algorithmic bytes at the measured HBM bandwidth vs FLOPs at the bf16 peak)."""
    step = Step(w, stream, straight=straight)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if int(step.status.item()) != 0:
        raise RuntimeError(f"device status {int(step.status.item())} during warm-up")
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(stream.device.index or 0) as clocks:
        start.record(stream)
        for _ in range(args.steps):
            step()
        stop.record(stream)
        torch.cuda.synchronize()
    ms = start.elapsed_time(stop) / args.steps
    roof = step_roofline(w, ms, step.N if step.cp else 0, pk)
    return {"ms_per_step": ms, "tokens_per_s": w.total_tokens / (ms / 1e3), "tokens": w.total_tokens,
            "num_v_heads": w.num_v_heads, "batch": w.batch, "gate_mode": w.gate_mode,
            "state_layout": w.state_layout, "pass": "context_parallel" if step.cp else "straight",
            "algorithmic_bytes": roof["algorithmic_bytes"], "gbs": roof["gbs"], "frac": roof["frac"],
            "gpu_launches": step.launches() * args.steps, "steps": args.steps, "warmup": args.warmup,
            "clocks": clocks.summary()}


def extra_workloads(w_main, args, stream, pk, dev):
    res = {}
    for label, name in EXTRA_WORKLOADS:
        w = w_main if name is None else W.make(name, device=dev)
        res[label] = time_workload(w, args, stream, pk, straight=name is None)
        del w
        torch.cuda.empty_cache()
    return res


def measure_e2e(w, args, stream, pg):
    """The step end to end through the public API from pinned host buffers: every input copied in,
    the step, the output rows and the final state copied out, all inside the timed region.  A
    single long bf16 sequence goes through kda_prefill_host_pipelined (the call for a sequence held
    in host memory: copies in and out pipelined with the kernels in 2048-token segments); other
    workloads copy in, call kda_chunk_fwd, and copy out."""
    dev = w.q.device
    if w.seg_offsets is not None and w.q.dtype == torch.bfloat16:
        return measure_e2e_host_pipelined(w, args, stream, pg)
    names = ["q", "k", "v", "raw_gate", "beta_logits", "a_log", "dt_bias", "cu_seqlens", "state_pool",
             "state_indices"] + (["seg_offsets"] if w.seg_offsets is not None else [])
    host = {n: getattr(w, n).cpu().pin_memory() for n in names}
    wd = W.Workload(**{k: getattr(w, k) for k in w.__dataclass_fields__})
    for n in names:
        setattr(wd, n, torch.empty_like(getattr(w, n)))
    step = Step(wd, stream, public=True)
    out_host = torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory()
    fin_src = step.fin if step.cp else step.pool
    fin_host = torch.empty(fin_src.shape, dtype=fin_src.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_host.numel() * out_host.element_size() + fin_host.numel() * fin_host.element_size()

    def one():
        for n in names:
            getattr(wd, n).copy_(host[n], non_blocking=True)
        if not step.cp:
            step.pool.copy_(wd.state_pool)
        step()
        out_host.copy_(step.out, non_blocking=True)
        fin_host.copy_(fin_src, non_blocking=True)

    for _ in range(max(1, min(args.warmup, 2))):
        one()
    torch.cuda.synchronize()
    if pg is not None:
        pg.barrier()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = max(1, min(args.steps, 5))
    start.record(stream)
    for _ in range(n):
        one()
    stop.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(start.elapsed_time(stop), pg, dev)
    world = pg.get_world_size() if pg is not None else 1
    return {"value": whole_job_throughput(w.total_tokens, world, ms / n), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": n}


def measure_e2e_host_pipelined(w, args, stream, pg):
    import kimi_delta_attention_23_b200 as kda
    dev = w.q.device
    T, Hk, Hv = w.total_tokens, w.k.shape[1], w.num_v_heads
    # pipeline granularity: 2048-token segments (8192: 104.1 ms, 4096: 102.8, 2048: 101.8, 1024:
    # 103.3 on the 131072-token, 32-head sequence; the copies in bound it near 100 ms)
    seg = min(2048, max(64, -(-T // 64) * 64))
    host = {n: getattr(w, n).cpu().contiguous().pin_memory()
            for n in ("q", "k", "v", "raw_gate", "beta_logits", "a_log", "dt_bias")}
    host["initial_state"] = w.state_pool[0].cpu().contiguous().pin_memory()
    out_host = torch.empty((T, Hv, w.dv), dtype=w.output_dtype, pin_memory=True)
    fin_host = torch.empty(host["initial_state"].shape, dtype=torch.float32, pin_memory=True)
    with torch.cuda.device(dev):
        ws = torch.empty(kda.kda_prefill_host_workspace_size(T, Hk, Hv, w.output_dtype, seg), dtype=torch.uint8,
                         device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_host.numel() * out_host.element_size() + fin_host.numel() * fin_host.element_size()

    def one():
        kda.kda_prefill_host_pipelined(host["q"], host["k"], host["v"], host["raw_gate"], host["beta_logits"],
                                       host["a_log"], host["dt_bias"], host["initial_state"], out_host,
                                       final_state=fin_host, segment_tokens=seg, workspace=ws,
                                       gate_mode=w.gate_mode, beta_mode=w.beta_mode, state_layout=w.state_layout,
                                       gate_lower_bound=w.gate_lower_bound, device_status=status, stream=stream,
                                       device=dev)

    for _ in range(max(1, min(args.warmup, 2))):
        one()
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} in the end-to-end call")
    if pg is not None:
        pg.barrier()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = max(1, min(args.steps, 5))
    start.record(stream)
    for _ in range(n):
        one()
    stop.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(start.elapsed_time(stop), pg, dev)
    world = pg.get_world_size() if pg is not None else 1
    return {"value": whole_job_throughput(T, world, ms / n), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": n, "api": "kda_prefill_host_pipelined",
            "path": "the plain chunk kernel over consecutive segments of the sequence, copies in and out "
                    "overlapped with it (not the context-parallel step timed on the device)",
            "segment_tokens": seg}


def cpu_baseline(w, args):
    import oracle
    wc = w.to("cpu")
    n = calibrate_oracle(wc, target_s=args.cpu_seconds)
    dt, n = oracle_time_sample(wc, n)
    return {"value": n / dt, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"first {n} tokens of the workload, all {w.num_v_heads} heads (fp64 token-by-token)",
            "seconds": dt}


def profile_launches(args):
    """Plain launches of one workload's step, nothing else (a target for ncu): the prefill kernel,
    or for a context-parallel workload the step's calls (build over the pieces, scan, composition,
    apply)."""
    import kimi_delta_attention_23_b200 as kda
    from kimi_delta_attention_23_b200 import build as kbuild
    kbuild.build()
    w = W.make(args.workload, device="cuda")
    if w.seg_offsets is not None and not args.straight:
        step = Step(w, torch.cuda.current_stream())
        for _ in range(args.profile_launches):
            step()
        torch.cuda.synchronize()
        print("launched", args.profile_launches, "context-parallel steps; pieces per segment", step.pieces)
        return 0
    if w.notes.get("decode"):
        pool = w.state_pool.clone()
        for _ in range(args.profile_launches):
            kda.kda_decode(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias, pool, w.state_indices,
                           output_dtype=w.output_dtype, gate_mode=w.gate_mode, beta_mode=w.beta_mode,
                           state_layout=w.state_layout, gate_lower_bound=w.gate_lower_bound)
        torch.cuda.synchronize()
        print("launched", args.profile_launches, "decode steps")
        return 0
    for _ in range(args.profile_launches):
        pool = w.state_pool.clone()
        kda.kda_chunk_fwd(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias, w.cu_seqlens, pool,
                          w.state_indices, output_dtype=w.output_dtype, gate_mode=w.gate_mode, beta_mode=w.beta_mode,
                          state_layout=w.state_layout, gate_lower_bound=w.gate_lower_bound)
    torch.cuda.synchronize()
    print("launched", args.profile_launches)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=W.WORKLOADS, default=DEFAULT_WORKLOAD)
    ap.add_argument("--straight", action="store_true",
                    help="segmented workloads: time one kda_chunk_fwd call over the whole sequence instead of "
                         "the context-parallel step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the other workloads timed after the default one (the 'workloads' key)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-step-seconds", type=float, default=4.0)
    ap.add_argument("--profile-launches", type=int, default=0,
                    help="only run this many kda_chunk_fwd launches on the workload (for ncu), no timing")
    args = ap.parse_args()
    if args.profile_launches:
        return profile_launches(args)
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
