"""Benchmark of the forward Differential Attention V2 hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

One step is one pass of the whole hot path over one batch of synthetic input, on the
largest single-GPU configurations:
  * prefill: causal bf16 DiffAttn V2 over B=1 x S=32768, Hq=64 (32 pairs), Hkv=8, D=128
    (one tcgen05 kernel launch), then
  * needle decode: one bf16 decode step for 8 sequences of 131072 cached tokens each
    ([8, 131072, 8, 128] KV cache with one planted needle key per sequence); the V1 lambda
    is computed on the device from its four re-parameterisation vectors (one small kernel),
    then one split-KV kernel whose last split per (b, KV head) merges the partials (a memset
    of its split counters precedes it).
`value` is the prefill throughput in TFLOP/s (algorithmic FLOPs = 4*D*Hq*B*S(S+1)/2 over
the prefill kernel's CUDA-event time inside the timed steps); the decode throughput in
GB/s (every visible K/V row once, plus q, lambda and out) is reported beside it. The same
run then times the second pair of workloads (B=4 x 4096 prefill; B=64 decode with lengths
uniform in [1024, 8192]) the same way, under `second_workload`.
Inputs are resident in HBM before the timed region and are larger than L2 (the prefill's
q alone is 537 MB and the decode streams 4.3 GB per step), so no extra L2 flush is done.
`e2e` repeats the step through host buffers: pinned uploads of every input and downloads
of both outputs, on their own streams, overlapped with the kernels across steps.

--impl reference times the float64 CPU oracle (the test oracle, as it stands) on a bounded
sample of the same workload on the host cores; with N > 1 only rank 0 runs it.

Multi-GPU (torchrun, one rank per GPU): every rank runs the same per-GPU workload on its
own seeded inputs (weak scaling: (b, KV-head) units are independent, so there is no
data-path collective); the timed region is bracketed by a barrier and a synchronize and
the time is the maximum over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "DiffAttnV2 fwd: prefill TFLOP/s (% bf16 peak); decode GB/s (% HBM)"
# The step the headline line times: the largest single-GPU configurations (32k-token causal
# prefill; needle decode over 8 x 131072 cached tokens with the V1 lambda).
PREFILL_CFG = "prefill_b1_s32768"
DECODE_CFG = "needle_decode_b8_s131072"
# The second prefill and decode workloads, timed the same way in the same run.
PREFILL_CFG_2 = "prefill_b4_s4096"
DECODE_CFG_2 = "decode_b64_s8192"

# Measured roofline denominators of this machine's B200s (measured copy bandwidth and
# cuBLAS bf16 GEMM); used when the peaks file is absent.
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic per launch from an ncu capture, keyed by the kernel source it was taken on;
# reported as null once the source differs from the one captured.
# B200 data-sheet figures (dense bf16 tensor throughput, HBM3e bandwidth), reported beside
# the measured peaks
SPEC_BF16_TFLOPS = 2250.0
SPEC_HBM_GBS = 8000.0

# DRAM traffic per launch from an ncu capture (dram__bytes_read.sum + dram__bytes_write.sum of
# one launch), keyed by workload and by the kernel source it was taken on; reported as null
# once the source differs from the one captured.
NCU_TRAFFIC = {
    # B=1 x 32768 causal prefill: 3469007104 read + 247027712 written
    ("prefill", "prefill_b1_s32768"): {"bytes": 3716034816, "source_sha": "9162a0e0f5575922"},
    # B=8 x 131072 needle decode (split kernel with the fused merge): 4304199936 + 12690688
    ("decode", "needle_decode_b8_s131072"): {"bytes": 4316890624, "source_sha": "ff96f9e2aabe4153"},
}


def _src_sha(name):
    """Hash of a kernel's source file together with the shared PTX wrappers it includes."""
    h = hashlib.sha256()
    for part in (name, "ptx.cuh"):
        with open(os.path.join(ROOT, "differential_attention_v2_b200", "csrc", part), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(",") for r in out.strip().splitlines() if r.strip()]
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for n, val in zip(names, r[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        loaded = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------- distributed
def _dist_init(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        return rank, world, local, dist
    if n_gpus != 1:
        print(f"warning: --gpus {n_gpus} without torchrun; running one process", file=sys.stderr)
    return 0, 1, 0, None


def head_shard(Hq, Hkv, world, rank):
    """KV heads and query heads of `rank` when the heads are split over `world` GPUs.

    Returns (kv0, kv1, q0, q1): KV heads [kv0, kv1) and their query heads [q0, q1). Whole
    GQA groups move together, so every pair of adjacent query heads keeps its K/V head and
    the ranks never exchange data: each computes out[..., q0/2:q1/2, :] on its own.
    """
    if Hkv % world:
        raise ValueError(f"Hkv={Hkv} KV heads do not split evenly over {world} ranks")
    group = Hq // Hkv
    per = Hkv // world
    kv0, kv1 = rank * per, (rank + 1) * per
    return kv0, kv1, kv0 * group, kv1 * group


def shard_prefill_inputs(inp, Hq, Hkv, world, rank):
    """Contiguous per-rank slices (q, k, v, lambda) of a head-sharded prefill."""
    kv0, kv1, q0, q1 = head_shard(Hq, Hkv, world, rank)
    return {"q": inp["q"][:, :, q0:q1].contiguous(), "k": inp["k"][:, :, kv0:kv1].contiguous(),
            "v": inp["v"][:, :, kv0:kv1].contiguous(), "lam": inp["lam"][:, :, q0 // 2:q1 // 2].contiguous()}


def _barrier(dist):
    if dist is not None:
        dist.barrier()


def _max_over_ranks(x, dist):
    if dist is None:
        return x
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# -------------------------------------------------------------------------- our arm
def _inputs(pc_name, dc_name, rank, do_pre=True, do_dec=True, world=1, strong=False):
    """Per-rank inputs. Weak scaling: every rank its own seeded batch of the full size.
    Strong scaling: one seeded problem, each rank its head shard (a whole number of GQA
    groups), so the ranks together compute exactly the single-GPU workload."""
    pc = workloads.CONFIGS[pc_name]
    dc = workloads.CONFIGS[dc_name]
    if not strong:
        pc = workloads.PrefillCase(**{**pc.__dict__, "seed": pc.seed + 100 * rank})
        dc = workloads.DecodeCase(**{**dc.__dict__, "seed": dc.seed + 100 * rank})
    pin = workloads.make_prefill(pc) if do_pre else None
    din = workloads.make_decode(dc) if do_dec else None
    if strong and world > 1:
        kv0, kv1, q0, q1 = head_shard(pc.Hq, pc.Hkv, world, rank)
        if pin is not None:
            pin = shard_prefill_inputs(pin, pc.Hq, pc.Hkv, world, rank)
        if din is not None:
            din = {**din, "q": din["q"][:, q0:q1].contiguous(), "kcache": din["kcache"][:, :, kv0:kv1].contiguous(),
                   "vcache": din["vcache"][:, :, kv0:kv1].contiguous()}
            for x in ("lam", "lq1", "lk1", "lq2", "lk2"):
                if din.get(x) is not None:
                    t = din[x]
                    din[x] = (t[:, q0 // 2:q1 // 2] if x == "lam" else t[q0 // 2:q1 // 2]).contiguous()
        pc = workloads.PrefillCase(**{**pc.__dict__, "Hq": q1 - q0, "Hkv": kv1 - kv0})
        dc = workloads.DecodeCase(**{**dc.__dict__, "Hq": q1 - q0, "Hkv": kv1 - kv0})
    return pc, pin, dc, din


class Step:
    """Device-resident inputs and outputs of one step (prefill + decode) and its launches.

    The decode of a V1-lambda workload computes lambda on the device first (one small
    kernel) from the four re-parameterisation vectors, as a caller of the operator would."""

    def __init__(self, da, pc, pin, dc, din, dev, stream, n_buffers=1):
        self.da, self.pc, self.dc, self.dev, self.stream = da, pc, dc, dev, stream
        self.pin, self.din = pin, din
        self.do_pre, self.do_dec = pin is not None, din is not None
        self.v1 = self.do_dec and din["lam"] is None
        self.bufs = []
        for _ in range(n_buffers):
            b = {}
            if self.do_pre:
                for x in ("q", "k", "v", "lam"):
                    b[x] = pin[x].to(dev)
                b["out"] = torch.empty(pc.B, pc.S, pc.Hq // 2, pc.D, dtype=torch.bfloat16, device=dev)
            if self.do_dec:
                for x in ("q", "seqlens") + (("lq1", "lk1", "lq2", "lk2") if self.v1 else ("lam",)):
                    b["d" + x] = din[x].to(dev)
                if self.v1:
                    b["dlam"] = torch.empty(dc.B, dc.Hq // 2, dtype=torch.float32, device=dev)
                b["dout"] = torch.empty(dc.B, dc.Hq // 2, dc.D, dtype=torch.bfloat16, device=dev)
            self.bufs.append(b)
        if self.do_dec:
            # the cache is state that lives on the device; one copy serves every buffer set
            self.kc = din["kcache"].to(dev)
            self.vc = din["vcache"].to(dev)
            self.ws = torch.empty(da.decode_workspace_size(dc.B, dc.Smax, dc.Hq, dc.Hkv, dc.D), dtype=torch.uint8,
                                  device=dev)
        self.flops = workloads.prefill_flops(pc.B, pc.S, pc.Hq, pc.D, causal=True) if self.do_pre else 0
        self.dbytes = workloads.decode_bytes(din["seqlens"].tolist(), dc.Hkv, dc.D, dc.Hq) if self.do_dec else 0
        # kernels of this library per step: prefill; V1 lambda; decode (the split counters'
        # memset is a runtime call, not a kernel of this library)
        self.launches = int(self.do_pre) + (int(self.v1) + 1 if self.do_dec else 0)

    def prefill(self, i=0, stream=None):
        b = self.bufs[i]
        self.da.prefill(b["q"], b["k"], b["v"], b["lam"], out=b["out"], stream=stream or self.stream)

    def decode(self, i=0, stream=None):
        b = self.bufs[i]
        st = stream or self.stream
        if self.v1:
            self.da.lambda_v1(b["dlq1"], b["dlk1"], b["dlq2"], b["dlk2"], self.din["lambda_init"], rows=self.dc.B,
                              out=b["dlam"], stream=st)
        self.da.decode(b["dq"], self.kc, self.vc, b["dseqlens"], b["dlam"], out=b["dout"], workspace=self.ws,
                       stream=st)

    def h2d_names(self):
        pre = ("q", "k", "v", "lam") if self.do_pre else ()
        dec = (("q", "seqlens") + (("lq1", "lk1", "lq2", "lk2") if self.v1 else ("lam",))) if self.do_dec else ()
        return pre, dec


def _time_steps(st, steps, dist):
    """Time `steps` steps on the step's stream: CUDA events around each step's prefill and
    decode; the whole region bracketed by a barrier and a synchronize on both sides."""
    stream, dev = st.stream, st.dev
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier(dist)
    torch.cuda.synchronize(dev)
    t0.record(stream)
    for i in range(steps):
        evs[i][0].record(stream)
        if st.do_pre:
            st.prefill()
        evs[i][1].record(stream)
        if st.do_dec:
            st.decode()
        evs[i][2].record(stream)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    _barrier(dist)
    total = _max_over_ranks(t0.elapsed_time(t1), dist)
    pre = _max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in evs), dist)
    dec = _max_over_ranks(sum(e[1].elapsed_time(e[2]) for e in evs), dist)
    return total, pre, dec


def _e2e(st, steps, dist):
    """The step end to end through the public API: every step copies its inputs from
    pinned host memory and its outputs back. Copies run on their own streams, ordered by
    events against the compute stream, so step i+1's uploads and step i's downloads overlap
    step i's kernels (two device buffer sets alternate). Returns (ms, h2d_bytes, d2h_bytes)
    per step, max over ranks."""
    dev, comp = st.dev, st.stream
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    pre, dec = st.h2d_names()
    host_in = {x: st.pin[x].pin_memory() for x in pre}
    host_in.update({"d" + x: st.din[x].pin_memory() for x in dec})
    outs = (["out"] if st.do_pre else []) + (["dout"] if st.do_dec else [])
    host_out = [{o: torch.empty(st.bufs[0][o].shape, dtype=st.bufs[0][o].dtype).pin_memory() for o in outs}
                for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(host_out[0][o].numel() * host_out[0][o].element_size() for o in outs)
    ev = lambda: torch.cuda.Event()

    def run(n, start_ev):
        loaded = [None] * n
        read = [None] * n     # buffer set i % 2 no longer read by step i's kernels
        fetched = [None] * n  # step i's outputs copied back
        for i in range(n):
            b = st.bufs[i % 2]
            with torch.cuda.stream(up):
                up.wait_event(start_ev)
                if i >= 2:
                    up.wait_event(read[i - 2])  # the buffer set's previous step is done with it
                for name, t in host_in.items():
                    b[name].copy_(t, non_blocking=True)
                loaded[i] = ev()
                loaded[i].record(up)
            comp.wait_event(loaded[i])
            if i >= 2:
                comp.wait_event(fetched[i - 2])  # outputs of the set's previous step are out
            if st.do_pre:
                st.prefill(i % 2, comp)
            if st.do_dec:
                st.decode(i % 2, comp)
            read[i] = ev()
            read[i].record(comp)
            with torch.cuda.stream(down):
                down.wait_event(read[i])
                for o in outs:
                    host_out[i % 2][o].copy_(b[o], non_blocking=True)
                fetched[i] = ev()
                fetched[i].record(down)
        comp.wait_event(fetched[n - 1])
        comp.wait_event(loaded[n - 1])

    s0 = torch.cuda.Event()
    s0.record(comp)
    run(2, s0)
    torch.cuda.synchronize(dev)
    _barrier(dist)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    run(steps, e0)
    e1.record(comp)
    torch.cuda.synchronize(dev)
    _barrier(dist)
    ms = _max_over_ranks(e0.elapsed_time(e1), dist) / steps
    return ms, h2d, d2h


def _traffic(kind, workload):
    tr = NCU_TRAFFIC.get((kind, workload))
    if tr is None:
        return None
    src = {"prefill": "prefill_sm100.cu", "decode": "decode_sm100.cu"}[kind]
    return tr["bytes"] if tr["source_sha"] == _src_sha(src) else None


def _describe(st, world, K, total_ms, pre_ms, dec_ms, peaks, peak_src):
    """Throughput and roofline objects of one timed step kind."""
    pre_launch_ms, dec_launch_ms = pre_ms / K, dec_ms / K
    tflops = st.flops / (pre_launch_ms * 1e-3) / 1e12 if st.do_pre else 0.0
    gbs = st.dbytes / (dec_launch_ms * 1e-3) / 1e9 if st.do_dec else 0.0
    peak_t = peaks["bf16_tflops"]
    pc, dc = st.pc, st.dc
    res = {
        "value": round(world * st.flops * K / (pre_ms * 1e-3) / 1e12, 2) if st.do_pre else 0.0,
        "ms_per_step": round(total_ms / K, 4),
        "roofline": {
            "bound": "tensor", "achieved": round(tflops, 2), "peak": peak_t, "unit": "TFLOP/s",
            "frac": round(tflops / peak_t, 4), "traffic": None,
            "kernel": "diffattn_prefill_sm100", "flops_per_launch": st.flops,
            "launch_ms": round(pre_launch_ms, 4), "peak_source": f"{peak_src} bf16_tflops (burst)",
            "frac_of_spec": round(tflops / SPEC_BF16_TFLOPS, 4), "spec_peak": SPEC_BF16_TFLOPS,
            # the same against cuBLAS held for seconds under the power cap (the prefill launches
            # run back to back for the whole timed region)
            "frac_of_sustained": (round(tflops / peaks["bf16_tflops_sustained"], 4)
                                  if peaks.get("bf16_tflops_sustained") else None),
        },
        "decode": {
            "value": round(world * st.dbytes * K / (dec_ms * 1e-3) / 1e9, 1) if st.do_dec else 0.0, "unit": "GB/s",
            "us_per_step": round(1000 * dec_launch_ms, 2),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm_gbs"], 4), "traffic": None,
                         "kernel": "diffattn_decode_split" + (" (+ lambda_v1_kernel)" if st.v1 else ""),
                         "bytes_per_launch": st.dbytes, "peak_source": f"{peak_src} hbm_gbs",
                         "frac_of_spec": round(gbs / SPEC_HBM_GBS, 4), "spec_peak": SPEC_HBM_GBS},
        },
        "prefill_cfg": {"B": pc.B, "S": pc.S, "Hq": pc.Hq, "Hkv": pc.Hkv, "D": pc.D, "causal": True,
                        "flops_per_step": st.flops} if st.do_pre else None,
        "decode_cfg": {"B": dc.B, "Smax": dc.Smax, "Hq": dc.Hq, "Hkv": dc.Hkv, "D": dc.D,
                       "sum_seqlens": int(st.din["seqlens"].sum()), "bytes_per_step": st.dbytes,
                       "lambda": "V1 (computed on the device each step)" if st.v1 else "V2 (given)"}
        if st.do_dec else None,
    }
    return res


def _workload_name(pc, dc, do_pre=True, do_dec=True):
    parts = []
    if do_pre:
        parts.append(f"causal bf16 prefill B={pc.B} S={pc.S} Hq={pc.Hq} Hkv={pc.Hkv} D={pc.D}")
    if do_dec:
        if dc.needle:
            parts.append(f"needle bf16 decode B={dc.B} x {dc.Smax} cached tokens Hq={dc.Hq} Hkv={dc.Hkv} D={dc.D}, "
                         "V1 lambda")
        else:
            parts.append(f"bf16 decode B={dc.B} Smax={dc.Smax} len U[{dc.len_lo},{dc.len_hi}] Hq={dc.Hq} "
                         f"Hkv={dc.Hkv} D={dc.D}")
    return " + ".join(parts)


def run_ours(args, rank, world, local, dist):
    import differential_attention_v2_b200 as da

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    do_pre = args.only in (None, "prefill")
    do_dec = args.only in (None, "decode")
    strong = args.scaling == "strong"
    stream = torch.cuda.current_stream(dev)
    K = args.steps
    W = max(args.warmup, 3)
    peaks, peak_src = _peaks()

    pc, pin, dc, din = _inputs(PREFILL_CFG, DECODE_CFG, rank, do_pre, do_dec, world, strong)
    st = Step(da, pc, pin if do_pre else None, dc, din if do_dec else None, dev, stream, n_buffers=2)

    def warm(s):
        for _ in range(W):
            if s.do_pre:
                s.prefill()
            if s.do_dec:
                s.decode()
        torch.cuda.synchronize(dev)
        if da.device_error(s.stream) != 0:
            raise RuntimeError("kernel reported a device-side error during warm-up")

    warm(st)
    clocks = ClockSampler(local) if rank == 0 else None
    if clocks:
        clocks.start()
    total_ms, pre_ms, dec_ms = _time_steps(st, K, dist)
    e2e_steps = max(3, min(K, 30))
    e2e_ms, h2d, d2h = _e2e(st, e2e_steps, dist)
    clk = clocks.stop() if clocks else None
    err = da.device_error(stream)
    if err:
        raise RuntimeError(f"kernel reported device error {err}")
    main = _describe(st, world, K, total_ms, pre_ms, dec_ms, peaks, peak_src)
    main_name = _workload_name(pc, dc, st.do_pre, st.do_dec)
    main_launches = st.launches
    main_flops = st.flops
    main["roofline"]["traffic"] = _traffic("prefill", PREFILL_CFG)
    main["decode"]["roofline"]["traffic"] = _traffic("decode", DECODE_CFG)

    # the second prefill and decode workloads, timed the same way in the same run
    also = None
    if not args.no_second and not args.only:
        pc2, pin2, dc2, din2 = _inputs(PREFILL_CFG_2, DECODE_CFG_2, rank, True, True, world, strong)
        del st
        torch.cuda.empty_cache()
        st2 = Step(da, pc2, pin2, dc2, din2, dev, stream)
        warm(st2)
        if clocks:
            clocks.start()
        t2, p2, d2 = _time_steps(st2, K, dist)
        clk2 = clocks.stop() if clocks else None
        err = da.device_error(stream)
        if err:
            raise RuntimeError(f"kernel reported device error {err}")
        also = _describe(st2, world, K, t2, p2, d2, peaks, peak_src)
        also["roofline"]["traffic"] = _traffic("prefill", PREFILL_CFG_2)
        also["decode"]["roofline"]["traffic"] = _traffic("decode", DECODE_CFG_2)
        also["workload"] = _workload_name(pc2, dc2)
        also["clocks"] = clk2
        also["gpu_launches"] = st2.launches * K

    if rank != 0:
        return None
    line = {
        "metric": METRIC,
        "value": main["value"],
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": main["ms_per_step"],
        "higher_is_better": True,
        "scaling": args.scaling,
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic: seeded N(0,1) q/k/v rounded to bf16, lambda = sigmoid(N(0,1)) fp32 for the prefill; "
                "needle decode: N(0,1) cache with one planted needle key per sequence, V1 lambda from "
                "N(0, 0.1^2) vectors",
        "config": {
            "workload": main_name,
            "prefill": main["prefill_cfg"],
            "decode": main["decode_cfg"],
            "parallelism": (f"head-parallel x{world} (whole GQA groups per rank, no data exchange)" if strong
                            else f"replicas x{world} (independent per-GPU batches)"),
            "l2": "no flush: inputs larger than L2 (prefill q 537 MB; the decode streams 4.3 GB per step)",
        },
        "decode": main["decode"],
        "roofline": main["roofline"],
        "e2e": {
            "value": round(world * main_flops / (e2e_ms * 1e-3) / 1e12, 3) if do_pre else None,
            "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
            "ms_per_step": round(e2e_ms, 3),
            "note": "prefill FLOPs over a step that copies the prefill's q/k/v/lambda and the decode's q, seqlens "
                    "and lambda inputs from pinned host memory, runs the kernels through the C ABI and copies both "
                    "outputs back; uploads, kernels and downloads run on three streams ordered by events, so step "
                    "i+1's uploads and step i's downloads overlap step i's kernels",
        },
        "gpu_launches": main_launches * K,
        "clocks": clk,
        "second_workload": also,
    }
    if args.only:
        line["only"] = args.only
    if world == 1 and not args.no_cpu_baseline and do_pre and do_dec:
        line["cpu_baseline"] = cpu_baseline(seconds=args.cpu_seconds, inputs=(pin, din))
    else:
        line["cpu_baseline"] = None
    return line


# ------------------------------------------------------------- the oracle on the host
def _oracle_threads():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _prefill_units(inp, case, n_units, seed):
    """Time the oracle on n_units random (b, pair, 128-row tile) units of the prefill."""
    from oracle import diffattn_f64 as ora
    import numpy as np

    rng = np.random.default_rng(seed)
    n_tiles = case.S // 128
    layout = ora.pair_layout(case.Hq, case.Hkv)
    flops = 0
    t0 = time.perf_counter()
    for _ in range(n_units):
        b = int(rng.integers(case.B))
        p = int(rng.integers(case.Hq // 2))
        t = int(rng.integers(n_tiles))
        _, h1, h2, g = layout[p]
        r0, r1 = 128 * t, 128 * t + 128
        kk = inp["k"][b, :r1, g].double().numpy()
        vv = inp["v"][b, :r1, g].double().numpy()
        q1 = inp["q"][b, r0:r1, h1].double().numpy()
        q2 = inp["q"][b, r0:r1, h2].double().numpy()
        lm = inp["lam"][b, r0:r1, p].double().numpy()
        ora.diff_attention_block(q1, q2, kk, vv, lm, ora.causal_mask(128, r1, r0))
        flops += 4 * case.D * 2 * sum(r + 1 for r in range(r0, r1))  # both heads of the pair
    return flops, time.perf_counter() - t0


def _decode_seqs(inp, case, n_seqs, seed):
    from oracle import diffattn_f64 as ora
    import numpy as np

    rng = np.random.default_rng(seed)
    byts = 0
    t0 = time.perf_counter()
    for _ in range(n_seqs):
        b = int(rng.integers(case.B))
        n = int(inp["seqlens"][b])
        sl = inp["seqlens"][b:b + 1]
        if inp["lam"] is None:  # V1 lambda: one value per pair from the four vectors
            lam = ora.lambda_v1(inp["lq1"], inp["lk1"], inp["lq2"], inp["lk2"], inp["lambda_init"])[None, :]
        else:
            lam = inp["lam"][b:b + 1]
        ora.decode(inp["q"][b:b + 1], inp["kcache"][b:b + 1], inp["vcache"][b:b + 1], sl, lam)
        byts += n * case.Hkv * case.D * 2 * 2
    return byts, time.perf_counter() - t0


def _blas_name():
    """Name of the BLAS library NumPy was built against (the oracle's matrix products)."""
    try:
        import numpy as np

        cfg = np.show_config(mode="dicts")
        blas = cfg.get("Build Dependencies", {}).get("blas", {})
        return f"{blas.get('name', '?')} {blas.get('version', '')}".strip()
    except Exception:  # older NumPy: no dict mode
        return "unknown"


def cpu_baseline(seconds=15.0, inputs=None):
    """The float64 oracle on a bounded sample of the same workload, timed on the host."""
    pc = workloads.CONFIGS[PREFILL_CFG]
    dc = workloads.CONFIGS[DECODE_CFG]
    if inputs is None:
        inputs = (workloads.make_prefill(pc), workloads.make_decode(dc))
    pin, din = inputs
    # calibrate with 4 units, then size the sample to about `seconds` of CPU work
    f, t = _prefill_units(pin, pc, 4, seed=1)
    n = max(4, int(0.8 * seconds / max(t / 4, 1e-6)))
    f, t = _prefill_units(pin, pc, n, seed=2)
    b, td = _decode_seqs(din, dc, 1, seed=3)
    return {"value": round(f / t / 1e12, 6), "unit": "TFLOP/s", "cores": _oracle_threads(), "kind": "oracle",
            "sample": f"{n} random (batch, pair, 128-row tile) units of the B={pc.B} S={pc.S} prefill "
                      f"({t:.1f} s); decode: 1 full sequence of the B={dc.B} x {dc.Smax} decode ({td:.1f} s)",
            "decode_gbs": round(b / td / 1e9, 4), "blas": _blas_name()}


def run_reference(args):
    """The oracle as the reference arm: each step a bounded sample of the same workload,
    sized so that the whole run stays within a few minutes of host time."""
    pc = workloads.CONFIGS[PREFILL_CFG]
    dc = workloads.CONFIGS[DECODE_CFG]
    pin, din = workloads.make_prefill(pc), workloads.make_decode(dc)
    f, t = _prefill_units(pin, pc, 2, seed=99)
    per_unit = t / 2
    budget = min(3.0, max(0.05, args.ref_seconds / max(1, args.steps + args.warmup)))
    units = max(1, int(0.8 * budget / per_unit))
    for i in range(args.warmup):
        _prefill_units(pin, pc, units, seed=100 + i)
    flops, secs = 0, 0.0
    dbytes, dsecs = 0, 0.0
    for i in range(args.steps):
        f, t = _prefill_units(pin, pc, units, seed=1000 + i)
        flops += f
        secs += t
        if i % max(1, args.steps // 8) == 0:
            b, td = _decode_seqs(din, dc, 1, seed=2000 + i)
            dbytes += b
            dsecs += td
    value = flops / secs / 1e12
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1000 * secs / args.steps, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic: the same seeded inputs as the GPU arm",
        "config": {"workload": _workload_name(pc, dc), "sample": "each step a bounded sample",
                   "prefill_units_per_step": units},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": _oracle_threads(), "kind": "oracle",
                         "sample": f"{units} random (batch, pair, 128-row tile) prefill units per step; "
                                   f"decode: one full sequence on every {max(1, args.steps // 8)}-th step"},
        "decode": {"value": round(dbytes / dsecs / 1e9, 4) if dsecs else None, "unit": "GB/s"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


# ------------------------------------------------------------ single-operation lines
def _time_op(fn, steps, warmup, stream):
    """Milliseconds per call of `fn` (which launches on the current stream): `warmup` eager
    calls, then `steps` calls captured in one CUDA graph and replayed once, timed with CUDA
    events around the replay (the graph removes the host launch gaps that back-to-back eager
    launches of a short kernel would add). Falls back to eager launches if capture fails.
    Returns (ms, how)."""
    for _ in range(max(warmup, 3)):
        fn()
    torch.cuda.synchronize()
    how = f"one CUDA graph of {steps} launches"
    try:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for _ in range(steps):
                fn()
        run = graph.replay
        run()  # one untimed replay
    except Exception:  # capture not possible here: time eager launches
        how = f"{steps} eager launches"
        torch.cuda.synchronize()

        def run():
            for _ in range(steps):
                fn()
    torch.cuda.synchronize()
    cur = torch.cuda.current_stream()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(cur)
    run()
    t1.record(cur)
    torch.cuda.synchronize()
    return t0.elapsed_time(t1) / steps, how


def run_workload(args):
    """One operation of the operator's scope on one GPU, timed alone (CUDA events over
    `steps` back-to-back launches after `warmup`): the second prefill and decode workloads
    and the next rows (sliding window, packed prefill, paged and multi-token decode, the V2
    lambda projection). Prints one JSON line with its own metric, work count and roofline."""
    import differential_attention_v2_b200 as da

    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    peaks, peak_src = _peaks()
    name = args.workload
    D = 128
    if name in ("prefill", "prefill_long", "window", "varlen"):
        if name == "varlen":
            g = torch.Generator().manual_seed(1010)
            lens = torch.randint(512, 3585, (8,), generator=g).tolist()
            T = sum(lens)
            case = workloads.PrefillCase(B=1, S=T, Hq=64, Hkv=8, D=D, seed=1010)
            inp = workloads.make_prefill(case)
            q, k, v, lam = (inp[x][0].to(dev) for x in ("q", "k", "v", "lam"))
            cu = torch.tensor([0] + list(torch.tensor(lens).cumsum(0).tolist()), dtype=torch.int32, device=dev)
            out = torch.empty(T, 32, D, dtype=torch.bfloat16, device=dev)
            fn = lambda: da.prefill_varlen(q, k, v, lam, cu, max(lens), out=out)
            flops = sum(4 * D * 64 * L * (L + 1) // 2 for L in lens)
            cfg = {"workload": f"packed causal prefill of 8 sequences, lengths U[512,3584] (total {T}), Hq=64 Hkv=8 D=128",
                   "lengths": lens}
        else:
            case = workloads.CONFIGS["prefill_b1_s32768"] if name == "prefill_long" else workloads.CONFIGS["prefill_b4_s4096"]
            inp = workloads.make_prefill(case)
            q, k, v, lam = (inp[x].to(dev) for x in ("q", "k", "v", "lam"))
            out = torch.empty(case.B, case.S, case.Hq // 2, D, dtype=torch.bfloat16, device=dev)
            if name == "window":
                W = 1024
                fn = lambda: da.prefill_window(q, k, v, lam, W, out=out)
                flops = 4 * D * case.Hq * case.B * sum(min(i + 1, W) for i in range(case.S))
                cfg = {"workload": f"sliding-window causal prefill, window {W}, B=4 S=4096 Hq=64 Hkv=8 D=128"}
            else:
                fn = lambda: da.prefill(q, k, v, lam, out=out)
                flops = workloads.prefill_flops(case.B, case.S, case.Hq, D)
                cfg = {"workload": f"causal prefill B={case.B} S={case.S} Hq=64 Hkv=8 D=128"}
        ms, how = _time_op(fn, args.steps, args.warmup, stream)
        val = flops / (ms * 1e-3) / 1e12
        unit, peak, bound = "TFLOP/s", peaks["bf16_tflops"], "tensor"
        launches = 1
    elif name == "decode_window":
        # the needle decode's caches (B=8 x 131072) read through a 4096-key window: bytes = the
        # window's K and V rows, plus q, lambda and out
        case = workloads.CONFIGS["needle_decode_b8_s131072"]
        inp = workloads.make_decode(case)
        kc, vc, sl, q = (inp[x].to(dev) for x in ("kcache", "vcache", "seqlens", "q"))
        lam = da.lambda_v1(*(inp[x].to(dev) for x in ("lq1", "lk1", "lq2", "lk2")), inp["lambda_init"], rows=case.B)
        W = 4096
        out = torch.empty(case.B, case.Hq // 2, D, dtype=torch.bfloat16, device=dev)
        ws = torch.empty(da.decode_workspace_size(case.B, case.Smax, case.Hq, case.Hkv, D), dtype=torch.uint8, device=dev)
        fn = lambda: da.decode(q, kc, vc, sl, lam, out=out, workspace=ws, window=W)
        nbytes = workloads.decode_bytes([min(int(n), W) for n in inp["seqlens"].tolist()], case.Hkv, D, case.Hq)
        ms, how = _time_op(fn, args.steps, args.warmup, stream)
        val = nbytes / (ms * 1e-3) / 1e9
        unit, peak, bound = "GB/s", peaks["hbm_gbs"], "hbm"
        launches = 1
        cfg = {"workload": "sliding-window decode (window 4096) of B=8 sequences of 131072 cached tokens, Hq=64 Hkv=8"}
    elif name in ("decode", "decode_needle", "paged", "multi"):
        case = workloads.CONFIGS["needle_decode_b8_s131072"] if name == "decode_needle" else workloads.CONFIGS["decode_b64_s8192"]
        inp = workloads.make_decode(case)
        kc, vc, sl = (inp[x].to(dev) for x in ("kcache", "vcache", "seqlens"))
        if inp["lam"] is None:
            lam = da.lambda_v1(*(inp[x].to(dev) for x in ("lq1", "lk1", "lq2", "lk2")), inp["lambda_init"], rows=case.B)
        else:
            lam = inp["lam"].to(dev)
        q = inp["q"].to(dev)
        nbytes = workloads.decode_bytes(inp["seqlens"].tolist(), case.Hkv, D, case.Hq)
        launches = 1
        if name == "paged":
            ps = 64
            max_pages = case.Smax // ps
            perm = torch.randperm(case.B * max_pages, generator=torch.Generator().manual_seed(7))
            table = perm.view(case.B, max_pages).to(torch.int32).to(dev)
            kp = torch.empty(case.B * max_pages, ps, case.Hkv, D, dtype=torch.bfloat16, device=dev)
            vp = torch.empty_like(kp)
            kp[perm.to(dev)] = kc.view(case.B * max_pages, ps, case.Hkv, D)
            vp[perm.to(dev)] = vc.view(case.B * max_pages, ps, case.Hkv, D)
            del kc, vc
            out = torch.empty(case.B, case.Hq // 2, D, dtype=torch.bfloat16, device=dev)
            ws = torch.empty(da.decode_workspace_size(case.B, case.Smax, case.Hq, case.Hkv, D), dtype=torch.uint8, device=dev)
            fn = lambda: da.decode_paged(q, kp, vp, table, sl, lam, out=out, workspace=ws)
            nbytes += case.B * max_pages * 4
            cfg = {"workload": "paged decode (page size 64, shuffled pages) of B=64, lengths U[1024,8192], Hq=64 Hkv=8"}
        elif name == "multi":
            Tn = 2
            g = torch.Generator().manual_seed(11)
            qm = torch.randn(case.B, Tn, case.Hq, D, generator=g).bfloat16().to(dev)
            lm = torch.sigmoid(torch.randn(case.B, Tn, case.Hq // 2, generator=g)).to(dev)
            out = torch.empty(case.B, Tn, case.Hq // 2, D, dtype=torch.bfloat16, device=dev)
            wsm = torch.empty(da.LIB.diffattn_v2_decode_multi_workspace_size(case.B, Tn, case.Smax, case.Hq, case.Hkv, D),
                              dtype=torch.uint8, device=dev)
            fn = lambda: da.decode_multi(qm, kc, vc, sl, lm, out=out, workspace=wsm)
            nbytes += (Tn - 1) * case.B * (case.Hq * D * 2 + case.Hq // 2 * (4 + D * 2))
            cfg = {"workload": "2-token (speculative) decode of B=64, lengths U[1024,8192], Hq=64 Hkv=8"}
        else:
            out = torch.empty(case.B, case.Hq // 2, D, dtype=torch.bfloat16, device=dev)
            ws = torch.empty(da.decode_workspace_size(case.B, case.Smax, case.Hq, case.Hkv, D), dtype=torch.uint8, device=dev)
            fn = lambda: da.decode(q, kc, vc, sl, lam, out=out, workspace=ws)
            cfg = {"workload": "needle decode B=8, 131072 cached tokens each, V1 lambda, Hq=64 Hkv=8" if name == "decode_needle"
                   else "decode B=64, lengths U[1024,8192], V2 lambda given, Hq=64 Hkv=8"}
        ms, how = _time_op(fn, args.steps, args.warmup, stream)
        val = nbytes / (ms * 1e-3) / 1e9
        unit, peak, bound = "GB/s", peaks["hbm_gbs"], "hbm"
    elif name == "backward":
        case = workloads.CONFIGS["prefill_b4_s4096"]
        inp = workloads.make_prefill(case)
        q, k, v, lam = (inp[x].to(dev) for x in ("q", "k", "v", "lam"))
        dout = workloads.make_prefill_grad(case).to(dev)
        out, ob, lse = da.prefill_train(q, k, v, lam)
        grads = [torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(lam)]
        ws = torch.empty(da.backward_workspace_size(case.B, case.S, case.Hq), dtype=torch.uint8, device=dev)
        fwd_ms, _ = _time_op(lambda: da.prefill_train(q, k, v, lam, out=out, o_branch=ob, lse=lse),
                             args.steps, args.warmup, stream)
        fn = lambda: da.backward(q, k, v, lam, ob, lse, dout, dq=grads[0], dk=grads[1], dv=grads[2], dlam=grads[3],
                                 workspace=ws)
        # chain-rule products per pair and visible (query, key): S_1, S_2 recomputed, dP shared
        # by both branches, dV from the combined weights, dK and dQ of both heads: 8 products
        # of 2*D flops each, twice the forward's 4
        flops = 2 * workloads.prefill_flops(case.B, case.S, case.Hq, D)
        ms, how = _time_op(fn, args.steps, args.warmup, stream)
        val = flops / (ms * 1e-3) / 1e12
        unit, peak, bound = "TFLOP/s", peaks["bf16_tflops"], "tensor"
        launches = 3
        cfg = {"workload": "backward of the causal prefill B=4 S=4096 Hq=64 Hkv=8 D=128 (dQ, dK, dV, dlambda)",
               "train_forward_ms": round(fwd_ms, 4),
               "train_forward_tflops": round(workloads.prefill_flops(case.B, case.S, case.Hq, D) / (fwd_ms * 1e-3) / 1e12, 2)}
    elif name == "backward_window":
        case = workloads.CONFIGS["prefill_b4_s4096"]
        W = 1024
        inp = workloads.make_prefill(case)
        q, k, v, lam = (inp[x].to(dev) for x in ("q", "k", "v", "lam"))
        dout = workloads.make_prefill_grad(case).to(dev)
        out, ob, lse = da.prefill_train(q, k, v, lam, window=W)
        ws = torch.empty(da.backward_workspace_size(case.B, case.S, case.Hq), dtype=torch.uint8, device=dev)
        fn = lambda: da.backward(q, k, v, lam, ob, lse, dout, workspace=ws, window=W)
        flops = 2 * 4 * D * case.Hq * case.B * sum(min(i + 1, W) for i in range(case.S))
        ms, how = _time_op(fn, args.steps, args.warmup, stream)
        val = flops / (ms * 1e-3) / 1e12
        unit, peak, bound = "TFLOP/s", peaks["bf16_tflops"], "tensor"
        launches = 3
        cfg = {"workload": f"backward of the sliding-window causal prefill, window {W}, B=4 S=4096 Hq=64 Hkv=8 D=128"}
    elif name == "backward_varlen":
        g = torch.Generator().manual_seed(1010)
        lens = torch.randint(512, 3585, (8,), generator=g).tolist()
        T = sum(lens)
        case = workloads.PrefillCase(B=1, S=T, Hq=64, Hkv=8, D=D, seed=1010)
        inp = workloads.make_prefill(case)
        q, k, v, lam = (inp[x][0].to(dev) for x in ("q", "k", "v", "lam"))
        dout = workloads.make_prefill_grad(case)[0].to(dev)
        cu = torch.tensor([0] + list(torch.tensor(lens).cumsum(0).tolist()), dtype=torch.int32, device=dev)
        out, ob, lse = da.prefill_varlen_train(q, k, v, lam, cu, max(lens))
        ws = torch.empty(da.backward_varlen_workspace_size(len(lens), T, 64), dtype=torch.uint8, device=dev)
        fn = lambda: da.backward_varlen(q, k, v, lam, ob, lse, dout, cu, max(lens), workspace=ws)
        flops = 2 * sum(4 * D * 64 * L * (L + 1) // 2 for L in lens)
        ms, how = _time_op(fn, args.steps, args.warmup, stream)
        val = flops / (ms * 1e-3) / 1e12
        unit, peak, bound = "TFLOP/s", peaks["bf16_tflops"], "tensor"
        launches = 4
        cfg = {"workload": f"backward of the packed causal prefill of 8 sequences, lengths U[512,3584] (total {T}), "
                           "Hq=64 Hkv=8 D=128", "lengths": lens}
    elif name == "lambda_v2":
        T, dm, npair = 16384, 4096, 32
        g = torch.Generator().manual_seed(12)
        x = torch.randn(T, dm, generator=g).bfloat16().to(dev)
        w = (torch.randn(dm, npair, generator=g) / dm ** 0.5).bfloat16().to(dev)
        b = torch.randn(npair, generator=g).to(dev)
        out = torch.empty(T, npair, dtype=torch.float32, device=dev)
        fn = lambda: da.lambda_v2(x, w, b, out=out)
        nbytes = T * dm * 2 + dm * npair * 2 + npair * 4 + T * npair * 4
        ms, how = _time_op(fn, args.steps, args.warmup, stream)
        val = nbytes / (ms * 1e-3) / 1e9
        unit, peak, bound = "GB/s", peaks["hbm_gbs"], "hbm"
        launches = 1
        cfg = {"workload": "V2 lambda projection sigmoid(x W + b): T=16384 tokens, d_model=4096, 32 pairs"}
    elif name == "prefill_fused_lambda":
        # B=4 x 4096 causal prefill whose V2 lambda comes from x [B,S,4096] inside the kernel,
        # timed against the two-launch path (projection on the tensor cores, then the prefill)
        case = workloads.CONFIGS["prefill_b4_s4096"]
        inp = workloads.make_prefill(case)
        q, k, v = (inp[x].to(dev) for x in ("q", "k", "v"))
        dm, npair = 4096, case.Hq // 2
        g = torch.Generator().manual_seed(13)
        xh = torch.randn(case.B * case.S, dm, generator=g).bfloat16().to(dev)
        w = (torch.randn(dm, npair, generator=g) / dm ** 0.5).bfloat16().to(dev)
        wt = w.t().contiguous()
        b = torch.randn(npair, generator=g).to(dev)
        out = torch.empty(case.B, case.S, npair, D, dtype=torch.bfloat16, device=dev)
        lam = torch.empty(case.B * case.S, npair, dtype=torch.float32, device=dev)
        x3 = xh.view(case.B, case.S, dm)
        fn = lambda: da.prefill_fused_lambda(q, k, v, x3, wt, b, out=out)
        flops = workloads.prefill_flops(case.B, case.S, case.Hq, D)
        ms, how = _time_op(fn, args.steps, args.warmup, stream)

        def two_launch():
            da.lambda_v2(xh, w, b, out=lam)
            da.prefill(q, k, v, lam.view(case.B, case.S, npair), out=out)

        ms2, _ = _time_op(two_launch, args.steps, args.warmup, stream)
        val = flops / (ms * 1e-3) / 1e12
        unit, peak, bound = "TFLOP/s", peaks["bf16_tflops"], "tensor"
        launches = 1
        cfg = {"workload": "causal prefill B=4 S=4096 Hq=64 Hkv=8 D=128 with the V2 lambda computed in the kernel "
                           "from x [4, 4096, 4096] bf16",
               "two_launch_ms": round(ms2, 4), "two_launch_tflops": round(flops / (ms2 * 1e-3) / 1e12, 2)}
    else:
        raise SystemExit(f"unknown workload {name}")
    err = da.device_error(stream)
    if err:
        raise RuntimeError(f"kernel reported device error {err}")
    line = {"metric": f"{name}: {unit}", "value": round(val, 2), "unit": unit, "n_gpus": 1, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic, seeded", "config": cfg,
            "roofline": {"bound": bound, "achieved": round(val, 2), "peak": peak, "unit": unit,
                         "frac": round(val / peak, 4), "traffic": None,
                         "frac_of_spec": round(val / (SPEC_BF16_TFLOPS if bound == "tensor" else SPEC_HBM_GBS), 4),
                         "peak_source": f"{peak_src} {'bf16_tflops (burst)' if bound == 'tensor' else 'hbm_gbs'}"},
            "gpu_launches": launches * args.steps, "workload": name, "timing": how}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-second", action="store_true",
                    help="skip the second prefill and decode workloads (B=4 x 4k prefill, B=64 decode)")
    ap.add_argument("--ref-seconds", type=float, default=120.0,
                    help="host-time budget of the whole reference run (warm-up and timed steps)")
    ap.add_argument("--workload", choices=("prefill", "decode", "prefill_long", "decode_needle", "decode_window",
                                           "window", "varlen",
                                           "paged", "multi", "prefill_fused_lambda",
                                           "lambda_v2", "backward", "backward_varlen", "backward_window"),
                    default=None,
                    help="time one other operation alone instead of the default step")
    ap.add_argument("--scaling", choices=("weak", "strong"), default="weak",
                    help="weak: each GPU runs the full per-GPU workload; strong: the heads of one workload "
                         "are split over the GPUs")
    ap.add_argument("--only", choices=("prefill", "decode"), default=None,
                    help="run one half of the step (for profiling a single kernel on less device memory)")
    args = ap.parse_args(argv)

    if args.workload:
        run_workload(args)
        return 0
    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) != 0:
            return 0
        print(json.dumps(run_reference(args)), flush=True)
        return 0

    rank, world, local, dist = _dist_init(args.gpus)
    try:
        line = run_ours(args, rank, world, local, dist)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if dist is not None:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
