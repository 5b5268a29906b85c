"""Benchmark of the FOCUS NVFP4 weight fake-quantizer on B200.

Workload: every linear weight of Llama-3.1-8B (32 layers x q, k, v, o, gate,
up, down: 224 tensors, 6,979,321,856 weights), synthetic: W ~ N(0, 0.02) bf16,
m = 1, q = 6, dW' ~ N(0, 1e-3) bf16, zero AdamW moments at step 1.  One step
is one pass of the whole hot path over all 224 tensors:
  the fused forward + straight-through backward + AdamW step with the NVFP4
  export of the updated parameters (one launch, W' written, W read once),
  which also reduces the block maxima it computes into each tensor's max |w|;
  then s2 = max/2688 of every tensor for the next step (one small launch).
  s2 of every tensor is computed by a separate pass once before the first
  step; W is frozen, so each step's s2 equals that pass's (tested).
Metric: Gelem/s = weights per second of whole steps (all ranks).  The
roofline object reports the fused step kernel against the measured HBM copy
bandwidth.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 it is launched by torch.distributed.run, one rank per GPU; every
rank steps its own model (seeded by rank: weak scaling, no data-path
collective), the time is the max over ranks.  The reference arm times the CPU
oracle on the host cores (rank 0 only), on a bounded row sample per step.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Gelem/s FOCUS fwd+STE-bwd+AdamW and % of B200 HBM roofline (ncu)"
WORKLOAD = "Llama-3.1-8B all 224 linear weights (32 layers x q,o[4096,4096] k,v[1024,4096] " \
           "gate,up[14336,4096] down[4096,14336]); step = one fused kernel: fwd (W' written), STE-bwd, " \
           "AdamW, NVFP4 export pack of the updated m and q, and the tensor maxima for s2; then s2 of every " \
           "tensor (one thread per tensor)"
# algorithmic bytes per weight of one step: the fused step reads W, dW' (2+2), m (0.25), q (0.5), four
# moments (1.5) and writes W' (2), m, q, moments (2.25), NVFP4 codes (0.5) and scales (0.0625); the s2 of
# the next step comes from the block maxima of the same read of W
BYTES_STEP = 11.0625
KERNEL_SOURCES = ("fp4_post_weight_b200/csrc/focus_kernels.cuh", "fp4_post_weight_b200/csrc/focus_device.cuh",
                  "fp4_post_weight_b200/csrc/focus_pipeline.cuh", "fp4_post_weight_b200/csrc/focus_capi.cu")
TRAFFIC_RECORD = "profiles/step_traffic.json"


def kernel_source_hash() -> str:
    """Hash of the code (comments and whitespace removed) of the kernel sources:
    the recorded DRAM traffic is valid while it is unchanged."""
    import re
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(os.path.join(ROOT, p)) as f:
            src = f.read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        h.update(re.sub(r"\s+", "", src).encode())
    return h.hexdigest()[:16]


def measured_peaks() -> dict:
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "source": "fallback"}


def recorded_traffic():
    """DRAM bytes per launch of the fused step kernel on the full workload, from the
    committed record of an ncu capture (profiles/step_traffic.json); None once the
    kernel sources differ from those the counters were taken with."""
    try:
        with open(os.path.join(ROOT, TRAFFIC_RECORD)) as f:
            d = json.load(f)
    except Exception:
        return None
    if d.get("kernel_source_hash") != kernel_source_hash():
        return None
    return d.get("dram_bytes_per_launch_full_workload")


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------

def init_dist(world, local):
    import datetime

    import torch
    import torch.distributed as dist
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local))


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = "clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active," \
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown," \
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap"

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(5)
        except Exception:
            self.proc.kill()
        self.out.flush()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.out.name) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) < 8:
                    continue
                try:
                    sm.append(float(p[0])); mx.append(float(p[1]))
                except ValueError:
                    continue
                for n, v in zip(names, p[4:8]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.out.name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# the workload
# ---------------------------------------------------------------------------

def model_tensors(layers: int):
    import synth
    return synth.LLAMA_8B.tensors()[:7 * layers]


def build_model(rank: int, device, layers: int = 32):
    import torch

    from fp4_post_weight_b200 import dist as D
    import synth
    from fp4_post_weight_b200.table import Entry
    ents = []
    for j, (_, sh) in enumerate(model_tensors(layers)):
        t = synth.llama_8b_tensor(j, sh, device, seed_base=D.seed_base(rank))
        o, i = sh
        e = Entry(W=t.W, m=t.m, q=t.q, s2=torch.zeros(1, device=device), dWq=t.dWq,
                  Wq=torch.empty_like(t.W), m_exp_avg=torch.zeros_like(t.m), m_exp_avg_sq=torch.zeros_like(t.m),
                  q_exp_avg=torch.zeros_like(t.q), q_exp_avg_sq=torch.zeros_like(t.q),
                  codes=torch.empty((o, i // 2), dtype=torch.uint8, device=device),
                  scales=torch.empty((o, i // 16), dtype=torch.uint8, device=device))
        ents.append(e)
    return ents


def run_ours(args, world, rank, local):
    import torch

    import synth
    from fp4_post_weight_b200 import dist as D
    from fp4_post_weight_b200 import focus as F
    from fp4_post_weight_b200.table import FocusTable, hparams

    init_dist(world, local)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    ents = build_model(rank, dev, args.layers)
    N = sum(o * i for _, (o, i) in model_tensors(args.layers))
    # one table: the step writes W' and exports the updated parameters as NVFP4
    step_tab = FocusTable(ents)
    hp = hparams()
    flags = F.FOCUS_STEP_PACK_UPDATED
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()

    t_counter = [0]

    def one_step(ev=None):
        # one pass of the whole path: the fused step (forward, straight-through
        # backward, AdamW, NVFP4 export of the updated parameters), which also
        # reduces the block maxima it computes into each tensor's max |w|, then s2
        # of every tensor for the next step (W is frozen: the value a separate
        # s2 pass would give)
        t_counter[0] += 1
        if ev is not None:
            ev[0].record(stream)
        F.focus_step_fused_amax(step_tab.dev, step_tab.n, step_tab.total_tiles, hp, t_counter[0], amax_ws, flags)
        if ev is not None:
            ev[1].record(stream)
        F.focus_s2_from_amax(step_tab.dev, step_tab.n, amax_ws)

    step_tab.s2()                  # s2 of every tensor before the first step
    amax_ws = torch.zeros(max(step_tab.n, 4), dtype=torch.int32, device=dev)
    # The CPU baseline times the oracle on a row sample of this workload; its
    # outputs are checked against what the first warm-up step computed for the
    # same rows (the inputs are the generator's, taken before that step).
    do_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    sample = None
    if do_cpu:
        sample = ParitySample(ents, int(_oracle_rate() * args.cpu_seconds))
    for w in range(args.warmup):
        one_step()
        if w == 0 and sample is not None:
            sample.read_outputs(ents)
    st = F.focus_get_error()
    if st != 0:
        raise SystemExit(f"device status after warm-up: {F.focus_status_string(st)}")
    torch.cuda.synchronize()
    D.barrier()

    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid).replace("GPU-", "")
    clocks = ClockSampler(gpu_id)
    clocks.start()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    torch.cuda.synchronize()
    D.barrier()
    start.record(stream)
    for k in range(args.steps):
        one_step(kev[k])
    end.record(stream)
    torch.cuda.synchronize()
    D.barrier()
    clk = clocks.stop()
    ms = start.elapsed_time(end)
    kms = [a.elapsed_time(b) for a, b in kev]
    step_kernel_ms = sum(kms) / args.steps
    if max(kms) > 1.5 * min(kms):
        print(f"warning: fused-step launch times vary from {min(kms):.2f} to {max(kms):.2f} ms "
              "(another job on this GPU?)", file=sys.stderr)
    ms_max = D.max_over_ranks(ms)
    st = F.focus_get_error()
    if st != 0:
        raise SystemExit(f"device status after timing: {F.focus_status_string(st)}")
    ms_per_step = ms_max / args.steps
    value = N * world / (ms_per_step * 1e-3) / 1e9

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, ents, N, world, dev)

    peaks = measured_peaks()
    achieved = N * BYTES_STEP / (step_kernel_ms * 1e-3) / 1e9
    roof = {"bound": "hbm", "kernel": "pipe_kernel<KIND_STEP> (focus_step_fused_amax: step, export pack, tensor maxima)", "achieved": round(achieved, 1),
            "peak": peaks["hbm_gbs"], "peak_source": peaks["source"] + " (MEASURED_PEAKS.json hbm_gbs, copy)",
            "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": recorded_traffic(),
            "nominal_gbs": 8000.0, "frac_of_nominal": round(achieved / 8000.0, 4),
            "bytes_per_elem": BYTES_STEP, "launch_ms": round(step_kernel_ms, 4)}
    rows = None
    if not args.no_rows:
        rows = measure_next_rows(ents, dev, N, peaks, world)
    cpu = parity = None
    if sample is not None:
        cpu, parity = cpu_baseline(ents, sample)
    if rank == 0:
        line = {"metric": METRIC, "value": round(value, 2), "unit": "Gelem/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic (seeded N(0,0.02) bf16 weights of the Llama-3.1-8B linear shapes; "
                        "no checkpoint)",
                "config": {"workload": WORKLOAD if args.layers == 32 else
                           f"first {args.layers} layers of: " + WORKLOAD, "tensors": len(ents), "elements_per_gpu": N,
                           "l2": f"inputs larger than L2 ({N * 8.25 / 1e9:.1f} GB resident per GPU vs 126 MB L2)",
                           "parallelism": f"dp{world} (one model per GPU, no collective)",
                           "bytes_per_elem_step": BYTES_STEP},
                "roofline": roof, "cpu_baseline": cpu, "parity": parity, "e2e": e2e, "next_rows": rows,
                "gpu_launches": 2 * args.steps, "clocks": clk,
                "kernel_ms": {"fused_step": round(step_kernel_ms, 4), "fused_step_min": round(min(kms), 4),
                              "fused_step_max": round(max(kms), 4),
                              "fused_step_median": round(statistics.median(kms), 4),
                              "fused_step_last5_mean": round(sum(kms[-5:]) / len(kms[-5:]), 4),
                              "fused_step_each": [round(x, 3) for x in kms],
                              "fused_step_ms_x_median_sm_mhz": (round(step_kernel_ms * clk["sm_mhz"], 1)
                                                                if clk.get("sm_mhz") else None)}}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def _timed(fn, stream, reps: int = 5, warm: int = 3):
    """Mean device time (ms) of fn() over reps calls, each bracketed by events on stream."""
    import torch
    for _ in range(warm):
        fn()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    torch.cuda.synchronize()
    for a, b in ev:
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in ev) / reps


def _roof(bytes_moved: float, ms: float, peak: float) -> dict:
    gbs = bytes_moved / (ms * 1e-3) / 1e9
    return {"ms": round(ms, 4), "achieved_gbs": round(gbs, 1), "frac": round(gbs / peak, 4)}


def measure_next_rows(ents, dev, N, peaks, world):
    """The rows after the hot path, each timed per launch with CUDA events on the
    launching stream, after the headline's timed region (inputs larger than L2):
      * FourOverSix round to nearest over the same 224 weights (one launch; codes
        and scales, and codes, scales and W');
      * FourOverSix with one scale per token over one decoder layer's linear
        inputs for a micro-batch of 4096 tokens (q/k/v, o and gate/up inputs
        [4096, 4096], the down input [4096, 14336]: 218 MB), one launch over
        the four tensors (and, for comparison, one launch per width);
      * a calibration step over four micro-batches: three table backward passes
        (the first overwriting dm/dq, then accumulating) and the fused step
        with FOCUS_STEP_ACCUMULATE | FOCUS_STEP_WQ_UPDATED;
      * the same step unfused (forward, backward, standalone AdamW: 15.5 B per
        weight in 450 launches), for what the fusion buys;
      * Llama-3.1-70B generated on the device and stepped one layer at a time
        (layers 0, 40, 79: s2, then the fused step with the export), per layer;
      * the MXFP4 variant's fused step over the same 224 weights (one launch per
        tensor; reads W, dW', m, q and moments, writes W', m, q and moments:
        9.75 B per weight)."""
    import torch

    import synth
    from fp4_post_weight_b200 import focus as F
    from fp4_post_weight_b200.table import PURPOSE_FOUROVERSIX, PURPOSE_MX, Entry, FocusTable, hparams
    from fp4_post_weight_b200 import dist as D
    stream = torch.cuda.current_stream(dev)
    peak = peaks["hbm_gbs"]
    out = {}
    # FourOverSix weights
    t_cs = FocusTable([Entry(W=e.W, m=None, q=None, s2=e.s2, codes=e.codes, scales=e.scales) for e in ents],
                      PURPOSE_FOUROVERSIX)
    t_all = FocusTable([Entry(W=e.W, m=None, q=None, s2=e.s2, codes=e.codes, scales=e.scales, Wq=e.Wq)
                        for e in ents], PURPOSE_FOUROVERSIX)
    ms = _timed(t_cs.fouroversix, stream)
    r = {"kernel": "pipe_kernel<KIND_F46>", "bytes_per_weight": 2.5625, **_roof(2.5625 * N, ms, peak)}
    ms = _timed(t_all.fouroversix, stream)
    r["with_Wq"] = {"bytes_per_weight": 4.5625, **_roof(4.5625 * N, ms, peak)}
    r["Gelem_s"] = round(N * world / (r["ms"] * 1e-3) / 1e9, 2)
    out["fouroversix_weights_llama8b"] = r
    # plain NVFP4 round to nearest of the weights (the target 6 alone), codes + scales
    ms = _timed(t_cs.nvfp4_rtn, stream)
    out["nvfp4_rtn_weights_llama8b"] = {"kernel": "pipe_kernel<KIND_RTN>", "bytes_per_weight": 2.5625,
                                        "Gelem_s": round(N * world / (ms * 1e-3) / 1e9, 2),
                                        **_roof(2.5625 * N, ms, peak)}
    # FourOverSix activations, one scale per token: one launch over the layer's four
    # activation tensors (rows staged in shared memory)
    from fp4_post_weight_b200.table import ActTable, act_entry
    Xs = [synth.activations(4096, h, dev, seed=50 + j) for j, h in enumerate((4096, 4096, 4096, 14336))]
    bufs = [(torch.empty(X.shape[0], device=dev), torch.empty((X.shape[0], X.shape[1] // 2), dtype=torch.uint8,
                                                                device=dev),
             torch.empty((X.shape[0], X.shape[1] // 16), dtype=torch.uint8, device=dev)) for X in Xs]
    n_act = sum(X.numel() for X in Xs)
    b_act = sum(X.numel() * (2 + 0.5 + 0.0625) + 4 * X.shape[0] for X in Xs)
    act_tab = ActTable([act_entry(X, ts, c, sc) for X, (ts, c, sc) in zip(Xs, bufs)])
    ms = _timed(act_tab.fouroversix, stream)
    out["fouroversix_act_4096_tokens_one_layer"] = {"kernel": "rows_staged_kernel", "launches": 1,
                                                     "elements": n_act, "bytes_per_elem": 2.5625,
                                                     "Gelem_s": round(n_act / (ms * 1e-3) / 1e9, 2),
                                                     **_roof(b_act, ms, peak)}
    # the same, one launch per width (the three 4096-wide tensors, then the 14336-wide one)
    t_a = ActTable([act_entry(X, ts, c, sc) for X, (ts, c, sc) in zip(Xs[:3], bufs[:3])])
    t_b = ActTable([act_entry(Xs[3], *bufs[3])])

    def act_by_width():
        t_a.fouroversix()
        t_b.fouroversix()
    ms = _timed(act_by_width, stream)
    out["fouroversix_act_4096_tokens_one_layer"]["by_width"] = {
        "launches": 2, "Gelem_s": round(n_act / (ms * 1e-3) / 1e9, 2), **_roof(b_act, ms, peak)}
    # the same writing the scales in the 128x4 layout of sm_100 block-scaled GEMMs
    # (4096 tokens and hidden/16 columns: no padding, the same bytes)
    swz = [torch.empty(F.focus_scales_swizzled_bytes(X.shape[0], X.shape[1] // 16), dtype=torch.uint8, device=dev)
           for X in Xs]
    swz_tab = ActTable([act_entry(X, ts, c, sw) for X, (ts, c, _), sw in zip(Xs, bufs, swz)], swizzled=True)
    ms = _timed(swz_tab.fouroversix, stream)
    out["fouroversix_act_4096_tokens_one_layer"]["scales_128x4"] = {
        "kernel": "rows_staged_kernel<SWZ>", "Gelem_s": round(n_act / (ms * 1e-3) / 1e9, 2), **_roof(b_act, ms, peak)}
    # plain NVFP4 round to nearest per token (the target 6 alone), same inputs and bytes
    ms = _timed(act_tab.nvfp4, stream)
    out["nvfp4_act_4096_tokens_one_layer"] = {"kernel": "rows_staged_kernel<RTN>", "launches": 1, "elements": n_act,
                                               "bytes_per_elem": 2.5625,
                                               "Gelem_s": round(n_act / (ms * 1e-3) / 1e9, 2),
                                               **_roof(b_act, ms, peak)}
    del Xs, bufs, swz, act_tab, swz_tab, t_a, t_b
    # the calibration step over four micro-batches
    for e in ents:
        e.dm = torch.zeros_like(e.m)
        e.dq = torch.zeros_like(e.q)
    tab = FocusTable(ents)
    hp = hparams()
    t_b0 = _timed(lambda: tab.bwd(accumulate=False), stream)
    t_b1 = _timed(lambda: tab.bwd(accumulate=True), stream)
    cnt = [100]

    def last():
        cnt[0] += 1
        tab.step(cnt[0], hp, F.FOCUS_STEP_ACCUMULATE | F.FOCUS_STEP_WQ_UPDATED)
    t_st = _timed(last, stream)
    tot = t_b0 + 2 * t_b1 + t_st
    out["micro_batch_step_llama8b"] = {
        "micro_batches": 4, "ms": round(tot, 3), "Gelem_s": round(N * world / (tot * 1e-3) / 1e9, 2),
        "bwd_first": {"kernel": "pipe_kernel<KIND_BWD>", "bytes_per_weight": 5.5, **_roof(5.5 * N, t_b0, peak)},
        "bwd_accumulate": {"kernel": "pipe_kernel<KIND_BWD>", "bytes_per_weight": 6.25,
                           **_roof(6.25 * N, t_b1, peak)},
        "step_accumulate_wq_updated": {"kernel": "pipe_kernel<KIND_STEP, true>", "bytes_per_weight": 11.25,
                                       **_roof(11.25 * N, t_st, peak)}}
    # the same step unfused: table forward (W'), table backward, then the
    # standalone AdamW on every tensor's m and q (448 launches)
    for e in ents:
        e.dm.zero_(); e.dq.zero_()
    cnt_u = [200]

    def unfused():
        cnt_u[0] += 1
        tab.fwd()
        tab.bwd(accumulate=False)
        for e in ents:
            F.focus_adamw_step(e.m, e.dm, e.m_exp_avg, e.m_exp_avg_sq, hp.lr_m, cnt_u[0])
            F.focus_adamw_step(e.q, e.dq, e.q_exp_avg, e.q_exp_avg_sq, hp.lr_q, cnt_u[0])
    t_f = _timed(tab.fwd, stream)
    t_u = _timed(unfused, stream)
    out["unfused_step_llama8b"] = {
        "kernels": "pipe_kernel<KIND_FWD> + pipe_kernel<KIND_BWD> + adamw_kernel x448", "bytes_per_weight": 15.5,
        "ms": round(t_u, 3), "Gelem_s": round(N * world / (t_u * 1e-3) / 1e9, 2),
        "fwd": {"kernel": "pipe_kernel<KIND_FWD>", "bytes_per_weight": 4.75, **_roof(4.75 * N, t_f, peak)},
        "vs_fused_step_without_export": "the fused step moves 10.5 B per weight in one launch"}
    for e in ents:
        e.dm = e.dq = None
    del tab
    # the MXFP4 variant: one fused step per tensor (224 launches), m = 1, q = 6, zero moments,
    # then the same as one launch over a table
    mx = []
    for e in ents:
        o, i = e.W.shape
        mx.append((torch.ones((o, i // 32), device=dev), torch.full((o, i // 8), 6.0, device=dev),
                   torch.zeros((o, i // 32), device=dev), torch.zeros((o, i // 32), device=dev),
                   torch.zeros((o, i // 8), device=dev), torch.zeros((o, i // 8), device=dev)))
    cnt_mx = [0]

    def mx_step():
        cnt_mx[0] += 1
        for e, (m, q, a1, a2, b1, b2) in zip(ents, mx):
            F.focus_mx_step(e.W, e.dWq, m, q, a1, a2, b1, b2, hp, cnt_mx[0], 0, e.Wq)
    ms = _timed(mx_step, stream)
    r = {"kernel": "mx_kernel<KIND_STEP>", "launches": len(ents), "bytes_per_weight": 9.75,
         "Gelem_s": round(N * world / (ms * 1e-3) / 1e9, 2), **_roof(9.75 * N, ms, peak)}
    # the same over a table of all the tensors: one launch
    mx_tab = FocusTable([Entry(W=e.W, m=m, q=q, s2=None, dWq=e.dWq, Wq=e.Wq, m_exp_avg=a1, m_exp_avg_sq=a2,
                               q_exp_avg=b1, q_exp_avg_sq=b2) for e, (m, q, a1, a2, b1, b2) in zip(ents, mx)],
                        PURPOSE_MX)

    def mx_step_table():
        cnt_mx[0] += 1
        mx_tab.mx_step(cnt_mx[0], hp)
    ms = _timed(mx_step_table, stream)
    r["one_launch"] = {"kernel": "mx_multi_kernel<KIND_STEP>", "launches": 1,
                       "Gelem_s": round(N * world / (ms * 1e-3) / 1e9, 2), **_roof(9.75 * N, ms, peak)}
    # the same with the MXFP4 export of the updated parameters (codes + E8M0 scales)
    mx_exp = FocusTable([Entry(W=e.W, m=m, q=q, s2=None, dWq=e.dWq, Wq=e.Wq, m_exp_avg=a1, m_exp_avg_sq=a2,
                               q_exp_avg=b1, q_exp_avg_sq=b2,
                               codes=torch.empty((e.W.shape[0], e.W.shape[1] // 2), dtype=torch.uint8, device=dev),
                               scales=torch.empty((e.W.shape[0], e.W.shape[1] // 32), dtype=torch.uint8, device=dev))
                         for e, (m, q, a1, a2, b1, b2) in zip(ents, mx)], PURPOSE_MX)

    def mx_step_export():
        cnt_mx[0] += 1
        mx_exp.mx_step(cnt_mx[0], hp, F.FOCUS_STEP_PACK_UPDATED)
    ms = _timed(mx_step_export, stream)
    r["one_launch_export"] = {"kernel": "mx_multi_kernel<KIND_STEP, EXPORT>", "launches": 1, "bytes_per_weight": 10.28125,
                              "Gelem_s": round(N * world / (ms * 1e-3) / 1e9, 2), **_roof(10.28125 * N, ms, peak)}
    out["mxfp4_step_llama8b"] = r
    del mx, mx_tab, mx_exp
    # Llama-3.1-70B, generated on the device one layer at a time and stepped there:
    # s2 of the layer, then the fused step with the export of the updated parameters
    # (timed per layer), layers 0, 40 and 79

    per_layer = []
    for layer in (0, 40, 79):
        lts = synth.llama_70b_layer(layer, dev)
        lents = []
        for t in lts:
            o, i = t.W.shape
            lents.append(Entry(W=t.W, m=t.m, q=t.q, s2=torch.zeros(1, device=dev), dWq=t.dWq, Wq=torch.empty_like(t.W),
                               m_exp_avg=torch.zeros_like(t.m), m_exp_avg_sq=torch.zeros_like(t.m),
                               q_exp_avg=torch.zeros_like(t.q), q_exp_avg_sq=torch.zeros_like(t.q),
                               codes=torch.empty((o, i // 2), dtype=torch.uint8, device=dev),
                               scales=torch.empty((o, i // 16), dtype=torch.uint8, device=dev)))
        ltab = FocusTable(lents)
        ltab.s2()
        cl = [0]

        def lstep():
            cl[0] += 1
            ltab.step_s2(cl[0], hp, F.FOCUS_STEP_PACK_UPDATED)
        per_layer.append(_timed(lstep, stream))
        del ltab, lents, lts
    n70 = sum(o * i for _, (o, i) in synth.LLAMA_70B.layer_shapes())
    t70 = sum(per_layer) / len(per_layer)
    out["llama70b_per_layer_step"] = {"kernel": "pipe_kernel<KIND_STEP> + s2_from_amax_kernel", "layers": [0, 40, 79],
                                      "weights_per_layer": n70, "bytes_per_weight": 11.0625,
                                      "Gelem_s": round(n70 * world / (t70 * 1e-3) / 1e9, 2),
                                      "ms_per_layer": [round(x, 3) for x in per_layer],
                                      **_roof(11.0625 * n70, t70, peak)}
    if F.focus_get_error() != 0:
        raise SystemExit("device status after the next-row measurements is not OK")
    D.barrier()
    return out


def host_budget_bytes(world: int) -> int:
    """Pinned host memory one rank may take for the e2e leg: 60% of the memory
    the host has available, shared by the ranks."""
    try:
        with open("/proc/meminfo") as f:
            kb = next(int(l.split()[1]) for l in f if l.startswith("MemAvailable:"))
        avail = kb * 1024
    except Exception:
        avail = 64 << 30
    return int(0.6 * avail / max(world, 1))


def run_e2e(args, ents, N, world, dev):
    """The same step through the C ABI with HOST buffers: focus_step_host, the
    library's host-buffer executor, uploads every input (W, dW', m, q, moments,
    s2) from pinned host memory, steps each tensor and reads every output (W',
    m, q, moments, codes, scales, s2) back, overlapping the uploads and
    read-backs of neighbouring tensors with the step; one blocking call per
    step.  It runs on as many whole decoder layers as the host's memory holds
    for every rank (all 32 on one B200 machine: 77 GB pinned); the rate is per
    weight, so it is the same metric."""
    import torch

    from fp4_post_weight_b200 import dist as D
    from fp4_post_weight_b200 import focus as F
    from fp4_post_weight_b200.table import Entry, HostTable, hparams
    ins = ("W", "dWq", "m", "q", "m_exp_avg", "m_exp_avg_sq", "q_exp_avg", "q_exp_avg_sq", "s2")
    outs = ("Wq", "m", "q", "m_exp_avg", "m_exp_avg_sq", "q_exp_avg", "q_exp_avg_sq", "codes", "scales", "s2")
    names = set(ins) | set(outs)
    per_layer = sum(getattr(e, n).numel() * getattr(e, n).element_size() for e in ents[:7] for n in names)
    layers = max(1, min(len(ents) // 7, host_budget_bytes(world) // per_layer))
    layers = int(D.min_over_ranks(layers)) if world > 1 else layers
    ents = ents[:7 * layers]
    N = sum(e.W.numel() for e in ents)
    hosts = []
    for e in ents:
        h = {}
        for n in names:
            t = getattr(e, n)
            h[n] = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
            h[n].copy_(t)
        hosts.append(Entry(W=h["W"], m=h["m"], q=h["q"], s2=h["s2"], dWq=h["dWq"], Wq=h["Wq"],
                           m_exp_avg=h["m_exp_avg"], m_exp_avg_sq=h["m_exp_avg_sq"], q_exp_avg=h["q_exp_avg"],
                           q_exp_avg_sq=h["q_exp_avg_sq"], codes=h["codes"], scales=h["scales"]))
    htab = HostTable(hosts, dev)
    hp = hparams()
    bi = sum(getattr(h, n).numel() * getattr(h, n).element_size() for h in hosts for n in ins)
    bo = sum(getattr(h, n).numel() * getattr(h, n).element_size() for h in hosts for n in outs)
    stream = torch.cuda.current_stream(dev)
    steps = max(1, args.e2e_steps)
    htab.step(1, hp, F.FOCUS_STEP_PACK_UPDATED, stream)          # warm-up (s2 is in the host copies)
    torch.cuda.synchronize()
    D.barrier()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for k in range(steps):
        htab.step(2 + k, hp, F.FOCUS_STEP_PACK_UPDATED, stream)  # blocking: results are in host memory
    e.record(stream)
    torch.cuda.synchronize()
    ms = D.max_over_ranks(s.elapsed_time(e)) / steps
    st = F.focus_get_error()
    if st != 0:
        raise SystemExit(f"device status after the host-buffer steps: {F.focus_status_string(st)}")
    del hosts, htab
    return {"value": round(N * world / (ms * 1e-3) / 1e9, 3), "unit": "Gelem/s", "h2d_bytes_per_step": bi,
            "d2h_bytes_per_step": bo, "ms_per_step": round(ms, 2), "steps": steps, "layers": layers,
            "weights_per_rank": N, "api": "focus_step_host (one blocking call per step)"}


# ---------------------------------------------------------------------------
# the CPU oracle (baseline and reference arm)
# ---------------------------------------------------------------------------

def oracle_sample_inputs(target: int, seed: int = 0):
    """A sample of about `target` weights with the Llama-3.1-8B shapes and the
    workload's recipe, generated on the host: the same fraction of the rows of
    each of the seven projection shapes, over as many layers as needed."""
    import math

    import numpy as np

    import synth
    shapes = synth.LLAMA_8B.layer_shapes()
    per_layer = sum(o * i for _, (o, i) in shapes)
    layers = max(1, math.ceil(target / per_layer))
    frac = min(1.0, target / (layers * per_layer))
    res = []
    for l in range(layers):
        for j, (_, (o, i)) in enumerate(shapes):
            rows = max(1, int(round(o * frac)))
            t = synth.llama_8b_tensor(1000 + 7 * l + j + seed, (rows, i), "cpu")
            z = np.zeros((rows, i // 16), np.float32)
            zq = np.zeros((rows, i // 8), np.float32)
            res.append([synth.bits(t.W), synth.bits(t.dWq), t.m.numpy().copy(), t.q.numpy().copy(),
                        z.copy(), z.copy(), zq.copy(), zq.copy()])
    return res, layers, frac


def oracle_step(sample):
    """The whole path on the CPU oracle: s2, forward + straight-through backward +
    AdamW, and the NVFP4 pack of the updated parameters, tensor by tensor."""
    import oracle
    n = 0
    for W, G, m, q, a, b, c, d in sample:
        s2 = oracle.s2(W)
        oracle.step(W, G, m, q, a, b, c, d, s2, 1, want_wq=True)
        oracle.pack(W, m, q, s2)
        n += W.size
    return n


def _oracle_rate() -> float:
    """Weights per second of oracle_step on this host (a small calibration sample)."""
    sample, _, _ = oracle_sample_inputs(4_000_000, seed=77)
    t0 = time.time()
    n = oracle_step(sample)
    return n / max(time.time() - t0, 1e-6)


def _cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            return next(l.split(":", 1)[1].strip() for l in f if l.startswith("model name"))
    except Exception:
        return "unknown"


class ParitySample:
    """A row sample of the benchmark's own tensors: every `stride`-th row of each
    of them (from an offset that varies by tensor), about `target` weights.  The
    inputs (W, dW', m, q, the moments) are taken from the device before the first
    step -- they are the seeded generator's -- and the first step's outputs for
    the same rows are read back right after it, outside any timed region."""

    def __init__(self, ents, target: int):
        import math

        import torch
        N = sum(e.W.numel() for e in ents)
        self.N = N
        self.stride = max(1, math.ceil(N / max(target, 1)))
        self.rows = []
        for j, e in enumerate(ents):
            o = e.W.shape[0]
            off = j % self.stride if j % self.stride < o else 0
            self.rows.append(torch.arange(off, o, self.stride, device=e.W.device))
        self.inputs = [self._take(e, r, ("W", "dWq", "m", "q", "m_exp_avg", "m_exp_avg_sq", "q_exp_avg",
                                          "q_exp_avg_sq")) for e, r in zip(ents, self.rows)]
        self.s2_before = [float(e.s2.item()) for e in ents]
        self.outputs = None

    @staticmethod
    def _take(e, rows, names):
        import numpy as np
        import torch
        out = {}
        for n in names:
            t = getattr(e, n).index_select(0, rows)
            if t.dtype == torch.bfloat16:
                out[n] = t.view(torch.int16).cpu().numpy().view(np.uint16)
            else:
                out[n] = t.cpu().numpy()
        return out

    def read_outputs(self, ents):
        import torch
        torch.cuda.synchronize()
        self.outputs = [self._take(e, r, ("Wq", "m", "q", "m_exp_avg", "m_exp_avg_sq", "q_exp_avg",
                                          "q_exp_avg_sq", "codes", "scales")) for e, r in zip(ents, self.rows)]
        self.s2_after = [float(e.s2.item()) for e in ents]


def _near_e4m3_boundary(x):
    """x (float64 array of scaled block maxima) within 2^-20 relative of an E4M3
    rounding boundary (a midpoint between neighbouring normal values) or of a
    clamp edge."""
    import numpy as np
    mids = []
    for b in range(0x08, 0x7E):
        e, mn = (b >> 3) & 15, b & 7
        e2, mn2 = (e, mn + 1) if mn < 7 else (e + 1, 0)
        mids.append(((1 + mn / 8) * 2.0 ** (e - 7) + (1 + mn2 / 8) * 2.0 ** (e2 - 7)) / 2)
    edges = np.array(mids + [2.0 ** -6, 448.0])
    edges.sort()
    x = np.asarray(x, np.float64)
    j = np.clip(np.searchsorted(edges, x), 1, len(edges) - 1)
    d = np.minimum(np.abs(x - edges[j - 1]), np.abs(x - edges[j]))
    return d <= 2.0 ** -20 * np.abs(x)


def cpu_baseline(ents, sample: ParitySample):
    """The CPU oracle on the host cores, on the benchmark's own workload: s2 of
    every tensor over all its weights, then on the sampled rows the forward (W',
    codes, rounding bands), the straight-through backward with AdamW at step 1,
    and the NVFP4 export of the updated m and q.  Reported as weights per second
    of the whole path, a1 charged per weight of the model and the rest per
    sampled weight.  Its outputs are then compared (outside the timing) with what
    the first GPU step wrote for the same rows, which gives the parity counts
    the method's correctness bar asks for: codes (seen through W', which the step
    writes from the forward's codes and scale bytes) may differ from the oracle's
    only where y lies within 2^-20 relative of a rounding boundary, and at most
    1e-6 of the elements; s2 not at all; the updated parameters and
    moments within |gpu - ref| <= 1e-7 + 1e-5 |ref|; the export of the updated
    parameters (compared with the oracle's pack of its own update, which agrees
    within that tolerance) may differ in a scale byte only where x_b lies within
    2^-20 of an E4M3 rounding boundary and in a code only inside the band."""
    import numpy as np

    import oracle
    import synth
    oracle.build()
    threads = oracle.num_threads()
    # single-threaded: W[2048, 2048] ~ N(0, 0.02), m = 1, q = 6, forward + pack
    c1 = synth.single_2048("cpu")
    W1 = synth.bits(c1.W)
    oracle.set_threads(1)
    t0 = time.time()
    s21 = oracle.s2(W1)
    oracle.fwd(W1, c1.m.numpy(), c1.q.numpy(), s21, want_y=False)
    oracle.pack(W1, c1.m.numpy(), c1.q.numpy(), s21)
    t_c1 = time.time() - t0
    oracle.set_threads(threads)
    # s2 of every tensor over all its rows
    import torch
    t_s2 = 0.0
    s2s = []
    for e in ents:
        wb = e.W.view(torch.int16).cpu().numpy().view(np.uint16)
        t0 = time.time()
        s2s.append(oracle.s2(wb))
        t_s2 += time.time() - t0
        del wb
    # the path on the sampled rows, each tensor's outputs compared (untimed) with
    # what the first GPU step wrote for the same rows
    tol = lambda g, r: np.abs(g.astype(np.float64) - r) > 1e-7 + 1e-5 * np.abs(r.astype(np.float64))
    c = {k: 0 for k in ("elements", "blocks", "band", "exact_ties", "code_mismatch", "code_mismatch_outside_band",
                        "s2_mismatch", "state_outside_tolerance", "export_scale_mismatch",
                        "export_scale_mismatch_off_boundary", "export_code_mismatch",
                        "export_code_mismatch_outside_band", "zero_blocks", "clamp_low", "clamp_high",
                        "out_of_range")}
    n = 0
    t_path = 0.0
    for j, (inp, out, s2) in enumerate(zip(sample.inputs, sample.outputs, s2s)):
        W, G = inp["W"], inp["dWq"]
        m, q = inp["m"].copy(), inp["q"].copy()
        mo = [inp[k].copy() for k in ("m_exp_avg", "m_exp_avg_sq", "q_exp_avg", "q_exp_avg_sq")]
        t0 = time.time()
        fwd = oracle.fwd(W, m, q, s2, want_y=False)
        oracle.step(W, G, m, q, *mo, s2, 1, want_wq=False)
        exp = oracle.fwd(W, m, q, s2, want_y=False)
        t_path += time.time() - t0
        n += W.size
        c["s2_mismatch"] += int(np.float32(sample.s2_before[j]) != s2) + int(np.float32(sample.s2_after[j]) != s2)
        c["elements"] += W.size
        c["blocks"] += W.size // 16
        for k in ("band", "exact_ties", "zero_blocks", "clamp_low", "clamp_high", "out_of_range"):
            c[k] += fwd.stats[k]
        # W' is the forward's (before the update): it differs only where a code does
        wbad = out["Wq"] != fwd.Wq
        c["code_mismatch"] += int(wbad.sum())
        c["code_mismatch_outside_band"] += int((wbad & (fwd.band != 1)).sum())
        skip = wbad.reshape(W.shape[0], -1, 16).any(-1)
        for g, r, sk in zip(("m", "q", "m_exp_avg", "m_exp_avg_sq", "q_exp_avg", "q_exp_avg_sq"), [m, q] + mo,
                            (1, 2, 1, 1, 2, 2)):
            c["state_outside_tolerance"] += int((tol(out[g], r) & ~np.repeat(skip, sk, axis=1)).sum())
        # the export of the updated parameters
        sbad = out["scales"] != exp.scales
        if sbad.any():
            A = ((W.astype(np.uint32) & 0x7FFF) << 16).view(np.float32).reshape(W.shape[0], -1, 16).max(-1)
            x = (A * m) / (np.float32(6) * np.float32(s2))
            c["export_scale_mismatch_off_boundary"] += int((~_near_e4m3_boundary(x[sbad])).sum())
        c["export_scale_mismatch"] += int(sbad.sum())
        codes = np.empty(W.shape, np.uint8)
        codes[:, 0::2], codes[:, 1::2] = out["codes"] & 0xF, out["codes"] >> 4
        cbad = (codes != exp.codes) & ~np.repeat(sbad, 16, axis=1)
        c["export_code_mismatch"] += int(cbad.sum())
        c["export_code_mismatch_outside_band"] += int((cbad & (exp.band != 1)).sum())
        del fwd, exp, codes
    value = n / (t_path + t_s2 * n / sample.N) / 1e9
    cpu = {"value": round(value, 5), "unit": "Gelem/s", "cores": threads, "kind": "oracle",
           "cpu_model": _cpu_model(), "nproc": os.cpu_count(),
           "sample": f"the benchmark's own weights: s2 of all {sample.N} weights ({t_s2:.1f} s), then every "
                     f"{sample.stride}th row of each of the {len(ents)} tensors ({n} weights): forward, "
                     f"STE-bwd + AdamW and the NVFP4 export of the update ({t_path:.1f} s), on {threads} "
                     f"OpenMP threads; s2 time charged per weight of the model",
           "single_thread_c1": {"value": round(W1.size / t_c1 / 1e9, 5), "unit": "Gelem/s", "seconds": round(t_c1, 3),
                                "work": "W[2048,2048] ~ N(0,0.02), m = 1, q = 6: s2 + forward + pack, 1 thread"}}
    c["meets_bar"] = bool(c["code_mismatch_outside_band"] == 0 and c["code_mismatch"] <= 1e-6 * c["elements"]
                          and c["s2_mismatch"] == 0
                          and c["state_outside_tolerance"] == 0 and c["export_scale_mismatch_off_boundary"] == 0
                          and c["export_code_mismatch_outside_band"] == 0
                          and 16 * c["export_scale_mismatch"] + c["export_code_mismatch"] <= 1e-6 * c["elements"])
    c["what"] = ("first GPU step of this run (the benchmarked launch) on every "
                 f"{sample.stride}th row of the {len(ents)} tensors, against the oracle of the CPU baseline")
    return cpu, c


def run_reference(args, world, rank):
    """The reference arm: the CPU oracle, timed on the host cores, on the same
    metric; each step is a bounded sample of the workload (about
    --reference-seconds of CPU work)."""
    if rank != 0:
        return
    import oracle
    oracle.build()
    threads = oracle.num_threads()
    target = int(_oracle_rate() * args.reference_seconds)
    for w in range(args.warmup):
        oracle_step(oracle_sample_inputs(max(target // 8, 1), seed=w)[0])
    samples = [oracle_sample_inputs(target, seed=100 + k) for k in range(args.steps)]
    t0 = time.time()
    n = 0
    for smp, _, _ in samples:
        n += oracle_step(smp)
    dt = time.time() - t0
    value = n / dt / 1e9
    _, layers, frac = samples[0]
    desc = (f"{frac:.3f} of the rows of each Llama-3.1-8B projection shape over {layers} layer(s) per step "
            f"({n // args.steps} weights): s2 + fwd + STE-bwd + AdamW + pack on {threads} OpenMP threads")
    line = {"metric": METRIC, "value": round(value, 5), "unit": "Gelem/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * dt / args.steps, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32 forward, f64 sums", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": WORKLOAD, "sample_weights_per_step": n // args.steps},
            "cpu_baseline": {"value": round(value, 5), "unit": "Gelem/s", "cores": threads, "kind": "oracle",
                             "cpu_model": _cpu_model(), "nproc": os.cpu_count(), "sample": desc},
            "e2e": {"value": round(value, 5), "unit": "Gelem/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--layers", type=int, default=32, help="decoder layers of the 8B shapes (32 = all)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-rows", action="store_true", help="skip the next-row measurements")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--reference-seconds", type=float, default=4.0)
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("note: at least 3 warm-up steps are used", file=sys.stderr)
        args.warmup = 3
    from fp4_post_weight_b200 import dist as D
    world, rank, local = D.env()
    if args.impl == "reference":
        run_reference(args, world, rank)
    else:
        run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
