#!/usr/bin/env python
"""Benchmark of libbdscan on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--no-extra]

A step is one bdscan_allblock call on the 87M-scale all-block training layer
(batch 16 x 1024 tokens in 32-token blocks, 24 heads x headdim 64, d_state 128,
one B/C group, bf16 inputs, fp32 state and outputs): the clean forward scan
with every boundary state, the block-local reverse of both streams, and every
noisy block continued from the clean boundary state before it - all rows of
the hot path.  Inputs are seeded synthetic tensors resident in HBM; they are
larger than L2 (126 MB), so no flush is needed between steps.

Prints one JSON line (rank 0).  For N > 1 (torchrun), every rank runs an
independent replica on its own GPU (the scan has no cross-GPU exchange);
timing is the max over ranks of CUDA-event time, and `value` counts the
tokens of all ranks.  `--impl reference` times the fp64 CPU oracle instead
(rank 0 only, a bounded sample per step).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from bidirectional_mamba_state_b200 import bdscan as bd  # noqa: E402
from bidirectional_mamba_state_b200 import roofline as RL  # noqa: E402
from bidirectional_mamba_state_b200 import workload as W  # noqa: E402

METRIC = "bidir block-scan tokens/s & denoise-step µs; % of HBM / tensor-core roofline"
WORKLOAD = "87m_allblock"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one bd_tc_kernel
# launch on this workload, from one ncu capture, and the hash of the kernel
# source it was taken on: reported while the source is unchanged, null after.
TC_TRAFFIC = {"bytes": 224_046_848 + 550_898_688,
              "sources": ("bidirectional_mamba_state_b200/csrc/scan_tc.cu",
                          "bidirectional_mamba_state_b200/csrc/sm100.cuh"),
              "sha256": "07b6300c12da2206b99f0503f29757428e187de9390ef1ff5e60b5175d511aed"}


def tc_traffic():
    import hashlib
    h = hashlib.sha256()
    try:
        for f in TC_TRAFFIC["sources"]:
            with open(os.path.join(ROOT, f), "rb") as fh:
                h.update(fh.read())
    except OSError:
        return None
    return TC_TRAFFIC["bytes"] if h.hexdigest() == TC_TRAFFIC["sha256"] else None


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        p["source"] = "measured"
        return p
    except (OSError, ValueError):
        p = dict(FALLBACK_PEAKS)
        p["source"] = "fallback"
        return p


# ----------------------------------------------------------------------------- clocks
_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
            0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
            0x100: "display_clock_setting"}


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (what nvidia-smi
    reads) every `period` seconds on a background thread."""

    def __init__(self, device_index: int, period: float = 0.01):
        self.period, self.samples, self.ok = period, [], False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = int(vis.split(",")[device_index]) if vis else device_index
            self.nv, self.h = pynvml, pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that instead of clocks
            self.err = repr(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self) -> dict:
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.err}
        mask = 0
        for _, r in self.samples:
            mask |= r
        reasons = [n for b, n in _REASONS.items() if mask & b and n != "gpu_idle"]
        mhz = [m for m, _ in self.samples]
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(mhz)}


# ----------------------------------------------------------------------------- distributed
def dist_init(backend: str = "nccl"):
    """One process per GPU (torchrun environment); ``gloo`` runs the same
    plumbing on CPU."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        import datetime
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int, dev) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job tokens/s: every rank processes its own replica's tokens each
    step; the step time is the max over ranks."""
    return tokens_per_rank * world / (ms_per_step * 1e-3)


# ----------------------------------------------------------------------------- workload
def make_inputs(s: W.Shape, dev):
    seed = W.SEEDS[WORKLOAD]
    return W.make_streams(s, seed, device=dev)


def cpu_baseline(s: W.Shape, target_s: float = 15.0) -> dict:
    """The fp64 oracle, as it stands, on the host's cores over a bounded sample
    of the same workload: whole allblock passes over a subset of the batch rows
    (all heads, full length), repeated until about ``target_s`` seconds of CPU
    work have run."""
    sys.path.insert(0, ROOT)
    import oracle
    cores = len(os.sched_getaffinity(0))
    oracle.set_threads(cores)
    one = s.with_(batch=1)
    streams = W.make_streams(one, W.SEEDS[WORKLOAD], device="cpu")
    t0 = time.perf_counter()
    oracle.allblock(one.as_dict(), *streams)
    t1 = max(time.perf_counter() - t0, 1e-3)
    nb = max(1, min(s.batch, int(target_s / t1)))
    sub = s.with_(batch=nb)
    streams = W.make_streams(sub, W.SEEDS[WORKLOAD], device="cpu")
    reps, tokens = 0, 0
    t0 = time.perf_counter()
    while True:
        oracle.allblock(sub.as_dict(), *streams)
        reps += 1
        tokens += nb * s.seqlen
        dt = time.perf_counter() - t0
        if dt >= target_s or dt / reps * (reps + 1) > 2 * target_s:
            break
    return {"value": tokens / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{reps} allblock pass(es) over {nb} of {s.batch} batch rows x "
                      f"{s.seqlen} tokens x {s.nheads} heads (fp64, OpenMP over batch x head), "
                      f"{dt:.1f} s"}


def workload_config(s: W.Shape, world: int) -> dict:
    return {"workload": WORKLOAD, "op": "bdscan_allblock", "batch": s.batch,
            "seqlen": s.seqlen, "nheads": s.nheads, "headdim": s.headdim,
            "dstate": s.dstate, "ngroups": s.ngroups, "block_len": s.block_len,
            "chunk_len": s.chunk_len, "in_dtype": s.in_dtype, "out_dtype": s.out_dtype,
            "l2": "inputs larger than L2 (no flush)",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


def run_ours(args):
    rank, world, local = dist_init()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    s = W.WORKLOADS[WORKLOAD]
    cf, cr, nf, nr = make_inputs(s, dev)
    ws = bd.workspace(s, bd.BDSCAN_OP_ALLBLOCK, dev)
    K = s.nblocks
    yc = torch.empty((s.batch, s.seqlen, s.nheads, s.headdim), device=dev, dtype=torch.float32)
    yn = torch.empty_like(yc)
    st = torch.empty((s.batch, K, s.nheads, s.headdim, s.dstate), device=dev, dtype=torch.float32)
    stream = torch.cuda.current_stream(dev)

    def step():
        bd.allblock(s, cf, cr, nf, nr, y_clean=yc, y_noisy=yn, states=st, ws=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    launches_per_step = bd.kernel_launches(s, bd.BDSCAN_OP_ALLBLOCK)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world)
    ms = e0.elapsed_time(e1)
    ms = max_over_ranks(ms, world, dev)
    ms_step = ms / args.steps
    value = job_throughput(s.batch * s.seqlen, world, ms_step)

    pk = peaks()
    bytes_step = RL.allblock_bytes(s)
    achieved = bytes_step / (ms_step * 1e-3) / 1e9
    flops = RL.allblock_flops(s)
    result = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16-in/fp32-state", "data": "synthetic",
        "config": workload_config(s, world),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / pk["hbm_gbs"], "traffic": tc_traffic(),
                     "algorithmic_bytes_per_launch": bytes_step,
                     "peak_source": f"{pk['source']} hbm_gbs",
                     "frac_of_nominal_8tbs": achieved / 8000.0,
                     "tensor_tflops": flops / (ms_step * 1e-3) / 1e12,
                     "tensor_frac_of_bf16": flops / (ms_step * 1e-3) / 1e12 / pk["bf16_tflops"]},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0:
        result["e2e"] = run_e2e(s, dev, cf, cr, nf, nr, ws, min(args.steps, 10), world, ref_y_noisy=yn)
    else:
        run_e2e(s, dev, cf, cr, nf, nr, ws, min(args.steps, 10), world)
    if rank == 0 and world == 1 and not args.no_extra:
        result["extra"] = run_extra(dev, pk)
    if rank == 0 and world == 1 and not args.no_cpu:
        result["cpu_baseline"] = cpu_baseline(s)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def run_e2e(s, dev, cf, cr, nf, nr, ws, steps, world, ref_y_noisy=None):
    """Same step through the public API from pinned host buffers: every step
    copies that step's inputs host->device, runs allblock, and copies all of its
    outputs (y_clean, y_noisy, boundary states) device->host.  The batch is
    processed in chunks of rows (rows are independent sequences) so that the
    copy-in of one chunk, the scan of the previous one and the copy-out of the
    one before overlap on three streams; steps do not overlap each other."""
    host = [{k: v.to("cpu").pin_memory() for k, v in d.items()} for d in (cf, cr, nf, nr)]
    devb = [{k: torch.empty_like(v) for k, v in d.items()} for d in (cf, cr, nf, nr)]
    K = s.nblocks
    yc = torch.empty((s.batch, s.seqlen, s.nheads, s.headdim), device=dev, dtype=torch.float32)
    yn = torch.empty_like(yc)
    st = torch.empty((s.batch, K, s.nheads, s.headdim, s.dstate), device=dev, dtype=torch.float32)
    hyc, hyn = torch.empty(yc.shape, pin_memory=True), torch.empty(yn.shape, pin_memory=True)
    hst = torch.empty(st.shape, pin_memory=True)
    comp = torch.cuda.current_stream(dev)
    cin, cout = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    h2d = sum(v.numel() * v.element_size() for d in host for v in d.values())
    d2h = sum(t.numel() * t.element_size() for t in (hyc, hyn, hst))
    rows = max(1, s.batch // 8)
    chunks = [(b0, min(s.batch, b0 + rows)) for b0 in range(0, s.batch, rows)]
    subs = {n: s.with_(batch=n) for n in {b1 - b0 for b0, b1 in chunks}}
    wss = {n: bd.workspace(sub, bd.BDSCAN_OP_ALLBLOCK, dev) for n, sub in subs.items()}

    def rows_of(d, b0, b1):
        return {k: (v if k in ("A", "D") else v[b0:b1]) for k, v in d.items()}

    def step():
        start = torch.cuda.Event()
        start.record(comp)
        cin.wait_event(start)
        for b0, b1 in chunks:
            with torch.cuda.stream(cin):
                for hd, dd in zip(host, devb):
                    for k in hd:
                        if k in ("A", "D"):
                            dd[k].copy_(hd[k], non_blocking=True)
                        else:
                            dd[k][b0:b1].copy_(hd[k][b0:b1], non_blocking=True)
            ev_in = torch.cuda.Event()
            ev_in.record(cin)
            comp.wait_event(ev_in)
            sub = subs[b1 - b0]
            bd.allblock(sub, *(rows_of(d, b0, b1) for d in devb), y_clean=yc[b0:b1], y_noisy=yn[b0:b1],
                        states=st[b0:b1], ws=wss[b1 - b0], stream=comp)
            ev_done = torch.cuda.Event()
            ev_done.record(comp)
            cout.wait_event(ev_done)
            with torch.cuda.stream(cout):
                hyc[b0:b1].copy_(yc[b0:b1], non_blocking=True)
                hyn[b0:b1].copy_(yn[b0:b1], non_blocking=True)
                hst[b0:b1].copy_(st[b0:b1], non_blocking=True)
        ev_out = torch.cuda.Event()
        ev_out.record(cout)
        comp.wait_event(ev_out)

    for _ in range(2):
        step()
    torch.cuda.synchronize(dev)
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    for _ in range(steps):
        step()
    e1.record(comp)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / steps
    out = {"value": s.batch * s.seqlen * world / (ms * 1e-3), "unit": "tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms,
           "steps": steps, "chunks": len(chunks)}
    if ref_y_noisy is not None:
        # the host copy of the noisy output against the device-resident run's
        ref = ref_y_noisy.float().cpu()
        out["check_max_abs_diff_vs_device_run"] = float((hyn - ref).abs().max())
        out["check_ref_max_abs"] = float(ref.abs().max())
    return out


def _time(fn, dev, reps, warm=3):
    for _ in range(warm):
        fn()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        fn()
    e1.record()
    torch.cuda.synchronize(dev)
    return e0.elapsed_time(e1) / reps


def _profile_case(name: str, dev, pk) -> dict:
    """One small case of a kernel for ncu (inputs of one layer, a few hundred MB
    on the device): three warm-up calls, then one call.  step_3b_b64: one 3B
    layer's denoising step at batch 64; step_700m_b1: one 700M layer's batch-1
    step (the one-launch instance); prefill_700m_8k: one 700M layer's 8K
    prefill (final state only)."""
    if name == "step_700m_b1":
        s = W.WORKLOADS["700m_step"]
        f, r = W.make_streams(s, W.SEEDS["700m_step"], device=dev, streams=(W.CLEAN_FWD, W.CLEAN_REV))
        state = W.make_state(s, W.SEEDS["700m_step"], device=dev)
        y = torch.empty((s.batch, s.seqlen, s.nheads, s.headdim), device=dev)
        ws = bd.workspace(s, bd.BDSCAN_OP_BLOCK_STEP, dev)
        call = lambda: bd.block_step(s, f, r, state, y=y, ws=ws)
        b = RL.block_step_bytes(s)
    elif name == "step_3b_b64":
        s = W.WORKLOADS["3b_step_b64"]
        f, r = W.make_streams(s, W.SEEDS["3b_step_b64"], device=dev, streams=(W.CLEAN_FWD, W.CLEAN_REV))
        state = W.make_state(s, W.SEEDS["3b_step_b64"], device=dev)
        y = torch.empty((s.batch, s.seqlen, s.nheads, s.headdim), device=dev)
        ws = bd.workspace(s, bd.BDSCAN_OP_BLOCK_STEP, dev)
        call = lambda: bd.block_step(s, f, r, state, y=y, ws=ws)
        b = RL.block_step_bytes(s)
    else:
        s = W.WORKLOADS["700m_prefill_8k"]
        f, r = W.make_streams(s, W.SEEDS["700m_prefill_8k"], device=dev, streams=(W.CLEAN_FWD, W.CLEAN_REV))
        y = torch.empty((s.batch, s.seqlen, s.nheads, s.headdim), device=dev)
        fin = torch.empty((s.batch, s.nheads, s.headdim, s.dstate), device=dev)
        ws = bd.workspace(s, bd.BDSCAN_OP_PREFIX, dev)
        call = lambda: bd.prefix(s, f, r, want_states=False, y=y, final=fin, ws=ws)
        b = RL.prefix_bytes(s, block_states=False)
    ms = _time(call, dev, 1, 3)
    return {"us": ms * 1e3, "algorithmic_bytes": b, "launches_per_call": bd.kernel_launches(
        s, bd.BDSCAN_OP_PREFIX if name.startswith("prefill") else bd.BDSCAN_OP_BLOCK_STEP)}


EXTRA = {
    "block_step_700m_b1_24layers": lambda dev, pk: _step_stack(W.WORKLOADS["700m_step"], 24, dev, pk),
    "block_step_3b_b1_40layers": lambda dev, pk: _step_stack(W.WORKLOADS["3b_step_b1"], 40, dev, pk),
    "block_step_3b_b64_40layers": lambda dev, pk: _step_stack(W.WORKLOADS["3b_step_b64"], 40, dev, pk),
    "tiny_allblock": lambda dev, pk: _allblock_line("tiny", dev, pk, reps=50),
    "allblock_350m": lambda dev, pk: _allblock_line("350m_allblock", dev, pk),
    "allblock_87m_gated": lambda dev, pk: _allblock_line("87m_allblock", dev, pk, gated=True),
    "prefill_700m_8k": lambda dev, pk: _prefill_line("700m_prefill_8k", 24, dev, pk),
    "prefill_700m_32k": lambda dev, pk: _prefill_line("700m_prefill_32k", 24, dev, pk),
    "prefill_700m_64k": lambda dev, pk: _prefill_line("700m_prefill_64k", 24, dev, pk),
    "prefill_3b_256k_40layers": lambda dev, pk: _prefill_3b(dev, pk),
    "profile_step_3b_b64": lambda dev, pk: _profile_case("step_3b_b64", dev, pk),
    "profile_step_700m_b1": lambda dev, pk: _profile_case("step_700m_b1", dev, pk),
    "profile_prefill_700m_8k": lambda dev, pk: _profile_case("prefill_700m_8k", dev, pk),
    "allblock_backward_87m": lambda dev, pk: _backward(W.WORKLOADS["87m_allblock"], dev, pk),
    "conv_allblock_87m": lambda dev, pk: _conv_allblock(W.WORKLOADS["87m_allblock"], 4, dev, pk),
    "conv_block_step_700m_b1_24layers": lambda dev, pk: _step_stack(W.WORKLOADS["700m_step"], 24, dev, pk,
                                                                    conv_width=4),
    "gated_rmsnorm_87m": lambda dev, pk: _norm(W.WORKLOADS["87m_allblock"], dev, pk),
    "step_flatness_700m": lambda dev, pk: _step_flatness(dev, pk),
    "conv_block_step_norm_700m_b1_24layers": lambda dev, pk: _step_stack(W.WORKLOADS["700m_step"], 24, dev,
                                                                         pk, conv_width=4, norm=True),
}


def run_extra(dev, pk, only=None) -> dict:
    """Secondary lines: the denoising step (block_step) over a layer stack captured
    in one CUDA graph, prefill of the 700M layer, the all-block backward and the
    short convolution.  Median of 20 graph replays after 5 warm-ups (the pages'
    own methodology) for the stacks; CUDA-event means for the rest."""
    out = {}
    try:
        for name, fn in EXTRA.items():
            if (only is None and not name.startswith("profile_")) or name == only:
                out[name] = fn(dev, pk)
    except Exception as e:  # report, never hide
        out["error"] = repr(e)
    return out


def run_only(args):
    """One secondary line alone (``--only NAME``): prints {"extra": {NAME: ...}}.
    Used to profile one operation under ncu without the rest of the bench."""
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    print(json.dumps({"extra": run_extra(dev, peaks(), only=args.only)}), flush=True)


def _step_stack(s: W.Shape, layers: int, dev, pk, conv_width: int = 0, norm: bool = False,
                two_calls: bool = False) -> dict:
    """With ``conv_width``, every layer's step starts with the short convolution
    of both directions from its cached conv state: one bdscan_conv_block_step
    call (convolution and scan step in one launch where the shape allows), or
    with ``two_calls`` bdscan_conv_prefix into the scan's x, B, C and then
    bdscan_block_step; with ``norm``, the gated RMSNorm of the summed output
    follows (bf16): the selective-scan core of a Mamba layer's denoising step."""
    seed = W.SEEDS["700m_step" if s.nheads == 48 else "3b_step_b1"]
    ins = [W.make_streams(s, seed, layer, device=dev, streams=(W.CLEAN_FWD, W.CLEAN_REV))
           for layer in range(layers)]
    states = [W.make_state(s, seed, layer, device=dev) for layer in range(layers)]
    ys = [torch.empty((s.batch, s.seqlen, s.nheads, s.headdim), device=dev) for _ in range(layers)]
    wss = [bd.workspace(s, bd.BDSCAN_OP_BLOCK_STEP, dev) for _ in range(layers)]
    if conv_width:
        convs = [[W.make_conv_dir(s, conv_width, seed, layer, st, device=dev) for st in (W.CLEAN_FWD, W.CLEAN_REV)]
                 for layer in range(layers)]
        cstates = [W.make_conv_state(s, conv_width, seed, layer, device=dev) for layer in range(layers)]
        # the convolution writes straight into the scan's x, B, C
        couts = [[{k: ins[l][i][k] for k in bd.CONV_KEYS} for i in range(2)] for l in range(layers)]
        cws = [bd.workspace(s, bd.BDSCAN_OP_CONV_BLOCK_STEP, dev) for _ in range(layers)]
    if norm:
        gz = torch.Generator(device=dev).manual_seed(11)
        zs = [torch.randn(ys[0].shape, generator=gz, device=dev).to(torch.bfloat16) for _ in range(layers)]
        nws = [torch.ones(s.nheads * s.headdim, device=dev) for _ in range(layers)]
        nouts = [torch.empty(ys[0].shape, dtype=torch.bfloat16, device=dev) for _ in range(layers)]
    g_stream = torch.cuda.Stream(dev)

    def stack():
        for l in range(layers):
            if conv_width and not two_calls:
                bd.conv_block_step(s, conv_width, True, convs[l][0], convs[l][1], cstates[l], ins[l][0], ins[l][1],
                                   states[l], y=ys[l], ws=cws[l], stream=torch.cuda.current_stream(dev))
            else:
                if conv_width:
                    bd.conv_prefix(s, conv_width, True, convs[l][0], convs[l][1], cstates[l],
                                   out_fwd=couts[l][0], out_rev=couts[l][1], stream=torch.cuda.current_stream(dev))
                bd.block_step(s, ins[l][0], ins[l][1], states[l], y=ys[l], ws=wss[l],
                              stream=torch.cuda.current_stream(dev))
            if norm:
                bd.gated_rmsnorm(s, ys[l], zs[l], nws[l], 1, 1e-5, out=nouts[l],
                                 stream=torch.cuda.current_stream(dev))

    with torch.cuda.stream(g_stream):
        stack()
    torch.cuda.synchronize(dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=g_stream):
        stack()
    torch.cuda.synchronize(dev)
    times = []
    for _ in range(5):
        graph.replay()
    torch.cuda.synchronize(dev)
    for _ in range(20):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        graph.replay()
        e1.record()
        torch.cuda.synchronize(dev)
        times.append(e0.elapsed_time(e1))
    ms = statistics.median(times)
    b = RL.block_step_bytes(s) * layers
    if conv_width:
        b += RL.conv_bytes(s, conv_width, 2, state_in=True) * layers
    if norm:
        b += RL.norm_bytes(s, gated=True) * layers
    del graph
    out = {"us_per_step": ms * 1e3, "tokens_per_s": s.batch * s.seqlen / (ms * 1e-3),
           "algorithmic_bytes": b, "hbm_frac": b / (ms * 1e-3) / 1e9 / pk["hbm_gbs"],
           "layers": layers, "batch": s.batch, "graph": True}
    if not conv_width and not norm:
        import oracle
        hf, hr, hst = _host(ins[0][0]), _host(ins[0][1]), states[0].to("cpu")
        out["cpu_baseline"] = _oracle_rate(
            lambda: oracle.block_step(s.as_dict(), hf, hr, hst), s.batch * s.seqlen * s.nheads,
            "token-heads/s", f"oracle block_step of layer 0 (all {s.batch} x {s.nheads} sequences, "
            f"forward from the cached state + block-local reverse)", target_s=1.0)
    if conv_width:
        out["conv_width"] = conv_width
    if norm:
        out["gated_rmsnorm"] = True
    return out


def _norm(s: W.Shape, dev, pk) -> dict:
    """Gated RMSNorm (one group over all H*P channels, bf16 result) of the 87M
    all-block layer's fp32 noisy output with a bf16 gate."""
    cf, cr, nf, nr = W.make_streams(s, W.SEEDS[WORKLOAD], device=dev)
    _, yn, _ = bd.allblock(s, cf, cr, nf, nr, want_clean=False)
    g = torch.Generator(device=dev).manual_seed(9)
    z = torch.randn(yn.shape, generator=g, device=dev).to(torch.bfloat16)
    w = torch.ones(s.nheads * s.headdim, device=dev)
    out = bd.gated_rmsnorm(s, yn, z, w, 1, 1e-5)
    ms = _time(lambda: bd.gated_rmsnorm(s, yn, z, w, 1, 1e-5, out=out), dev, 20)
    b = RL.norm_bytes(s, gated=True)
    achieved = b / (ms * 1e-3) / 1e9
    return {"us_per_call": ms * 1e3, "tokens_per_s": s.batch * s.seqlen / (ms * 1e-3),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / pk["hbm_gbs"], "algorithmic_bytes": b},
            "cpu_baseline": _guarded(_norm_oracle_rate, s, yn, z, w)}


def _guarded(fn, *args) -> dict:
    """A secondary line's oracle rate; a failure there is reported in the line
    instead of ending the remaining lines."""
    try:
        return fn(*args)
    except Exception as e:  # report, never hide
        return {"kind": "oracle", "error": repr(e)}


def _norm_oracle_rate(s: W.Shape, yn, z, w) -> dict:
    """The oracle's gated RMSNorm on the first batch row, timed on the host cores."""
    import oracle
    hy, hz, hw = yn[:1].to("cpu"), z[:1].to("cpu"), w.to("cpu")
    return _oracle_rate(lambda: oracle.gated_rmsnorm(hy, hz, hw, 1, 1e-5), s.seqlen, "tokens/s",
                        f"oracle gated_rmsnorm on 1 of {s.batch} batch rows ({s.seqlen} tokens x "
                        f"{s.nheads * s.headdim} channels)")


def _conv_allblock(s: W.Shape, width: int, dev, pk) -> dict:
    """Short convolution (+SiLU) of the all-block layer's four directions, the
    noisy blocks continuing from the clean rows before them."""
    dirs = [W.make_conv_dir(s, width, W.SEEDS[WORKLOAD], stream=i, device=dev) for i in range(4)]
    outs = bd.conv_allblock(s, width, True, *dirs)
    ms = _time(lambda: bd.conv_allblock(s, width, True, *dirs, outs=outs), dev, 20)
    b = RL.conv_bytes(s, width, 4)
    achieved = b / (ms * 1e-3) / 1e9
    return {"us_per_call": ms * 1e3, "tokens_per_s": s.batch * s.seqlen / (ms * 1e-3), "width": width,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / pk["hbm_gbs"], "algorithmic_bytes": b,
                         "algorithmic_flops": RL.conv_flops(s, width, 4)},
            "cpu_baseline": _guarded(_conv_oracle_rate, s, width, dirs)}


def _conv_oracle_rate(s: W.Shape, width: int, dirs) -> dict:
    """The oracle's all-block convolution (four directions) on the first batch
    row, timed on the host cores."""
    import oracle
    one = s.with_(batch=1)
    hd = [_host({k: (v if k in ("weight", "bias") else v[:1]) for k, v in d.items()}) for d in dirs]
    return _oracle_rate(lambda: oracle.conv_allblock(one.as_dict(), width, True, *hd), one.seqlen, "tokens/s",
                        f"oracle conv_allblock (width {width}, four directions) on 1 of {s.batch} batch rows, "
                        f"all {s.seqlen} tokens")


def _backward(s: W.Shape, dev, pk) -> dict:
    """Backward of the all-block layer (gradients of every input of the four
    directions and of h0), from the forward's boundary states."""
    cf, cr, nf, nr = W.make_streams(s, W.SEEDS[WORKLOAD], device=dev)
    _, yn, st = bd.allblock(s, cf, cr, nf, nr)
    g = torch.Generator(device=dev).manual_seed(7)
    dyn = torch.randn(yn.shape, generator=g, device=dev)
    dyc = torch.randn(yn.shape, generator=g, device=dev)
    ws = bd.workspace(s, bd.BDSCAN_OP_ALLBLOCK_BACKWARD, dev)
    grads, dh0 = bd.allblock_backward(s, cf, cr, nf, nr, st, dyn, dy_clean=dyc, ws=ws)
    ms = _time(lambda: bd.allblock_backward(s, cf, cr, nf, nr, st, dyn, dy_clean=dyc, grads=grads, ws=ws),
               dev, 5)
    flops = RL.allblock_backward_flops(s)
    bytes_ = RL.allblock_backward_bytes(s)
    # fp32 CUDA-core peak: 148 SMs x 128 FMA lanes x 2 flops x the max SM clock
    alu_peak = 148 * 128 * 2 * pk["sm_max_mhz"] * 1e6 / 1e12
    tf = flops / (ms * 1e-3) / 1e12
    return {"us_per_call": ms * 1e3, "tokens_per_s": s.batch * s.seqlen / (ms * 1e-3),
            "kernel": "generic CUDA-core backward (per-block adjoint in shared memory)",
            "roofline": {"bound": "alu", "achieved": tf, "peak": alu_peak, "unit": "TFLOP/s",
                         "frac": tf / alu_peak, "algorithmic_flops": flops,
                         "algorithmic_bytes": bytes_,
                         "hbm_frac": bytes_ / (ms * 1e-3) / 1e9 / pk["hbm_gbs"]},
            "cpu_baseline": _guarded(_backward_oracle_rate, s, (cf, cr, nf, nr), dyn, dyc)}


def _backward_oracle_rate(s: W.Shape, dirs, dyn, dyc) -> dict:
    """The oracle's backward on the first batch row of the same inputs and output
    gradients (all heads, all tokens, four directions), timed on the host cores."""
    import oracle
    one = s.with_(batch=1)
    hs = [_host({k: (v if k in ("A", "D") else v[:1]) for k, v in d.items()}) for d in dirs]
    hdyn, hdyc = dyn[:1].to("cpu"), dyc[:1].to("cpu")
    return _oracle_rate(lambda: oracle.allblock_backward(one.as_dict(), *hs, dy_clean=hdyc, dy_noisy=hdyn),
                        one.seqlen, "tokens/s",
                        f"oracle allblock_backward on 1 of {s.batch} batch rows, all {s.nheads} heads, "
                        f"all {s.seqlen} tokens, loss on y_clean and y_noisy")


def _oracle_rate(call, units: float, unit: str, sample: str, target_s: float = 3.0) -> dict:
    """The fp64 oracle, as it stands, timed on the host's cores: ``call`` is run
    until about ``target_s`` seconds have passed; ``units`` of work per run."""
    import oracle
    cores = len(os.sched_getaffinity(0))
    oracle.set_threads(cores)
    reps = 0
    t0 = time.perf_counter()
    while True:
        call()
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= target_s or dt / reps * (reps + 1) > 2 * target_s:
            break
    return {"value": units * reps / dt, "unit": unit, "cores": cores, "kind": "oracle",
            "sample": f"{sample}; {reps} run(s) in {dt:.1f} s"}


def _host(d: dict) -> dict:
    return {k: v.to("cpu") for k, v in d.items()}


def _heads_host(d: dict, hs: list) -> dict:
    """Host copy of one direction's inputs restricted to the heads ``hs`` (one
    B/C group: B and C are shared by all heads)."""
    return {k: (v[hs] if k in ("A", "D") else v if k in ("B", "C") else v[:, :, hs]).to("cpu")
            for k, v in d.items()}


def _allblock_line(name: str, dev, pk, reps: int = 10, gated: bool = False) -> dict:
    """One bdscan_allblock call on a whole workload (CUDA events), with the
    oracle's rate on one batch row (all heads, full length); gated: every
    direction with its gate z (y_dir silu(z_dir) before the sum, fused in the
    scan kernel's epilogue)."""
    import oracle
    s = W.WORKLOADS[name]
    cf, cr, nf, nr = W.make_streams(s, W.SEEDS[name], device=dev, gated=gated)
    yc, yn, st = bd.allblock(s, cf, cr, nf, nr)
    ws = bd.workspace(s, bd.BDSCAN_OP_ALLBLOCK, dev)
    ms = _time(lambda: bd.allblock(s, cf, cr, nf, nr, y_clean=yc, y_noisy=yn, states=st, ws=ws), dev, reps)
    b = RL.allblock_bytes(s, gated=gated)
    del yc, yn, st
    one = s.with_(batch=1)
    hs = [_host({k: (v if k in ("A", "D") else v[:1]) for k, v in d.items()}) for d in (cf, cr, nf, nr)]
    cpu = _oracle_rate(lambda: oracle.allblock(one.as_dict(), *hs), one.seqlen, "tokens/s",
                       f"oracle allblock on 1 of {s.batch} batch rows, all {s.nheads} heads, "
                       f"all {s.seqlen} tokens")
    return {"us_per_call": ms * 1e3, "tokens_per_s": s.batch * s.seqlen / (ms * 1e-3),
            "roofline": {"bound": "hbm", "achieved": b / (ms * 1e-3) / 1e9, "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": b / (ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                         "algorithmic_bytes": b},
            "cpu_baseline": cpu}


def _prefill_line(name: str, layers: int, dev, pk, oracle_heads=None) -> dict:
    """Prefill (bdscan_prefix, final state only, block-local reverse) of one
    layer and of a stack of ``layers`` layers with independent weights, each
    layer's inputs resident (the stack's calls back to back, CUDA events);
    with the oracle's rate per token-head on one layer."""
    import oracle
    s = W.WORKLOADS[name]
    seed = W.SEEDS[name]
    ins = [W.make_streams(s, seed, l, device=dev, streams=(W.CLEAN_FWD, W.CLEAN_REV)) for l in range(layers)]
    y = torch.empty((s.batch, s.seqlen, s.nheads, s.headdim), device=dev)
    fins = [torch.empty((s.batch, s.nheads, s.headdim, s.dstate), device=dev) for _ in range(layers)]
    ws = bd.workspace(s, bd.BDSCAN_OP_PREFIX, dev)
    one = lambda l: bd.prefix(s, ins[l][0], ins[l][1], want_states=False, y=y, final=fins[l], ws=ws)
    ms1 = _time(lambda: one(0), dev, 20, 5)

    def stack():
        for l in range(layers):
            one(l)
    ms = _time(stack, dev, 3, 1)
    b = RL.prefix_bytes(s, block_states=False)
    out = {"us_per_layer": ms1 * 1e3, "tokens_per_s_per_layer": s.batch * s.seqlen / (ms1 * 1e-3),
           "algorithmic_bytes_per_layer": b, "hbm_frac": b / (ms1 * 1e-3) / 1e9 / pk["hbm_gbs"],
           f"ms_{layers}_layers": ms, f"hbm_frac_{layers}_layers": b * layers / (ms * 1e-3) / 1e9 / pk["hbm_gbs"],
           "layers": layers}
    hs = list(range(s.nheads)) if oracle_heads is None else list(range(oracle_heads))
    f, r = _heads_host(ins[0][0], hs), _heads_host(ins[0][1], hs)
    del ins
    sub = s.with_(nheads=len(hs))
    out["cpu_baseline"] = _oracle_rate(
        lambda: oracle.prefix(sub.as_dict(), f, r, want_states=False), s.batch * s.seqlen * len(hs),
        "token-heads/s", f"oracle prefix of layer 0, {len(hs)} of {s.nheads} heads, all {s.seqlen} tokens, "
        f"forward + block-local reverse")
    return out


def _prefill_3b(dev, pk, layers: int = 40) -> dict:
    """The 3B layer's 262,144-token prefill (final state only): ``layers`` layers
    with independent weights, each layer's inputs drawn just before its call
    (untimed; 40 layers' inputs would not fit the device at once), every call
    timed with CUDA events; per layer (median) and the 40-layer sum."""
    import oracle
    s = W.WORKLOADS["3b_prefill_256k"]
    seed = W.SEEDS["3b_prefill_256k"]
    y = torch.empty((s.batch, s.seqlen, s.nheads, s.headdim), device=dev)
    fin = torch.empty((s.batch, s.nheads, s.headdim, s.dstate), device=dev)
    ws = bd.workspace(s, bd.BDSCAN_OP_PREFIX, dev)
    times = []
    for l in range(layers):
        f, r = W.make_streams(s, seed, l, device=dev, streams=(W.CLEAN_FWD, W.CLEAN_REV))
        if l == 0:
            bd.prefix(s, f, r, want_states=False, y=y, final=fin, ws=ws)
        times.append(_time(lambda: bd.prefix(s, f, r, want_states=False, y=y, final=fin, ws=ws), dev, 1, 0))
        if l == 0:
            hf, hr = _heads_host(f, list(range(16))), _heads_host(r, list(range(16)))
        del f, r
    ms = statistics.median(times)
    b = RL.prefix_bytes(s, block_states=False)
    sub = s.with_(nheads=16)
    cpu = _oracle_rate(lambda: oracle.prefix(sub.as_dict(), hf, hr, want_states=False),
                       s.seqlen * 16, "token-heads/s",
                       "oracle prefix of layer 0, 16 of 80 heads, all 262144 tokens, forward + block-local "
                       "reverse", target_s=1.0)
    return {"us_per_layer_median": ms * 1e3, "ms_40_layers_sum": sum(times),
            "tokens_per_s_per_layer": s.seqlen / (ms * 1e-3), "algorithmic_bytes_per_layer": b,
            "hbm_frac": b / (ms * 1e-3) / 1e9 / pk["hbm_gbs"], "layers": layers,
            "timing": "each layer's call timed alone (CUDA events), inputs drawn before it",
            "cpu_baseline": cpu}


def _step_flatness(dev, pk) -> dict:
    """Per-step cost against context length: prefill one layer (final state
    only) at several lengths, then time a denoising step (block_step over the
    active 32-token block) from each cached state.  The step reads only the
    fixed-size state, so its time must not grow with the context: 700M at
    8K/32K/64K, 3B at 8K/64K/256K."""
    out = {}
    for model, step_name, lens in (("700m", "700m_step", (8192, 32768, 65536)),
                                   ("3b", "3b_step_b1", (8192, 65536, 262144))):
        st = W.WORKLOADS[step_name]
        a, r = W.make_streams(st, 7, device=dev, streams=(W.CLEAN_FWD, W.CLEAN_REV))
        ws = bd.workspace(st, bd.BDSCAN_OP_BLOCK_STEP, dev)
        y = torch.empty((st.batch, st.seqlen, st.nheads, st.headdim), device=dev)
        row = {}
        for L in lens:
            s = st.with_(seqlen=L, chunk_len=128)
            f, rr = W.make_streams(s, W.SEEDS[step_name], device=dev, streams=(W.CLEAN_FWD, W.CLEAN_REV))
            _, _, fin = bd.prefix(s, f, rr, want_states=False)
            del f, rr
            ms = _time(lambda: bd.block_step(st, a, r, fin, y=y, ws=ws), dev, 50, 5)
            row[f"us_per_step_after_{L // 1024}k"] = ms * 1e3
        v = list(row.values())
        row["max_over_min"] = max(v) / min(v)
        out[model] = row
    out["layers"] = 1
    return out


def run_reference(args):
    """The fp64 CPU oracle as the reference arm: rank 0 only, each step the
    oracle's allblock on a bounded sample (one batch row, all heads, full
    length) of the same workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    s = W.WORKLOADS[WORKLOAD]
    cores = len(os.sched_getaffinity(0))
    oracle.set_threads(cores)
    one = s.with_(batch=1)
    streams = W.make_streams(one, W.SEEDS[WORKLOAD], device="cpu")
    for _ in range(args.warmup):
        oracle.allblock(one.as_dict(), *streams)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.allblock(one.as_dict(), *streams)
    dt = (time.perf_counter() - t0) / args.steps
    value = one.batch * one.seqlen / dt
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(s, args.gpus),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"each step: oracle allblock on 1 of {s.batch} batch rows, "
                                       f"all {s.nheads} heads, all {s.seqlen} tokens"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extra", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--only", choices=sorted(EXTRA), help="run one secondary line alone")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.only:
        run_only(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
