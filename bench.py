"""Benchmark of the rf_v2 block-sparse attention call on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload minimax] [--impl reference]
                    [--sparsity S] [--dtype bf16|f16] [--precision native|fp8] [--mode replicas|ulysses]

One step = one full call (token reorder + pooling, block scores + top-k mask,
block-sparse attention with the inverse reorder fused) on one batch of seeded
synthetic bf16 Q/K/V resident in HBM.  The metric is the effective
throughput over the kept blocks: FLOPs = 4 * D * sum over query rows of the
number of keys the row attends to (dense prefix and first-frame rows count
all S keys), divided by the device time of the step.  Under torchrun each rank
runs its own replica (the call shards by independent problems; no collective
on the data path), so the aggregate is the sum over ranks divided by the
slowest rank's time.

``--mode ulysses`` runs the call sequence-parallel instead (vllm-omni
"RainFusion Attention", "Requirements and compatibility"): each rank holds a
sequence shard [B, S/P, N, D] of q, k and v; one all-to-all turns them into
head shards [B, S, N/P, D], the library's call runs on the local heads, and a
second all-to-all returns the output's sequence shard.  The exchanges are
NCCL collectives (a process group of one rank without torchrun); the work of
the whole problem is fixed as P grows ("scaling": "strong"), and the line
reports the two exchanges and the call separately.

``--impl reference`` times the plain CPU oracle on the host cores instead, on
a bounded sample of the same workload.

``--dtype f16`` runs fp16 inputs and output; ``--precision fp8`` runs the
attention's two products on e4m3 operands (quantised in the first stage) and
takes the fp8 tensor peak as twice the measured bf16 one (the nominal
ratio).
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "rf_v2 sparse-attn ms/call & effective TFLOPS (kept blocks) at MiniMax-H3 shape"
UNIT = "TFLOP/s"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def _stages(w, plan, prec, ms_prepare, ms_attention, k3_tflops, hbm_gbs, ms_k1=None):
    """Per-stage times with the HBM-bound stages' algorithmic bytes: K1 reads q, k, v in the caller's layout and
    writes the internal copies (fp8: e4m3 codes and one fp32 scale per 128-row tile) plus the fp32 block means
    of q and k, K2 reads the block means and writes the mask, kept counts and margins.  ``ms_k1`` (K1 alone,
    from the library's stage event) splits the prepare stage into K1 and the kernel after it."""
    heads = w.B * w.N
    row = 128 * 2                                          # one token's head vector, bytes
    pooled = 2 * plan.nb * 128 * 4                         # q and k block means, bytes per head
    words = (plan.nb + 31) // 32
    written = 3 * plan.S_int * 128 + 3 * plan.n_tiles * 4 if prec == "fp8" else 3 * plan.S_int * row
    k1 = heads * (3 * w.S * row + written + pooled)
    k2 = heads * (pooled + plan.nb * (words * 4 + 8))
    moved = k1 + k2
    gbs = moved / (ms_prepare * 1e-3) / 1e9
    k1_name = "K1 reorder + block means" + (" + e4m3 codes" if prec == "fp8" else "")
    out = {"prepare": {"kernels": k1_name + ", K2 block scores + top-k",
                       "ms": ms_prepare, "algorithmic_bytes": moved, "gbs": gbs, "frac_of_hbm": gbs / hbm_gbs}}
    if ms_k1 is not None and 0 < ms_k1 < ms_prepare:
        g1 = k1 / (ms_k1 * 1e-3) / 1e9
        rest = ms_prepare - ms_k1
        g2 = k2 / (rest * 1e-3) / 1e9
        out["permute_pool"] = {"kernels": k1_name, "ms": ms_k1, "algorithmic_bytes": k1,
                               "gbs": g1, "frac_of_hbm": g1 / hbm_gbs}
        out["after_permute_pool"] = {"kernels": "K2", "ms": rest,
                                     "algorithmic_bytes": k2, "gbs": g2, "frac_of_hbm": g2 / hbm_gbs}
    out["attention"] = {"kernels": "K3", "ms": ms_attention, "tflops": k3_tflops}
    return out


def _kv_stream(flops, prec, ms_attention, sm_mhz, sms):
    """K and V brought from L2 into the SMs by K3: each (query row, kept key) pair costs 4 bytes (a 128 x 128
    tile pair of 64 KB serves 128 x 128 pairs; e4m3: 2 bytes) and 4 D = 512 FLOPs.  Per SM cycle at the median
    SM clock sampled in the timed region (two TMA threads per SM stream about 74 bytes per SM cycle from L2)."""
    pairs = flops / (4 * 128)
    nbytes = pairs * (2 if prec == "fp8" else 4)
    out = {"bytes": nbytes, "tbs": nbytes / (ms_attention * 1e-3) / 1e12}
    if sm_mhz:
        out["bytes_per_sm_cycle"] = nbytes / (ms_attention * 1e-3 * sms * sm_mhz * 1e6)
    return out


# The attention kernels' sources, hashed together to tie a traffic capture to the code it measured.
K3_SOURCES = ("rf_attn_common.cuh", "rf_attn_chain.cu", "rf_attn.cu")


# Nominal dense tensor peaks of B200 (TFLOP/s), for context beside the measured ones.
NOMINAL_TFLOPS = {"bf16": 2250.0, "fp8": 4500.0}


def _roofline(k3_tflops: float, prec: str, dtype: str, peaks: dict, src: str, traffic):
    """K3 against the measured sustained matmul peak (the kernel runs back to
    back for the whole timed region, under the power cap), with the measured
    burst and the nominal dense peaks beside it.  fp8 takes twice the bf16
    figures (the nominal fp8 / bf16 ratio)."""
    mult = 2.0 if prec == "fp8" else 1.0
    sustained = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) * mult
    burst = peaks["bf16_tflops"] * mult
    nominal = NOMINAL_TFLOPS["fp8" if prec == "fp8" else "bf16"]
    note = f"{src} bf16_tflops_sustained"
    if prec == "fp8":
        note += " x 2 (nominal fp8 / bf16 ratio)"
    elif dtype == "f16":
        note += " (fp16 and bf16 have the same nominal peak)"
    return {"kernel": "rf attention (K3)", "bound": "tensor", "achieved": k3_tflops, "peak": sustained,
            "unit": "TFLOP/s", "frac": k3_tflops / sustained, "traffic": traffic, "peak_source": note,
            "frac_of_measured_burst": k3_tflops / burst, "measured_burst_peak": burst,
            "frac_of_nominal": k3_tflops / nominal, "nominal_peak": nominal}


def _mask_stats(stats: dict, plan) -> dict:
    """The mask of the timed call, from the library's statistics: kept key
    blocks, the realised density of (query, key) pairs, and the selections
    that sat on a near-tie (k-th and (k+1)-th block scores within 1e-5,
    relative), which the bit-exact mask check excuses."""
    return {"k": plan.k, "nb": plan.nb, "ff": plan.ff, "kept_blocks": stats["kept_blocks"],
            "query_blocks": stats["query_blocks"],
            "kept_per_query_block": stats["kept_blocks"] / max(stats["query_blocks"], 1),
            "density": stats["density"], "near_ties": stats["near_ties"],
            "near_tie_rule": "k-th and (k+1)-th block scores within 1e-5 (relative)",
            "second_pass_tiles": stats["redo_tiles"]}


def _k3_traffic(heads: int, label: str = "k3"):
    """DRAM bytes per attention launch from the committed ncu summary (label
    k3: 16-bit operands, k3_fp8: e4m3 operands), scaled to ``heads``; None
    when the kernel source changed since the capture."""
    import hashlib
    csrc = os.path.join(ROOT, "block_sparse_video_rf_b200", "csrc")
    path = os.path.join(ROOT, "profiles", "k3_traffic.txt")
    if not os.path.exists(path):
        return None
    h = hashlib.sha256()
    for name in K3_SOURCES:
        h.update(open(os.path.join(csrc, name), "rb").read())
    digest = h.hexdigest()[:16]
    for line in open(path):
        parts = line.split()
        if len(parts) >= 3 and not line.startswith("#") and parts[0] == label and parts[1] == digest:
            return int(parts[2]) * heads / 56.0
    return None


def _describe(w, dtype="bf16", precision="native") -> str:
    t, h, wd = w.latent
    prec = "" if precision == "native" else f", {precision} e4m3 attention operands"
    return (f"{w.name}: B={w.B}, {w.N} heads, D={w.D}, txt_len={w.txt_len}, latent ({t},{h},{wd}) -> S={w.S}, "
            f"sparsity {w.sparsity}, {w.layout}, {dtype} synthetic ({w.kind}){prec}")


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock, power and throttle reasons sampled every 20 ms while the
    timed region runs (NVML in a thread of this process; nvidia-smi at 200 ms
    where NVML cannot be loaded).  Only samples taken inside the region count,
    so the median is the clock under load."""
    PERIOD_S = 0.02
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.device_index = device_index
        self.samples = []           # (sm_mhz, max_mhz, watts, reason names)
        self.source = None
        self._stop = None
        self._thread = None
        self._proc = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            pr = torch.cuda.get_device_properties(self.device_index)
            bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.device_index)

    def __enter__(self):
        import threading
        try:
            nv, h = self._nvml_handle()
        except Exception:
            nv = None
        if nv is not None:
            bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
            self._stop = threading.Event()

            def run():
                while not self._stop.is_set():
                    try:
                        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
                        watts = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                        r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.samples.append((float(sm), float(mx), watts, [n for n, b in bits.items() if r & b]))
                    except Exception:
                        pass
                    self._stop.wait(self.PERIOD_S)

            self.source = "nvml"
            self._thread = threading.Thread(target=run, daemon=True)
            self._thread.start()
            return self
        try:
            self._proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.device_index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi"
        except OSError:
            self._proc = None
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=2)
        if self._proc is not None:
            self._proc.terminate()
            try:
                out, _ = self._proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self._proc.kill()
                out, _ = self._proc.communicate()
            for line in out.splitlines():
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm, mx, watts = float(parts[1]), float(parts[2]), float(parts[3])
                except ValueError:
                    continue
                self.samples.append((sm, mx, watts, [n for n, v in zip(self.NAMES, parts[5:9])
                                                     if v.lower().startswith("active")]))

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        reasons = sorted({n for smp in self.samples for n in smp[3]})
        return {"sm_mhz": statistics.median(smp[0] for smp in self.samples), "sm_max_mhz": self.samples[-1][1],
                "reasons": reasons, "samples": len(self.samples),
                "power_w_median": round(statistics.median(smp[2] for smp in self.samples), 1),
                "source": self.source}


# ---------------------------------------------------------------- multi-rank aggregation
def reduce_max(values, dist=None, device="cpu"):
    """Element-wise max over ranks (the slowest rank decides every time)."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def aggregate(flops_per_rank_step: float, world: int, ms_per_step_max: float) -> float:
    """Whole-job throughput in TFLOP/s: every rank runs the same replica."""
    return world * flops_per_rank_step / (ms_per_step_max * 1e-3) / 1e12


# ---------------------------------------------------------------- CPU oracle sample
def oracle_sample(q, k, v, w, budget_s: float = 15.0, heads_total=None):
    """Times the CPU oracle on head 0: its own mask, then attention for evenly
    spaced query tiles until about ``budget_s`` of CPU work.  Returns
    (TFLOP/s, threads, description)."""
    import oracle
    from threadpoolctl import threadpool_info
    qh = q[0, :, 0].float().cpu().numpy() if w.layout == "BSND" else q[0, 0].float().cpu().numpy()
    kh = k[0, :, 0].float().cpu().numpy() if w.layout == "BSND" else k[0, 0].float().cpu().numpy()
    vh = v[0, :, 0].float().cpu().numpy() if w.layout == "BSND" else v[0, 0].float().cpu().numpy()
    t0 = time.perf_counter()
    g = oracle.geometry(w.S, w.txt_len, *w.latent)
    mask, _ = oracle.build_mask(qh[None, None], kh[None, None], g, float(np.float32(w.sparsity)))
    mask = mask[0, 0]
    # query tiles in the oracle's own terms: prefix rows in chunks of 128, then sparse blocks
    tiles = [("prefix", g.prefix[i:i + 128]) for i in range(0, len(g.prefix), 128)]
    tiles += [("block", g.blocks[i]) for i in range(g.nb)] if not g.dense else []
    order = list(range(0, len(tiles), 7)) + [i for i in range(len(tiles)) if i % 7]
    flops, done = 0.0, 0
    scale = w.D ** -0.5
    for idx in order:
        kind, rows = tiles[idx]
        out = oracle.attention_rows(qh, kh, vh, g, None if g.dense else mask, scale, rows=rows)
        blk = None if kind == "prefix" else idx - (len(tiles) - g.nb)
        nkeys = len(oracle.key_set(g, mask, blk)) if not g.dense else g.S
        flops += 4.0 * w.D * len(rows) * nkeys
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    threads = max([p.get("num_threads", 1) for p in threadpool_info()] + [1])
    desc = (f"head 0 of {heads_total or w.N}: mask of all {g.nb} blocks + attention of {done} of {len(tiles)} query tiles "
            f"(every 7th first), {flops / 1e12:.3f} TFLOP in {dt:.1f} s")
    return flops / dt / 1e12, threads, desc


# ---------------------------------------------------------------- reference arm
def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from block_sparse_video_rf_b200 import synth
    q, k, v = synth.make_inputs(synth.workload(w.name, N=1, seed=w.seed), device="cpu")
    vals, walls = [], []
    desc = threads = None
    w1 = synth.workload(w.name, N=1, **({} if args.sparsity is None else {"sparsity": args.sparsity}))
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        val, threads, desc = oracle_sample(q, k, v, w1, budget_s=args.ref_budget, heads_total=w.N)
        if i >= args.warmup:
            vals.append(val)
            walls.append(time.perf_counter() - t0)
    value = statistics.mean(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(walls),
        "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": _describe(w), "sample": "one head per step, bounded CPU time"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- sequence-parallel arm
def shard_rows(x, rank: int, world: int):
    """This rank's sequence shard of a BSND tensor: tokens [r S/P, (r + 1) S/P)."""
    S = x.shape[1]
    if S % world:
        raise ValueError(f"sequence length {S} is not a multiple of the {world} ranks")
    Sl = S // world
    return x[:, rank * Sl:(rank + 1) * Sl].contiguous()


def _free_port() -> int:
    import socket
    sk = socket.socket()
    sk.bind(("127.0.0.1", 0))
    port = sk.getsockname()[1]
    sk.close()
    return port


def run_ulysses(args, w):
    """--mode ulysses: the call on sequence shards, Ulysses all-to-all to head
    shards and back around the library's call on N / P heads (see the module
    docstring).  Timed per step with CUDA events: the first exchange, the
    call (and its attention stage alone), the second exchange; the slowest
    rank decides each."""
    import datetime
    import torch.distributed as dist
    from block_sparse_video_rf_b200 import rfsa, synth, ulysses
    if w.layout != "BSND":
        raise SystemExit("--mode ulysses takes BSND workloads")
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("RANK", "0")
    os.environ.setdefault("WORLD_SIZE", "1")
    os.environ.setdefault("LOCAL_RANK", "0")
    if "MASTER_PORT" not in os.environ:
        os.environ["MASTER_PORT"] = str(_free_port())
    world, rank, local = int(os.environ["WORLD_SIZE"]), int(os.environ["RANK"]), int(os.environ["LOCAL_RANK"])
    if w.S % world or w.N % world:
        raise SystemExit(f"S = {w.S} and N = {w.N} must be multiples of the {world} ranks")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    try:
        return _ulysses_timed(args, w, dist, rfsa, synth, ulysses, world, rank, local, dev)
    finally:
        dist.destroy_process_group()


def _ulysses_timed(args, w, dist, rfsa, synth, ulysses, world, rank, local, dev):
    prec = args.precision
    tdtype = torch.float16 if args.dtype == "f16" else torch.bfloat16
    sp = np.float32(w.sparsity)
    Nl = w.N // world
    # every rank draws the whole seeded problem and keeps its sequence shard
    q, k, v = synth.make_inputs(w, device=dev, dtype=tdtype)
    q_sh, k_sh, v_sh = (shard_rows(t, rank, world) for t in (q, k, v))
    del q, k, v
    torch.cuda.empty_cache()
    ws = rfsa.alloc_workspace(w.B, w.S, Nl, w.D, w.txt_len, w.latent, device=dev, precision=prec)
    plan = rfsa.rf_plan(w.S, w.txt_len, w.latent, sp)
    views = rfsa.workspace_views(ws, w.B, Nl, plan, dtype=tdtype, precision=prec)
    out_h = torch.empty((w.B, w.S, Nl, w.D), dtype=tdtype, device=dev)
    stream = torch.cuda.current_stream(dev)
    cur = {"ev": None}

    def attend(qh, kh, vh):
        rfsa.rf_prepare(qh, kh, vh, "BSND", w.txt_len, w.latent, sp, ws, precision=prec)
        if cur["ev"] is not None:
            cur["ev"][4].record(stream)            # the attention stage starts
        rfsa.rf_attend(out_h, "BSND", w.txt_len, w.latent, sp, ws, precision=prec)
        return out_h

    def step(ev=None):
        cur["ev"] = ev
        marks = (lambda i: ev[i].record(stream)) if ev is not None else None
        return ulysses.rf_sparse_attention_ulysses(q_sh, k_sh, v_sh, w.txt_len, w.latent, sp, attend=attend,
                                                   marks=marks)

    for _ in range(max(args.warmup, 1)):
        step()
    torch.cuda.synchronize(dev)
    if rfsa.rf_read_status(ws, w.B, Nl, w.D, plan) != 0:
        raise RuntimeError("device status after warm-up")
    flops_local = rfsa.kept_block_flops(plan, views["kept"], w.B, Nl, w.D)
    stats = rfsa.rf_read_stats(ws, w.B, Nl, w.D, plan, precision=prec)
    tot = torch.tensor([flops_local, float(stats["near_ties"]), float(stats["kept_blocks"]),
                        float(stats["query_blocks"])], dtype=torch.float64, device=dev)
    dist.all_reduce(tot)
    flops, near, kept_blocks, query_blocks = tot.tolist()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        t0.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t1.record(stream)
        torch.cuda.synchronize(dev)
    dist.barrier()
    ms_total = t0.elapsed_time(t1)
    a2a_in = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    call = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    k3 = statistics.mean(e[4].elapsed_time(e[2]) for e in evs)
    a2a_out = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)

    # end to end: this rank's shards from pinned host memory, the output shard back
    e2e_steps = args.e2e_steps if args.e2e_steps is not None else min(args.steps, 10)
    hq, hk, hv = (t.cpu().pin_memory() for t in (q_sh, k_sh, v_sh))
    ho = torch.empty(q_sh.shape, dtype=tdtype, pin_memory=True)

    def e2e_call():
        dq, dk, dv = (t.to(dev, non_blocking=True) for t in (hq, hk, hv))
        o = ulysses.rf_sparse_attention_ulysses(dq, dk, dv, w.txt_len, w.latent, sp, attend=attend)
        ho.copy_(o, non_blocking=True)
        torch.cuda.current_stream(dev).synchronize()

    e2e_call()
    dist.barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_call()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / max(e2e_steps, 1)
    ms_total, e2e_ms, a2a_in, call, k3, a2a_out = reduce_max([ms_total, e2e_ms, a2a_in, call, k3, a2a_out], dist, dev)
    ms_step = ms_total / args.steps
    if rank == 0:
        peaks, src = _peaks()
        k3_tflops_rank = flops / world / (k3 * 1e-3) / 1e12          # the slowest rank's K3 over its share
        shard_bytes = q_sh.numel() * q_sh.element_size()
        line = {
            "metric": METRIC, "value": flops / (ms_step * 1e-3) / 1e12, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None,
            "dtype": args.dtype if prec == "native" else f"e4m3 ({args.dtype} in/out)", "data": "synthetic",
            "config": {"workload": _describe(w, args.dtype, prec), "mode": "ulysses",
                       "parallelism": f"ulysses sequence parallel over {world} rank(s): [B, S/{world}, {w.N}, D] "
                                      f"-> [B, S, {Nl}, D] -> [B, S/{world}, {w.N}, D]",
                       "l2": "inputs larger than L2 (no flush)", "kept_block_tflop_per_call": flops / 1e12},
            "e2e": {"value": flops / (e2e_ms * 1e-3) / 1e12, "unit": UNIT, "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": 3 * shard_bytes, "d2h_bytes_per_step": shard_bytes, "per": "rank"},
            "roofline": _roofline(k3_tflops_rank, prec, args.dtype, peaks, src, None),
            "mask_stats": {"k": plan.k, "nb": plan.nb, "kept_blocks": int(kept_blocks),
                           "query_blocks": int(query_blocks), "near_ties": int(near),
                           "near_tie_rule": "k-th and (k+1)-th block scores within 1e-5 (relative)"},
            # per rank and step: K1, K2, K3 and its second pass (the exchanges are NCCL's kernels)
            "gpu_launches": 4 * args.steps,
            "stages": {"all_to_all_in": {"ms": a2a_in, "bytes_per_rank": 3 * shard_bytes * (world - 1) / world},
                       "call": {"ms": call, "heads_per_rank": Nl},
                       "attention": {"kernels": "K3", "ms": k3, "tflops_per_rank": k3_tflops_rank},
                       "all_to_all_out": {"ms": a2a_out, "bytes_per_rank": shard_bytes * (world - 1) / world}},
            "clocks": clocks.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            from block_sparse_video_rf_b200 import synth as _s
            qc, kc, vc = _s.make_inputs(_s.workload(w.name, N=1, seed=w.seed), device="cpu")
            val, threads, desc = oracle_sample(qc, kc, vc, _s.workload(w.name, N=1, sparsity=w.sparsity),
                                               heads_total=w.N)
            line["cpu_baseline"] = {"value": val, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc}
        print(json.dumps(line), flush=True)
    dist.barrier()
    return 0


# ---------------------------------------------------------------- CUDA arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="minimax")
    ap.add_argument("--sparsity", type=float, default=None)
    ap.add_argument("--heads", type=int, default=None, help="override the head count (small profiling cases)")
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-budget", type=float, default=6.0, help="seconds of oracle work per reference step")
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--dtype", default="bf16", choices=["bf16", "f16"])
    ap.add_argument("--precision", default="native", choices=["native", "fp8"])
    ap.add_argument("--mode", default="replicas", choices=["replicas", "ulysses"],
                    help="replicas: every rank runs the whole call; ulysses: sequence-parallel over the ranks")
    args = ap.parse_args()

    from block_sparse_video_rf_b200 import synth
    over = {} if args.sparsity is None else {"sparsity": args.sparsity}
    if args.heads is not None:
        over["N"] = args.heads
    w = synth.workload(args.workload, **over)
    if args.impl == "reference":
        return run_reference(args, w)
    if args.mode == "ulysses":
        return run_ulysses(args, w)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))

    from block_sparse_video_rf_b200 import rfsa
    dev = torch.device("cuda", local)
    tdtype = torch.float16 if args.dtype == "f16" else torch.bfloat16
    prec = args.precision
    q, k, v = synth.make_inputs(w, device=dev, dtype=tdtype)
    out = torch.empty_like(q)
    sp = np.float32(w.sparsity)
    ws = rfsa.alloc_workspace(w.B, w.S, w.N, w.D, w.txt_len, w.latent, device=dev, precision=prec)
    plan = rfsa.rf_plan(w.S, w.txt_len, w.latent, sp)
    views = rfsa.workspace_views(ws, w.B, w.N, plan, dtype=tdtype, precision=prec)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
            rfsa.rf_debug_set_stage_event(ev[3])       # the library records it after K1
        rfsa.rf_prepare(q, k, v, w.layout, w.txt_len, w.latent, sp, ws, precision=prec)
        if ev is not None:
            ev[1].record(stream)
        rfsa.rf_attend(out, w.layout, w.txt_len, w.latent, sp, ws, precision=prec)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(max(args.warmup, 1)):
        step()
    torch.cuda.synchronize(dev)
    status = rfsa.rf_read_status(ws, w.B, w.N, w.D, plan)
    if status != 0:
        raise RuntimeError(f"device status {status} after warm-up")
    flops = rfsa.kept_block_flops(plan, views["kept"], w.B, w.N, w.D)
    stats = rfsa.rf_read_stats(ws, w.B, w.N, w.D, plan, precision=prec)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for e in evs:
        e[3].record(stream)                            # creates the CUDA event the library records
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        t_start.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    rfsa.rf_debug_set_stage_event(None)
    if dist is not None:
        dist.barrier()
    ms_total = t_start.elapsed_time(t_end)
    k1 = [e[0].elapsed_time(e[3]) for e in evs]
    k1k2 = [e[0].elapsed_time(e[1]) for e in evs]
    k3 = [e[1].elapsed_time(e[2]) for e in evs]
    status = rfsa.rf_read_status(ws, w.B, w.N, w.D, plan)
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed steps")

    # end to end through host buffers: H2D of q, k, v and D2H of the output inside the timed region
    e2e_steps = args.e2e_steps if args.e2e_steps is not None else min(args.steps, 10)
    qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
    oh = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)

    def e2e_call():      # the library's own host-buffer entry point
        rfsa.rf_sparse_attention_host(qh, kh, vh, w.layout, w.txt_len, w.latent, sp, oh, precision=prec)

    e2e_call()   # warm the caches
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_call()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / max(e2e_steps, 1)

    # slowest rank decides
    ms_total, e2e_ms, k3_ms = reduce_max([ms_total, e2e_ms, statistics.mean(k3)], dist, dev)
    ms_step = ms_total / args.steps
    value = aggregate(flops, world, ms_step)
    e2e_value = aggregate(flops, world, e2e_ms)

    if rank == 0:
        peaks, src = _peaks()
        k3_tflops = flops / (k3_ms * 1e-3) / 1e12
        tensor_bytes = q.numel() * q.element_size()
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": args.dtype if prec == "native" else f"e4m3 ({args.dtype} in/out)",
            "data": "synthetic",
            "config": {"workload": _describe(w, args.dtype, prec), "l2": "inputs larger than L2 (no flush)",
                       "kept_block_tflop_per_call": flops / 1e12, "k": plan.k, "nb": plan.nb, "ff": plan.ff,
                       "P": plan.P, "ms_prepare": statistics.mean(k1k2), "ms_attention": k3_ms},
            "e2e": {"value": e2e_value, "unit": UNIT, "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": 3 * tensor_bytes, "d2h_bytes_per_step": tensor_bytes},
            # the committed capture is of the MiniMax-H3 shape: other workloads' traffic is not a multiple of it
            "roofline": _roofline(k3_tflops, prec, args.dtype, peaks, src,
                                  _k3_traffic(w.N, "k3_fp8" if prec == "fp8" else "k3")
                                  if args.dtype == "bf16" and w.name == "minimax" else None),
            "mask_stats": _mask_stats(stats, plan),
            # K1, K2 and K3 (the chain kernel and its second pass, which returns at once when no unit was
            # handed to it)
            "gpu_launches": 4 * args.steps,
            "stages": _stages(w, plan, prec, statistics.mean(k1k2), k3_ms, k3_tflops, peaks["hbm_gbs"],
                              statistics.mean(k1)),
            "clocks": clocks.summary(),
        }
        line["stages"]["attention"]["kv_stream"] = _kv_stream(flops, prec, k3_ms, line["clocks"].get("sm_mhz"),
                                                              torch.cuda.get_device_properties(dev).multi_processor_count)
        if world == 1 and not args.no_cpu_baseline:
            val, threads, desc = oracle_sample(q, k, v, w)
            line["cpu_baseline"] = {"value": val, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc}
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
