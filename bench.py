"""Benchmark of the NSA hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl nsa|reference]

One step = one NSA forward (compression + block scores, top-k, selection,
sliding window, gated combination) over the 340M-shape workload: B=1,
T=8192, 16 query heads, 4 KV heads (GQA-4), head dim 64, block 64, top-k 16,
window 512, bf16, with inputs resident in HBM.  L2 is flushed (256 MiB
write) between timed steps; each step is timed with CUDA events on the
launching stream.  Rank 0 prints one JSON line.  Its `e2e` figure times the
same forward through nsa_forward_host from page-locked host buffers, the
copies in and out inside each timed step.

With N > 1 (torchrun), every rank runs its own independent copy of the
workload (NSA has no cross-sequence exchange: weak scaling, no data-path
collective); the reported time is the max over ranks and the value sums the
tokens of all ranks.

--impl reference times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import sparse_attention_nsa_b200 as nsa  # noqa: E402
from sparse_attention_nsa_b200 import inputs as W  # noqa: E402

METRIC = "NSA fwd tokens/s & TFLOP/s (frac of bf16 peak) @8192 GQA-4; decode HBM GB/s"
WORK = W.NSA_340M
DECODE = W.DECODE_32K


def kernels_per_forward(w) -> int:
    """Kernels one nsa_forward of workload w launches (as its ncu launch list
    shows): pooling, compression branch + scores, top-k, window, then either
    the query-tiled selection with the combination, or (block-major, from Nb
    >= 8 top-k and Tq >= 64) the reverse map's scan and fill (the top-k does
    its counting), the selection kernel and the merge with the combination."""
    nb = -(-w.T // w.sel_block)
    block_major = w.dtype == torch.bfloat16 and nb >= 8 * w.topk and w.T >= 64
    return 4 + (4 if block_major else 1)


# ------------------------------------------------------------------ work model
def fwd_flops(w, branch_mask=None) -> dict:
    """Algorithmic FLOPs of one forward: 4*D per (query row, attended key)
    (QK^T and PV); the compression branch counts 2*D per key when only its
    scores are needed."""
    m = w.branch_mask if branch_mask is None else branch_mask
    l, n, win, D = w.sel_block, w.topk, w.window, w.D
    sel = swa = cmp = 0
    for t in range(w.T):
        sel += min(t + 1, (n - 1) * l + t % l + 1)
        swa += min(t + 1, win)
        cmp += min((t + 1) // w.cmp_block, w.Nc)
    rows = w.B * w.Hq
    out = {"sel": 4 * D * sel * rows if m & 2 else 0,
           "swa": 4 * D * swa * rows if m & 4 else 0,
           "cmp": (4 if m & 1 else 2) * D * cmp * rows if m & 3 else 0}
    out["total"] = sum(out.values())
    return out


def executed_sel_flops(w, idx) -> float:
    """MMA FLOPs the selection kernel actually issues: each 128-row tile
    (128/G tokens x G heads of one group) runs S = QK^T and O += PV over the
    union of its tokens' selected 64-key blocks (2 x 2*128*64*64 FLOP per
    union block), whatever fraction of its rows selected each block."""
    import numpy as np
    ii = idx.cpu().numpy()  # [B, T, Hkv, topk]
    tq = 128 // (w.Hq // w.Hkv)
    blocks = 0
    for b in range(w.B):
        for g in range(w.Hkv):
            for t0 in range(0, w.T, tq):
                sel = ii[b, t0:t0 + tq, g].ravel()
                blocks += len(np.unique(sel[sel >= 0]))
    return blocks * 2 * 2.0 * 128 * 64 * 64


def load_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def profiled_traffic(kernel_src: str, profile_json: str):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum)
    recorded in a committed machine-readable ncu summary, if that summary was
    taken on the current source of the kernel (its sha1 prefix matches);
    otherwise None (the counters are stale)."""
    import hashlib
    try:
        sha = hashlib.sha1(open(os.path.join(ROOT, kernel_src), "rb").read()).hexdigest()[:12]
        with open(os.path.join(ROOT, profile_json)) as f:
            rec = json.load(f)
        if rec.get("source_sha1") != sha:
            return None
        return int(rec["dram_bytes_per_launch"])
    except Exception:
        return None


def sel_compulsory_bytes(w) -> int:
    """HBM bytes the selection branch must move at the least: q, k, v and
    the block indices read once; o_sel (path dtype) and lse_sel written."""
    es = 2 if w.dtype == torch.bfloat16 else 4
    return (w.B * w.T * w.Hq * w.D * es + 2 * w.B * w.T * w.Hkv * w.D * es
            + w.B * w.T * w.Hkv * w.topk * 4 + w.B * w.T * w.Hq * w.D * es + w.B * w.T * w.Hq * 4)


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (read only)."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            try:  # NVML indexes every GPU of the host; match ours by UUID
                uuid = str(torch.cuda.get_device_properties(index).uuid)
                uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
                self._h = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if mask & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self._nv:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self) -> dict:
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ------------------------------------------------------------------ timing helpers
class Flusher:
    def __init__(self, dev):
        self.buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def __call__(self):
        self.buf.fill_(1)


def timed_steps(fn, steps: int, flush, stream) -> list[float]:
    """Per-step device time (ms) of fn, with an L2 flush outside each timing."""
    times = []
    for _ in range(steps):
        flush()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        times.append((a, b))
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in times]


def kernel_event_times(fn, steps: int, flush, stream) -> list[float]:
    """Device time (ms) of the block-major selection kernel inside fn: the
    library records a CUDA event pair around it on the launching stream."""
    times = []
    for _ in range(steps):
        flush()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)  # creates the events; the library records them again
        b.record(stream)
        nsa.nsa_set_kernel_events(a, b)
        fn()
        times.append((a, b))
    nsa.nsa_set_kernel_events(None, None)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in times]


def sel_bm_algorithmic_bytes(w, idx) -> int:
    """HBM bytes the block-major selection kernel must move: one fp16 partial
    row (128 B) and one float lse per (query row, used slot) written, plus Q,
    K and V read once and the reverse-map list entries (4 B per used slot)."""
    import numpy as np
    ii = idx.cpu().numpy()  # [B, T, Hkv, topk]
    t = np.arange(w.T)[None, :, None, None]
    used = (ii >= 0) & (ii <= t // w.sel_block)
    slots = int(used.sum())  # (token, group, slot) triples
    G = w.Hq // w.Hkv
    es = 2
    return (slots * G * (128 + 4) + slots * 4
            + w.B * w.T * w.Hq * w.D * es + 2 * w.B * w.T * w.Hkv * w.D * es)


def roofline_line(kernel: str, flops: float, ms: float, peaks: dict, traffic, compulsory: int,
                  design: dict | None = None) -> dict:
    """Roofline record of a tensor-bound kernel: algorithmic TFLOP/s per
    launch against the measured bf16 peak."""
    achieved = flops / (ms * 1e-3) / 1e12
    r = {"bound": "tensor", "kernel": kernel, "achieved": achieved,
         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
         "frac": achieved / peaks["bf16_tflops"], "traffic": traffic,
         "peak_source": f"{peaks['source']} bf16 dense GEMM (burst)",
         "algorithmic_flops": flops, "ms_per_launch": ms,
         "compulsory_bytes": compulsory,
         "traffic_over_algorithmic": (traffic / compulsory) if traffic else None}
    if design:
        r["design_min_bytes"] = design
    return r


def barrier_sync(dist_on):
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()


def max_over_ranks(x: float, dist_on: bool, device: str = "cuda") -> float:
    """Job time = the slowest rank's time (all ranks must call this)."""
    if not dist_on:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_rank_step: int, world: int, job_ms: float) -> float:
    """Weak scaling: every rank processes its own copy of the workload, so
    the job processes world x tokens per step in the slowest rank's time."""
    return tokens_per_rank_step * world / (job_ms * 1e-3)


# ------------------------------------------------------------------ CPU oracle leg
def oracle_tokens_per_s(budget_s: float, seed: int = 0) -> dict:
    """Time the fp64 CPU oracle on a bounded sample of the bench workload:
    whole tokens (all heads, all branches), spread over the sequence."""
    import numpy as np

    import oracle as orc
    w = WORK
    inp = W.make_inputs(w, seed=seed)
    c = orc.Cfg(B=w.B, T=w.T, Hq=w.Hq, Hkv=w.Hkv, D=w.D, cmp_block=w.cmp_block,
                cmp_stride=w.cmp_stride, sel_block=w.sel_block, topk=w.topk,
                window=w.window, scale=w.scale, kv_round=orc.KV_BF16,
                branch_mask=w.branch_mask)
    q, k, v, g = (inp[n].double().numpy() for n in ("q", "k", "v", "gates"))
    kc, vc = orc.compress(c, k, v)
    rng = np.random.default_rng(seed)
    # calibrate on a small sample, then size the timed sample to the budget
    n = 64
    while True:
        rows = np.stack([np.zeros(n, dtype=int), rng.integers(0, w.T, n)], 1)
        t0 = time.perf_counter()
        orc.forward_rows(c, q, k, v, g, rows, kc, vc)
        dt = time.perf_counter() - t0
        if dt >= budget_s or n >= w.B * w.T:
            break
        n = int(min(w.B * w.T, max(2 * n, n * budget_s / max(dt, 1e-3) * 1.05)))
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": n / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} whole tokens (16 heads, 3 branches) drawn uniformly from the "
                      f"T=8192 sequence of {w.name}; compression of the full sequence "
                      f"precomputed; {dt:.1f} s"}


def workload_config(w, world: int) -> dict:
    """The JSON line's config, the same for both arms: the workload, the L2
    treatment between timed GPU steps, and how the ranks divide the work."""
    return {"workload": w.name, "B": w.B, "T": w.T, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D,
            "block": w.sel_block, "topk": w.topk, "window": w.window,
            "l2": "flushed between GPU steps (256 MiB write); the CPU oracle reads a "
                  "fresh sample each step",
            "parallelism": f"replicas x{world} (independent sequences, no collective "
                           "on the data path)"}


# ------------------------------------------------------------------ main legs
def run_reference(args, rank: int, world: int) -> None:
    if rank != 0:
        return
    budget = max(2.0, min(20.0, 25.0 / max(args.steps, 1)))
    vals = []
    cb = None
    for i in range(args.warmup + args.steps):
        r = oracle_tokens_per_s(budget if i >= args.warmup else 1.0, seed=0)
        if i >= args.warmup:
            vals.append(r["value"])
            cb = r
    v = statistics.median(vals)
    cb["value"] = v
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": WORK.B * WORK.T / v * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(WORK, world),
            "cpu_baseline": cb,
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_gpu(args, rank: int, world: int, dist_on: bool) -> None:
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    nsa.load()
    stream = torch.cuda.current_stream()
    flush = Flusher(dev)
    w = WORK
    p = nsa.params_for(w)
    inp = W.make_inputs(w, seed=rank)
    q, k, v, g = (inp[n].to(dev) for n in ("q", "k", "v", "gates"))
    out = torch.empty_like(q)
    ws = nsa.alloc_workspace(p, dev)
    saved = {"idx": torch.empty((w.B, w.T, w.Hkv, w.topk), dtype=torch.int32, device=dev)}

    def step():
        nsa.nsa_forward(p, q, k, v, g, out, saved, ws)

    for _ in range(args.warmup):
        flush()
        step()
    if nsa.nsa_last_device_error() != 0:
        raise RuntimeError("device-side check failed during warm-up")
    # clocks are sampled across every timed region of this run (forward,
    # selection alone, end to end, decode, training step)
    sampler = ClockSampler(local)
    barrier_sync(dist_on)
    sampler.__enter__()
    times = timed_steps(step, args.steps, flush, stream)
    barrier_sync(dist_on)
    ms = max_over_ranks(sum(times) / len(times), dist_on)
    flops = fwd_flops(w)
    tokens_per_step = w.B * w.T
    value = job_tokens_per_s(tokens_per_step, world, ms)

    # the forward's dominant kernel (block-major selection, sel_bm_kernel):
    # CUDA events the library records around that kernel on this stream,
    # inside the same forward call, flushed as above
    bm_ms = statistics.mean(kernel_event_times(step, args.steps, flush, stream))
    bm_bytes = sel_bm_algorithmic_bytes(w, saved["idx"])
    # context: the query-tiled selection kernel on the same indices
    o_sel = torch.empty_like(q)
    for _ in range(2):
        nsa.nsa_sel_attn_fwd(p, q, k, v, saved["idx"], o_sel, None)
    sel_ms = statistics.mean(timed_steps(
        lambda: nsa.nsa_sel_attn_fwd(p, q, k, v, saved["idx"], o_sel, None),
        args.steps, flush, stream))
    peaks = load_peaks()
    sel_tflops = flops["sel"] / (sel_ms * 1e-3) / 1e12
    sel_exec_flops = executed_sel_flops(w, saved["idx"])

    # end to end through the C ABI with host buffers (pinned): nsa_forward_host
    # copies the inputs in, runs the forward and copies out back, all timed
    hq, hk, hv, hg = (x.cpu().pin_memory() for x in (q, k, v, g))
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    hws = torch.empty(nsa.nsa_forward_host_workspace_size(p), dtype=torch.uint8, device=dev)

    def e2e_step():
        nsa.nsa_forward_host(p, hq, hk, hv, hg, hout, hws, stream)

    for _ in range(2):
        e2e_step()
    e2e_ms = max_over_ranks(statistics.mean(timed_steps(e2e_step, args.steps, flush, stream)),
                            dist_on)
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hg))
    d2h = hout.numel() * hout.element_size()

    del hq, hk, hv, hg, hout, hws
    if args.leg == "forward":  # the forward alone (for profiling it)
        sampler.__exit__(None, None, None)
        print(json.dumps({"forward": {"ms_per_step": ms, "tokens_per_s": value,
                                      "sel_bm_kernel_ms": bm_ms,
                                      "sel_bm_kernel_gbs": bm_bytes / (bm_ms * 1e-3) / 1e9}}))
        return
    # decode (B=64 sequences, 32768-token caches): HBM GB/s
    dec = run_decode(dev, flush, stream, args.steps, peaks)
    # training step (B=8 forward + backward)
    train = run_train(dev, flush, stream, max(3, args.steps // 4), peaks)
    # long context (32768 tokens, block-major selection)
    long_ctx = run_long(dev, flush, stream, max(3, args.steps // 4), peaks)
    # the 1.3B-shape forward (B=4, GQA-4 with 8 KV heads)
    onep3b = run_1p3b(dev, flush, stream, max(3, args.steps // 2), peaks)
    # MoBA block attention (block 512, top-3) on the selection kernels
    moba = run_moba(dev, flush, stream, max(3, args.steps // 2), peaks)
    # NSA on its parametric compressor (blocks of 32 every 16 tokens)
    mlp = run_mlp(dev, flush, stream, max(3, args.steps // 2), peaks)
    # the pages' branch pruning: sel + window, cmp + window, window alone
    pruned = run_pruned(dev, flush, stream, max(3, args.steps // 2), peaks)
    # selection backward, two-pass against single-pass atomic
    selbwd = run_sel_bwd_compare(dev, flush, stream, 3, peaks)
    sampler.__exit__(None, None, None)

    barrier_sync(dist_on)
    if rank != 0:
        return
    clocks = sampler.summary()
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": workload_config(w, world),
        "tflops": flops["total"] * world / (ms * 1e-3) / 1e12,
        "frac_bf16_peak": flops["total"] / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
        "flops_per_step": flops,
        # dominant kernel of the timed forward: the block-major selection
        # kernel, rated on the selection branch's algorithmic FLOPs (4 D per
        # selected (query row, key)) against the measured bf16 peak (burst:
        # the kernel is timed inside a 0.3 ms forward).  traffic is its ncu
        # DRAM bytes per launch; traffic_over_algorithmic divides that by the
        # branch's compulsory bytes (q, k, v, indices in; o_sel, lse out).
        # The design's own minimum bytes (the per-(row, slot) partials it
        # writes) are given as a labelled extra.
        "roofline": roofline_line(
            "block-major selection (sel_bm_kernel)", flops["sel"], bm_ms, peaks,
            profiled_traffic("sparse_attention_nsa_b200/csrc/k_sel_bm.cu",
                             "profiles/sel_bm_340m.json"),
            sel_compulsory_bytes(w),
            design={"bytes": bm_bytes, "what": "fp16 partial row + lse per used (row, slot), "
                    "list entries, q/k/v once",
                    "gbs": bm_bytes / (bm_ms * 1e-3) / 1e9,
                    "frac_of_hbm": bm_bytes / (bm_ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}),
        # context: the query-tiled selection kernel (the forward's path for
        # Nb < 8 top-k) on the same indices; on structure-free selections the
        # union of a tile's blocks is near dense, so it issues more MMA work
        # than the algorithmic count
        "selection_query_tiled": {"ms_per_launch": sel_ms, "tflops": sel_tflops,
                                  "frac_bf16_peak": sel_tflops / peaks["bf16_tflops"],
                                  "executed_tflops": sel_exec_flops / (sel_ms * 1e-3) / 1e12,
                                  "executed_over_algorithmic": sel_exec_flops / flops["sel"]},
        "decode": dec,
        "train": train,
        "long_context": long_ctx,
        "nsa_1p3b": onep3b,
        "moba": moba,
        "mlp_compression": mlp,
        "pruned_branches": pruned,
        "sel_bwd_two_pass_vs_atomic": selbwd,
        "e2e": {"value": job_tokens_per_s(tokens_per_step, world, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": kernels_per_forward(w) * args.steps,
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_tokens_per_s(budget_s=12.0)
    print(json.dumps(line), flush=True)


def run_train(dev, flush, stream, steps, peaks, batch=None) -> dict:
    """One training step of attention: NSA forward (intermediates kept) and
    the whole backward, B=8 x 8192 tokens, 340M shape (batch overrides B, to
    profile a smaller case of the same kernels)."""
    w = W.TRAIN_340M if batch is None else W.TRAIN_340M.replace(B=batch)
    inp = W.make_inputs(w, seed=1, with_dout=True)
    q, k, v, g, dout = (inp[n].to(dev) for n in ("q", "k", "v", "gates", "dout"))
    p = nsa.params_for(w)
    out = torch.empty_like(q)
    ws = nsa.alloc_workspace(p, dev)
    f32 = torch.float32
    saved = {"kc": torch.empty((w.B, w.Nc, w.Hkv, w.D), dtype=w.dtype, device=dev),
             "vc": torch.empty((w.B, w.Nc, w.Hkv, w.D), dtype=w.dtype, device=dev),
             "o_cmp": torch.empty_like(q), "o_sel": torch.empty_like(q), "o_swa": torch.empty_like(q),
             "lse_cmp": torch.empty((w.B, w.T, w.Hq), dtype=f32, device=dev),
             "lse_sel": torch.empty((w.B, w.T, w.Hq), dtype=f32, device=dev),
             "lse_swa": torch.empty((w.B, w.T, w.Hq), dtype=f32, device=dev),
             "idx": torch.empty((w.B, w.T, w.Hkv, w.topk), dtype=torch.int32, device=dev)}
    dq = torch.empty((w.B, w.T, w.Hq, w.D), dtype=f32, device=dev)
    dk = torch.empty((w.B, w.T, w.Hkv, w.D), dtype=f32, device=dev)
    dv = torch.empty_like(dk)
    dg = torch.empty((w.B, w.T, w.Hq, 3), dtype=f32, device=dev)
    bws = torch.empty(nsa.nsa_backward_workspace_size(p), dtype=torch.uint8, device=dev)

    def fwd():
        nsa.nsa_forward(p, q, k, v, g, out, saved, ws)

    def bwd():
        nsa.nsa_backward(p, q, k, v, g, dout, saved, dq, dk, dv, dg, bws)

    for _ in range(2):
        fwd()
        bwd()
    fwd_ms = statistics.mean(timed_steps(fwd, steps, flush, stream))
    bwd_ms = statistics.mean(timed_steps(bwd, steps, flush, stream))
    flops = fwd_flops(w)["total"]
    step_ms = fwd_ms + bwd_ms
    return {"workload": w.name, "fwd_ms": fwd_ms, "bwd_ms": bwd_ms, "ms_per_step": step_ms,
            "tokens_per_s": w.B * w.T / (step_ms * 1e-3),
            "tflops_fwd_plus_bwd": 3.5 * flops / (step_ms * 1e-3) / 1e12,
            "flops_note": "algorithmic: forward + backward counted as 2.5x forward"}


def run_sel_bwd_compare(dev, flush, stream, steps, peaks, batch=8) -> dict:
    """The selection backward at the training shape (B=8, T=8192, GQA-4) two
    ways on the same forward: the two-pass kernels (query-stationary dQ, then
    key-stationary dK/dV over the reverse map) and the single pass that adds
    dK/dV with atomics from the query-stationary pass; the pages compare
    these two designs and find the two-pass one faster."""
    w = W.TRAIN_340M.replace(B=batch)
    inp = W.make_inputs(w, seed=6, with_dout=True)
    q, k, v, g = (inp[n].to(dev) for n in ("q", "k", "v", "gates"))
    p = nsa.params_for(w)
    out = torch.empty_like(q)
    f32 = torch.float32
    saved = {"idx": torch.empty((w.B, w.T, w.Hkv, w.topk), dtype=torch.int32, device=dev),
             "o_sel": torch.empty_like(q),
             "lse_sel": torch.empty((w.B, w.T, w.Hq), dtype=f32, device=dev)}
    nsa.nsa_forward(p, q, k, v, g, out, saved, nsa.alloc_workspace(p, dev))
    dO = inp["dout"].to(dev).float()
    dq = torch.zeros((w.B, w.T, w.Hq, w.D), dtype=f32, device=dev)
    dk = torch.zeros((w.B, w.T, w.Hkv, w.D), dtype=f32, device=dev)
    dv = torch.zeros_like(dk)
    ws = torch.empty(nsa.nsa_backward_workspace_size(p), dtype=torch.uint8, device=dev)
    args = (p, q, k, v, saved["idx"], saved["o_sel"], saved["lse_sel"], dO, dq, dk, dv, ws)

    def two_pass():
        nsa.nsa_sel_attn_bwd(*args)

    def single_pass():
        nsa.nsa_sel_attn_bwd_atomic(*args)

    for _ in range(2):
        two_pass()
        single_pass()
    t2 = statistics.mean(timed_steps(two_pass, steps, flush, stream))
    t1 = statistics.mean(timed_steps(single_pass, steps, flush, stream))
    if nsa.nsa_last_device_error() != 0:
        raise RuntimeError("device-side check failed in the selection-backward comparison")
    flops = 2.5 * fwd_flops(w)["sel"]
    return {"workload": w.name, "two_pass_ms": t2, "single_pass_atomic_ms": t1,
            "two_pass_tflops": flops / (t2 * 1e-3) / 1e12,
            "atomic_over_two_pass": t1 / t2,
            "flops_note": "algorithmic selection backward counted as 2.5x its forward"}


def run_1p3b(dev, flush, stream, steps, peaks) -> dict:
    """The 1.3B-shape forward: B=4 x 8192 tokens, 32 query heads on 8 KV
    heads (GQA-4), block 64, top-k 16, window 512, bf16."""
    w = W.NSA_1P3B
    inp = W.make_inputs(w, seed=4)
    q, k, v, g = (inp[n].to(dev) for n in ("q", "k", "v", "gates"))
    p = nsa.params_for(w)
    out = torch.empty_like(q)
    ws = nsa.alloc_workspace(p, dev)

    def fwd():
        nsa.nsa_forward(p, q, k, v, g, out, None, ws)

    for _ in range(3):
        fwd()
    ms = statistics.mean(timed_steps(fwd, steps, flush, stream))
    if nsa.nsa_last_device_error() != 0:
        raise RuntimeError("device-side check failed in the 1.3B-shape leg")
    flops = fwd_flops(w)
    tf = flops["total"] / (ms * 1e-3) / 1e12
    return {"workload": w.name, "fwd_ms": ms, "tokens_per_s": w.B * w.T / (ms * 1e-3),
            "tflops": tf, "frac_bf16_peak": tf / peaks["bf16_tflops"],
            "flops_per_step": flops}


def run_moba(dev, flush, stream, steps, peaks) -> dict:
    """MoBA block attention at the 340M shape (B=1, T=8192, GQA-4; block 512,
    top-k 3, the pages' MoBA setting) through nsa_moba_forward: gate and
    top-k, then the selection attention kernels on the chosen blocks."""
    w = W.NSA_340M.replace(name="moba_340m_gqa4_t8192_L512_k3_bf16")
    L, k = 512, 3
    inp = W.make_inputs(w, seed=5)
    q, kk, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    p = nsa.make_moba_params(w.B, w.T, w.Hq, w.Hkv, block=L, topk=k, dtype=w.dtype)
    out = torch.empty_like(q)
    ws = torch.empty(nsa.nsa_moba_workspace_size(p), dtype=torch.uint8, device=dev)

    def fwd():
        nsa.nsa_moba_forward(p, q, kk, v, out, None, None, ws)

    for _ in range(3):
        fwd()
    ms = statistics.mean(timed_steps(fwd, steps, flush, stream))
    if nsa.nsa_last_device_error() != 0:
        raise RuntimeError("device-side check failed in the MoBA leg")
    keys = sum(min(t + 1, (k - 1) * L + t % L + 1) for t in range(w.T))
    flops = 4 * w.D * keys * w.B * w.Hq
    tf = flops / (ms * 1e-3) / 1e12
    return {"workload": w.name, "fwd_ms": ms, "tokens_per_s": w.B * w.T / (ms * 1e-3),
            "tflops": tf, "frac_bf16_peak": tf / peaks["bf16_tflops"], "flops_per_step": flops}


def run_mlp(dev, flush, stream, steps, peaks) -> dict:
    """NSA with its own parametric compressor (one linear layer over each
    block's rows) at the 340M shape with NSA's original compression geometry
    (blocks of 32 every 16 tokens; selection block 64, top-k 16, window
    512), B=1 x 8192 tokens: the compressor forward and backward alone, the
    whole forward and a training step (forward + backward), beside the same
    forward on the mean pool."""
    w = W.NSA_340M.replace(name="nsa_mlp_340m_gqa4_t8192_l32_d16_bf16", cmp_block=32,
                           cmp_stride=16)
    inp = W.make_inputs(w, seed=7, with_dout=True)
    q, k, v, g, dout = (inp[n].to(dev) for n in ("q", "k", "v", "gates", "dout"))
    wk, wv = (t.to(dev) for t in W.make_mlp_weights(w, seed=8))
    p = nsa.params_for(w)
    out = torch.empty_like(q)
    ws = torch.empty(nsa.nsa_forward_mlp_workspace_size(p), dtype=torch.uint8, device=dev)
    mws = nsa.alloc_workspace(p, dev)
    fws = torch.empty(max(nsa.nsa_compress_mlp_workspace_size(p), 1), dtype=torch.uint8,
                      device=dev)
    f32 = torch.float32
    kc = torch.empty((w.B, w.Nc, w.Hkv, w.D), dtype=w.dtype, device=dev)
    vc = torch.empty_like(kc)
    dkc = torch.randn((w.B, w.Nc, w.Hkv, w.D), dtype=f32, device=dev)
    dvc = torch.randn_like(dkc)
    dk = torch.zeros((w.B, w.T, w.Hkv, w.D), dtype=f32, device=dev)
    dv = torch.zeros_like(dk)
    dwk = torch.empty((w.cmp_block * w.D, w.D), dtype=f32, device=dev)
    dwv = torch.empty_like(dwk)
    cws = torch.empty(nsa.nsa_compress_mlp_bwd_workspace_size(p), dtype=torch.uint8, device=dev)
    saved = nsa.alloc_saved(p, dev)
    bws = torch.empty(nsa.nsa_backward_mlp_workspace_size(p), dtype=torch.uint8, device=dev)
    dq = torch.empty((w.B, w.T, w.Hq, w.D), dtype=f32, device=dev)
    dkk, dvv = torch.empty_like(dk), torch.empty_like(dk)
    dg = torch.empty((w.B, w.T, w.Hq, 3), dtype=f32, device=dev)

    def cfwd():
        nsa.nsa_compress_mlp(p, k, v, wk, wv, kc, vc, fws)

    def cbwd():
        nsa.nsa_compress_mlp_bwd(p, k, v, wk, wv, dkc, dvc, dk, dv, dwk, dwv, cws)

    def fwd_mlp():
        nsa.nsa_forward_mlp(p, q, k, v, wk, wv, g, out, None, ws)

    def fwd_mean():
        nsa.nsa_forward(p, q, k, v, g, out, None, mws)

    def train():
        nsa.nsa_forward_mlp(p, q, k, v, wk, wv, g, out, saved, ws)
        nsa.nsa_backward_mlp(p, q, k, v, wk, wv, g, dout, saved, dq, dkk, dvv, dwk, dwv, dg, bws)

    for fn in (cfwd, cbwd, fwd_mlp, fwd_mean, train, train):
        fn()
    res = {}
    for name, fn in (("compress_fwd_ms", cfwd), ("compress_bwd_ms", cbwd),
                     ("fwd_ms", fwd_mlp), ("fwd_mean_pool_ms", fwd_mean), ("train_step_ms", train)):
        res[name] = statistics.mean(timed_steps(fn, steps, flush, stream))
    if nsa.nsa_last_device_error() != 0:
        raise RuntimeError("device-side check failed in the parametric-compression leg")
    # the compressor's GEMM work: kc and vc, one (l*D) x D product per block row
    rows = w.B * w.Nc * w.Hkv
    cflops = 2 * 2 * rows * (w.cmp_block * w.D) * w.D
    ctf = cflops / (res["compress_fwd_ms"] * 1e-3) / 1e12
    btf = 2 * cflops / (res["compress_bwd_ms"] * 1e-3) / 1e12
    res.update({"workload": w.name, "tokens_per_s": w.B * w.T / (res["fwd_ms"] * 1e-3),
                "compress_fwd_tflops": ctf, "compress_bwd_tflops": btf,
                "compress_flops": cflops,
                "note": "compressor FLOPs 2 x (kc, vc) x rows x (l D) x D; its backward "
                        "(dW and the rows' gradient) twice that"})
    return res


def run_pruned(dev, flush, stream, steps, peaks) -> dict:
    """The pages' branch pruning at the 340M shape (B=1, T=8192, GQA-4): the
    same forward with every branch, with selection + window (compression
    gate 0), and with the window alone, as later layers run once their
    unused branches are pruned; speedups are against the full forward."""
    res = {}
    for name, mask in (("all", W.BR_ALL), ("sel_swa", W.BR_SEL | W.BR_SWA),
                       ("cmp_swa", W.BR_CMP | W.BR_SWA), ("swa", W.BR_SWA)):
        w = W.NSA_340M.replace(name=f"nsa_340m_gqa4_t8192_{name}_bf16", branch_mask=mask,
                               cmp_gate_zero=not (mask & W.BR_CMP))
        inp = W.make_inputs(w, seed=9)
        q, k, v, g = (inp[n].to(dev) for n in ("q", "k", "v", "gates"))
        p = nsa.params_for(w)
        out = torch.empty_like(q)
        ws = nsa.alloc_workspace(p, dev)

        def fwd():
            nsa.nsa_forward(p, q, k, v, g, out, None, ws)

        for _ in range(3):
            fwd()
        ms = statistics.mean(timed_steps(fwd, steps, flush, stream))
        res[name] = {"fwd_ms": ms, "tokens_per_s": w.B * w.T / (ms * 1e-3)}
    if nsa.nsa_last_device_error() != 0:
        raise RuntimeError("device-side check failed in the pruned-branch leg")
    for name in res:
        res[name]["speedup_vs_all"] = res["all"]["fwd_ms"] / res[name]["fwd_ms"]
    return res


def run_long(dev, flush, stream, steps, peaks) -> dict:
    """Long-context forward: the pruned MQA workload (B=1, 32768 tokens,
    selection + window).  Its selection runs block-major (Nb = 32 top-k);
    the query-tiled kernel is timed beside it on the same indices."""
    w = W.PRUNED_32K
    inp = W.make_inputs(w, seed=2)
    q, k, v, g = (inp[n].to(dev) for n in ("q", "k", "v", "gates"))
    p = nsa.params_for(w)
    out = torch.empty_like(q)
    ws = nsa.alloc_workspace(p, dev)
    saved = {"idx": torch.empty((w.B, w.T, w.Hkv, w.topk), dtype=torch.int32, device=dev)}

    def fwd():
        nsa.nsa_forward(p, q, k, v, g, out, saved, ws)

    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.T, w.Hq), dtype=torch.float32, device=dev)
    sws = torch.empty(nsa.nsa_sel_workspace_size(p), dtype=torch.uint8, device=dev)

    def sel_bm():
        nsa.nsa_sel_attn_fwd_ws(p, q, k, v, saved["idx"], o, lse, sws)

    def sel_tiled():
        nsa.nsa_sel_attn_fwd(p, q, k, v, saved["idx"], o, lse)

    for _ in range(2):
        fwd()
    fwd_ms = statistics.mean(timed_steps(fwd, steps, flush, stream))
    bm_ms = statistics.mean(timed_steps(sel_bm, steps, flush, stream))
    tiled_ms = statistics.mean(timed_steps(sel_tiled, steps, flush, stream))
    if nsa.nsa_last_device_error() != 0:
        raise RuntimeError("device-side check failed in the long-context leg")
    flops = fwd_flops(w)
    return {"workload": w.name, "fwd_ms": fwd_ms, "tokens_per_s": w.B * w.T / (fwd_ms * 1e-3),
            "tflops": flops["total"] / (fwd_ms * 1e-3) / 1e12,
            "sel_block_major_ms": bm_ms, "sel_query_tiled_ms": tiled_ms,
            "sel_block_major_tflops": flops["sel"] / (bm_ms * 1e-3) / 1e12}


def run_decode(dev, flush, stream, steps, peaks) -> dict:
    w = DECODE
    inp = W.make_decode_inputs(w, seed=0)
    kcache, vcache = inp["k_cache"].to(dev), inp["v_cache"].to(dev)
    pk = nsa.params_for(w)
    kc = torch.empty((w.B, w.Nc, w.Hkv, w.D), dtype=w.dtype, device=dev)
    vc = torch.empty_like(kc)
    nsa.nsa_compress(pk, kcache, vcache, kc, vc)
    p = nsa.params_for(w, Tq=1)
    q = inp["q"].to(dev).unsqueeze(1).contiguous()
    g = inp["gates"].to(dev).unsqueeze(1).contiguous()
    out = torch.empty_like(q)
    idx = torch.empty((w.B, 1, w.Hkv, w.topk), dtype=torch.int32, device=dev)
    ws = nsa.alloc_workspace(p, dev)

    def step():
        nsa.nsa_decode(p, q, kcache, vcache, kc, vc, g, out, idx, ws)

    for _ in range(3):
        step()
    us = statistics.mean(timed_steps(step, steps, flush, stream)) * 1e3
    # algorithmic bytes: q, gates, out, the whole compressed cache, and the
    # union of selected-block keys and window keys (K and V) per sequence
    ii = idx.cpu().numpy()
    t = w.T - 1
    keys = 0
    for b in range(w.B):
        for g_ in range(w.Hkv):
            s = set()
            for j in ii[b, 0, g_]:
                if j >= 0:
                    s.update(range(j * w.sel_block, min(j * w.sel_block + w.sel_block, t + 1)))
            s.update(range(max(0, t - w.window + 1), t + 1))
            keys += len(s)
    es = 2
    bytes_ = (w.B * w.Hq * w.D * es * 2 + w.B * w.Hq * 3 * 4
              + w.B * w.Nc * w.Hkv * w.D * es * 2 + keys * w.D * es * 2)
    gbs = bytes_ / (us * 1e-6) / 1e9
    return {"workload": w.name, "us_per_step": us, "algorithmic_bytes": bytes_,
            "gbs": gbs, "peak_gbs": peaks["hbm_gbs"], "frac": gbs / peaks["hbm_gbs"],
            "tokens_per_s": w.B / (us * 1e-6)}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="nsa", choices=["nsa", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--leg", default="all",
                    choices=["all", "forward", "decode", "train", "long", "onep3b", "moba",
                             "selbwd", "mlp", "pruned"],
                    help="forward / decode / train / long / onep3b / moba / selbwd / mlp / pruned: run only that leg on one GPU "
                         "and print its numbers (for profiling that leg alone); all: the "
                         "benchmark")
    ap.add_argument("--batch", type=int, default=None,
                    help="--leg train / selbwd only: batch size instead of 8 (a smaller case "
                         "of the same kernels, for profiling)")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.leg not in ("all", "forward"):
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        nsa.load()
        flush, stream, peaks = Flusher(dev), torch.cuda.current_stream(), load_peaks()
        if args.leg == "decode":
            print(json.dumps({"decode": run_decode(dev, flush, stream, args.steps, peaks)}))
        elif args.leg == "long":
            print(json.dumps({"long_context": run_long(dev, flush, stream, args.steps, peaks)}))
        elif args.leg == "selbwd":
            print(json.dumps({"sel_bwd_two_pass_vs_atomic": run_sel_bwd_compare(
                dev, flush, stream, args.steps, peaks,
                batch=args.batch if args.batch else 8)}))
        elif args.leg == "moba":
            print(json.dumps({"moba": run_moba(dev, flush, stream, args.steps, peaks)}))
        elif args.leg == "mlp":
            print(json.dumps({"mlp_compression": run_mlp(dev, flush, stream, args.steps, peaks)}))
        elif args.leg == "pruned":
            print(json.dumps({"pruned_branches": run_pruned(dev, flush, stream, args.steps, peaks)}))
        elif args.leg == "onep3b":
            print(json.dumps({"nsa_1p3b": run_1p3b(dev, flush, stream, args.steps, peaks)}))
        else:
            print(json.dumps({"train": run_train(dev, flush, stream, args.steps, peaks,
                                                 batch=args.batch)}))
        return
    dist_on = world > 1
    if dist_on:
        import datetime
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_gpu(args, rank, world, dist_on)
    finally:
        if dist_on:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
