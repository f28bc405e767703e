"""Benchmark of the mask-aware attention hot path on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
for each mask of the workload, the tile metadata pass, the forward and the
backward; plus one clip-shift-max localization of the first mask's vectors to
8 simulated context-parallel ranks (dual-chunk assignment) and their KV-chunk
pair counts.

Default workload (N=1): n = 131072, B = 1, H = 16, D = 128, bf16, Q/K/V/dO ~
N(0,1), the sweep of 12 seeded structured masks (full, causal, sliding window
2K and 8K, causal and bidirectional documents, prefix-LM, prefix-LM documents,
share-question, causal blockwise, global + sliding window, random eviction),
forward and backward timed per mask.  --config n8192 | n32768 select the
smaller workloads (two masks each).

Metric: effective TFLOP/s counting only unmasked score entries
(forward 4*D*U, backward 10*D*U per (b, h), U = unmasked (i, j) pairs).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                       [--config n131072|n32768|n8192] [--masks a,b,...]
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "mask-aware attn effective TFLOPs fwd/bwd (unmasked FLOPs), % of BF16 peak"
UNIT = "TFLOP/s"
L2_FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="n131072", choices=["n131072", "n32768", "n8192"])
    ap.add_argument("--masks", default=None, help="comma list of mask names (default: the config's)")
    ap.add_argument("--heads", type=int, default=None,
                    help="override the config's head count (small ncu captures; the bench line then names it)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch the phases eagerly instead of graph replays")
    ap.add_argument("--no-aux", action="store_true", help="skip the batched integer-pass measurement")
    ap.add_argument("--aux-only", action="store_true",
                    help="run only the batched integer-pass measurement (N=262144 localization and KV-chunk "
                         "pairs, 16-head metadata) and print its JSON; not a bench line (profiling runs)")
    return ap.parse_args()


# ----------------------------------------------------------------------------- workload
def workload(config: str, rank: int, masks_arg=None, heads=None):
    if config == "n8192":
        n, B, H, D = 8192, 2, 16, 128
        masks = ["sliding_window_1024", "causal_document_512_4096"]
        desc = "n=8192 B=2 H=16 D=128 bf16; masks: causal sliding window w=1024, causal documents L~U[512,4096]"
    elif config == "n32768":
        n, B, H, D = 32768, 1, 32, 128
        masks = ["prefix_lm", "share_question"]
        desc = "n=32768 B=1 H=32 D=128 bf16; masks: prefix-LM, share-question"
    else:
        n, B, H, D = 131072, 1, 16, 128
        masks = list(synth.SWEEP_FAMILIES)
        desc = ("n=131072 B=1 H=16 D=128 bf16; 12-mask sweep: full, causal, sliding window 2K, sliding window 8K, "
                "causal documents, bidirectional documents, prefix-LM, prefix-LM documents, share-question, "
                "causal blockwise 64, global + sliding window, random eviction")
    if masks_arg:
        masks = masks_arg.split(",")
        desc = desc.split(";")[0] + "; masks: " + ", ".join(masks)
    if heads:
        desc = desc.replace(f"H={H} ", f"H={heads} ", 1)
        H = heads
    cfg_id = {"n8192": 2, "n32768": 3, "n131072": 4}[config]
    specs = []
    for m_idx, name in enumerate(masks):
        rows = []
        for b in range(B):
            seed = 1000 * cfg_id + 10 * b + m_idx + 100000 * rank
            if name == "sliding_window_1024":
                s = synth.mask_sliding_window(n, 1024)
            elif name == "causal_document_512_4096":
                s = synth.mask_causal_document(n, synth.draw_docs(synth.Rng(seed), n, 512, 4096))
            else:
                s = synth.make_family(name, n, seed)
            rows.append(s)
        specs.append((name, rows))
    return dict(n=n, B=B, H=H, D=D, masks=specs, desc=desc, seed=1000 * cfg_id + 100000 * rank)


def workload_config(wl, world):
    """The `config` keys both arms report for a workload."""
    return {"workload": wl["desc"], "B": wl["B"], "H": wl["H"], "seq_len": wl["n"], "head_dim": wl["D"],
            "masks": [m for m, _ in wl["masks"]],
            "unmasked_pairs_per_head": [unmasked_pairs(specs, wl["n"]) for _, specs in wl["masks"]],
            "localize": "8 simulated ranks, dual-chunk, 16 chunks", "parallelism": f"replicas x{world}"}


def unmasked_pairs(spec_rows, n):
    """U per batch row from interval lengths (plain per-column count)."""
    out = []
    for s in spec_rows:
        lts, lte, uts, ute = (x.astype(np.int64) for x in s.vectors())
        a0, a1 = np.clip(lts, 0, n), np.clip(lte, 0, n)
        b0, b1 = np.clip(uts, 0, n), np.clip(ute, 0, n)
        la, lb = np.maximum(a1 - a0, 0), np.maximum(b1 - b0, 0)
        ov = np.maximum(np.minimum(a1, b1) - np.maximum(a0, b0), 0) * ((la > 0) & (lb > 0))
        out.append(int(np.sum(n - (la + lb - ov))))
    return out


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event reasons of this process's GPU during the timed region, read (never
    set) through NVML every ~5 ms from a thread; the device is found by its PCI bus id.  Falls back
    to an `nvidia-smi -lms 200` stream when NVML is unavailable."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, dev_index):
        self.dev = dev_index
        self.proc = self.thread = None
        self.samples, self.lines, self.max_mhz = [], [], None

    def _nvml_start(self):
        import threading

        import pynvml
        import torch
        pynvml.nvmlInit()
        pr = torch.cuda.get_device_properties(self.dev)
        bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
        h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
        bits = [pynvml.nvmlClocksEventReasonHwSlowdown, pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                pynvml.nvmlClocksEventReasonSwThermalSlowdown, pynvml.nvmlClocksEventReasonSwPowerCap]
        self.stop = threading.Event()

        def run():
            while True:
                try:
                    mhz = float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                    rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.samples.append((mhz, [n for n, bit in zip(self.NAMES, bits) if rs & bit]))
                except Exception:
                    pass
                if self.stop.wait(0.005):
                    break

        self.thread = threading.Thread(target=run, daemon=True)
        self.thread.start()

    def __enter__(self):
        try:
            self._nvml_start()
        except Exception:
            self.thread = None
            try:
                self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.Q}",
                                              "--format=csv,noheader,nounits", "-lms", "200"],
                                             stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except Exception:
                self.proc = None
        return self

    def __exit__(self, *a):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            for ln in out.splitlines():
                f = [x.strip() for x in ln.split(",")]
                if len(f) < 9:
                    continue
                try:
                    self.samples.append((float(f[1]), [n for k, n in enumerate(self.NAMES)
                                                       if f[5 + k].lower().startswith("active")]))
                    self.max_mhz = float(f[2])
                except ValueError:
                    continue

    def summary(self):
        sm = [x for x, _ in self.samples]
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"]}
        reasons = sorted({r for _, rs in self.samples for r in rs})
        load = [x for x in sm if x > 0.5 * (self.max_mhz or max(sm))] or sm
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(sm), "source": "nvml" if self.thread is not None else "nvidia-smi"}


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["bf16_tflops"], p.get("bf16_tflops_sustained"), p["hbm_gbs"], "measured"
    except Exception:
        return 1590.0, 1400.0, 6650.0, "fallback"


KERNEL_SOURCES = {  # the files whose device code each timed kernel is built from
    "bwd_kernel": ["mask_aware_flash_b200/csrc/fm_bwd.cu", "mask_aware_flash_b200/csrc/fm_common.cuh", "include/fm.h"],
    "fwd_kernel": ["mask_aware_flash_b200/csrc/fm_fwd.cu", "mask_aware_flash_b200/csrc/fm_common.cuh", "include/fm.h"],
}


def source_hash(kernel: str) -> str:
    """Hash of the sources a kernel is built from (a committed traffic figure is valid for it)."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, config: str):
    """DRAM bytes per launch from a committed ncu summary, if it matches the kernel's current sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        e = t[config][kernel]
        return e["bytes_per_launch"] if e.get("source_hash") == source_hash(kernel) else None
    except Exception:
        return None


# ----------------------------------------------------------------------------- CPU oracle baseline
def cpu_baseline(wl, budget_s=15.0):
    """The oracle as it stands, on the host cores: sampled query rows of head (0, 0), one mask per
    call in turn.  For each unmasked pair of those rows the oracle runs the forward (score, O: 4*D
    FLOPs in the effective count) and the dQ half of the backward (dP, dQ: 4*D of the backward's
    10*D); it runs no dK / dV column work here, so it is credited 8*D FLOPs per pair, the FLOPs it
    actually ran."""
    import oracle
    n, B, H, D = wl["n"], wl["B"], wl["H"], wl["D"]
    scale = 1.0 / math.sqrt(D)
    # inputs of the sampled heads only (the oracle reads q/k/v/do of (b, h))
    q = synth.bf16_bits_to_f32(synth.normal_bf16_bits(wl["seed"], 1, (1, n, 1, D)))
    k = synth.bf16_bits_to_f32(synth.normal_bf16_bits(wl["seed"], 2, (1, n, 1, D)))
    v = synth.bf16_bits_to_f32(synth.normal_bf16_bits(wl["seed"], 3, (1, n, 1, D)))
    do = synth.bf16_bits_to_f32(synth.normal_bf16_bits(wl["seed"], 4, (1, n, 1, D)))
    rows_per_call = 128
    done_pairs, t_used, calls = 0, 0.0, 0
    rng = synth.Rng(wl["seed"] + 7)
    while t_used < budget_s and calls < 100000:
        name, specs = wl["masks"][calls % len(wl["masks"])]
        s = specs[0]
        rows = np.array(rng.sample_distinct(0, n - 1, rows_per_call), np.int32)
        vecs = [x[None, None] for x in s.vectors()]
        allowed_rows = 0
        for i in rows:  # unmasked pairs of the sampled rows (interval test per key, vectorised)
            lts, lte, uts, ute = s.vectors()
            m = ((lts <= i) & (i < lte)) | ((uts <= i) & (i < ute))
            allowed_rows += int(n - m.sum())
        t0 = time.perf_counter()
        oracle.attention_head(q, k, v, vecs, 0, 0, scale, rows=rows, dout=do)
        t_used += time.perf_counter() - t0
        done_pairs += allowed_rows
        calls += 1
    flops = 8.0 * D * done_pairs
    return {"value": flops / t_used / 1e12, "unit": UNIT, "cores": oracle.max_threads(), "kind": "oracle",
            "sample": f"{calls} oracle calls x {rows_per_call} sampled query rows (forward + dQ, fp64) of head (0,0), "
                      f"the workload's masks in turn, {done_pairs} unmasked pairs in {t_used:.1f} s; "
                      f"effective FLOPs = 8*D*pairs (forward 4*D + the dQ half of the backward 4*D)"}


# ----------------------------------------------------------------------------- ranks
def reduce_max(values, world, device):
    """Element-wise maximum over all ranks (device time of the slowest rank)."""
    import torch
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_tflops(world, flops_per_rank_step, steps, max_ms):
    """Whole-job throughput: every rank processes its own replica's work in the slowest rank's time."""
    return world * flops_per_rank_step * steps / (max_ms * 1e-3) / 1e12


# ----------------------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    import torch
    import mask_aware_flash_b200 as fm
    from mask_aware_flash_b200 import _build
    _build.build()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = workload(args.config, rank, args.masks, args.heads)
    n, B, H, D = wl["n"], wl["B"], wl["H"], wl["D"]
    scale = 1.0 / math.sqrt(D)

    def bf16(t_id):
        bits = synth.normal_bf16_bits(wl["seed"], t_id, (B, n, H, D))
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)

    host = {name: bf16(t).pin_memory() for name, t in (("q", 1), ("k", 2), ("v", 3), ("do", 4))}
    q, k, v, do = (host[x].to(dev) for x in ("q", "k", "v", "do"))
    vec_host, vec_dev = [], []
    for name, specs in wl["masks"]:
        vs = [torch.from_numpy(np.stack([s.vectors()[c] for s in specs])[:, None, :].copy()).pin_memory()
              for c in range(4)]
        vec_host.append(vs)
        vec_dev.append([x.to(dev) for x in vs])
    # dual-chunk assignment of 16 chunks to 8 simulated ranks
    nch = 16
    chunk = n // nch
    loc_starts = [[r * chunk, (nch - 1 - r) * chunk] for r in range(nch // 2)]
    loc_lens = [[chunk, chunk]] * (nch // 2)
    U = [unmasked_pairs(specs, n) for _, specs in wl["masks"]]
    fwd_flops_m = [sum(4.0 * D * u * H for u in us) for us in U]
    bwd_flops_m = [sum(10.0 * D * u * H for u in us) for us in U]
    flops_fwd, flops_bwd = sum(fwd_flops_m), sum(bwd_flops_m)

    stream = torch.cuda.current_stream()
    o = torch.empty_like(q)
    lse = torch.empty((B, H, n), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    bws = torch.empty(fm.fm_attn_bwd_workspace_bytes(q, k, v), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731

    n_loc = [sum(x) for x in loc_lens]
    nm = len(wl["masks"])

    def build_phases(bs):
        """The step over one buffer set, as an ordered list of phases (kind, mask index, callable,
        kernel launches): localization of the simulated ranks, their KV-chunk pair counts, then
        metadata, forward and backward per mask."""
        bs["last"], bs["state"] = {"meta": [None] * nm}, {}
        last, state, vd = bs["last"], bs["state"], bs["vec"]

        def p_loc():
            state["loc"] = fm.fm_localize([vd[0][c] for c in range(4)], loc_starts, loc_lens)

        def p_kv():
            last["pairs"] = fm.fm_kv_chunk_pairs(state["loc"], n_loc, chunk)

        ph = [("localize", -1, p_loc, 1), ("kv_chunk_pairs", -1, p_kv, 1)]
        for mi in range(nm):
            def p_meta(mi=mi):
                last["meta"][mi] = fm.fm_build_mask_meta(*vd[mi], n_q=n)

            def p_fwd(mi=mi):
                fm.fm_attn_fwd(bs["q"], bs["k"], bs["v"], last["meta"][mi], vd[mi], scale, o=bs["o"], lse=bs["lse"])

            def p_bwd(mi=mi):
                fm.fm_attn_bwd(bs["q"], bs["k"], bs["v"], bs["o"], bs["lse"], bs["do"], last["meta"][mi], vd[mi], scale,
                               dq=bs["dq"], dk=bs["dk"], dv=bs["dv"], ws=bws)
            ph += [("meta", mi, p_meta, fm.META_LAUNCHES), ("fwd", mi, p_fwd, 1), ("bwd", mi, p_bwd, fm.BWD_LAUNCHES)]
        return ph

    def capture(ph):
        """Each phase in its own CUDA graph (the host cost of the ctypes calls and output allocations
        would otherwise leave the GPU idle between the small kernels); eager launches if capture fails."""
        if args.no_graph:
            return [x[2] for x in ph], False
        try:
            graphs = []
            for x in ph:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    x[2]()
                graphs.append(g)
            for g in graphs:  # one replay of the whole step before timing
                g.replay()
            torch.cuda.synchronize()
            return [g.replay for g in graphs], True
        except Exception as exc:  # keep the eager launches (same kernels)
            print(f"bench: graph capture failed ({exc}); timing eager launches", file=sys.stderr)
            return [x[2] for x in ph], False

    bs0 = dict(q=q, k=k, v=v, do=do, o=o, lse=lse, dq=dq, dk=dk, dv=dv, vec=vec_dev)
    phases = build_phases(bs0)
    last = bs0["last"]
    launches_per_step = sum(x[3] for x in phases)

    import torch.distributed as dist
    for _ in range(args.warmup):
        for x in phases:
            x[2]()
    torch.cuda.synchronize()
    runners, graphs_used = capture(phases)
    if world > 1:
        dist.barrier()

    def step(evs=None):
        for i, run in enumerate(runners):
            run()
            if evs is not None:
                evs[i + 1].record(stream)
        return launches_per_step

    step_ev = [[ev() for _ in range(len(phases) + 1)] for _ in range(args.steps)]
    launches = 0
    with ClockSampler(local_rank) as clk:
        torch.cuda.synchronize()
        for s in range(args.steps):
            flush.fill_(s & 0xFF)  # L2 flush between steps, outside the step events
            step_ev[s][0].record(stream)
            launches += step(step_ev[s])
        torch.cuda.synchronize()
    step_ms = [step_ev[s][0].elapsed_time(step_ev[s][-1]) for s in range(args.steps)]

    def phase_ms(kind, mi=None):
        return sum(step_ev[s][i].elapsed_time(step_ev[s][i + 1]) for s in range(args.steps)
                   for i, ph in enumerate(phases) if ph[0] == kind and (mi is None or ph[1] == mi))

    steps = args.steps
    per_mask_ms = [[phase_ms("fwd", mi), phase_ms("bwd", mi), phase_ms("meta", mi)] for mi in range(nm)]
    meta_ms = phase_ms("meta")
    loc_ms, kvc_ms = phase_ms("localize"), phase_ms("kv_chunk_pairs")
    flat = [sum(step_ms)] + [x for row in per_mask_ms for x in row[:2]]
    flat = reduce_max(flat, world, dev)  # slowest rank, per quantity
    total_ms = flat[0]
    per_mask_ms = [[flat[1 + 2 * mi], flat[2 + 2 * mi], per_mask_ms[mi][2]] for mi in range(nm)]
    fwd_ms = sum(x[0] for x in per_mask_ms)
    bwd_ms = sum(x[1] for x in per_mask_ms)
    value = job_tflops(world, flops_fwd + flops_bwd, steps, total_ms)

    e2e = None if args.no_e2e else run_e2e(fm, torch, dev, stream, wl, host, vec_host, scale, bws, steps,
                                             2, world, flops_fwd + flops_bwd)
    assert fm.fm_get_device_status() == 0, "device-side timeout during the bench"

    burst, sustained, hbm, src = peaks()

    def bw(nbytes, ms_total, calls):
        us = ms_total * 1e3 / calls
        gbs = nbytes / (us * 1e-6) / 1e9
        return {"us_per_launch": round(us, 2), "algorithmic_bytes": int(nbytes), "gbs": round(gbs, 1),
                "frac_of_hbm": round(gbs / hbm, 4)}

    # algorithmic bytes of the integer passes (untimed bookkeeping after the timed region)
    T = n // 128
    meta_bytes = 0
    for mt in last["meta"]:
        ent = int(mt.row_count.sum().item() + mt.col_count.sum().item())
        meta_bytes += B * (16 * n + 32 * T + T * T + 8 * T + 4 * (T // 2 + T)) + 4 * ent
    meta_bytes /= nm
    R = len(loc_starts)
    pairs = last["pairs"]
    rank_work = pairs.sum(dim=(1, 2, 3)).double()
    integer_passes = {
        "meta": dict(bw(meta_bytes, meta_ms, steps * nm), note="one fm_build_mask_meta call per mask"),
        "localize": dict(bw(16 * B * n * (1 + R), loc_ms, steps), ranks=R),
        "kv_chunk_pairs": dict(bw(16 * B * n * R + 8 * pairs.numel(), kvc_ms, steps), ranks=R,
                               chunks_pruned=int((pairs == 0).sum().item()), chunks=int(pairs.numel()),
                               rank_work_max_over_mean=round(float(rank_work.max() / rank_work.mean()), 4)),
        "batched_n262144_r16": None if args.no_aux else aux_localize(fm, torch, dev, stream, hbm),
    }
    fwd_tf = flops_fwd * steps / (fwd_ms * 1e-3) / 1e12
    bwd_tf = flops_bwd * steps / (bwd_ms * 1e-3) / 1e12
    long_step = total_ms / steps > 200.0  # seconds-long loops run under the power cap
    peak = sustained if (long_step and sustained) else burst
    peak_name = "sustained" if peak == sustained and long_step else "burst"

    def frac(tf):
        return {"effective_tflops": round(tf, 2), "frac_of_2250_nominal": round(tf / 2250.0, 4),
                "frac_of_measured_burst": round(tf / burst, 4),
                "frac_of_measured_sustained": round(tf / sustained, 4) if sustained else None}

    masks_out = []
    for mi, (name, _) in enumerate(wl["masks"]):
        f_ms, b_ms, m_ms = per_mask_ms[mi]
        masks_out.append({"mask": name, "unmasked_pairs_per_head": U[mi],
                          "fwd_ms": round(f_ms / steps, 4), "bwd_ms": round(b_ms / steps, 4),
                          "meta_ms": round(m_ms / steps, 4),
                          "fwd": frac(fwd_flops_m[mi] * steps / (f_ms * 1e-3) / 1e12),
                          "bwd": frac(bwd_flops_m[mi] * steps / (b_ms * 1e-3) / 1e12)})
    dominant = "bwd_kernel" if bwd_ms >= fwd_ms else "fwd_kernel"
    ach = bwd_tf if dominant == "bwd_kernel" else fwd_tf
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": round(total_ms / steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1), seeded masks)",
        "config": dict(workload_config(wl, world),
                       launch="one CUDA graph per phase, replayed" if graphs_used else "eager",
                       l2=f"flushed between steps ({L2_FLUSH_BYTES >> 20} MiB write outside the step events); "
                          f"inputs {4 * q.numel() * 2 >> 20} MiB > L2"),
        "fwd": dict(frac(fwd_tf), ms_per_step=round(fwd_ms / steps, 4)),
        "bwd": dict(frac(bwd_tf), ms_per_step=round(bwd_ms / steps, 4),
                    note=f"fm_attn_bwd phase: {fm.BWD_LAUNCHES} launches per call"),
        "per_mask": masks_out,
        "meta_ms_per_step": round(meta_ms / steps, 4),
        "integer_passes": integer_passes,
        "roofline": {"bound": "tensor", "kernel": dominant, "achieved": round(ach, 2), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(ach / peak, 4),
                     "peak_source": f"{src} bf16 {peak_name} (MEASURED_PEAKS.json)",
                     "traffic": traffic_for(dominant, args.config)},
        "e2e": e2e, "gpu_launches": launches, "clocks": clk.summary(),
    }
    return line, wl


def run_e2e(fm, torch, dev, stream, wl, host, vec_host, scale, bws, steps, warmup, world, flops_step):
    """End to end through the public API (eager calls, the ones a user makes) with host buffers: every
    step copies its inputs (Q, K, V, dO and every mask's vectors) from pinned host memory to the GPU,
    and every mask's results (O, LSE, dQ, dK, dV) back to pinned host memory.  Inputs are
    double-buffered per step (the inputs of step s+1 go up on one copy stream while step s computes)
    and outputs per mask (the results of mask m come back on another copy stream while mask m+1
    computes); events order every reuse of a buffer."""
    n, B, H = wl["n"], wl["B"], wl["H"]
    nm = len(wl["masks"])
    ins = [{x: torch.empty_like(host[x], device=dev) for x in host} for _ in range(2)]
    for s_ in ins:
        s_["vec"] = [[torch.empty_like(t, device=dev) for t in vs] for vs in vec_host]
    outs = [{x: torch.empty_like(ins[0]["q"]) for x in ("o", "dq", "dk", "dv")} for _ in range(2)]
    for o_ in outs:
        o_["lse"] = torch.empty((B, H, n), dtype=torch.float32, device=dev)
    out_host = [{x: torch.empty_like(outs[0][x], device="cpu").pin_memory() for x in outs[0]} for _ in range(2)]
    h2d = sum(host[x].numel() * 2 for x in host) + sum(t_.numel() * 4 for vs in vec_host for t_ in vs)
    d2h = nm * sum(t_.numel() * t_.element_size() for t_ in outs[0].values())
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    new_ev = torch.cuda.Event
    inputs_ready, inputs_free = [new_ev(), new_ev()], [new_ev(), new_ev()]
    mask_done, outputs_read = [new_ev(), new_ev()], [new_ev(), new_ev()]

    def upload(s_):
        bs = ins[s_ % 2]
        with torch.cuda.stream(up):
            if s_ >= 2:
                up.wait_event(inputs_free[s_ % 2])  # step s_-2 has finished reading this set
            for x in ("q", "k", "v", "do"):
                bs[x].copy_(host[x], non_blocking=True)
            for mi, vs in enumerate(vec_host):
                for c in range(4):
                    bs["vec"][mi][c].copy_(vs[c], non_blocking=True)
            inputs_ready[s_ % 2].record(up)

    def compute_and_download(s_):
        bs = ins[s_ % 2]
        stream.wait_event(inputs_ready[s_ % 2])
        for mi in range(nm):
            g = s_ * nm + mi
            ob, oh = outs[g % 2], out_host[g % 2]
            if g >= 2:
                stream.wait_event(outputs_read[g % 2])  # results of mask g-2 are home
            meta = fm.fm_build_mask_meta(*bs["vec"][mi], n_q=n)
            fm.fm_attn_fwd(bs["q"], bs["k"], bs["v"], meta, bs["vec"][mi], scale, o=ob["o"], lse=ob["lse"])
            fm.fm_attn_bwd(bs["q"], bs["k"], bs["v"], ob["o"], ob["lse"], bs["do"], meta, bs["vec"][mi], scale,
                           dq=ob["dq"], dk=ob["dk"], dv=ob["dv"], ws=bws)
            mask_done[g % 2].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(mask_done[g % 2])
                for x in ("o", "lse", "dq", "dk", "dv"):
                    oh[x].copy_(ob[x], non_blocking=True)
                outputs_read[g % 2].record(down)
        inputs_free[s_ % 2].record(stream)

    def pipeline(nsteps, e_start=None, e_end=None):
        torch.cuda.synchronize()
        if e_start is not None:
            e_start.record(stream)
            up.wait_event(e_start)
            down.wait_event(e_start)
        upload(0)
        for s_ in range(nsteps):
            if s_ + 1 < nsteps:
                upload(s_ + 1)
            compute_and_download(s_)
        stream.wait_event(outputs_read[(nsteps * nm - 1) % 2])
        stream.wait_event(outputs_read[(nsteps * nm - 2) % 2])
        if e_end is not None:
            e_end.record(stream)
        torch.cuda.synchronize()

    pipeline(warmup)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    pipeline(steps, e0, e1)
    (te_ms,) = reduce_max([e0.elapsed_time(e1)], world, dev)
    return {"value": job_tflops(world, flops_step, steps, te_ms), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "note": "eager API calls; inputs of step s+1 uploaded while step s computes, every mask's results "
                    "downloaded while the next mask computes"}


def aux_localize(fm, torch, dev, stream, hbm, reps=20):
    """The batched form of the integer passes at the localization workload's size: causal documents
    (L ~ U[4096, 65536]) over N = 262144 keys, 32 chunks of 8192 dealt to 16 simulated ranks (rank r
    gets chunks r and 31 - r), all ranks in one launch; then the per-rank KV-chunk pair counts."""
    N, nch = 262144, 32
    chunk, R = N // nch, nch // 2
    spec = synth.mask_causal_document(N, synth.draw_docs(synth.Rng(5000), N, 4096, 65536))
    vt = [torch.from_numpy(np.ascontiguousarray(x[None, None])).to(dev) for x in spec.vectors()]
    starts = [[r * chunk, (nch - 1 - r) * chunk] for r in range(R)]
    lens = [[chunk, chunk]] * R
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    loc = fm.fm_localize(vt, starts, lens)
    pairs = fm.fm_kv_chunk_pairs(loc, [2 * chunk] * R, chunk)
    g_loc, g_kv = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()  # reps back-to-back launches each
    with torch.cuda.graph(g_loc):
        for _ in range(reps):
            fm.fm_localize(vt, starts, lens, out=loc)
    with torch.cuda.graph(g_kv):
        for _ in range(reps):
            fm.fm_kv_chunk_pairs(loc, [2 * chunk] * R, chunk, out=pairs)
    g_loc.replay()
    g_kv.replay()
    torch.cuda.synchronize()
    ev[0].record(stream)
    g_loc.replay()
    ev[1].record(stream)
    g_kv.replay()
    ev[2].record(stream)
    torch.cuda.synchronize()
    out = {}
    for name, ms, nbytes in (("localize", ev[0].elapsed_time(ev[1]), 16 * N * (1 + R)),
                             ("kv_chunk_pairs", ev[1].elapsed_time(ev[2]), 16 * N * R + 8 * pairs.numel())):
        us = ms * 1e3 / reps
        gbs = nbytes / (us * 1e-6) / 1e9
        out[name] = {"us_per_launch": round(us, 2), "algorithmic_bytes": int(nbytes), "gbs": round(gbs, 1),
                     "frac_of_hbm": round(gbs / hbm, 4)}
    out["meta_hm16_n131072"] = aux_meta(fm, torch, dev, stream, hbm, reps)
    work = pairs.sum(dim=(1, 2, 3)).double()
    out["kv_chunk_pairs"].update(chunks_pruned=int((pairs == 0).sum().item()), chunks=int(pairs.numel()),
                                 rank_work_max_over_mean=round(float(work.max() / work.mean()), 4))
    # sparsity-aware assignment: per-chunk work from the same passes; dual-chunk, longest-first and
    # refined assignments against the bound set by the chunk granularity
    from mask_aware_flash_b200 import cp_balance as cb
    cost = cb.chunk_costs(fm, vt, chunk)
    out["balance"] = cb.balance_report(cost, R, 2)
    return out


def aux_meta(fm, torch, dev, stream, hbm, reps):
    """The metadata pass batched over mask heads: one fm_build_mask_meta call on 16 per-head masks
    (the 12 sweep masks and four more seeds of the first four) of n = 131072 keys, [1, 16, n] vectors
    (32 MiB).  Algorithmic bytes: the vectors read once; min/max, class matrix, both lists, their
    counts and both dispatch orders written once."""
    n, Hm = 131072, 16
    names = list(synth.SWEEP_FAMILIES) + list(synth.SWEEP_FAMILIES[:4])
    specs = [synth.make_family(nm, n, 6000 + i) for i, nm in enumerate(names[:Hm])]
    vt = [torch.from_numpy(np.stack([sp.vectors()[c] for sp in specs])[None].copy()).to(dev) for c in range(4)]
    meta = fm.fm_build_mask_meta(*vt, n_q=n)
    ws = meta.ws
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(reps):
            fm.fm_build_mask_meta(*vt, n_q=n, ws=ws)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / reps
    T = n // 128
    ent = int(meta.row_count.sum().item() + meta.col_count.sum().item())
    nbytes = Hm * (16 * n + 32 * T + T * T + 4 * (T + T) + 4 * (T // 2 + T)) + 4 * ent
    gbs = nbytes / (us * 1e-6) / 1e9
    return {"us_per_launch": round(us, 2), "algorithmic_bytes": int(nbytes), "gbs": round(gbs, 1),
            "frac_of_hbm": round(gbs / hbm, 4), "mask_heads": Hm, "launches_per_call": fm.META_LAUNCHES}


def run_reference(args):
    wl = workload(args.config, 0, args.masks, args.heads)
    cb = cpu_baseline(wl, budget_s=max(5.0, min(20.0, 3.0 * args.steps)))
    return {"metric": METRIC, "value": cb["value"], "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1), seeded masks)",
            "config": workload_config(wl, args.gpus), "impl": "reference", "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)))
        return
    if args.aux_only:
        import torch
        import mask_aware_flash_b200 as fm
        from mask_aware_flash_b200 import _build
        _build.build()
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        if rank == 0:
            print(json.dumps({"integer_passes_batched": aux_localize(fm, torch, dev, torch.cuda.current_stream(),
                                                                      peaks()[2])}))
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    line, wl = run_ours(args, rank, world, local_rank)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(wl)
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
