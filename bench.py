#!/usr/bin/env python
"""Benchmark of the attention-map-reuse hot path: prefill tokens/s for compress + retrieve at L=32K.

One step = one pass of the whole path over one synthetic layer of the L=32768 workload
(32 sender heads -> 64 receiver heads, d=128, bf16, block 128, p=0.9): block top-p compression of
every sender head's causal map (mr_compress) followed by the fused translated retrieval for every
receiver head (mr_retrieve).  value = tokens of all ranks / device time (max over ranks).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

For N > 1 it runs under torchrun, one rank per GPU; every rank compresses and retrieves its own
independent sequence (weak scaling, no data-path collective).  ``--impl reference`` times the fp64
CPU oracle on bounded samples of the same workload on the host cores (rank 0 only).
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
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from cross_model_attention_mr_b200.workloads import config, draw_batch, draw_layers, iter_layers, shrink  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "prefill tokens/s for compress+retrieve at L=32K; % TC peak and % HBM peak"


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------------------------------------
# clocks during the timed region
# ------------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: str):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", self.gpu], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def gpu_index_for(local_rank: int) -> str:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return str(local_rank)


# ------------------------------------------------------------------------------------------------
# algorithmic work of the path (what the method must do, independent of the implementation)
# ------------------------------------------------------------------------------------------------
def dense_causal_flops(H: int, d: int, d_v: int, first_pos: int, n_rows: int) -> int:
    """QK^T and PV flops of exact causal attention for rows at positions first_pos .. + n_rows - 1
    (row at position i sees i + 1 keys)."""
    keys = n_rows * first_pos + n_rows * (n_rows + 1) // 2
    return 2 * H * keys * (d + d_v)


def algorithmic(spec, nnz: int, union_tiles: int, n_req: int = 1, suffixes=None, fp8: bool = False):
    B, d, L = spec.block, spec.d, spec.L
    # bytes per stored tile: values (bf16, or e4m3 plus one fp32 scale per 32 x 64 piece) + column index
    tile_bytes = (B * B + 4 * (B // 32) * (B // 64) if fp8 else B * B * 2) + 4
    dense = 0
    if suffixes is not None:  # receiver heads' dense rows after the shared prefix
        dense = sum(dense_causal_flops(spec.H_r, d, spec.d_v, L, int(x)) for x in suffixes)
    return {
        "dense_flops": dense,
        # one causal QK^T per sender head: H_s * d * L * (L + 1) flops
        "compress_flops": spec.H_s * d * L * (L + 1),
        # the stored map: kept tiles of B*B probabilities plus one int32 column index each
        "map_bytes": nnz * tile_bytes,
        # translated map times V over the union of kept key blocks, per receiver head and request
        "retrieve_av_flops": spec.H_r * n_req * union_tiles * 2 * B * B * spec.d_v,
        # head mixing: each kept sender tile is weighted into every receiver head
        "retrieve_mix_flops": spec.H_r * nnz * 2 * B * B,
        # where the retrieval mixes heads: the library takes the tensor-core path for bf16 maps of
        # 128-key blocks with at most 32 sender heads and one request group of 4 receiver heads
        "mix_path": ("tensor" if (not fp8 and B == 128 and spec.H_s <= 32 and n_req < 2 and spec.dtype == "bf16")
                     else "cuda_core"),
    }


def mean_work(per_layer):
    """Layer mean of the algorithmic work dicts: numbers averaged, labels (the first layer's) kept."""
    return {k: (sum(w[k] for w in per_layer) / len(per_layer) if isinstance(v, (int, float)) else v)
            for k, v in per_layer[0].items()}


def kernel_work(name: str, work: dict):
    """(bound, amount, unit) of a kernel's algorithmic work per launch, against the roof the method
    names for its stage: the tensor-core peak for the contractions (QK^T in compression; the head
    mixing and X.V in retrieval), the HBM peak for writing the map."""
    if name in ("mr_compress_stats", "mr_compress_tc"):
        return "tensor", work["compress_flops"], "flop"
    if name in ("mr_emit", "mr_emit_tc"):
        return "hbm", work["map_bytes"], "byte"
    if name in ("mr_retrieve", "mr_retrieve_tc"):
        return "tensor", work["retrieve_av_flops"] + work["retrieve_mix_flops"], "flop"
    if name in ("mr_dense", "mr_dense_tc"):
        return "tensor", work.get("dense_flops", 0), "flop"
    return None, 0, None


def stage_rooflines(prof: dict, work: dict, pk: dict, sms: int):
    """Per launched kernel: algorithmic work / average launch time against the measured peaks
    (tensor: bf16 sustained; hbm: copy bandwidth).  The retrieval also reports its map bytes
    against HBM, and its head-mixing rate as a diagnostic of the implementation (not the method's
    roof): on the CUDA-core path against the cores' fp32 FMA rate."""
    out = {}
    tc_peak = float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"]))
    hbm_peak = float(pk["hbm_gbs"])
    for name, (ms, cnt) in prof.items():
        bound, amount, _ = kernel_work(name, work)
        if bound is None or cnt == 0 or amount == 0:
            continue
        avg_s = ms / cnt / 1e3
        e = {"ms_per_launch": ms / cnt, "bound": bound}
        if bound == "tensor":
            e.update(achieved_tflops=amount / avg_s / 1e12, peak_tflops=tc_peak,
                     frac=amount / avg_s / 1e12 / tc_peak)
        else:
            e.update(achieved_gbs=amount / avg_s / 1e9, peak_gbs=hbm_peak, frac=amount / avg_s / 1e9 / hbm_peak)
        if name in ("mr_retrieve", "mr_retrieve_tc"):
            e["map_gbs"] = work["map_bytes"] / avg_s / 1e9
            e["map_hbm_frac"] = e["map_gbs"] / hbm_peak
            if work.get("mix_path") == "tensor":
                e["diagnostic_mixing"] = {"achieved_tflops": work["retrieve_mix_flops"] / avg_s / 1e12,
                                          "path": "tensor core: mma.sync m16n8k16, bf16 in, fp32 accumulate",
                                          "note": "mixing rate over the whole launch; the launch is bound by "
                                                  "its L2 gather, not by this contraction"}
            else:
                fma_peak = sms * 128 * 2 * float(pk.get("sm_max_mhz", 1965.0)) * 1e6 / 1e12
                e["diagnostic_fp32_mixing"] = {"achieved_tflops": work["retrieve_mix_flops"] / avg_s / 1e12,
                                               "fp32_fma_peak_tflops": fma_peak,
                                               "note": "head mixing on CUDA cores; the roof of that choice"}
        out[name] = e
    return out


def roofline_of(name: str, ms: float, cnt: int, work: dict, pk: dict, pk_src: str):
    """The bench line's roofline object for one kernel (its stage's roof, see kernel_work)."""
    bound, amount, _ = kernel_work(name, work)
    avg_s = ms / cnt / 1e3
    if bound == "hbm":
        achieved, peak, runit, kind = amount / avg_s / 1e9, float(pk["hbm_gbs"]), "GB/s", "copy"
    else:
        achieved, runit, kind = amount / avg_s / 1e12, "TFLOP/s", "bf16 sustained"
        peak = float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"]))
    return {"bound": bound, "achieved": achieved, "peak": peak, "unit": runit, "frac": achieved / peak,
            "traffic": None, "kernel": name, "peak_source": pk_src, "peak_kind": kind}


def phase_split(stages: dict, tokens: float):
    """Per step of the headline workload (one retrieval launch per step): the time of the
    compression (statistics, scan, emit) and of the retrieval, and the retrieval-only rate, since
    a compressed prefix can serve several receivers."""
    comp_k = ("mr_compress_tc", "mr_emit_tc", "mr_scan_counts", "mr_compress_stats", "mr_emit")
    retr_k = ("mr_retrieve_tc", "mr_retrieve")
    comp = sum(v["ms_per_launch"] * v["launches"] for k, v in stages.items() if k in comp_k)
    retr = sum(v["ms_per_launch"] * v["launches"] for k, v in stages.items() if k in retr_k)
    n = sum(v["launches"] for k, v in stages.items() if k in retr_k)
    if not n or retr <= 0:
        return None
    return {"t_compress_ms": comp / n, "t_retrieve_ms": retr / n, "retrieve_only_tokens_per_s": tokens / (retr / n / 1e3)}


def source_hash(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, workload: str):
    """Per-launch DRAM bytes of `kernel` on `workload` from the committed ncu summary, if its
    sources are unchanged since the counters were taken (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            d = json.load(f)
        if d.get("workload") != workload:
            return None
        ent = d.get(kernel)
        if not ent:
            return None
        if source_hash(ent["sources"]) != ent["source_hash"]:
            return None
        return float(ent["bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


# ------------------------------------------------------------------------------------------------
# CPU oracle timing (baseline / reference arm)
# ------------------------------------------------------------------------------------------------
def oracle_sample_time(spec, lay, units_I, rows, threads):
    """Time the fp64 oracle on sampled compression units and retrieval rows and extrapolate to the
    full step by exact per-unit work.  Returns (full-step seconds, description)."""
    import oracle
    B, L = spec.block, spec.L
    nqb = L // B
    units = [int((k * 7) % spec.H_s) * nqb + int(I) for k, I in enumerate(units_I)]
    t0 = time.perf_counter()
    r = oracle.compress(lay.Q, lay.K, spec.scale, float(np.float32(spec.p)), B, lay.bias, units=units,
                        n_threads=threads)
    tc = time.perf_counter() - t0
    # work of a unit: B rows x (I+1)*B keys; total over all units of all heads
    w_sample = sum((I + 1) for I in units_I)
    w_total = spec.H_s * nqb * (nqb + 1) / 2
    t_compress = tc * w_total / w_sample
    kept = np.tril(np.ones((nqb, nqb), np.uint8))[None].repeat(spec.H_s, 0)
    for u in units:
        h, I = divmod(u, nqb)
        kept[h, I] = r.kept[h, I]
    t0 = time.perf_counter()
    oracle.retrieve_rows(lay.Q, lay.K, spec.scale, B, kept, lay.W, lay.V, np.asarray(rows), lay.bias,
                         n_threads=threads)
    tr = time.perf_counter() - t0
    t_retrieve = tr * (L * (L + 1) / 2) / sum(i + 1 for i in rows)
    desc = (f"{len(units)} compression units (h, I), I in [{min(units_I)}, {max(units_I)}], and "
            f"{len(rows)} retrieval rows i in [{min(rows)}, {max(rows)}] of the L={L} workload, "
            f"extrapolated by per-unit work ((I+1) key blocks per unit, (i+1) keys per row); "
            f"sample took {tc + tr:.1f} s (compress {tc:.1f} s, retrieve {tr:.1f} s)")
    return t_compress + t_retrieve, desc, tc + tr


def oracle_sample_calibrated(spec, lay, threads, target_s, rng):
    """One bounded oracle sample of about `target_s` seconds: a calibration pass with one unit and
    one row per thread, then units and rows (multiples of the thread count, so the pool stays full)
    scaled to the target.  Returns (full-step seconds, description)."""
    nqb = spec.L // spec.block

    def draw(n):
        return (rng.integers(nqb // 2, nqb, size=n).tolist(), rng.integers(spec.L // 2, spec.L, size=n).tolist())

    u, r = draw(threads)
    _, _, took = oracle_sample_time(spec, lay, u, r, threads)
    reps = int(max(1, min(64, round(target_s / max(took, 1e-3)))))
    u, r = draw(threads * reps)
    t_full, desc, _ = oracle_sample_time(spec, lay, u, r, threads)
    return t_full, desc


# ------------------------------------------------------------------------------------------------
# multi-rank host logic (one process per GPU; independent sequences, no data-path collective)
# ------------------------------------------------------------------------------------------------
def rank_spec(spec, rank: int):
    """Rank r processes its own sequence: the same workload drawn from seed + 7919 r."""
    if spec.seed is None or rank == 0:
        return spec
    from dataclasses import replace
    return replace(spec, seed=spec.seed + 7919 * rank)


def max_over_ranks(ms: float, dist, device) -> float:
    """Slowest rank's time (the job is done when every rank is)."""
    if dist is None:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def all_ranks_ok(ok: bool, dist, device) -> bool:
    """Every rank learns whether all ranks are fine, so an error path takes the same collective
    steps everywhere (no rank is left waiting in a later collective)."""
    if dist is None:
        return ok
    import torch
    t = torch.tensor([1 if ok else 0], dtype=torch.int32, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MIN)
    return bool(t.item())


def job_tokens_per_s(world: int, L: int, ms: float) -> float:
    """Whole-job throughput: every rank processed L tokens in the slowest rank's time."""
    return world * L / (ms / 1e3)


def line_config(spec, world: int) -> dict:
    """The `config` of the headline line; the reference arm prints the same dict."""
    return {"workload": spec.name, "L": spec.L, "H_s": spec.H_s, "H_r": spec.H_r, "d": spec.d,
            "d_v": spec.d_v, "block": spec.block, "p": spec.p, "layers": 1,
            "l2": "inputs larger than L2 (Q, K %d MB each, V %d MB, the map tens of GB)" % (
                spec.H_s * spec.L * spec.d * 2 // 10**6, spec.H_r * spec.L * spec.d_v * 2 // 10**6),
            "parallelism": f"replicas{world}"}


def run_reference(args, spec, rank):
    if rank != 0:
        return
    lay = draw_layers(spec)[0]
    threads = os.cpu_count() or 1
    nqb = spec.L // spec.block
    rng = np.random.default_rng(11)
    vals, took = [], []
    desc = ""
    for step in range(args.warmup + args.steps):
        if step < args.warmup:  # warm-up: one small pass (page-in, thread pool start)
            u, r = rng.integers(nqb // 2, nqb, size=threads).tolist(), rng.integers(spec.L // 2, spec.L, size=threads).tolist()
            oracle_sample_time(spec, lay, u, r, threads)
            continue
        t0 = time.perf_counter()
        t_full, desc = oracle_sample_calibrated(spec, lay, threads, 8.0, rng)
        took.append(time.perf_counter() - t0)
        vals.append(spec.L / t_full)
    value = float(statistics.median(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * spec.L / value,
        "ms_per_step_extrapolated": True,
        "sample_seconds_per_step": float(statistics.median(took)),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": line_config(spec, args.gpus),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": "per step: " + desc},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------------------
# measurement lines for the other workloads (one GPU; the headline line is the default, config 4)
# ------------------------------------------------------------------------------------------------
CONFIG_METRIC = {
    2: "prefill tokens/s for compress+retrieve, 1 layer, L=4K, 32 -> 40 heads, block 64",
    3: "prefill tokens/s for compress+retrieve summed over 28 layers, L=8K, 32 -> 28 heads, block 64",
    5: "prefill tokens/s: shared 4K prefix compressed once, retrieval for 16 requests, dense causal "
       "rows for their 512-2048-token suffixes",
}


def config_tokens_per_step(spec, suffixes=None) -> int:
    """Tokens one step processes: the sequence, or (config 5) every request's prefix + suffix."""
    if suffixes is None:
        return spec.L
    return int(sum(spec.L + int(x) for x in suffixes))


def run_config_line(args, spec, n):
    """One timed measurement line for workload n in {2, 3, 5} on one GPU (same JSON contract;
    end-to-end and CPU baseline are reported for the headline workload only)."""
    import torch
    from cross_model_attention_mr_b200 import mr
    torch.cuda.set_device(0)
    stream = torch.cuda.current_stream()
    bf = torch.bfloat16
    to_dev = lambda x: torch.from_numpy(x).to(bf).cuda().contiguous()  # noqa: E731
    p = float(np.float32(spec.p))
    cap = mr.max_tiles(spec.H_s, spec.L, spec.block)
    m = mr.Map(spec.H_s, spec.L, spec.block, mr.MR_BF16, cap, "cuda")
    ws_c = mr.Workspace(mr.compress_workspace_bytes(spec.H_s, spec.L, spec.d, spec.block))
    suffixes = None
    nqb = spec.L // spec.block
    if n in (2, 3):
        # layer by layer: each layer goes to the device before the next is drawn
        dev = [(to_dev(l.Q), to_dev(l.K), to_dev(l.V), torch.from_numpy(l.W).cuda(), mr.Bias.from_spec(l.bias))
               for l in iter_layers(spec)]
        ws_r = mr.Workspace(mr.retrieve_workspace_bytes(m, spec.H_r, spec.d_v, 1))
        O = torch.empty((1, spec.H_r, spec.L, spec.d_v), dtype=bf, device="cuda")
        wss = [ws_c, ws_r]

        def step():
            for Q, K, V, W, bias in dev:
                mr.compress(Q, K, p, spec.block, bias=bias, scale=spec.scale, out=m, ws=ws_c, stream=stream)
                mr.retrieve(m, W, V, out=O, ws=ws_r, stream=stream)

        def per_layer_maps():
            out = []
            for Q, K, V, W, bias in dev:
                mr.compress(Q, K, p, spec.block, bias=bias, scale=spec.scale, out=m, ws=ws_c, stream=stream)
                out.append((m.nnz_host(), int(np.any(m.kept_bits_host(), axis=0).sum())))
            return out
    else:
        b = draw_batch(spec)
        P, R = spec.L, spec.n_req
        suffixes = [r.suffix for r in b.requests]
        lens_k = [P + x for x in suffixes]
        cu_k = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
        cu_q = np.concatenate([[0], np.cumsum(suffixes)]).astype(np.int32)
        Qs, Ks = to_dev(b.Qs), to_dev(b.Ks)
        W = torch.from_numpy(b.W).cuda()
        bias_s = mr.Bias.from_spec(b.bias)
        bias_r = mr.Bias(b.bias.sink_len, b.bias.sink_bias, b.bias.window, b.bias.window_bias)
        Vp = to_dev(np.concatenate([r.V for r in b.requests], axis=1))        # [H_r][total_k][d_v]
        Kp = to_dev(np.concatenate([r.K for r in b.requests], axis=1))        # [H_r][total_k][d]
        Qsuf = to_dev(np.concatenate([r.Q[:, P:] for r in b.requests], axis=1))  # [H_r][total_q][d]
        off = torch.tensor(cu_k[:-1].astype(np.int64) * spec.d_v, dtype=torch.int64, device="cuda")
        cu_q_d, cu_k_d = torch.from_numpy(cu_q).cuda(), torch.from_numpy(cu_k).cuda()
        q_off = torch.full((R,), P, dtype=torch.int32, device="cuda")
        ws_r = mr.Workspace(mr.retrieve_workspace_bytes(m, spec.H_r, spec.d_v, R))
        ws_d = mr.Workspace(mr.LIB.mr_dense_ref_workspace_bytes(R))
        O_ret = torch.empty((R, spec.H_r, P, spec.d_v), dtype=bf, device="cuda")
        O_suf = torch.empty((spec.H_r, int(cu_q[-1]), spec.d_v), dtype=bf, device="cuda")
        wss = [ws_c, ws_r, ws_d]

        def step():
            mr.compress(Qs, Ks, p, spec.block, bias=bias_s, scale=spec.scale, out=m, ws=ws_c, stream=stream)
            mr.retrieve(m, W, Vp, out=O_ret, v_req_off=off, v_head_stride=int(cu_k[-1]) * spec.d_v, n_req=R,
                        ws=ws_r, stream=stream)
            mr.dense_ref(Qsuf, Kp, Vp, cu_q_d, cu_k_d, q_off, int(cu_q[-1]), int(cu_k[-1]), bias=bias_r,
                         scale=spec.scale, out=O_suf, ws=ws_d, stream=stream)

        def per_layer_maps():
            mr.compress(Qs, Ks, p, spec.block, bias=bias_s, scale=spec.scale, out=m, ws=ws_c, stream=stream)
            return [(m.nnz_host(), int(np.any(m.kept_bits_host(), axis=0).sum()))]

    maps = per_layer_maps()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if any(w.sync_status() for w in wss):
        raise SystemExit(f"device status after warm-up: {[w.sync_status() for w in wss]}")
    sampler = ClockSampler(gpu_index_for(0))
    sampler.start()
    time.sleep(0.3)
    launches0 = mr.kernel_launches()
    mr.profile_enable(True)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    prof = mr.profile_read()
    mr.profile_enable(False)
    launches = mr.kernel_launches() - launches0
    if any(w.sync_status() for w in wss):
        raise SystemExit(f"device status in the timed steps: {[w.sync_status() for w in wss]}")
    ms = ev0.elapsed_time(ev1) / args.steps
    tokens = config_tokens_per_step(spec, suffixes)
    n_req = spec.n_req if n == 5 else 1
    per_layer = [algorithmic(spec, nnz, un, n_req, suffixes) for nnz, un in maps]
    work = mean_work(per_layer)  # per launch, layer mean
    pk, pk_src = peaks()
    dname, (dms, dcnt) = max(prof.items(), key=lambda kv: kv[1][0])
    roofline = roofline_of(dname, dms, dcnt, work, pk, pk_src)
    roofline["traffic"] = None
    total = sum(v[0] for v in prof.values())
    stages = {k: {"ms_per_launch": v[0] / v[1], "launches": v[1], "share": v[0] / total} for k, v in prof.items()}
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for k, r in stage_rooflines(prof, work, pk, sms).items():
        stages[k].update(r)
    nnz_all = sum(x[0] for x in maps)
    tiles_all = len(maps) * spec.H_s * nqb * (nqb + 1) / 2
    line = {
        "metric": CONFIG_METRIC[n], "value": tokens / (ms / 1e3), "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": spec.name, "L": spec.L, "H_s": spec.H_s, "H_r": spec.H_r, "d": spec.d,
                   "block": spec.block, "p": spec.p, "layers": len(maps) if n == 3 else 1,
                   "requests": n_req, "tokens_per_step": tokens,
                   "l2": "inputs larger than L2 (maps %.2f GB per step)" % (nnz_all * spec.block ** 2 * 2 / 1e9),
                   "parallelism": "replicas1"},
        "gpu_launches": int(launches), "clocks": clocks, "roofline": roofline,
        "cpu_baseline": None, "e2e": None, "stages": stages,
        "map": {"nnz_tiles": nnz_all, "kept_fraction": nnz_all / tiles_all,
                "union_fraction": sum(x[1] for x in maps) / (len(maps) * nqb * (nqb + 1) / 2)},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------------------
# the retrieval's map reads alone (gather-only measurement)
# ------------------------------------------------------------------------------------------------
def run_gather_probe(args, spec):
    """Compress the workload once, then time mr_gather_probe: every stored tile moved to shared
    memory by 1 CTA (from DRAM) and by 16 CTAs side by side (the retrieval's re-read factor at 4
    receiver heads per CTA), with the retrieval's copy mechanism and no arithmetic."""
    import torch
    from cross_model_attention_mr_b200 import mr
    torch.cuda.set_device(0)
    stream = torch.cuda.current_stream()
    lay = draw_layers(spec)[0]
    bf = torch.bfloat16
    fp8 = args.map == "fp8"
    m = mr.compress(torch.from_numpy(lay.Q).to(bf).cuda(), torch.from_numpy(lay.K).to(bf).cuda(),
                    float(np.float32(spec.p)), spec.block, bias=mr.Bias.from_spec(lay.bias), scale=spec.scale,
                    map_dtype=mr.MR_FP8_E4M3 if fp8 else None)
    torch.cuda.synchronize()
    nnz = m.nnz_host()
    tile_bytes = spec.block * spec.block * (1 if fp8 else 2)
    pk, pk_src = peaks()
    ws = mr.Workspace(256)
    out = {}
    for readers in (1, 16):
        for slots in (8, 16, 24):
            for _ in range(args.warmup):
                mr.gather_probe(m, readers, ws, stream, slots)
            ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ev0.record(stream)
            for _ in range(args.steps):
                mr.gather_probe(m, readers, ws, stream, slots)
            ev1.record(stream)
            torch.cuda.synchronize()
            ms = ev0.elapsed_time(ev1) / args.steps
            gbs = readers * nnz * tile_bytes / (ms / 1e3) / 1e9
            out[f"{readers}x{slots}"] = {"readers": readers, "slots_per_thread": slots, "ms": ms, "GB/s": gbs,
                                         "hbm_frac": gbs / float(pk["hbm_gbs"])}
    line = {"metric": "map gather alone: stored tiles moved to shared memory, GB/s", "unit": "GB/s",
            "value": max(v["GB/s"] for v in out.values() if v["readers"] == 1), "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": True, "dtype": "fp8" if fp8 else "bf16", "data": "synthetic",
            "config": {"workload": spec.name, "map_tiles": nnz, "tile_bytes": tile_bytes,
                       "map_bytes": nnz * tile_bytes},
            "readers": out, "peak_gbs": float(pk["hbm_gbs"]), "peak_source": pk_src}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------------------
# one sequence split across ranks (strong scaling)
# ------------------------------------------------------------------------------------------------
def run_split(args, spec, dist, world: int, rank: int, local: int):
    """Each rank owns a contiguous, work-balanced range of query blocks and the token rows of that
    range.  A step all-gathers the ranks' K and V row shards (the path's one exchange), then
    compresses its query blocks and retrieves its output rows; maps and outputs stay local.
    value = L / (slowest rank's step time)."""
    import torch
    from cross_model_attention_mr_b200 import mr
    torch.cuda.set_device(local)
    stream = torch.cuda.current_stream()
    bf = torch.bfloat16
    lay = draw_layers(spec)[0]
    nqb = spec.L // spec.block
    ranges = mr.split_query_blocks(nqb, world, 1 if spec.block == 128 else 2)
    shards = mr.row_shards(spec.L, ranges, spec.block)
    q0, q1 = ranges[rank]
    b, e = shards[rank]
    Q = torch.from_numpy(lay.Q).to(bf).cuda()   # rows outside this rank's range are never read
    Kl = torch.from_numpy(np.ascontiguousarray(lay.K[:, b:e])).to(bf).cuda()
    Vl = torch.from_numpy(np.ascontiguousarray(lay.V[:, b:e])).to(bf).cuda()
    W = torch.from_numpy(lay.W).cuda()
    bias = mr.Bias.from_spec(lay.bias)
    p = float(np.float32(spec.p))
    m = mr.Map(spec.H_s, spec.L, spec.block, mr.MR_BF16, max(1, mr.max_tiles(spec.H_s, spec.L, spec.block)), "cuda")
    ws_c = mr.Workspace(mr.compress_workspace_bytes(spec.H_s, spec.L, spec.d, spec.block))
    ws_r = mr.Workspace(mr.retrieve_workspace_bytes(m, spec.H_r, spec.d_v, 1))
    O = torch.empty((1, spec.H_r, spec.L, spec.d_v), dtype=bf, device="cuda")

    def step():
        K = mr.gather_row_shards(Kl, shards) if world > 1 else Kl
        V = mr.gather_row_shards(Vl, shards) if world > 1 else Vl
        if q1 > q0:
            mr.compress(Q, K, p, spec.block, bias=bias, scale=spec.scale, out=m, ws=ws_c, stream=stream,
                        blocks=(q0, q1))
            mr.retrieve(m, W, V, out=O, ws=ws_r, stream=stream, blocks=(q0, q1))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ok = (q1 == q0) or not (ws_c.sync_status() or ws_r.sync_status())
    if not all_ranks_ok(ok, dist, "cuda"):
        raise SystemExit("device status after warm-up")
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1) / args.steps, dist, "cuda")
    ok = (q1 == q0) or not (ws_c.sync_status() or ws_r.sync_status())
    if not all_ranks_ok(ok, dist, "cuda"):
        raise SystemExit("device status in the timed steps")
    if rank == 0:
        line = {
            "metric": METRIC + " (one sequence split across ranks)", "value": spec.L / (ms / 1e3),
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(line_config(spec, world), parallelism=f"query-block split x{world}",
                           ranges=[list(r) for r in ranges]),
            "exchange": "all-gather of K and V row shards per step (torch.distributed)",
        }
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------------------
# native arm
# ------------------------------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--L", type=int, default=None,
                    help="shorter sequence of the same workload shape (profiling captures); default 32768")
    ap.add_argument("--gather-probe", action="store_true",
                    help="time the retrieval's map reads alone (mr_gather_probe) on the workload's map")
    ap.add_argument("--split", action="store_true",
                    help="split one sequence across the ranks by query-block range (strong scaling)")
    ap.add_argument("--map", default="bf16", choices=["bf16", "fp8"],
                    help="map value type: bf16 (default, the headline) or fp8 (e4m3 with per-piece scales)")
    ap.add_argument("--config", type=int, default=4, choices=[2, 3, 4, 5],
                    help="workload: 4 = the headline line (default); 2, 3, 5 = one-GPU measurement lines")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    spec = config(args.config)
    if args.L is not None and args.L != spec.L:
        name = spec.name.replace("L32768", f"L{args.L}") if "L32768" in spec.name else f"{spec.name}_at_L{args.L}"
        spec = shrink(spec, L=args.L, name=name)
    if args.gather_probe:
        run_gather_probe(args, spec)
        return
    if args.config != 4 and args.impl != "reference":
        if int(os.environ.get("WORLD_SIZE", "1")) > 1:
            raise SystemExit("--config 2/3/5 lines are one-GPU measurements")
        run_config_line(args, spec, args.config)
        return

    if args.impl == "reference":
        run_reference(args, spec, rank)
        return

    import torch
    from cross_model_attention_mr_b200 import mr

    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    if args.split:
        try:
            run_split(args, spec, dist, world, rank, local)
        finally:
            if dist is not None:
                dist.destroy_process_group()
        return
    spec = rank_spec(spec, rank)  # independent sequence per rank

    lay = draw_layers(spec)[0]
    bf = torch.bfloat16
    host = {
        "Q": torch.from_numpy(lay.Q).to(bf).pin_memory(),
        "K": torch.from_numpy(lay.K).to(bf).pin_memory(),
        "V": torch.from_numpy(lay.V).to(bf).pin_memory(),
        "W": torch.from_numpy(lay.W).pin_memory(),
    }
    Q, K, V, W = (host[k].cuda(non_blocking=True) for k in ("Q", "K", "V", "W"))
    bias = mr.Bias.from_spec(lay.bias)
    p = float(np.float32(spec.p))
    cap = mr.max_tiles(spec.H_s, spec.L, spec.block)
    fp8 = args.map == "fp8"
    m = mr.Map(spec.H_s, spec.L, spec.block, mr.MR_FP8_E4M3 if fp8 else mr.MR_BF16, cap, "cuda")
    ws_c = mr.Workspace(mr.compress_workspace_bytes(spec.H_s, spec.L, spec.d, spec.block))
    ws_r = mr.Workspace(mr.retrieve_workspace_bytes(m, spec.H_r, spec.d_v, 1))
    O = torch.empty((1, spec.H_r, spec.L, spec.d_v), dtype=bf, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        mr.compress(Q, K, p, spec.block, bias=bias, scale=spec.scale, out=m, ws=ws_c, stream=stream)
        mr.retrieve(m, W, V, out=O, ws=ws_r, stream=stream)

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st_c, st_r = ws_c.sync_status(), ws_r.sync_status()
    if not all_ranks_ok(not (st_c or st_r), dist, "cuda"):
        raise SystemExit(f"device status (this rank) compress={st_c} retrieve={st_r}")
    nnz = m.nnz_host()
    kept = m.kept_bits_host()
    nqb = spec.L // spec.block
    union_tiles = int(np.any(kept, axis=0).sum())
    work = algorithmic(spec, nnz, union_tiles, fp8=fp8)

    # ---- timed region (device time, CUDA events on the launching stream) ----
    sampler = ClockSampler(gpu_index_for(local))
    barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    launches0 = mr.kernel_launches()
    mr.profile_enable(True)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    prof = mr.profile_read()
    mr.profile_enable(False)
    launches = mr.kernel_launches() - launches0
    ms = ev0.elapsed_time(ev1) / args.steps
    st_c, st_r = ws_c.sync_status(), ws_r.sync_status()
    if not all_ranks_ok(not (st_c or st_r), dist, "cuda"):
        raise SystemExit(f"device status in the timed steps (this rank): compress={st_c} retrieve={st_r}")
    ms = max_over_ranks(ms, dist, "cuda")
    value = job_tokens_per_s(world, spec.L, ms)

    # ---- roofline of the dominant kernel, and of every stage ----
    pk, pk_src = peaks()
    dname, (dms, dcnt) = max(prof.items(), key=lambda kv: kv[1][0])
    roofline = roofline_of(dname, dms, dcnt, work, pk, pk_src)
    roofline["traffic"] = traffic_for(dname, spec.name + ("+fp8" if fp8 else ""))
    stages = {k: {"ms_per_launch": v[0] / v[1], "launches": v[1], "share": v[0] / sum(x[0] for x in prof.values())}
              for k, v in prof.items()}
    sms = torch.cuda.get_device_properties(local).multi_processor_count
    for k, r in stage_rooflines(prof, work, pk, sms).items():
        stages[k].update(r)

    # ---- end to end through the public API with host buffers ----
    # Every step copies its inputs from pinned host memory and reads its result back inside the
    # timed region.  Double-buffered: step k + 1's inputs go up on a copy stream and step k - 1's
    # output comes down on another while step k computes; the compute itself stays on one stream.
    # Q and K go up first: the compression needs only them, and the retrieval waits for V and W.
    e2e = None
    if not args.no_e2e:
        h2d = sum(host[k].numel() * host[k].element_size() for k in host)
        dev_bufs = [{"Q": Q, "K": K, "V": V, "W": W, "O": O},
                    {k: torch.empty_like(t) for k, t in (("Q", Q), ("K", K), ("V", V), ("W", W), ("O", O))}]
        Ohs = [torch.empty(O.shape, dtype=bf).pin_memory() for _ in range(2)]
        d2h = Ohs[0].numel() * Ohs[0].element_size()
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev = {name: [torch.cuda.Event() for _ in range(2)] for name in ("qk", "vw", "done", "out")}

        def e2e_steps(n):
            for k in range(n):
                b, d = k % 2, dev_bufs[k % 2]
                with torch.cuda.stream(s_in):
                    if k >= 2:
                        s_in.wait_event(ev["done"][b])  # step k - 2 has finished with this buffer
                    for name in ("Q", "K"):
                        d[name].copy_(host[name], non_blocking=True)
                    ev["qk"][b].record(s_in)
                    for name in ("V", "W"):
                        d[name].copy_(host[name], non_blocking=True)
                    ev["vw"][b].record(s_in)
                stream.wait_event(ev["qk"][b])
                if k >= 2:
                    stream.wait_event(ev["out"][b])  # step k - 2's output has been read back
                mr.compress(d["Q"], d["K"], p, spec.block, bias=bias, scale=spec.scale, out=m, ws=ws_c, stream=stream)
                stream.wait_event(ev["vw"][b])
                mr.retrieve(m, d["W"], d["V"], out=d["O"], ws=ws_r, stream=stream)
                ev["done"][b].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev["done"][b])
                    Ohs[b].copy_(d["O"], non_blocking=True)
                    ev["out"][b].record(s_out)

        e2e_steps(2)
        torch.cuda.synchronize()
        barrier()
        n_e2e = max(3, args.steps)  # the same step count as the device-timed run; the pipeline fills and drains once
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        e2e_steps(n_e2e)
        for b in range(2):
            s_out.wait_event(ev["out"][b])
        e1.record(s_out)
        torch.cuda.synchronize()
        st_c, st_r = ws_c.sync_status(), ws_r.sync_status()
        if not all_ranks_ok(not (st_c or st_r), dist, "cuda"):
            raise SystemExit(f"device status in the end-to-end steps (this rank): compress={st_c} retrieve={st_r}")
        ems = e0.elapsed_time(e1) / n_e2e
        ems = max_over_ranks(ems, dist, "cuda")
        e2e = {"value": job_tokens_per_s(world, spec.L, ems), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "ms_per_step": ems,
               "pipeline": ("inputs of step k+1 and output of step k-1 copied while step k computes; "
                            "a step's compression starts once its Q and K are up")}
        del dev_bufs

    # ---- what the receiver would otherwise run: dense causal attention of its 64 heads ----
    dense = None
    if not args.no_dense:
        import torch as _t
        cu = _t.tensor([0, spec.L], dtype=_t.int32, device="cuda")
        Qr = Q.repeat(2, 1, 1)[: spec.H_r].contiguous()  # receiver-shaped queries/keys (synthetic)
        Kr = K.repeat(2, 1, 1)[: spec.H_r].contiguous()
        Od = _t.empty_like(V)
        ws_d = mr.Workspace(mr.LIB.mr_dense_ref_workspace_bytes(1))
        mr.dense_ref(Qr, Kr, V, cu, cu, None, spec.L, spec.L, bias=None, scale=spec.scale, out=Od, ws=ws_d)
        _t.cuda.synchronize()
        d0, d1 = _t.cuda.Event(enable_timing=True), _t.cuda.Event(enable_timing=True)
        d0.record(stream)
        mr.dense_ref(Qr, Kr, V, cu, cu, None, spec.L, spec.L, bias=None, scale=spec.scale, out=Od, ws=ws_d)
        d1.record(stream)
        _t.cuda.synchronize()
        dms_ = d0.elapsed_time(d1)
        dfl = dense_causal_flops(spec.H_r, spec.d, spec.d_v, 0, spec.L)
        pkd, _ = peaks()
        dense = {"tokens_per_s": spec.L / (dms_ / 1e3), "ms": dms_, "heads": spec.H_r, "flops": dfl,
                 "achieved_tflops": dfl / (dms_ / 1e3) / 1e12,
                 "frac_of_bf16_burst": dfl / (dms_ / 1e3) / 1e12 / float(pkd["bf16_tflops"]),
                 "note": "exact causal attention of the receiver heads, one launch timed alone"}
        del Qr, Kr, Od

    # ---- CPU oracle baseline (rank 0, N = 1 only) ----
    cpu = None
    if not args.no_cpu_baseline and world == 1 and rank == 0:
        threads = os.cpu_count() or 1
        t_full, desc = oracle_sample_calibrated(spec, lay, threads, 15.0, np.random.default_rng(11))
        cpu = {"value": spec.L / t_full, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": desc}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded Gaussian Q/K/V, sink+window+retrieval-block logit bias, row-softmax W)",
            "config": dict(line_config(spec, world), **({"map_values": "fp8 e4m3, scale per 32 x 64 piece"} if fp8 else {})),
            "gpu_launches": int(launches),
            "clocks": clocks,
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "stages": stages,
            "map": {"nnz_tiles": nnz, "kept_fraction": nnz / (spec.H_s * nqb * (nqb + 1) / 2),
                    "union_fraction": union_tiles / (nqb * (nqb + 1) / 2)},
            "algorithmic": work,
            "dense_ref": dense,
            "phases": phase_split(stages, spec.L),
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
