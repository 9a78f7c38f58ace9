"""Benchmark: selected query-tokens/s of causal IVF route+refine on B200.

One step = the whole hot path over the last R/T prefill chunks of the
workload (one refit period): per chunk, append its keys, seal its windows
(the refit they trigger runs on the side stream) and route + refine its
queries; then publish the refit.  The index state before those chunks is
restored (checkpoint/rollback) between steps, and L2 is flushed between
steps.  Inputs are seeded synthetic data of the workload's shapes.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload glm_bf16_L128k]

N > 1 runs under torch.distributed.run: every rank holds an independent
request (its own seed) and runs the same step; no collective is on the data
path (weak scaling).  `--impl reference` times the float64 CPU oracle on the
host cores (rank 0 only) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from synth import workloads as S  # noqa: E402

METRIC = "selected query-tokens/s at 128K-1M prefix (route+refine) & recall vs exhaustive"
UNIT = "query-tokens/s"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default="glm_bf16_L128k", choices=sorted(S.WORKLOADS))
    p.add_argument("--refine-kernel", type=int, default=0, choices=[0, 1, 2, 3, 4],
                   help="force a tensor-core refine variant (0 = the library's choice)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--cpu-sample", type=int, default=48, help="queries timed per oracle step")
    p.add_argument("--budget", type=int, default=0, help="candidate budget C (0: the workload's)")
    p.add_argument("--refit-period", type=int, default=-1,
                   help="refit period R in keys (0: seal only, no refit; -1: the workload's)")
    p.add_argument("--routing", default="ivf", choices=["ivf", "blocks"],
                   help="ivf: the causal inverted-file index; blocks: the contiguous-block baseline "
                        "(blocks of W/m consecutive keys with mean representatives, no refit)")
    p.add_argument("--refit-overlap", action="store_true",
                   help="also time one refit (64 seeds from the last 16384 keys) alone, the route "
                        "alone and both together, and report the hidden fraction")
    p.add_argument("--exh-reps", type=int, default=10, help="timed exhaustive calls (after one warm-up)")
    p.add_argument("--no-exhaustive", dest="exhaustive", action="store_false",
                   help="skip recall and the exhaustive baseline (it holds up to 4 GiB of score rows)")
    p.add_argument("--decode", type=int, default=0,
                   help="also time N decode steps after the prefill (one key appended, one query "
                        "selected per step) with route+refine and with the exhaustive selection")
    p.add_argument("--mode", default="replicas", choices=["replicas", "sharded"],
                   help="N > 1: replicas = an independent request per rank (weak scaling); sharded = one "
                        "request, every rank rescoring its share of each candidate list, partial top-k "
                        "all-gathered over NCCL and merged (strong scaling)")
    p.add_argument("--no-1m", dest="with_1m", action="store_false",
                   help="skip the 1M-key sub-result of the default workload")
    return p.parse_args()


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), \
        int(os.environ.get("LOCAL_RANK", 0))


def chunks_per_step(wl):
    """A step spans one refit period (R / T chunks) so that it holds the
    refit the method runs every R tokens."""
    return max(1, wl.refit_period // wl.T) if wl.refit_period else 1


def config_block(wl, n, mode="replicas"):
    return {"workload": wl.name, "chunks_per_step": chunks_per_step(wl),
            "queries_per_step": chunks_per_step(wl) * wl.T, "prefix_tokens": wl.L, "chunk_queries": wl.T, "heads": wl.H,
            "head_dim": wl.d, "key_dtype": wl.key_dtype, "k": wl.k, "budget_C": wl.budget,
            "window_W": wl.window, "clusters_per_window": wl.clusters_per_window,
            "refit_period_R": wl.refit_period, "sinks": wl.n_sinks,
            "routing": "contiguous blocks (baseline)" if wl.block_routing else "ivf",
            "step": "last R/T chunks: per chunk append + seal (+side-stream refit) + route/refine; then publish",
            "l2": "flushed between steps (256 MiB write)",
            "parallelism": f"cluster-sharded rescore x{n}" if mode == "sharded" and n > 1 else f"replicas x{n}"}


def wl_for_rank(name, rank, budget=0, refit_period=-1, routing="ivf", sharded=False):
    """Every rank runs an independent request: same shapes, its own seed (or,
    sharded, the same request on every rank).  budget / refit_period /
    routing override the workload's (ablations)."""
    wl = S.scaled(S.WORKLOADS[name], seed=0 if sharded else rank)
    if budget:
        wl = S.scaled(wl, budget=budget)
    if routing == "blocks":
        wl = S.scaled(wl, block_routing=True, refit_period=0)
    elif refit_period >= 0:
        wl = S.scaled(wl, refit_period=refit_period)
    return wl


def max_over_ranks(x: float, device) -> float:
    """Max of a per-rank number over all ranks (identity without a group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank: int, steps: int, world: int, max_total_ms: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's timed device time."""
    return world * units_per_rank * steps / (max_total_ms / 1e3)


# ------------------------------------------------------------- inputs --

def bf16_dev(x, device):
    import torch
    bits = S.to_bf16_bits(x)
    return torch.from_numpy(bits.view(np.int16)).to(device).view(torch.bfloat16)


def chunk_keys_dev(wl, p0, p1, device):
    import torch
    kf = S.keys_f64(wl, p0, p1)
    if wl.key_dtype == "fp32":
        return torch.from_numpy(kf.astype(np.float32)).to(device), None
    kb = bf16_dev(kf, device)
    if wl.key_dtype == "bf16":
        return kb, None
    from ivf_top_key_b200 import quantize_fp8
    return quantize_fp8(kb)


def queries_dev(wl, p0, p1, device):
    import torch
    q, w = S.queries_f64(wl, p0, p1)
    wd = torch.from_numpy(w.astype(np.float32)).to(device)
    if wl.q_dtype == "fp32":
        return torch.from_numpy(q.astype(np.float32)).to(device), wd
    return bf16_dev(q, device), wd


# ------------------------------------------------------------- clocks --

class Clocks:
    """nvidia-smi sampling during the timed region."""

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"ai_bench_clocks_{os.getpid()}.csv")

    def __enter__(self):
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            self.proc.wait(timeout=10)
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return None
        rows = [r.split(",") for r in open(self.path).read().strip().splitlines() if r.strip()]
        try:
            os.remove(self.path)
        except OSError:
            pass
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = max(mx, float(r[2]))
                for nm, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(nm)
            except (ValueError, IndexError):
                continue
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------ roofline --

def measured_peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def traffic_from_profile(kernel_src: str, profile_md: str):
    """DRAM bytes per launch recorded by an ncu capture summary, if the
    kernel source has not changed since (sha256 prefix recorded there)."""
    try:
        txt = open(profile_md).read()
        src = open(kernel_src, "rb").read()
    except OSError:
        return None
    h = hashlib.sha256(src).hexdigest()[:16]
    m_h = re.search(r"source_sha256_16:\s*([0-9a-f]{16})", txt)
    m_t = re.search(r"dram_bytes_per_launch_fullsize:\s*([0-9.eE+]+)", txt)
    if not m_h or not m_t or m_h.group(1) != h:
        return None
    return float(m_t.group(1))


# ------------------------------------------------------------ our arm --

def l2_read_peak(dev, reps=20):
    """A plain L2-resident read: torch row sums over 16 stride-0 repeats of
    one 64 MiB fp32 buffer (1 GiB read per launch, so the launch cost does
    not weigh in; the buffer fits the 126 MB L2 but not L1), best of
    `reps`, read bytes.  The bound of a gather whose rows are served from
    L2.  (The same reduction over a 4 GiB buffer reads at the measured HBM
    copy rate.)"""
    import torch
    x = torch.ones(64 << 18, dtype=torch.float32, device=dev)
    v = x.unsqueeze(0).expand(16, -1)
    out = torch.empty(16, dtype=torch.float32, device=dev)
    for _ in range(3):
        torch.sum(v, dim=1, out=out)
    best = float("inf")
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        torch.sum(v, dim=1, out=out)
        e1.record()
        e1.synchronize()
        best = min(best, e0.elapsed_time(e1))
    return 16 * x.numel() * 4 / (best / 1e3) / 1e9


def build_index(wl, args, dev):
    """The workload's index up to the timed chunks (untimed setup), its
    checkpoint, and the timed chunks' inputs on the device."""
    from ivf_top_key_b200 import AttentionIndex
    T, L = wl.T, wl.L
    ncs = chunks_per_step(wl)
    p_first = L - ncs * T
    idx = AttentionIndex(d=wl.d, H=wl.H, key_dtype=wl.key_dtype, q_dtype=wl.q_dtype,
                         n_sinks=wl.n_sinks, window=wl.window,
                         clusters_per_window=wl.clusters_per_window,
                         refit_period=wl.refit_period, refit_new_seeds=0,
                         refit_seed_window=0, seal_iters=wl.seal_iters, async_refit=True,
                         max_query_chunk=T, max_budget=wl.budget, max_k=wl.k, max_keys=L,
                         seed=wl.seed,
                         encoder_weights=S.encoder_weights(wl) if wl.encoder == "random" else None,
                         block_routing=wl.block_routing)
    if args.refine_kernel:
        idx.debug_refine_kernel(args.refine_kernel)
    for c in range(wl.n_chunks - ncs):
        kd, ks = chunk_keys_dev(wl, c * T, (c + 1) * T, dev)
        idx.append_keys(kd, ks)
        idx.seal()
    idx.publish()
    idx.sync()
    idx.checkpoint()
    chunks = []
    for c in range(ncs):
        a = p_first + c * T
        kd, ks = chunk_keys_dev(wl, a, a + T, dev)
        qd, wd = queries_dev(wl, a, a + T, dev)
        chunks.append((a, kd, ks, qd, wd))
    return idx, chunks


def measure_exhaustive(idx, wl, qd, wd, pos0, stream, reps):
    """The in-library exhaustive selection of one chunk: one warm-up call
    (it allocates its score rows on first use), then `reps` timed calls
    with phase events on.  Returns (ids of the last call, median ms,
    phase ms per call {exh_scores, exh_topk})."""
    import torch
    exh = torch.empty((wl.T, wl.k), dtype=torch.int32, device=qd.device)
    idx.select_exhaustive(qd, wd, pos0, wl.k, out=exh)
    idx.sync()
    idx.profile_read()
    idx.profile(True)
    ms = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        idx.select_exhaustive(qd, wd, pos0, wl.k, out=exh)
        e1.record(stream)
        idx.sync()
        ms.append(e0.elapsed_time(e1))
    idx.profile(False)
    ph = idx.profile_read()
    per = {k: ph[k][0] / reps for k in ("exh_scores", "exh_topk")}
    return exh, float(np.median(ms)), per


def measure_workload(wl, args, dev, stream, world, steps, warmup, e2e_on, overlap_on):
    """Time `steps` steps of the workload (after `warmup`), then recall and
    the exhaustive baseline on its final chunk, the rooflines of the
    refine and GEMM kernels, and optionally the end-to-end number and the
    refit overlap.  Returns a dict of results (the index is closed)."""
    import torch
    import torch.distributed as dist
    from ivf_top_key_b200 import C as capi
    T, L = wl.T, wl.L
    ncs = chunks_per_step(wl)
    pos0 = L - T                   # last chunk (recall is measured on it)
    idx, chunks = build_index(wl, args, dev)
    kd, ks, qd, wd = chunks[-1][1:]
    out = torch.empty((T, wl.k), dtype=torch.int32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    sharded = getattr(args, "mode", "replicas") == "sharded" and world > 1
    if sharded:
        from ivf_top_key_b200 import sharded as shd

    def step():
        for a, kd_, ks_, qd_, wd_ in chunks:
            idx.append_keys(kd_, ks_)
            idx.seal()
            if sharded:
                out.copy_(shd.sharded_route_refine(idx, qd_, wd_, a, wl.k, wl.budget))
            else:
                idx.route_refine(qd_, wd_, a, wl.k, wl.budget, out=out)
        idx.publish()

    for _ in range(warmup):
        flush.fill_(1)
        idx.rollback()
        step()
    idx.sync()
    idx.profile_read()
    idx.profile(True)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = capi.ai_kernel_launches()
    clk = Clocks(torch.cuda.current_device())
    with clk:
        t_wall = time.perf_counter()
        for i in range(steps):
            flush.fill_(i & 0xFF)
            idx.rollback()
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        t_wall = time.perf_counter() - t_wall
    if world > 1:
        dist.barrier()
    launches = capi.ai_kernel_launches() - launches0
    idx.profile(False)
    phases = idx.profile_read()
    idx.sync()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = max_over_ranks(float(np.sum(step_ms)), dev)
    units = T * ncs                # query tokens per step
    # sharded: the ranks share one request, so its queries count once
    value = weak_scaling_value(units, steps, 1 if sharded else world, total_ms)
    st = idx.stats()
    nC = st["n_clusters"]

    # the route GEMM and the refine kernel alone: the final chunk routed
    # again with no refit in flight (inside a step the side-stream refit
    # shares the GPU with them)
    idx.publish()
    idx.sync()
    idx.profile_read()
    idx.profile(True)
    for _ in range(args.exh_reps):
        idx.route_refine(qd, wd, pos0, wl.k, wl.budget, out=out)
    idx.sync()
    idx.profile(False)
    iso = idx.profile_read()

    # recall vs the in-library exhaustive selection (final chunk, after the
    # last step), and the exhaustive's own timing
    recall, exh_ms, exh_ph = None, None, {"exh_scores": 0.0, "exh_topk": 0.0}
    if args.exhaustive:
        exh, exh_ms, exh_ph = measure_exhaustive(idx, wl, qd, wd, pos0, stream, args.exh_reps)
        rows = torch.arange(T, device=dev, dtype=torch.int64)[:, None] * (L + 1)
        sel_c = (out.to(torch.int64) + rows)[out >= 0]
        exh_c = (exh.to(torch.int64) + rows)[exh >= 0]
        recall = float(torch.isin(exh_c, sel_c).sum().item() / max(1, exh_c.numel()))

    # rooflines (live CUDA events of the library's phases)
    peaks, peak_kind = measured_peaks()
    esz = {"bf16": 2, "fp8": 1, "fp32": 4}[wl.key_dtype]
    row_bytes = wl.d * esz + (4 if wl.key_dtype == "fp8" else 0)
    refine_ms, refine_n = phases["refine"]
    route_ms, route_n = phases["route"]
    # algorithmic bytes per refine launch: gathered candidate rows, query,
    # weights, cluster-score row, CSR offsets, output ids
    qbytes = wl.H * wl.d * (2 if wl.q_dtype == "bf16" else 4)
    refine_bytes = T * (wl.budget * row_bytes + qbytes + wl.H * 4 + nC * 8 + wl.k * 4)
    # (nC: clusters of the final chunk's index; per launch = one chunk of T queries)
    route_flops = 2.0 * T * wl.H * wl.d * nC
    dom = max(phases.items(), key=lambda kv: kv[1][0])[0]
    roofline = None
    if refine_n:
        avg = refine_ms / refine_n / 1e3
        ach = refine_bytes / avg / 1e9
        traffic = traffic_from_profile(os.path.join(ROOT, "ivf_top_key_b200", "csrc", "route_refine.cu"),
                                       os.path.join(ROOT, "profiles", f"refine_{wl.name}.md"))
        kname = {0: "k_refine_simt", 1: "k_refine_tc (list in shared memory)",
                 2: "k_refine_tc (list in global scratch)",
                 3: "k_refine_pipe (warp-specialised: build / gather + rescore / top-k overlapped)",
                 4: "k_refine_pipe (warp-specialised, one TMEM score buffer)"}[
            idx.refine_kernel_choice(wl.budget)]
        roofline = {"kernel": kname,
                    "bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": round(ach / peaks["hbm_gbs"], 4),
                    "traffic": traffic, "peak_source": f"{peak_kind} hbm_gbs",
                    "algorithmic_bytes_per_launch": refine_bytes,
                    "avg_launch_ms": round(refine_ms / refine_n, 4)}
    route_roof = None
    if route_n:
        avg = route_ms / route_n / 1e3
        tf = route_flops / avg / 1e12
        iso_ms, iso_n = iso["route"]
        tf_iso = route_flops / (iso_ms / iso_n / 1e3) / 1e12 if iso_n else None
        route_roof = {"kernel": "k_scores_tc (route GEMM)", "bound": "tensor",
                      "achieved": round(tf, 1), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                      "frac": round(tf / peaks["bf16_tflops"], 4),
                      "peak_source": f"{peak_kind} bf16_tflops (burst)",
                      "avg_launch_ms": round(route_ms / route_n, 4),
                      "isolated": {"achieved": round(tf_iso, 1), "frac": round(tf_iso / peaks["bf16_tflops"], 4),
                                   "avg_launch_ms": round(iso_ms / iso_n, 4),
                                   "note": "final chunk routed again with no refit in flight"}
                      if tf_iso else None}
    if roofline is not None and iso["refine"][1]:
        ams = iso["refine"][0] / iso["refine"][1]
        ach = refine_bytes / (ams / 1e3) / 1e9
        roofline["isolated"] = {"achieved": round(ach, 1), "frac": round(ach / peaks["hbm_gbs"], 4),
                                "avg_launch_ms": round(ams, 4),
                                "note": "final chunk routed again with no refit in flight"}
    exh_roof = None
    if exh_ph["exh_scores"] > 0:
        # causal: query i scores keys 0 .. pos0 + i
        flops = 2.0 * wl.H * wl.d * (T * pos0 + T * (T + 1) / 2)
        tf = flops / (exh_ph["exh_scores"] / 1e3) / 1e12
        exh_roof = {"kernel": "k_scores_tc (exhaustive GEMM, causal)", "bound": "tensor",
                    "achieved": round(tf, 1), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                    "frac": round(tf / peaks["bf16_tflops"], 4),
                    "peak_source": f"{peak_kind} bf16_tflops (burst)",
                    "ms_per_chunk": round(exh_ph["exh_scores"], 4)}

    # end to end through the public API with host buffers
    e2e = measure_e2e(idx, chunks, wl, out, stream, flush, steps, warmup, world, units) \
        if e2e_on and not sharded else None
    refit_overlap = None
    if overlap_on:  # last: it moves the checkpoint to the full prefix
        refit_overlap = measure_refit_overlap(idx, chunks, wl, out, stream)
    idx.close()
    return {
        "value": value, "total_ms": total_ms, "steps": steps, "units": units,
        "recall": recall, "nC": nC,
        "exhaustive": {"value": round(T / (exh_ms / 1e3), 1), "unit": UNIT,
                       "ms_per_chunk": round(exh_ms, 4),
                       "note": f"in-library exhaustive selection of the final chunk (warm; median of "
                               f"{args.exh_reps} calls)",
                       "phases_ms_per_chunk": {k: round(v, 4) for k, v in exh_ph.items()},
                       "route_refine_speedup": round(value / world / (T / (exh_ms / 1e3)), 2)}
        if exh_ms else None,
        "roofline": roofline, "roofline_route_gemm": route_roof, "roofline_exhaustive_gemm": exh_roof,
        "phases": phases, "dominant_phase": dom, "launches": launches, "clocks": clk.summary(),
        "e2e": e2e, "refit_overlap": refit_overlap, "wall_s": t_wall,
    }


def measure_e2e(idx, chunks, wl, out, stream, flush, steps, warmup, world, units):
    """The same step through the public API with pinned host buffers: every
    step copies its inputs host-to-device and its result back inside the
    timed region."""
    import torch
    dev = out.device
    T = wl.T
    kd, ks, qd, wd = chunks[-1][1:]
    host = []
    for a, kd_, ks_, qd_, wd_ in chunks:
        host.append((a, kd_.cpu().pin_memory(), ks_.cpu().pin_memory() if ks_ is not None else None,
                     qd_.cpu().pin_memory(), wd_.cpu().pin_memory(),
                     torch.empty((T, wl.k), dtype=torch.int32).pin_memory()))
    # Two device input/output sets; host-to-device copies of chunk c+1
    # and the device-to-host copy of chunk c's result run on copy streams
    # while chunk c is processed (every copy stays inside the timed region).
    bufs = [(torch.empty_like(kd), torch.empty_like(ks) if ks is not None else None,
             torch.empty_like(qd), torch.empty_like(wd), torch.empty_like(out)) for _ in range(2)]
    h2d_s = torch.cuda.Stream(device=dev)
    d2h_s = torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def load(c):
        _, kh, sh, qh, wh, _ = host[c]
        kb, sb, qb, wb, _ = bufs[c % 2]
        with torch.cuda.stream(h2d_s):
            if c >= 2:
                h2d_s.wait_event(ev_done[c % 2])  # chunk c-2 no longer reads the set
            kb.copy_(kh, non_blocking=True)
            if sh is not None:
                sb.copy_(sh, non_blocking=True)
            qb.copy_(qh, non_blocking=True)
            wb.copy_(wh, non_blocking=True)
            ev_in[c % 2].record(h2d_s)

    def e2e_step():
        n = len(host)
        h2d_s.wait_stream(stream)  # after the work already queued (and the start event)
        load(0)
        for c in range(n):
            a = host[c][0]
            kb, sb, qb, wb, ob = bufs[c % 2]
            stream.wait_event(ev_in[c % 2])
            if c >= 2:
                stream.wait_event(ev_out[c % 2])  # chunk c-2's result has left
            idx.append_keys(kb, sb)
            idx.seal()
            idx.route_refine(qb, wb, a, wl.k, wl.budget, out=ob)
            ev_done[c % 2].record(stream)
            if c + 1 < n:
                load(c + 1)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(ev_done[c % 2])
                host[c][5].copy_(ob, non_blocking=True)
                ev_out[c % 2].record(d2h_s)
        idx.publish()
        stream.wait_event(ev_out[(n - 1) % 2])

    for _ in range(max(1, warmup)):
        idx.rollback()
        e2e_step()
    torch.cuda.synchronize()
    ee = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for i in range(steps):
        flush.fill_(i & 0xFF)
        idx.rollback()
        ee[i][0].record(stream)
        e2e_step()
        ee[i][1].record(stream)
    torch.cuda.synchronize()
    e_ms = max_over_ranks(float(np.sum([a.elapsed_time(b) for a, b in ee])), dev)
    h2d = sum(kh.numel() * kh.element_size() + qh.numel() * qh.element_size() +
              wh.numel() * wh.element_size() + (sh.numel() * 4 if sh is not None else 0)
              for _, kh, sh, qh, wh, _ in host)
    d2h = sum(oh.numel() * 4 for *_, oh in host)
    return {"value": weak_scaling_value(units, steps, world, e_ms), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": e_ms / steps}


def measure_decode(wl, args, dev, stream, n_steps):
    """Decode after a full prefill of the workload: every step appends the
    next key, seals (a window completes every W steps; refits follow their
    period) and selects the top-k of one query at the newest position.
    The same steps are timed with route+refine and with the exhaustive
    selection (the index is rolled back between the two); CUDA events
    around all steps."""
    import torch
    from ivf_top_key_b200 import AttentionIndex
    T, L = wl.T, wl.L
    wl_d = S.scaled(wl, L=L + n_steps)
    idx = AttentionIndex(d=wl.d, H=wl.H, key_dtype=wl.key_dtype, q_dtype=wl.q_dtype,
                         n_sinks=wl.n_sinks, window=wl.window,
                         clusters_per_window=wl.clusters_per_window,
                         refit_period=wl.refit_period, seal_iters=wl.seal_iters, async_refit=True,
                         max_query_chunk=T, max_budget=wl.budget, max_k=wl.k, max_keys=L + n_steps,
                         seed=wl.seed, block_routing=wl.block_routing)
    for c in range(wl.n_chunks):
        kd, ks = chunk_keys_dev(wl, c * T, (c + 1) * T, dev)
        idx.append_keys(kd, ks)
        idx.seal()
    idx.publish()
    idx.sync()
    idx.checkpoint()
    kd, ks = chunk_keys_dev(wl_d, L, L + n_steps, dev)
    qd, wd = queries_dev(wl_d, L, L + n_steps, dev)
    out = torch.empty((1, wl.k), dtype=torch.int32, device=dev)

    def run(select, n):
        for i in range(n):
            idx.append_keys(kd[i:i + 1], None if ks is None else ks[i:i + 1])
            idx.seal()
            select(qd[i:i + 1], wd[i:i + 1], L + i)
        idx.publish()

    def rr(q, w, t):
        idx.route_refine(q, w, t, wl.k, wl.budget, out=out)

    def ex(q, w, t):
        idx.select_exhaustive(q, w, t, wl.k, out=out)

    res = {}
    for name, fn in (("route_refine", rr), ("exhaustive", ex)):
        idx.rollback()
        run(fn, min(8, n_steps))  # warm-up
        idx.sync()
        idx.rollback()
        idx.sync()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run(fn, n_steps)
        e1.record(stream)
        idx.sync()
        ms = e0.elapsed_time(e1)
        res[name] = {"us_per_token": round(ms * 1e3 / n_steps, 2),
                     "tokens_per_s": round(n_steps / (ms / 1e3), 1)}
    idx.close()
    return {"workload": wl.name, "prefix_tokens": L, "steps": n_steps, "batch": 1,
            "step": "append one key + seal (+ refit on its period) + select for one query",
            **res, "speedup_vs_exhaustive": round(res["exhaustive"]["us_per_token"] /
                                                  res["route_refine"]["us_per_token"], 2)}


def run_ours(args):
    import torch
    import torch.distributed as dist
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    # the selection path runs on a high-priority stream so that the refit the
    # library runs on its own (default-priority) side stream stays in the
    # background, as in a serving engine
    lo_pri, hi_pri = torch.cuda.Stream.priority_range()
    main_stream = torch.cuda.Stream(device=dev, priority=hi_pri)
    torch.cuda.set_stream(main_stream)
    stream = torch.cuda.current_stream()
    wl = wl_for_rank(args.workload, rank, args.budget, args.refit_period, args.routing,
                     sharded=args.mode == "sharded" and world > 1)
    r = measure_workload(wl, args, dev, stream, world, args.steps, args.warmup, not args.no_e2e,
                         args.refit_overlap)
    # the 1M-key prefix (one final chunk routed over ~8200 clusters, plus
    # the concurrent full refit) rides along with the default workload
    r1m = None
    if args.with_1m and args.workload == "glm_bf16_L128k" and args.routing == "ivf" and args.refit_period < 0 \
            and not args.budget:
        wl1 = wl_for_rank("glm_bf16_L1m", rank, 0, sharded=args.mode == "sharded" and world > 1)
        r1m = measure_workload(wl1, args, dev, stream, world, max(3, args.steps // 2), max(3, args.warmup),
                               False, True)
    l2 = None
    if r["roofline"] is not None and wl.L * wl.d * 2 <= (64 << 20):
        # key store L2-resident: the rescore's rows come from L2, so its
        # algorithmic bytes are also set against an L2-resident read
        l2p = l2_read_peak(dev)
        ach = r["roofline"]["achieved"]
        l2 = {"kernel": r["roofline"]["kernel"], "achieved": ach, "peak": round(l2p, 1), "unit": "GB/s",
              "frac": round(ach / l2p, 4),
              "peak_source": "torch row sums over 16 stride-0 repeats of a 64 MiB L2-resident fp32 buffer, "
                             "best of 20 (read bytes)",
              "note": f"key store {wl.L * wl.d * 2 >> 20} MiB fits L2: rows are served from L2"}
    dec = measure_decode(wl, args, dev, stream, args.decode) if args.decode else None
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_baseline(wl, args.cpu_sample)
    if rank == 0:
        phases = r["phases"]
        line = {
            "metric": METRIC, "value": round(r["value"], 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["total_ms"] / args.steps,
            "higher_is_better": True,
            "scaling": "strong" if args.mode == "sharded" and world > 1 else "weak", "vs_baseline": None,
            "dtype": wl.key_dtype, "data": "synthetic (seeded Gaussian-mixture keys/queries)",
            "config": config_block(wl, world, args.mode),
            "recall_vs_exhaustive": round(r["recall"], 4) if r["recall"] is not None else None,
            "exhaustive": r["exhaustive"],
            "roofline": r["roofline"], "l2": l2, "roofline_route_gemm": r["roofline_route_gemm"],
            "roofline_exhaustive_gemm": r["roofline_exhaustive_gemm"],
            "phases_ms_per_step": {k: round(v[0] / args.steps, 4) for k, v in phases.items()},
            "dominant_phase": r["dominant_phase"],
            "gpu_launches": int(r["launches"]), "gpu_launches_per_step": r["launches"] / args.steps,
            "refit_overlap": r["refit_overlap"],
            "clocks": r["clocks"], "e2e": r["e2e"], "cpu_baseline": cpu,
            "wall_s_timed_region": round(r["wall_s"], 3),
        }
        if dec is not None:
            line["decode"] = dec
        if r1m is not None:
            line["at_1m"] = {
                "workload": "glm_bf16_L1m", "prefix_tokens": wl1.L, "clusters": r1m["nC"],
                "value": round(r1m["value"], 1), "unit": UNIT, "steps": r1m["steps"],
                "ms_per_step": r1m["total_ms"] / r1m["steps"],
                "recall_vs_exhaustive": round(r1m["recall"], 4) if r1m["recall"] is not None else None,
                "exhaustive": r1m["exhaustive"], "roofline": r1m["roofline"],
                "roofline_route_gemm": r1m["roofline_route_gemm"],
                "roofline_exhaustive_gemm": r1m["roofline_exhaustive_gemm"],
                "phases_ms_per_step": {k: round(v[0] / r1m["steps"], 4) for k, v in r1m["phases"].items()},
                "refit_overlap": r1m["refit_overlap"], "clocks": r1m["clocks"],
                "gpu_launches": int(r1m["launches"]),
            }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def measure_refit_overlap(idx, chunks, wl, out, stream, reps=3):
    """One warm-started refit over the whole prefix (64 new seeds from the
    last 16384 keys) on the side stream, concurrent with routing the final
    chunk: hidden = (t_refit + t_route - t_both) / t_refit, all from CUDA
    events on the main stream (the refit is joined by ai_publish)."""
    import torch
    idx.rollback()
    for a, kd_, ks_, qd_, wd_ in chunks:
        idx.append_keys(kd_, ks_)
        idx.seal()
    idx.publish()
    idx.sync()
    idx.checkpoint()
    a, _, _, qd, wd = chunks[-1]

    def timed(fn):
        best = []
        for _ in range(reps):
            idx.rollback()
            idx.sync()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            idx.sync()
            best.append(e0.elapsed_time(e1))
        return float(np.median(best))

    def refit_only():
        idx.refit(64, 16384)
        idx.publish()

    def route_only():
        idx.route_refine(qd, wd, a, wl.k, wl.budget, out=out)

    def both():
        idx.refit(64, 16384)
        idx.route_refine(qd, wd, a, wl.k, wl.budget, out=out)
        idx.publish()

    t_refit, t_route, t_both = timed(refit_only), timed(route_only), timed(both)
    st = idx.stats()
    return {"t_refit_ms": t_refit, "t_route_ms": t_route, "t_both_ms": t_both,
            "hidden_fraction": (t_refit + t_route - t_both) / t_refit if t_refit > 0 else None,
            "keys": st["n_keys"], "clusters_after": st["n_clusters"],
            "keys_fully_scanned": st["last_refit_scanned"],
            "keys_rechecked_f64": st["last_refit_rechecked"]}


# --------------------------------------------------------- oracle arm --

def _threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def _oracle_prefix(wl):
    from oracle import ai_oracle as O
    orc = O.OracleIndex(d=wl.d, n_sinks=wl.n_sinks, window=wl.window,
                        clusters_per_window=wl.clusters_per_window,
                        refit_period=wl.refit_period, refit_new_seeds=wl.refit_new_seeds,
                        refit_seed_window=wl.refit_seed_window, seal_iters=wl.seal_iters,
                        seed=wl.seed,
                        encoder=S.encoder_weights(wl) if wl.encoder == "random" else None,
                        block_routing=wl.block_routing)
    keys = oracle_keys(wl, 0, wl.L)
    for c in range(wl.n_chunks - chunks_per_step(wl)):
        orc.append(keys[c * wl.T:(c + 1) * wl.T])
        orc.seal()
    orc.publish()
    return orc, keys


def oracle_keys(wl, p0, p1):
    from oracle import ai_oracle as O
    kf = S.keys_f64(wl, p0, p1)
    if wl.key_dtype == "fp32":
        return kf.astype(np.float32).astype(np.float64)
    vals = S.bf16_bits_to_f64(S.to_bf16_bits(kf))
    if wl.key_dtype == "bf16":
        return vals
    codes, sc = O.quantize_fp8_keys(vals.astype(np.float32))
    return codes * sc.astype(np.float64)[:, None]


def oracle_queries(wl, p0, p1):
    q, w = S.queries_f64(wl, p0, p1)
    w = w.astype(np.float32).astype(np.float64)
    if wl.q_dtype == "fp32":
        return q.astype(np.float32).astype(np.float64), w
    return S.bf16_bits_to_f64(S.to_bf16_bits(q)), w


def oracle_step(orc0, keys, wl, sample_idx, qv, wv):
    """One oracle step over the timed chunks: maintenance (append, seal,
    refit) of every chunk plus route+refine of a sample of their queries.
    sample_idx indexes the queries of the timed chunks.  Returns
    (maintenance seconds, seconds per query)."""
    import copy
    orc = copy.deepcopy(orc0)
    ncs = chunks_per_step(wl)
    p_first = wl.L - ncs * wl.T
    t_m = t_q = 0.0
    nq = 0
    for c in range(ncs):
        a = p_first + c * wl.T
        t0 = time.perf_counter()
        orc.append(keys[a:a + wl.T])
        orc.seal()
        t_m += time.perf_counter() - t0
        t0 = time.perf_counter()
        for i in sample_idx:
            if c * wl.T <= i < (c + 1) * wl.T:
                orc.route_refine(qv[i], wv[i], p_first + int(i), wl.k, wl.budget)
                nq += 1
        t_q += time.perf_counter() - t0
    return t_m, t_q / max(nq, 1)


def oracle_baseline(wl, n_sample):
    orc, keys = _oracle_prefix(wl)
    nq = chunks_per_step(wl) * wl.T
    qv, wv = oracle_queries(wl, wl.L - nq, wl.L)
    rng = np.random.default_rng(0)
    sample = np.sort(rng.choice(nq, size=min(n_sample, nq), replace=False))
    t_m, t_q = oracle_step(orc, keys, wl, sample, qv, wv)
    step_s = t_m + nq * t_q
    return {"value": round(nq / step_s, 2), "unit": UNIT, "cores": _threads(), "kind": "oracle",
            "sample": (f"last {nq} queries of {wl.name} (one step): full maintenance (append, "
                       f"seal, refit) timed ({t_m:.2f} s) + {len(sample)} sampled queries' "
                       f"route+refine ({t_q * 1e3:.1f} ms each), extrapolated to the step")}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    wl = wl_for_rank(args.workload, 0, args.budget, args.refit_period, args.routing)
    orc, keys = _oracle_prefix(wl)
    nq = chunks_per_step(wl) * wl.T
    qv, wv = oracle_queries(wl, wl.L - nq, wl.L)
    rng = np.random.default_rng(0)
    n = max(4, min(args.cpu_sample, nq) // 4)
    for _ in range(args.warmup):
        oracle_step(orc, keys, wl, rng.choice(nq, size=2, replace=False), qv, wv)
    tot = 0.0
    t_ms, t_qs = [], []
    for _ in range(args.steps):
        sample = np.sort(rng.choice(nq, size=n, replace=False))
        t_m, t_q = oracle_step(orc, keys, wl, sample, qv, wv)
        t_ms.append(t_m)
        t_qs.append(t_q)
        tot += t_m + nq * t_q
    value = nq * args.steps / tot
    cores = _threads()
    sample_desc = (f"per step: maintenance of the last {nq} positions of {wl.name} "
                   f"(mean {np.mean(t_ms):.2f} s) + {n} sampled queries' route+refine "
                   f"(mean {np.mean(t_qs) * 1e3:.1f} ms each), extrapolated to the step")
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded Gaussian-mixture keys/queries)",
        "config": config_block(wl, world), "impl": "reference",
        "cpu_baseline": {"kind": "oracle", "cores": cores, "sample": sample_desc,
                         "value": round(value, 2), "unit": UNIT},
        "e2e": {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
