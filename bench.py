"""Benchmark of the CSA / HCA compressed-attention decode step on B200.

One step = one decode step of one layer for a batch of requests: compressor
append of the new token (csa_compress_append), lightning-indexer scores and
top-k (csa_index_scores + csa_topk, or csa_index_topk in one launch with
--select fused) and multi-query attention (csa_hca_decode_attn), all through
the C ABI.  Inputs are seeded synthetic
data of the workload's shapes; caches are filled through the same append
path before timing.

Default workload: CSA Pro-like decode at 1M context (1,048,576 tokens =
262,144 compressed entries per request), batch 4, 128 query heads x 512, 64
RoPE dims, indexer 64 x 128 MXFP4, top-1024, window 128.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl reference] [--no-cpu-baseline] [--no-other-workloads]

At N = 1 the line also carries `other_workloads`: the tiny fp32 CSA layer,
HCA at 128K, CSA Flash-like at 128K and HCA at 1M, each with its own
throughput, breakdown, rooflines and clock record (fewer steps each).

Prints one JSON line (rank 0).  For N > 1 run under torch.distributed.run:
each rank serves its own batch (requests shard across GPUs, no collective on
the data path); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from compressed_sparse_long_hca_b200 import inputs as I  # noqa: E402

METRIC = "CSA/HCA decode queries/s per layer at 128K–1M ctx; HBM GB/s vs ~8 TB/s"
UNIT = "queries/s"


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], "measured", d
    return 6650.0, "fallback", {}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def _profiled_traffic(select: str = "separate"):
    """DRAM bytes (read + write) per launch of the roofline's kernel from the
    committed ncu summary, or None when the kernel's sources changed since
    the capture."""
    import hashlib
    name = "index_topk_csa-pro-1m.md" if select == "fused" else "index_tc_csa-pro-1m.md"
    path = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(path):
        return None
    fields = {}
    for line in open(path, encoding="utf-8"):
        k, _, v = line.strip().partition(": ")
        if k in ("sources_sha256", "traffic_bytes_per_launch"):
            fields[k] = v.strip()
    h = hashlib.sha256()
    for f in ("index_tc.cu", "layout.cuh", "tc.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "compressed_sparse_long_hca_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    if fields.get("sources_sha256") != h.hexdigest() or "traffic_bytes_per_launch" not in fields:
        return None
    return int(fields["traffic_bytes_per_launch"])


def workload_config(wl, ws: int, select: str = "separate") -> dict:
    """The `config` object both arms print."""
    return {"workload": wl.name, "context": wl.context, "batch_per_gpu": wl.batch, "heads": wl.H,
            "head_dim": wl.D, "rope_dims": wl.R, "indexer": f"{wl.H_I}x{wl.d_I}", "topk": wl.k,
            "window": wl.W, "layers_per_step": 1,
            "l2": "flushed before every timed step: 256 MB written, then 256 MB read (not timed)",
            "parallelism": f"request-sharded x{ws}",
            "select": ("csa_index_topk" if select == "fused" else "csa_index_scores + csa_topk") if wl.kind == "csa" else None}


def rank_seed(wl, rank: int) -> int:
    """Seed of the requests a rank owns: ranks hold disjoint requests."""
    return wl.seed + 7919 * rank


def max_over_ranks(vals, ws: int, device) -> list:
    """Element-wise maximum of per-rank device timings (all ranks call it)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(vals), dtype=torch.float64, device=device)
    if ws > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_rate(ws: int, batch_per_rank: int, steps: int, ms: float) -> float:
    """Queries per second of the whole job: every rank's queries over the
    slowest rank's time."""
    return ws * batch_per_rank * steps / (ms / 1e3)


class Clocks:
    """SM clock and clock-event reasons of this rank's GPU, sampled every
    millisecond through NVML (read-only queries) by a background thread
    during the timed region; nvidia-smi polling when NVML is unavailable."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap"}

    def __init__(self, gpu_index: int):
        import torch
        try:
            self.uuid = "GPU-" + str(torch.cuda.get_device_properties(gpu_index).uuid)
        except Exception:
            self.uuid = None
        self.gpu_index = gpu_index
        self.proc = None
        self.thread = None
        self.samples = []
        import tempfile
        self.path = os.path.join(tempfile.gettempdir(), f"csa_bench_clocks_{os.getpid()}_{gpu_index}.csv")

    def _nvml_loop(self, handle, nv):
        while not self.stop_flag:
            try:
                sm = nv.nvmlDeviceGetClockInfo(handle, nv.NVML_CLOCK_SM)
                mx = nv.nvmlDeviceGetMaxClockInfo(handle, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(handle)
                self.samples.append((sm, mx, rs))
            except Exception:
                pass
            time.sleep(0.001)

    def start(self):
        self.stop_flag = False
        try:
            import pynvml as nv
            import threading
            nv.nvmlInit()
            handle = nv.nvmlDeviceGetHandleByUUID(self.uuid) if self.uuid else nv.nvmlDeviceGetHandleByIndex(self.gpu_index)
            self.nv = nv
            self.thread = threading.Thread(target=self._nvml_loop, args=(handle, nv), daemon=True)
            self.thread.start()
            return
        except Exception:
            self.thread = None
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.uuid or self.gpu_index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.stop_flag = True
            self.thread.join(timeout=5)
            if not self.samples:
                return None
            sm = [x[0] for x in self.samples]
            reasons = sorted({nm for _, _, rs in self.samples for bit, nm in self.REASONS.items() if rs & bit})
            return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(x[1] for x in self.samples)),
                    "reasons": reasons, "samples": len(sm), "source": "nvml, 1 ms"}
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvidia-smi, 100 ms"}


# ---------------------------------------------------------------- GPU arm

def key_bytes(wl, fmt: str) -> int:
    """Bytes of one stored index key: MXFP4 codes + E8M0 scales, or fp32."""
    return wl.d_I * 4 if fmt == "f32" else wl.d_I // 2 + wl.d_I // 32


def row_bytes(wl, fmt: str) -> int:
    """Bytes of one stored KV row: E4M3 non-RoPE part + BF16 RoPE part + fp32
    scale, or fp32."""
    return wl.D * 4 if fmt == "f32" else (wl.D - wl.R) + 2 * wl.R + 4


def workload_fmt(wl) -> str:
    """Storage format of a workload: the tiny configuration is the fp32 one."""
    return "f32" if wl.name == "tiny-csa" else "mixed"


def measure(wl, rank: int, ws: int, steps: int, warm: int, with_e2e: bool, select: str = "separate") -> dict:
    """Fill a cache of the workload through the append path, then time
    `steps` decode steps (after `warm` eager warm-up steps) as CUDA graph
    replays with the L2 flushed before each; returns the figures of the
    bench line (times are this rank's; the caller takes the max over ranks)."""
    import torch

    from compressed_sparse_long_hca_b200 import _lib
    from compressed_sparse_long_hca_b200.api import Cache, DecodeStep, topk

    B, T0 = wl.batch, wl.context
    csa = wl.kind == "csa"
    fmt = workload_fmt(wl)
    cap = T0 + 5 * steps + warm + 256       # every timed or warm-up step (and graph warm-up) appends one token
    nb = (cap + 511) // 512
    layer = 0
    b_kv, b_idx, sink = I.layer_params(wl.seed, layer, wl.kind, wl.D, wl.d_I or 32, wl.H)
    cache = Cache(n_csa=1 if csa else 0, n_hca=0 if csa else 1, H=wl.H, D=wl.D, D_rope=wl.R,
                  H_I=wl.H_I or 1, d_I=wl.d_I or 32, max_requests=B, max_pages_per_request=nb,
                  pool_pages=nb * B, b_pos_csa=b_kv[None] if csa else None,
                  b_pos_idx=b_idx[None] if csa else None, b_pos_hca=None if csa else b_kv[None], fmt=fmt)
    qdt = cache.qdtype
    rid = torch.arange(B, dtype=torch.int32, device="cuda")
    for r in range(B):
        cache.request_alloc(r, cap)
    # ---- fill the caches to the workload's context through the append path
    dI = wl.d_I if csa else 0
    t = 0
    while t < T0:
        n_tok = min(I.CHUNK, T0 - t)
        chunk = t // I.CHUNK
        parts = [I.device_token_inputs(rank_seed(wl, rank), layer, r, chunk, wl.D, dI) for r in range(B)]
        st = lambda k: torch.stack([p[k][:n_tok] for p in parts]).contiguous() if parts[0][k] is not None else None
        cache.compress_append(layer, rid, st(0), st(1), st(2), st(3))
        t += n_tok
    torch.cuda.synchronize()
    cache.check_device_error()
    # ---- per-step inputs (device), generated up front
    total_steps = 3 * steps + warm
    g = torch.Generator(device="cuda")
    g.manual_seed(rank_seed(wl, rank) * 31)
    step_c = torch.randn((total_steps, B, 1, wl.D), generator=g, device="cuda")
    step_z = torch.randn((total_steps, B, 1, wl.D), generator=g, device="cuda")
    step_ci = torch.randn((total_steps, B, 1, dI), generator=g, device="cuda") if csa else None
    step_zi = torch.randn((total_steps, B, 1, dI), generator=g, device="cuda") if csa else None
    q = torch.randn((B, wl.H, wl.D), generator=g, device="cuda").to(qdt)
    qi = torch.randn((B, wl.H_I, dI), generator=g, device="cuda") if csa else None
    w = torch.randn((B, wl.H_I), generator=g, device="cuda") if csa else None
    sink_d = torch.from_numpy(sink).cuda()
    ld = (cap // 4 + 127) // 128 * 128
    scores = torch.empty((B, ld), device="cuda") if csa else None
    nv = torch.empty(B, dtype=torch.int32, device="cuda")
    idx = torch.empty((B, max(wl.k, 1)), dtype=torch.int32, device="cuda")
    out = torch.empty((B, wl.H, wl.D), dtype=qdt, device="cuda")
    flush = torch.empty(256 * 2**20, dtype=torch.uint8, device="cuda")    # > 126 MB L2
    flush_rd = torch.ones(256 * 2**20 // 4, dtype=torch.int32, device="cuda")

    def flush_l2():
        """Evict the step's inputs from L2 (not timed): write a buffer larger
        than L2, then read another one, so that the lines left in L2 are
        clean and the step is not charged for the flush's own write-backs."""
        flush.zero_()
        flush_rd.sum()

    stream = torch.cuda.current_stream()

    # Static per-step inputs: the timed steps replay CUDA graphs of the step
    # (append | index + top-k | attention); before each replay the step's
    # token inputs are copied into these buffers (outside the timed region).
    in_c, in_z = torch.empty_like(step_c[0]), torch.empty_like(step_z[0])
    in_ci = torch.empty_like(step_ci[0]) if csa else None
    in_zi = torch.empty_like(step_zi[0]) if csa else None

    def load_inputs(s):
        in_c.copy_(step_c[s])
        in_z.copy_(step_z[s])
        if csa:
            in_ci.copy_(step_ci[s])
            in_zi.copy_(step_zi[s])

    def part_append():
        cache.compress_append(layer, rid, in_c, in_z, in_ci, in_zi)

    tk_ws = torch.empty(cache.index_topk_workspace_bytes(B, ld) + 256, dtype=torch.uint8, device="cuda") if csa else None

    def part_index_topk():                  # scores and selection in one launch
        cache.index_topk(layer, rid, qi, w, scores, nv, wl.k, idx, workspace=tk_ws)

    def part_index():                       # scores materialised ...
        cache.index_scores(layer, rid, qi, w, scores, nv)

    def part_topk():                        # ... then selected
        topk(scores, nv, wl.k, idx)

    def part_attn():
        # on a CSA layer the call directly follows the step's index_topk
        cache.decode_attn(layer, rid, q, idx if csa else None, sink_d, out, state_ready=csa)

    sel_parts = ([("index_topk", part_index_topk)] if select == "fused" else
                 [("index", part_index), ("topk", part_topk)]) if csa else []
    parts = [("append", part_append)] + sel_parts + [("attention", part_attn)]
    for s in range(warm):                   # eager warm-up (also sizes the attention workspace)
        load_inputs(s)
        for _, f in parts:
            f()
    torch.cuda.synchronize()
    cache.check_device_error()
    lib = _lib.load()
    # The step as CUDA graphs: plain (the headline), with events around the
    # roofline kernel, with events around every part (the breakdown).  Event
    # nodes inside a graph cost a few microseconds each, so each figure comes
    # from its own pass of `steps` timed steps.
    def capture(marks):
        evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(parts) + 1)]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for x, (nm, f) in enumerate(parts):
                if nm in marks or (x > 0 and parts[x - 1][0] in marks):
                    evs[x].record()
                f()
            if parts[-1][0] in marks:
                evs[len(parts)].record()
        return g, evs

    launches0 = lib.csa_launch_count()
    g_plain, _ = capture(())
    kernels_per_step = lib.csa_launch_count() - launches0   # libcsa kernels inside the graph
    # the kernel the roofline is reported for: the index scan (CSA), the attention (HCA)
    roof_part = ("index_topk" if select == "fused" else "index") if csa else "attention"
    g_idx, ev_idx = capture((roof_part,))
    g_all, ev_all = capture(tuple(nm for nm, _ in parts))
    for gr in (g_plain, g_idx, g_all):      # a graph's first replay also uploads it: not timed
        load_inputs(0)
        gr.replay()
    torch.cuda.synchronize()
    cache.check_device_error()
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed_pass(g, first, after=None):
        total = 0.0
        for s in range(steps):
            load_inputs(first + s)
            flush_l2()                      # L2 flushed between timed steps (not timed)
            ev0.record(stream)
            g.replay()
            ev1.record(stream)
            ev1.synchronize()
            total += ev0.elapsed_time(ev1)
            if after:
                after()
        return total

    clocks = Clocks(torch.cuda.current_device())
    clocks.start()
    step_ms = timed_pass(g_plain, warm)
    clk = clocks.stop()
    idx_sum = [0.0]
    names = [nm for nm, _ in parts]
    x = names.index(roof_part)
    timed_pass(g_idx, warm + steps, lambda: idx_sum.__setitem__(0, idx_sum[0] + ev_idx[x].elapsed_time(ev_idx[x + 1])))
    part_ms = {nm: 0.0 for nm in names}

    def add_parts():
        for x, nm in enumerate(names):
            part_ms[nm] += ev_all[x].elapsed_time(ev_all[x + 1])

    timed_pass(g_all, warm + 2 * steps, add_parts)
    idx_ms = idx_sum[0] / steps
    res = {"step_ms": step_ms, "idx_ms": idx_ms, "clocks": clk, "launches": kernels_per_step * steps,
           "breakdown": {nm: round(v / steps * 1e3, 2) for nm, v in part_ms.items()}, "e2e_ms": None}
    del g_plain, g_idx, g_all
    if with_e2e:
        # ---- end to end through the public API with host buffers: DecodeStep
        # replays one graph that copies the step's packed inputs from its
        # pinned host buffer, runs the step and copies the output back
        e2e = DecodeStep(cache, layer, list(range(B)), wl.k if csa else 0, sink_d, fused_select=select == "fused")
        host_in = []
        for s in range(steps):              # each step's own inputs, packed up front (not timed)
            buf = torch.zeros(e2e.input_bytes, dtype=torch.uint8)
            v = e2e.views(buf)
            v["q"].copy_(q.cpu())
            v["c"].copy_(step_c[s].cpu())
            v["z"].copy_(step_z[s].cpu())
            if csa:
                v["ci"].copy_(step_ci[s].cpu())
                v["zi"].copy_(step_zi[s].cpu())
                v["q_idx"].copy_(qi.cpu())
                v["w"].copy_(w.cpu())
            host_in.append(buf)

        def produce(s):
            """The step's inputs written into the step's pinned buffer by
            their producer (not timed; the transfer from it is)."""
            e2e.host_in.copy_(host_in[s])

        produce(0)
        e2e()                               # first replay of the step's graph: not timed
        e2e(timed=True)
        torch.cuda.synchronize()
        e2e_ms = 0.0
        for s in range(steps):
            produce(s)
            flush_l2()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            e2e()
            b.record(stream)
            b.synchronize()
            e2e_ms += a.elapsed_time(b)
        # the same again with marks between the phases (input copy, step,
        # output copy) where the step is composed in Python (the C step's
        # copies happen inside the one call)
        phase = [0.0, 0.0, 0.0]
        for s in range(steps if e2e.fused_select else 0):
            produce(s)
            flush_l2()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            e2e(timed=True)
            b.record(stream)
            b.synchronize()
            ev = [a, e2e.marks[0], e2e.marks[1], b]
            for x in range(3):
                phase[x] += ev[x].elapsed_time(ev[x + 1])
        res["e2e_ms"] = e2e_ms
        res["e2e_phases"] = ({nm: round(v / steps * 1e3, 2) for nm, v in zip(("h2d", "step", "d2h"), phase)}
                             if e2e.fused_select else None)
        res["e2e_api"] = "api.DecodeStep -> " + ("csa_compress_append + csa_index_topk + csa_hca_decode_attn"
                                                 if e2e.fused_select else "csa_decode_step (host buffers)")
        res["h2d"] = e2e.input_bytes
        res["d2h"] = e2e.host_out.numel() * e2e.host_out.element_size()
        del e2e
    cache.check_device_error()
    # tokens per request half-way through the pass that timed the roofline
    # kernel: eager warm-up steps, one untimed replay of each of the three
    # graphs, the plain pass, then half of the timed pass
    res["t_mid"] = T0 + warm + 3 + steps + steps // 2
    del cache
    return res


def rooflines(wl, m: dict, steps: int, select: str = "separate") -> dict:
    """The dominant kernel's roofline and the whole step's, from the
    algorithmic bytes (or flops) of the workload."""
    peak, peak_kind, peaks = _peaks()
    csa = wl.kind == "csa"
    fmt = workload_fmt(wl)
    t_mid, idx_ms, step_ms = m["t_mid"], m["idx_ms"], m["step_ms"]
    B = wl.batch
    kb, rb = key_bytes(wl, fmt) if csa else 0, row_bytes(wl, fmt)
    out = {}
    if csa:
        n_c = t_mid // 4
        alg = B * (n_c * kb + wl.H_I * wl.d_I * 4 + wl.H_I * 4)
        ach = alg / (idx_ms / 1e3) / 1e9
        out["roofline"] = {"bound": "hbm", "kernel": "csa_index_topk" if select == "fused" else "csa_index_scores",
                           "achieved": ach, "peak": peak,
                           "unit": "GB/s", "frac": ach / peak,
                           "traffic": _profiled_traffic(select) if wl.name == "csa-pro-1m" else None,
                           "peak_source": peak_kind, "ms_per_launch": idx_ms,
                           "algorithmic_bytes_per_launch": alg}
    else:
        # HCA: the attention over every compressed entry is the dominant
        # kernel; QK^T and PV are 2 * H * rows * D flops each per query
        rows = t_mid // 128 + wl.W
        flops = B * 4.0 * wl.H * rows * wl.D
        ach = flops / (idx_ms / 1e3) / 1e12
        tpeak = peaks.get("bf16_tflops", 1590.0)
        out["roofline"] = {"bound": "tensor", "kernel": "csa_hca_decode_attn", "achieved": ach, "peak": tpeak,
                           "unit": "TFLOP/s", "frac": ach / tpeak, "traffic": None,
                           "peak_source": "measured bf16 burst" if "bf16_tflops" in peaks else "fallback",
                           "ms_per_launch": idx_ms, "algorithmic_flops_per_launch": flops,
                           "rows_per_query": rows}
    # the whole step against HBM: the algorithmic bytes of every part (index
    # keys scanned, selected and window rows gathered, q in and out) over the
    # step time, against the measured copy peak and the nominal 8 TB/s
    rows_q = (wl.k if csa else t_mid // 128) + wl.W
    qb = 4 if fmt == "f32" else 2
    step_bytes = B * ((t_mid // 4 * kb + wl.H_I * wl.d_I * 4 + wl.H_I * 4 if csa else 0)
                      + rows_q * rb + 2 * wl.H * wl.D * qb)
    step_gbs = step_bytes / (step_ms / steps / 1e3) / 1e9
    out["step_roofline"] = {"bound": "hbm", "achieved": step_gbs, "peak": peak, "unit": "GB/s",
                            "frac": step_gbs / peak, "frac_of_8tbs": step_gbs / 8000.0,
                            "algorithmic_bytes_per_step": step_bytes, "peak_source": peak_kind}
    return out


def measure_projections(steps: int = 10, n_tok: int = 4) -> dict:
    """The projections around the decode step at the Pro-like shapes (hidden
    7168, query latent 1024, 128 heads x 512, indexer 64 x 128, 16 output
    groups of 1024), for a batch of `n_tok` tokens, through csa_gemm_bf16:
    each call timed with CUDA events after an L2 flush, against the HBM
    roofline (at decode batch sizes a projection streams its weight)."""
    import torch

    from compressed_sparse_long_hca_b200.api import Linear
    d, D, dI, HI, dc, H, G, dg, dm = 7168, 512, 128, 64, 1024, 128, 16, 1024, 7168
    shapes = [  # name, n_out, k_in, groups, output dtype
        ("h -> c, z, c_I, z_I, w, c_q", 2 * D + 2 * dI + HI + dc, d, 1, torch.float32),
        ("c_q -> q, q_I", H * D + HI * dI, dc, 1, torch.bfloat16),
        ("attention -> grouped (16 x 1024)", G * dg, H * D, G, torch.bfloat16),
        ("grouped -> model width", dm, G * dg, 1, torch.float32),
    ]
    rng = np.random.default_rng(2026)
    peak, peak_kind, _ = _peaks()
    flush = torch.empty(256 * 2**20, dtype=torch.uint8, device="cuda")
    flush_rd = torch.ones(256 * 2**20 // 4, dtype=torch.int32, device="cuda")
    calls, total_us, total_bytes = {}, 0.0, 0
    for name, n_out, k_in, groups, odt in shapes:
        w = (rng.standard_normal((n_out, k_in // groups), dtype=np.float32) / np.float32(np.sqrt(k_in // groups)))
        lin = Linear(w, groups=groups)
        del w
        x = torch.randn((n_tok, k_in), device="cuda").to(torch.bfloat16)
        y = torch.empty((n_tok, n_out), dtype=odt, device="cuda")
        lin(x, y)                               # warm-up (workspace, launch set-up)
        torch.cuda.synchronize()
        ms = 0.0
        for _ in range(steps):
            flush.zero_()
            flush_rd.sum()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            lin(x, y)
            b.record()
            b.synchronize()
            ms += a.elapsed_time(b)
        Linear.check_device_error()
        us = ms / steps * 1e3
        nbytes = n_out * (k_in // groups) * 2 + n_tok * k_in * 2 + n_tok * n_out * y.element_size()
        calls[name] = {"us": round(us, 2), "weight_mb": round(n_out * (k_in // groups) * 2 / 1e6, 1),
                       "achieved_gbs": round(nbytes / (us / 1e6) / 1e9, 1),
                       "frac": round(nbytes / (us / 1e6) / 1e9 / peak, 3)}
        total_us += us
        total_bytes += nbytes
        del lin, x, y
    return {"tokens": n_tok, "calls": calls, "total_us": round(total_us, 2),
            "roofline": {"bound": "hbm", "achieved": total_bytes / (total_us / 1e6) / 1e9, "peak": peak,
                         "unit": "GB/s", "frac": total_bytes / (total_us / 1e6) / 1e9 / peak,
                         "algorithmic_bytes": total_bytes, "peak_source": peak_kind}}


def measure_prefill(wl, n_tok: int = 128, reps: int = 3) -> dict:
    """Chunks of queries with causal visibility (csa_prefill_chunk) at the end
    of the workload's context: each request of the batch appends n_tok new
    tokens that are all queries.  The cache is filled through the append path
    first; each chunk is timed with CUDA events after an L2 flush."""
    import torch

    from compressed_sparse_long_hca_b200.api import Cache
    B, T0 = wl.batch, wl.context
    csa = wl.kind == "csa"
    cap = T0 + (reps + 1) * n_tok + 512
    nb = (cap + 511) // 512
    b_kv, b_idx, sink = I.layer_params(wl.seed, 0, wl.kind, wl.D, wl.d_I or 32, wl.H)
    cache = Cache(n_csa=1 if csa else 0, n_hca=0 if csa else 1, H=wl.H, D=wl.D, D_rope=wl.R,
                  H_I=wl.H_I or 1, d_I=wl.d_I or 32, max_requests=B, max_pages_per_request=nb,
                  pool_pages=nb * B, b_pos_csa=b_kv[None] if csa else None,
                  b_pos_idx=b_idx[None] if csa else None, b_pos_hca=None if csa else b_kv[None],
                  fmt=workload_fmt(wl))
    rid = torch.arange(B, dtype=torch.int32, device="cuda")
    for r in range(B):
        cache.request_alloc(r, cap)
    dI = wl.d_I if csa else 0
    t = 0
    while t < T0:
        n = min(I.CHUNK, T0 - t)
        parts = [I.device_token_inputs(wl.seed, 0, r, t // I.CHUNK, wl.D, dI) for r in range(B)]
        st = lambda k: torch.stack([p[k][:n] for p in parts]).contiguous() if parts[0][k] is not None else None
        cache.compress_append(0, rid, st(0), st(1), st(2), st(3))
        t += n
    torch.cuda.synchronize()
    cache.check_device_error()
    g = torch.Generator(device="cuda")
    g.manual_seed(wl.seed * 7 + 1)
    shp = (B, n_tok)
    c, z = torch.randn(shp + (wl.D,), generator=g, device="cuda"), torch.randn(shp + (wl.D,), generator=g, device="cuda")
    ci = torch.randn(shp + (dI,), generator=g, device="cuda") if csa else None
    zi = torch.randn(shp + (dI,), generator=g, device="cuda") if csa else None
    q = torch.randn(shp + (wl.H, wl.D), generator=g, device="cuda").to(cache.qdtype)
    qi = torch.randn(shp + (wl.H_I, dI), generator=g, device="cuda") if csa else None
    w = torch.randn(shp + (wl.H_I,), generator=g, device="cuda") if csa else None
    out = torch.empty(shp + (wl.H, wl.D), dtype=cache.qdtype, device="cuda")
    sink_d = torch.from_numpy(sink).cuda()
    flush = torch.empty(256 * 2**20, dtype=torch.uint8, device="cuda")
    flush_rd = torch.ones(256 * 2**20 // 4, dtype=torch.int32, device="cuda")
    cache.prefill_chunk(0, rid, c, z, ci, zi, q, qi, w, wl.k if csa else 0, sink_d, out)    # warm-up chunk
    torch.cuda.synchronize()
    ms = 0.0
    for _ in range(reps):
        flush.zero_()
        flush_rd.sum()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        cache.prefill_chunk(0, rid, c, z, ci, zi, q, qi, w, wl.k if csa else 0, sink_d, out)
        b.record()
        b.synchronize()
        ms += a.elapsed_time(b)
    cache.check_device_error()
    us = ms / reps * 1e3
    toks = B * n_tok
    del cache
    return {"workload": wl.name, "context": T0, "batch": B, "tokens_per_request": n_tok, "chunks": reps,
            "us_per_chunk": round(us, 1), "tokens_per_s": toks / (us / 1e6),
            "api": "Cache.prefill_chunk -> csa_prefill_chunk",
            "l2": "flushed before each chunk (256 MiB write + read)"}


# Configurations measured beside the headline at N = 1 (fewer steps each):
# the tiny fp32 CSA layer, HCA at 128K (batch 32), CSA Flash-like at 128K
# (batch 32) and the HCA layer at 1M (batch 4).
OTHER_WORKLOADS = ("tiny-csa", "hca-128k", "csa-flash-128k", "hca-pro-1m")


def run_gpu(args):
    import gc

    import torch
    import torch.distributed as dist

    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    if ws > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    wl = I.WORKLOADS[args.workload]
    steps, warm = args.steps, args.warmup
    m = measure(wl, rank, ws, steps, warm, with_e2e=True, select=args.select)
    # ---- max over ranks
    step_ms, e2e_ms, idx_ms = max_over_ranks([m["step_ms"], m["e2e_ms"], m["idx_ms"]], ws, "cuda")
    m.update(step_ms=step_ms, idx_ms=idx_ms)
    value = whole_job_rate(ws, wl.batch, steps, step_ms)
    e2e_value = whole_job_rate(ws, wl.batch, steps, e2e_ms)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": steps, "warmup": warm,
        "ms_per_step": step_ms / steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32 on fp32" if workload_fmt(wl) == "f32" else "f32 on mxfp4/fp8/bf16", "data": "synthetic",
        "config": workload_config(wl, ws, args.select),
        "gpu_launches": m["launches"],
        "step_breakdown_us": m["breakdown"],
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(m["h2d"]),
                "d2h_bytes_per_step": int(m["d2h"]), "phases_us": m["e2e_phases"], "through": m["e2e_api"]},
        "clocks": m["clocks"],
    }
    line.update(rooflines(wl, m, steps, args.select))
    if ws == 1 and args.others:
        others = {}
        o_steps = max(3, min(steps, 10))
        for name in OTHER_WORKLOADS:
            if name == wl.name:
                continue
            gc.collect()
            torch.cuda.empty_cache()
            wo = I.WORKLOADS[name]
            mo = measure(wo, rank, ws, o_steps, 3, with_e2e=False, select=args.select)
            rec = {"value": whole_job_rate(1, wo.batch, o_steps, mo["step_ms"]), "unit": UNIT,
                   "ms_per_step": mo["step_ms"] / o_steps, "steps": o_steps, "warmup": 3,
                   "config": workload_config(wo, 1, args.select), "step_breakdown_us": mo["breakdown"],
                   "gpu_launches": mo["launches"], "clocks": mo["clocks"]}
            rec.update(rooflines(wo, mo, o_steps, args.select))
            others[name] = rec
        line["other_workloads"] = others
        gc.collect()
        torch.cuda.empty_cache()
        line["projections"] = measure_projections()
        gc.collect()
        torch.cuda.empty_cache()
        line["prefill"] = measure_prefill(wl)
    if rank == 0 and args.cpu_baseline and ws == 1:
        line["cpu_baseline"] = cpu_baseline(wl, budget_s=args.cpu_budget)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()


# ---------------------------------------------------------------- oracle (CPU) arm

def _oracle_cache(wl, rng):
    """Stored rows in the oracle's format for one request of the workload
    (random valid codes: the oracle's cost does not depend on the values)."""
    from oracle import csa_oracle as O
    T = wl.context + 1
    N = T // 4 if wl.kind == "csa" else T // 128
    fp8 = rng.integers(0, 0x7E, (N, wl.D - wl.R), dtype=np.uint8) | (rng.integers(0, 2, (N, 1)) << 7).astype(np.uint8)
    rope = O.bf16_bits_from_f32(rng.standard_normal((N, wl.R)).astype(np.float32))
    scale = (np.abs(rng.standard_normal(N)) / 448 + 1e-3).astype(np.float32)
    kv = O.KVRow(fp8=fp8, rope=rope, scale=scale)
    keys = None
    if wl.kind == "csa":
        keys = O.MXFP4(codes=rng.integers(0, 16, (N, wl.d_I), dtype=np.uint8),
                       scales=rng.integers(124, 130, (N, wl.d_I // 32), dtype=np.uint8))
    win = O.quantize_kv(rng.standard_normal((min(T, 128), wl.D)), wl.R)
    return kv, keys, win, T


def oracle_setup(wl):
    """Untimed set-up of the oracle arm: one request's stored rows."""
    from oracle import csa_oracle as O
    rng = np.random.default_rng(wl.seed)
    kv, keys, win, T = _oracle_cache(wl, rng)
    p = O.LayerParams(wl.kind, wl.D, wl.R, np.zeros((8, wl.D)), np.zeros((8, wl.d_I or 32)),
                      m=4 if wl.kind == "csa" else 128)
    return dict(p=p, kv=kv, keys=keys, win=win, T=T, rng=rng)


def oracle_queries(wl, setup, n: int | None = None, budget_s: float | None = None):
    """Run the fp64 oracle, as it stands, on decode queries of the workload
    (index scan, top-k and attention over one request's stored rows).
    Returns (queries done, seconds)."""
    from oracle import csa_oracle as O
    rng = setup["rng"]
    done, t0 = 0, time.perf_counter()
    while True:
        q = I.bf16_grid(rng.standard_normal((wl.H, wl.D)).astype(np.float32))
        qi = rng.standard_normal((wl.H_I, wl.d_I)).astype(np.float32) if wl.kind == "csa" else None
        w = rng.standard_normal(wl.H_I).astype(np.float32) if wl.kind == "csa" else None
        O.decode_query(setup["p"], None, q, rng.standard_normal(wl.H), k=wl.k, q_idx=qi, w=w,
                       entries=(setup["kv"], setup["keys"]), window=setup["win"], T=setup["T"])
        done += 1
        el = time.perf_counter() - t0
        if (n is not None and done >= n) or (n is None and el >= budget_s):
            return done, el


def _cores():
    try:
        from threadpoolctl import threadpool_info
        return int(max([d.get("num_threads", 1) for d in threadpool_info()] + [1]))
    except Exception:
        return os.cpu_count()


def _sample_text(wl, done, el):
    n_ent = (wl.context + 1) // 4 if wl.kind == "csa" else (wl.context + 1) // 128
    return (f"{done} decode queries of the {wl.name} workload on one request's stored rows "
            f"({n_ent} compressed entries + 128-token window; index scan, top-k and attention in "
            f"fp64 numpy), {el:.1f} s")


def cpu_baseline(wl, budget_s: float = 15.0):
    setup = oracle_setup(wl)
    done, el = oracle_queries(wl, setup, budget_s=budget_s)
    return {"value": done / el, "unit": UNIT, "cores": _cores(), "kind": "oracle",
            "sample": _sample_text(wl, done, el)}


def run_reference(args):
    """The oracle, as it stands, timed on the host cores.  A step is a
    bounded sample of the workload: q queries of one request (q <= batch,
    chosen from the warm-up so that the whole run stays within ~3 minutes)."""
    ws, rank, _ = _dist()
    if rank != 0:
        return
    wl = I.WORKLOADS[args.workload]
    setup = oracle_setup(wl)
    _, el_w = oracle_queries(wl, setup, n=args.warmup)       # untimed warm-up queries
    per_q = el_w / max(args.warmup, 1)
    q_step = max(1, min(wl.batch, int(180.0 / max(per_q * args.steps, 1e-9))))
    done, el = oracle_queries(wl, setup, n=args.steps * q_step)
    value = done / el
    sample = _sample_text(wl, done, el) + f"; {q_step} quer{'y' if q_step == 1 else 'ies'} per step"
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": el * 1e3 / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": workload_config(wl, ws),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": _cores(), "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="csa-pro-1m", choices=sorted(I.WORKLOADS))
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--select", default="separate", choices=["fused", "separate"],
                    help="CSA selection: csa_index_scores + csa_topk (two launches, the faster on one "
                         "B200) or csa_index_topk (one cooperative launch)")
    ap.add_argument("--no-other-workloads", dest="others", action="store_false",
                    help="skip the other configurations measured beside the headline at N = 1")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
