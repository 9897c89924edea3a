#!/usr/bin/env python
"""Benchmark of one sparse decode step (top-k token-level sparse attention under GQA, JSSA-style).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

A step is the whole hot path for one batch: projection-and-append of the newest key, then the
decode step (group-mean query, projected score scan with top-k per KV head, gather-free split-K
attention and combine) through the C ABI.  Inputs are seeded synthetic tensors resident in
HBM.  Rank 0 prints one JSON line.  Multi-GPU runs (torchrun) are independent replicas of
the workload on every rank (no data-path collective): weak scaling, time = max over ranks.
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
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sparse decode steps/s & achieved HBM GB/s at N=128K, B=1/16; speedup vs dense"
UNIT = "steps/s"
DEFAULT_WORKLOAD = "long-128k-b16"
SECONDARY_WORKLOAD = "long-128k-b1"
FP8_WORKLOAD = "long-128k-b16-fp8"
# kernels one step launches: append, score scan, selection, split attention, split merge
STEP_KERNELS = 5
L2_BYTES = 126 * 1024 * 1024


# ------------------------------------------------------------------------------ accounting
NOMINAL_HBM_GBS = 8000.0


def roofline_bytes(B, Hq, Hkv, d, r, seqlens, ks, lam, kp_bytes=2):
    """Algorithmic HBM bytes of one step, per kernel and in total.

    Per (sequence b, KV head): N_b*r*kp_bytes (projected cache scan; 2 for bf16, 1 for FP8) +
    k_b*2*d*2 (selected K and V rows) + G*d*2 (queries) + G*d*4 (fp32 output) [+ N_b*4 gate
    inputs when lambda != 0].
    """
    G = Hq // Hkv
    kproj = sum(int(n) * r * kp_bytes for n in seqlens) * Hkv
    kv = sum(min(int(k), int(n)) * 2 * d * 2 for n, k in zip(seqlens, ks)) * Hkv
    q = B * Hq * d * 2
    out = B * Hq * d * 4
    lg = sum(int(n) * 4 for n in seqlens) * Hkv if lam != 0.0 else 0
    lg_sel = sum(min(int(k), int(n)) * 4 for n, k in zip(seqlens, ks)) * Hkv if lam != 0.0 else 0
    return {
        "score": kproj + q + lg,
        "select": 0,
        "attend": kv + q + out + lg_sel,
        "step": kproj + kv + q + out + lg,
        "kproj": kproj, "kv": kv,
    }


def dense_bytes(B, Hq, Hkv, d, seqlens):
    return sum(int(n) * 2 * d * 2 for n in seqlens) * Hkv + B * Hq * d * 2 + B * Hq * d * 4


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def kernel_source_sha(name):
    path = os.path.join(ROOT, "token_level_sparse_head_b200", "csrc", name)
    h = hashlib.sha256()
    for p in (path, os.path.join(ROOT, "token_level_sparse_head_b200", "csrc", "sas_device.cuh")):
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_file, workload):
    """DRAM bytes per launch from the committed ncu summary, if it matches the current source."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
        e = t[kernel_file][workload]
        if e.get("source_sha") == kernel_source_sha(kernel_file):
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


# ------------------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_id: str):
        self.proc = None
        self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", device_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=self.tmp, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.06)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.tmp.flush()
        rows = []
        with open(self.tmp.name) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 8:
                    rows.append(parts)
        os.unlink(self.tmp.name)
        if not rows:
            return None
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def smi_device_id(torch, dev):
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        return vis.split(",")[dev] if vis else str(dev)


# ------------------------------------------------------------------------------ our arm
class Workload:
    def __init__(self, name, device, torch, batch=None):
        from synth import CONFIGS, make_config
        from token_level_sparse_head_b200 import DecodeSession, lib, shape_of

        self.name = name
        self.torch = torch
        self.lib = lib
        p = make_config(name, device=device, **({"B": batch} if batch else {}))
        self.p = p
        self.shape = shape_of(p)
        self.sess = DecodeSession(self.shape, p.k_max, device=device)
        self.fp8 = p.kproj_scale is not None
        kdt = torch.uint8 if self.fp8 else torch.bfloat16   # FP8 E4M3 codes or bf16 values
        if p.paged:
            self.kproj = torch.zeros(p.num_pages, p.Hkv, 64, p.r, dtype=kdt, device=device)
        else:
            self.kproj = torch.zeros(p.B, p.Hkv, p.n_cap, p.r, dtype=kdt, device=device)
        lib.sas_build_proj_cache(self.shape, p.K, p.M, self.kproj, p.page_table, p.seqlens)
        # the newest key of every sequence (position N_b - 1), for the append of each step
        sl = p.seqlens.tolist()
        knew = torch.empty(p.B, p.Hkv, p.d, dtype=torch.bfloat16, device=device)
        for b, n in enumerate(sl):
            if p.paged:
                pg = int(p.page_table[b, (n - 1) // 64])
                knew[b] = p.K[pg, :, (n - 1) % 64]
            else:
                knew[b] = p.K[b, :, n - 1]
        self.knew = knew
        self.seqlens_h = sl
        self.ks_h = p.k.tolist()
        self.bytes = roofline_bytes(p.B, p.Hq, p.Hkv, p.d, p.r, sl, self.ks_h, p.lam, kp_bytes=1 if self.fp8 else 2)
        self.dense_bytes = dense_bytes(p.B, p.Hq, p.Hkv, p.d, sl)
        self.cfg = dict(CONFIGS[name])

    def step(self):
        p, L = self.p, self.lib
        L.sas_append_proj(self.shape, self.knew, p.M, self.kproj, p.page_table, p.seqlens)
        L.sas_decode_step(self.shape, p.q, p.M, self.kproj, p.K, p.V, p.page_table, p.seqlens, p.k, p.k_max,
                          p.lam, p.log_g, self.sess.out, self.sess.idx, self.sess.workspace, self.sess.ws_bytes)

    def step_parts(self, ev):
        """The same step through the component entry points, with events between kernels."""
        p, L, s = self.p, self.lib, self.sess
        ev[0].record()
        L.sas_append_proj(self.shape, self.knew, p.M, self.kproj, p.page_table, p.seqlens)
        ev[1].record()
        L.sas_score_scan(self.shape, p.q, p.M, self.kproj, p.page_table, p.seqlens, p.k, p.k_max, p.lam, p.log_g,
                         None, s.workspace, s.ws_bytes)
        ev[2].record()
        L.sas_select_from_scores(self.shape, p.seqlens, p.k, p.k_max, s.idx, s.workspace, s.ws_bytes)
        ev[3].record()
        L.sas_sparse_attention(self.shape, p.q, p.K, p.V, p.page_table, p.seqlens, s.idx, p.k, p.k_max, p.lam,
                               p.log_g, s.out, s.workspace, s.ws_bytes)
        ev[4].record()

    def parts(self):
        """The step's four component calls (append, score scan, selection, attention with its split
        merge) as separate entry-point calls."""
        p, L, s = self.p, self.lib, self.sess
        return {
            "append": lambda: L.sas_append_proj(self.shape, self.knew, p.M, self.kproj, p.page_table, p.seqlens),
            "score": lambda: L.sas_score_scan(self.shape, p.q, p.M, self.kproj, p.page_table, p.seqlens, p.k,
                                              p.k_max, p.lam, p.log_g, None, s.workspace, s.ws_bytes),
            "select": lambda: L.sas_select_from_scores(self.shape, p.seqlens, p.k, p.k_max, s.idx, s.workspace,
                                                       s.ws_bytes),
            "attend": lambda: L.sas_sparse_attention(self.shape, p.q, p.K, p.V, p.page_table, p.seqlens, s.idx,
                                                     p.k, p.k_max, p.lam, p.log_g, s.out, s.workspace, s.ws_bytes),
        }

    def dense(self):
        p = self.p
        self.lib.sas_dense_decode(self.shape, p.q, p.K, p.V, p.page_table, p.seqlens, self.sess.out,
                                  self.sess.workspace, self.sess.ws_bytes)

    def free(self):
        del self.p, self.kproj, self.sess, self.knew
        self.torch.cuda.empty_cache()


def max_over_ranks(t, dist=None):
    """The slowest rank's time (every rank gets it); t itself without a process group."""
    if dist is None:
        return t
    import torch

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    tt = torch.tensor([t], dtype=torch.float64, device=dev)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt.item())


def job_throughput(steps, world, t_max):
    """Whole-job steps/s: every rank ran `steps` steps of its own replica in at most t_max s."""
    return steps * world / t_max


def timed_block(torch, fn, steps, dist=None):
    """Time `steps` calls of fn as one block: barrier + sync on both sides, CUDA events on the
    current stream; returns the max over ranks of the elapsed seconds."""
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    return max_over_ranks(e0.elapsed_time(e1) / 1e3, dist)


def step_distribution(torch, fn, min_steps=50, min_seconds=1.0, flush_buf=None):
    """Per-step device times of fn (CUDA events around each call), over at least min_steps
    calls and at least min_seconds of calls; an L2 flush before each call when flush_buf is
    given.  Returns {median, p10, p90, mean, n} in milliseconds."""
    ts = []
    t_end = time.perf_counter() + min_seconds
    chunk = 50
    while len(ts) < min_steps or time.perf_counter() < t_end:
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(chunk)]
        for e0, e1 in evs:
            if flush_buf is not None:
                flush_l2(flush_buf)
            e0.record()
            fn()
            e1.record()
        torch.cuda.synchronize()
        ts.extend(e0.elapsed_time(e1) for e0, e1 in evs)
        if len(ts) >= 200000:
            break
    ts.sort()
    q = lambda f: ts[min(len(ts) - 1, int(f * (len(ts) - 1) + 0.5))]
    return {"median": q(0.5), "p10": q(0.1), "p90": q(0.9), "mean": statistics.mean(ts), "n": len(ts)}


def flush_l2(flush_buf):
    """Evict L2: write a buffer twice the L2 size, then read it back, so the lines left in L2
    are clean and the timed step does not pay for the flush's write-back."""
    flush_buf.zero_()
    flush_buf.sum()


def flushed_steps(torch, fn, steps, flush_buf):
    """Per-step event timing with an L2 flush (write, then read, of 2x the L2 size) between steps."""
    ts = []
    for _ in range(steps):
        flush_l2(flush_buf)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) / 1e3)
    return statistics.median(ts)


def selection_recall(torch, wl, gate=True):
    """Oracle top-k recall of the selection the last step made: the mean over (sequence, KV head)
    of |selected set  ∩  exact top-k| / k, where the exact set ranks the full-dimension key
    sigma * q-bar . k_i (+ lambda * log g_i when `gate` and the workload is gated).  Sequences
    whose budget covers them are skipped.  A report, not a check."""
    p = wl.p
    G = p.Hq // p.Hkv
    idx = wl.sess.idx
    lam = float(getattr(p, "lam", 0.0) or 0.0)
    rec = []
    for b in range(p.B):
        n = int(wl.seqlens_h[b])
        k = min(int(wl.ks_h[b]), n)
        if k <= 0 or k >= n:
            continue
        for h in range(p.Hkv):
            if p.paged:
                pages = p.page_table[b, :(n + 63) // 64].long()
                rows = p.K[pages, h].reshape(-1, p.K.shape[-1])[:n]
            else:
                rows = p.K[b, h, :n]
            qbar = p.q[b, h * G:(h + 1) * G].float().mean(0)
            key = (rows.float() @ qbar) / math.sqrt(rows.shape[-1])
            if gate and lam != 0.0:
                key = key + lam * p.log_g[b, h, :n].float()
            exact = torch.topk(key, k).indices
            sel = idx[b, h, :k].long()
            rec.append(float(torch.isin(sel, exact).sum()) / k)
    return statistics.mean(rec) if rec else None


def run_recall_report(args):
    """One line per named workload: the oracle top-k recall of one decode step's selection."""
    import torch

    from synth import CONFIGS

    torch.cuda.set_device(0)
    for name in CONFIGS:
        wl = Workload(name, "cuda:0", torch)
        wl.step()
        torch.cuda.synchronize()
        p = wl.p
        line = {"report": "selection_recall", "workload": name, "B": p.B, "N_max": max(wl.seqlens_h),
                "k_max": p.k_max, "r": p.r, "d": p.d, "lam": p.lam, "fp8_kproj": wl.fp8,
                "recall": selection_recall(torch, wl)}
        if p.lam:
            line["recall_vs_ungated_score"] = selection_recall(torch, wl, gate=False)
        print(json.dumps(line), flush=True)
        wl.free()
        del wl


def capture_graph(torch, fn):
    """fn captured into a CUDA graph (the library's calls allocate nothing and never synchronise,
    so a step can be captured as it is); None if capture is not possible here."""
    try:
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            fn()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        torch.cuda.synchronize()
        return g
    except Exception as e:  # report, keep the stream-launch numbers
        print(f"# graph capture unavailable: {e}", file=sys.stderr)
        return None


def run_ours(args):
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as tdist

        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=torch.device("cuda", local))
        dist = tdist
    dev = f"cuda:{local}"
    peak, peak_kind = measured_peaks()

    wl = Workload(args.workload, dev, torch, batch=args.batch)
    p = wl.p
    for _ in range(args.warmup):
        wl.step()
    torch.cuda.synchronize()

    # --- headline: K steps of sas_append_proj + sas_decode_step, inputs resident in HBM, replayed
    # from a CUDA graph of the step (as a decode server runs it); the same K steps launched
    # call by call are reported beside it
    graph = capture_graph(torch, wl.step)
    replay = graph.replay if graph is not None else wl.step
    t_stream = timed_block(torch, wl.step, args.steps, dist)
    # clocks are sampled over a window of at least a second under load: the per-step
    # distribution (each replay between two events) and then the headline block itself
    sampler = ClockSampler(smi_device_id(torch, local))
    dist_ms = step_distribution(torch, replay, min_steps=50, min_seconds=args.dist_seconds)
    t = timed_block(torch, replay, args.steps, dist)
    clocks = sampler.stop()
    ms = t / args.steps * 1e3
    value = job_throughput(args.steps, world, t)

    # --- per-kernel durations (component entry points, events between the kernels)
    nk = max(3, min(args.steps, 200))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(nk)]
    torch.cuda.synchronize()
    for i in range(nk):
        wl.step_parts(evs[i])
    torch.cuda.synchronize()
    names = ("append", "score", "select", "attend")
    k_ms = {nm: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs) for i, nm in enumerate(names)}
    dom = max(("score", "attend"), key=lambda nm: k_ms[nm])  # the kernels with algorithmic HBM bytes
    dom_bytes = wl.bytes[dom]
    head_bytes = dict(wl.bytes)
    head_dense_bytes = wl.dense_bytes
    achieved = dom_bytes / (k_ms[dom] * 1e-3) / 1e9
    traffic = recorded_traffic({"score": "score.cu", "select": "select.cu", "attend": "attend.cu"}[dom], args.workload)

    recall = selection_recall(torch, wl)

    # --- gather-then-attend foil on the same selected rows: copy the rows, then dense decode
    foil = None
    if not args.no_foil:
        from token_level_sparse_head_b200 import DecodeSession, lib as L

        Kg = torch.empty(p.B, p.Hkv, p.k_max, p.d, dtype=torch.bfloat16, device=dev)
        Vg = torch.empty_like(Kg)
        counts = torch.empty(p.B, dtype=torch.int32, device=dev)
        gshape = L.Shape(p.B, p.Hq, p.Hkv, p.d, p.r, p.k_max)
        gsess = DecodeSession(gshape, p.k_max, device=dev)
        gout = torch.empty_like(wl.sess.out)
        idx_sel = wl.sess.idx

        def gather():
            L.sas_gather_selected(wl.shape, p.K, p.V, p.page_table, p.seqlens, idx_sel, p.k, p.k_max, Kg, Vg, counts)

        def attend_gathered():
            gsess.dense(p.q, Kg, Vg, None, counts, out=gout)

        nf = max(5, min(args.steps, 100))
        evf = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(nf)]
        for _ in range(3):
            gather()
            attend_gathered()
        torch.cuda.synchronize()
        for i in range(nf):
            evf[i][0].record()
            gather()
            evf[i][1].record()
            attend_gathered()
            evf[i][2].record()
        torch.cuda.synchronize()
        g_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evf)
        a_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evf)
        foil = {"gather_ms": g_ms, "attend_gathered_ms": a_ms, "total_ms": g_ms + a_ms,
                "gather_free_attend_ms": k_ms["attend"], "gather_free_speedup": (g_ms + a_ms) / k_ms["attend"],
                "note": "same selected rows; gather copies them to a contiguous buffer, then dense decode"}
        del Kg, Vg, gsess

    # --- dense full-KV baseline on the same workload
    for _ in range(2):
        wl.dense()
    nd = max(3, min(args.steps // 10, 50))
    td = timed_block(torch, wl.dense, nd, dist)
    dense_ms = td / nd * 1e3

    # --- end to end through the C ABI with host buffers (pinned), copies inside the timed region
    q_host = torch.empty_like(p.q, device="cpu").pin_memory()
    q_host.copy_(p.q)
    knew_host = torch.empty_like(wl.knew, device="cpu").pin_memory()
    knew_host.copy_(wl.knew)
    out_host = torch.empty_like(wl.sess.out, device="cpu").pin_memory()

    def e2e_step():
        p.q.copy_(q_host, non_blocking=True)
        wl.knew.copy_(knew_host, non_blocking=True)
        wl.step()
        out_host.copy_(wl.sess.out, non_blocking=True)
        torch.cuda.current_stream().synchronize()

    for _ in range(3):
        e2e_step()
    ne = max(3, min(args.steps, 200))
    te = timed_block(torch, e2e_step, ne, dist)
    e2e = {"value": job_throughput(ne, world, te), "unit": UNIT,
           "h2d_bytes_per_step": q_host.numel() * 2 + knew_host.numel() * 2,
           "d2h_bytes_per_step": out_host.numel() * 4}

    # --- secondary workload: B = 1 at 128K (L2 flushed between steps; its 84 MB fit in L2)
    secondary = None
    if not args.no_secondary and args.workload == DEFAULT_WORKLOAD:
        wl.free()
        del wl
        w1 = Workload(SECONDARY_WORKLOAD, dev, torch)
        flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
        for _ in range(3):
            w1.step()
        n1 = max(10, min(args.steps, 100))
        t1_stream = flushed_steps(torch, w1.step, n1, flush)
        g1 = capture_graph(torch, w1.step)
        d1 = step_distribution(torch, g1.replay if g1 is not None else w1.step, min_steps=100, min_seconds=0.3,
                               flush_buf=flush)
        t1 = d1["median"] * 1e-3
        gd1 = capture_graph(torch, w1.dense)
        td1 = flushed_steps(torch, gd1.replay if gd1 is not None else w1.dense, 10, flush)
        # each kernel alone, replayed from its own graph after an L2 flush
        kt = {}
        for kname, fn in w1.parts().items():
            gk = capture_graph(torch, fn)
            kt[kname] = flushed_steps(torch, gk.replay if gk is not None else fn, 20, flush) * 1e3
        secondary = {"workload": SECONDARY_WORKLOAD, "ms_per_step": t1 * 1e3, "steps_per_s": 1.0 / t1,
                     "ms_per_step_stream": t1_stream * 1e3, "p10": d1["p10"], "p90": d1["p90"], "n": d1["n"],
                     "hbm_gbs": w1.bytes["step"] / t1 / 1e9, "dense_ms_per_step": td1 * 1e3,
                     "speedup_vs_dense": td1 / t1, "l2": "flushed between steps (2x L2 written, then read)",
                     "timing": "CUDA graph replay of the step" if g1 is not None else "stream launches",
                     "kernels_ms": kt}
        wl = w1

    # --- the same 128K B=16 workload with the projected cache in FP8 E4M3 (the pages' setting)
    fp8 = None
    if not args.no_fp8 and args.workload == DEFAULT_WORKLOAD:
        wl.free()
        del wl
        w8 = Workload(FP8_WORKLOAD, dev, torch)
        for _ in range(3):
            w8.step()
        g8 = capture_graph(torch, w8.step)
        n8 = max(10, min(args.steps, 300))
        t8 = timed_block(torch, g8.replay if g8 is not None else w8.step, n8, dist)
        evs8 = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(20)]
        for i in range(20):
            w8.step_parts(evs8[i])
        torch.cuda.synchronize()
        k8 = {nm: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs8) for i, nm in enumerate(names)}
        ms8 = t8 / n8 * 1e3
        fp8 = {"workload": FP8_WORKLOAD, "ms_per_step": ms8, "steps_per_s": 1e3 / ms8,
               "hbm_gbs": w8.bytes["step"] / (ms8 * 1e-3) / 1e9, "step_bytes": w8.bytes["step"],
               "speedup_vs_bf16_kproj": ms / ms8, "kernels_ms": k8,
               "score_hbm_gbs": w8.bytes["score"] / (k8["score"] * 1e-3) / 1e9,
               "selection_recall": selection_recall(torch, w8),
               "timing": "CUDA graph replay of the step" if g8 is not None else "stream launches"}
        wl = w8

    # --- the other named workloads: 8B-shaped 32K, paged variable-length B=16, gated budget sweep
    others = None
    if not args.no_workloads and args.workload == DEFAULT_WORKLOAD:
        wl.free()
        del wl
        wl = None
        others = {name: time_workload(torch, name, dev) for name in OTHER_WORKLOADS}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.workload, budget_s=args.cpu_seconds)

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "ms_per_step_stream": t_stream / args.steps * 1e3,
        "ms_per_step_dist": dist_ms,
        "timing": "CUDA graph replay of the step" if graph is not None else "stream launches",
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "storage_dtype": "bf16", "data": "synthetic",
        "config": config_view(args.workload, world),
        "hbm_gbs": None, "speedup_vs_dense": dense_ms / ms,
        "dense": {"ms_per_step": dense_ms, "steps_per_s": 1e3 / dense_ms},
        "kernels_ms": k_ms,
        "roofline": {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": peak_kind,
                     "algorithmic_bytes_per_launch": dom_bytes, "traffic": traffic},
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": STEP_KERNELS * args.steps, "clocks": clocks,
    }
    line["hbm_gbs"] = head_bytes["step"] / (ms * 1e-3) / 1e9
    line["step_roofline_frac"] = line["hbm_gbs"] / peak
    # the same step against the nominal B200 HBM3e figure (about 8 TB/s), for context
    line["step_frac_of_nominal_8tbs"] = line["hbm_gbs"] / NOMINAL_HBM_GBS
    line["dense"]["hbm_gbs"] = head_dense_bytes / (dense_ms * 1e-3) / 1e9
    if secondary:
        line["b1"] = secondary
    if fp8:
        line["fp8_kproj"] = fp8
    if foil:
        line["gather_foil"] = foil
    if others:
        line["workloads"] = others
    line["selection_recall"] = {"value": recall, "definition": "mean over (sequence, KV head) of the fraction of "
                                "the exact top-k by q-bar . k_i (full dimension) that the projected selection keeps; "
                                "synthetic data"}
    print(json.dumps(line), flush=True)


OTHER_WORKLOADS = ("8b-32k", "paged-b16", "gated-b4-k256", "gated-b4-k1024", "gated-b4-k4096", "gated-b4-k16384")


def workload_bytes(name):
    """Roofline bytes of one step of a named workload from its definition (the paged workload:
    at the mean sequence length of its uniform draw)."""
    from synth import CONFIGS

    c = CONFIGS[name]
    kp = 1 if c.get("kproj_fp8") else 2
    n = c["N"] if c["N"] else (c["n_lo"] + c["n_hi"]) / 2
    k = c["k"] if c["k"] else n / c["k_div"]
    return roofline_bytes(c["B"], c["Hq"], c["Hkv"], c["d"], c["r"], [n] * c["B"], [k] * c["B"],
                          c.get("lam", 0.0), kp_bytes=kp)["step"]


def l2_policy(step_bytes):
    """Steps that read less than twice the L2 are timed with an L2 flush before each step."""
    return step_bytes < 2 * L2_BYTES


def config_view(name, world):
    """The config dict both arms print for a workload: its shape, the L2 treatment of the timing
    and the parallelism."""
    from synth import CONFIGS

    c = dict(CONFIGS[name])
    v = {k: c[k] for k in ("B", "Hq", "Hkv", "d", "r", "N", "k") if k in c}
    if c.get("lam"):
        v["lam"] = c["lam"]
    if c.get("paged"):
        v.update(n_lo=c["n_lo"], n_hi=c["n_hi"], k="N_b/%d" % c["k_div"], page_size=64)
    if c.get("kproj_fp8"):
        v["kproj"] = "fp8_e4m3"
    step = workload_bytes(name)
    v["l2"] = (f"L2 flushed before each step (a step reads {step / 1e9:.3f} GB, L2 is 0.13 GB)" if l2_policy(step)
               else f"inputs larger than L2: each step reads {step / 1e9:.2f} GB, L2 is 0.13 GB")
    v["parallelism"] = f"replicas x{world}"
    return dict(workload=name, **v)


def time_workload(torch, name, dev):
    """One named workload: the step (append + decode step, CUDA graph replay) and the dense decode,
    each as a median over replays, with its roofline bytes and bandwidth."""
    w = Workload(name, dev, torch)
    step_bytes = w.bytes["step"]
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev) if l2_policy(step_bytes) else None
    for _ in range(3):
        w.step()
    g = capture_graph(torch, w.step)
    st = step_distribution(torch, g.replay if g is not None else w.step, min_steps=50, min_seconds=0.2,
                           flush_buf=flush)
    gd = capture_graph(torch, w.dense)
    dn = step_distribution(torch, gd.replay if gd is not None else w.dense, min_steps=20, min_seconds=0.1,
                           flush_buf=flush)
    out = {"ms_per_step": st["median"], "p10": st["p10"], "p90": st["p90"], "steps_per_s": 1e3 / st["median"],
           "step_bytes": step_bytes, "hbm_gbs": step_bytes / (st["median"] * 1e-3) / 1e9,
           "dense_ms_per_step": dn["median"], "dense_hbm_gbs": w.dense_bytes / (dn["median"] * 1e-3) / 1e9,
           "speedup_vs_dense": dn["median"] / st["median"],
           "l2": "flushed before each step" if flush is not None else "inputs larger than L2",
           "timing": "median of CUDA graph replays"}
    del g, gd, flush
    w.free()
    del w
    return out


# ------------------------------------------------------------------------------ oracle arm
# The oracle runs one (sequence, KV head) pair at a time; a step is every pair of the workload.
# Pairs are independent, so a pool of single-threaded worker processes (spawned, so nothing of
# a CUDA context is inherited) takes them in parallel.  Each worker holds one seeded draw of the
# workload's pair shape and runs the oracle on it for every pair it is handed: the oracle's
# arithmetic does not depend on the values.
_ORACLE_PAIR = None


def _oracle_worker_init(name):
    import multiprocessing

    global _ORACLE_PAIR
    ident = multiprocessing.current_process()._identity
    _ORACLE_PAIR = oracle_head_problem(name, seed=2000 + (ident[0] if ident else 0))


def _oracle_worker_run(_):
    return oracle_head_seconds(_ORACLE_PAIR)


class OraclePool:
    """Worker processes for whole oracle steps of a workload."""

    THREAD_VARS = ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")

    def __init__(self, name, workers=None):
        import multiprocessing

        from synth import CONFIGS

        c = CONFIGS[name]
        self.pairs = c["B"] * c["Hkv"]
        self.workers = max(1, min(workers or (os.cpu_count() or 1), self.pairs, 32))
        saved = {k: os.environ.get(k) for k in self.THREAD_VARS}
        for k in self.THREAD_VARS:
            os.environ[k] = "1"  # every worker single-threaded: cores = workers
        try:
            self.pool = multiprocessing.get_context("spawn").Pool(self.workers, initializer=_oracle_worker_init,
                                                                 initargs=(name,))
        finally:
            for k, v in saved.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v

    def step(self):
        """Wall seconds of one step: the oracle on every (sequence, KV head) pair."""
        t0 = time.perf_counter()
        self.pool.map(_oracle_worker_run, range(self.pairs), chunksize=1)
        return time.perf_counter() - t0

    def close(self):
        self.pool.close()
        self.pool.join()

    def sample(self, steps):
        return (f"{steps} whole oracle steps; each step runs the oracle on all {self.pairs} (sequence, KV head) "
                f"pairs, spread over {self.workers} single-threaded worker processes, each holding one seeded "
                f"draw of the workload's pair")


def oracle_head_problem(name, seed):
    """One (sequence, KV head) of the named workload, drawn on the CPU (heads are independent
    and identically distributed), with its projected cache built by the oracle."""
    from oracle import sas_oracle as O
    from synth import CONFIGS, make_problem

    c = CONFIGS[name]
    G = c["Hq"] // c["Hkv"]
    n = c["N"] if c["N"] else (c["n_lo"] + c["n_hi"]) // 2
    k = c["k"] if c["k"] else n // c["k_div"]
    p = make_problem(B=1, Hq=G, Hkv=1, d=c["d"], r=c["r"], seqlens=[n], k=[k], lam=c.get("lam", 0.0),
                     basis=c["basis"], aniso=c["aniso"], seed=seed)
    f = lambda t: None if t is None else t.to(__import__("torch").float64).numpy()
    q, K, V, M = f(p.q)[0], f(p.K)[0, 0, :n], f(p.V)[0, 0, :n], f(p.M)[0]
    lg = None if p.log_g is None else f(p.log_g)[0, 0, :n]
    kp = O.project_keys(K, M)
    return dict(q=q, K=K, V=V, M=M, kp=kp, lg=lg, k=k, lam=c.get("lam", 0.0))


def oracle_head_seconds(h):
    from oracle import sas_oracle as O

    t0 = time.perf_counter()
    O.decode_head(h["q"], h["M"], h["kp"], h["K"], h["V"], h["k"], h["lam"], h["lg"])
    return time.perf_counter() - t0


def cpu_baseline(name, budget_s=15.0):
    """The oracle, as it stands, on whole steps of the workload for about budget_s seconds of CPU
    time (wall time x workers), at least one step."""
    pool = OraclePool(name)
    try:
        pool.step()  # warm-up: workers have loaded their pair
        ts = []
        while not ts or (sum(ts) * pool.workers < budget_s and len(ts) < 1000):
            ts.append(pool.step())
    finally:
        pool.close()
    per_step = statistics.mean(ts)
    return {"value": 1.0 / per_step, "unit": UNIT, "cores": pool.workers, "kind": "oracle",
            "sample": pool.sample(len(ts)), "ms_per_step": per_step * 1e3}


def run_reference(args):
    """The reference arm: the oracle (numpy, fp64) on whole steps of the workload on the host
    cores, --warmup untimed steps then --steps timed ones; rank 0 only."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    pool = OraclePool(args.workload)
    try:
        for _ in range(args.warmup):
            pool.step()
        ts = [pool.step() for _ in range(args.steps)]
    finally:
        pool.close()
    total = sum(ts)
    value = args.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_view(args.workload, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": pool.workers, "kind": "oracle",
                         "sample": pool.sample(args.steps)},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--batch", type=int, default=None, help="override the workload's batch (profiling)")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-fp8", action="store_true", help="skip the FP8 projected-cache line")
    ap.add_argument("--no-foil", action="store_true", help="skip the gather-then-attend line")
    ap.add_argument("--no-workloads", action="store_true", help="skip the other named workloads")
    ap.add_argument("--dist-seconds", type=float, default=1.0,
                    help="least wall time of the per-step distribution and clock window (0: 50 steps)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--recall-report", action="store_true",
                    help="print the selection recall of every named workload instead of timing")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.recall_report:
        run_recall_report(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
