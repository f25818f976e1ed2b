#!/usr/bin/env python
"""Benchmark of the ParisKV decode-time retrieval path on B200.

One *step* = pk_search + pk_attend for every (sequence, KV head) pair of one
decoder layer: query preparation, collision scan, candidate compaction +
4-bit rerank + Top-k, and gather + exact attention, on a fresh query.

Default workload (the metric's 128K point): 8 sequences x n = 131072 keys,
8 KV heads, 32 query heads, head_dim 128, bf16 K/V in HBM, Top-100, ratio-table
budgets.  The line also carries the metric's 1M point (n = 1048576, 8 KV
heads, K/V in pinned host memory read through UVA) under "million_token".

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload throughput|million|llama|tiny|drift|sweep|longgen|heads] [--no-million]
                  [--no-cpu-baseline] [--no-e2e] [--no-dense] [--graph] [--drift-steps T]

For N > 1 launch under torch.distributed.run: every rank runs its own copy of
the workload (pairs shard with no data-path collective: weak scaling); the
time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("retrieval+attend steps/sec per layer (all KV heads) at 128K and 1M; "
          "HBM % peak; Recall@100")
L2_BYTES = 126 * 1024 * 1024
FLUSH_BYTES = 256 * 1024 * 1024

WORKLOADS = {
    "throughput": dict(name="throughput_8x131072", batch=8, n=131072, H=8, G=4, cand=0, kv_host=False),
    "million": dict(name="million_1x1048576_uva", batch=1, n=1 << 20, H=8, G=4, cand=0, kv_host=True),
    "llama": dict(name="llama_1x32768", batch=1, n=32768, H=8, G=4, cand=2048, kv_host=False),
    "tiny": dict(name="tiny_1x4096", batch=1, n=4096, H=1, G=1, cand=512, kv_host=False),
    # Recall@100 and step time over a grid of candidate / collision ratios
    "sweep": dict(name="ratio_sweep", batch=1, n=0, H=8, G=4, cand=0, kv_host=False,
                  ns=(32768, 131072, 524288, 1048576), betas=(0.02, 0.05, 0.1, 0.2),
                  rhos=(0.05, 0.1, 0.2, 0.35, 0.5), queries=8),
    # aggregated vs per-query-head retrieval on the throughput shape
    "heads": dict(name="heads_8x131072", batch=8, n=131072, H=8, G=4, cand=0, kv_host=False, queries=16),
    # the same with K/V in pinned host memory: the per-head attention gathers
    # the union of a pair's lists once; timed alone on lists made to overlap
    "heads_uva": dict(name="heads_uva_8x131072", batch=8, n=131072, H=8, G=4, cand=0, kv_host=True, queries=8),
    # sink / local / update-buffer decoding after an 8 x 131072 prefill
    "longgen": dict(name="longgen_8x131072+1024", batch=8, n=131072, H=8, G=4, cand=0, kv_host=False,
                    steps=1024, sink=64, local=512, update=512),
    # prefill 65536 keys per KV head, then 16384 decode steps of append + search
    "drift": dict(name="drift_65536+16384", batch=1, n=65536, H=8, G=1, cand=0, kv_host=False,
                  steps=16384, recall_every=256),
}


# ----------------------------------------------------------------- helpers
def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="throughput", choices=sorted(WORKLOADS))
    ap.add_argument("--no-million", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--graph", action="store_true",
                    help="time one CUDA-graph launch per step instead of eager launches")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--drift-steps", type=int, default=0,
                    help="decode steps of the drift workload (default: all 16384)")
    return ap.parse_args()


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), \
        int(os.environ.get("LOCAL_RANK", 0))


def max_over_ranks(values, world: int, device=None):
    """Element-wise max of per-rank timings (one all-reduce, every rank calls
    it in the same order).  At world == 1 the values come back unchanged."""
    vals = [float(v) for v in values]
    if world <= 1:
        return vals
    import torch
    import torch.distributed as dist
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_rate(units_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job throughput: the units every rank processed over the slowest
    rank's time (weak scaling: each rank owns the same amount of work)."""
    return units_per_rank * world / (ms_max / 1000.0)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "MEASURED_PEAKS.json hbm_gbs (of measured)"
    return 6650.0, "fallback 6.65 TB/s (of fallback)"


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 50 ms."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,"
              "utilization.gpu")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="pk_clocks_", suffix=".csv")
            os.close(fd)
            cmd = ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits", "-lms", "50"]
            if self.uuid:
                cmd += ["--id=" + self.uuid]
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower().startswith("active")})

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        loaded = [r for r in rows if (num(r[8]) or 0) > 0] or rows
        sm = [num(r[0]) for r in loaded if num(r[0]) is not None]
        mx = [num(r[1]) for r in rows if num(r[1]) is not None]
        pw = [num(r[2]) for r in loaded if num(r[2]) is not None]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(pw) if pw else None, "reasons": reasons, "samples": len(rows),
                "samples_under_load": len(loaded)}


def src_hash(*names):
    h = hashlib.sha256()
    for nm in names:
        with open(os.path.join(ROOT, "kv_cache_top_b200", "csrc", nm), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` from a committed ncu summary in
    profiles/, or None when there is none or the kernel source changed since."""
    path = os.path.join(ROOT, "profiles", "%s_%s.md" % (kernel, workload))
    if not os.path.exists(path):
        return None
    txt = open(path).read()
    m = re.search(r"dram_bytes_per_full_launch:\s*([0-9.eE+]+)", txt)
    hm = re.search(r"source_sha256_16:\s*([0-9a-f]+)", txt)
    files = {"collision_scan": ["k_collision_scan.cu", "pk_internal.cuh"],
             "rerank_topk": ["k_rerank_topk.cu", "pk_internal.cuh"],
             "compact": ["k_compact.cu", "pk_internal.cuh"],
             "topk_merge": ["k_rerank_topk.cu", "pk_internal.cuh"],
             "query_prep": ["k_query_prep.cu", "pk_internal.cuh"],
             "gather_attend": ["k_gather_attend.cu", "pk_internal.cuh"]}.get(kernel)
    if not m or not hm or not files or hm.group(1) != src_hash(*files):
        return None
    return float(m.group(1))


def cpu_model() -> str:
    """The host CPU's model name (for the CPU-baseline lines)."""
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# -------------------------------------------------------- algorithmic bytes
def alg_bytes(kernel: str, wl: dict, C: int, topk: int = 100):
    """Bytes a launch must move at minimum (per launch, all pairs)."""
    bh, n, G = wl["batch"] * wl["H"], wl["n"], wl["G"]
    if kernel == "query_prep":
        return bh * (G * 128 * 2 + 16 * 256 * 4 + 16 * 32 * 4 + 128 * 4)
    if kernel == "collision_scan":
        return bh * (16 * n + n)                     # codes read + S written
    if kernel == "compact":
        return bh * (n + 4 * C)                      # S read + candidate ids written
    if kernel == "rerank_topk":
        return bh * (132 * C)                        # ids + candidate records
    if kernel == "topk_merge":
        return bh * 16 * topk * max(1, C // 1472)    # per-slice sets read + result (estimate)
    if kernel == "gather_attend":
        return bh * (2 * topk * 128 * 2 + G * 128 * (2 + 4))   # K/V rows + q + o
    raise KeyError(kernel)


# --------------------------------------------------------------- our arm
def run_ours(args, wl, rank, world, local_rank, want_cpu, peaks):
    import torch
    import kv_cache_top_b200 as pk
    import workloads

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    seed = args.seed + rank
    batch, n, H, G = wl["batch"], wl["n"], wl["H"], wl["G"]
    bh, topk, nq = batch * H, 100, 64
    w = workloads.llama_layer(batch, n, H=H, G=G, seed=seed, device=dev, n_queries=nq)
    n_app = 4096                                       # keys per pair appended after the timed passes
    p = pk.pk_default_params(batch=batch, n_kv_heads=H, group=G, topk=topk, cand_budget=wl["cand"],
                             kv_dtype=pk.PK_BF16, n_cap=n + n_app,
                             kv_location=pk.PK_KV_HOST_PINNED if wl["kv_host"] else pk.PK_KV_DEVICE)
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()
    t_b = time.perf_counter()
    h = pk.pk_build_index(w["K"], w["V"], n, p)
    torch.cuda.synchronize()
    build_s = time.perf_counter() - t_b
    k_app = torch.randn(batch, H, n_app, 128, device=dev).to(torch.bfloat16)
    C, R = pk.pk_resolve(n, wl["cand"], 0.0, topk)
    info = pk.pk_get_info(h)
    q = w["q"]
    idx = torch.empty(bh, topk, dtype=torch.int32, device=dev)
    score = torch.empty(bh, topk, dtype=torch.float32, device=dev)
    out = torch.empty(batch, H * G, 128, dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)

    # Recall@100 against exact Top-100 of <k_i, q_agg> (fp32 matmul, metric only)
    recalls = []
    for qi in range(4):
        pk.pk_search(h, q[qi], topk, idx, score)
        got = idx.cpu()
        qa = q[qi].float().view(batch, H, G, 128).sum(2)                     # [batch][H][D]
        for b in range(batch):
            for hh in range(H):
                s = w["K"][b, hh].float() @ qa[b, hh]
                ex = torch.topk(s, topk).indices.cpu()
                recalls.append(len(set(ex.tolist()) & set(got[b * H + hh].tolist())) / topk)
    recall = sum(recalls) / len(recalls)
    if wl["kv_host"]:
        del w["K"], w["V"]
        torch.cuda.empty_cache()

    def step(i):
        pk.pk_search(h, q[i % nq], topk, idx, score)
        pk.pk_attend(h, q[i % nq], idx, topk, out)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()

    # one CUDA graph per query of the pool: a step is then one graph launch
    # (the library's programmatic dependent launches become graph edges)
    graphs = None
    if args.graph:
        graphs = []
        for i in range(nq):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step(i)
            graphs.append(g)
        for i in range(min(args.warmup, nq)):
            graphs[i].replay()
        torch.cuda.synchronize()

    def timed_step(i, trace):
        if graphs is not None and not trace:
            graphs[i % nq].replay()
        else:
            step(i)

    sampler = ClockSampler(None)
    if rank == 0:
        try:
            sampler.uuid = str(torch.cuda.get_device_properties(dev).uuid)
            if not sampler.uuid.startswith("GPU-"):
                sampler.uuid = "GPU-" + sampler.uuid
        except Exception:
            sampler.uuid = None
        sampler.start()
        time.sleep(0.3)

    def timed_pass(trace: bool):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        if trace:
            pk.pk_trace_enable(h, True)
            pk.pk_trace_read(h)
        t0 = time.perf_counter()
        for i in range(args.steps):
            flush.zero_()                      # L2 flush outside the timed events
            evs[i][0].record(stream)
            timed_step(i, trace)
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        wall = time.perf_counter() - t0
        if world > 1:
            torch.distributed.barrier()
        ms = sum(a.elapsed_time(b) for a, b in evs)
        kern = None
        if trace:
            kern = pk.pk_trace_read(h)
            pk.pk_trace_enable(h, False)
        return ms, wall, kern

    ms_clean, wall_clean, _ = timed_pass(False)
    ms_traced, _, kern = timed_pass(True)

    # end-to-end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        q_host = q.cpu().pin_memory()
        q_dev = torch.empty_like(q[0])
        o_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()   # the step's result
        ks = min(args.steps, 500)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(ks)]
        torch.cuda.synchronize()
        for i in range(ks):
            flush.zero_()
            evs[i][0].record(stream)
            q_dev.copy_(q_host[i % nq], non_blocking=True)
            pk.pk_search(h, q_dev, topk, idx, score)
            pk.pk_attend(h, q_dev, idx, topk, out)
            o_host.copy_(out, non_blocking=True)
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        e2e_copy_ms = sum(a.elapsed_time(b) for a, b in evs)
        # the same calls given the pinned host buffers themselves: the kernels
        # read the query and write the output over the host link (UVA), so
        # no separate copy is launched
        o_host2 = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        torch.cuda.synchronize()
        for i in range(ks):
            flush.zero_()
            evs[i][0].record(stream)
            pk.pk_search(h, q_host[i % nq], topk, idx, score)
            pk.pk_attend(h, q_host[i % nq], idx, topk, o_host2)
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        e2e_uva_ms = sum(a.elapsed_time(b) for a, b in evs)
        assert torch.isfinite(o_host2).all()
        e2e = {"steps": ks, "ms_total": min(e2e_copy_ms, e2e_uva_ms),
               "copy_ms_total": e2e_copy_ms, "uva_ms_total": e2e_uva_ms,
               "h2d_bytes_per_step": q_dev.numel() * q_dev.element_size(),
               "d2h_bytes_per_step": out.numel() * 4}

    clocks = sampler.stop() if rank == 0 else None

    # max over ranks of the device times (every rank takes the same step)
    ms_clean, e2e_max = max_over_ranks([ms_clean, e2e["ms_total"] if e2e else 0.0], world, dev)
    if e2e:
        e2e = {"value": job_rate(e2e["steps"], world, e2e_max), "unit": "steps/s",
               "ms_per_step": e2e_max / e2e["steps"],
               "h2d_bytes_per_step": e2e["h2d_bytes_per_step"],
               "d2h_bytes_per_step": e2e["d2h_bytes_per_step"],
               "path": "the faster of two forms of the public calls with host buffers, both timed: "
                       "(copy) query copied in and output copied out around pk_search + pk_attend; "
                       "(uva) pk_search + pk_attend given the pinned host buffers, which the kernels "
                       "read and write over the host link",
               "copy_ms_per_step": e2e["copy_ms_total"] / e2e["steps"],
               "uva_ms_per_step": e2e["uva_ms_total"] / e2e["steps"]}

    # index build (host wall clock: allocation, K/V copy-in, encode) and the
    # encode kernel alone on one append of n_app keys per pair
    torch.cuda.synchronize()
    pk.pk_trace_enable(h, True)
    pk.pk_trace_read(h)
    pk.pk_append(h, k_app, k_app, n_app)
    enc = pk.pk_trace_read(h)["encode"]
    pk.pk_trace_enable(h, False)
    enc_us = enc[1] * 1000.0 / max(1, enc[0])
    keys_app = bh * n_app
    build = {"build_s_wall": build_s, "keys": bh * n,
             "build_keys_per_s": bh * n / build_s,
             "append_keys": keys_app, "encode_us": enc_us, "encode_keys_per_s": keys_app / (enc_us * 1e-6),
             "encode_gbs": keys_app * (128 * 2 + 16 + 128) / (enc_us * 1e-3) / 1e6,
             "encode_bytes_per_key": "256 B of K read + 144 B of codes and record written"}
    del k_app

    res = dict(ms_total=ms_clean, wall=wall_clean, kern=kern, recall=recall, C=C, R=R, info=info,
               e2e=e2e, clocks=clocks, ms_traced=ms_traced, graph=graphs is not None, build=build)
    del graphs

    # dense-attention comparator on the same tensors (HBM workloads only)
    if rank == 0 and not wl["kv_host"] and not args.no_dense:
        try:
            import torch.nn.functional as F
            qd = q[0].view(batch, H * G, 1, 128)
            Kd, Vd = w["K"], w["V"]
            for _ in range(3):
                F.scaled_dot_product_attention(qd, Kd, Vd, enable_gqa=True)
            torch.cuda.synchronize()
            ds = []
            for _ in range(10):
                flush.zero_()
                a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a_.record(stream)
                F.scaled_dot_product_attention(qd, Kd, Vd, enable_gqa=True)
                b_.record(stream)
                torch.cuda.synchronize()
                ds.append(a_.elapsed_time(b_))
            dms = statistics.median(ds)
            res["dense"] = {"kind": "torch SDPA over all n keys (same K/V, same queries)",
                            "ms_per_step": dms, "steps_s": 1000.0 / dms,
                            "bytes_per_step": 2 * bh * n * 128 * 2,
                            "gbs": 2 * bh * n * 128 * 2 / dms / 1e6}
        except Exception as e:                  # comparator only; never the product
            res["dense"] = {"error": str(e)[:200]}

    # host-link reference (pinned H2D copy) for UVA workloads
    if rank == 0 and wl["kv_host"]:
        hb = torch.empty(256 << 20, dtype=torch.uint8).pin_memory()
        db = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        best = 1e9
        for _ in range(5):
            a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a_.record(stream)
            db.copy_(hb, non_blocking=True)
            b_.record(stream)
            torch.cuda.synchronize()
            best = min(best, a_.elapsed_time(b_))
        res["h2d_gbs"] = (256 << 20) / best / 1e6
        # the same pinned buffer read in place by a kernel over UVA (a torch
        # reduction over a device view of the host pointer): the contiguous
        # kernel-read rate of the host link
        hb.fill_(1)

        class _HostView:
            __cuda_array_interface__ = {"shape": (64 << 20,), "typestr": "<i4",
                                        "data": (hb.data_ptr(), False), "version": 3}
        hv = torch.as_tensor(_HostView(), device=dev)
        best = 1e9
        for _ in range(5):
            a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a_.record(stream)
            s_ = hv.sum()
            b_.record(stream)
            torch.cuda.synchronize()
            best = min(best, a_.elapsed_time(b_))
        assert int(s_) == (64 << 20) * 0x01010101
        res["uva_read_gbs"] = (256 << 20) / best / 1e6
        del hv, hb, db

    # CPU baseline: the oracle on a bounded sample of the same workload, on
    # one core and on all host cores
    if want_cpu:
        single = cpu_baseline(wl, seed, w if not wl["kv_host"] else None, dev)
        res["cpu"] = single
        try:
            par = cpu_baseline_parallel(wl, seed, queries=64 if wl["n"] <= 200000 else 4 * bh)
            par["single_core"] = single
            res["cpu"] = par
        except Exception as e:          # the one-core figure stands
            single["parallel_error"] = str(e)[:200]

    pk.pk_free(h)
    del w, flush
    torch.cuda.empty_cache()
    return res


def cpu_baseline(wl, seed, w, dev, pairs_wanted=4, queries=32):
    """Time the oracle (as it stands, 1 thread) on sampled pairs of the same
    workload: index build untimed, then search + attend per query."""
    import torch
    import oracle
    import workloads
    batch, n, H, G = wl["batch"], wl["n"], wl["H"], wl["G"]
    bh = batch * H
    pairs = sorted({(i * bh) // pairs_wanted for i in range(pairs_wanted)})
    if n > 200000:                      # one pair, 4 steps' worth of pair-searches (4 x bh)
        pairs, queries = pairs[:1], 4 * bh
    tot, cnt = 0.0, 0
    for pidx in pairs:
        b, hh = divmod(pidx, H)
        K, V, qq = workloads.llama_pair(b, hh, n, H=H, G=G, seed=seed, device=dev, n_queries=queries)
        Kn, Vn, qn = workloads.to_np_f32(K), workloads.to_np_f32(V), workloads.to_np_f32(qq)
        del K, V, qq
        enc = oracle.build_index(Kn)
        for i in range(queries):
            t0 = time.perf_counter()
            o = oracle.search(enc, qn[i], topk_k=100, cand_budget=wl["cand"])
            oracle.attend(qn[i], Kn, Vn, o["idx"], 1.0 / math.sqrt(128))
            tot += time.perf_counter() - t0
            cnt += 1
    per_pair = tot / cnt
    return {"value": 1.0 / (per_pair * bh), "unit": "steps/s", "cores": 1, "kind": "oracle", "cpu": cpu_model(),
            "sample": "%d of %d (sequence, KV head) pairs x %d queries each (%.1f s of timed "
                      "search+attend, index build untimed); one step = %d pair-searches" %
                      (len(pairs), bh, queries, tot, bh),
            "ms_per_pair": per_pair * 1000.0}


_barrier = None


def _oracle_worker_init(barrier):
    global _barrier
    _barrier = barrier


def _oracle_worker(job):
    """One host core: build one pair's oracle index (untimed), wait for the
    other workers, then time search + attend for `queries` queries."""
    pidx, wl, seed, queries = job
    import oracle
    import workloads
    b, hh = divmod(pidx, wl["H"])
    K, V, qq = workloads.llama_pair(b, hh, wl["n"], H=wl["H"], G=wl["G"], seed=seed, device="cpu",
                                    n_queries=queries)
    Kn, Vn, qn = workloads.to_np_f32(K), workloads.to_np_f32(V), workloads.to_np_f32(qq)
    del K, V, qq
    enc = oracle.build_index(Kn)
    _barrier.wait(timeout=600)
    t0 = time.perf_counter()
    for i in range(queries):
        o = oracle.search(enc, qn[i], topk_k=100, cand_budget=wl["cand"])
        oracle.attend(qn[i], Kn, Vn, o["idx"], 1.0 / math.sqrt(128))
    return queries, time.perf_counter() - t0


def cpu_baseline_parallel(wl, seed, queries=64, max_workers=32):
    """The oracle on all host cores: one process (spawn-started, so it is safe
    after GPU use) per core, each on its own sampled pair, all timing their
    searches at once.  Throughput = searches done / the slowest worker's time."""
    import multiprocessing as mp
    from concurrent.futures import ProcessPoolExecutor
    bh = wl["batch"] * wl["H"]
    P = max(1, min(os.cpu_count() or 1, max_workers, bh))
    ctx = mp.get_context("spawn")
    barrier = ctx.Barrier(P)
    jobs = [((i * bh) // P, wl, seed, queries) for i in range(P)]
    # a worker that dies raises here (BrokenProcessPool) instead of being respawned
    with ProcessPoolExecutor(P, mp_context=ctx, initializer=_oracle_worker_init, initargs=(barrier,)) as ex:
        res = list(ex.map(_oracle_worker, jobs, timeout=900))
    done = sum(r[0] for r in res)
    tmax = max(r[1] for r in res)
    return {"value": done / tmax / bh, "unit": "steps/s", "cores": P, "kind": "oracle", "cpu": cpu_model(),
            "sample": "%d processes, one (sequence, KV head) pair each, %d queries each, timed together "
                      "(%.1f s; index build untimed); one step = %d pair-searches" % (P, queries, tmax, bh)}


def kernel_table(kern, steps, wl, C, peak):
    tot = sum(v[1] for v in kern.values()) or 1.0
    out = {}
    for k, (nl, ms) in kern.items():
        if nl == 0:
            continue
        avg_ms = ms / nl
        ab = alg_bytes(k, wl, C)
        out[k] = {"launches": nl, "avg_us": avg_ms * 1000.0, "share": ms / tot,
                  "alg_bytes_per_launch": ab, "gbs": ab / avg_ms / 1e6, "hbm_frac": ab / avg_ms / 1e6 / peak}
    return out


def main():
    args = parse_args()
    rank, world, local_rank = dist_env()
    if args.impl == "reference":
        return run_reference(args, rank, world)
    import torch
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    peak, peak_src = load_peaks()
    wl = WORKLOADS[args.workload]
    if args.workload == "drift":
        if world > 1:
            raise SystemExit("the drift mode runs on one GPU")
        return run_drift(args, wl, peak)
    if args.workload in ("heads", "heads_uva"):
        if world > 1:
            raise SystemExit("the per-head comparison runs on one GPU")
        return run_heads(args, wl)
    if args.workload == "longgen":
        if world > 1:
            raise SystemExit("the long-generation mode runs on one GPU")
        return run_longgen(args, wl)
    if args.workload == "sweep":
        if world > 1:
            raise SystemExit("the sweep runs on one GPU")
        return run_sweep(args, wl)
    want_cpu = (rank == 0 and world == 1 and not args.no_cpu_baseline)
    res = run_ours(args, wl, rank, world, local_rank, want_cpu, peak)

    mil = None
    if args.workload == "throughput" and not args.no_million:
        wl_m = WORKLOADS["million"]
        margs = argparse.Namespace(**vars(args))
        margs.steps = min(args.steps, 500)
        margs.no_e2e = True
        rm = run_ours(margs, wl_m, rank, world, local_rank, want_cpu, peak)
        km = kernel_table(rm["kern"], margs.steps, wl_m, rm["C"], peak)
        link_bytes = wl_m["batch"] * wl_m["H"] * 100 * 2 * 128 * 2
        att = km.get("gather_attend", {})
        mil = {"workload": wl_m["name"], "steps_s": job_rate(margs.steps, world, rm["ms_total"]),
               "ms_per_step": rm["ms_total"] / margs.steps, "steps": margs.steps,
               "search_us": sum(km[k]["avg_us"] for k in ("query_prep", "collision_scan", "compact", "rerank_topk",
                                          "topk_merge")
                                if k in km),
               "attend_us": att.get("avg_us"), "recall_at_100": rm["recall"],
               "uva_bytes_per_step": link_bytes,
               "host_link_gbs": (link_bytes / (att["avg_us"] * 1e-6) / 1e9) if att else None,
               "h2d_copy_gbs": rm.get("h2d_gbs"),
               "host_link_frac_of_h2d_copy": ((link_bytes / (att["avg_us"] * 1e-6) / 1e9) / rm["h2d_gbs"])
               if att and rm.get("h2d_gbs") else None,
               "uva_read_gbs": rm.get("uva_read_gbs"),
               "host_link_frac_of_uva_read": ((link_bytes / (att["avg_us"] * 1e-6) / 1e9) / rm["uva_read_gbs"])
               if att and rm.get("uva_read_gbs") else None,
               "kernels": km, "cand_budget": rm["C"], "collision_budget": rm["R"],
               "index_build": rm["build"], "cpu_baseline": rm.get("cpu")}

    if world > 1:
        torch.distributed.barrier()
    if rank != 0:
        if world > 1:
            torch.distributed.destroy_process_group()
        return

    km = kernel_table(res["kern"], args.steps, wl, res["C"], peak)
    dom = max(km, key=lambda k: km[k]["share"])
    step_bytes = sum(alg_bytes(k, wl, res["C"]) for k in km)
    ms_per_step = res["ms_total"] / args.steps
    value = job_rate(args.steps, world, res["ms_total"])
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "steps/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": wl["name"], "batch": wl["batch"], "n": wl["n"], "kv_heads": wl["H"],
                   "q_heads": wl["H"] * wl["G"], "head_dim": 128, "topk": 100,
                   "cand_budget": res["C"], "collision_budget": res["R"],
                   "kv_location": "pinned host (UVA)" if wl["kv_host"] else "hbm",
                   "kv_dtype": "bf16", "index": "16 B codes + 128 B 4-bit record per key",
                   "l2": "flushed between timed steps (256 MiB write outside the events)",
                   "queries": "fresh query per step from a 64-query pool",
                   "launch": "one CUDA graph per step" if res["graph"] else "eager launches",
                   "parallelism": "replicas: each rank its own %d pairs" % (wl["batch"] * wl["H"])},
        "recall_at_100": res["recall"],
        "hbm": {"alg_bytes_per_step": step_bytes, "gbs": step_bytes / ms_per_step / 1e6,
                "frac": step_bytes / ms_per_step / 1e6 / peak},
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": km[dom]["gbs"], "peak": peak,
                     "unit": "GB/s", "frac": km[dom]["gbs"] / peak,
                     "traffic": profiled_traffic(dom, wl["name"]), "peak_source": peak_src},
        "kernels": km,
        "gpu_launches": sum(v["launches"] for v in km.values()),
        "clocks": res["clocks"],
        "e2e": res["e2e"],
        "cpu_baseline": res.get("cpu"),
        "wall_s_timed_region": res["wall"],
        "ms_per_step_traced": res["ms_traced"] / args.steps,
        "index_build": res["build"],
    }
    if "dense" in res:
        line["dense_attention"] = res["dense"]
    if mil is not None:
        line["million_token"] = mil
    print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


# ------------------------------------------------------------ drift mode
def run_drift(args, wl, peaks):
    """Append + search per decode step over a drifting key stream (one KV
    head group per step, G = 1); Recall@100 against the exact Top-100 of
    <k_i, q> in fp64 over all keys so far, every `recall_every` steps."""
    import torch
    import kv_cache_top_b200 as pk
    import workloads
    dev = torch.device("cuda", 0)
    n0, T, H, every = wl["n"], wl["steps"], wl["H"], wl["recall_every"]
    if args.drift_steps > 0:
        T = max(every, (min(args.drift_steps, T) // every) * every)
    w = workloads.drift_stream(n0, T, H=H, seed=args.seed, device=dev)
    p = pk.pk_default_params(batch=1, n_kv_heads=H, group=1, topk=100, n_cap=n0 + T, kv_dtype=pk.PK_BF16)
    h = pk.pk_build_index(w["K"], w["V"], n0, p)
    idx = torch.empty(H, 100, dtype=torch.int32, device=dev)
    Kall = torch.cat([w["K"][0].double(), w["k_new"][:, 0, :, 0].permute(1, 0, 2).double()], dim=1)  # [H][n0+T][D]
    stream = torch.cuda.current_stream()
    for t in range(min(args.warmup, 8)):          # warm-up searches without appends
        pk.pk_search(h, w["q"][0], 100, idx)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(T)]
    recalls = []
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    for t in range(T):
        flush.zero_()                                 # the index (~95 MB) would stay in L2 otherwise
        ev[t][0].record(stream)
        pk.pk_append(h, w["k_new"][t], w["v_new"][t], 1)
        pk.pk_search(h, w["q"][t], 100, idx)
        ev[t][1].record(stream)
        if (t + 1) % every == 0:
            n = n0 + t + 1
            s = torch.einsum("hnd,hd->hn", Kall[:, :n], w["q"][t][0].double())
            ex = torch.topk(s, 100, dim=1).indices
            got = idx.long()
            r = [len(set(ex[i].tolist()) & set(got[i].tolist())) / 100.0 for i in range(H)]
            recalls.append((t + 1, sum(r) / H))
    torch.cuda.synchronize()
    ms = [a.elapsed_time(b) for a, b in ev]
    pk.pk_free(h)
    ms_tot = sum(ms)
    line = {"metric": "append+search steps/s under key drift; Recall@100 every %d steps" % every,
            "value": T / (ms_tot / 1000.0), "unit": "steps/s", "n_gpus": 1, "steps": T, "warmup": args.warmup,
            "ms_per_step": ms_tot / T, "ms_per_step_median": statistics.median(ms), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": wl["name"], "n_prefill": n0, "kv_heads": H, "q_heads": H, "head_dim": 128,
                       "topk": 100, "step": "pk_append (1 key per KV head) + pk_search",
                       "l2": "flushed between steps (256 MiB write outside the events)"},
            "recall_at_100": [{"step": a, "recall": b} for a, b in recalls],
            "recall_at_100_mean": sum(b for _, b in recalls) / max(1, len(recalls)),
            "gpu_launches": None}
    print(json.dumps(line), flush=True)


# ------------------------------------------- per-query-head retrieval
def run_heads(args, wl):
    """The aggregated query (one search per KV head) against every query
    head searching on its own: Recall@100 against each query head's exact
    Top-100 of <k_i, q_g> (fp32), and the retrieval + attention time per
    step (CUDA events, L2 flushed between steps)."""
    import torch
    import kv_cache_top_b200 as pk
    import workloads
    dev = torch.device("cuda", 0)
    B, n, H, G, nq = wl["batch"], wl["n"], wl["H"], wl["G"], wl["queries"]
    w = workloads.llama_layer(B, n, H=H, G=G, seed=args.seed, device=dev, n_queries=nq)
    p = pk.pk_default_params(batch=B, n_kv_heads=H, group=G, topk=100, kv_dtype=pk.PK_BF16,
                             kv_location=pk.PK_KV_HOST_PINNED if wl["kv_host"] else pk.PK_KV_DEVICE)
    h = pk.pk_build_index(w["K"], w["V"], n, p)
    BH, U = B * H, B * H * G
    idx_a = torch.empty(BH, 100, dtype=torch.int32, device=dev)
    idx_h = torch.empty(U, 100, dtype=torch.int32, device=dev)
    out = torch.empty(B, H * G, 128, dtype=torch.float32, device=dev)
    rec_a, rec_h, union_rows = [], [], []
    for qi in range(nq):
        q = w["q"][qi]
        pk.pk_search(h, q, 100, idx_a)
        pk.pk_search_heads(h, q, 100, idx_h)
        ga, gh = idx_a.cpu(), idx_h.cpu()
        # rows the per-head attention gathers per pair: the union of its G lists
        union_rows += [len(set(gh[p * G:(p + 1) * G].flatten().tolist())) for p in range(BH)]
        qs = q.float().view(B, H, G, 128)
        for b in range(B):
            for hh in range(H):
                s_ = w["K"][b, hh].float() @ qs[b, hh].T                     # [n][G]
                ex = torch.topk(s_, 100, dim=0).indices.T.cpu()             # [G][100]
                for g in range(G):
                    e = set(ex[g].tolist())
                    rec_a.append(len(e & set(ga[b * H + hh].tolist())) / 100)
                    rec_h.append(len(e & set(gh[(b * H + hh) * G + g].tolist())) / 100)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    def timed(step, k=200):
        for i in range(5):
            step(i)
        ev = []
        for i in range(k):
            flush.zero_()
            a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a_.record(stream)
            step(i)
            b_.record(stream)
            ev.append((a_, b_))
        torch.cuda.synchronize()
        return sum(a_.elapsed_time(b_) for a_, b_ in ev) / k

    step_a = lambda i: (pk.pk_search(h, w["q"][i % nq], 100, idx_a),
                        pk.pk_attend(h, w["q"][i % nq], idx_a, 100, out))
    step_h = lambda i: (pk.pk_search_heads(h, w["q"][i % nq], 100, idx_h),
                        pk.pk_attend_heads(h, w["q"][i % nq], idx_h, 100, out))
    ms_a = timed(step_a)
    ms_h = timed(step_h)

    def kernels(step, k=50):          # per-kernel event times (traced pass)
        pk.pk_trace_enable(h, True)
        pk.pk_trace_read(h)
        for i in range(k):
            flush.zero_()
            step(i)
        kern = pk.pk_trace_read(h)
        pk.pk_trace_enable(h, False)
        return {name: round(ms / nl * 1000.0, 2) for name, (nl, ms) in kern.items() if nl}

    kern_a, kern_h = kernels(step_a), kernels(step_h)

    overlap = None
    if wl["kv_host"]:
        # pk_attend_heads alone on the heads' own lists, and on lists made to
        # overlap: heads 1.. of a pair take the first half of head 0's list,
        # or all of it.  Each distinct row of a pair crosses the host link once.
        own = []
        for i in range(nq):
            pk.pk_search_heads(h, w["q"][i], 100, idx_h)
            own.append(idx_h.clone())

        def shared(ix, m):
            v = ix.view(BH, G, 100).clone()
            v[:, 1:, :m] = v[:, :1, :m]
            return v.view(U, 100)

        overlap = {}
        for name, lists in (("own", own), ("half", [shared(x, 50) for x in own]),
                            ("same", [shared(x, 100) for x in own])):
            us = 1000.0 * timed(lambda i: pk.pk_attend_heads(h, w["q"][i % nq], lists[i % nq], 100, out))
            rows = sum(len(set(x[p_ * G:(p_ + 1) * G].flatten().tolist())) for x in lists for p_ in range(BH))
            overlap[name] = {"attend_us": us, "rows_per_pair": rows / (len(lists) * BH),
                             "host_bytes_per_call": rows / len(lists) * 2 * 128 * 2}
    pk.pk_free(h)
    print(json.dumps({
        "metric": "Recall@100 against each query head's exact Top-100, and step time: aggregated vs "
                  "per-query-head retrieval",
        "aggregated": {"recall_at_100": sum(rec_a) / len(rec_a), "ms_per_step": ms_a,
                       "steps_s": 1000.0 / ms_a, "kernel_us": kern_a},
        "per_head": {"recall_at_100": sum(rec_h) / len(rec_h), "ms_per_step": ms_h, "steps_s": 1000.0 / ms_h,
                     "kernel_us": kern_h,
                     "attend_rows_per_pair": {"union": sum(union_rows) / len(union_rows), "lists": G * 100}},
        "attend_heads_overlap": overlap,
        "data": "synthetic", "dtype": "f32",
        "config": {"workload": wl["name"], "batch": B, "n": n, "kv_heads": H, "q_heads": H * G, "topk": 100,
                   "queries": nq, "kv_location": "pinned host (UVA)" if wl["kv_host"] else "hbm",
                   "l2": "flushed between steps (outside the events)"}}), flush=True)


# ------------------------------------------------------ long generation
def run_longgen(args, wl):
    """Decode steps with the sink / local / update-buffer layout: each step
    adds one token per pair to the dense tail, retrieves the zone's Top-k and
    attends over sink + tail + retrieved rows.  Re-indexing of `update` tokens
    runs either in line on the decode stream (pk_append) or asynchronously
    (pk_append_stage on a side stream in 4 pieces over 4 steps,
    pk_append_publish one step after the last); both
    modes run on the same inputs.  CUDA events per step on the decode stream,
    L2 flushed between steps; steps that re-index (stage, publish) are
    reported apart."""
    import torch
    import workloads
    from kv_cache_top_b200.decode_cache import DecodeCache
    dev = torch.device("cuda", 0)
    B, n, H, G, T = wl["batch"], wl["n"], wl["H"], wl["G"], wl["steps"]
    w = workloads.llama_layer(B, n + T, H=H, G=G, seed=args.seed, device=dev, n_queries=64)
    K, V, q = w["K"], w["V"], w["q"]
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()
    toks = [(K[:, :, n + t:n + t + 1].contiguous(), V[:, :, n + t:n + t + 1].contiguous()) for t in range(T)]

    def run(async_reindex):
        cache = DecodeCache(K[:, :, :n].contiguous(), V[:, :, :n].contiguous(), group=G, sink=wl["sink"],
                            local=wl["local"], update=wl["update"], max_len=n + T, async_reindex=async_reindex)
        torch.cuda.synchronize()
        ev, kind = [], []
        for t in range(T):
            flush.zero_()
            a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            before = (cache.reindexed, getattr(cache, "staged_for", -1))
            a_.record(stream)
            cache.step(q[t % 64], *toks[t])
            b_.record(stream)
            ev.append((a_, b_))
            after = (cache.reindexed, getattr(cache, "staged_for", -1))
            if async_reindex:
                kind.append("publish" if after[0] > before[0] else ("stage" if after[1] >= 0 else "plain"))
            else:
                kind.append("reindex" if after[0] > before[0] else "plain")
        torch.cuda.synchronize()
        ms = [a_.elapsed_time(b_) for a_, b_ in ev]
        info = cache.info()
        cache.close()
        out = {"steps_s": T / (sum(ms) / 1000.0), "ms_per_step": sum(ms) / T,
               "ms_per_plain_step_median": statistics.median([m for m, k in zip(ms, kind) if k == "plain"]),
               "zone_keys_at_end": info.n}
        for k in sorted(set(kind) - {"plain"}):
            sel = [m for m, kk in zip(ms, kind) if kk == k]
            out["%s_steps" % k] = len(sel)
            out["ms_per_%s_step" % k] = sum(sel) / len(sel)
        return out

    sync = run(False)
    asy = run(True)
    print(json.dumps({
        "metric": "decode steps/s with the sink / local / update-buffer layout (retrieval + attention over "
                  "sink, local and retrieved rows)",
        "value": asy["steps_s"], "unit": "steps/s", "n_gpus": 1, "steps": T, "higher_is_better": True,
        "ms_per_step": asy["ms_per_step"], "async_reindex": asy, "inline_reindex": sync,
        "dtype": "f32", "data": "synthetic",
        "config": {"workload": wl["name"], "batch": B, "prefill": n, "kv_heads": H, "q_heads": H * G,
                   "sink": wl["sink"], "local": wl["local"], "update": wl["update"], "topk": 100,
                   "timing": "CUDA events per step on the decode stream; side-stream staging counts where "
                             "the decode stream waits for it",
                   "l2": "flushed between steps (outside the events)"}}),
          flush=True)


# ------------------------------------------------------------ ratio sweep
def run_sweep(args, wl):
    """Recall@100 (against the exact Top-100 of <k_i, q_agg>, fp32) and the
    search + attend time per step for candidate ratio beta (C = ceil(beta n))
    and collision ratio rho, plus the ratio table's own choice, at several n
    (1 sequence x 8 KV heads, Llama-shaped keys, K/V in HBM)."""
    import torch
    import kv_cache_top_b200 as pk
    import workloads
    dev = torch.device("cuda", 0)
    H, G, topk, nq = wl["H"], wl["G"], 100, wl["queries"]
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()
    grid = []
    for n in wl["ns"]:
        w = workloads.llama_layer(1, n, H=H, G=G, seed=args.seed, device=dev, n_queries=nq)
        exact = []
        for qi in range(nq):
            qa = w["q"][qi].float().view(H, G, 128).sum(1)
            s_ = torch.einsum("hnd,hd->hn", w["K"][0].float(), qa)
            exact.append(torch.topk(s_, topk, dim=1).indices.cpu())
        idx = torch.empty(H, topk, dtype=torch.int32, device=dev)
        out = torch.empty(1, H * G, 128, dtype=torch.float32, device=dev)
        points = [(0.0, 0.0)] + [(b, r) for b in wl["betas"] for r in wl["rhos"]]
        for beta, rho in points:
            cand = math.ceil(beta * n) if beta > 0 else 0
            p = pk.pk_default_params(batch=1, n_kv_heads=H, group=G, topk=topk, cand_budget=cand,
                                     collision_ratio=rho, kv_dtype=pk.PK_BF16)
            h = pk.pk_build_index(w["K"], w["V"], n, p)
            C, R = pk.pk_resolve(n, cand, rho, topk)
            rec = []
            for qi in range(nq):
                pk.pk_search(h, w["q"][qi], topk, idx)
                got = idx.cpu()
                rec += [len(set(exact[qi][i].tolist()) & set(got[i].tolist())) / topk for i in range(H)]
            ev = []
            for i in range(3 + 10):
                flush.zero_()
                a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a_.record(stream)
                pk.pk_search(h, w["q"][i % nq], topk, idx)
                pk.pk_attend(h, w["q"][i % nq], idx, topk, out)
                b_.record(stream)
                ev.append((a_, b_))
            torch.cuda.synchronize()
            ms = statistics.median([a_.elapsed_time(b_) for a_, b_ in ev[3:]])
            grid.append({"n": n, "beta": beta if beta > 0 else "table", "rho": rho if rho > 0 else "table",
                         "C": C, "R": R, "recall_at_100": sum(rec) / len(rec), "ms_per_step": ms})
            pk.pk_free(h)
        del w
        torch.cuda.empty_cache()
    print(json.dumps({"metric": "Recall@100 and step time vs candidate / collision ratio",
                      "unit": "recall", "data": "synthetic", "dtype": "f32",
                      "config": {"workload": wl["name"], "batch": 1, "kv_heads": H, "q_heads": H * G,
                                 "head_dim": 128, "topk": topk, "queries": nq,
                                 "step": "pk_search + pk_attend for all 8 KV heads, L2 flushed, median of 10"},
                      "grid": grid}), flush=True)


# ---------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    """The reference arm is the CPU oracle as it stands, on one host core.
    A timed step searches and attends a sample of P of the workload's
    (sequence, KV head) pairs, P chosen from a one-pair trial so that the
    --steps K run takes about a minute (P = all pairs when that fits); the
    value extrapolates a step's time to all pairs, and the line says so.
    Index builds (up to 16 distinct pairs, cycled) run untimed in threads."""
    if rank != 0:
        return
    from concurrent.futures import ThreadPoolExecutor
    import torch
    import oracle
    import workloads
    wl = WORKLOADS[args.workload]
    batch, n, H, G = wl["batch"], wl["n"], wl["H"], wl["G"]
    bh = batch * H
    dev = torch.device("cuda", 0) if torch.cuda.is_available() else torch.device("cpu")
    nd = min(bh, 16 if n <= 200000 else 4)
    nq = 16
    C, R = oracle.resolve(n, wl["cand"], 0.0, 100)

    def load(i):
        pidx = (i * bh) // nd
        b, hh = divmod(pidx, H)
        K, V, qq = workloads.llama_pair(b, hh, n, H=H, G=G, seed=args.seed, device=dev, n_queries=nq)
        return workloads.to_np_f32(K), workloads.to_np_f32(V), workloads.to_np_f32(qq)

    raw = [load(i) for i in range(nd)]
    with ThreadPoolExecutor(min(nd, os.cpu_count() or 1)) as ex:
        encs = list(ex.map(lambda r: oracle.build_index(r[0]), raw))
    data = [(e,) + r for e, r in zip(encs, raw)]

    def one(j):
        enc, Kn, Vn, qn = data[j % nd]
        qv = qn[(j // nd) % nq]
        o = oracle.search(enc, qv, topk_k=100, cand_budget=wl["cand"])
        oracle.attend(qv, Kn, Vn, o["idx"], 1.0 / math.sqrt(128))

    t0 = time.perf_counter()
    one(0)
    t_pair = time.perf_counter() - t0
    budget_s = 60.0
    P = int(max(1, min(bh, budget_s / max(1, args.steps) / max(t_pair, 1e-6))))
    j = 1
    for _ in range(args.warmup):
        for _ in range(P):
            one(j)
            j += 1
    t0 = time.perf_counter()
    for _ in range(args.steps):
        for _ in range(P):
            one(j)
            j += 1
    dt = time.perf_counter() - t0
    ms_step = dt / args.steps * 1000.0                # one timed step: P pair-searches
    value = 1000.0 / (ms_step * bh / P)               # full steps (all bh pairs) per second
    sample = ("each timed step searches + attends %d of the %d (sequence, KV head) pairs (%d distinct "
              "oracle indices, built untimed, cycled; fresh query per search); value = full steps/s "
              "extrapolated from the sample (x %d / %d)" % (P, bh, nd, bh, P))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "ms_per_full_step_extrapolated": ms_step * bh / P, "pairs_per_timed_step": P,
            "extrapolated": P < bh,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": wl["name"], "batch": batch, "n": n, "kv_heads": H, "q_heads": H * G,
                       "head_dim": 128, "topk": 100, "cand_budget": C, "collision_budget": R,
                       "kv_location": "host memory (CPU oracle)", "kv_dtype": "bf16 values in fp32",
                       "index": "oracle index (codes, level indices, fp32 weights, fp64 signed levels)",
                       "queries": "fresh query per search from a %d-query pool" % nq,
                       "parallelism": "one host core"},
            "cpu_baseline": {"value": value, "unit": "steps/s", "cores": 1, "kind": "oracle", "cpu": cpu_model(),
                             "sample": sample},
            "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
