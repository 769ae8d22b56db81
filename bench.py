#!/usr/bin/env python
"""Benchmark of the ParisKV decode-step retrieval path on B200.

Metric: keys searched per second per decode step (query prep + collision vote + candidate
select + RSQ-IP rerank + top-k), i.e. batch * query heads * cached keys / search time, and
the achieved fraction of the HBM roofline of the dominant kernel.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload million_offload]
    python bench.py --workload drift_32k    # long-generation drift: append + search per step
    python bench.py --impl reference ...   # the CPU oracle on a bounded sample

Default workload: the million-token offload decode step (batch 1, 32 query / 8 KV heads,
d = 128, N = 1,048,576 cached keys, 5% candidates, k = 4096; index in HBM, bf16 K/V in pinned
host memory read over UVA by the sparse attention). Inputs are synthetic (seeded, see
long_context_kv_srht_b200/workload.py). Multi-GPU runs are weak-scaled replicas: every rank
holds its own sequences; the only collectives are the timing barrier and max-reduction.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_FLUSH_BYTES = 256 << 20
L2_NOTE = (f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MiB write, then "
           f"{L2_FLUSH_BYTES >> 20} MiB read of another buffer)")
APPEND_SLACK = 64
LEARNED_ITERS = 10          # spherical k-means iterations of the learned-centroid comparator


class L2Flush:
    """Evicts the step's data from L2 between timed steps: writes a buffer larger than L2,
    then reads another buffer as large, so that L2 is left holding clean lines (the write's
    dirty lines are written back here, outside the timed region, rather than during the
    next step's own DRAM traffic)."""

    def __init__(self, dev):
        import torch
        self.w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(L2_FLUSH_BYTES // 8, dtype=torch.int64, device=dev)

    def __call__(self, s: int) -> None:
        self.w.fill_(s & 255)
        self.r.sum()


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="million_offload")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cache", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the search and dense-comparator lines of the other workloads")
    ap.add_argument("--profile-run", action="store_true",
                    help="for profilers: build the index, run --warmup + --steps searches (and "
                         "with --attend the sparse attention over the top-k) and exit; no "
                         "timing, no JSON line, no extra device buffers")
    ap.add_argument("--attend", action="store_true",
                    help="with --profile-run: also run the sparse attention after each search")
    ap.add_argument("--n", type=int, default=None,
                    help="with --profile-run: index this many keys instead of the workload's n "
                         "(a reduced case for captures that replay each launch many times)")
    ap.add_argument("--centroids", choices=["analytic", "learned"], default="analytic",
                    help="drift_32k: coarse centroids (analytic, or learned from the prefill "
                         "by spherical k-means: the comparator of the drift claim)")
    ap.add_argument("--levels", choices=["uniform", "prior"], default="uniform",
                    help="magnitude levels of the RSQ codes (uniform, or the rotation prior's)")
    return ap.parse_args()


# ------------------------------------------------------------------------------------ dist
def dist_setup(args=None):
    """One process per GPU from the torchrun environment: NCCL over the local GPU, or gloo on
    the host cores where no GPU is visible (the reference arm and the multi-rank tests)."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch
        import torch.distributed as dist
        timeout = datetime.timedelta(seconds=120)
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timeout,
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=timeout)
    return ws, rank, local


def rank_spec(name: str, rank: int):
    """The workload of one rank: weak scaling gives every rank its own sequences (the seed is
    offset by 1000 per rank), the same shapes."""
    from long_context_kv_srht_b200 import workload
    return workload.spec(name, seed=workload.spec(name).seed + 1000 * rank)


def dist_max(x: float, ws: int) -> float:
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_barrier(ws: int):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi sampled every 100 ms while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu: int):
        try:
            import torch
            self.gpu = "GPU-" + str(torch.cuda.get_device_properties(gpu).uuid)
        except Exception:
            self.gpu = str(gpu)
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = sorted(float(r[1]) for r in rows if r[1].replace(".", "").isdigit())
        smax = max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": smax,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------------------------ helpers
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def kernel_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, only while the kernel's source
    and the shared device headers are unchanged since the capture (their sha256 is stored
    next to the figure)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get("kernels", {}).get(kernel, {}).get(workload)
    if not e:
        return None
    h = hashlib.sha256()
    for name in e["sources"]:
        with open(os.path.join(ROOT, "long_context_kv_srht_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return e["dram_bytes_per_launch"] if h.hexdigest() == e["sha256"] else None


def algorithmic_bytes(stage: str, sp, C: int) -> int:
    """Bytes a stage must move per launch: the vote reads 16 B of ids per key per KV head;
    the rerank reads one 128 B record per candidate per query head."""
    units = sp.batch * sp.num_kv_heads
    packs = -(-sp.group // 4)
    if stage == "vote":
        return units * packs * sp.n * 16
    if stage == "rerank":
        return sp.batch * sp.num_q_heads * C * 128
    return 0


def candidate_count(n, k, bp):
    return min(n, max(k, -(-n * bp // 10000)))


# ------------------------------------------------------------------------------------ oracle
def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_sample(sp, data, reps: int, heads: int = 4):
    """Times the CPU oracle (as it stands) on one (sequence, KV head) unit of the workload:
    index build untimed, then `reps` searches of `heads` query heads over all n keys."""
    import oracle
    keys = data["keys"][0, 0, :sp.n].float().cpu().numpy()
    qs = data["queries"][0, :heads].float().cpu().numpy()
    signs = data["signs"].numpy()
    p = oracle.SearchParams(m=sp.m, rho=sp.rho, cand_bp=sp.cand_bp)
    enc = oracle.build_unit(keys, signs, sp.m)
    t0 = time.perf_counter()
    for _ in range(reps):
        for g in range(heads):
            oracle.search(enc, qs[g], signs, sp.k, p)
    dt = time.perf_counter() - t0
    keys_done = reps * heads * keys.shape[0]
    return keys_done / dt, dt, oracle.num_threads()


def run_reference(args, ws, rank):
    """The reference arm: the CPU oracle on the host cores, for the same metric/workload."""
    if rank != 0:
        return
    import torch
    from long_context_kv_srht_b200 import workload
    sp = workload.spec(args.workload)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    one = workload.spec(args.workload, batch=1, num_kv_heads=1)
    data = workload.generate_torch(one, dev)
    import oracle
    keys = data["keys"][0, 0].float().cpu().numpy()
    qs = data["queries"][0].float().cpu().numpy()
    signs = data["signs"].numpy()
    p = oracle.SearchParams(m=sp.m, rho=sp.rho, cand_bp=sp.cand_bp)
    enc = oracle.build_unit(keys, signs, sp.m)
    for i in range(args.warmup):
        oracle.search(enc, qs[i % sp.group], signs, sp.k, p)
    t0 = time.perf_counter()
    for i in range(args.steps):
        oracle.search(enc, qs[i % sp.group], signs, sp.k, p)
    dt = time.perf_counter() - t0
    value = args.steps * keys.shape[0] / dt
    line = {
        "impl": "reference", "metric": "keys searched/s per decode step (vote+rerank+top-k)",
        "value": value, "unit": "keys/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": sp.name, "sample": "1 query head x 1 (sequence, KV head) unit",
                   "n": sp.n, "k": sp.k, "cand_bp": sp.cand_bp},
        "cpu_baseline": {"value": value, "unit": "keys/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "cpu_model": cpu_model(),
                         "sample": f"each step: one query head over one unit's {sp.n} keys"},
        "e2e": {"value": value, "unit": "keys/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def decode_step(args, ix, cfg, sp, keys, vals, qs, idx, est, k, H, dev, kv_host):
    import numpy as np
    import torch
    from long_context_kv_srht_b200 import pariskv as pk
    ix.profile(True)
    e0 = torch.cuda.Event(enable_timing=True)
    ea = torch.cuda.Event(enable_timing=True)
    es = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    app_ms = srch_ms = att_ms = 0.0
    stage = {}
    nwarm, nrep = 3, 10        # warm-up steps touch the host pages (GPU TLB) before timing
    out = torch.empty(qs.shape, dtype=torch.float32, device=dev)
    assert nwarm + nrep <= APPEND_SLACK
    pk.union_rows()   # reset the union-row counter of the group-union attention
    for s in range(nwarm + nrep):
        new_k = keys[:, :, ix.size:ix.size + 1].to(dev)
        e0.record()
        ix.append(new_k)
        ea.record()
        ix.search(qs, k, idx, est)
        es.record()
        pk.sparse_attend(cfg, qs, keys, vals, idx, k, 1.0 / float(np.sqrt(sp.d)), n=ix.size,
                         out=out)
        e1.record()
        e1.synchronize()
        if s < nwarm:
            ix.stage_ms()
            continue
        for name, ms in ix.stage_ms().items():
            stage[name] = stage.get(name, 0.0) + ms / nrep
        app_ms += e0.elapsed_time(ea) / nrep
        srch_ms += ea.elapsed_time(es) / nrep
        att_ms += es.elapsed_time(e1) / nrep
    # K/V rows the attention fetched per step: the GQA-group union when it is used (each row
    # once per KV head), else every head's own k rows
    urows = pk.union_rows() / (nwarm + nrep)
    rows = urows if urows else H * k
    kv_bytes = int(rows * 2 * sp.d * 2)
    decode = {"append_ms": app_ms, "search_ms": srch_ms, "sparse_attend_ms": att_ms,
              "total_ms": app_ms + srch_ms + att_ms,
              "kv_source": "pinned host (UVA)" if kv_host else "HBM",
              "attend_rows_per_step": rows, "attend_rows_per_head_selection": H * k,
              "attend_kv_bytes_per_step": kv_bytes,
              "attend_gbs": kv_bytes / (att_ms / 1e3) / 1e9}
    if kv_host:
        # the PCIe roofline of the attention: one coalesced pass over 256 MiB of the pinned K
        # array, read by the device the same way (UVA)
        nb = min(256 << 20, keys.numel() * keys.element_size()) // 16 * 16
        sink = torch.zeros(1, dtype=torch.int32, device=dev)
        pk.read_stream(keys, nb, sink)
        torch.cuda.synchronize()
        ts = []
        for _ in range(3):
            e0.record()
            pk.read_stream(keys, nb, sink)
            e1.record()
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
        pcie = nb / (min(ts) / 1e3) / 1e9
        decode["pcie_read_gbs"] = pcie
        decode["attend_pcie_frac"] = decode["attend_gbs"] / pcie
    decode["search_stage_ms"] = stage
    return decode


# ------------------------------------------------------------------------------------ main
def dense_comparator(cfg, sp, data, ix, k, dev, peak_gbs):
    """Full attention over all n tokens (pariskv_dense_attend, K/V in HBM) against ParisKV's
    retrieval + sparse attention over the top-k with the same K/V in HBM (the one-key append,
    about 0.02 ms, is in the decode-step figures): the synthetic analogue of the comparison
    with full attention in "Technical Summary: ParisKV" (Experimental Results). Both are
    timed with CUDA events around 20 steps enqueued back to back after 3 warm-up steps; K/V
    (4 GiB at the million-token workload) exceed L2, so no flush is needed between steps."""
    import numpy as np
    import torch
    from long_context_kv_srht_b200 import pariskv as pk
    if sp.dtype != "bf16" or sp.group > 8:
        return None
    keys, vals, qs = data["keys"], data["values"], data["queries"]
    Kd = keys if keys.is_cuda else keys.to(dev)
    Vd = vals if vals.is_cuda else vals.to(dev)
    n = sp.n
    scale = 1.0 / float(np.sqrt(sp.d))
    out = torch.empty(qs.shape, dtype=torch.float32, device=dev)
    H = sp.batch * sp.num_q_heads
    idx = torch.empty((H, k), dtype=torch.int32, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed(fn, reps=20, warm=3):
        # steps enqueued back to back (no host synchronisation between them), so the time is
        # the device's, not the host's launch latency; mean over the reps
        for _ in range(warm):
            fn()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        e1.synchronize()
        return e0.elapsed_time(e1) / reps

    dense_ms = timed(lambda: pk.dense_attend(cfg, qs, Kd, Vd, scale, n=n, out=out))
    # the ParisKV retrieval and sparse attention on the same K/V in HBM (the index as it is;
    # this measurement does not grow it)
    size = ix.size

    def paris():
        ix.search(qs, k, idx)
        pk.sparse_attend(cfg, qs, Kd, Vd, idx, k, scale, n=size, out=out)
    paris_ms = timed(paris)
    kv_bytes = 2 * sp.batch * sp.num_kv_heads * n * sp.d * 2
    del Kd, Vd
    return {"dense_ms": dense_ms,
            "dense_gbs": kv_bytes / (dense_ms / 1e3) / 1e9,
            "dense_frac_of_measured_hbm": kv_bytes / (dense_ms / 1e3) / 1e9 / peak_gbs,
            "dense_bytes_per_step": kv_bytes,
            "dense_roofline_ms": kv_bytes / (peak_gbs * 1e9) * 1e3,
            "paris_hbm_ms": paris_ms, "speedup_vs_dense_hbm": dense_ms / paris_ms,
            "speedup_vs_dense_roofline": kv_bytes / (peak_gbs * 1e9) * 1e3 / paris_ms,
            "kv": "HBM (both)", "n": n, "k": k}


def side_workload(name, args, dev, flush):
    """The search of another workload (K/V in HBM), timed like the headline (L2 flushed
    between steps, CUDA events per step), with its roofline fraction and the ParisKV step
    (search + sparse attention) against full attention on the same K/V."""
    import numpy as np
    import torch
    from long_context_kv_srht_b200 import pariskv as pk
    from long_context_kv_srht_b200 import workload
    sp = workload.spec(name)
    data = workload.generate_torch(sp, dev, n=sp.n)
    cfg = pk.config(batch=sp.batch, num_kv_heads=sp.num_kv_heads, group=sp.group,
                    capacity=sp.n, dtype=sp.dtype, rho=sp.rho, cand_bp=sp.cand_bp,
                    levels=args.levels)
    ix = pk.build_index(cfg, data["signs"], data["keys"], n=sp.n)
    H, k = sp.batch * sp.num_q_heads, sp.k
    C = candidate_count(sp.n, k, sp.cand_bp)
    idx = torch.empty((H, k), dtype=torch.int32, device=dev)
    est = torch.empty((H, k), dtype=torch.float32, device=dev)
    qs = data["queries"]
    for _ in range(max(3, args.warmup)):
        ix.search(qs, k, idx, est)
    torch.cuda.synchronize()
    steps = max(10, min(args.steps, 50))
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for s in range(steps):
        flush(s)
        ev0[s].record()
        ix.search(qs, k, idx, est)
        ev1[s].record()
    torch.cuda.synchronize()
    ms = float(np.mean([a.elapsed_time(b) for a, b in zip(ev0, ev1)]))
    peak = measured_peaks()[0]
    step_bytes = algorithmic_bytes("vote", sp, C) + algorithmic_bytes("rerank", sp, C)
    out = {"ms_per_step": ms, "keys_per_s": H * sp.n / (ms / 1e3), "steps": steps,
           "step_algorithmic_bytes": step_bytes,
           "step_frac": step_bytes / (ms / 1e3) / 1e9 / peak,
           "config": {"batch": sp.batch, "q_heads": sp.num_q_heads, "kv_heads": sp.num_kv_heads,
                      "n": sp.n, "k": k, "candidates": C, "key_dtype": sp.dtype, "kv_in": "HBM"}}
    dense = dense_comparator(cfg, sp, data, ix, k, dev, peak)
    if dense:
        out["dense_ms"] = dense["dense_ms"]
        out["paris_step_ms"] = dense["paris_hbm_ms"]
        out["paris_vs_dense"] = dense["speedup_vs_dense_hbm"]
    ix.sync()
    ix.destroy()
    del data
    torch.cuda.empty_cache()
    return out


# Region sizes of the four-region cache measurement ("Technical Summary: ParisKV" gives none;
# 64 sink tokens as in the sink-token convention of "Self-Indexing KVCache", a 2048-token local
# window, a 256-token buffer).
CACHE_REGIONS = dict(n_sink=64, n_local=2048, n_buffer=256)


def cache_decode(cfg, sp, data, k, dev):
    """Decode steps through the four-region cache (pariskv_cache_step): prefill of all but the
    last T_WARM + T tokens of the workload, then one token per step; each step appends the
    token, promotes a full buffer (evicting the oldest Local tokens to the Retrieval zone in
    pinned host memory and to its index), searches the Retrieval zone and attends over
    Sink + Local + buffer + the top-k. Every step is timed with events on the stream."""
    import numpy as np
    import torch
    from long_context_kv_srht_b200 import pariskv as pk
    t_warm, T = 8, 512
    r = CACHE_REGIONS
    n0 = sp.n - t_warm - T
    if n0 < r["n_sink"] + r["n_local"] + k:
        return None
    keys, vals, qs = data["keys"], data["values"], data["queries"]
    H = sp.batch * sp.num_q_heads
    cache = pk.Cache(cfg, data["signs"], r["n_sink"], r["n_local"], r["n_buffer"], k,
                     retrieval_capacity=sp.n)
    t0 = time.perf_counter()
    cache.prefill(keys, vals, n=n0)
    torch.cuda.synchronize()
    prefill_s = time.perf_counter() - t0
    kn = keys[:, :, n0:sp.n].to(dev)
    vn = vals[:, :, n0:sp.n].to(dev)
    kn = [kn[:, :, s].contiguous() for s in range(t_warm + T)]
    vn = [vn[:, :, s].contiguous() for s in range(t_warm + T)]
    out = torch.empty((sp.batch, sp.num_q_heads, sp.d), dtype=torch.float32, device=dev)
    scale = 1.0 / float(np.sqrt(sp.d))
    for s in range(t_warm):
        cache.step(qs, kn[s], vn[s], scale, out=out)
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(T + 1)]
    promo, launches, before = [], 0, cache.counts()["retrieval"]
    ev[0].record()
    for s in range(T):
        cache.step(qs, kn[t_warm + s], vn[t_warm + s], scale, out=out)
        ev[s + 1].record()
        launches += pk.last_launch_count()
        now = cache.counts()["retrieval"]
        if now != before:
            promo.append(s)
        before = now
    torch.cuda.synchronize()
    ts = np.array([ev[s].elapsed_time(ev[s + 1]) for s in range(T)])
    plain = np.delete(ts, promo)
    counts = cache.counts()
    cache.destroy()
    return {"regions": r, "k": k, "prefill_tokens": n0, "prefill_s": prefill_s,
            "steps": T, "ms_per_step": float(ts.mean()), "ms_per_step_median": float(np.median(ts)),
            "promotion_steps": len(promo),
            "promotion_step_ms": float(ts[promo].mean()) if promo else None,
            "other_step_ms": float(plain.mean()),
            "counts_after": counts, "gpu_launches_per_step": launches / T,
            "tokens_attended_per_head": counts["sink"] + counts["local"] + counts["buffer"] + k,
            "retrieval_kv": "pinned host (UVA)", "heads": H}


def run_drift(args, ws, rank, local):
    """Long-generation drift (8 KV heads, 32768 prefill keys, then one appended key per KV
    head per decode step while the keys' mean vector drifts; k = 1024). Every timed step
    appends one key per KV head and searches once over the grown index; L2 is flushed between
    steps. Recall of the returned top-k against the exact inner-product top-k (computed on
    the device, outside the timed region) is tracked at sampled steps. The warm-up steps are
    the first decode steps of the sequence; all remaining steps are timed."""
    import numpy as np
    import torch
    from long_context_kv_srht_b200 import pariskv as pk
    from long_context_kv_srht_b200 import workload

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    sp = rank_spec("drift_32k", rank)
    T, H, n0, k = sp.decode_steps, sp.num_kv_heads, sp.n, sp.k
    w = workload.generate_drift(sp)
    bf = lambda a: torch.from_numpy(workload.bf16_bits(a)).view(torch.bfloat16).to(dev)
    pre, app, qs = bf(w.prefill[None]), bf(w.appended), bf(w.queries)
    cfg = pk.config(batch=1, num_kv_heads=H, group=1, capacity=n0 + T, dtype=sp.dtype,
                    rho=sp.rho, cand_bp=sp.cand_bp, levels=args.levels)
    train_ms = None
    if args.centroids == "learned":
        # the comparator: centroids learned from the prefill keys, then frozen
        t0 = time.perf_counter()
        cent = pk.train_centroids(cfg, w.signs, pre, LEARNED_ITERS)
        train_ms = (time.perf_counter() - t0) * 1e3
        ix = pk.build_index(cfg, w.signs, pre, n=0)
        ix.set_centroids(cent)
        ix.append(pre)
    else:
        ix = pk.build_index(cfg, w.signs, pre)
    idx = torch.empty((H, k), dtype=torch.int32, device=dev)
    est = torch.empty((H, k), dtype=torch.float32, device=dev)
    flush = L2Flush(dev)
    W = max(0, min(args.warmup, T - 1))
    for t in range(W):
        ix.append(app[t].view(1, H, 1, 128))
        ix.search(qs[t].view(1, H, 128), k, idx, est)
    torch.cuda.synchronize()

    steps = T - W
    sample = set(range(W, T, 2048)) | {T - 1}
    kept = {}
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    dist_barrier(ws)
    torch.cuda.synchronize()
    launches = 0
    for i, t in enumerate(range(W, T)):
        flush(t)
        ev[i][0].record()
        ix.append(app[t].view(1, H, 1, 128))
        ev[i][1].record()
        ix.search(qs[t].view(1, H, 128), k, idx, est)
        ev[i][2].record()
        launches += pk.last_launch_count() + 1
        if t in sample:
            kept[t] = idx.clone()
    torch.cuda.synchronize()
    dist_barrier(ws)
    clk = clocks.stop()
    app_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in ev]))
    srch_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in ev]))
    step_ms = dist_max(app_ms + srch_ms, ws)
    keys_searched = sum(H * (n0 + t + 1) for t in range(W, T))
    value = ws * keys_searched / (step_ms * steps / 1e3)

    # recall against the exact top-k by <q, k> over the keys present at each sampled step
    allk = torch.cat([pre[0], app.permute(1, 0, 2)], dim=1).float()   # [H, n0 + T, d]
    rec = {}
    for t, got in sorted(kept.items()):
        sc = torch.einsum("hnd,hd->hn", allk[:, : n0 + t + 1], qs[t].float())
        ex = torch.topk(sc, k, dim=1).indices
        hit = 0
        for h in range(H):
            hit += np.intersect1d(got[h].cpu().numpy(), ex[h].cpu().numpy()).size
        rec[str(t)] = hit / (H * k)

    if rank == 0:
        line = {
            "metric": "keys searched/s per decode step (vote+rerank+top-k)",
            "value": value, "unit": "keys/s", "n_gpus": ws, "steps": steps,
            "warmup": W, "ms_per_step": step_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": sp.name, "kv_heads": H, "q_heads_per_kv": 1, "d": sp.d,
                       "n_prefill": n0, "decode_steps": T, "k": k, "B": sp.B, "m": sp.m,
                       "rho": sp.rho, "cand_bp": sp.cand_bp, "key_dtype": sp.dtype,
                       "levels": args.levels, "centroids": args.centroids,
                       "step": "append one key per KV head + one search",
                       "l2": L2_NOTE},
            "decode_step": {"append_ms": app_ms, "search_ms": srch_ms},
            "recall_vs_exact_topk": rec,
            "recall_mean": float(np.mean(list(rec.values()))),
            "centroid_training_ms": train_ms,
            "roofline": None,
            "gpu_launches": launches,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    ix.sync()
    ix.destroy()
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def profile_run(args, local):
    """The search (and optionally the sparse attention) of the workload, untimed, for an
    ncu capture: K/V in pinned host memory at the million-token workload as in the bench,
    on the device otherwise; --n reduces the number of keys."""
    import numpy as np
    import torch
    from long_context_kv_srht_b200 import pariskv as pk
    from long_context_kv_srht_b200 import workload
    dev = torch.device("cuda", local)
    torch.cuda.set_device(local)
    sp = workload.spec(args.workload)
    if args.n:
        sp = workload.spec(args.workload, n=args.n)
    kv_host = sp.name == "million_offload"
    data = workload.generate_torch(sp, dev, n=sp.n, kv_on_host=kv_host)
    cfg = pk.config(batch=sp.batch, num_kv_heads=sp.num_kv_heads, group=sp.group,
                    capacity=sp.n, dtype=sp.dtype, rho=sp.rho, cand_bp=sp.cand_bp,
                    levels=args.levels)
    ix = pk.build_index(cfg, data["signs"], data["keys"], n=sp.n)
    H, k = sp.batch * sp.num_q_heads, min(sp.k, sp.n)
    idx = torch.empty((H, k), dtype=torch.int32, device=dev)
    est = torch.empty((H, k), dtype=torch.float32, device=dev)
    out = torch.empty(data["queries"].shape, dtype=torch.float32, device=dev)
    for _ in range(args.warmup + args.steps):
        ix.search(data["queries"], k, idx, est)
        if args.attend:
            pk.sparse_attend(cfg, data["queries"], data["keys"], data["values"], idx, k,
                             1.0 / float(np.sqrt(sp.d)), out=out)
    torch.cuda.synchronize()
    ix.sync()
    ix.destroy()
    print(f"profile run: {sp.name}, n = {sp.n}, {args.warmup + args.steps} searches"
          + (" + attention" if args.attend else ""), flush=True)


def main():
    args = parse()
    ws, rank, local = dist_setup(args)
    if args.impl == "reference":
        run_reference(args, ws, rank)
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    if args.workload == "drift_32k":
        run_drift(args, ws, rank, local)
        return
    if args.profile_run:
        profile_run(args, local)
        return
    import numpy as np
    import torch
    from long_context_kv_srht_b200 import pariskv as pk
    from long_context_kv_srht_b200 import workload

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    sp = rank_spec(args.workload, rank)
    kv_host = sp.name == "million_offload"
    # K/V hold APPEND_SLACK extra tokens after the n indexed ones: the decode-step measurement
    # appends them to the index, so every index the search can return has a K/V row
    data = workload.generate_torch(sp, dev, n=sp.n + APPEND_SLACK, kv_on_host=kv_host)
    keys, vals, qs = data["keys"], data["values"], data["queries"]
    cfg = pk.config(batch=sp.batch, num_kv_heads=sp.num_kv_heads, group=sp.group,
                    capacity=sp.n + APPEND_SLACK, dtype=sp.dtype, rho=sp.rho,
                    cand_bp=sp.cand_bp, levels=args.levels)
    ix = pk.build_index(cfg, data["signs"], keys, n=sp.n)
    H = sp.batch * sp.num_q_heads
    k = sp.k
    C = candidate_count(sp.n, k, sp.cand_bp)
    idx = torch.empty((H, k), dtype=torch.int32, device=dev)
    est = torch.empty((H, k), dtype=torch.float32, device=dev)
    flush = L2Flush(dev)
    for _ in range(args.warmup):
        ix.search(qs, k, idx, est)
    torch.cuda.synchronize()

    # the timed steps: searches enqueued back to back (no host synchronisation inside the
    # loop), each bracketed by events on the search stream, L2 flushed between them
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    dist_barrier(ws)
    torch.cuda.synchronize()
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    launches = 0
    for s in range(args.steps):
        flush(s)                    # L2 flushed between timed steps
        ev0[s].record()
        ix.search(qs, k, idx, est)
        ev1[s].record()
        launches += pk.last_launch_count()
    torch.cuda.synchronize()
    dist_barrier(ws)
    clk = clocks.stop()
    step_times = [a.elapsed_time(b) for a, b in zip(ev0, ev1)]
    step_ms = float(np.mean(step_times))
    step_ms_max = dist_max(step_ms, ws)
    step_median = dist_max(float(np.median(step_times)), ws)
    keys_per_step = sp.batch * sp.num_q_heads * sp.n
    value = ws * keys_per_step / (step_ms_max / 1e3)

    # per-stage device time: the same searches with the library's stage events (a separate
    # loop, because reading the events synchronises the host every step)
    ix.profile(True)
    stage_tot = {}
    for s in range(args.steps):
        flush(s)
        ix.search(qs, k, idx, est)
        for name, ms in ix.stage_ms().items():
            stage_tot[name] = stage_tot.get(name, 0.0) + ms
    ix.profile(False)
    torch.cuda.synchronize()
    stage_avg = {kname: v / args.steps for kname, v in stage_tot.items()}

    # roofline of the dominant kernel (HBM-bound; no tensor-core work on this path)
    dom = max(stage_avg, key=stage_avg.get)
    peak, peak_kind = measured_peaks()
    abytes = algorithmic_bytes(dom, sp, C)
    achieved = abytes / (stage_avg[dom] / 1e3) / 1e9 if abytes else None
    step_bytes = algorithmic_bytes("vote", sp, C) + algorithmic_bytes("rerank", sp, C)
    roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak,
                "unit": "GB/s", "frac": (achieved / peak) if achieved else None,
                "peak_kind": peak_kind, "algorithmic_bytes_per_launch": abytes,
                "traffic": kernel_traffic(dom, sp.name),
                "step_algorithmic_bytes": step_bytes,
                "step_frac": step_bytes / (step_ms_max / 1e3) / 1e9 / peak,
                "step_frac_of_nominal_8tbs": step_bytes / (step_ms_max / 1e3) / 8e12}

    # the rerank's gathers alone: the last search's candidate records read once per query head
    # with the rerank's access pattern and no arithmetic, timed like the stages (L2 flushed).
    # A random 128-byte gather cannot reach the copy rate, so this rate is the rerank's
    # practical ceiling; the rerank's fraction of it shows what its arithmetic costs.
    sink = torch.zeros(1, dtype=torch.int32, device=dev)
    for _ in range(3):
        ix.gather_candidates(sink)
    for s in range(args.steps):
        flush(s)
        ev0[s].record()
        ix.gather_candidates(sink)
        ev1[s].record()
    torch.cuda.synchronize()
    gather_ms = dist_max(float(np.mean([a.elapsed_time(b) for a, b in zip(ev0, ev1)])), ws)
    rbytes = algorithmic_bytes("rerank", sp, C)
    gather_gbs = rbytes / (gather_ms / 1e3) / 1e9
    rerank_gbs = rbytes / (stage_avg["rerank"] / 1e3) / 1e9
    roofline["gather_ceiling"] = {"kernel": "record gather without arithmetic",
                                  "ms": gather_ms, "achieved": gather_gbs, "unit": "GB/s",
                                  "frac_of_peak": gather_gbs / peak,
                                  "rerank_frac_of_ceiling": rerank_gbs / gather_gbs}

    # host cost of enqueueing one search (the device is kept busy meanwhile), and the same
    # search replayed as a CUDA graph (one launch per step, no host work between kernels)
    ix.profile(False)
    big = torch.empty(4 << 30, dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    big.fill_(1)
    t0 = time.perf_counter()
    for _ in range(10):
        ix.search(qs, k, idx, est)
    host_us = (time.perf_counter() - t0) / 10 * 1e6
    torch.cuda.synchronize()
    del big
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        ix.search(qs, k, idx, est)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    with torch.cuda.graph(graph, capture_error_mode="thread_local"):
        ix.search(qs, k, idx, est)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    gtimes = []
    for s in range(args.steps):
        flush(s)
        ev0[s].record()
        graph.replay()
        ev1[s].record()
    torch.cuda.synchronize()
    graph_ms = dist_max(float(np.mean([a.elapsed_time(b) for a, b in zip(ev0, ev1)])), ws)
    graph_value = ws * keys_per_step / (graph_ms / 1e3)
    del graph
    ix.profile(True)

    # end to end through the C ABI: pinned host query in, top-k indices and estimates out
    e2e = None
    if not args.no_e2e:
        q_host = qs.cpu().pin_memory()
        q_dev = torch.empty_like(qs)
        i_host = torch.empty((H, k), dtype=torch.int32).pin_memory()
        e_host = torch.empty((H, k), dtype=torch.float32).pin_memory()
        ix.profile(False)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        tot = 0.0
        nrep = max(3, min(args.steps, 50))
        for s in range(nrep + 2):
            flush(s)
            e0.record()
            q_dev.copy_(q_host, non_blocking=True)
            ix.search(q_dev, k, idx, est)
            i_host.copy_(idx, non_blocking=True)
            e_host.copy_(est, non_blocking=True)
            e1.record()
            e1.synchronize()
            if s >= 2:
                tot += e0.elapsed_time(e1)
        e2e_ms = dist_max(tot / nrep, ws)
        e2e = {"value": ws * keys_per_step / (e2e_ms / 1e3), "unit": "keys/s",
               "ms_per_step": e2e_ms, "h2d_bytes_per_step": q_host.numel() * q_host.element_size(),
               "d2h_bytes_per_step": i_host.numel() * 4 + e_host.numel() * 4}

    # the full decode step around the search: append one key per (sequence, KV head), search,
    # sparse attention over the top-k (K/V read from pinned host memory over UVA here)
    decode = None
    if not args.no_decode:
        decode = decode_step(args, ix, cfg, sp, keys, vals, qs, idx, est, k, H, dev, kv_host)

    # full attention over every token, the baseline "Technical Summary: ParisKV" compares with
    dense = None
    if not args.no_dense:
        dense = dense_comparator(cfg, sp, data, ix, k, dev, measured_peaks()[0])
        if dense and decode:
            dense["speedup_vs_dense_offloaded_step"] = dense["dense_ms"] / decode["total_ms"]

    # the same decode step through the four-region cache (Sink / Local / buffer in HBM, the
    # Retrieval zone in pinned host memory)
    cache_step = None
    if not args.no_cache:
        cache_step = cache_decode(cfg, sp, data, k, dev)

    # the search on the other workloads of the pages' tables (one GPU, rank 0 only)
    others = None
    if rank == 0 and ws == 1 and not args.no_workloads and sp.name == "million_offload":
        others = {name: side_workload(name, args, dev, flush)
                  for name in ("llama3_8b_128k", "batched_64k")}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        v, dt, cores = oracle_sample(sp, data, reps=1)
        cpu = {"value": v, "unit": "keys/s", "cores": cores, "kind": "oracle",
               "cpu_model": cpu_model(),
               "sample": f"one (sequence, KV head) unit: 4 query heads x {sp.n} keys, "
                         f"index build untimed ({dt:.1f} s timed)"}

    if rank == 0:
        line = {
            "metric": "keys searched/s per decode step (vote+rerank+top-k)",
            "value": value, "unit": "keys/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_ms_max, "ms_per_step_median": step_median,
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": sp.name, "batch": sp.batch, "q_heads": sp.num_q_heads,
                       "kv_heads": sp.num_kv_heads, "d": sp.d, "n": sp.n, "k": k,
                       "candidates": C, "B": sp.B, "m": sp.m, "rho": sp.rho,
                       "key_dtype": sp.dtype, "kv_in": "pinned host" if kv_host else "HBM",
                       "levels": args.levels,
                       "l2": L2_NOTE},
            "stage_ms": stage_avg,
            "host_enqueue_us_per_search": host_us,
            "graph": {"ms_per_step": graph_ms, "value": graph_value},
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "decode_step": decode,
            "cache_step": cache_step,
            "dense_comparator": dense,
            "workloads": others,
            "gpu_launches": launches,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    ix.sync()   # raises if a device-side consistency flag or bounded wait fired
    ix.destroy()
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
