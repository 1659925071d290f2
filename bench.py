"""Benchmark: one serving step of RVQ-compressed decode attention per timed step.

A step is one pass of the whole hot path over one batch: each sequence's new token enters the
fp16 window, the evicted oldest window token is RVQ-encoded onto the compressed prefix
(rotation, greedy stages, code packing), then decode attention runs over the compressed prefix
plus the window (query rotation, lookup tables, scoring, online softmax, value histograms, the
log-sum-exp merge with the window).  Workload: Llama-3-8B-shaped single layer, batch 8, 32 query
heads over 8 kv heads, head_dim 128, 32K context, 4+4 RVQ stages, 128-token window (synthetic
data, seeded k-means codebooks).  Inputs rotate over R replicas (different layers' caches) whose
total size exceeds the 126 MB L2, so every step reads its codes from HBM.

Metric: compressed tokens attended per second (sum over sequences of compressed-prefix length,
per step, over the step time), whole job over all ranks.  Multi-GPU: independent replicas per
rank (the path has no exchange step), timed as the max over ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attn compressed tokens/s/GPU & HBM GB/s (% roofline); encode vectors/s"
UNIT = "compressed tokens/s"
WORKLOAD = "llama3_8b_32k"

# DRAM bytes (read + write) of one scan2_kernel launch on this workload, the mean of three
# launches of one ncu capture (profiles/scan2_kernel_llama3_8b_32k.md), valid while the scan's
# source (csrc/scan_rvq.cuh) is unchanged.
SCAN_TRAFFIC = {"scan_src_sha1": "3d61919446712b2c54318221c11f4e278f9964f3",
                "bytes_per_launch": 17825280}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--replicas", type=int, default=8)
    ap.add_argument("--soak-s", type=float, default=1.0, help="extra warm-up time (clocks)")
    ap.add_argument("--no-encode", action="store_true", help="skip the bulk-encode extra")
    ap.add_argument("--no-smooth", action="store_true",
                    help="skip the serving step with key smoothing (extra)")
    ap.add_argument("--no-paged", action="store_true",
                    help="skip the serving step with the paged code layout (extra)")
    ap.add_argument("--no-ragged", action="store_true",
                    help="skip the serving step on the ragged 64-sequence batch (extra)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


# --------------------------------------------------------------------------------------------
# Clock sampling during the timed region
# --------------------------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        rows = [r.split(",") for r in out.strip().splitlines() if r.strip()]
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax = float(r[2])
                for n, v in zip(names, r[5:9]):
                    if v.strip().lower() in ("active", "1", "0x1"):
                        reasons.add(n)
            except Exception:
                continue
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------------------------
# Workload state on the GPU
# --------------------------------------------------------------------------------------------

_BOOKS = {}


def codebooks(wl, kind, smooth=None):
    """The workload's seeded k-means codebooks (float32 numpy), memoised: the main line and
    several extras train the same ones."""
    from compressed_decode_attention_zkv_b200 import inputs as I
    key = (wl, kind, None if smooth is None else np.asarray(smooth).tobytes())
    if key not in _BOOKS:
        _BOOKS[key] = I.train_codebooks(wl, kind, smooth=smooth)
    return _BOOKS[key]


def build_state(wl, R, Tcap_extra, dev, smooth=False, tcap_multiple=16):
    """Encode the workload's prefixes on the GPU (prefill) and make R replicas.  smooth: key
    smoothing factors calibrated on the calibration sample, key codebooks trained on smoothed
    keys, prefixes encoded with them (each replica carries "k_smooth")."""
    import torch

    from compressed_decode_attention_zkv_b200 import inputs as I
    from compressed_decode_attention_zkv_b200 import zkv

    lam_np = I.key_smooth_factors(wl) if smooth else None
    lam = None if lam_np is None else torch.from_numpy(lam_np).to(dev)
    Ck = torch.from_numpy(codebooks(wl, "k", smooth=lam_np)).to(dev)
    Cv = torch.from_numpy(codebooks(wl, "v")).to(dev)
    Tc = wl.Tc
    Tcap = (Tc + Tcap_extra + tcap_multiple - 1) // tcap_multiple * tcap_multiple
    kc = torch.zeros((wl.B, wl.Hkv, Tcap, wl.Sk), dtype=torch.uint8, device=dev)
    vc = torch.zeros((wl.B, wl.Hkv, Tcap, wl.Sv), dtype=torch.uint8, device=dev)
    wk = torch.empty((wl.B, wl.Hkv, wl.W, wl.d), dtype=torch.float16, device=dev)
    wv = torch.empty((wl.B, wl.Hkv, wl.W, wl.d), dtype=torch.float16, device=dev)
    for b in range(wl.B):
        for kind, codes, books, win in (("k", kc, Ck, wk), ("v", vc, Cv, wv)):
            x = torch.from_numpy(I.kv_tokens(wl, kind, b, 0, wl.T)).to(dev)   # [Hkv][T][d]
            zkv.rvq_encode(x[:, :Tc].permute(1, 0, 2)[None], books,
                           codes=codes[b, :, :Tc].permute(1, 0, 2)[None], with_norms=False,
                           smooth=lam if kind == "k" else None)
            win[b].copy_(x[:, Tc:])
            del x
    torch.cuda.synchronize()
    reps = []
    for r in range(R):
        reps.append(dict(
            Ck=Ck.clone(), Cv=Cv.clone(), k_codes=kc.clone(), v_codes=vc.clone(),
            win_k=wk.clone(), win_v=wv.clone(),
            comp_len=torch.full((wl.B,), Tc, dtype=torch.int32, device=dev),
            win_len=torch.full((wl.B,), wl.W, dtype=torch.int32, device=dev),
            win_head=torch.zeros((wl.B,), dtype=torch.int32, device=dev),
            q=torch.from_numpy(I.queries(wl, step=r)).to(dev),
            new_k=torch.from_numpy(I.new_tokens(wl, r, "k", np.full(wl.B, wl.T))).to(dev),
            new_v=torch.from_numpy(I.new_tokens(wl, r, "v", np.full(wl.B, wl.T))).to(dev),
            out=torch.empty((wl.B, wl.Hq, wl.d), dtype=torch.float32, device=dev),
            lse=torch.empty((wl.B, wl.Hq), dtype=torch.float32, device=dev),
            err=torch.zeros(1, dtype=torch.int32, device=dev),
            k_smooth=None if lam is None else lam.clone()))
    del kc, vc, wk, wv
    return reps, Tcap


def replica_bytes(rep):
    return sum(t.numel() * t.element_size() for k, t in rep.items()
               if k in ("Ck", "Cv", "k_codes", "v_codes", "win_k", "win_v", "q", "k_smooth")
               and t is not None)


def step_fn(rep, ws, max_comp, events=None):
    """One serving step through the library's single serving-step call (append of the new
    tokens, then decode attention over the updated cache)."""
    from compressed_decode_attention_zkv_b200 import zkv
    zkv.rvq_serve_step(rep["new_k"], rep["new_v"], rep["q"], rep["win_k"], rep["win_v"],
                       rep["win_len"], rep["win_head"], rep["comp_len"], rep["k_codes"],
                       rep["v_codes"], rep["Ck"], rep["Cv"], out=rep["out"], lse=rep["lse"],
                       max_comp_len=max_comp, workspace=ws, error_flag=rep["err"],
                       trace_events=events, k_smooth=rep.get("k_smooth"),
                       block_table=rep.get("bt"))


# --------------------------------------------------------------------------------------------
# CPU oracle baseline (bounded sample)
# --------------------------------------------------------------------------------------------

def oracle_sample(wl, n_max: int):
    """The oracle's bounded sample of the serving step: the (b=0, kv head 0) group with its G
    query heads, n_max compressed tokens of codes from the input generator, the window, and the
    seeded codebooks (numpy, float32 / uint8 / fp16)."""
    from compressed_decode_attention_zkv_b200 import inputs as I
    one = I.workload(wl.name, B=1, Hkv=1, Hq=wl.G, n_cal=1024, kmeans_iters=2)
    return dict(q=I.queries(one), kc=I.random_codes(one, "k", max(n_max, 16)),
                vc=I.random_codes(one, "v", max(n_max, 16)), Ck=I.train_codebooks(one, "k"),
                Cv=I.train_codebooks(one, "v"), wk=I.window_tokens(one, "k", np.array([wl.T])),
                wv=I.window_tokens(one, "v", np.array([wl.T])), W=wl.W)


def oracle_step(smp, n):
    """One oracle serving step on the sample: the encode of the evicted window token (K and V)
    and the decode attention over n compressed tokens plus the window.  Returns seconds."""
    from oracle import zkv_oracle as O
    t0 = time.perf_counter()
    O.rvq_encode(smp["wk"][0, 0, :1], smp["Ck"][0])
    O.rvq_encode(smp["wv"][0, 0, :1], smp["Cv"][0])
    O.decode_attn(smp["q"], smp["kc"][:, :, :max(n, 16)], smp["vc"][:, :, :max(n, 16)], [n],
                  smp["Ck"], smp["Cv"], smp["wk"], smp["wv"], [smp["W"]])
    return time.perf_counter() - t0


def oracle_rate(wl, seconds: float, n_tok_cap: int | None = None):
    """Time the oracle's serving step on one host core (BLAS limited to one thread) on the
    bounded sample, its compressed length doubled from 2048 until one step takes a quarter of
    the budget.  Returns (tokens/s in the metric's unit, detail with the sample and n)."""
    from threadpoolctl import threadpool_limits

    smp = oracle_sample(wl, wl.Tc)
    with threadpool_limits(1):
        n = min(2048, wl.Tc)
        t = oracle_step(smp, n)
        while t < seconds / 4 and n < wl.Tc:
            n = min(wl.Tc, n * 2)
            t = oracle_step(smp, n)
        if n_tok_cap:
            n = min(n, n_tok_cap)
        reps, total = 0, 0.0
        while total < seconds and reps < 64:
            total += oracle_step(smp, n)
            reps += 1
    tokens = reps * n / wl.Hkv          # one kv-head group = 1/Hkv of a sequence's heads
    return tokens / total, {"sample": f"oracle serving step on 1 of {wl.B * wl.Hkv} (seq, kv-head) "
                                      f"groups (all {wl.G} query heads), {n} compressed + {wl.W} "
                                      f"window tokens, 2 evicted-token encodes; {reps} reps, "
                                      f"{total:.1f} s; scaled by 1/Hkv to sequence-tokens",
                            "cores": 1, "n": n, "smp": smp}


def _oracle_worker(smp, n, seconds, barrier, queue):
    """One host core's share of the all-core oracle timing (a spawned process): after the start
    barrier, serving steps on the sample until `seconds` have passed."""
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(1):
            oracle_step(smp, min(n, 64))            # imports and first-call costs
            barrier.wait(timeout=300)
            t0 = time.perf_counter()
            reps = 0
            while True:
                oracle_step(smp, n)
                reps += 1
                el = time.perf_counter() - t0
                if el >= seconds:
                    break
        queue.put((reps, el))
    except Exception as exc:   # reported to the parent, which then gives no all-core number
        queue.put(("error", f"{type(exc).__name__}: {exc}"))


def host_cores() -> int:
    """The host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_rate_all_cores(wl, smp, n, seconds: float):
    """The oracle's serving step on every host core at once: one spawned process per core, each
    running the single-core sample (BLAS one thread) from a common start for `seconds`.
    Throughput = all processes' tokens / the longest process time.  Returns (tokens/s, cores)."""
    import multiprocessing as mp
    cores = host_cores()
    ctx = mp.get_context("spawn")   # the parent holds a CUDA context: never fork
    barrier = ctx.Barrier(cores)
    queue = ctx.Queue()
    saved = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS",
                                            "MKL_NUM_THREADS")}
    for k in saved:
        os.environ[k] = "1"
    procs = []
    try:
        for _ in range(cores):
            pr = ctx.Process(target=_oracle_worker, args=(smp, n, seconds, barrier, queue))
            pr.start()
            procs.append(pr)
    finally:
        for k, v in saved.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v
    results = []
    try:
        for _ in procs:
            results.append(queue.get(timeout=300 + 4 * seconds))
    finally:
        for pr in procs:
            pr.join(timeout=10)
            if pr.is_alive():
                pr.kill()
                pr.join()
    errs = [r[1] for r in results if r[0] == "error"]
    if errs:
        raise RuntimeError(errs[0])
    tokens = sum(r[0] for r in results) * n / wl.Hkv
    return tokens / max(r[1] for r in results), cores


def encode_match(dev, sample4=None):
    """The oracle's RVQ encode beside the GPU's codes: the tiny workload's keys and values in
    full, and (sample4, from encode_extra) every 64th token of the 64K-token prefill encode on
    all 8 heads.  Codes are walked stage by stage against the oracle's float64 greedy rule:
    exact, near-tie exceptions (distance gap within 1e-5 relative), mismatches.  Also the
    oracle's single-core encode rate on those rows."""
    import torch
    from threadpoolctl import threadpool_limits

    from compressed_decode_attention_zkv_b200 import inputs as I
    from compressed_decode_attention_zkv_b200 import zkv
    from oracle import zkv_oracle as O

    def walk(x, books, codes):   # x [H][n][d], books [H][S][256][d], codes [n][H][S]
        tot = {"rows": 0, "exact": 0, "exceptions": 0, "mismatches": 0}
        t = 0.0
        with threadpool_limits(1):
            for h in range(x.shape[0]):
                w = O.rvq_match_walk(x[h], books[h], codes[:, h])
                for k in ("exact", "exceptions", "mismatches"):
                    tot[k] += w[k]
                tot["rows"] += x.shape[1]
                t0 = time.perf_counter()
                O.rvq_encode(x[h], books[h])
                t += time.perf_counter() - t0
        tot["oracle_encode_vectors_per_s_1core"] = tot["rows"] / t
        tot["code_decisions"] = tot["exact"] + tot["exceptions"] + tot["mismatches"]
        return tot

    out = {}
    wl = I.workload("tiny")
    parts = []
    for kind in ("k", "v"):
        books = codebooks(wl, kind)
        x = I.kv_tokens(wl, kind, 0, 0, wl.T)            # [Hkv][T][d]
        codes, _ = zkv.rvq_encode(torch.from_numpy(x).to(dev).permute(1, 0, 2),
                                  torch.from_numpy(books).to(dev), with_norms=False)
        parts.append(walk(x, books, codes[0].cpu().numpy()))
    out["tiny_full"] = {k: sum(p[k] for p in parts) for k in ("rows", "exact", "exceptions",
                                                               "mismatches", "code_decisions")}
    out["tiny_full"]["what"] = "tiny K and V, all 1024 tokens, 1 head, S = 2"
    if sample4 is not None:
        parts = [walk(sample4[k]["x"], sample4[k]["books"], sample4[k]["codes"]) for k in ("k", "v")]
        out["prefill_encode_64k_sample"] = {
            k: sum(p[k] for p in parts) for k in ("rows", "exact", "exceptions", "mismatches",
                                                  "code_decisions")}
        out["prefill_encode_64k_sample"]["what"] = (
            "every 64th of 65536 tokens x 8 heads x {K, V}, S = 8, codes from the timed encode")
        out["prefill_encode_64k_sample"]["oracle_encode_vectors_per_s_1core"] = (
            sum(p["rows"] for p in parts) / sum(p["rows"] / p["oracle_encode_vectors_per_s_1core"]
                                               for p in parts))
    return out


def workload_config(wl):
    """The workload fields both arms report."""
    return {"workload": WORKLOAD, "batch": wl.B, "q_heads": wl.Hq, "kv_heads": wl.Hkv,
            "head_dim": wl.d, "context": wl.T, "window": wl.W, "stages_k": wl.Sk,
            "stages_v": wl.Sv, "codewords": 256,
            "step": "append (evict+encode 1 token/seq) + decode attention"}


_POOL_SMP = None
_POOL_LIMIT = None


def _pool_init(smp):
    """Worker set-up for the reference arm's process pool: the sample, BLAS on one thread."""
    global _POOL_SMP, _POOL_LIMIT
    from threadpoolctl import threadpool_limits
    _POOL_SMP = smp
    _POOL_LIMIT = threadpool_limits(1)   # kept alive for the worker's life


def _pool_step(n):
    return oracle_step(_POOL_SMP, n)


def run_reference(args):
    """The reference arm: the oracle's serving step, as it stands, on every host core (one
    process per core, BLAS one thread each, all running the same bounded sample per step)."""
    import multiprocessing as mp

    from compressed_decode_attention_zkv_b200 import inputs as I
    wl = I.workload(WORKLOAD)
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    # bound the whole run to about two minutes: per-step sample sized from a calibration
    per_step = max(0.02, 120.0 / max(1, args.steps + args.warmup))
    rate, info = oracle_rate(wl, seconds=0.5)
    n_cap = int(max(64, min(wl.Tc, rate * wl.Hkv * per_step)))
    smp = info["smp"]
    cores = host_cores()
    saved = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS",
                                            "MKL_NUM_THREADS")}
    for k in saved:
        os.environ[k] = "1"
    times = []
    try:
        with mp.get_context("spawn").Pool(cores, initializer=_pool_init, initargs=(smp,)) as pool:
            pool.map(_pool_step, [64] * cores)   # imports and first-call costs
            for i in range(args.warmup + args.steps):
                t0 = time.perf_counter()
                pool.map(_pool_step, [n_cap] * cores, chunksize=1)
                dt = time.perf_counter() - t0
                if i >= args.warmup:
                    times.append(dt)
    finally:
        for k, v in saved.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v
    total = sum(times)
    value = (len(times) * cores * n_cap / wl.Hkv) / total
    cpu = {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
           "host_cores": cores,
           "sample": f"each step: {cores} processes (one per host core, BLAS one thread), each the "
                     f"oracle serving step on one (seq, kv-head) group of the {WORKLOAD} workload "
                     f"({wl.G} query heads, {n_cap} compressed + {wl.W} window tokens, 2 "
                     f"evicted-token encodes), scaled by 1/Hkv to sequence-tokens",
           "single_core": {"value": rate, "cores": 1, "sample": info["sample"]}}
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * total / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(workload_config(wl), sample="bounded CPU sample per step"),
            "cpu_baseline": cpu,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------------------------
# Our implementation
# --------------------------------------------------------------------------------------------

def scan_src_sha1():
    """sha1 of the scan kernel's source file (the traffic figure stays valid while it is
    unchanged)."""
    return sha1_of(os.path.join(ROOT, "compressed_decode_attention_zkv_b200", "csrc",
                                "scan_rvq.cuh"))


def max_over_ranks(seconds: float, world: int, dev) -> float:
    """The slowest rank's time (every rank calls this at the same point; a no-op for one
    rank).  dev: the rank's device (a CUDA device under NCCL, the CPU under gloo)."""
    if world <= 1:
        return seconds
    import torch
    import torch.distributed as dist
    t = torch.tensor([seconds], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(tokens_per_rank: int, world: int, seconds: float) -> float:
    """Whole-job throughput of the replicated step: every rank processes its own copy of the
    workload, so the job attends world times the tokens of one rank in the slowest rank's
    time."""
    return tokens_per_rank * world / seconds


def sha1_of(path):
    with open(path, "rb") as f:
        return hashlib.sha1(f.read()).hexdigest()


def encode_extra(dev, hbm, bf16):
    """Bulk prefill encode of the 64K-token x 8-head workload (K and V): vectors/s."""
    import torch

    from compressed_decode_attention_zkv_b200 import inputs as I
    from compressed_decode_attention_zkv_b200 import zkv
    wl = I.workload("prefill_encode_64k")
    books = {k: torch.from_numpy(codebooks(wl, k)).to(dev) for k in ("k", "v")}
    xs = {k: torch.from_numpy(I.kv_tokens(wl, k, 0, 0, wl.T)).to(dev).permute(1, 0, 2)
          for k in ("k", "v")}                                          # [T, H, d] views
    codes = {k: torch.empty((wl.T, wl.Hkv, wl.Sk), dtype=torch.uint8, device=dev) for k in xs}
    norms = {k: torch.empty((wl.T, wl.Hkv, wl.Sk), dtype=torch.float32, device=dev) for k in xs}

    def call():
        for k in ("k", "v"):
            zkv.rvq_encode(xs[k], books[k], codes=codes[k], norms=norms[k])

    call()
    torch.cuda.synchronize()
    n_iter = 3
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(n_iter):
        call()
    e.record()
    torch.cuda.synchronize()
    sec = s.elapsed_time(e) / 1000.0 / n_iter
    # every 64th token of each head, for the oracle's code check in the CPU-baseline leg
    sample = {k: {"x": xs[k][::64].permute(1, 0, 2).contiguous().cpu().numpy(),
                  "books": codebooks(wl, k), "codes": codes[k][::64].cpu().numpy()}
              for k in ("k", "v")}
    rows = 2 * wl.T * wl.Hkv
    flops = 2.0 * rows * wl.Sk * 256 * wl.d
    byts = rows * wl.d * 2 + rows * wl.Sk * (1 + 4) + 2 * wl.Hkv * wl.Sk * 256 * wl.d * 4
    # the distance GEMM runs on tcgen05 (kind::tf32): its peak is the measured bf16 GEMM peak
    # times the nominal dense tf32 / bf16 ratio (1.1 / 2.25 PFLOP/s)
    tf32_peak = bf16 * (1.1 / 2.25)
    return {"workload": "prefill_encode_64k (65536 tok x 8 kv heads x {K,V}, d=128, S=8)",
            "vectors_per_s": rows / sec, "ms_per_call": sec * 1000.0,
            "tflops": flops / sec / 1e12, "hbm_gbs": byts / sec / 1e9,
            "bound": "tensor", "peak": tf32_peak, "peak_unit": "TFLOP/s tf32",
            "peak_kind": "measured bf16 GEMM (burst) x nominal tf32/bf16 ratio",
            "frac": flops / sec / 1e12 / tf32_peak,
            "note": "tcgen05 kind::tf32 distance GEMM (M=128 rows, N=256 codewords) into TMEM; "
                    "exact decision: TF32-margin candidates re-scored in float32, then float64",
            "_sample": sample}


def ragged_extra(dev, hbm_peak, R=4, steps=100):
    """The serving step on the ragged batch: 64 sequences with seeded lengths U{1024..16384}
    (Hq 32, Hkv 8, d 128, Sk = Sv = 4, full 128-token windows), one appended token per sequence
    per step.  Codes drawn from the input generator's skewed code distribution (encoding half a
    million prefix tokens on the host would dominate the run), R rotating replicas larger than
    L2, one CUDA graph per replica step, CUDA-event timed."""
    import torch

    from compressed_decode_attention_zkv_b200 import inputs as I
    from compressed_decode_attention_zkv_b200 import zkv
    wl = I.workload("ragged_serving_64")
    lens = I.ragged_lengths(wl)
    comp = (lens - wl.W).astype(np.int64)
    grow = (3 + steps + 2 * R + R - 1) // R + 2
    Tcap = int((comp.max() + grow + 15) // 16 * 16)
    kc = torch.from_numpy(I.random_codes(wl, "k", Tcap)).to(dev)
    vc = torch.from_numpy(I.random_codes(wl, "v", Tcap, seed=1)).to(dev)
    Ck = torch.from_numpy(codebooks(wl, "k")).to(dev)
    Cv = torch.from_numpy(codebooks(wl, "v")).to(dev)
    wk = torch.from_numpy(I.window_tokens(wl, "k", lens)).to(dev)
    wv = torch.from_numpy(I.window_tokens(wl, "v", lens)).to(dev)
    reps = []
    for r in range(R):
        reps.append(dict(
            Ck=Ck.clone(), Cv=Cv.clone(), k_codes=kc.clone(), v_codes=vc.clone(),
            win_k=wk.clone(), win_v=wv.clone(),
            comp_len=torch.from_numpy(comp.astype(np.int32)).to(dev),
            win_len=torch.full((wl.B,), wl.W, dtype=torch.int32, device=dev),
            win_head=torch.zeros((wl.B,), dtype=torch.int32, device=dev),
            q=torch.from_numpy(I.queries(wl, step=r)).to(dev),
            new_k=torch.from_numpy(I.new_tokens(wl, r, "k", lens)).to(dev),
            new_v=torch.from_numpy(I.new_tokens(wl, r, "v", lens)).to(dev),
            out=torch.empty((wl.B, wl.Hq, wl.d), dtype=torch.float32, device=dev),
            lse=torch.empty((wl.B, wl.Hq), dtype=torch.float32, device=dev),
            err=torch.zeros(1, dtype=torch.int32, device=dev)))
    del kc, vc, wk, wv
    max_comp = int(comp.max()) + grow
    need = zkv.decode_workspace_size(reps[0]["q"], reps[0]["k_codes"], reps[0]["v_codes"],
                                     reps[0]["comp_len"], reps[0]["Ck"], reps[0]["Cv"],
                                     reps[0]["win_k"], reps[0]["win_v"], reps[0]["win_len"],
                                     max_comp_len=max_comp)
    wss = [torch.empty(need, dtype=torch.uint8, device=dev) for _ in range(R)]
    host_comp = [int(comp.sum())] * R   # compressed tokens of all sequences, per replica
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(R)]
    for ev in (ev for row in evs for ev in row):   # torch times only events it saw recorded
        ev.record()
    for r in range(R):   # eager call per replica (kernel attributes before capture)
        step_fn(reps[r], wss[r], max_comp)
        host_comp[r] += wl.B
    torch.cuda.synchronize()
    graphs = []
    for r in range(R):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step_fn(reps[r], wss[r], max_comp)
        graphs.append(g)
    for i in range(3):
        graphs[i % R].replay()
        host_comp[i % R] += wl.B
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    tokens = 0
    s.record()
    for i in range(steps):
        r = (3 + i) % R
        graphs[r].replay()
        host_comp[r] += wl.B            # the step's append grows every prefix first
        tokens += host_comp[r]
    e.record()
    torch.cuda.synchronize()
    sec = s.elapsed_time(e) / 1000.0
    assert sum(int(rep["err"].item()) for rep in reps) == 0
    del graphs
    # per-kernel times: graphs with event nodes between the kernels, 2 rounds over the replicas
    # (each replay appends a token to every sequence of its replica; the prefixes have room)
    spans = None
    try:
        tg = []
        for r in range(R):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step_fn(reps[r], wss[r], max_comp, events=evs[r])
            tg.append(g)
        acc = [[], [], []]
        for _ in range(2):
            for r in range(R):
                tg[r].replay()
            torch.cuda.synchronize()
            for r in range(R):
                for i in range(3):
                    acc[i].append(evs[r][i].elapsed_time(evs[r][i + 1]) * 1e3)
        del tg
        spans = {"tables+window+partition+append": statistics.mean(acc[0]),
                 "scan": statistics.mean(acc[1]), "combine": statistics.mean(acc[2]),
                 "unit": "us", "timing": "event nodes between the kernels (no overlap there)"}
    except Exception as exc:
        spans = {"error": f"{type(exc).__name__}: {exc}"}
    step_s = sec / steps
    tc_avg = tokens / steps
    byts = (tc_avg * wl.Hkv * (wl.Sk + wl.Sv) + wl.B * wl.Hkv * wl.W * wl.d * 2 * 2
            + wl.Hkv * (wl.Sk + wl.Sv) * 256 * wl.d * 4 + wl.B * wl.Hq * wl.d * (2 + 4))
    rep_mb = replica_bytes(reps[0]) / 1e6
    return {"workload": "ragged_serving_64 (64 seqs, lengths U{1024..16384} seed 3, Hq 32, "
                        "Hkv 8, d 128, Sk = Sv = 4, W 128)",
            "value": tokens / sec, "unit": UNIT, "ms_per_step": 1000.0 * step_s,
            "seq_tokens_per_s": wl.B / step_s, "compressed_tokens_per_step": tc_avg,
            "kernels_us": spans,
            "step_gbs": byts / step_s / 1e9, "step_frac": byts / step_s / 1e9 / hbm_peak,
            "steps": steps,
            "note": f"one zkv_rvq_serve_step per step; graphs over {R} rotating replicas x "
                    f"{rep_mb:.0f} MB (> L2); codes from the skewed code distribution"}


def decode_only_extra(dev, hbm_peak, name, R, calls, label):
    """Decode attention alone on a named workload: one zkv_rvq_decode_attn per call, replayed
    from CUDA graphs over R rotating replicas of all inputs (R chosen so that they exceed L2).
    Codes from the input generator's code distribution; codebooks trained as for the main
    line."""
    import torch

    from compressed_decode_attention_zkv_b200 import inputs as I
    from compressed_decode_attention_zkv_b200 import zkv
    wl = I.workload(name)
    Tc = wl.Tc
    Tcap = (Tc + 15) // 16 * 16
    kc = torch.from_numpy(I.random_codes(wl, "k", Tcap)).to(dev)
    vc = torch.from_numpy(I.random_codes(wl, "v", Tcap, seed=1)).to(dev)
    Ck = torch.from_numpy(codebooks(wl, "k")).to(dev)
    Cv = torch.from_numpy(codebooks(wl, "v")).to(dev)
    lens = np.full(wl.B, wl.T)
    wk = torch.from_numpy(I.window_tokens(wl, "k", lens)).to(dev)
    wv = torch.from_numpy(I.window_tokens(wl, "v", lens)).to(dev)
    reps = []
    for r in range(R):
        reps.append(dict(q=torch.from_numpy(I.queries(wl, step=r)).to(dev), k_codes=kc.clone(),
                         v_codes=vc.clone(), Ck=Ck.clone(), Cv=Cv.clone(), win_k=wk.clone(),
                         win_v=wv.clone(),
                         comp_len=torch.full((wl.B,), Tc, dtype=torch.int32, device=dev),
                         win_len=torch.full((wl.B,), wl.W, dtype=torch.int32, device=dev),
                         out=torch.empty((wl.B, wl.Hq, wl.d), dtype=torch.float32, device=dev),
                         lse=torch.empty((wl.B, wl.Hq), dtype=torch.float32, device=dev),
                         err=torch.zeros(1, dtype=torch.int32, device=dev)))
    del kc, vc, wk, wv
    keys = ("q", "k_codes", "v_codes", "comp_len", "Ck", "Cv", "win_k", "win_v", "win_len")
    need = zkv.decode_workspace_size(*(reps[0][k] for k in keys), max_comp_len=Tc)
    wss = [torch.empty(need, dtype=torch.uint8, device=dev) for _ in range(R)]

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(R)]
    for ev in (ev for row in evs for ev in row):   # torch times only events it saw recorded
        ev.record()

    def call(r, traced=False):
        rep = reps[r]
        zkv.rvq_decode_attn(*(rep[k] for k in keys), out=rep["out"], lse=rep["lse"],
                            max_comp_len=Tc, workspace=wss[r], error_flag=rep["err"],
                            trace_events=evs[r] if traced else None)
    for r in range(R):   # eager call per replica (kernel attributes before capture)
        call(r)
    torch.cuda.synchronize()
    graphs = []
    for r in range(R):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            call(r)
        graphs.append(g)
    for i in range(2 * R):
        graphs[i % R].replay()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for i in range(calls):
        graphs[i % R].replay()
    e.record()
    torch.cuda.synchronize()
    sec = s.elapsed_time(e) / 1000.0 / calls
    assert sum(int(rep["err"].item()) for rep in reps) == 0
    del graphs
    # per-kernel times: graphs with event nodes between the kernels, 4 rounds over the replicas
    spans = None
    try:
        tg = []
        for r in range(R):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                call(r, traced=True)
            tg.append(g)
        acc = [[], [], []]
        for _ in range(4):
            for r in range(R):
                tg[r].replay()
            torch.cuda.synchronize()
            for r in range(R):
                for i in range(3):
                    acc[i].append(evs[r][i].elapsed_time(evs[r][i + 1]) * 1e3)
        del tg
        spans = {"tables+window+partition": statistics.mean(acc[0]),
                 "scan": statistics.mean(acc[1]), "combine": statistics.mean(acc[2]),
                 "unit": "us", "timing": "event nodes between the kernels (no overlap there)"}
    except Exception as exc:
        spans = {"error": f"{type(exc).__name__}: {exc}"}
    rep_mb = replica_bytes(reps[0]) / 1e6
    byts = (wl.B * wl.Hkv * Tc * (wl.Sk + wl.Sv) + wl.B * wl.Hkv * wl.W * wl.d * 2 * 2
            + wl.Hkv * (wl.Sk + wl.Sv) * 256 * wl.d * 4 + wl.B * wl.Hq * wl.d * 2
            + wl.B * wl.Hq * (wl.d + 1) * 4)
    return {"workload": label,
            "value": wl.B * Tc / sec, "unit": UNIT, "us_per_call": sec * 1e6,
            "call_gbs": byts / sec / 1e9, "call_frac": byts / sec / 1e9 / hbm_peak,
            "calls": calls,
            "algorithmic_bytes": byts, "kernels_us": spans,
            "note": f"zkv_rvq_decode_attn (3 kernels: tables + window + partition, scan, "
                    f"combine) from CUDA graphs over {R} rotating replicas x {rep_mb:.2f} MB "
                    f"(> L2)"}


def pq_encode_extra(dev):
    """Product-VQ (VecInfer) encode of the prefill_encode_64k keys (65536 tokens x 8 kv heads,
    d = 128, sub-vectors of 4 with the smoothing factors): vectors/s."""
    import torch

    from compressed_decode_attention_zkv_b200 import inputs as I
    from compressed_decode_attention_zkv_b200 import zkv
    # a smaller calibration for the codebook: the encode scans all 256 codewords of every
    # sub-vector whatever they are, and full k-means here would take ~45 s of host time
    wl = I.workload("prefill_encode_64k", n_cal=2048, kmeans_iters=4)
    m = 4
    lam_np = I.key_smooth_factors(wl)
    lam = torch.from_numpy(lam_np).to(dev)
    book = torch.from_numpy(I.train_pq_codebook(wl, "k", m, smooth=lam_np)).to(dev)
    x = torch.from_numpy(I.kv_tokens(wl, "k", 0, 0, wl.T)).to(dev).permute(1, 0, 2)   # [T, H, d]
    codes = torch.empty((wl.T, wl.Hkv, wl.d // m), dtype=torch.uint8, device=dev)
    zkv.pq_encode(x, book, codes=codes, smooth=lam)
    torch.cuda.synchronize()
    n_iter = 5
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(n_iter):
        zkv.pq_encode(x, book, codes=codes, smooth=lam)
    e.record()
    torch.cuda.synchronize()
    sec = s.elapsed_time(e) / 1000.0 / n_iter
    rows = wl.T * wl.Hkv
    return {"workload": "prefill_encode_64k keys (65536 tok x 8 kv heads, d=128), product VQ "
                        "with 4-dim sub-vectors (2 bits/elem) and key smoothing",
            "vectors_per_s": rows / sec, "ms_per_call": sec * 1000.0,
            "fp64_gflops": 2.0 * rows * (wl.d // m) * 256 * m / sec / 1e9,
            "note": "one warp per row; float64 distances to all 256 codewords of every "
                    "sub-vector; codebook from 2048 calibration vectors x 4 k-means iterations"}


def pq_decode_extra(dev, hbm_peak, m=4):
    """Product-VQ decode (m-dim sub-vectors: 2 bits/elem at m = 4, 1 at m = 8, on K and V) on
    the llama3_8b_32k shape: seeded codes and codebooks, 2 rotating replicas (268 MB > L2 at
    m = 4, 134 MB at m = 8), CUDA-event timed calls."""
    import torch

    from compressed_decode_attention_zkv_b200 import inputs as I
    from compressed_decode_attention_zkv_b200 import zkv
    wl = I.workload(WORKLOAD)
    R = 2
    Tc, nsub = wl.Tc, wl.d // m
    g = torch.Generator(device=dev).manual_seed(11)
    reps = []
    for r in range(R):
        kc = torch.randint(0, 256, (wl.B, wl.Hkv, Tc, nsub), dtype=torch.uint8, device=dev, generator=g)
        vc = torch.randint(0, 256, (wl.B, wl.Hkv, Tc, nsub), dtype=torch.uint8, device=dev, generator=g)
        Ck = torch.randn((wl.Hkv, 256, m), device=dev, generator=g) * 0.25
        Cv = torch.randn((wl.Hkv, 256, m), device=dev, generator=g)
        q = torch.randn((wl.B, wl.Hq, wl.d), device=dev, generator=g).half()
        wk = torch.randn((wl.B, wl.Hkv, wl.W, wl.d), device=dev, generator=g).half()
        wv = torch.randn((wl.B, wl.Hkv, wl.W, wl.d), device=dev, generator=g).half()
        comp = torch.full((wl.B,), Tc, dtype=torch.int32, device=dev)
        win = torch.full((wl.B,), wl.W, dtype=torch.int32, device=dev)
        reps.append((q, kc, vc, comp, Ck, Cv, wk, wv, win))
    ws = torch.empty(zkv.pq_decode_workspace_size(reps[0][0], reps[0][1], reps[0][4], reps[0][6]),
                     dtype=torch.uint8, device=dev)
    outs = [zkv.pq_decode_attn(*rp, workspace=ws) for rp in reps]   # warm-up, kernel attributes
    torch.cuda.synchronize()
    steps = 100
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for i in range(steps):
        rp = reps[i % R]
        zkv.pq_decode_attn(*rp, out=outs[i % R][0], lse=outs[i % R][1], workspace=ws)
    e.record()
    torch.cuda.synchronize()
    sec = s.elapsed_time(e) / 1000.0 / steps
    code_bytes = 2 * wl.B * wl.Hkv * Tc * nsub
    byts = code_bytes + 2 * wl.B * wl.Hkv * wl.W * wl.d * 2 + wl.B * wl.Hq * wl.d * (2 + 4)
    return {"workload": f"{wl.name} shape, product VQ with {m}-dim sub-vectors on K and V "
                        f"({8 // m} bits/elem, {2 * nsub} code bytes per token and kv head)",
            "value": wl.B * Tc / sec, "unit": UNIT, "us_per_call": sec * 1e6,
            "hbm_gbs": byts / sec / 1e9, "hbm_frac": byts / sec / 1e9 / hbm_peak,
            "note": "zkv_pq_decode_attn (lane = sub-vector scan + finalize), eager calls over "
                    f"{R} rotating replicas"}


def paginate_replica(rep, P, seed):
    """Move a replica's codes into page pools [n_pages, Hkv, P, S] (pages shuffled through a
    pool with spare pages) and give it the block table."""
    import torch
    Bn, Hkv, Tcap, _ = rep["k_codes"].shape
    mp = Tcap // P
    n_pages = Bn * mp + 16
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(n_pages, generator=g)[:Bn * mp].to(rep["k_codes"].device)
    for key in ("k_codes", "v_codes"):
        c = rep[key]
        S = c.shape[3]
        pages = c.view(Bn, Hkv, mp, P, S).permute(0, 2, 1, 3, 4).reshape(Bn * mp, Hkv, P, S)
        pool = torch.zeros((n_pages, Hkv, P, S), dtype=torch.uint8, device=c.device)
        pool[perm] = pages
        rep[key] = pool
    rep["bt"] = perm.view(Bn, mp).to(torch.int32).contiguous()


def variant_extra(wl, args, dev, R, base_ms, smooth=False, page_tokens=0):
    """The serving step of the main line in a variant on the same workload: with the VecInfer
    key smoothing (per-channel factors before the rotation, absorbed into the query; codebooks
    trained on smoothed keys) or with the paged code layout (pages of page_tokens tokens behind
    a block table).  Own replicas, CUDA graphs, the same timing rules.  Returns a dict."""
    import torch

    from compressed_decode_attention_zkv_b200 import zkv
    steps = min(args.steps, 200)
    per_rep = (R + 3 + steps + R - 1) // R + 2
    reps, Tcap = build_state(wl, R, per_rep, dev, smooth=smooth,
                             tcap_multiple=page_tokens if page_tokens else 16)
    if page_tokens:
        for r, rep in enumerate(reps):
            paginate_replica(rep, page_tokens, 1000 + r)
    max_comp = wl.Tc + per_rep
    need = zkv.decode_workspace_size(reps[0]["q"], reps[0]["k_codes"], reps[0]["v_codes"],
                                     reps[0]["comp_len"], reps[0]["Ck"], reps[0]["Cv"],
                                     reps[0]["win_k"], reps[0]["win_v"], reps[0]["win_len"],
                                     max_comp_len=max_comp, block_table=reps[0].get("bt"))
    wss = [torch.empty(need, dtype=torch.uint8, device=dev) for _ in range(R)]
    host_comp = [wl.Tc] * R
    for r in range(R):   # eager call per replica (kernel attributes before capture)
        step_fn(reps[r], wss[r], max_comp)
        host_comp[r] += 1
    torch.cuda.synchronize()
    graphs = []
    for r in range(R):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step_fn(reps[r], wss[r], max_comp)
        graphs.append(g)
    for i in range(3):
        graphs[i % R].replay()
        host_comp[i % R] += 1
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    tokens = 0
    s.record()
    for i in range(steps):
        r = (3 + i) % R
        graphs[r].replay()
        host_comp[r] += 1
        tokens += wl.B * host_comp[r]
    e.record()
    torch.cuda.synchronize()
    sec = s.elapsed_time(e) / 1000.0
    assert sum(int(rep["err"].item()) for rep in reps) == 0
    del graphs
    what = ("VecInfer key smoothing (lambda_i = sqrt(max|K_i|), codebooks trained on smoothed "
            "keys)" if smooth else f"paged codes ({page_tokens}-token pages shuffled through a "
            f"pool, block table [B][{Tcap // page_tokens}])")
    return {"workload": f"{wl.name} with {what}",
            "value": tokens / sec, "unit": UNIT, "ms_per_step": 1000.0 * sec / steps,
            "steps": steps, "main_step_over_this_step": base_ms / (1000.0 * sec / steps),
            "note": "one zkv_rvq_serve_step per step; graphs over "
                    f"{R} rotating replicas (inputs larger than L2)"}


def run_ours(args):
    import torch
    import torch.distributed as dist

    from compressed_decode_attention_zkv_b200 import build as Bld
    from compressed_decode_attention_zkv_b200 import inputs as I
    from compressed_decode_attention_zkv_b200 import zkv

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if rank == 0:
        Bld.build()
    if world > 1:
        dist.barrier()
    zkv.lib()
    hbm_peak, bf16_peak, peak_kind = peaks()

    wl = I.workload(WORKLOAD)
    R = args.replicas
    n_e2e = min(args.steps, 400)
    n_trace_rounds = 8
    # every step (eager warm-up, graph warm-up, timed, traced, e2e, eager fallback) grows one
    # replica's prefixes by 1
    per_rep = (R + args.warmup + args.steps + n_e2e + 2 * n_trace_rounds * R + R - 1) // R + 2
    reps, Tcap = build_state(wl, R, per_rep, dev)
    rep_mb = replica_bytes(reps[0]) / 1e6
    max_comp = wl.Tc + per_rep        # host bound on every prefix length during the run
    need = zkv.decode_workspace_size(reps[0]["q"], reps[0]["k_codes"], reps[0]["v_codes"],
                                     reps[0]["comp_len"], reps[0]["Ck"], reps[0]["Cv"],
                                     reps[0]["win_k"], reps[0]["win_v"], reps[0]["win_len"],
                                     max_comp_len=max_comp)
    wss = [torch.empty(need, dtype=torch.uint8, device=dev) for _ in range(R)]
    host_comp = [wl.Tc] * R          # compressed length of every sequence of each replica

    # trace events per replica: start of the step (tables, partition, encode and length update
    # follow), before the scan, before the combine, after the last kernel
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(R)]
    for e in (e for row in evs for e in row):   # torch only times events it has seen recorded;
        e.record()                               # the library re-records the same handles
    torch.cuda.synchronize()

    def one_step(r, traced=False):
        step_fn(reps[r], wss[r], max_comp, events=evs[r] if traced else None)

    def decode_only(r):
        from compressed_decode_attention_zkv_b200 import zkv as Z
        rep = reps[r]
        Z.rvq_decode_attn(rep["q"], rep["k_codes"], rep["v_codes"], rep["comp_len"], rep["Ck"],
                          rep["Cv"], rep["win_k"], rep["win_v"], rep["win_len"], out=rep["out"],
                          lse=rep["lse"], max_comp_len=max_comp, workspace=wss[r],
                          error_flag=rep["err"])

    # eager warm-up call per replica (sets kernel attributes before capture)
    stream = torch.cuda.Stream(device=dev)
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        for r in range(R):
            one_step(r)
            host_comp[r] += 1
    torch.cuda.current_stream().wait_stream(stream)
    torch.cuda.synchronize()
    # the timed graphs carry no events; a second set with event nodes between the kernels
    # (which end the programmatic overlap at those points) gives the per-kernel times
    graphs, soak_graphs, traced_graphs = [], [], []
    for r in range(R):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            one_step(r)
        graphs.append(g)
        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2):
            decode_only(r)
        soak_graphs.append(g2)
    trace_err = None
    try:
        for r in range(R):
            g3 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g3):
                one_step(r, traced=True)
            traced_graphs.append(g3)
    except Exception as exc:   # no per-kernel times from graphs: the eager pass below
        trace_err = f"{type(exc).__name__}: {exc}"
        traced_graphs = []
    # capture does not execute: the state is unchanged

    step_counter = [0]

    def launch(n):
        for _ in range(n):
            r = step_counter[0] % R
            graphs[r].replay()
            host_comp[r] += 1
            step_counter[0] += 1

    clocks = ClockSampler(local)
    clocks.start()
    launch(args.warmup)
    torch.cuda.synchronize()
    # soak (decode only: leaves the cache unchanged) so clocks reach their loaded state
    t_end = time.perf_counter() + args.soak_s
    while time.perf_counter() < t_end:
        for i in range(64):
            soak_graphs[i % R].replay()
        torch.cuda.synchronize()
    # timed region
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    comp_before = list(host_comp)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    first = step_counter[0]
    launch(args.steps)
    stop.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    elapsed = max_over_ranks(start.elapsed_time(stop) / 1000.0, world, dev)
    # tokens attended in the timed steps: step i uses replica i % R whose prefix grew by one
    tokens = 0
    comp_now = list(comp_before)
    for i in range(first, first + args.steps):
        r = i % R
        comp_now[r] += 1                 # the append inside the step grows the prefix first
        tokens += wl.B * comp_now[r]
    value = weak_scaling_value(tokens, world, elapsed)
    errs = sum(int(rep["err"].item()) for rep in reps)
    assert errs == 0, f"device error flag set: {errs}"

    # per-kernel durations: the traced graphs replayed back to back in the timed rotation, right
    # after the timed region; the spans of each replica's replay are read after each round
    def span(r, a, b):
        return evs[r][a].elapsed_time(evs[r][b]) / 1000.0
    acc = {k: [] for k in ("pre", "scan", "comb")}
    if traced_graphs:
        try:
            for _ in range(n_trace_rounds):
                for r in range(R):
                    traced_graphs[r].replay()
                    host_comp[r] += 1
                torch.cuda.synchronize()
                for r in range(R):
                    acc["pre"].append(span(r, 0, 1))
                    acc["scan"].append(span(r, 1, 2))
                    acc["comb"].append(span(r, 2, 3))
            trace_src = (f"CUDA event nodes in the step graphs: {n_trace_rounds} rounds of the {R} "
                         f"replicas replayed back to back after the timed region")
        except Exception as exc:
            trace_err = f"{type(exc).__name__}: {exc}"
            acc = {k: [] for k in acc}
    if not acc["scan"]:   # event timing inside graphs unavailable: eager steps instead
        print(f"[bench] graph-captured event timing failed ({trace_err}); timing kernels eagerly",
              file=sys.stderr)
        for i in range(n_trace_rounds * R):
            r = i % R
            one_step(r, traced=True)
            host_comp[r] += 1
            torch.cuda.synchronize()
            acc["pre"].append(span(r, 0, 1))
            acc["scan"].append(span(r, 1, 2))
            acc["comb"].append(span(r, 2, 3))
        trace_src = f"CUDA events around each kernel, eager steps ({trace_err})"
    t_pre, t_scan, t_merge = (statistics.mean(acc[k]) for k in ("pre", "scan", "comb"))
    del traced_graphs
    per = {"tables+window+partition+append": t_pre, "scan": t_scan, "combine": t_merge}
    Tc_avg = tokens / (wl.B * args.steps)
    # algorithmic bytes (counted once per distinct byte).  The scan kernel reads the codes of
    # every compressed token: (Sk + Sv) bytes per (token, kv head).
    scan_bytes = wl.B * wl.Hkv * Tc_avg * (wl.Sk + wl.Sv)
    # the whole step: codes, window, codebooks (read by the encode and the decode alike), q,
    # out + lse; the append's new tokens (read, written to the window), evicted rows and codes
    call_bytes = (scan_bytes + wl.B * wl.Hkv * wl.W * wl.d * 2 * 2
                  + wl.Hkv * (wl.Sk + wl.Sv) * 256 * wl.d * 4
                  + wl.B * wl.Hq * wl.d * 2 + wl.B * wl.Hq * (wl.d + 1) * 4
                  + wl.B * wl.Hkv * 2 * (3 * wl.d * 2) + wl.B * wl.Hkv * (wl.Sk + wl.Sv))
    step_time = t_pre + t_scan + t_merge
    traffic = (SCAN_TRAFFIC["bytes_per_launch"]
               if SCAN_TRAFFIC["scan_src_sha1"] == scan_src_sha1() else None)
    roof = {"bound": "hbm", "kernel": "scan2_kernel", "achieved": scan_bytes / t_scan / 1e9,
            "peak": hbm_peak, "unit": "GB/s", "frac": scan_bytes / t_scan / 1e9 / hbm_peak,
            "traffic": traffic, "peak_kind": f"{peak_kind} (hbm_gbs copy, burst)",
            "algorithmic_bytes_per_launch": scan_bytes, "avg_launch_s": t_scan,
            "timing": trace_src}

    # e2e: public API, inputs copied from pinned host memory, result read back, every step.
    # Per replica the step's inputs (new K, new V, q) are views of one device buffer filled by
    # one copy from one pinned host buffer; out and lse are views of one buffer read back by
    # one copy.  The call is the binding's prepared serving step (one library call).
    e2e = None
    if True:
        nk = wl.B * wl.Hkv * wl.d
        nq = wl.B * wl.Hq * wl.d
        n_in, n_out = 2 * nk + nq, nq + wl.B * wl.Hq
        host_in, host_out, dev_in, dev_out, calls = [], [], [], [], []
        for r in range(R):
            rep = reps[r]
            hin = torch.cat([rep["new_k"].flatten(), rep["new_v"].flatten(),
                             rep["q"].flatten()]).cpu().pin_memory()
            din = torch.empty(n_in, dtype=torch.float16, device=dev)
            dout = torch.empty(n_out, dtype=torch.float32, device=dev)
            new_k = din[:nk].view(wl.B, wl.Hkv, wl.d)
            new_v = din[nk:2 * nk].view(wl.B, wl.Hkv, wl.d)
            q = din[2 * nk:].view(wl.B, wl.Hq, wl.d)
            out = dout[:nq].view(wl.B, wl.Hq, wl.d)
            lse = dout[nq:].view(wl.B, wl.Hq)
            call = zkv.PreparedServeStep(new_k, new_v, q, rep["win_k"], rep["win_v"],
                                         rep["win_len"], rep["win_head"], rep["comp_len"],
                                         rep["k_codes"], rep["v_codes"], rep["Ck"], rep["Cv"],
                                         out=out, lse=lse, max_comp_len=max_comp,
                                         workspace=wss[r], error_flag=rep["err"])
            host_in.append(hin)
            host_out.append(torch.empty(n_out, dtype=torch.float32).pin_memory())
            dev_in.append(din)
            dev_out.append(dout)
            calls.append(call)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record()
        tok2 = 0
        for i in range(n_e2e):
            r = i % R
            dev_in[r].copy_(host_in[r], non_blocking=True)
            calls[r]()
            host_out[r].copy_(dev_out[r], non_blocking=True)
            host_comp[r] += 1
            tok2 += wl.B * host_comp[r]
        e2.record()
        torch.cuda.synchronize()
        t2 = max_over_ranks(s2.elapsed_time(e2) / 1000.0, world, dev)
        h2d = n_in * 2
        d2h = n_out * 4
        e2e = {"value": tok2 * world / t2, "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": n_e2e,
               "path": "zkv.PreparedServeStep (one ctypes C-ABI call: zkv_rvq_serve_step), eager, "
                       "per step; one pinned H2D copy of the step's inputs, one D2H copy of "
                       "out + lse"}

    extras = {}
    sample4 = None
    # the extras are single-GPU measurements: a run on several GPUs leaves them to the one-GPU
    # run (rank 0 timing them would keep the other ranks waiting at the final barrier)
    solo = rank == 0 and world == 1
    if rank == 0:
        del graphs, soak_graphs
    if not args.no_encode and solo:
        try:
            extras["encode"] = encode_extra(dev, hbm_peak, bf16_peak)
            sample4 = extras["encode"].pop("_sample")
        except Exception as exc:   # an extra never takes the main line down
            extras["encode"] = {"error": f"{type(exc).__name__}: {exc}"}
    base_ms = 1000.0 * elapsed / args.steps
    for name, kw, skip in (("smooth", dict(smooth=True), args.no_smooth),
                           ("paged", dict(page_tokens=256), args.no_paged)):
        if skip or not solo:
            continue
        reps.clear()
        wss.clear()
        torch.cuda.empty_cache()
        try:
            extras[name] = variant_extra(wl, args, dev, R, base_ms, **kw)
        except Exception as exc:   # an extra never takes the main line down
            extras[name] = {"error": f"{type(exc).__name__}: {exc}"}
    if solo and not args.no_ragged:
        for key, kw in (("decode_only", dict(
                            name="llama3_8b_32k", R=12, calls=600,
                            label="llama3_8b_32k decode only (B 8, Hq 32 / Hkv 8, context 32768, "
                                  "W 128, Sk = Sv = 4)")),
                        ("long_context", dict(
                            name="qwen25_7b_128k", R=24, calls=240,
                            label="qwen25_7b_128k decode (B 1, Hq 28 / Hkv 4, context 131072, "
                                  "W 256, Sk 2, Sv 4)")),
                        ("tiny", dict(
                            name="tiny", R=256, calls=1000,
                            label="tiny decode (1 kv head, d 128, 960 compressed + 64 window "
                                  "tokens, Sk = Sv = 2)"))):
            try:
                extras[key] = decode_only_extra(dev, hbm_peak, **kw)
            except Exception as exc:   # an extra never takes the main line down
                extras[key] = {"error": f"{type(exc).__name__}: {exc}"}
        try:
            extras["ragged_serving"] = ragged_extra(dev, hbm_peak)
        except Exception as exc:   # an extra never takes the main line down
            extras["ragged_serving"] = {"error": f"{type(exc).__name__}: {exc}"}
        torch.cuda.empty_cache()
    # the product-VQ extras come last: nothing measured above depends on them
    for name, fn in (("pq_encode", lambda: pq_encode_extra(dev)),
                     ("pq_decode", lambda: pq_decode_extra(dev, hbm_peak)),
                     ("pq_decode_m8", lambda: pq_decode_extra(dev, hbm_peak, m=8))):
        if args.no_encode or not solo:
            continue
        try:
            extras[name] = fn()
        except Exception as exc:   # an extra never takes the main line down
            extras[name] = {"error": f"{type(exc).__name__}: {exc}"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # the oracle as it stands, on one core and on every host core (one process per core
        # running the same sample); the encode check reports its matching counts
        v1, info = oracle_rate(wl, seconds=args.cpu_seconds)
        try:
            vall, cores = oracle_rate_all_cores(wl, info["smp"], info["n"], args.cpu_seconds / 2)
            cpu = {"value": vall, "unit": UNIT, "cores": cores, "kind": "oracle",
                   "sample": f"{cores} processes (one per host core, BLAS one thread), each: "
                             + info["sample"].split(";")[0]
                             + f"; for {args.cpu_seconds / 2:.1f} s from a common start",
                   "host_cores": host_cores(), "single_core": {"value": v1, "cores": 1,
                                                               "sample": info["sample"]}}
        except Exception as exc:   # the single-core figure stands alone
            cpu = {"value": v1, "unit": UNIT, "cores": 1, "kind": "oracle",
                   "sample": info["sample"], "host_cores": host_cores(),
                   "all_cores_error": f"{type(exc).__name__}: {exc}"}
        try:
            cpu["encode_match"] = encode_match(dev, sample4)
        except Exception as exc:
            cpu["encode_match"] = {"error": f"{type(exc).__name__}: {exc}"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * elapsed / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": dict(workload_config(wl), compressed_tokens_per_seq_avg=Tc_avg,
                           l2=f"{R} rotating replicas x {rep_mb:.1f} MB = {R * rep_mb:.0f} MB > 126 MB L2",
                           parallelism=f"replicas x{world}, no collective",
                           graph="one CUDA graph per replica step"),
            "gpu_launches": 4 * args.steps,   # tables+window+partition, encode, scan, combine
            "roofline": roof,
            "kernels_s": per,
            "step_call": {"seconds": step_time, "algorithmic_bytes": call_bytes,
                          "gbs": call_bytes / step_time / 1e9,
                          "frac": call_bytes / step_time / 1e9 / hbm_peak},
            "clocks": clk,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        line.update(extras)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
