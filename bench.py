#!/usr/bin/env python
"""Throughput of one FOCUS focused denoising step on B200: decoded tokens/s, step latency, roofline.

    python bench.py [--gpus N --steps K --warmup W] [--workload NAME] [--impl reference]

One "step" is one pass of the whole focused step (embed, layers 0-1 with importance, delta / budget /
top-k, compaction, layers 2..L-1 on the kept rows, LM head + decode) over one batch.  The default
workload is the largest one-GPU configuration: the SDAR-8B-shaped random-init bf16 model (36 layers,
hidden 4096, 32 / 8 heads) with 256 ragged requests, block 64, prefixes U[512, 2048] in 64-token pages,
masked fraction U[0.3, 1.0], k_max 16.  Other workloads: sdar1.7b_n32_b32, sdar1.7b_n128_b32 and the
kernel-sweep points sweep_n{N}_b{B}_f{f} (1.7B shape, forced keep fraction f, prefixes U[256, 4096]).
Under torchrun each rank runs an independent replica on its own requests (requests are independent: no
collective on the data path), so the scaling is weak.

`--impl reference` times the CPU oracle (test infrastructure, float64 numpy) on the host cores instead,
one request of the same workload per step.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import focus_synth as fs  # noqa: E402

METRIC = "decoded tokens/s per focused step on 1 B200; step latency; % of roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["focus", "reference"], default="focus")
    ap.add_argument("--workload", default="sdar8b_n256_b64",
                    help="named workload, or sweep_n{N}_b{B}_f{f} for a kernel-sweep point")
    ap.add_argument("--roofline-kernel", default="auto", help="kernel class for the roofline (default: dominant)")
    ap.add_argument("--cpu-baseline-requests", type=int, default=None,
                    help="requests the CPU oracle baseline runs (default: about 20 s of float64 work)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--eager", action="store_true", help="time eager focus_step calls instead of graph replays")
    ap.add_argument("--layers", type=int, default=None, help="override the layer count (profiling cases)")
    ap.add_argument("--requests", type=int, default=None, help="override the request count (profiling cases)")
    ap.add_argument("--mode", choices=["step", "block", "schedule"], default="step",
                    help="step: one focused step (the default measurement); block: whole blocks decoded to "
                         "completion and committed (dense first step, focused steps, dense refresh, commit); "
                         "schedule: a trace of requests through the effective-batch scheduler, focused vs dense")
    return ap.parse_args()


def resolve_workload(name: str):
    """(model shape, workload, base seed) of a named workload or of a sweep point sweep_n{N}_b{B}_f{f}."""
    m = re.fullmatch(r"sweep_n(\d+)_b(\d+)_f([0-9.]+)", name)
    if m:
        return (fs.MODEL_SHAPES["sdar1.7b"], fs.sweep_workload(int(m[1]), int(m[2]), float(m[3])), fs.SEEDS["sweep"])
    sname, wname = fs.CASES[name]
    return fs.MODEL_SHAPES[sname], fs.WORKLOADS[wname], fs.SEEDS.get(name, 1234)


def make_workload(args, seed, device, requests=None):
    """The named workload, optionally with fewer layers / other request counts for small profiling cases."""
    shape, work, _ = resolve_workload(args.workload)
    if args.layers is not None:
        shape = dataclasses.replace(shape, n_layers=args.layers)
    n = requests if requests is not None else args.requests
    if n is not None:
        work = dataclasses.replace(work, n_requests=n)
    return fs.make_case(args.workload, seed=seed, device=device, shape=shape, work=work)


def workload_desc(case: fs.Case) -> str:
    s, w = case.shape, case.work
    return (f"{s.n_layers}L D{s.hidden} {s.n_q_heads}/{s.n_kv_heads} heads d{s.head_dim} F{s.ffn} V{s.vocab} {s.dtype}; "
            f"N={w.n_requests} B={w.block} prefix {w.prefix} page {w.page_size} masked {w.masked} "
            f"k_min {w.k_min} k_max {w.k_max} tau {w.tau} threshold {w.conf_threshold}")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        try:
            d = json.load(open(p))
            return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
        except Exception:
            pass
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.samples = []
        self.proc = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "50", "-i", uuid], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), [x.strip() for x in line.split(",")]))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self, t0, t1):
        rows = [r for t, r in self.samples if t0 <= t <= t1 + 0.06]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no sample inside the timed region"],
                    "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[2]) for r in rows if num(r[2]) is not None]
        mx = [num(r[3]) for r in rows if num(r[3]) is not None]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in rows for n, v in zip(names, r[6:10]) if v.strip().lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max((num(r[4]) or 0.0) for r in rows)}


# ------------------------------------------------------------------ roofline bookkeeping
def algorithmic_work(kclass: str, case: fs.Case, R: int, kept_per_req, plen, splits=1):
    """(bytes, flops) one launch of `kclass` must move / compute at the minimum (operands at the path's
    storage type: bf16, or float32 for the float32 path)."""
    s = case.shape
    D, F, V, Hq, Hkv, d = s.hidden, s.ffn, s.vocab, s.n_q_heads, s.n_kv_heads, s.head_dim
    qkv = (Hq + 2 * Hkv) * d
    N, B = case.work.n_requests, case.work.block
    e = 2 if s.dtype == "bf16" else 4
    full = kclass.startswith("gemm_full")
    M = N * B if full else R
    # outputs: q and the cache rows (bf16) for QKV; the float32 residual read and written for O / down;
    # the SwiGLU activations (bf16) for gate / up; per-tile statistics only (no logits) for the LM head
    gem = {"qkv": (qkv, D, M * qkv * e), "o": (D, Hq * d, M * D * 8), "gateup": (2 * F, D, M * F * e),
           "down": (D, F, M * D * 8), "lmhead": (V, D, M * ((V + 127) // 128) * 12)}
    for key, (n, k, out_bytes) in gem.items():
        if kclass.endswith("_" + key) or kclass == "gemm_" + key:
            return n * k * e + M * k * e + out_bytes, 2.0 * M * n * k
    if kclass in ("attn_score", "attn_ragged"):
        rows = [B] * N if kclass == "attn_score" else list(kept_per_req)
        by = fl = 0.0
        for b in range(N):
            if rows[b] == 0:
                continue
            keys = int(plen[b]) + B
            by += keys * Hkv * d * e * 2 + rows[b] * Hq * d * e * 2
            fl += 4.0 * rows[b] * Hq * d * keys
        return by, fl
    return None, None


def step_work(case: fs.Case, R: int, kept_per_req, plen):
    """Every launch of one step as (kernel class, launches, algorithmic bytes, flops per launch), in the
    step's order: embedding + norm; layers 0-1 on all N*B rows (QKV, attention with importance, O,
    norm, gate/up, down, and a norm between the layers); selection and the row map; the norm that gathers
    the kept rows;
    layers 2..L-1 on the R kept rows (QKV, ragged attention, O, norm, gate/up, down, norm); LM head;
    combine + decode.  Norms read the float32 residual and write bf16 rows (the gathering norm also
    writes the compacted float32 rows).  With more than 256 kept-row slots (N x k_max, bf16) every
    kept-row GEMM is two launches, of which the one whose range misses the live row count does no work."""
    s = case.shape
    L, D = s.n_layers, s.hidden
    N, B = case.work.n_requests, case.work.block
    e = 2 if s.dtype == "bf16" else 4
    rows_full = N * B
    n_kept_layers = L - 2
    work = [("embed_norm", 1, rows_full * D * (e + 4 + e), 0.0)]
    for kc, n in (("gemm_full_qkv", 2), ("attn_score", 2), ("gemm_full_o", 2), ("gemm_full_gateup", 2),
                  ("gemm_full_down", 2)):
        by, fl = algorithmic_work(kc, case, R, kept_per_req, plen)
        work.append((kc, n, by, fl))
    work.append(("row_norm", 3, rows_full * D * (4 + e), 0.0))
    # the importance partials (per KV head and 64-vector query tile) and the mask, then the row map
    q_tiles = -(-(B * (s.n_q_heads // s.n_kv_heads)) // 64) if s.dtype == "bf16" else 1
    work.append(("select", 1, 2 * N * s.n_kv_heads * q_tiles * B * 4 + N * B, 0.0))
    work.append(("select", 1, N * 4 * 2 + R * 3 * 4, 0.0))
    work.append(("row_norm", 1, R * D * (4 + 4 + e), 0.0))
    for kc in ("gemm_qkv", "attn_ragged", "gemm_o", "gemm_gateup", "gemm_down"):
        by, fl = algorithmic_work(kc, case, R, kept_per_req, plen)
        work.append((kc, n_kept_layers, by, fl))
    w = case.work
    k_cap = (min(B, math.ceil(w.forced_keep_frac * B)) if w.forced_keep_frac is not None and w.forced_keep_frac >= 0
             else w.k_max)
    work.append(("row_norm", 2 * n_kept_layers, R * D * (4 + e), 0.0))
    by, fl = algorithmic_work("gemm_lmhead", case, R, kept_per_req, plen)
    work.append(("gemm_lmhead", 1, by, fl))
    if s.dtype == "bf16" and N * k_cap > 256:
        # kept-row bound above 256: each kept-row GEMM is a few-row and a many-row launch, and the one whose
        # range the live row count misses exits after its wait (no work)
        for kc in ("gemm_qkv", "gemm_o", "gemm_gateup", "gemm_down"):
            work.append((kc, n_kept_layers, 0.0, 0.0))
        work.append(("gemm_lmhead", 1, 0.0, 0.0))
    work.append(("decode", 2, R * ((s.vocab + 127) // 128) * 12 + 3 * N * B * 4, 0.0))
    return work


def step_roofline(work, peaks: dict, ms_per_step: float) -> dict:
    """Sum over the step's launches of max(bytes / HBM peak, flops / sustained bf16 peak), against the
    measured step time (a step is seconds of back-to-back kernels, so the sustained tensor figure)."""
    bw, tf = peaks["hbm_gbs"] * 1e9, peaks["bf16_tflops_sustained"] * 1e12
    t_hbm = t_tensor = 0.0
    total_bytes = total_flops = 0.0
    for _kc, n, by, fl in work:
        tb, tt = by / bw, fl / tf
        if tt > tb:
            t_tensor += n * tt
        else:
            t_hbm += n * tb
        total_bytes += n * by
        total_flops += n * fl
    t_roof_ms = (t_hbm + t_tensor) * 1e3
    return {"t_roof_ms": t_roof_ms, "measured_ms": ms_per_step,
            "frac": t_roof_ms / ms_per_step if ms_per_step > 0 else None,
            "hbm_bound_ms": t_hbm * 1e3, "tensor_bound_ms": t_tensor * 1e3,
            "algorithmic_gb": total_bytes / 1e9, "algorithmic_tflop": total_flops / 1e12}


# kernel families: the launches of one role in the step, whichever kernel runs them (the kept-row GEMMs
# run on the swapped few-row kernel up to 256 kept rows and on the row-major kernel above)
FAMILIES = {
    "gemm_kept_rows": ("gemm_qkv", "gemm_o", "gemm_gateup", "gemm_down"),
    "gemm_full_block": ("gemm_full_qkv", "gemm_full_o", "gemm_full_gateup", "gemm_full_down"),
    "gemm_lm_head": ("gemm_lmhead",),
    "attention_ragged": ("attn_ragged",),
    "attention_scoring": ("attn_score",),
    "norms": ("embed_norm", "row_norm", "qkv_finalize"),
    "select_compact": ("select",),
    "decode": ("decode",),
}


def family_rooflines(per_class: dict, work, peaks: dict) -> dict:
    """Per family: device ms per step (summed over its launches), algorithmic bytes and flops per step, the
    bound (tensor when flops / sustained bf16 exceed bytes / HBM) and the achieved rate against that peak."""
    bw, tf = peaks["hbm_gbs"] * 1e9, peaks["bf16_tflops_sustained"] * 1e12
    out = {}
    for fam, classes in FAMILIES.items():
        ms = sum(per_class.get(k, (0.0, 0))[0] for k in classes)
        n = sum(per_class.get(k, (0.0, 0))[1] for k in classes)
        by = sum(cnt * b for kc, cnt, b, f in work if kc in classes)
        fl = sum(cnt * f for kc, cnt, b, f in work if kc in classes)
        if ms <= 0 or n == 0:
            continue
        tensor = fl / tf > by / bw
        ach = fl / (ms / 1e3) / 1e12 if tensor else by / (ms / 1e3) / 1e9
        peak = peaks["bf16_tflops_sustained"] if tensor else peaks["hbm_gbs"]
        out[fam] = {"bound": "tensor" if tensor else "hbm", "achieved": round(ach, 1), "peak": peak,
                    "unit": "TFLOP/s" if tensor else "GB/s", "frac": round(ach / peak, 4), "ms_per_step": round(ms, 4),
                    "launches": n, "algorithmic_gb": round(by / 1e9, 4), "algorithmic_tflop": round(fl / 1e12, 4)}
    return out


def source_digest(kclass: str) -> str:
    """Digest of the sources that build a kernel class (recorded traffic is used only while it matches)."""
    shared = ["common.cuh", "launch.h"]
    files = {"gemm": ["tc_gemm.cu", "tc_gemm_kernel.cuh", "tc_gemm_persist.cuh", "gemm_simt.cu"],
             "attn": ["attention_tc.cu", "attention_t5.cu", "attention_pages.cuh", "attention.cu",
                      "tc_gemm_kernel.cuh"], "row": ["rows.cu"],
             "qkv": ["rows.cu"], "embed": ["rows.cu"], "select": ["select.cu"], "decode": ["decode.cu"]}
    key = kclass.split("_")[0]
    h = hashlib.sha256()
    for f in files.get(key, []) + shared:
        p = os.path.join(ROOT, "decodability_aware_token_b200", "csrc", f)
        if os.path.exists(p):
            h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kclass: str):
    """DRAM bytes per launch of a kernel class from an ncu capture, as recorded in profiles/traffic.md
    (a table row `| class | source digest | bytes per launch | ... |`); None if absent or stale."""
    p = os.path.join(ROOT, "profiles", "traffic.md")
    if not os.path.exists(p):
        return None
    for line in open(p):
        cells = [c.strip() for c in line.strip().strip("|").split("|")]
        if len(cells) >= 3 and cells[0] == kclass and cells[1] == source_digest(kclass):
            try:
                return float(cells[2])
            except ValueError:
                return None
    return None


# ------------------------------------------------------------------ CPU oracle timings
def oracle_tokens_per_s(case_host: fs.Case, requests, model=None):
    from oracle import focus_oracle as fo
    w = case_host.work
    t0 = time.perf_counter()
    r = fo.focus_step(case_host.shape, model if model is not None else case_host.model, case_host.batch, tau=w.tau,
                      k_min=w.k_min, k_max=w.k_max, conf_threshold=w.conf_threshold, alpha=w.alpha,
                      forced_keep_frac=w.forced_keep_frac, requests=list(requests))
    dt = time.perf_counter() - t0
    return int((r.decoded_ids >= 0).sum()), dt


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def oracle_model(model: dict, share: float = 0.5):
    """The weights as float64 arrays (an input form the oracle takes as is) when they fit in `share` of the
    host's free memory, else as given (the oracle then converts the layers it reads on every call).
    Returns (model, converted)."""
    import psutil
    tensors = [t for v in model.values() for t in (v if isinstance(v, list) else [v])]
    if sum(t.numel() for t in tensors) * 8 > share * psutil.virtual_memory().available:
        return model, False
    f64 = lambda t: t.detach().cpu().to(torch.float64).numpy()
    return {k: ([f64(t) for t in v] if isinstance(v, list) else f64(v)) for k, v in model.items()}, True


def cpu_oracle_sample(case: fs.Case, model, seconds: float, max_requests=None):
    """Time the oracle one request per call, in request order, until `seconds` of CPU work have run (at
    least one request).  Returns (decoded tokens, seconds, requests run)."""
    N = case.work.n_requests
    limit = N if max_requests is None else min(N, max_requests)
    tok, secs, n = 0, 0.0, 0
    while n < limit and (secs < seconds or n == 0):
        t, dt = oracle_tokens_per_s(case, [n], model)
        tok, secs, n = tok + t, secs + dt, n + 1
    return tok, secs, n


def run_reference(args):
    """The oracle on the host cores: each step is one request of the workload (requests cycle).  Only the
    requests the run visits are generated (same shapes, distributions and seed), so that the 8B shape's
    page pool fits on the host; the weights are converted to float64 once, before the timed steps, when
    the host has room for them."""
    shape, work, base = resolve_workload(args.workload)
    n_used = max(1, min(work.n_requests if args.requests is None else args.requests, args.warmup + args.steps))
    case = make_workload(args, base, "cpu", requests=n_used)
    full = fs.Case(case.shape, dataclasses.replace(case.work, n_requests=work.n_requests if args.requests is None
                                                   else args.requests), None, None, case.seed)
    model, converted = oracle_model(case.model)
    for i in range(args.warmup):
        oracle_tokens_per_s(case, [i % n_used], model)
    tok, secs = 0, 0.0
    for i in range(args.steps):
        t, dt = oracle_tokens_per_s(case, [(args.warmup + i) % n_used], model)
        tok += t
        secs += dt
    value = tok / secs if secs > 0 else 0.0
    cores = blas_threads()
    sample = (f"one request per step, cycling over the first {n_used} requests of the workload (same shapes "
              f"and distributions), float64 oracle, " +
              ("weights converted to float64 once before the timed steps" if converted else
               "weights converted inside every step (host memory too small to hold them in float64)"))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / max(1, args.steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "desc": workload_desc(full), "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ replicas (one process per GPU)
# Requests are independent, so N GPUs run N replicas, each on its own batch of the workload (no
# collective on the data path); the ranks meet only to time the job: the slowest rank's device time
# and the sum of the tokens all ranks decoded.
def rank_seed(base: int, rank: int) -> int:
    """Seed of rank `rank`'s requests (same shapes and distributions, different draws)."""
    return base + 7919 * rank


def reduce_over_ranks(elapsed_ms: float, decoded: float, world: int, device) -> tuple[float, float]:
    """(max over ranks of elapsed_ms, sum over ranks of decoded); a collective only when world > 1."""
    import torch.distributed as dist
    t = torch.tensor([elapsed_ms], dtype=torch.float64, device=device)
    tk = torch.tensor([decoded], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.all_reduce(tk, op=dist.ReduceOp.SUM)
    return float(t.item()), float(tk.item())


def whole_job_rate(total_units: float, max_ms: float) -> float:
    """Units all ranks processed per second of the slowest rank's time."""
    return total_units / (max_ms / 1e3) if max_ms > 0 else 0.0


# ------------------------------------------------------------------ whole blocks
def run_block_mode(args, case, dev, world, barrier):
    """Decode whole blocks through focus_decode_block: the dense first step, focused steps until nothing is
    masked (the loop reads the remaining count after every step), the dense refresh and the commit of
    the block's K/V into the prefix pages.  Each timed block starts from the workload's initial block
    state and prefix lengths.  tokens/s = masked positions decoded / device time of the blocks."""
    from decodability_aware_token_b200 import FocusContext, StepParams
    w, shp = case.work, case.shape
    N, B = w.n_requests, w.block
    batch = fs.with_block_pages(case.batch, B)
    params = StepParams(w.tau, w.k_min, w.k_max, w.conf_threshold, w.alpha, -1.0)
    ctx = FocusContext(shp, case.model, max_requests=N, max_block=B, max_keep=B,
                       max_pages_per_req=int(batch["page_table"].shape[1]))
    init = {k: batch[k].clone() for k in ("block_tokens", "mask", "ibc", "prefix_len")}
    st = dict(batch)
    masked = int(init["mask"].sum())

    def one_block():
        for k, v in init.items():
            st[k].copy_(v)
        return ctx.decode_block(st, params)[1]

    for _ in range(max(1, args.warmup)):
        one_block()
    torch.cuda.synchronize(dev)
    K = max(1, min(args.steps, 20))
    sampler = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    tw0 = time.time()
    ev0.record(stream)
    steps = [one_block() for _ in range(K)]
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    tw1 = time.time()
    barrier()
    sampler.stop()
    elapsed = ev0.elapsed_time(ev1)
    max_ms, total = reduce_over_ranks(elapsed, masked * K, world, dev)
    if int(os.environ.get("RANK", "0")) == 0:
        line = {
            "metric": "decoded tokens/s, whole blocks (dense first step, focused steps, dense refresh, commit)",
            "value": whole_job_rate(total, max_ms), "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_block": max_ms / K, "focused_steps_per_block": statistics.mean(steps) - 1,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": shp.dtype,
            "data": "synthetic", "clocks": sampler.summary(tw0, tw1),
            "config": {"workload": args.workload, "mode": "block", "desc": workload_desc(case),
                       "masked_per_block": masked, "requests_per_gpu": N,
                       "launch": "eager calls; the loop synchronises after every step to read the masked count"},
        }
        print(json.dumps(line), flush=True)
    ctx.close()


# ------------------------------------------------------------------ a trace through the scheduler
class _DenseEngine:
    """A plain block-diffusion engine for comparison: every step of every block keeps the whole block."""

    def __init__(self, engine):
        self.engine = engine

    def capacity_check(self, slots, block):
        self.engine.capacity_check(slots, block)

    def step(self, view, dense):
        self.engine.step(view, True)

    def commit(self, view):
        self.engine.commit(view)


def run_schedule_mode(args, case, dev, world, barrier):
    """Continuous batching of a request trace through the effective-batch scheduler (host loop around
    focus_step / focus_commit_block): 2N requests of the workload's model and prefix distribution, one or two
    blocks each, arriving a few per iteration, over N slots and the row budget of a dense engine on N
    requests (N x B).  Run twice on this GPU: with focused steps (a focused request costs k_max rows, so more
    requests share the budget) and with a dense engine (every step keeps the whole block, every request
    costs B rows).  tokens/s = block positions decoded / device time of the whole trace (the scheduler reads
    the mask state after every iteration, so host work is inside that time)."""
    from decodability_aware_token_b200 import FocusContext, StepParams
    from decodability_aware_token_b200.scheduler import EffectiveBatchScheduler, FocusEngine, Request
    w, shp = case.work, case.shape
    N, B = w.n_requests, w.block
    pool0, table, plen = case.batch["kv_pool"], case.batch["page_table"].cpu(), case.batch["prefix_len"].cpu()
    S = int(pool0.shape[4])
    n_req = 2 * N
    g = torch.Generator().manual_seed(7)
    src = torch.randint(0, N, (n_req,), generator=g).tolist()            # prompt of request r: that of src[r]
    nblk = (1 + torch.randint(0, 2, (n_req,), generator=g)).tolist()
    arrive = [r // max(1, N // 4) for r in range(n_req)]
    max_pages = max(-(-(int(plen[b]) + 2 * B) // S) for b in range(N)) + 1
    # requests share their source's full prompt pages (read only); a partly filled last page receives the
    # first committed positions, so every request gets its own copy of it
    n0 = int(pool0.shape[0])
    prompt_pages, copies = [], []
    for r in range(n_req):
        b = src[r]
        n_pg = -(-int(plen[b]) // S)
        pg = table[b, :n_pg].tolist()
        if int(plen[b]) % S:
            copies.append(pg[-1])
            pg[-1] = n0 + len(copies) - 1
        prompt_pages.append(pg)
    spare = n_req * (-(-2 * B // S) + 1)
    extra = torch.zeros((len(copies) + spare,) + tuple(pool0.shape[1:]), dtype=pool0.dtype, device=pool0.device)
    if copies:
        extra[: len(copies)] = pool0[torch.tensor(copies, device=pool0.device)]
    pool_init = torch.cat([pool0, extra], 0)
    free0 = list(range(n0 + len(copies), int(pool_init.shape[0])))
    params = StepParams(w.tau, w.k_min, w.k_max, w.conf_threshold, w.alpha)

    def trace(dense: bool):
        pool = pool_init.clone()
        reqs = [Request(r, arrive[r], int(plen[src[r]]), prompt_pages[r], nblk[r]) for r in range(n_req)]
        with FocusContext(shp, case.model, max_requests=N, max_block=B, max_keep=B,
                          max_pages_per_req=max_pages) as ctx:
            eng = FocusEngine(ctx, params)
            sch = EffectiveBatchScheduler(_DenseEngine(eng) if dense else eng, slots=N, block=B,
                                          n_layers=shp.n_layers, n_kv_heads=shp.n_kv_heads, head_dim=shp.head_dim,
                                          max_pages_per_req=max_pages, kv_pool=pool, free_pages=free0,
                                          mask_token=shp.vocab - 1, k_max=B if dense else w.k_max,
                                          row_budget=N * B, keep_pages=True)
            for rq in reqs:
                sch.submit(rq)
            torch.cuda.synchronize(dev)
            barrier()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            sch.run(max_iterations=100_000)
            e1.record()
            torch.cuda.synchronize(dev)
            ms = e0.elapsed_time(e1)
        decoded = sum(nblk) * B
        return ms, decoded, sch.iteration, max(st.active for st in sch.stats)

    sampler = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    time.sleep(0.3)
    tw0 = time.time()
    f_ms, f_tok, f_it, f_peak = trace(False)
    d_ms, d_tok, d_it, d_peak = trace(True)
    tw1 = time.time()
    sampler.stop()
    f_max, f_total = reduce_over_ranks(f_ms, f_tok, world, dev)
    d_max, d_total = reduce_over_ranks(d_ms, d_tok, world, dev)
    if int(os.environ.get("RANK", "0")) == 0:
        line = {
            "metric": "decoded tokens/s over a request trace (effective-batch scheduler, focused vs dense steps)",
            "value": whole_job_rate(f_total, f_max), "unit": UNIT, "n_gpus": world, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": shp.dtype, "data": "synthetic",
            "dense_engine": {"value": whole_job_rate(d_total, d_max), "ms": d_max, "iterations": d_it,
                             "max_active": d_peak},
            "focused": {"ms": f_max, "iterations": f_it, "max_active": f_peak},
            "speedup_vs_dense": (d_max / f_max) if f_max > 0 else None,
            "clocks": sampler.summary(tw0, tw1),
            "config": {"workload": args.workload, "mode": "schedule", "desc": workload_desc(case),
                       "requests": n_req, "slots": N, "row_budget": N * B, "blocks": sum(nblk),
                       "launch": "eager calls; the scheduler reads the mask state after every iteration"},
        }
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ the GPU arm
def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            run_reference(args)
        return
    import torch.distributed as dist
    from decodability_aware_token_b200 import FocusContext, StepParams, StepOutputs

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    base = fs.SEEDS.get(args.workload, 1234)
    case = make_workload(args, rank_seed(base, rank), dev)    # this rank's requests
    w, shp = case.work, case.shape
    N, B = w.n_requests, w.block
    if args.mode in ("block", "schedule"):
        (run_block_mode if args.mode == "block" else run_schedule_mode)(args, case, dev, world, barrier)
        if world > 1:
            dist.destroy_process_group()
        return
    params = StepParams(w.tau, w.k_min, w.k_max, w.conf_threshold, w.alpha, w.forced_keep_frac)
    mk = B if w.forced_keep_frac >= 0 else w.k_max
    ctx = FocusContext(shp, case.model, max_requests=N, max_block=B, max_keep=mk,
                       max_pages_per_req=case.max_pages_per_req)
    K, Wm = args.steps, max(3, args.warmup)
    tok0, mask0, ibc0 = case.batch["block_tokens"], case.batch["mask"], case.batch["ibc"]

    # The step decodes in place: every timed step starts from the workload's initial tokens and mask
    # (two small copies).  The intra-block KV cache needs no reset: a step rewrites every entry it reads
    # before reading it (all positions at layers 0-1, the kept rows at later layers), so after one step
    # it is a fixed point and each step repeats the same work.
    st = dict(case.batch)
    st["block_tokens"], st["mask"], st["ibc"] = tok0.clone(), mask0.clone(), ibc0.clone()
    out = StepOutputs.alloc(N, B, mk, shp.hidden, dev, importance=False, hidden=False)
    stream = torch.cuda.current_stream(dev)

    def one_step():
        st["block_tokens"].copy_(tok0)
        st["mask"].copy_(mask0)
        ctx.step(st, params, out)

    for i in range(Wm):
        one_step()
    torch.cuda.synchronize(dev)
    launches_per_step = ctx.last_step_launches()
    kept = out.keep_count.cpu()
    R = int(kept.sum())
    plen = case.batch["prefix_len"].cpu()

    # device time per kernel class (untimed: one captured step per class, event pairs around its launches)
    from decodability_aware_token_b200 import _abi
    per_class = {}
    if args.roofline_kernel == "auto":
        for kc in _abi.KERNEL_CLASSES:
            ctx.profile_begin(kc, 4096)
            try:
                if args.eager:
                    one_step()
                else:
                    probe = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(probe):
                        one_step()
                    probe.replay()
                    torch.cuda.synchronize(dev)
                ms, n = ctx.profile_end()
            except RuntimeError:
                ms, n = 0.0, 0
            per_class[kc] = (ms, n)
        roof_class = max(per_class, key=lambda k: per_class[k][0])
    else:
        roof_class = args.roofline_kernel
    torch.cuda.synchronize(dev)

    # the step is captured as a CUDA graph (its launch sequence depends only on host-visible sizes), once
    # plain -- the timed replays -- and once with event pairs around every launch of the roofline kernel
    # class, replayed in a second timed loop for that kernel's launch durations (event nodes between
    # kernels would interrupt the programmatic launch chain of the plain graph)
    graph = graph_prof = None
    if not args.eager:
        try:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                one_step()
            graph.replay()
            ctx.profile_begin(roof_class, 4096)
            graph_prof = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph_prof):
                one_step()
            graph_prof.replay()
            torch.cuda.synchronize(dev)
        except RuntimeError as exc:  # capture refused: time eager calls instead, and say so
            print(f"CUDA graph capture failed ({exc}); timing eager calls", file=sys.stderr)
            graph = graph_prof = None
            args.eager = True
            try:
                ctx.profile_end()
            except RuntimeError:
                pass

    # ---- timed region: device events on the launching stream, max over ranks
    sampler = ClockSampler(local)
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize(dev)
    if args.eager:
        ctx.profile_begin(roof_class, max(1, K * 64))
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    tw0 = time.time()
    ev0.record(stream)
    for i in range(K):
        if graph is not None:
            graph.replay()
        else:
            one_step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    tw1 = time.time()
    if graph_prof is not None:  # the roofline kernel's launches, timed over K profiled replays
        for i in range(K):
            graph_prof.replay()
        torch.cuda.synchronize(dev)
    try:
        kern_ms, kern_n = ctx.profile_end()   # graph: the event pairs of the last replay
    except RuntimeError as exc:
        print(f"kernel timing unavailable ({exc})", file=sys.stderr)
        kern_ms, kern_n = 0.0, 0
    barrier()
    time.sleep(0.1)
    sampler.stop()
    clocks = sampler.summary(tw0, tw1)
    elapsed = ev0.elapsed_time(ev1)
    decoded = int((out.decoded_ids >= 0).sum()) * K     # every step repeats the same (deterministic) work
    max_ms, total_decoded = reduce_over_ranks(elapsed, decoded, world, dev)
    value = whole_job_rate(total_decoded, max_ms)
    del graph, graph_prof

    # ---- end to end through the public API (eager calls) with pinned host buffers
    e2e = None
    if not args.no_e2e:
        host_in = {k: case.batch[k].cpu().pin_memory() for k in ("block_tokens", "mask", "prefix_len", "page_table")}
        out_h = StepOutputs.alloc(N, B, mk, shp.hidden, "cpu", importance=False, hidden=False, pin_memory=True)
        names = ("keep_count", "retained_idx", "decoded_ids", "conf", "top_id")
        h2d = sum(v.numel() * v.element_size() for v in host_in.values())
        d2h = sum(getattr(out_h, k).numel() * getattr(out_h, k).element_size() for k in names)
        torch.cuda.synchronize(dev)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e_dec = 0
        e0.record(stream)
        for i in range(K):
            for k_, v in host_in.items():
                st[k_].copy_(v, non_blocking=True)
            o = ctx.step(st, params, out)
            for k_ in names:
                getattr(out_h, k_).copy_(getattr(o, k_), non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = e0.elapsed_time(e1)
        e_dec = int((out_h.decoded_ids >= 0).sum()) * K
        e_max_ms, e_total = reduce_over_ranks(e_ms, e_dec, world, dev)
        e2e = {"value": whole_job_rate(e_total, e_max_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h}

    # ---- roofline of the dominant kernel class
    peaks, peak_src = load_peaks()
    by, fl = algorithmic_work(roof_class, case, R, kept.tolist(), plen.tolist())
    roofline = None
    if by is not None and kern_n > 0:
        avg_s = kern_ms / kern_n / 1e3
        t_b = by / (peaks["hbm_gbs"] * 1e9)
        t_f = fl / (peaks["bf16_tflops_sustained"] * 1e12)
        if t_f > t_b:
            ach = fl / avg_s / 1e12
            roofline = {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                        "frac": ach / peaks["bf16_tflops_sustained"]}
        else:
            ach = by / avg_s / 1e9
            roofline = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": ach / peaks["hbm_gbs"]}
        roofline.update({"traffic": recorded_traffic(roof_class), "kernel": roof_class,
                         "peak_source": f"{peak_src} ({'sustained bf16' if roofline['bound'] == 'tensor' else 'HBM copy'})",
                         "launches_timed": kern_n, "avg_launch_us": avg_s * 1e6,
                         "algorithmic_bytes_per_launch": by, "algorithmic_flops_per_launch": fl,
                         "kept_rows": R})

    # ---- the whole step against its roofline (sum over launches of the slower of bytes and flops)
    work_list = step_work(case, R, kept.tolist(), plen.tolist())
    step_roof = step_roofline(work_list, peaks, max_ms / K)
    step_roof["peak_source"] = f"{peak_src} (HBM copy; sustained bf16)"
    families = family_rooflines(per_class, work_list, peaks) if per_class else None
    weights_gb = sum(t.numel() * t.element_size() for v in case.model.values()
                     for t in (v if isinstance(v, list) else [v])) / 1e9
    kv_gb = float(plen.sum()) * shp.n_layers * 2 * shp.n_kv_heads * shp.head_dim * case.batch["kv_pool"].element_size() / 1e9

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # the oracle reads the model and the batch from host copies, and the page pool (tens of GB at the 8B
        # shape) page by page from the device
        del st
        host_batch = {k: (v if k == "kv_pool" else v.cpu()) for k, v in case.batch.items()}
        host_batch["block_tokens"], host_batch["mask"], host_batch["ibc"] = tok0.cpu(), mask0.cpu(), ibc0.cpu()
        host = fs.Case(shp, w, None, host_batch, case.seed)
        model64, converted = oracle_model(case.model)
        ctok, csec, nreq = cpu_oracle_sample(host, model64, 20.0, args.cpu_baseline_requests)
        cpu = {"value": ctok / csec, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"{nreq} of {N} requests of the same batch, one oracle call each ({csec:.1f} s of "
                         f"float64 work; weights converted to float64 " +
                         ("once, untimed)" if converted else "inside every call)")}
        del model64

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": Wm,
            "ms_per_step": max_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if shp.dtype == "bf16" else "f32", "data": "synthetic",
            "config": {"workload": args.workload + ("" if args.layers is None and args.requests is None else
                                                    f" (layers={shp.n_layers}, requests={N})"),
                       "desc": workload_desc(case), "requests_per_gpu": N,
                       "global_batch": N * world, "block": B, "kept_rows_per_step": R,
                       "decoded_per_step": total_decoded / K / world,
                       "launch": "eager focus_step calls" if args.eager else
                                 "CUDA graph of one focus_step, one replay per step (tokens/mask restored by two copies)",
                       "l2": f"inputs larger than L2 ({weights_gb:.1f} GB of weights and {kv_gb:.1f} GB of prefix KV "
                             f"pages read per step, against a 126 MB L2)",
                       "parallelism": f"replicas x{world} (requests sharded, no collective)"},
            "gpu_launches": launches_per_step * K,
            "clocks": clocks, "roofline": roofline, "step_roofline": step_roof, "families": families,
            "cpu_baseline": cpu, "e2e": e2e,
            "per_class_ms_per_step": {k: round(v[0], 4) for k, v in per_class.items()} if per_class else None,
        }
        print(json.dumps(line), flush=True)
    ctx.close()
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
