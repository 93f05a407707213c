"""Seeded synthetic inputs for one FOCUS focused denoising step.

This module is shared by the CPU oracle side (tests, CPU baseline) and the CUDA
side (tests, bench).  It only draws random numbers and lays them out; it holds
none of the step's arithmetic (no norm, projection, attention, selection or
decoding).

Model shapes follow the two model families the FOCUS pages name (SDAR and
LLaDA2.0; "FOCUS: DLLMs Know How to Tame Their Compute Bound", project page,
Overview and Efficiency): the weights are random-init because no trained
checkpoint is available.  Workload structure (block size, ragged prefixes held
in fixed-size KV pages, a masked subset of each block) follows the same page's
Overview -- Motivation and Runtime Action: a block of B tokens is denoised at
each step on top of an exactly cached prefix.

Recipe (all seeded; every tensor gets its own generator seeded from
(base seed, tensor name, layer), so generation order does not matter; tensors of more than 2^30
elements are drawn in 2^28-element slices with one generator per slice):
  * weights  ~ N(0, 0.02), norms gamma ~ 1 + N(0, 0.1), embeddings ~ N(0, 1),
    rounded to the model dtype (bf16, or fp32 for the tiny model);
  * prefix KV pages and the intra-block KV cache ~ N(0, 1), model dtype;
  * prefix lengths per request from the workload's distribution, pages of
    `page_size` tokens, physical page ids a seeded permutation;
  * masked positions: a seeded random subset of each block, count fixed or
    round(u * B) with u uniform; masked positions hold the mask token id V-1,
    the others uniform random ids in [0, V-1).
"""
from __future__ import annotations

import dataclasses
import hashlib
import math
from concurrent.futures import ThreadPoolExecutor
from typing import Optional

import torch

__all__ = [
    "ModelShape", "Workload", "Case", "MODEL_SHAPES", "WORKLOADS",
    "make_model", "make_batch", "make_case", "sweep_workload",
]


@dataclasses.dataclass(frozen=True)
class ModelShape:
    n_layers: int
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    dtype: str = "bf16"          # "bf16" or "f32"
    rms_eps: float = 1e-6
    rope_theta: float = 10000.0

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def qkv_dim(self):
        return (self.n_q_heads + 2 * self.n_kv_heads) * self.head_dim


@dataclasses.dataclass(frozen=True)
class Workload:
    n_requests: int
    block: int
    page_size: int
    prefix: tuple                 # ("fixed", P) | ("uniform", lo, hi) | ("lognormal", median, sigma, lo, hi)
    masked: tuple                 # ("count", n) | ("frac", lo, hi)
    k_min: int = 1
    k_max: int = 8
    tau: float = 0.0
    conf_threshold: float = 0.9
    alpha: float = 1.0
    forced_keep_frac: float = -1.0
    spare_pages: int = 3


MODEL_SHAPES = {
    # random-init 4-layer fp32 model for the tiny step
    "tiny": ModelShape(4, 256, 4, 4, 64, 1024, 1024, "f32"),
    # SDAR-1.7B-shaped
    "sdar1.7b": ModelShape(28, 2048, 16, 8, 128, 6144, 151936, "bf16"),
    # SDAR-8B-shaped
    "sdar8b": ModelShape(36, 4096, 32, 8, 128, 12288, 151936, "bf16"),
    # reduced bf16 shapes: several GEMM / attention tiles and ragged tails,
    # small enough for the oracle to finish in seconds
    "small_bf16": ModelShape(4, 512, 8, 4, 128, 1536, 4000, "bf16"),
    "small_bf16_g4": ModelShape(3, 512, 8, 2, 128, 1024, 2100, "bf16"),
    "small_f32": ModelShape(3, 256, 4, 2, 64, 768, 700, "f32"),
    # hidden 2048 with enough block rows that the many-row GEMMs run on the persistent kernel, still
    # small enough (3 layers, vocabulary 4096) for the oracle
    "wide_bf16": ModelShape(3, 2048, 16, 8, 128, 3072, 4096, "bf16"),
}

WORKLOADS = {
    "tiny": Workload(2, 16, 16, ("fixed", 64), ("count", 10), k_min=2, k_max=8, tau=0.0, conf_threshold=0.9),
    "sdar1.7b_n32_b32": Workload(32, 32, 64, ("uniform", 256, 1024), ("frac", 0.3, 1.0), k_min=1, k_max=8),
    "sdar1.7b_n128_b32": Workload(128, 32, 64, ("lognormal", 600.0, 0.8, 64, 4096), ("frac", 0.3, 1.0), k_min=1, k_max=12),
    "sdar8b_n256_b64": Workload(256, 64, 64, ("uniform", 512, 2048), ("frac", 0.3, 1.0), k_min=1, k_max=16),
    # reduced workloads for parity at oracle-friendly sizes
    "small": Workload(5, 32, 64, ("uniform", 0, 300), ("frac", 0.3, 1.0), k_min=1, k_max=8),
    "small_b16": Workload(6, 16, 16, ("uniform", 0, 90), ("frac", 0.0, 1.0), k_min=2, k_max=6),
    "wide": Workload(41, 64, 64, ("uniform", 0, 600), ("frac", 0.3, 1.0), k_min=1, k_max=16),
}

# seed of each named case: 1234 + the workload's index among the five
# workloads (tiny, 1.7B N32, 1.7B N128, 8B N256, 1.7B sweep); reduced cases from 2001
SEEDS = {
    "tiny": 1235, "sdar1.7b_n32_b32": 1236, "sdar1.7b_n128_b32": 1237, "sdar8b_n256_b64": 1238,
    "sweep": 1239, "small_bf16": 2001, "small_bf16_g4": 2002, "small_f32": 2003, "wide_bf16": 2004,
}

# named cases: (model shape, workload)
CASES = {
    "tiny": ("tiny", "tiny"),
    "sdar1.7b_n32_b32": ("sdar1.7b", "sdar1.7b_n32_b32"),
    "sdar1.7b_n128_b32": ("sdar1.7b", "sdar1.7b_n128_b32"),
    "sdar8b_n256_b64": ("sdar8b", "sdar8b_n256_b64"),
    "small_bf16": ("small_bf16", "small"),
    "small_bf16_g4": ("small_bf16_g4", "small_b16"),
    "small_f32": ("small_f32", "small_b16"),
    "wide_bf16": ("wide_bf16", "wide"),
}


def sweep_workload(n_requests: int, block: int, keep_frac: float) -> Workload:
    """Kernel-sweep workload on the 1.7B shape: forced keep fraction, prefixes U[256, 4096]."""
    return Workload(n_requests, block, 64, ("uniform", 256, 4096), ("frac", 0.3, 1.0),
                    k_min=1, k_max=block, forced_keep_frac=keep_frac)


@dataclasses.dataclass
class Case:
    shape: ModelShape
    work: Workload
    model: dict                    # name -> tensor (per-layer tensors in lists)
    batch: dict                    # name -> tensor
    seed: int

    @property
    def max_pages_per_req(self) -> int:
        return int(self.batch["page_table"].shape[1])


def _seed_of(base: int, name: str, layer: int = -1) -> int:
    h = hashlib.blake2b(f"{base}/{name}/{layer}".encode(), digest_size=8).digest()
    return int.from_bytes(h, "little") & ((1 << 62) - 1)


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


_SLICE = 1 << 28  # elements drawn per generator for very large tensors


def _normal(shape, std, mean, seed, device, dtype):
    """N(mean, std^2) in float32, rounded to `dtype`.  Tensors of more than 2^30 elements (the page pools of
    the full-size workloads) are drawn in slices of 2^28 elements, each from its own generator seeded from
    (seed, slice index), straight into the result: the float32 draw of a whole 60 GB page pool would not fit
    on the device next to it."""
    n = math.prod(shape)
    if n <= (1 << 30):
        g = _gen(device, seed)
        t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        if std != 1.0:
            t.mul_(std)
        if mean != 0.0:
            t.add_(mean)
        return t.to(dtype)
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(-1)
    for i, lo in enumerate(range(0, n, _SLICE)):
        hi = min(n, lo + _SLICE)
        g = _gen(device, _seed_of(seed, "slice", i))
        t = torch.randn(hi - lo, generator=g, device=device, dtype=torch.float32)
        if std != 1.0:
            t.mul_(std)
        if mean != 0.0:
            t.add_(mean)
        flat[lo:hi].copy_(t)
    return out


def make_model(shape: ModelShape, seed: int, device="cpu", lm_boost_rows: Optional[torch.Tensor] = None,
               lm_boost: float = 1.0) -> dict:
    """Random-init weights in the layout the C ABI takes (row-major [out, in])."""
    dt = shape.torch_dtype
    D, F, V = shape.hidden, shape.ffn, shape.vocab
    jobs = {
        "embed": ((V, D), 1.0, 0.0, -1),
        "final_norm": ((D,), 0.1, 1.0, -1),
        "lm_head": ((V, D), 0.02, 0.0, -1),
    }
    for l in range(shape.n_layers):
        jobs[f"wqkv.{l}"] = ((shape.qkv_dim, D), 0.02, 0.0, l)
        jobs[f"wo.{l}"] = ((D, shape.n_q_heads * shape.head_dim), 0.02, 0.0, l)
        jobs[f"wgate.{l}"] = ((F, D), 0.02, 0.0, l)
        jobs[f"wup.{l}"] = ((F, D), 0.02, 0.0, l)
        jobs[f"wdown.{l}"] = ((D, F), 0.02, 0.0, l)
        jobs[f"attn_norm.{l}"] = ((D,), 0.1, 1.0, l)
        jobs[f"mlp_norm.{l}"] = ((D,), 0.1, 1.0, l)

    def run(item):
        name, (shp, std, mean, layer) = item
        key = name.split(".")[0]
        return name, _normal(shp, std, mean, _seed_of(seed, key, layer), device, dt)

    if str(device) == "cpu":
        with ThreadPoolExecutor(max_workers=8) as ex:
            made = dict(ex.map(run, jobs.items()))
    else:
        made = dict(map(run, jobs.items()))
    if lm_boost_rows is not None:
        rows = lm_boost_rows.to(made["lm_head"].device)
        made["lm_head"][rows] = (made["lm_head"][rows].float() * lm_boost).to(dt)
    out = {k: made[k] for k in ("embed", "final_norm", "lm_head")}
    for key in ("wqkv", "wo", "wgate", "wup", "wdown", "attn_norm", "mlp_norm"):
        out[key] = [made[f"{key}.{l}"] for l in range(shape.n_layers)]
    return out


def _prefix_lengths(work: Workload, g: torch.Generator) -> torch.Tensor:
    N = work.n_requests
    kind = work.prefix[0]
    if kind == "fixed":
        return torch.full((N,), int(work.prefix[1]), dtype=torch.int32)
    if kind == "uniform":
        lo, hi = work.prefix[1], work.prefix[2]
        return torch.randint(lo, hi + 1, (N,), generator=g, dtype=torch.int64).to(torch.int32)
    if kind == "lognormal":
        median, sigma, lo, hi = work.prefix[1:]
        z = torch.randn((N,), generator=g, dtype=torch.float64)
        p = torch.exp(math.log(median) + sigma * z).round().clamp(lo, hi)
        return p.to(torch.int32)
    raise ValueError(kind)


def _masks(work: Workload, g: torch.Generator) -> torch.Tensor:
    N, B = work.n_requests, work.block
    mask = torch.zeros((N, B), dtype=torch.uint8)
    for b in range(N):
        if work.masked[0] == "count":
            n = int(work.masked[1])
        else:
            lo, hi = work.masked[1], work.masked[2]
            u = lo + (hi - lo) * torch.rand((), generator=g, dtype=torch.float64).item()
            n = int(round(u * B))
        perm = torch.randperm(B, generator=g)
        mask[b, perm[:n]] = 1
    return mask


def make_batch(shape: ModelShape, work: Workload, seed: int, device="cpu",
               prefix_len: Optional[torch.Tensor] = None, mask: Optional[torch.Tensor] = None) -> dict:
    """Ragged batch: block tokens, mask state, prefix lengths, page tables, KV pool, intra-block KV cache."""
    g = _gen("cpu", _seed_of(seed, "batch-structure"))
    N, B, S = work.n_requests, work.block, work.page_size
    P = _prefix_lengths(work, g) if prefix_len is None else prefix_len.to(torch.int32).clone()
    m = _masks(work, g) if mask is None else mask.to(torch.uint8).clone()
    V = shape.vocab
    tokens = torch.randint(0, V - 1, (N, B), generator=g, dtype=torch.int64).to(torch.int32)
    tokens[m.bool()] = V - 1
    pages_per = [(int(p) + S - 1) // S for p in P]
    max_pages = max(1, max(pages_per))
    n_pages = sum(pages_per) + work.spare_pages
    perm = torch.randperm(n_pages, generator=g).to(torch.int32)
    table = torch.full((N, max_pages), -1, dtype=torch.int32)
    at = 0
    for b in range(N):
        table[b, :pages_per[b]] = perm[at:at + pages_per[b]]
        at += pages_per[b]
    dt = shape.torch_dtype
    L, H, d = shape.n_layers, shape.n_kv_heads, shape.head_dim
    kv_pool = _normal((n_pages, L, 2, H, S, d), 1.0, 0.0, _seed_of(seed, "kv_pool"), device, dt)
    ibc = _normal((N, L, 2, H, B, d), 1.0, 0.0, _seed_of(seed, "ibc"), device, dt)
    dev = torch.device(device)
    return {
        "block_tokens": tokens.to(dev), "mask": m.to(dev), "prefix_len": P.to(dev),
        "page_table": table.to(dev), "kv_pool": kv_pool, "ibc": ibc,
    }


def with_block_pages(batch: dict, block: int) -> dict:
    """A copy of `batch` whose page tables also cover positions P_b .. P_b + block - 1 of every request
    (the block about to be committed to the prefix): the last prefix page is shared, further pages are
    appended to the pool (zero-filled) in request order.  Input preparation only: no step arithmetic."""
    pool, table, plen = batch["kv_pool"], batch["page_table"].cpu(), batch["prefix_len"].cpu()
    S = int(pool.shape[4])
    N = int(table.shape[0])
    need = [(int(p) + block + S - 1) // S for p in plen]
    have = [(int(p) + S - 1) // S for p in plen]
    width = max(int(table.shape[1]), max(need))
    new_table = torch.full((N, width), -1, dtype=torch.int32)
    new_table[:, : table.shape[1]] = table
    n_old = int(pool.shape[0])
    at = n_old
    for b in range(N):
        for i in range(have[b], need[b]):
            new_table[b, i] = at
            at += 1
    extra = torch.zeros((at - n_old,) + tuple(pool.shape[1:]), dtype=pool.dtype, device=pool.device)
    out = dict(batch)
    out["kv_pool"] = torch.cat([pool, extra], 0)
    out["page_table"] = new_table.to(batch["page_table"].device)
    return out


def make_case(name: str = "tiny", seed: Optional[int] = None, device="cpu", *, shape: Optional[ModelShape] = None,
              work: Optional[Workload] = None, lm_boost_frac: float = 0.0, lm_boost: float = 50.0,
              **work_overrides) -> Case:
    """Build a seeded case by name, or from an explicit (shape, work)."""
    if shape is None or work is None:
        sname, wname = CASES[name]
        shape = shape or MODEL_SHAPES[sname]
        work = work or WORKLOADS[wname]
    if work_overrides:
        work = dataclasses.replace(work, **work_overrides)
    if seed is None:
        seed = SEEDS.get(name, 1234)
    boost_rows = None
    if lm_boost_frac > 0:
        g = _gen("cpu", _seed_of(seed, "lm-boost-rows"))
        n = max(1, int(lm_boost_frac * shape.vocab))
        boost_rows = torch.randperm(shape.vocab - 1, generator=g)[:n]
    model = make_model(shape, seed, device, boost_rows, lm_boost)
    batch = make_batch(shape, work, seed, device)
    return Case(shape, work, model, batch, seed)
