"""Plain float64 CPU oracle of one FOCUS focused denoising step (test infrastructure only).

Source: "FOCUS: DLLMs Know How to Tame Their Compute Bound" (Liang, Tan, Zhong,
Xu, Canini), the authors' project page and the arXiv abstract, plus a news
article on the same paper ("FOCUS: novo sistema aumenta throughput de Diffusion
LLMs ...").  What the pages fix:

  * project page, Overview -- Motivation: block-diffusion decoding runs a full
    token block per denoising step on top of an exactly cached prefix;
  * project page, Overview -- Design: importance is estimated after the early
    Q/K projections; likely-decodable positions are kept under an adaptive
    budget and the rest leave the later layers;
  * project page, Overview -- Decodability Signal: the signal is the layer-0-to-1
    importance delta;
  * project page, Overview -- Runtime Action: dynamic budgeting, token eviction,
    ragged execution and intra-block KV caching;
  * news article, "Arquitetura do FOCUS": importance scoring (training-free,
    early layers), target token selection, state compaction, ragged paged
    attention;
  * project page, Quality table: decoding uses a confidence threshold
    ("Conf." 0.7 / 0.8 / 0.9).

The pages print no formula.  The readings taken where they are silent:

  * importance I_l[j] of block position j at layer l = sum over all query heads
    h and all block query rows i of softmax_i(q_i K^T / sqrt(d))[P + j], the
    softmax running over the P prefix keys and the B block keys;
  * delta = I_1 - I_0;  c = #{masked j : delta_j > tau};
    k = min(clamp(ceil(alpha * c), k_min, k_max), #masked), the product and
    ceil taken in float32 as the kernel does;
  * the kept positions are the first k masked positions under the key
    (delta descending, j ascending), listed in ascending j;
  * a forced keep fraction f >= 0 keeps ceil(f * B) of all B positions under the
    key (masked first, delta descending, j ascending) -- f = 1 is the dense step;
  * layers 2..L-1 run only on kept rows; a kept row's fresh K/V overwrite the
    intra-block KV cache before attention, and every query attends to the
    prefix keys plus all B cache entries of its layer; layers 0 and 1 refresh
    the cache for all B positions;
  * confidence = max softmax of the logits, top id = lowest id among the maxima;
    a kept masked position decodes when conf > theta; if none does and the
    request kept any masked position, the kept masked position with the highest
    confidence (lowest j on ties) decodes;
  * the model layer is a standard pre-norm decoder layer: RMSNorm, grouped-query
    attention with rotate-half RoPE at absolute position P + j, residual,
    RMSNorm, SwiGLU MLP, residual; a final RMSNorm feeds an untied LM head;
  * around the step (decode_block, commit_block): a block starts with a dense
    step, focused steps follow until no position is masked, the decoded block is
    run densely once more, and its K/V then join the prefix pages at positions
    P .. P + B - 1 (project page, Overview -- Motivation: the prefix is cached
    exactly).

Parity pins: tests/test_oracle_*.py (closed forms, invariants, brute force,
an independent dense forward).  Method quality -- whether the delta predicts
decodability -- is parity unpinned: it needs trained weights and datasets.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np

try:  # torch is only used to read bf16 tensors into float64
    import torch
except ImportError:  # pragma: no cover
    torch = None


def _f64(t) -> np.ndarray:
    if torch is not None and isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def _i64(t) -> np.ndarray:
    if torch is not None and isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.int64).numpy()
    return np.asarray(t, dtype=np.int64)


# --------------------------------------------------------------------------
# model pieces (the standard decoder layer the pages' models use)
# --------------------------------------------------------------------------

def rms_norm(x: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * gamma."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * gamma


def rope(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half rotary embedding of the last axis (pairs (i, i + d/2)).

    Pair i turns by angle pos * theta^(-2i/d).  x: [..., n, d], pos: [n].
    """
    d = x.shape[-1]
    half = d // 2
    inv_freq = theta ** (-(2.0 * np.arange(half, dtype=np.float64)) / d)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * inv_freq[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def _keep(x: np.ndarray) -> np.ndarray:
    return x


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round to the nearest bfloat16 (ties to even), returned as float64."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64)).to(torch.bfloat16).to(torch.float64).numpy()


STORAGE = {"f64": _keep, "bf16": round_bf16}


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray):
    """Grouped-query softmax attention, no mask (block diffusion attends bidirectionally).

    q: [Hq, n, d]; k, v: [Hkv, T, d]; query head h reads KV head h // (Hq / Hkv).
    Returns (o [Hq, n, d], p [Hq, n, T]) with p the softmax probabilities.
    """
    hq, n, d = q.shape
    hkv = k.shape[0]
    group = hq // hkv
    o = np.empty((hq, n, v.shape[-1]))
    p_all = np.empty((hq, n, k.shape[1]))
    for h in range(hq):
        g = h // group
        s = (q[h] @ k[g].T) / math.sqrt(d)
        s = s - s.max(axis=1, keepdims=True)
        e = np.exp(s)
        p = e / e.sum(axis=1, keepdims=True)
        o[h] = p @ v[g]
        p_all[h] = p
    return o, p_all


def importance_from_probs(p: np.ndarray, prefix_len: int) -> np.ndarray:
    """Column sum of the attention probabilities over heads and query rows, block columns only.

    Project page, Overview -- Design / Decodability Signal: importance taken from
    the early layers' Q/K attention.  p: [Hq, n_queries, P + B] -> [B].
    """
    return p[:, :, prefix_len:].sum(axis=(0, 1))


def gather_prefix(kv_pool: np.ndarray, page_row: np.ndarray, prefix_len: int, layer: int, page_size: int):
    """Read a request's prefix K, V for one layer out of its pages -> ([Hkv, P, d], [Hkv, P, d])."""
    n_pages = (prefix_len + page_size - 1) // page_size
    hkv, d = kv_pool.shape[3], kv_pool.shape[5]
    if n_pages == 0:
        z = np.zeros((hkv, 0, d))
        return z, z.copy()
    pages = [int(page_row[i]) for i in range(n_pages)]
    kk = np.concatenate([_f64(kv_pool[pg, layer, 0]) for pg in pages], axis=1)[:, :prefix_len]
    vv = np.concatenate([_f64(kv_pool[pg, layer, 1]) for pg in pages], axis=1)[:, :prefix_len]
    return kk, vv


def layer_forward(x, lw, shape, positions, rows, prefix_k, prefix_v, cache_k, cache_v, store=_keep):
    """One pre-norm decoder layer on the rows `rows` (ascending block positions) of one request.

    cache_k / cache_v ([Hkv, B, d], float64) are the intra-block KV cache of this
    layer; the rows' fresh K/V overwrite it first (project page, Overview --
    Runtime Action: intra-block KV caching), then every row attends to the
    prefix keys plus all B cache entries.  Returns (x_out, attention probs).

    `store` is applied to every activation a kernel keeps in its storage type
    (normalised rows, q / k / v, attention output, MLP activation): the identity
    for plain float64, or bf16 rounding to take decisions in the kernel's
    precision.  Sums and the residual stream stay float64 either way.
    """
    hq, hkv, d = shape.n_q_heads, shape.n_kv_heads, shape.head_dim
    n = x.shape[0]
    h = store(rms_norm(x, lw["attn_norm"], shape.rms_eps))
    qkv = h @ lw["wqkv"].T
    q = qkv[:, : hq * d].reshape(n, hq, d).transpose(1, 0, 2)
    k = qkv[:, hq * d:(hq + hkv) * d].reshape(n, hkv, d).transpose(1, 0, 2)
    v = qkv[:, (hq + hkv) * d:].reshape(n, hkv, d).transpose(1, 0, 2)
    pos = positions[rows]
    q = store(rope(q, pos, shape.rope_theta))
    k = store(rope(k, pos, shape.rope_theta))
    cache_k[:, rows] = k
    cache_v[:, rows] = store(v)
    keys = np.concatenate([prefix_k, cache_k], axis=1)
    vals = np.concatenate([prefix_v, cache_v], axis=1)
    o, p = attention(q, keys, vals)
    x = x + store(o).transpose(1, 0, 2).reshape(n, hq * d) @ lw["wo"].T
    h2 = store(rms_norm(x, lw["mlp_norm"], shape.rms_eps))
    a = store(silu(h2 @ lw["wgate"].T) * (h2 @ lw["wup"].T))
    x = x + a @ lw["wdown"].T
    return x, p


# --------------------------------------------------------------------------
# budget, selection, compaction, LM head, decode
# --------------------------------------------------------------------------

def _ceil_f32(a: float, c: float) -> int:
    """ceil(a * c) evaluated in float32, as the kernel evaluates it."""
    return int(np.ceil(np.float32(np.float32(a) * np.float32(c))))


def select_positions(delta: np.ndarray, masked: np.ndarray, *, tau: float, k_min: int, k_max: int,
                     alpha: float = 1.0, forced_keep_frac: float = -1.0):
    """Adaptive budget + top-k with index tie-break for one request.

    Project page, Overview -- Design ("keeps likely decodable candidates under an
    adaptive budget") and Runtime Action ("dynamic budgeting, token eviction");
    news article, "Target Token Selection".  Returns (kept positions ascending,
    cut gap, tau gap) -- the two gaps say how far the decision is from flipping.
    """
    B = delta.shape[0]
    masked = np.asarray(masked).astype(bool)
    tau32 = float(np.float32(tau))
    if forced_keep_frac >= 0:
        k = min(B, _ceil_f32(forced_keep_frac, B))
        order = sorted(range(B), key=lambda j: (0 if masked[j] else 1, -delta[j], j))
        tau_gap = math.inf
        groups = [0 if masked[j] else 1 for j in order]
    else:
        eligible = [j for j in range(B) if masked[j]]
        c = sum(1 for j in eligible if delta[j] > tau32)
        k = min(max(_ceil_f32(alpha, c), k_min), k_max)
        k = min(k, len(eligible))
        order = sorted(eligible, key=lambda j: (-delta[j], j))
        tau_gap = min((abs(delta[j] - tau32) for j in eligible), default=math.inf)
        groups = [0] * len(order)
    if 0 < k < len(order) and groups[k - 1] == groups[k]:
        cut_gap = float(delta[order[k - 1]] - delta[order[k]])
    else:
        cut_gap = math.inf
    return sorted(order[:k]), cut_gap, tau_gap


def compact_rows(kept: Sequence[Sequence[int]], max_keep: int):
    """Ragged row map of the kept rows: requests in order, positions ascending.

    News article, "State Compaction"; project page, Runtime Action ("ragged
    execution").  Returns keep_count [N], retained_idx [N, max_keep] (-1 padded),
    row_offsets [N+1] (exclusive scan), row_map [R, 2] = (request, position).
    """
    n = len(kept)
    keep_count = np.array([len(s) for s in kept], dtype=np.int64)
    retained = np.full((n, max_keep), -1, dtype=np.int64)
    offsets = np.zeros(n + 1, dtype=np.int64)
    rows = []
    for b, s in enumerate(kept):
        retained[b, : len(s)] = s
        offsets[b + 1] = offsets[b] + len(s)
        rows.extend((b, j) for j in s)
    row_map = np.array(rows, dtype=np.int64).reshape(-1, 2)
    return keep_count, retained, offsets, row_map


def lm_head_conf(x: np.ndarray, final_norm: np.ndarray, lm_head: np.ndarray, eps: float, store=_keep):
    """Final RMSNorm, logits, max-softmax confidence and top id (lowest id among equal maxima).

    Project page, Quality table: decoding is gated by a confidence ("Conf.").
    Returns (conf, top_id, log_conf, top-1 logit margin) per row.
    """
    h = store(rms_norm(x, final_norm, eps))
    z = h @ lm_head.T
    top = np.argmax(z, axis=1)               # first maximum = lowest id
    zmax = z[np.arange(z.shape[0]), top]
    sumexp = np.exp(z - zmax[:, None]).sum(axis=1)
    conf = 1.0 / sumexp
    log_conf = -np.log(sumexp)
    if z.shape[1] > 1:
        part = np.partition(z, -2, axis=1)
        margin = part[:, -1] - part[:, -2]
    else:
        margin = np.full(z.shape[0], math.inf)
    return conf, top, log_conf, margin


def threshold_decode(kept: Sequence[int], masked: np.ndarray, conf: np.ndarray, top_id: np.ndarray,
                     threshold: float):
    """Which kept positions decode this step, and to which ids.

    A kept masked position decodes when conf > threshold (strict); if none does
    but some kept position is masked, the one with the highest conf decodes
    (lowest position on ties), so every step makes progress.
    Returns (dict position -> id, decision gaps for tolerance-aware checks).
    """
    thr = float(np.float32(threshold))
    cand = [t for t, j in enumerate(kept) if masked[j]]
    dec = [t for t in cand if conf[t] > thr]
    thr_gap = min((abs(conf[t] - thr) for t in cand), default=math.inf)
    fallback_gap = math.inf
    if not dec and cand:
        best = max(cand, key=lambda t: (conf[t], -kept[t]))
        dec = [best]
        others = [conf[t] for t in cand if t != best]
        if others:
            fallback_gap = float(np.log(conf[best]) - np.log(max(others)))
    return {int(kept[t]): int(top_id[t]) for t in dec}, thr_gap, fallback_gap


# --------------------------------------------------------------------------
# the step
# --------------------------------------------------------------------------

@dataclasses.dataclass
class OracleResult:
    importance: np.ndarray       # [2, N, B]
    delta: np.ndarray            # [N, B]
    keep_count: np.ndarray       # [N]
    retained_idx: np.ndarray     # [N, max_keep], ascending, -1 padded
    row_offsets: np.ndarray      # [N + 1]
    row_map: np.ndarray          # [R, 2]
    hidden: np.ndarray           # [R, D] residual stream after the last layer
    conf: np.ndarray             # [N, max_keep] (0 where unused)
    top_id: np.ndarray           # [N, max_keep] (-1 where unused)
    decoded_ids: np.ndarray      # [N, B], -1 where nothing decoded
    block_tokens: np.ndarray     # [N, B] after decoding
    mask: np.ndarray             # [N, B] after decoding
    ibc: np.ndarray              # [N, L, 2, Hkv, B, d] after the step
    cut_gap: np.ndarray          # [N] delta gap at the top-k cut
    tau_gap: np.ndarray          # [N] min |delta - tau| over eligible positions
    log_conf: np.ndarray         # [N, max_keep]
    logit_margin: np.ndarray     # [N, max_keep] top-1 minus top-2 logit
    thr_gap: np.ndarray          # [N] min |conf - threshold| over kept masked rows
    fallback_gap: np.ndarray     # [N] log-conf gap of the fallback choice


def focus_step(shape, model: dict, batch: dict, *, tau: float, k_min: int, k_max: int, conf_threshold: float,
               alpha: float = 1.0, forced_keep_frac: float = -1.0, max_keep: Optional[int] = None,
               forced_keep: Optional[Sequence[Sequence[int]]] = None, requests: Optional[Sequence[int]] = None,
               page_size: Optional[int] = None, storage: str = "f64") -> OracleResult:
    """One focused denoising step over a batch of ragged requests.

    shape: model shape (n_layers, hidden, n_q_heads, n_kv_heads, head_dim, ffn,
    vocab, rms_eps, rope_theta); model / batch: tensors in the C ABI's layout.
    `forced_keep` replaces the selection (per request, any order) -- used to
    compare the later layers on a set chosen elsewhere.  `requests` restricts
    the step to a subset of the batch (requests are independent).  `storage`
    "bf16" rounds activations where a bf16 kernel stores them (see
    layer_forward), so that decisions are taken in the kernel's precision.
    """
    store = STORAGE[storage]
    tokens = _i64(batch["block_tokens"])
    mask = _i64(batch["mask"]).astype(bool)
    prefix_len = _i64(batch["prefix_len"])
    table = _i64(batch["page_table"])
    kv_pool = batch["kv_pool"]
    if requests is not None:
        req = list(requests)
        tokens, mask, prefix_len, table = tokens[req], mask[req], prefix_len[req], table[req]
        ibc = _f64(batch["ibc"][req]).copy()
        if forced_keep is not None:
            forced_keep = [forced_keep[b] for b in req]
    else:
        ibc = _f64(batch["ibc"]).copy()
    N, B = tokens.shape
    L = shape.n_layers
    if L < 2:
        raise ValueError("the importance delta needs at least two layers")
    S = page_size if page_size is not None else int(kv_pool.shape[4])
    if max_keep is None:
        max_keep = B if forced_keep_frac >= 0 else k_max
    embed = model["embed"]

    def layer_weights(l):
        return {key: _f64(model[key][l]) for key in
                ("wqkv", "wo", "wgate", "wup", "wdown", "attn_norm", "mlp_norm")}

    positions = [int(prefix_len[b]) + np.arange(B) for b in range(N)]
    x = [_f64(embed[tokens[b]]) for b in range(N)]
    all_rows = np.arange(B)

    # layers 0 and 1 on the full block, importance at both
    importance = np.zeros((2, N, B))
    for l in (0, 1):
        lw = layer_weights(l)
        for b in range(N):
            pk, pv = gather_prefix(kv_pool, table[b], int(prefix_len[b]), l, S)
            x[b], p = layer_forward(x[b], lw, shape, positions[b], all_rows, pk, pv, ibc[b, l, 0], ibc[b, l, 1],
                                    store)
            importance[l, b] = importance_from_probs(p, int(prefix_len[b]))
    delta = importance[1] - importance[0]

    # budget + selection
    kept, cut_gap, tau_gap = [], np.full(N, math.inf), np.full(N, math.inf)
    for b in range(N):
        if forced_keep is not None:
            kept.append(sorted(int(j) for j in forced_keep[b]))
            continue
        s, cg, tg = select_positions(delta[b], mask[b], tau=tau, k_min=k_min, k_max=k_max, alpha=alpha,
                                     forced_keep_frac=forced_keep_frac)
        kept.append(s)
        cut_gap[b], tau_gap[b] = cg, tg
    if any(len(s) > max_keep for s in kept):
        raise ValueError("kept more positions than max_keep")
    keep_count, retained, offsets, row_map = compact_rows(kept, max_keep)

    # later layers on the kept rows only
    xc = [x[b][np.asarray(kept[b], dtype=np.int64)] for b in range(N)]
    for l in range(2, L):
        lw = layer_weights(l)
        for b in range(N):
            if not kept[b]:
                continue
            pk, pv = gather_prefix(kv_pool, table[b], int(prefix_len[b]), l, S)
            xc[b], _ = layer_forward(xc[b], lw, shape, positions[b], np.asarray(kept[b]), pk, pv,
                                     ibc[b, l, 0], ibc[b, l, 1], store)

    # LM head, confidence, decode
    final_norm, lm_head = _f64(model["final_norm"]), _f64(model["lm_head"])
    conf = np.zeros((N, max_keep))
    top_id = np.full((N, max_keep), -1, dtype=np.int64)
    log_conf = np.full((N, max_keep), -math.inf)
    margin = np.full((N, max_keep), math.inf)
    decoded = np.full((N, B), -1, dtype=np.int64)
    thr_gap, fb_gap = np.full(N, math.inf), np.full(N, math.inf)
    new_tokens, new_mask = tokens.copy(), mask.copy()
    for b in range(N):
        k = len(kept[b])
        if k == 0:
            continue
        c, t, lc, mg = lm_head_conf(xc[b], final_norm, lm_head, shape.rms_eps, store)
        conf[b, :k], top_id[b, :k], log_conf[b, :k], margin[b, :k] = c, t, lc, mg
        dec, thr_gap[b], fb_gap[b] = threshold_decode(kept[b], mask[b], c, t, conf_threshold)
        for j, tok in dec.items():
            decoded[b, j] = tok
            new_tokens[b, j] = tok
            new_mask[b, j] = False
    hidden = np.concatenate(xc, axis=0) if xc else np.zeros((0, shape.hidden))
    return OracleResult(importance, delta, keep_count, retained, offsets, row_map, hidden, conf, top_id, decoded,
                        new_tokens, new_mask.astype(np.uint8), ibc, cut_gap, tau_gap, log_conf, margin,
                        thr_gap, fb_gap)


# --------------------------------------------------------------------------
# around the step: one block to completion, then its K/V into the prefix
# --------------------------------------------------------------------------

def commit_block(kv_pool, ibc, prefix_len, page_table):
    """Write every request's block K/V into its prefix pages at positions P_b .. P_b + B - 1 and grow the
    prefix by B.

    Project page, Overview -- Motivation: the prefix is served from an exactly cached KV; a block that
    has been decoded becomes part of that prefix.  `ibc` is the intra-block cache [N, L, 2, Hkv, B, d]
    after the block's final refresh; the pages hold [pages, L, 2, Hkv, S, d].  Returns (pool, prefix_len)
    as new float64 / int64 arrays."""
    pool = _f64(kv_pool).copy()
    cache = _f64(ibc)
    plen = _i64(prefix_len).copy()
    table = _i64(page_table)
    S = pool.shape[4]
    N, B = cache.shape[0], cache.shape[4]
    for b in range(N):
        for j in range(B):
            pos = int(plen[b]) + j
            page = int(table[b, pos // S])
            pool[page, :, :, :, pos % S, :] = cache[b, :, :, :, j, :]
    return pool, plen + B


@dataclasses.dataclass
class BlockResult:
    steps: list                  # OracleResult of every decoding step (the first one dense)
    block_tokens: np.ndarray     # [N, B] the decoded block
    ibc: np.ndarray              # [N, L, 2, Hkv, B, d] after the final dense refresh
    kv_pool: np.ndarray          # pages after the commit
    prefix_len: np.ndarray       # [N] grown by B


def decode_block(shape, model: dict, batch: dict, *, tau: float, k_min: int, k_max: int, conf_threshold: float,
                 alpha: float = 1.0, max_steps: Optional[int] = None, storage: str = "f64") -> BlockResult:
    """Denoise one block to completion and commit it.

    Project page, Overview -- Motivation / Runtime Action: a block is decoded over several denoising
    steps, each computing the block on top of the cached prefix; FOCUS runs the later layers only on the
    kept positions, whose fresh K/V refresh the intra-block cache while evicted positions keep theirs.
    Readings: the block's first step is dense (every position computed, which fills the intra-block
    cache); then focused steps run until no position is masked (the decode rule's fallback decodes at
    least one masked position of every request that has one, so at most B steps); the fully decoded
    block is computed once more densely so that its cache holds the K/V of the final tokens, and that
    cache is committed to the prefix pages."""
    B = int(_i64(batch["block_tokens"]).shape[1])
    max_steps = B if max_steps is None else max_steps
    state = {k: v for k, v in batch.items()}
    steps = []

    def run(frac):
        r = focus_step(shape, model, state, tau=tau, k_min=k_min, k_max=k_max, conf_threshold=conf_threshold,
                       alpha=alpha, forced_keep_frac=frac, max_keep=B, storage=storage)
        state["block_tokens"], state["mask"], state["ibc"] = r.block_tokens, r.mask, r.ibc
        return r

    steps.append(run(1.0))
    while np.asarray(state["mask"]).any() and len(steps) < max_steps:
        steps.append(run(-1.0))
    if np.asarray(state["mask"]).any():
        raise ValueError("block not decoded within max_steps")
    refresh = run(1.0)
    pool, plen = commit_block(state["kv_pool"], refresh.ibc, state["prefix_len"], state["page_table"])
    return BlockResult(steps, np.asarray(state["block_tokens"]), refresh.ibc, pool, plen)
