"""Plants plausible mistakes in the oracle (CPU only) and checks that the pins catch each one.

Each mutation swaps one oracle function for a copy with one deliberate slip (a
dropped term, a wrong sign, index or tie-break, operations in the wrong order);
at least one pin of tests/test_oracle_pins.py must then fail.
"""
import math

import numpy as np
import pytest

from oracle import focus_oracle as fo
import test_oracle_pins as pins


def _rope_sign(x, pos, theta):
    d = x.shape[-1]
    half = d // 2
    ang = np.asarray(pos, dtype=np.float64)[:, None] * (theta ** (-(2.0 * np.arange(half)) / d))[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c + x2 * s, x2 * c - x1 * s], axis=-1)          # slip: turns the other way


def _rope_interleaved(x, pos, theta):
    d = x.shape[-1]
    ang = np.asarray(pos, dtype=np.float64)[:, None] * (theta ** (-(2.0 * np.arange(d // 2)) / d))[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., 0::2], x[..., 1::2]                                          # slip: pairs (2i, 2i+1)
    out = np.empty_like(x)
    out[..., 0::2], out[..., 1::2] = x1 * c - x2 * s, x2 * c + x1 * s
    return out


def _attention_variant(scale_by_sqrt_d=True, group_of=lambda h, hq, hkv: h // (hq // hkv)):
    def attn(q, k, v):
        hq, hkv = q.shape[0], k.shape[0]
        o = np.empty((hq, q.shape[1], v.shape[-1]))
        p_all = np.empty((hq, q.shape[1], k.shape[1]))
        for h in range(hq):
            g = group_of(h, hq, hkv)
            s = q[h] @ k[g].T / (math.sqrt(q.shape[-1]) if scale_by_sqrt_d else 1.0)
            e = np.exp(s - s.max(1, keepdims=True))
            p = e / e.sum(1, keepdims=True)
            o[h], p_all[h] = p @ v[g], p
        return o, p_all
    return attn


def _importance_leading_columns(p, prefix_len):
    return p[:, :, : p.shape[2] - prefix_len].sum(axis=(0, 1))                  # slip: wrong column range


def _rms_no_gamma(x, gamma, eps):
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)             # slip: gamma dropped


def _select_high_index_on_ties(delta, masked, *, tau, k_min, k_max, alpha=1.0, forced_keep_frac=-1.0):
    masked = np.asarray(masked).astype(bool)
    eligible = [j for j in range(len(delta)) if masked[j]]
    c = sum(1 for j in eligible if delta[j] > np.float32(tau))
    k = min(min(max(math.ceil(alpha * c), k_min), k_max), len(eligible))
    if forced_keep_frac >= 0:
        return _orig["select_positions"](delta, masked, tau=tau, k_min=k_min, k_max=k_max, alpha=alpha,
                                         forced_keep_frac=forced_keep_frac)
    order = sorted(eligible, key=lambda j: (-delta[j], -j))                       # slip: higher j wins ties
    return sorted(order[:k]), math.inf, math.inf


def _layer_variant(write_cache_first=True, mlp_residual=True):
    def layer(x, lw, shape, positions, rows, prefix_k, prefix_v, cache_k, cache_v, store=fo._keep):
        hq, hkv, d = shape.n_q_heads, shape.n_kv_heads, shape.head_dim
        n = x.shape[0]
        h = fo.rms_norm(x, lw["attn_norm"], shape.rms_eps)
        qkv = h @ lw["wqkv"].T
        q = qkv[:, : hq * d].reshape(n, hq, d).transpose(1, 0, 2)
        k = qkv[:, hq * d:(hq + hkv) * d].reshape(n, hkv, d).transpose(1, 0, 2)
        v = qkv[:, (hq + hkv) * d:].reshape(n, hkv, d).transpose(1, 0, 2)
        pos = positions[rows]
        q, k = fo.rope(q, pos, shape.rope_theta), fo.rope(k, pos, shape.rope_theta)
        if write_cache_first:
            cache_k[:, rows], cache_v[:, rows] = k, v
        keys = np.concatenate([prefix_k, cache_k], axis=1)
        vals = np.concatenate([prefix_v, cache_v], axis=1)
        o, p = fo.attention(q, keys, vals)
        if not write_cache_first:                                                 # slip: stale cache read
            cache_k[:, rows], cache_v[:, rows] = k, v
        x = x + o.transpose(1, 0, 2).reshape(n, hq * d) @ lw["wo"].T
        h2 = fo.rms_norm(x, lw["mlp_norm"], shape.rms_eps)
        a = fo.silu(h2 @ lw["wgate"].T) * (h2 @ lw["wup"].T)
        mlp = a @ lw["wdown"].T
        return (x + mlp if mlp_residual else mlp), p                              # slip: residual dropped
    return layer


def _storage_variant(round_residual=False, round_attention_output=True, round_q_after_rope=True):
    """The oracle's layer with one slip in where bf16 storage rounds (the float64 mode is unaffected)."""
    def layer(x, lw, shape, positions, rows, prefix_k, prefix_v, cache_k, cache_v, store=fo._keep):
        hq, hkv, d = shape.n_q_heads, shape.n_kv_heads, shape.head_dim
        n = x.shape[0]
        h = store(fo.rms_norm(x, lw["attn_norm"], shape.rms_eps))
        qkv = h @ lw["wqkv"].T
        q = qkv[:, : hq * d].reshape(n, hq, d).transpose(1, 0, 2)
        k = qkv[:, hq * d:(hq + hkv) * d].reshape(n, hkv, d).transpose(1, 0, 2)
        v = qkv[:, (hq + hkv) * d:].reshape(n, hkv, d).transpose(1, 0, 2)
        pos = positions[rows]
        if round_q_after_rope:
            q = store(fo.rope(q, pos, shape.rope_theta))
        else:
            q = fo.rope(store(q), pos, shape.rope_theta)                          # slip: rounds before RoPE
        k = store(fo.rope(k, pos, shape.rope_theta))
        cache_k[:, rows] = k
        cache_v[:, rows] = store(v)
        keys = np.concatenate([prefix_k, cache_k], axis=1)
        vals = np.concatenate([prefix_v, cache_v], axis=1)
        o, p = fo.attention(q, keys, vals)
        o = store(o) if round_attention_output else o                             # slip: output not rounded
        x = x + o.transpose(1, 0, 2).reshape(n, hq * d) @ lw["wo"].T
        if round_residual:
            x = store(x)                                                          # slip: residual rounded
        h2 = store(fo.rms_norm(x, lw["mlp_norm"], shape.rms_eps))
        a = store(fo.silu(h2 @ lw["wgate"].T) * (h2 @ lw["wup"].T))
        x = x + a @ lw["wdown"].T
        return (store(x) if round_residual else x), p
    return layer


def _lm_head_highest_id(x, g, w, eps, store=fo._keep):
    conf, top, lc, mg = _orig["lm_head_conf"](x, g, w, eps, store)
    z = fo.rms_norm(x, g, eps) @ w.T
    return conf, z.shape[1] - 1 - np.argmax(z[:, ::-1], axis=1), lc, mg          # slip: highest id on ties


def _decode_not_strict(kept, masked, conf, top_id, threshold):
    thr = float(np.float32(threshold))
    cand = [t for t, j in enumerate(kept) if masked[j]]
    dec = [t for t in cand if conf[t] >= thr]                                     # slip: >= instead of >
    if not dec and cand:
        dec = [max(cand, key=lambda t: (conf[t], -kept[t]))]
    return {int(kept[t]): int(top_id[t]) for t in dec}, math.inf, math.inf


def _select_variant(*, count_all=False, floor_budget=False, no_kmin=False, unmasked_first=False):
    def sel(delta, masked, *, tau, k_min, k_max, alpha=1.0, forced_keep_frac=-1.0):
        masked = np.asarray(masked).astype(bool)
        B = len(delta)
        tau32 = float(np.float32(tau))
        if forced_keep_frac >= 0:
            k = min(B, fo._ceil_f32(forced_keep_frac, B))
            first = (lambda j: 1 if masked[j] else 0) if unmasked_first else (lambda j: 0 if masked[j] else 1)
            order = sorted(range(B), key=lambda j: (first(j), -delta[j], j))    # slip (optional): key order
            return sorted(order[:k]), math.inf, math.inf
        eligible = [j for j in range(B) if masked[j]]
        pool = range(B) if count_all else eligible                                # slip (optional): count all
        c = sum(1 for j in pool if delta[j] > tau32)
        k = int(np.floor(np.float32(alpha) * np.float32(c))) if floor_budget else fo._ceil_f32(alpha, c)
        k = min(k if no_kmin else max(k, k_min), k_max)                           # slip (optional): no k_min
        k = min(k, len(eligible))
        order = sorted(eligible, key=lambda j: (-delta[j], j))
        return sorted(order[:k]), math.inf, math.inf
    return sel


def _importance_block_normalised(p, prefix_len):
    blk = p[:, :, prefix_len:]
    return (blk / blk.sum(axis=2, keepdims=True)).sum(axis=(0, 1))               # slip: softmax over block only


def _compact_descending(kept, max_keep):
    return _orig["compact_rows"]([sorted(s, reverse=True) for s in kept], max_keep)  # slip: order reversed


def _decode_fallback_any(kept, masked, conf, top_id, threshold):
    thr = float(np.float32(threshold))
    cand = [t for t, j in enumerate(kept) if masked[j]]
    dec = [t for t in cand if conf[t] > thr]
    if not dec and cand:
        dec = [max(range(len(kept)), key=lambda t: (conf[t], -kept[t]))]           # slip: fallback may pick unmasked
    return {int(kept[t]): int(top_id[t]) for t in dec}, math.inf, math.inf


def _decode_fallback_high_j(kept, masked, conf, top_id, threshold):
    thr = float(np.float32(threshold))
    cand = [t for t, j in enumerate(kept) if masked[j]]
    dec = [t for t in cand if conf[t] > thr]
    if not dec and cand:
        dec = [max(cand, key=lambda t: (conf[t], kept[t]))]                      # slip: higher j wins ties
    return {int(kept[t]): int(top_id[t]) for t in dec}, math.inf, math.inf


_orig = {n: getattr(fo, n) for n in ("select_positions", "lm_head_conf", "compact_rows")}

MUTATIONS = {
    "rope_sign": ("rope", _rope_sign),
    "rope_interleaved_pairs": ("rope", _rope_interleaved),
    "attention_without_sqrt_d": ("attention", _attention_variant(scale_by_sqrt_d=False)),
    "kv_group_modulo": ("attention", _attention_variant(group_of=lambda h, hq, hkv: h % hkv)),
    "importance_wrong_columns": ("importance_from_probs", _importance_leading_columns),
    "norm_drops_gamma": ("rms_norm", _rms_no_gamma),
    "select_high_index_on_ties": ("select_positions", _select_high_index_on_ties),
    "cache_written_after_attention": ("layer_forward", _layer_variant(write_cache_first=False)),
    "mlp_residual_dropped": ("layer_forward", _layer_variant(mlp_residual=False)),
    "argmax_highest_id": ("lm_head_conf", _lm_head_highest_id),
    "decode_threshold_not_strict": ("threshold_decode", _decode_not_strict),
    "budget_counts_unmasked_positions": ("select_positions", _select_variant(count_all=True)),
    "budget_floor_instead_of_ceil": ("select_positions", _select_variant(floor_budget=True)),
    "budget_without_k_min": ("select_positions", _select_variant(no_kmin=True)),
    "forced_keep_unmasked_first": ("select_positions", _select_variant(unmasked_first=True)),
    "importance_softmax_over_block_only": ("importance_from_probs", _importance_block_normalised),
    "compaction_descending": ("compact_rows", _compact_descending),
    "fallback_may_pick_unmasked": ("threshold_decode", _decode_fallback_any),
    "fallback_higher_position_on_ties": ("threshold_decode", _decode_fallback_high_j),
    "bf16_storage_rounds_the_residual": ("layer_forward", _storage_variant(round_residual=True)),
    "bf16_storage_skips_the_attention_output": ("layer_forward", _storage_variant(round_attention_output=False)),
    "bf16_storage_rounds_q_before_rope": ("layer_forward", _storage_variant(round_q_after_rope=False)),
}

PINS = [getattr(pins, n) for n in sorted(dir(pins)) if n.startswith("test_") and n not in (
    "test_column_sums_total_heads_times_queries", "test_forced_full_keep_equals_dense_forward")]


def _run_pins():
    failed = []
    for fn in PINS:
        try:
            fn()
        except AssertionError:
            failed.append(fn.__name__)
    try:
        pins.test_forced_full_keep_equals_dense_forward("tiny")
    except AssertionError:
        failed.append("test_forced_full_keep_equals_dense_forward")
    return failed


@pytest.mark.parametrize("mutation", sorted(MUTATIONS))
def test_planted_mistake_is_caught(mutation, monkeypatch):
    attr, bad = MUTATIONS[mutation]
    monkeypatch.setattr(fo, attr, bad)
    assert _run_pins(), f"no pin caught the planted mistake {mutation}"
