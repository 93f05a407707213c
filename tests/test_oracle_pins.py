"""Pins of the CPU oracle against things other than itself.

Closed forms, invariants, library special cases, hand-worked fixtures
(tests/golden/), brute force on tiny inputs, an independently written dense
forward (tests/dense_reference.py) and a pure-Python scalar-loop step
(tests/scalar_bruteforce.py).  CPU only.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import focus_synth as fs
from oracle import focus_oracle as fo

from dense_reference import dense_block_forward
from scalar_bruteforce import scalar_step

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(7)


# ---------------------------------------------------------------- attention
def _rand_qkv(hq, hkv, n, t, d, scale=1.0):
    return (rng.normal(size=(hq, n, d)) * scale, rng.normal(size=(hkv, t, d)) * scale, rng.normal(size=(hkv, t, d)))


def test_softmax_rows_sum_to_one():
    q, k, v = _rand_qkv(4, 2, 5, 37, 16, 2.0)
    _, p = fo.attention(q, k, v)
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=0, atol=1e-13)
    assert (p > 0).all()


@pytest.mark.parametrize("hq,hkv,n,prefix,blk", [(4, 2, 16, 40, 16), (8, 8, 7, 0, 7), (6, 1, 3, 100, 3)])
def test_column_sums_total_heads_times_queries(hq, hkv, n, prefix, blk):
    """Summed over every key column (prefix and block), the column sums equal Hq * n."""
    q, k, v = _rand_qkv(hq, hkv, n, prefix + blk, 32, 1.5)
    _, p = fo.attention(q, k, v)
    total = p.sum(axis=(0, 1))
    assert abs(total.sum() - hq * n) < 1e-10 * hq * n
    # the block-column importance is the tail of these column sums
    np.testing.assert_allclose(fo.importance_from_probs(p, prefix), total[prefix:], rtol=0, atol=1e-13)


def test_importance_identical_keys_closed_form():
    """Identical keys: every probability is 1/(P+B), so each block column gets Hq*B/(P+B)."""
    hq, hkv, B, P, d = 6, 3, 8, 24, 16
    q = rng.normal(size=(hq, B, d))
    krow = rng.normal(size=d)
    k = np.broadcast_to(krow, (hkv, P + B, d)).copy()
    v = rng.normal(size=(hkv, P + B, d))
    _, p = fo.attention(q, k, v)
    np.testing.assert_allclose(fo.importance_from_probs(p, P), hq * B / (P + B), rtol=1e-13)


def test_attention_without_prefix_is_textbook_attention():
    """P = 0 and Hkv = Hq: plain multi-head softmax attention (torch SDPA, float64)."""
    q, k, v = _rand_qkv(4, 4, 9, 9, 16, 1.3)
    o, _ = fo.attention(q, k, v)
    ref = F.scaled_dot_product_attention(torch.from_numpy(q)[None], torch.from_numpy(k)[None],
                                         torch.from_numpy(v)[None])[0].numpy()
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-12)


def test_grouped_query_heads_read_their_kv_group():
    """GQA equals MHA with each KV head repeated for its consecutive group of query heads."""
    q, k, v = _rand_qkv(8, 2, 5, 21, 16, 1.0)
    o, _ = fo.attention(q, k, v)
    kr, vr = np.repeat(k, 4, axis=0), np.repeat(v, 4, axis=0)
    o2, _ = fo.attention(q, kr, vr)
    np.testing.assert_allclose(o, o2, rtol=1e-14, atol=1e-14)
    # and head 5 must read group 1, not group 5 % 2
    ref5 = F.scaled_dot_product_attention(torch.from_numpy(q[5:6])[None], torch.from_numpy(k[1:2])[None],
                                          torch.from_numpy(v[1:2])[None])[0].numpy()
    np.testing.assert_allclose(o[5:6], ref5, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- rope / norm / silu
def test_rope_is_a_relative_rotation():
    d = 32
    q, k = rng.normal(size=(1, 1, d)), rng.normal(size=(1, 1, d))
    pq, pk, shift = 37, 5, 1000
    s1 = (fo.rope(q, np.array([pq]), 1e4) * fo.rope(k, np.array([pk]), 1e4)).sum()
    s2 = (fo.rope(q, np.array([pq + shift]), 1e4) * fo.rope(k, np.array([pk + shift]), 1e4)).sum()
    assert abs(s1 - s2) < 1e-10
    # norm preserving, identity at position 0, composition of turns
    x = rng.normal(size=(2, 3, d))
    pos = np.array([3, 11, 250])
    np.testing.assert_allclose(np.linalg.norm(fo.rope(x, pos, 1e4), axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    np.testing.assert_allclose(fo.rope(x, np.zeros(3), 1e4), x, rtol=0, atol=0)
    np.testing.assert_allclose(fo.rope(fo.rope(x, pos, 1e4), pos + 7, 1e4), fo.rope(x, 2 * pos + 7, 1e4),
                               rtol=1e-10, atol=1e-10)


def test_rope_two_dims_is_planar_rotation_by_position():
    """d = 2: one pair with frequency 1, so position p turns (a, b) by p radians counter-clockwise."""
    a, b, p = 0.6, -1.7, 2.5
    out = fo.rope(np.array([[[a, b]]]), np.array([p]), 1e4)[0, 0]
    assert abs(out[0] - (a * math.cos(p) - b * math.sin(p))) < 1e-15
    assert abs(out[1] - (a * math.sin(p) + b * math.cos(p))) < 1e-15


def test_rms_norm_closed_forms():
    x = rng.normal(size=(5, 64)) * 3.0
    y = fo.rms_norm(x, np.ones(64), 0.0)
    np.testing.assert_allclose(np.sqrt((y * y).mean(-1)), 1.0, rtol=1e-13)
    np.testing.assert_allclose(fo.rms_norm(7.5 * x, np.ones(64), 0.0), y, rtol=1e-13)
    g = rng.normal(size=64)
    c = np.full((1, 64), -2.0)
    np.testing.assert_allclose(fo.rms_norm(c, g, 0.0)[0], -g, rtol=1e-14)


def test_silu_identities():
    x = rng.normal(size=100) * 4
    np.testing.assert_allclose(fo.silu(x) - fo.silu(-x), x, rtol=1e-12, atol=1e-12)
    assert fo.silu(np.array([0.0]))[0] == 0.0
    assert abs(fo.silu(np.array([40.0]))[0] - 40.0) < 1e-12


def test_bf16_storage_rounding_closed_forms():
    """bf16 keeps 8 significant bits: 1 + 2^-8 is a tie (to even: 1), just above it rounds up to 1 + 2^-7."""
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 2 ** -8 + 2 ** -20, 1.0 + 3 * 2 ** -8, -3.0 - 2 ** -7, 2.0 ** -130])
    want = np.array([1.0, 1.0, 1.0 + 2 ** -7, 1.0 + 2 ** -6, -3.0, 2.0 ** -130])
    np.testing.assert_array_equal(fo.round_bf16(x), want)
    y = rng.normal(size=1000) * 10
    r = fo.round_bf16(y)
    assert np.all(np.abs(r - y) <= np.abs(y) * 2.0 ** -8)        # half an ulp of an 8-bit significand
    np.testing.assert_array_equal(fo.round_bf16(r), r)             # idempotent


def test_bf16_storage_only_rounds_activations():
    """storage='f64' is the plain step; storage='bf16' moves hidden states by about the bf16 ulp."""
    case = fs.make_case("tiny")
    w = case.work
    kw = dict(tau=w.tau, k_min=w.k_min, k_max=w.k_max, conf_threshold=w.conf_threshold, forced_keep_frac=1.0)
    a = fo.focus_step(case.shape, case.model, case.batch, **kw)
    b = fo.focus_step(case.shape, case.model, case.batch, storage="f64", **kw)
    c = fo.focus_step(case.shape, case.model, case.batch, storage="bf16", **kw)
    np.testing.assert_array_equal(a.hidden, b.hidden)
    rel = np.abs(c.hidden - a.hidden).max() / np.sqrt(np.mean(a.hidden ** 2))
    assert 1e-5 < rel < 2e-2
    assert np.all(fo.round_bf16(c.ibc) == c.ibc)                   # the cache holds bf16 values


# ---------------------------------------------------------------- selection / compaction
def test_select_golden_cases():
    data = json.load(open(os.path.join(GOLDEN, "select_cases.json")))
    for c in data["cases"]:
        kept, _, _ = fo.select_positions(np.array(c["delta"]), np.array(c["mask"]), tau=c["tau"], k_min=c["k_min"],
                                         k_max=c["k_max"], alpha=c["alpha"], forced_keep_frac=c["f"])
        assert kept == c["keep"], c["name"]


def _brute_select(delta, masked, tau, k_min, k_max):
    elig = [j for j in range(len(delta)) if masked[j]]
    c = sum(1 for j in elig if delta[j] > tau)
    k = min(min(max(c, k_min), k_max), len(elig))
    # the unique size-k subset that beats every left-out eligible position under (delta desc, j asc)
    found = []
    for sub in itertools.combinations(elig, k):
        rest = [j for j in elig if j not in sub]
        if all((delta[a] > delta[r]) or (delta[a] == delta[r] and a < r) for a in sub for r in rest):
            found.append(list(sub))
    assert len(found) == 1
    return found[0]


def test_select_matches_brute_force_random():
    for _ in range(300):
        B = int(rng.integers(1, 10))
        delta = rng.integers(-3, 4, size=B) / 4.0          # many exact ties
        masked = rng.integers(0, 2, size=B)
        k_min, k_max = int(rng.integers(0, 4)), int(rng.integers(1, 8))
        kept, _, _ = fo.select_positions(delta, masked, tau=0.0, k_min=k_min, k_max=k_max)
        assert kept == _brute_select(delta, masked, 0.0, k_min, k_max)


def test_select_exhaustive_over_masks_b4():
    for bits in range(16):
        masked = np.array([(bits >> j) & 1 for j in range(4)])
        for delta in itertools.product([-0.5, 0.0, 0.5], repeat=4):
            delta = np.array(delta)
            for k_min, k_max in [(0, 4), (1, 2), (2, 3), (4, 4)]:
                kept, _, _ = fo.select_positions(delta, masked, tau=0.0, k_min=k_min, k_max=k_max)
                assert kept == _brute_select(delta, masked, 0.0, k_min, k_max)


def test_compaction_is_order_preserving_and_inverts_the_gather():
    kept = [[0, 3, 7], [], [2], [1, 5]]
    kc, ret, off, rmap = fo.compact_rows(kept, 4)
    assert kc.tolist() == [3, 0, 1, 2] and off.tolist() == [0, 3, 3, 4, 6]
    assert ret.tolist() == [[0, 3, 7, -1], [-1] * 4, [2, -1, -1, -1], [1, 5, -1, -1]]
    keys = [tuple(r) for r in rmap.tolist()]
    assert keys == sorted(keys) and len(set(keys)) == len(keys)
    # gather then scatter back restores every kept row
    full = rng.normal(size=(4, 8, 3))
    comp = np.stack([full[b, j] for b, j in keys])
    back = np.zeros_like(full)
    for r, (b, j) in enumerate(keys):
        back[b, j] = comp[r]
    for b, s in enumerate(kept):
        np.testing.assert_array_equal(back[b, s], full[b, s])


# ---------------------------------------------------------------- LM head / decode
def test_lm_head_conf_against_direct_softmax():
    base = rng.normal(size=32)
    x = base + 0.05 * rng.normal(size=(6, 32))
    g = np.abs(rng.normal(size=32)) + 0.5
    w = rng.normal(size=(50, 32)) * 0.3
    w[3] = w[7] = base * g / np.linalg.norm(base * g) * 4.0   # an exact tie at the top of every row
    conf, top, log_conf, margin = fo.lm_head_conf(x, g, w, 1e-6)
    z = fo.rms_norm(x, g, 1e-6) @ w.T
    direct = np.exp(z) / np.exp(z).sum(1, keepdims=True)     # no max shift: a different evaluation
    np.testing.assert_allclose(conf, direct.max(1), rtol=1e-12)
    np.testing.assert_allclose(log_conf, np.log(direct.max(1)), rtol=1e-12)
    for r in range(6):
        best = [i for i in range(50) if z[r, i] == z[r].max()]
        assert best == [3, 7] and top[r] == 3
        srt = np.sort(z[r])
        assert margin[r] == pytest.approx(srt[-1] - srt[-2], abs=1e-14)
    # and away from ties the margin is the top-1 minus top-2 gap
    conf2, top2, _, margin2 = fo.lm_head_conf(x, g, w[:7], 1e-6)
    z2 = fo.rms_norm(x, g, 1e-6) @ w[:7].T
    np.testing.assert_allclose(margin2, np.sort(z2, 1)[:, -1] - np.sort(z2, 1)[:, -2], rtol=1e-12)


def test_decode_golden_cases():
    data = json.load(open(os.path.join(GOLDEN, "decode_cases.json")))
    for c in data["cases"]:
        dec, _, _ = fo.threshold_decode(c["kept"], np.array(c["mask"]), np.array(c["conf"], dtype=float),
                                        np.array(c["top"]), c["threshold"])
        assert dec == {int(k): v for k, v in c["decoded"].items()}, c["name"]


# ---------------------------------------------------------------- whole step
MICRO = fs.ModelShape(3, 8, 4, 2, 4, 12, 11, "f32")
MICRO_WORK = fs.Workload(2, 4, 2, ("uniform", 0, 5), ("count", 3), k_min=1, k_max=3, tau=0.0, conf_threshold=0.9)


def _step(case, **kw):
    w = case.work
    args = dict(tau=w.tau, k_min=w.k_min, k_max=w.k_max, conf_threshold=w.conf_threshold, alpha=w.alpha,
                forced_keep_frac=w.forced_keep_frac)
    args.update(kw)
    return fo.focus_step(case.shape, case.model, case.batch, **args)


def test_whole_step_matches_scalar_brute_force():
    for seed in (11, 12, 13):
        case = fs.make_case(shape=MICRO, work=MICRO_WORK, seed=seed)
        # a larger weight scale so attention is far from uniform and every term matters
        for key in ("wqkv", "wo", "wgate", "wup", "wdown"):
            case.model[key] = [t * 20 for t in case.model[key]]
        case.model["lm_head"] = case.model["lm_head"] * 40
        r = _step(case)
        s = scalar_step(case.shape, case.model, case.batch, 0.0, 1, 3, 0.9)
        np.testing.assert_allclose(r.importance, np.array(s["importance"]), rtol=1e-11, atol=1e-12)
        kept = [r.retained_idx[b, : r.keep_count[b]].tolist() for b in range(2)]
        assert kept == s["kept"]
        hid = np.array([row for b in range(2) for row in s["hidden"][b]])
        np.testing.assert_allclose(r.hidden, hid, rtol=1e-11, atol=1e-11)
        for b in range(2):
            k = r.keep_count[b]
            np.testing.assert_allclose(r.conf[b, :k], s["conf"][b], rtol=1e-11)
            assert r.top_id[b, :k].tolist() == s["top"][b]
            got = {j: int(r.decoded_ids[b, j]) for j in range(4) if r.decoded_ids[b, j] >= 0}
            assert got == s["decoded"][b]
        np.testing.assert_allclose(r.ibc, np.array(s["cache"]), rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("name", ["tiny", "small_f32"])
def test_forced_full_keep_equals_dense_forward(name):
    """Keep fraction 1: the focused step is exactly the dense full-block step."""
    case = fs.make_case(name)
    r = _step(case, forced_keep_frac=1.0)
    ref = dense_block_forward(case.shape, case.model, case.batch)
    N, B = case.batch["block_tokens"].shape
    assert r.keep_count.tolist() == [B] * N
    np.testing.assert_allclose(r.hidden, ref["hidden"].reshape(N * B, -1).numpy(), rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(r.importance, ref["colsum"].numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(r.ibc, ref["kv"].numpy(), rtol=1e-10, atol=1e-10)
    z = ref["logits"].reshape(N * B, -1).numpy()
    top = z.argmax(1)
    assert r.top_id.reshape(-1).tolist() == top.tolist()
    np.testing.assert_allclose(r.conf.reshape(-1), 1.0 / np.exp(z - z.max(1, keepdims=True)).sum(1), rtol=1e-10)


def test_bf16_storage_points_match_an_independent_bf16_forward():
    """storage='bf16' rounds where the bf16 kernels store activations -- the normalised rows, q and k after
    RoPE, v, the attention output, the SwiGLU product, the row normalised for the LM head -- and nowhere
    else (never the residual stream): with every position kept it equals an independently written forward
    that rounds at exactly those points and accumulates in float64."""
    case = fs.make_case("tiny")
    r = _step(case, forced_keep_frac=1.0, storage="bf16")
    ref = dense_block_forward(case.shape, case.model, case.batch, storage="bf16")
    N, B = case.batch["block_tokens"].shape
    np.testing.assert_allclose(r.hidden, ref["hidden"].reshape(N * B, -1).numpy(), rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(r.importance, ref["colsum"].numpy(), rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(r.ibc, ref["kv"].numpy(), rtol=1e-9, atol=1e-9)
    z = ref["logits"].reshape(N * B, -1).numpy()
    np.testing.assert_allclose(r.conf.reshape(-1), 1.0 / np.exp(z - z.max(1, keepdims=True)).sum(1), rtol=1e-9)


def test_page_permutation_leaves_the_step_unchanged():
    case = fs.make_case("small_f32")
    r1 = _step(case)
    pool, table = case.batch["kv_pool"], case.batch["page_table"]
    perm = torch.randperm(pool.shape[0], generator=torch.Generator().manual_seed(5))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(len(perm))
    case.batch["kv_pool"] = pool[perm]              # physical page p moves to slot inv[p]
    case.batch["page_table"] = torch.where(table >= 0, inv[table.clamp(min=0).long()].int(), table)
    r2 = _step(case)
    np.testing.assert_array_equal(r1.retained_idx, r2.retained_idx)
    np.testing.assert_allclose(r1.hidden, r2.hidden, rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(r1.decoded_ids, r2.decoded_ids)


def test_request_subset_equals_full_batch_rows():
    """Requests are independent: running a subset gives the same rows as the full batch."""
    case = fs.make_case("small_f32")
    full = _step(case)
    sub = _step(case, requests=[1, 4])
    rows = list(range(full.row_offsets[1], full.row_offsets[2])) + list(range(full.row_offsets[4], full.row_offsets[5]))
    np.testing.assert_allclose(sub.hidden, full.hidden[rows], rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(sub.decoded_ids, full.decoded_ids[[1, 4]])


def test_forced_keep_set_reproduces_own_selection():
    case = fs.make_case("tiny")
    r = _step(case)
    kept = [r.retained_idx[b, : r.keep_count[b]].tolist() for b in range(2)]
    r2 = _step(case, forced_keep=kept)
    np.testing.assert_array_equal(r.hidden, r2.hidden)
    np.testing.assert_array_equal(r.decoded_ids, r2.decoded_ids)


def test_step_updates_tokens_and_mask_only_where_decoded():
    case = fs.make_case("small_f32")
    r = _step(case)
    tok0, mask0 = case.batch["block_tokens"].numpy(), case.batch["mask"].numpy()
    dec = r.decoded_ids >= 0
    assert dec.sum(1).min() >= 0
    np.testing.assert_array_equal(r.block_tokens[~dec], tok0[~dec])
    np.testing.assert_array_equal(r.block_tokens[dec], r.decoded_ids[dec])
    assert (r.mask[dec] == 0).all() and (mask0[dec] == 1).all()
    np.testing.assert_array_equal(r.mask[~dec], mask0[~dec])
    # every request that kept a masked position decodes at least one
    for b in range(r.keep_count.shape[0]):
        if any(mask0[b, j] for j in r.retained_idx[b, : r.keep_count[b]]):
            assert dec[b].any()
