"""Pins of the oracle's block loop and commit (CPU only).

The loop around the focused step: a dense first step, focused steps until nothing is masked, a dense
refresh of the decoded block, and the commit of its K/V into the prefix pages.  The commit is pinned to
an independently written dense block forward (exact prefix caching), and a planted indexing slip must
be caught.
"""
import numpy as np
import pytest
import torch

import focus_synth as fs
from dense_reference import dense_block_forward
from oracle import focus_oracle as fo


def _block(name):
    case = fs.make_case(name)
    batch = fs.with_block_pages(case.batch, case.work.block)
    w = case.work
    r = fo.decode_block(case.shape, case.model, batch, tau=w.tau, k_min=w.k_min, k_max=w.k_max,
                        conf_threshold=w.conf_threshold)
    return case, batch, r


def test_block_loop_decodes_every_position_with_progress():
    case, batch, r = _block("tiny")
    N, B = case.batch["block_tokens"].shape
    mask0 = case.batch["mask"].numpy().astype(bool)
    assert r.steps[0].keep_count.tolist() == [B] * N            # the first step is dense
    assert len(r.steps) <= B
    prev = mask0
    for s in r.steps:
        now = s.mask.astype(bool)
        assert not (now & ~prev).any()                            # nothing becomes masked again
        for b in range(N):
            if prev[b].any():
                assert (prev[b] & ~now[b]).sum() >= 1             # every step decodes in every unfinished request
        prev = now
    assert not prev.any()
    # unmasked positions keep their tokens; decoded ones hold the step's decoded ids
    t0 = case.batch["block_tokens"].numpy()
    assert (r.block_tokens[~mask0] == t0[~mask0]).all()
    dec = np.full((N, B), -1)
    for s in r.steps:
        dec = np.where(s.decoded_ids >= 0, s.decoded_ids, dec)
    assert (r.block_tokens[mask0] == dec[mask0]).all()
    np.testing.assert_array_equal(r.prefix_len, case.batch["prefix_len"].numpy() + B)


@pytest.mark.parametrize("name", ["tiny", "small_f32"])
def test_commit_holds_the_dense_kv_of_the_decoded_block(name):
    """Exact prefix caching: the pages now hold, at positions P .. P + B - 1, the K/V an independent dense
    forward of the decoded block computes on top of the same prefix."""
    case, batch, r = _block(name)
    done = dict(batch)
    done["block_tokens"] = torch.from_numpy(r.block_tokens.astype(np.int32))
    ref = dense_block_forward(case.shape, case.model, done)["kv"].numpy()      # [N, L, 2, Hkv, B, d]
    plen0 = batch["prefix_len"].numpy()
    table = batch["page_table"].numpy()
    S = batch["kv_pool"].shape[4]
    N, B = r.block_tokens.shape
    for b in range(N):
        for j in range(B):
            pos = int(plen0[b]) + j
            got = r.kv_pool[table[b, pos // S], :, :, :, pos % S, :]
            np.testing.assert_allclose(got, ref[b, :, :, :, j, :], rtol=1e-10, atol=1e-10)
    # everything else in the pool is untouched
    pool0 = batch["kv_pool"].double().numpy()
    touched = np.zeros(pool0.shape[0:1] + pool0.shape[4:5], dtype=bool)
    for b in range(N):
        for j in range(B):
            pos = int(plen0[b]) + j
            touched[table[b, pos // S], pos % S] = True
    keep = ~touched
    np.testing.assert_array_equal(np.moveaxis(r.kv_pool, 4, 1)[keep], np.moveaxis(pool0, 4, 1)[keep])


def test_commit_brute_force_positions():
    """A distinct value per (request, block position) lands at exactly its page slot."""
    rng = np.random.default_rng(3)
    N, L, H, B, d, S = 3, 2, 2, 5, 4, 4
    plen = np.array([0, 3, 9])
    pages = [(p + B + S - 1) // S for p in plen]
    table = np.full((N, max(pages)), -1)
    perm = rng.permutation(sum(pages))
    at = 0
    for b in range(N):
        table[b, : pages[b]] = perm[at:at + pages[b]]
        at += pages[b]
    pool = rng.normal(size=(sum(pages), L, 2, H, S, d))
    ibc = np.zeros((N, L, 2, H, B, d))
    for b in range(N):
        for j in range(B):
            ibc[b, :, :, :, j, :] = 1000 * b + j
    out, plen2 = fo.commit_block(pool, ibc, plen, table)
    for b in range(N):
        for j in range(B):
            pos = plen[b] + j
            assert (out[table[b, pos // S], :, :, :, pos % S, :] == 1000 * b + j).all()
    assert plen2.tolist() == (plen + B).tolist()


def test_planted_commit_offset_is_caught(monkeypatch):
    real = fo.commit_block

    def shifted(kv_pool, ibc, prefix_len, page_table):   # slip: one position too far
        return real(kv_pool, ibc, np.asarray(prefix_len) + 1, page_table)[0], np.asarray(prefix_len) + ibc.shape[4]

    monkeypatch.setattr(fo, "commit_block", shifted)
    with pytest.raises(AssertionError):
        test_commit_brute_force_positions()
