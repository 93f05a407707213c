"""GPU: the loop around the focused step (dense first step, focused steps, dense refresh, commit).

Every step of a GPU-run block loop is checked against the oracle on that step's own inputs (so a
near-tie in one step does not compound), the commit is checked bit for bit against the oracle's
commit of the same cache, and the native loop (focus_decode_block) must reproduce the loop driven step
by step through the C ABI exactly.
"""
import numpy as np
import pytest
import torch

import focus_synth as fs
from gpu_harness import check, step_params, to_device
from oracle import focus_oracle as fo

pytestmark = pytest.mark.gpu


def _limits(case, batch):
    B = case.work.block
    return dict(max_requests=case.work.n_requests, max_block=B, max_keep=B,
                max_pages_per_req=int(batch["page_table"].shape[1]))


def _dev(batch):
    return {k: v.to("cuda:0").clone() for k, v in batch.items()}


@pytest.mark.parametrize("name", ["tiny", "small_bf16"])
def test_commit_block_copies_the_cache_into_the_pages(name):
    from decodability_aware_token_b200 import FocusContext
    case = fs.make_case(name)
    batch = fs.with_block_pages(case.batch, case.work.block)
    gb = _dev(batch)
    with FocusContext(case.shape, to_device(case), **_limits(case, batch)) as ctx:
        ctx.commit_block(gb)
        torch.cuda.synchronize()
        rc, bits = ctx.device_error()
    assert rc == 0, bits
    want_pool, want_plen = fo.commit_block(batch["kv_pool"], batch["ibc"], batch["prefix_len"], batch["page_table"])
    np.testing.assert_array_equal(gb["kv_pool"].cpu().double().numpy(), want_pool)   # a copy: bit-exact
    np.testing.assert_array_equal(gb["prefix_len"].cpu().numpy(), want_plen)


def _gpu_record(step_out, state):
    rec = {k: (v.cpu() if v is not None else None) for k, v in step_out.tensors().items()}
    rec.update(block_tokens=state["block_tokens"].cpu(), mask=state["mask"].cpu(), ibc=state["ibc"].cpu(),
               device_status=0, device_bits=0)
    return rec


@pytest.mark.parametrize("name,checked", [("tiny", None), ("small_bf16", (0, 1, 2, -2, -1))])
def test_block_loop_steps_match_oracle_and_native_loop(name, checked):
    from decodability_aware_token_b200 import FocusContext, StepParams
    case = fs.make_case(name)
    batch = fs.with_block_pages(case.batch, case.work.block)
    model = to_device(case)
    lim = _limits(case, batch)
    N, B = case.work.n_requests, case.work.block
    base = step_params(case.work)
    state = _dev(batch)
    steps = []
    with FocusContext(case.shape, model, **lim) as ctx:
        def run(frac):
            before = {k: state[k].cpu().clone() for k in ("block_tokens", "mask", "ibc")}
            p = dict(base, forced_keep_frac=frac)
            out = ctx.step(state, StepParams(**p))
            torch.cuda.synchronize()
            steps.append((before, p, _gpu_record(out, state)))
        run(1.0)
        while bool(state["mask"].any()) and len(steps) < B:
            run(-1.0)
        assert not bool(state["mask"].any())
        n_decoding = len(steps)
        run(1.0)                                        # dense refresh of the decoded block
        ctx.commit_block(state)
        torch.cuda.synchronize()
        rc, bits = ctx.device_error()
        assert rc == 0, bits

        # the native loop from the same start reproduces it exactly
        native = _dev(batch)
        _, n_native = ctx.decode_block(native, StepParams(**base))
        torch.cuda.synchronize()
    assert n_native == n_decoding
    for k in ("block_tokens", "mask", "ibc", "kv_pool", "prefix_len"):
        assert torch.equal(native[k].cpu(), state[k].cpu()), k

    # every (or every sampled) step against the oracle on that step's own inputs
    idx = range(len(steps)) if checked is None else sorted({i % len(steps) for i in checked})
    for i in idx:
        before, p, rec = steps[i]
        host = dict(batch)
        host.update(before)
        sc = fs.Case(case.shape, case.work, case.model, host, case.seed)
        rep = check(sc, p, model, gpu=rec, limits=lim)
        print(name, "step", i, {k: v for k, v in rep.items() if k in ("flipped",)})
    # the commit holds the refreshed cache
    want_pool, want_plen = fo.commit_block(batch["kv_pool"], steps[-1][2]["ibc"], batch["prefix_len"],
                                           batch["page_table"])
    np.testing.assert_array_equal(state["kv_pool"].cpu().double().numpy(), want_pool)
    np.testing.assert_array_equal(state["prefix_len"].cpu().numpy(), want_plen)
