"""GPU: the effective-batch scheduler driving the library (FocusEngine: focus_step and focus_commit_block on
slot views of one batch), on a trace of ragged requests that arrive staggered, share slots, sit in
different phases of their block loops and run under a row budget that defers dense steps.

  * sampled engine calls are checked against the oracle on that call's own inputs (the reduced 4-layer
    bf16 shape: the plain float64 oracle, no allowance), so a near-tie in one step does not compound;
  * every commit is checked bit for bit against the oracle's commit of the same cache into the same
    pool, so the slot and page bookkeeping (which pages, which positions) is exact;
  * every request decodes what it decodes alone: the same blocks in the same number of steps as a run of
    that request by itself through the same engine.  (Requests are independent in the step; the GPU's
    attention splits long key walks into a number of pieces that depends on the batch, so agreement is up
    to float summation order -- on these seeded inputs no decision is that close.)
"""
import numpy as np
import pytest
import torch

import focus_synth as fs
from gpu_harness import check, step_params, to_device
from oracle import focus_oracle as fo

pytestmark = pytest.mark.gpu

B, S, MAX_PAGES, N_REQ, SLOTS = 16, 16, 12, 12, 5


def _trace(seed=31):
    g = torch.Generator().manual_seed(seed)
    prompts = torch.randint(0, 121, (N_REQ,), generator=g).tolist()
    arrivals = sorted(torch.randint(0, 12, (N_REQ,), generator=g).tolist())
    blocks = (1 + torch.randint(0, 2, (N_REQ,), generator=g)).tolist()
    return prompts, arrivals, blocks


def _pool(shape, prompts, spare=40, seed=5):
    need = [-(-p // S) for p in prompts]
    n_pages = sum(need) + spare
    g = torch.Generator().manual_seed(seed)
    pool = torch.randn(n_pages, shape.n_layers, 2, shape.n_kv_heads, S, shape.head_dim, generator=g)
    order = torch.randperm(n_pages, generator=g).tolist()
    pages, at = [], 0
    for n in need:
        pages.append(order[at:at + n])
        at += n
    return pool.to(torch.bfloat16), pages, order[at:]


class RecordingEngine:
    """FocusEngine plus a record of sampled steps (inputs, pool, outputs) and a check of every commit."""

    def __init__(self, engine, every):
        self.engine, self.every, self.calls = engine, every, 0
        self.records, self.commits = [], 0

    def capacity_check(self, slots, block):
        self.engine.capacity_check(slots, block)

    def step(self, view, dense):
        self.calls += 1
        if self.calls % self.every:
            return self.engine.step(view, dense)
        before = {k: view[k].cpu().clone() for k in ("block_tokens", "mask", "prefix_len", "page_table", "ibc")}
        pool = view["kv_pool"].cpu().clone()
        p = self.engine.dense if dense else self.engine.focused
        n, block = view["block_tokens"].shape
        out = self.engine.ctx.step(view, p, out=self.engine.ctx.alloc_outputs(n, block))
        torch.cuda.synchronize()
        rec = {k: (v.cpu() if v is not None else None) for k, v in out.tensors().items()}
        rec.update(block_tokens=view["block_tokens"].cpu(), mask=view["mask"].cpu(), ibc=view["ibc"].cpu(),
                   device_status=0, device_bits=0)
        self.records.append((before, pool, dense, rec))

    def commit(self, view):
        pool0, ibc = view["kv_pool"].cpu().double().numpy(), view["ibc"].cpu()
        plen0, table = view["prefix_len"].cpu(), view["page_table"].cpu()
        self.engine.commit(view)
        torch.cuda.synchronize()
        want_pool, want_plen = fo.commit_block(pool0, ibc, plen0, table)
        np.testing.assert_array_equal(view["kv_pool"].cpu().double().numpy(), want_pool)   # a copy: bit-exact
        np.testing.assert_array_equal(view["prefix_len"].cpu().numpy(), want_plen)
        self.commits += 1


def _run(case, model, pool, pages, free, reqs, slots, row_budget, every=0):
    from decodability_aware_token_b200 import FocusContext, StepParams
    from decodability_aware_token_b200.scheduler import EffectiveBatchScheduler, FocusEngine, Request
    s, w = case.shape, case.work
    params = StepParams(w.tau, w.k_min, w.k_max, w.conf_threshold, w.alpha)
    with FocusContext(s, model, max_requests=slots, max_block=B, max_keep=B, max_pages_per_req=MAX_PAGES) as ctx:
        eng = FocusEngine(ctx, params)
        if every:
            eng = RecordingEngine(eng, every)
        sch = EffectiveBatchScheduler(eng, slots=slots, block=B, n_layers=s.n_layers, n_kv_heads=s.n_kv_heads,
                                      head_dim=s.head_dim, max_pages_per_req=MAX_PAGES, kv_pool=pool, free_pages=free,
                                      mask_token=s.vocab - 1, k_max=w.k_max, row_budget=row_budget, keep_pages=True)
        for r in reqs:
            sch.submit(Request(*r))
        res = sch.run(max_iterations=2000)
        rc, bits = ctx.device_error()
    assert rc == 0, bits
    return sch, res, eng


def test_scheduled_requests_match_the_oracle_step_by_step_and_decode_as_alone():
    case = fs.make_case("small_bf16", k_min=1, k_max=4)
    s, w = case.shape, case.work
    model = to_device(case)
    prompts, arrivals, nblocks = _trace()
    pool_host, pages, free = _pool(s, prompts)
    reqs = [(r, arrivals[r], prompts[r], pages[r], nblocks[r]) for r in range(N_REQ)]
    pool = pool_host.cuda()
    sch, res, eng = _run(case, model, pool, pages, free, reqs, SLOTS, row_budget=2 * B, every=3)

    assert sorted(res) == list(range(N_REQ))
    assert max(st.active for st in sch.stats) > 2          # more than a dense engine's 2 requests at once
    assert all(st.row_cost <= 2 * B for st in sch.stats)   # the budget holds in every iteration
    assert any(st.focused and st.dense for st in sch.stats)
    assert eng.commits == sum(nblocks)

    # sampled calls against the oracle on their own inputs
    params_f = step_params(w, forced_keep_frac=-1.0)
    params_d = step_params(w, forced_keep_frac=1.0)
    for before, pool_then, dense, rec in eng.records:
        n = before["block_tokens"].shape[0]
        batch = dict(before, kv_pool=pool_then)
        wk = fs.Workload(n, B, S, ("fixed", 0), ("count", 0), k_min=w.k_min, k_max=w.k_max, tau=w.tau,
                         conf_threshold=w.conf_threshold, alpha=w.alpha, forced_keep_frac=1.0 if dense else -1.0)
        sc = fs.Case(s, wk, case.model, batch, case.seed)
        lim = dict(max_requests=SLOTS, max_block=B, max_keep=B, max_pages_per_req=MAX_PAGES)
        check(sc, params_d if dense else params_f, model, gpu=rec, limits=lim)
    assert len(eng.records) >= 10

    # every request alone, through the same engine and a pool in the same starting state
    for r in range(N_REQ):
        pool_r = pool_host.cuda()
        _, alone, _ = _run(case, model, pool_r, pages, free, [(r, 0, prompts[r], pages[r], nblocks[r])], 1,
                           row_budget=B)
        got, want = res[r], alone[r]
        assert [b.tolist() for b in got.blocks] == [b.tolist() for b in want.blocks], f"request {r}"
        assert got.steps == want.steps, f"request {r}"
        assert got.prefix_len == prompts[r] + nblocks[r] * B
