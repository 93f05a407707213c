"""The effective-batch scheduler (continuous batching around the focused step), on the CPU with the oracle
as its engine.  The step treats requests independently, so whatever the schedule -- arrivals, slot
reuse, requests in different phases of their block loops sharing an iteration -- every request must
decode exactly what it decodes alone through the oracle's block loop, and commit exactly the same K/V."""
import dataclasses

import numpy as np
import pytest
import torch

import focus_synth as fs
from oracle import focus_oracle as fo
from decodability_aware_token_b200.scheduler import EffectiveBatchScheduler, Request

B = 8          # block size of these runs (the oracle takes any)
S = 16         # page size
MAX_PAGES = 6


class OracleEngine:
    """The scheduler's engine with the oracle's step and commit (float64 state, so nothing is rounded
    between steps and the comparison with the oracle's own block loop is exact)."""

    def __init__(self, case):
        self.shape, self.model, self.w = case.shape, case.model, case.work
        self.calls = []

    def step(self, view, dense):
        w = self.w
        r = fo.focus_step(self.shape, self.model, view, tau=w.tau, k_min=w.k_min, k_max=w.k_max,
                          conf_threshold=w.conf_threshold, alpha=w.alpha,
                          forced_keep_frac=1.0 if dense else -1.0, max_keep=B)
        view["block_tokens"].copy_(torch.as_tensor(r.block_tokens))
        view["mask"].copy_(torch.as_tensor(r.mask))
        view["ibc"].copy_(torch.as_tensor(r.ibc))
        self.calls.append(("dense" if dense else "focused", view["block_tokens"].shape[0]))

    def commit(self, view):
        pool, plen = fo.commit_block(view["kv_pool"], view["ibc"], view["prefix_len"], view["page_table"])
        view["kv_pool"].copy_(torch.as_tensor(pool))
        view["prefix_len"].copy_(torch.as_tensor(plen))
        self.calls.append(("commit", 1))


def _setup(prompts, seed=7, spare=24):
    """A float64 page pool holding every request's prompt K/V (N(0,1), seeded) in shuffled pages, plus
    `spare` free pages; returns (pool, prompt pages per request, free pages)."""
    case = fs.make_case("tiny")
    s = case.shape
    need = [-(-p // S) for p in prompts]
    n_pages = sum(need) + spare
    g = torch.Generator().manual_seed(seed)
    pool = torch.randn(n_pages, s.n_layers, 2, s.n_kv_heads, S, s.head_dim, generator=g, dtype=torch.float64)
    order = torch.randperm(n_pages, generator=g).tolist()
    pages, at = [], 0
    for n in need:
        pages.append(order[at:at + n])
        at += n
    return case, pool, pages, order[at:]


_ALONE = {}


def _alone(case, pool, prompt_len, prompt_pages, n_blocks):
    """Decode one request by itself through the oracle's block loop, block after block (memoised on the
    inputs: several tests compare against the same requests)."""
    key = (prompt_len, tuple(prompt_pages), n_blocks, case.work, float(pool.sum()), pool.shape)
    if key not in _ALONE:
        _ALONE[key] = _alone_uncached(case, pool, prompt_len, prompt_pages, n_blocks)
    return _ALONE[key]


def _alone_uncached(case, pool, prompt_len, prompt_pages, n_blocks):
    s, w = case.shape, case.work
    pool = pool.clone().numpy()
    used = set(range(pool.shape[0])) - set(prompt_pages)
    free = sorted(used)
    pages = list(prompt_pages)
    plen = prompt_len
    blocks, steps = [], []
    for _ in range(n_blocks):
        while len(pages) * S < plen + B:
            pages.append(free.pop(0))
        row = np.full((1, MAX_PAGES), -1, dtype=np.int64)
        row[0, : len(pages)] = pages
        batch = {"block_tokens": np.full((1, B), s.vocab - 1), "mask": np.ones((1, B)),
                 "prefix_len": np.array([plen]), "page_table": row, "kv_pool": pool,
                 "ibc": np.zeros((1, s.n_layers, 2, s.n_kv_heads, B, s.head_dim))}
        res = fo.decode_block(s, case.model, batch, tau=w.tau, k_min=w.k_min, k_max=w.k_max,
                              conf_threshold=w.conf_threshold, alpha=w.alpha)
        blocks.append(res.block_tokens[0].copy())
        steps.append(len(res.steps))
        pool, plen = res.kv_pool, int(res.prefix_len[0])
    return blocks, steps, _kv(pool, pages, plen)


def _kv(pool, pages, plen):
    """The request's K/V by position: [plen, L, 2, Hkv, d]."""
    pool = np.asarray(pool)
    return np.stack([pool[pages[p // S], :, :, :, p % S, :] for p in range(plen)])


def _scheduler(case, pool, free, **kw):
    s = case.shape
    return EffectiveBatchScheduler(OracleEngine(case), block=B, n_layers=s.n_layers, n_kv_heads=s.n_kv_heads,
                                   head_dim=s.head_dim, max_pages_per_req=MAX_PAGES, kv_pool=pool, free_pages=free,
                                   mask_token=s.vocab - 1, k_max=case.work.k_max, **kw)


PROMPTS = [24, 0, 40, 16, 7]
ARRIVALS = [0, 0, 1, 2, 6]
NBLOCKS = [2, 1, 2, 1, 2]


def test_every_request_decodes_what_it_decodes_alone():
    case, pool, pages, free = _setup(PROMPTS)
    init = pool.clone()
    sch = _scheduler(case, pool, free, slots=3, keep_pages=True)
    for r, (p, a, nb) in enumerate(zip(PROMPTS, ARRIVALS, NBLOCKS)):
        sch.submit(Request(r, a, p, pages[r], nb))
    res = sch.run(max_iterations=400)
    assert sorted(res) == list(range(len(PROMPTS)))
    for r, (p, nb) in enumerate(zip(PROMPTS, NBLOCKS)):
        blocks, steps, kv = _alone(case, init, p, pages[r], nb)
        got = res[r]
        assert got.prefix_len == p + nb * B
        assert [b.tolist() for b in got.blocks] == [b.tolist() for b in blocks], f"request {r}"
        assert got.steps == steps, f"request {r}"
        np.testing.assert_array_equal(_kv(sch.kv_pool.numpy(), got.pages, got.prefix_len), kv)
    # the schedule really mixed phases: some iteration ran a focused and a dense call together
    assert any(st.focused and st.dense for st in sch.stats)
    assert all(st.active <= 3 for st in sch.stats)


def test_slots_and_pages_are_recycled():
    case, pool, pages, free = _setup(PROMPTS, spare=8)
    total = len(free) + sum(len(p) for p in pages)
    sch = _scheduler(case, pool, free, slots=2)
    for r, (p, a, nb) in enumerate(zip(PROMPTS, ARRIVALS, NBLOCKS)):
        sch.submit(Request(r, a, p, pages[r], nb))
    sch.run(max_iterations=400)
    assert sch.done() and not sch.slot_req
    assert sorted(sch.free) == list(range(total))          # every page is back in the pool
    for r, a in enumerate(ARRIVALS):
        assert sch.results[r].admitted >= a
    # first come, first served
    adm = [sch.results[r].admitted for r in range(len(PROMPTS))]
    assert adm == sorted(adm)


def test_row_budget_sets_the_effective_batch():
    """With the budget of a dense engine on 2 requests (2 x B rows), focused requests (k_max rows each)
    let more requests run at once than slots counted densely would."""
    prompts = [16] * 6
    case, pool, pages, free = _setup(prompts)
    k_max = 2
    case = dataclasses.replace(case, work=dataclasses.replace(case.work, k_min=1, k_max=k_max))
    dense_budget = 2 * B
    sch = _scheduler(case, pool, free, slots=6, row_budget=dense_budget)
    for r, p in enumerate(prompts):
        sch.submit(Request(r, 2 * r, p, pages[r], 1))   # staggered: each arrives while others are focused
    sch.run(max_iterations=400)
    # a dense engine with this budget runs 2 requests; focused ones cost k_max rows, so more fit
    assert max(st.active for st in sch.stats) > dense_budget // B
    for st in sch.stats:
        assert st.row_cost == st.focused * k_max + st.dense * B
    # no iteration ran more rows than the budget
    assert all(st.row_cost <= dense_budget for st in sch.stats)


def test_requests_that_cannot_fit_are_refused():
    case, pool, pages, free = _setup([24])
    sch = _scheduler(case, pool, free, slots=1)
    with pytest.raises(ValueError):
        sch.submit(Request(0, 0, 24, pages[0], (MAX_PAGES * S - 24) // B + 1))   # beyond the page table
    with pytest.raises(ValueError):
        sch.submit(Request(1, 0, 24, pages[0][:1], 1))                            # prompt pages missing
    with pytest.raises(ValueError):
        _scheduler(case, pool, free, slots=1, row_budget=B - 1)


class _MarshalOnlyContext:
    """Stands in for a FocusContext on the CPU: every call goes through the binding's own argument
    marshalling (dtype, device, contiguity and shape checks, ctypes structs), then the oracle does the
    work.  It checks that FocusEngine hands the library well-formed slot views and output slices."""

    def __init__(self, case, max_requests):
        from decodability_aware_token_b200 import _abi
        self.shape, self.model, self.w = case.shape, case.model, case.work
        self.dtype, self.device = torch.float64, torch.device("cpu")
        self.limits = _abi.Limits(max_requests, B, B, MAX_PAGES)
        self.params_seen = []
        self.calls = []

    @property
    def max_keep(self):
        return self.limits.max_keep

    def alloc_outputs(self, n, block, importance=True, hidden=True):
        from decodability_aware_token_b200 import FocusContext
        return FocusContext.alloc_outputs(self, n, block, importance, hidden)

    def step(self, batch, params, out=None, stream=None):
        from decodability_aware_token_b200 import FocusContext
        FocusContext._marshal(self, batch, params, out)
        self.params_seen.append(params.forced_keep_frac)
        OracleEngine.step(self, batch, dense=params.forced_keep_frac == 1.0)

    def commit_block(self, batch, stream=None):
        from decodability_aware_token_b200 import FocusContext, StepParams
        n, block = batch["block_tokens"].shape
        FocusContext._marshal(self, batch, StepParams(), self.alloc_outputs(n, block))
        OracleEngine.commit(self, batch)


def test_focus_engine_marshals_slot_views_for_the_library():
    from decodability_aware_token_b200 import StepParams
    from decodability_aware_token_b200.scheduler import FocusEngine
    case, pool, pages, free = _setup(PROMPTS)
    init = pool.clone()
    w = case.work
    ctx = _MarshalOnlyContext(case, max_requests=3)
    params = StepParams(w.tau, w.k_min, w.k_max, w.conf_threshold, w.alpha)
    s = case.shape
    sch = EffectiveBatchScheduler(FocusEngine(ctx, params), slots=3, block=B, n_layers=s.n_layers,
                                  n_kv_heads=s.n_kv_heads, head_dim=s.head_dim, max_pages_per_req=MAX_PAGES,
                                  kv_pool=pool, free_pages=free, mask_token=s.vocab - 1, k_max=w.k_max,
                                  keep_pages=True)
    for r, (p, a, nb) in enumerate(zip(PROMPTS, ARRIVALS, NBLOCKS)):
        sch.submit(Request(r, a, p, pages[r], nb))
    res = sch.run(max_iterations=400)
    assert set(ctx.params_seen) == {1.0, -1.0}          # dense and focused calls, nothing else
    for r, (p, nb) in enumerate(zip(PROMPTS, NBLOCKS)):
        blocks, _, kv = _alone(case, init, p, pages[r], nb)
        assert [b.tolist() for b in res[r].blocks] == [b.tolist() for b in blocks]
        np.testing.assert_array_equal(_kv(sch.kv_pool.numpy(), res[r].pages, res[r].prefix_len), kv)


def test_admission_reserves_every_page_a_request_needs():
    """A pool with room for one long request at a time: the second waits for the first to finish
    instead of starting and running out of pages mid-flight."""
    prompts = [16, 16]
    case, pool, pages, free = _setup(prompts, spare=3)            # 3 free pages: 3 blocks of 8 over 16 tokens
    sch = _scheduler(case, pool, free, slots=2)
    sch.submit(Request(0, 0, 16, pages[0], 3))                     # needs ceil((16 + 24) / 16) - 1 = 2 pages
    sch.submit(Request(1, 0, 16, pages[1], 3))                     # 2 more: only 1 left while 0 runs
    res = sch.run(max_iterations=400)
    assert res[1].admitted > res[0].admitted
    assert res[1].admitted >= res[0].finished


def test_focus_engine_refuses_a_context_too_small_for_the_slots_or_block():
    from decodability_aware_token_b200 import StepParams
    from decodability_aware_token_b200.scheduler import FocusEngine
    case, pool, pages, free = _setup([16])
    s = case.shape
    eng = FocusEngine(_MarshalOnlyContext(case, max_requests=2), StepParams())
    kw = dict(block=B, n_layers=s.n_layers, n_kv_heads=s.n_kv_heads, head_dim=s.head_dim, max_pages_per_req=MAX_PAGES,
              kv_pool=pool, free_pages=free, mask_token=s.vocab - 1, k_max=2)
    with pytest.raises(ValueError):
        EffectiveBatchScheduler(eng, slots=3, **kw)                       # more slots than max_requests
    small = _MarshalOnlyContext(case, max_requests=2)
    small.limits.max_keep = B // 2
    with pytest.raises(ValueError):
        EffectiveBatchScheduler(FocusEngine(small, StepParams()), slots=2, **kw)   # dense steps need max_keep >= B
    EffectiveBatchScheduler(eng, slots=2, **kw)                           # fits


class _OnePerStepEngine:
    """Decodes the lowest masked position of every request at each step with a masked position -- what
    the fallback of the decode rule does with random weights -- and grows the prefix at a commit.  Fast
    stand-in for the scheduling logic alone."""

    def step(self, view, dense):
        m = view["mask"]
        for r in range(m.shape[0]):
            left = torch.nonzero(m[r]).flatten()
            if left.numel():
                view["block_tokens"][r, left[0]] = 7
                m[r, left[0]] = 0

    def commit(self, view):
        view["prefix_len"] += B


def _trace_iterations(k_max, budget, n_req=12):
    pool = torch.zeros(64, 1, 2, 1, S, 4)
    sch = EffectiveBatchScheduler(_OnePerStepEngine(), slots=n_req, block=B, n_layers=1, n_kv_heads=1, head_dim=4,
                                  max_pages_per_req=MAX_PAGES, kv_pool=pool, free_pages=range(64), mask_token=9,
                                  k_max=k_max, row_budget=budget)
    for r in range(n_req):
        sch.submit(Request(r, 0, 0, [], 1 + r % 3))
    sch.run(max_iterations=10_000)
    assert all(st.row_cost <= budget for st in sch.stats)   # the budget holds in every iteration
    rows = sum(st.row_cost for st in sch.stats)
    return sch.iteration, max(st.active for st in sch.stats), rows, sum(st.deferred for st in sch.stats)


def test_focused_accounting_finishes_a_trace_in_fewer_steps():
    """The same row budget (that of a dense engine on 2 requests) and the same trace: counting focused
    requests at k_max rows runs more of them at once and finishes in fewer iterations than counting every
    request at B rows."""
    dense_iters, dense_peak, dense_rows, _ = _trace_iterations(k_max=B, budget=2 * B)
    focus_iters, focus_peak, focus_rows, deferred = _trace_iterations(k_max=2, budget=2 * B)
    assert dense_peak == 2 and focus_peak > dense_peak
    assert focus_iters < dense_iters and focus_rows < dense_rows
    assert deferred > 0   # refreshes that would have run past the budget waited for a later iteration
