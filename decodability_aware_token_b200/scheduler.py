"""Continuous batching of ragged requests around the focused step: an effective-batch scheduler.

FOCUS turns the compute it saves on evicted block positions into a larger effective batch
("FOCUS: DLLMs Know How to Tame Their Compute Bound": arXiv abstract; project page, Overview -- the saved
FLOPs become throughput).  This module is the host-side loop that does so.  It is orchestration only:
every step and every commit runs through an engine (``FocusEngine``: the library's ``focus_step`` and
``focus_commit_block``); nothing of the method's arithmetic is here.

Requests arrive with their prompt already in the KV pool (the step serves blocks on top of an exactly
cached prefix, project page, Overview -- Motivation) and ask for a number of blocks.  Each block of
each request goes through the block loop of ``focus_decode_block``: a dense first step, focused steps
until no position is masked, a dense refresh, and the commit of the block's K/V into the prefix pages.
Requests sit in the slots of one batch; they are in different phases of that loop at the same time, so
each iteration runs at most two calls on contiguous slot ranges -- the focused steps, then the dense
steps (first steps and refreshes) -- and then commits the blocks whose refresh just ran.  Finished
requests leave their slot at once and waiting ones take it (continuous batching).

The row budget (the effective batch): a request in a focused step costs at most k_max rows in layers
2..L-1, one in a dense step costs B, and no iteration runs more than ``row_budget`` rows.  A waiting
request is admitted while a slot is free, the pages for all its blocks can be reserved, and the summed
cost of the active requests plus B (its dense first step) stays within the budget.  Every iteration then
runs all focused steps and as many dense steps (first steps and refreshes, oldest admission first) as
still fit; the other dense steps wait for a later iteration.  The focused steps always fit (each
admission kept every active request's cost, at least k_max, within the budget), and when no request is
focused at least one dense step runs, so every request keeps moving.  A dense engine spending N x B rows
per step admits N requests; with the same budget, focused requests cost k_max, so up to N x B / k_max of
them run at once.

Readings (the pages describe no scheduler): first come, first served among arrived requests; a
request's prompt pages and the pages allocated for its blocks return to the pool when it finishes
(unless ``keep_pages``).  The step treats requests independently, so every request decodes what it
decodes alone: exactly with the oracle as engine; on the GPU up to the float summation order, since the
attention splits long key walks into pieces only when a batch has few (request, head) units.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import torch

from . import StepOutputs

__all__ = ["Request", "RequestResult", "IterationStats", "EffectiveBatchScheduler", "FocusEngine"]

_DENSE_FIRST, _FOCUSED, _DENSE_REFRESH = 0, 1, 2


@dataclasses.dataclass
class Request:
    rid: int
    arrival: int                  # first iteration at which the request may be admitted
    prompt_len: int               # P: prompt tokens whose K/V are already in the pool
    prompt_pages: List[int]       # pool pages holding them, in position order (owned by the request)
    n_blocks: int                 # blocks to generate (>= 1)


@dataclasses.dataclass
class RequestResult:
    rid: int
    blocks: List[torch.Tensor]    # the decoded blocks, [B] int32 each, on the host
    admitted: int                 # iteration of admission
    finished: int                 # iteration whose commit completed the last block
    prefix_len: int               # prompt_len + n_blocks * B
    pages: List[int]              # pages covering positions 0 .. prefix_len - 1, in order
    steps: List[int]              # decoding steps of each block (the dense first step included)


@dataclasses.dataclass
class IterationStats:
    iteration: int
    active: int                   # requests in slots during the iteration
    focused: int                  # of which in a focused step
    dense: int                    # of which ran a dense step (first step or refresh)
    row_cost: int                 # focused * k_max + dense * B: rows run, at most row_budget
    committed: int                # blocks committed at the end of the iteration
    deferred: int = 0             # requests whose dense step waits for a later iteration (budget full)


class FocusEngine:
    """Runs the scheduler's calls on the GPU through a FocusContext (steps and commits on slot views)."""

    def __init__(self, ctx, params, stream: Optional[torch.cuda.Stream] = None):
        self.ctx = ctx
        self.focused = dataclasses.replace(params, forced_keep_frac=-1.0, forced_keep_idx=None,
                                           forced_keep_count=None)
        self.dense = dataclasses.replace(self.focused, forced_keep_frac=1.0)
        self.stream = stream
        self._out = None

    def capacity_check(self, slots: int, block: int) -> None:
        """The context must take every slot in one call and keep all B positions in the dense steps."""
        lim = self.ctx.limits
        if slots > lim.max_requests:
            raise ValueError(f"{slots} slots exceed the context's max_requests ({lim.max_requests})")
        if block > lim.max_block or block > lim.max_keep:
            raise ValueError(f"block {block}: the context needs max_block and max_keep >= B for the dense steps")

    def _outputs(self, n: int, block: int):
        if self._out is None or self._out.keep_count.shape[0] < n or self._out.decoded_ids.shape[1] != block:
            self._out = self.ctx.alloc_outputs(max(n, 1), block, importance=False, hidden=False)
        o = self._out
        return StepOutputs(o.keep_count[:n], o.retained_idx[:n], o.row_offsets[:n + 1], o.decoded_ids[:n],
                           o.conf[:n], o.top_id[:n])

    def step(self, view: Dict[str, torch.Tensor], dense: bool) -> None:
        n, block = view["block_tokens"].shape
        self.ctx.step(view, self.dense if dense else self.focused, out=self._outputs(n, block), stream=self.stream)

    def commit(self, view: Dict[str, torch.Tensor]) -> None:
        self.ctx.commit_block(view, stream=self.stream)


class EffectiveBatchScheduler:
    """Continuous batching of block-diffusion requests over `slots` batch slots (see the module notes).

    engine:       object with step(view, dense) and commit(view) acting in place on slot views
    kv_pool:      [pages, L, 2, Hkv, S, d] tensor shared by every request (prompts already written)
    free_pages:   pool pages not holding any prompt, available for generated blocks
    mask_token:   token id of a masked position (the block starts all masked)
    row_budget:   admission budget in layers-2..L-1 rows per iteration (default slots x B: no gain
                  counted); k_max: the focused steps' budget ceiling
    """

    def __init__(self, engine, *, slots: int, block: int, n_layers: int, n_kv_heads: int, head_dim: int,
                 max_pages_per_req: int, kv_pool: torch.Tensor, free_pages, mask_token: int, k_max: int,
                 row_budget: Optional[int] = None, keep_pages: bool = False):
        if slots < 1 or block < 1 or k_max < 1 or max_pages_per_req < 1:
            raise ValueError("slots, block, k_max and max_pages_per_req must be positive")
        check = getattr(engine, "capacity_check", None)
        if check is not None:
            check(slots, block)
        self.engine = engine
        self.slots, self.B, self.k_max = slots, block, min(k_max, block)
        self.page_size = int(kv_pool.shape[4])
        self.max_pages = max_pages_per_req
        self.kv_pool = kv_pool
        self.free = list(free_pages)
        self.mask_token = int(mask_token)
        self.row_budget = slots * block if row_budget is None else int(row_budget)
        if self.row_budget < block:
            raise ValueError("row_budget must admit at least one dense step (B rows)")
        self.keep_pages = keep_pages
        dev = kv_pool.device
        self.tokens = torch.full((slots, block), self.mask_token, dtype=torch.int32, device=dev)
        self.mask = torch.zeros(slots, block, dtype=torch.uint8, device=dev)
        self.prefix_len = torch.zeros(slots, dtype=torch.int32, device=dev)
        self.page_table = torch.full((slots, max_pages_per_req), -1, dtype=torch.int32, device=dev)
        self.ibc = torch.zeros(slots, n_layers, 2, n_kv_heads, block, head_dim, dtype=kv_pool.dtype, device=dev)
        self.waiting: List[Request] = []
        self.slot_req: List[dict] = []               # per active slot: the request's host-side record
        self.results: Dict[int, RequestResult] = {}
        self.stats: List[IterationStats] = []
        self.iteration = 0

    # ---- requests -------------------------------------------------------------------------------
    def submit(self, req: Request) -> None:
        S = self.page_size
        if req.n_blocks < 1 or req.prompt_len < 0:
            raise ValueError(f"request {req.rid}: needs n_blocks >= 1 and prompt_len >= 0")
        if len(req.prompt_pages) != -(-req.prompt_len // S):
            raise ValueError(f"request {req.rid}: {len(req.prompt_pages)} prompt pages for {req.prompt_len} tokens")
        if -(-(req.prompt_len + req.n_blocks * self.B) // S) > self.max_pages:
            raise ValueError(f"request {req.rid}: prompt plus {req.n_blocks} blocks exceed the page table")
        self.waiting.append(req)
        self.waiting.sort(key=lambda r: (r.arrival, r.rid))

    def _pages_needed(self, rec: dict) -> int:
        """Pages to add so that positions up to prefix + B are mapped."""
        return max(0, -(-(rec["prefix_len"] + self.B) // self.page_size) - len(rec["pages"]))

    def _pages_for_request(self, req: Request) -> int:
        """Pages a request needs beyond its prompt pages to hold all its blocks."""
        return max(0, -(-(req.prompt_len + req.n_blocks * self.B) // self.page_size) - len(req.prompt_pages))

    def _cost(self, rec: dict) -> int:
        return self.k_max if rec["phase"] == _FOCUSED else self.B

    def _write_slot(self, i: int, rec: dict) -> None:
        self.tokens[i].fill_(self.mask_token)
        self.mask[i].fill_(1)
        self.prefix_len[i] = rec["prefix_len"]
        row = torch.full((self.max_pages,), -1, dtype=torch.int32)
        row[: len(rec["pages"])] = torch.tensor(rec["pages"], dtype=torch.int32)
        self.page_table[i].copy_(row)

    def _start_block(self, rec: dict) -> None:
        need = self._pages_needed(rec)  # taken from the pages reserved at admission
        rec["pages"].extend(rec["reserved"][:need])
        del rec["reserved"][:need]
        rec["phase"] = _DENSE_FIRST
        rec["block_steps"] = 0

    def _admit(self) -> None:
        while self.waiting and self.waiting[0].arrival <= self.iteration and len(self.slot_req) < self.slots:
            req = self.waiting[0]
            cost = sum(self._cost(r) for r in self.slot_req)
            need = self._pages_for_request(req)
            if cost + self.B > self.row_budget or need > len(self.free):
                break  # first come, first served: nobody overtakes the head of the queue
            self.waiting.pop(0)
            # every page the request will need is reserved now, so no request stalls mid-flight
            rec = {"req": req, "prefix_len": req.prompt_len, "pages": list(req.prompt_pages), "blocks": [],
                   "steps": [], "admitted": self.iteration, "reserved": self.free[:need]}
            del self.free[:need]
            self._start_block(rec)
            self.slot_req.append(rec)
            self._write_slot(len(self.slot_req) - 1, rec)

    # ---- slot moves -----------------------------------------------------------------------------
    def _swap(self, i: int, j: int) -> None:
        if i == j:
            return
        idx, rev = torch.tensor([i, j], device=self.tokens.device), torch.tensor([j, i], device=self.tokens.device)
        for t in (self.tokens, self.mask, self.prefix_len, self.page_table, self.ibc):
            t[idx] = t[rev]
        self.slot_req[i], self.slot_req[j] = self.slot_req[j], self.slot_req[i]

    def _partition(self) -> int:
        """Order the active slots as [focused | dense]; returns the number of focused ones."""
        n = len(self.slot_req)
        lo, hi = 0, n - 1
        while True:
            while lo < n and self.slot_req[lo]["phase"] == _FOCUSED:
                lo += 1
            while hi >= 0 and self.slot_req[hi]["phase"] != _FOCUSED:
                hi -= 1
            if lo >= hi:
                return lo
            self._swap(lo, hi)

    def _order_dense(self, start: int) -> None:
        """Sort the dense slots [start, n) by admission (oldest first), so the ones that fit come first."""
        n = len(self.slot_req)
        key = lambda i: (self.slot_req[i]["admitted"], self.slot_req[i]["req"].rid)
        for i in range(start, n):  # selection sort through slot swaps (a handful of slots)
            j = min(range(i, n), key=key)
            self._swap(i, j)

    def _view(self, a: int, b: int) -> Dict[str, torch.Tensor]:
        return {"block_tokens": self.tokens[a:b], "mask": self.mask[a:b], "prefix_len": self.prefix_len[a:b],
                "page_table": self.page_table[a:b], "kv_pool": self.kv_pool, "ibc": self.ibc[a:b]}

    # ---- the loop -------------------------------------------------------------------------------
    def done(self) -> bool:
        return not self.waiting and not self.slot_req

    def iterate(self) -> IterationStats:
        """Admit, run the focused and the dense steps, move every request to its next phase, commit the
        blocks whose refresh ran, retire finished requests."""
        self._admit()
        n_active = len(self.slot_req)
        n_f = self._partition()
        self._order_dense(n_f)
        fit = (self.row_budget - n_f * self.k_max) // self.B
        n = n_f + max(0, min(n_active - n_f, fit))     # slots [0, n) run; dense slots beyond wait
        cost = n_f * self.k_max + (n - n_f) * self.B
        if n_f > 0:
            self.engine.step(self._view(0, n_f), dense=False)
        if n > n_f:
            self.engine.step(self._view(n_f, n), dense=True)
        masked = self.mask[:n].to("cpu").bool().any(dim=1).tolist() if n else []
        committed = 0
        finished = []
        for i, rec in enumerate(self.slot_req[:n]):
            rec["block_steps"] += 1 if rec["phase"] != _DENSE_REFRESH else 0
            if rec["phase"] == _DENSE_REFRESH:
                self.engine.commit(self._view(i, i + 1))
                committed += 1
                rec["blocks"].append(self.tokens[i].to("cpu").clone())
                rec["steps"].append(rec["block_steps"])
                rec["prefix_len"] += self.B
                if len(rec["blocks"]) < rec["req"].n_blocks:
                    self._start_block(rec)
                    self._write_slot(i, rec)
                else:
                    finished.append(i)
            elif masked[i]:
                if rec["block_steps"] >= self.B:  # as focus_decode_block: at most B decoding steps a block
                    raise RuntimeError(f"request {rec['req'].rid}: block not decoded within {self.B} steps")
                rec["phase"] = _FOCUSED
            else:
                rec["phase"] = _DENSE_REFRESH
        for i in sorted(finished, reverse=True):
            rec = self.slot_req[i]
            self._swap(i, len(self.slot_req) - 1)
            self.slot_req.pop()
            req = rec["req"]
            self.results[req.rid] = RequestResult(req.rid, rec["blocks"], rec["admitted"], self.iteration,
                                                  rec["prefix_len"], list(rec["pages"]), rec["steps"])
            if not self.keep_pages:
                self.free.extend(rec["pages"])
            self.free.extend(rec["reserved"])  # none left once every block is placed
        st = IterationStats(self.iteration, n_active, n_f, n - n_f, cost, committed, n_active - n)
        self.stats.append(st)
        self.iteration += 1
        return st

    def run(self, max_iterations: int = 1 << 20) -> Dict[int, RequestResult]:
        """Iterate until every submitted request has finished."""
        while not self.done():
            if self.iteration >= max_iterations:
                raise RuntimeError("scheduler did not finish within max_iterations")
            self.iterate()
        return self.results
