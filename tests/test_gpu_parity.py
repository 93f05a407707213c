"""GPU parity: the CUDA focused step (through the C ABI) against the CPU oracle.

Small cases span several GEMM / attention tiles and ragged tails; the full-size workloads are
checked on sampled requests (requests are independent, so the oracle can run a subset).
"""
import dataclasses
import gc

import pytest
import torch

import focus_synth as fs
from gpu_harness import check, run_gpu, run_oracle, step_params, to_device, limits_for

pytestmark = pytest.mark.gpu

_models = {}


def _case(name, **kw):
    return fs.make_case(name, **kw)


def _model(name, case):
    if name not in _models:
        _models.clear()
        _models[name] = to_device(case)
    return _models[name]


@pytest.mark.parametrize("name", ["tiny", "small_f32", "small_bf16", "small_bf16_g4"])
def test_adaptive_step_matches_oracle(name):
    case = _case(name)
    rep = check(case, step_params(case.work), _model(name, case))
    print(name, rep)


@pytest.mark.parametrize("name", ["tiny", "small_bf16"])
@pytest.mark.parametrize("frac", [1.0, 0.25])
def test_forced_fraction_matches_oracle(name, frac):
    """Keep fraction 1 is the dense full-block step (the oracle's f = 1 is pinned to a dense forward)."""
    case = _case(name)
    check(case, step_params(case.work, forced_keep_frac=frac), _model(name, case))


@pytest.mark.parametrize("name,frac,boost", [("tiny", 0.02, 60.0), ("small_bf16", 0.001, 25.0)])
def test_confidence_threshold_path(name, frac, boost):
    """LM-head rows of a few vocabulary entries scaled up so that some confidences clear the threshold.

    The boost multiplies those logits, and with them the logit error of bf16 operands; a few rows at
    25x keep the confidence error inside the bf16 tolerance while pushing most confidences past 0.9."""
    case = _case(name, lm_boost_frac=frac, lm_boost=boost)
    p = step_params(case.work)
    gpu = run_gpu(case, p)
    conf = gpu["conf"][gpu["conf"] > 0]
    assert (conf > p["conf_threshold"]).any(), "the variant should exercise the threshold"
    check(case, p, gpu=gpu)


@pytest.mark.parametrize("name", ["small_f32", "small_bf16"])
def test_alpha_tau_kmin_variants(name):
    case = _case(name)
    m = _model(name, case)
    check(case, step_params(case.work, alpha=1.5, tau=0.002, k_min=3, k_max=case.work.k_max), m)
    check(case, step_params(case.work, alpha=0.5, tau=-0.01, k_min=0, k_max=case.work.k_max), m)


@pytest.mark.parametrize("frac", [-1.0, 1.0])
def test_many_row_gemms_match_oracle(frac):
    """Hidden 2048, 41 requests of block 64: the 2624 block rows (a ragged last 128-row tile) give the
    layers-0-1 GEMMs enough tiles for the persistent kernel, with 256-wide tiles for some GEMMs and 128-wide
    for others.  Adaptive: the kept rows (up to 656) run on the one-tile-per-CTA kernel; keep fraction 1:
    the last layer's 2624 kept rows run on the persistent kernel too."""
    case = _case("wide_bf16")
    check(case, step_params(case.work, forced_keep_frac=frac), _model("wide_bf16", case))


def _with_batch(case, **fields):
    b = dict(case.batch)
    b.update(fields)
    return fs.Case(case.shape, case.work, case.model, b, case.seed)


@pytest.mark.parametrize("name", ["tiny", "small_bf16"])
def test_edge_no_prefix(name):
    case = _case(name)
    N = case.work.n_requests
    c2 = _with_batch(case, prefix_len=torch.zeros(N, dtype=torch.int32))
    check(c2, step_params(case.work), _model(name, case))


@pytest.mark.parametrize("name", ["tiny", "small_bf16"])
def test_edge_nothing_masked_keeps_nothing(name):
    case = _case(name)
    c2 = _with_batch(case, mask=torch.zeros_like(case.batch["mask"]))
    gpu = run_gpu(c2, step_params(case.work), _model(name, case))
    assert int(gpu["keep_count"].sum()) == 0 and bool((gpu["decoded_ids"] == -1).all())
    check(c2, step_params(case.work), gpu=gpu)


@pytest.mark.parametrize("name", ["tiny", "small_bf16"])
def test_edge_everything_masked(name):
    case = _case(name)
    tok = case.batch["block_tokens"].clone()
    tok[:] = case.shape.vocab - 1
    c2 = _with_batch(case, mask=torch.ones_like(case.batch["mask"]), block_tokens=tok)
    check(c2, step_params(case.work), _model(name, case))


def test_edge_single_request_full_block_budget():
    """N = 1, k_max = B: every masked position may be kept."""
    case = _case("small_bf16")
    w = dataclasses.replace(case.work, n_requests=1)
    c2 = fs.Case(case.shape, w, case.model, {k: (v[:1] if k != "kv_pool" else v) for k, v in case.batch.items()},
                 case.seed)
    check(c2, step_params(w, k_max=w.block, k_min=w.block), _model("small_bf16", case))


def test_caller_forced_set_is_honoured():
    case = _case("small_bf16")
    p = step_params(case.work)
    forced = [[0, 5, 31], [], [1, 2, 3, 4, 6, 7, 8, 9], [30], [10, 20]]
    gpu = run_gpu(case, p, _model("small_bf16", case), forced=forced)
    for b, s in enumerate(forced):
        assert gpu["retained_idx"][b, : gpu["keep_count"][b]].tolist() == s
    import parity
    # a 4-layer model: the plain float64 oracle, no allowance
    ora = run_oracle(case, p, forced=forced, max_keep=p["k_max"])
    rep, fl = parity.compare(case, p, ora, gpu, parity.tolerance(case.shape), case.batch["ibc"],
                             check_selection=False)
    assert not fl


def test_bad_page_id_sets_device_error_and_does_not_fault():
    case = _case("tiny")
    table = case.batch["page_table"].clone()
    table[0, 1] = 10_000                                  # no such page: the kernel skips it and flags it
    c2 = _with_batch(case, page_table=table)
    gpu = run_gpu(c2, step_params(case.work), _model("tiny", case))
    from decodability_aware_token_b200 import _abi
    assert gpu["device_status"] == _abi.FOCUS_ERR_DEVICE_BOUNDS
    assert gpu["device_bits"] & _abi.FOCUS_DEVERR_PAGE_ID


def test_prefix_beyond_page_table_is_clamped_and_flagged():
    case = _case("tiny")
    plen = case.batch["prefix_len"].clone()
    plen[1] = 10_000
    gpu = run_gpu(_with_batch(case, prefix_len=plen), step_params(case.work), _model("tiny", case))
    from decodability_aware_token_b200 import _abi
    assert gpu["device_bits"] & _abi.FOCUS_DEVERR_PREFIX


def test_bounded_wait_expires_with_a_timeout_status_and_the_context_stays_usable():
    """Failure detection without a fault: a pipeline wait that nothing satisfies gives up after about a
    second, the error word says so, and the same context then runs a clean step."""
    from decodability_aware_token_b200 import FocusContext, _abi
    case = _case("tiny")
    m = _model("tiny", case)
    p = step_params(case.work)
    lim = limits_for(case, p)
    batch = {k: v.cuda().clone() for k, v in case.batch.items()}
    with FocusContext(case.shape, m, **lim) as ctx:
        ctx.probe_wait_timeout()
        rc, bits = ctx.device_error()
        assert rc == _abi.FOCUS_ERR_TIMEOUT and bits & _abi.FOCUS_DEVERR_TIMEOUT
        from decodability_aware_token_b200 import StepParams
        ctx.step(batch, StepParams(**p))
        rc, bits = ctx.device_error()
        assert rc == _abi.FOCUS_OK and bits == 0


def test_host_validation_rejects_bad_arguments():
    from decodability_aware_token_b200 import FocusContext, StepParams, FocusError, _abi
    case = _case("tiny")
    m = _model("tiny", case)
    lim = limits_for(case, step_params(case.work))
    batch = {k: v.cuda() for k, v in case.batch.items()}
    with FocusContext(case.shape, m, **lim) as ctx:
        with pytest.raises(FocusError) as e:
            ctx.step(batch, StepParams(k_min=1, k_max=case.work.block + 1))
        assert e.value.code in (_abi.FOCUS_ERR_INVALID_ARG, _abi.FOCUS_ERR_LIMITS)
        with pytest.raises(FocusError) as e:
            ctx.step(batch, StepParams(k_min=1, k_max=lim["max_keep"] + 1 if lim["max_keep"] < case.work.block else 99))
        with pytest.raises(FocusError) as e:
            ctx.step(batch, StepParams(k_min=5, k_max=2))
        assert e.value.code == _abi.FOCUS_ERR_INVALID_ARG


def test_step_is_deterministic():
    case = _case("small_bf16")
    p = step_params(case.work)
    m = _model("small_bf16", case)
    a, b = run_gpu(case, p, m), run_gpu(case, p, m)
    for k in ("importance", "keep_count", "retained_idx", "hidden", "conf", "top_id", "decoded_ids"):
        assert torch.equal(a[k], b[k]), k
    assert torch.equal(a["ibc"], b["ibc"])


def test_step_replays_from_cuda_graph():
    """focus_step makes no host synchronisation: a captured step replays with the eager step's results."""
    from decodability_aware_token_b200 import FocusContext, StepParams
    case = _case("small_bf16")
    w = case.work
    m = _model("small_bf16", case)
    lim = limits_for(case, step_params(w))
    dev = torch.device("cuda:0")
    batch = {k: v.to(dev).clone() for k, v in case.batch.items()}
    tok0, mask0 = batch["block_tokens"].clone(), batch["mask"].clone()
    p = StepParams(w.tau, w.k_min, w.k_max, w.conf_threshold)
    with FocusContext(case.shape, m, **lim) as ctx:
        eager = ctx.step(batch, p)
        torch.cuda.synchronize()
        ref = {k: v.clone() for k, v in eager.tensors().items() if v is not None}
        ref_ibc = batch["ibc"].clone()
        out = ctx.alloc_outputs(w.n_requests, w.block)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            batch["block_tokens"].copy_(tok0)
            batch["mask"].copy_(mask0)
            ctx.step(batch, p, out)
        for _ in range(2):
            g.replay()
            torch.cuda.synchronize()
            for k, v in ref.items():
                assert torch.equal(getattr(out, k), v), k
            assert torch.equal(batch["ibc"], ref_ibc)
        rc, bits = ctx.device_error()
        assert rc == 0, bits


# ---------------------------------------------------------------- full-size workloads, sampled requests
@pytest.fixture
def free_device_memory():
    """The full-size cases hold tens of GB on the device: release them before and after each test."""
    _models.clear()
    gc.collect()
    torch.cuda.empty_cache()
    yield
    gc.collect()
    torch.cuda.empty_cache()


def pick_requests(case, gpu, params, n):
    """Requests worth the oracle's time at full size, chosen rather than drawn: the longest and the shortest
    prefix, a prefix that ends inside a page, a request that kept more than k_min, the tightest cut of the
    GPU's own deltas, the first and the last request; seeded others fill up to n."""
    N, B, S = case.work.n_requests, case.work.block, case.work.page_size
    plen = case.batch["prefix_len"].cpu().long()
    kc = gpu["keep_count"].long()
    mask = case.batch["mask"].cpu().bool()
    delta = (gpu["importance"][1] - gpu["importance"][0]).double()
    picks = [int(torch.argmax(plen)), int(torch.argmin(plen))]
    ragged = [b for b in range(N) if int(plen[b]) % S]
    picks += ragged[:1]
    more = [b for b in range(N) if int(kc[b]) > params["k_min"]]
    picks += more[:1]
    gaps = []
    for b in range(N):
        elig = [j for j in range(B) if mask[b, j]] if params["forced_keep_frac"] < 0 else list(range(B))
        d = sorted((float(delta[b, j]) for j in elig), reverse=True)
        k = int(kc[b])
        if 0 < k < len(d):
            gaps.append((d[k - 1] - d[k], b))
    if gaps:
        picks.append(min(gaps)[1])
    picks += [0, N - 1]
    picks += torch.randperm(N, generator=torch.Generator().manual_seed(17)).tolist()
    order = list(dict.fromkeys(picks))   # first occurrence wins: the chosen ones, then the seeded fill
    return sorted(order[:n])


def _sampled_check(case, n_requests=8, params=None):
    """Full-size case on the GPU (model, pages and cache stay on the device); the oracle runs only the
    chosen requests (requests are independent) and reads their pages from the device.  The case's device
    tensors are released on the way out, pass or fail (a failure's traceback would keep them alive)."""
    p = params or step_params(case.work)
    host_batch = {}
    try:
        gpu = run_gpu(case, p, case.model)
        host_batch.update({k: (v if k == "kv_pool" else v.cpu()) for k, v in case.batch.items()})
        host = fs.Case(case.shape, case.work, case.model, host_batch, case.seed)
        reqs = pick_requests(host, gpu, p, n_requests)
        rep = check(host, p, requests=reqs, gpu=gpu)
        rep["checked"] = reqs
        return rep
    finally:
        host_batch.clear()
        case.batch.clear()
        case.model.clear()


@pytest.mark.slow
@pytest.mark.usefixtures("free_device_memory")
def test_sdar_1p7b_n32_b32_sampled():
    # the 1.7B shape, 32 requests with prefixes U[256, 1024], block 32, k_max 8
    case = fs.make_case("sdar1.7b_n32_b32", device="cuda:0")
    rep = _sampled_check(case)
    del case
    print(rep)


@pytest.mark.slow
@pytest.mark.usefixtures("free_device_memory")
def test_sdar_1p7b_n128_lognormal_sampled():
    # 128 ragged requests, prefixes log-normal (median 600, clipped to 64..4096), k_max 12
    case = fs.make_case("sdar1.7b_n128_b32", device="cuda:0")
    rep = _sampled_check(case)
    del case
    print(rep)


@pytest.mark.slow
@pytest.mark.usefixtures("free_device_memory")
def test_sdar_8b_n256_b64_sampled():
    # 8B shape (hidden 4096, 32 / 8 heads: four query heads per KV head), block 64, k_max 16: the kept rows
    # (several thousand) run on the row-major tensor-core GEMMs
    case = fs.make_case("sdar8b_n256_b64", device="cuda:0")
    rep = _sampled_check(case)
    del case
    print(rep)


@pytest.mark.slow
@pytest.mark.usefixtures("free_device_memory")
@pytest.mark.parametrize("n,block,frac", [(32, 16, 0.25), (64, 64, 0.5), (128, 32, 0.1), (256, 64, 1.0)])
def test_kernel_sweep_points_sampled(n, block, frac):
    """Sweep points on the 1.7B shape with a forced keep fraction (prefixes U[256, 4096]): every batch size
    32 / 64 / 128 / 256 and block size 16 / 32 / 64 once.  Keep fraction 1 at 256 x 64 is the dense
    full-block step at full size (the oracle's f = 1 is pinned to an independent dense forward)."""
    case = fs.make_case("sweep", seed=fs.SEEDS["sweep"], device="cuda:0", shape=fs.MODEL_SHAPES["sdar1.7b"],
                        work=fs.sweep_workload(n, block, frac))
    rep = _sampled_check(case, n_requests=3)
    if frac == 1.0:
        assert rep["decisions_vs_f64"]["kept_equal"] == len(rep["checked"])
    del case
    print(rep)


# ---------------------------------------------------------------- budget / decode variants
@pytest.mark.parametrize("alpha", [1.2, 1.5, 1.8])
@pytest.mark.parametrize("threshold", [0.7, 0.8, 0.9])
def test_quality_table_knobs(alpha, threshold):
    """The knobs of the project page's Quality table: the budget multiplier alpha (1.2 / 1.5 / 1.8) and the
    confidence threshold "Conf." (0.7 / 0.8 / 0.9), with boosted LM-head rows so that the threshold
    decides (bf16 shape, several tiles)."""
    case = _case("small_bf16", lm_boost_frac=0.001, lm_boost=25.0)
    p = step_params(case.work, alpha=alpha, conf_threshold=threshold)
    gpu = run_gpu(case, p)
    check(case, p, gpu=gpu)


@pytest.mark.parametrize("block", [16, 64])
def test_other_block_sizes(block):
    """Block sizes 16 and 64 on the reduced bf16 shape (the project page's efficiency figures use several)."""
    case = _case("small_bf16", block=block, k_max=min(8, block))
    check(case, step_params(case.work), _model("small_bf16_b%d" % block, case))
