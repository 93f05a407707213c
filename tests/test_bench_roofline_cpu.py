"""bench.py's roofline bookkeeping (host arithmetic, no GPU): the algorithmic work of each launch and the
whole-step roofline, checked against closed forms written out here from the shapes."""
import dataclasses
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import focus_synth as fs  # noqa: E402


def _case(name="sdar1.7b_n32_b32"):
    s, w = fs.CASES[name]
    return fs.Case(fs.MODEL_SHAPES[s], fs.WORKLOADS[w], model=None, batch=None, seed=0)


def test_step_work_has_every_launch_of_the_step():
    # embedding + norm; per full layer QKV, attention, O, norm, gate/up, down (+ one norm between the two
    # full layers); selection; the gathering norm; per kept layer QKV, attention, O, norm, gate/up, down,
    # norm; LM head; combine + decode; selection and the row map are two launches: 7 L + 6 launches.
    # With more than 256 kept-row slots (N x k_max) each kept-row GEMM and the LM head are two launches
    # (few-row and many-row kernel, one of which exits on the live row count): 4 (L - 2) + 1 more
    for name, few in (("sdar1.7b_n32_b32", True), ("sdar8b_n256_b64", False), ("small_bf16", True),
                      ("sdar1.7b_n128_b32", False)):
        case = _case(name)
        N, L = case.work.n_requests, case.shape.n_layers
        assert (N * case.work.k_max <= 256) == few
        work = bench.step_work(case, R=N, kept_per_req=[1] * N, plen=[64] * N)
        assert sum(n for _, n, _, _ in work) == 7 * L + 6 + (0 if few else 4 * (L - 2) + 1)


def test_kept_row_gemm_bytes_are_the_weights_plus_rows():
    case = _case()
    s = case.shape
    R = 32
    by, fl = bench.algorithmic_work("gemm_gateup", case, R, [1] * 32, [512] * 32)
    weights = 2 * s.ffn * s.hidden * 2
    assert by == weights + R * s.hidden * 2 + R * s.ffn * 2
    assert fl == 2.0 * R * 2 * s.ffn * s.hidden
    by, _ = bench.algorithmic_work("gemm_down", case, R, [1] * 32, [512] * 32)
    assert by == s.hidden * s.ffn * 2 + R * s.ffn * 2 + R * s.hidden * 8  # residual read + written in float32


def test_ragged_attention_bytes_closed_form():
    case = _case()
    s, B = case.shape, case.work.block
    kept = [1, 0, 3, 2]
    plen = [256, 1024, 640, 0]
    case = fs.Case(s, dataclasses.replace(case.work, n_requests=4), None, None, 0)
    by, fl = bench.algorithmic_work("attn_ragged", case, sum(kept), kept, plen)
    kv = sum((p + B) * s.n_kv_heads * s.head_dim * 2 * 2 for p, k in zip(plen, kept) if k)
    qo = sum(k * s.n_q_heads * s.head_dim * 2 * 2 for k in kept)
    assert by == kv + qo
    assert fl == sum(4.0 * k * s.n_q_heads * s.head_dim * (p + B) for p, k in zip(plen, kept))


def test_step_roofline_sums_the_slower_bound_of_each_launch():
    peaks = {"hbm_gbs": 1000.0, "bf16_tflops_sustained": 1000.0}
    # two HBM-bound launches of 1 GB (1 ms each), one tensor-bound launch of 1 TFLOP (1 ms), and one
    # launch whose bytes (0.5 ms) are below its flops (2 ms)
    work = [("a", 2, 1e9, 0.0), ("b", 1, 0.0, 1e12), ("c", 1, 5e8, 2e12)]
    r = bench.step_roofline(work, peaks, ms_per_step=10.0)
    assert abs(r["t_roof_ms"] - 5.0) < 1e-12
    assert abs(r["hbm_bound_ms"] - 2.0) < 1e-12 and abs(r["tensor_bound_ms"] - 3.0) < 1e-12
    assert abs(r["frac"] - 0.5) < 1e-12
    assert abs(r["algorithmic_gb"] - 2.5) < 1e-12 and abs(r["algorithmic_tflop"] - 3.0) < 1e-12


def test_step_roofline_of_the_bench_workload_is_dominated_by_streams():
    # 1.7B shape, 32 requests with one kept row each: the kept layers stream their weights and KV pages,
    # so the step's roofline time is mostly HBM-bound and well below a millisecond and a half
    case = _case()
    N = case.work.n_requests
    work = bench.step_work(case, R=N, kept_per_req=[1] * N, plen=[640] * N)
    peaks = {"hbm_gbs": 6541.8, "bf16_tflops_sustained": 1365.2}
    r = bench.step_roofline(work, peaks, ms_per_step=2.6)
    assert r["hbm_bound_ms"] > r["tensor_bound_ms"]
    assert 0.5 < r["t_roof_ms"] < 1.5
    s = case.shape
    weights = s.n_layers * (s.hidden * (s.n_q_heads + 2 * s.n_kv_heads) * s.head_dim + s.n_q_heads * s.head_dim * s.hidden
                            + 3 * s.hidden * s.ffn) * 2 + s.vocab * s.hidden * 2
    assert r["algorithmic_gb"] * 1e9 > weights  # every weight is read at least once per step


def test_families_sum_their_kernel_classes_and_take_the_slower_bound():
    # the 8B shape with 14 kept rows per request: the kept-row GEMMs are one tensor-bound family, the ragged
    # attention an HBM-bound one
    case = _case("sdar8b_n256_b64")
    N = case.work.n_requests
    work = bench.step_work(case, R=14 * N, kept_per_req=[14] * N, plen=[1280] * N)
    per_class = {kc: (2.0, 34) for kc, _, _, _ in work}
    peaks = {"hbm_gbs": 6541.8, "bf16_tflops_sustained": 1365.2}
    fam = bench.family_rooflines(per_class, work, peaks)
    kept = fam["gemm_kept_rows"]
    assert kept["ms_per_step"] == 8.0 and kept["launches"] == 4 * 34 and kept["bound"] == "tensor"
    fl = sum(n * f for kc, n, _, f in work if kc in ("gemm_qkv", "gemm_o", "gemm_gateup", "gemm_down"))
    assert abs(kept["algorithmic_tflop"] - fl / 1e12) < 1e-3
    assert abs(kept["achieved"] - fl / 8e-3 / 1e12) < 0.1
    assert fam["attention_ragged"]["bound"] == "hbm" and fam["attention_ragged"]["unit"] == "GB/s"


def test_sweep_workload_names_resolve_to_the_sweep_recipe():
    shape, work, seed = bench.resolve_workload("sweep_n256_b64_f1.0")
    assert shape == fs.MODEL_SHAPES["sdar1.7b"] and seed == fs.SEEDS["sweep"]
    assert (work.n_requests, work.block, work.forced_keep_frac, work.prefix) == (256, 64, 1.0, ("uniform", 256, 4096))
    shape, work, seed = bench.resolve_workload("sdar8b_n256_b64")
    assert shape == fs.MODEL_SHAPES["sdar8b"] and work.n_requests == 256 and seed == fs.SEEDS["sdar8b_n256_b64"]
