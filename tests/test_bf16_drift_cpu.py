"""How far a bf16 evaluation of the step may lie from the float64 oracle, shown with an evaluation that
shares nothing with the oracle (CPU only).

The GPU path stores activations in bf16 and accumulates in float32.  Deep random-weight stacks amplify
bf16-level perturbations, so on the 28- and 36-layer shapes the GPU's hidden states and confidences are
compared with the float64 oracle within 2e-2 x RMS plus twice the drift that bf16 storage alone causes
(tests/parity.py).  These tests back that allowance with a second, independently written bf16 evaluation
(tests/dense_reference.py with bf16 storage, float32 accumulation and bf16 probabilities before P.V, the
way tensor-core kernels take them):

  * at depth, the independent evaluation lies about as far from float64 as the oracle's bf16 mode, the
    two bf16 evaluations differ from each other by about that drift (so neither is "the" bf16 answer),
    and 2e-2 x RMS plus twice the drift covers the independent one -- while 2e-2 x RMS alone does not;
  * on a shallow model the strict 2e-2 x RMS bound holds for the independent evaluation with no
    allowance, which is why the GPU tests hold models of at most 4 layers to it.

The deep models keep the reduced width of the CPU-sized shapes but scale the weights so that each layer
has the gain (hidden size x weight variance) of the 1.7B (2048 x 0.02^2) and 8B (4096 x 0.02^2) shapes;
the width-2048 28-layer model itself gives the same picture (drift 4.3 %, independent 4.0 %, cross 5.0 %
of RMS max-abs) but takes minutes on a CPU.
"""
import math

import numpy as np
import pytest
import torch

import focus_synth as fs
from oracle import focus_oracle as fo

from dense_reference import dense_block_forward

STATED = 2e-2  # the stated max-abs bound, relative to the RMS of the float64 values


def _deep_case(n_layers, gain_width, n_kv_heads, seed):
    shape = fs.ModelShape(n_layers, 512, 8, n_kv_heads, 64, 1536, 2000, "bf16")
    work = fs.Workload(2, 16, 16, ("uniform", 32, 200), ("frac", 0.3, 1.0), k_min=1, k_max=16)
    case = fs.make_case(shape=shape, work=work, seed=seed)
    scale = math.sqrt(gain_width / shape.hidden)   # weight std 0.02 * scale: D * std^2 = gain_width * 0.02^2
    for key in ("wqkv", "wo", "wgate", "wup", "wdown"):
        case.model[key] = [(w.float() * scale).to(torch.bfloat16) for w in case.model[key]]
    return case


def _evaluations(case):
    B = case.work.block
    kw = dict(tau=0.0, k_min=1, k_max=B, conf_threshold=0.9, forced_keep_frac=1.0)
    f64 = fo.focus_step(case.shape, case.model, case.batch, **kw)
    ora_bf16 = fo.focus_step(case.shape, case.model, case.batch, storage="bf16", **kw)
    ind = dense_block_forward(case.shape, case.model, case.batch, storage="bf16", accum="f32", round_probs=True)
    N = case.work.n_requests
    z = ind["logits"].reshape(N * B, -1).numpy()
    ind_conf = 1.0 / np.exp(z - z.max(1, keepdims=True)).sum(1)
    return f64, ora_bf16, ind["hidden"].reshape(N * B, -1).numpy(), ind_conf, z


def _rel(a, b, scale):
    return float(np.abs(a - b).max()) / scale, float(np.sqrt(np.mean((a - b) ** 2))) / scale


@pytest.mark.parametrize("n_layers,gain_width,n_kv_heads,seed", [(28, 2048, 4, 77), (36, 4096, 2, 77)])
def test_two_bf16_evaluations_differ_from_float64_by_the_same_drift(n_layers, gain_width, n_kv_heads, seed):
    case = _deep_case(n_layers, gain_width, n_kv_heads, seed)
    f64, ora_bf16, ind_hidden, ind_conf, _ = _evaluations(case)
    rms = float(np.sqrt(np.mean(f64.hidden ** 2)))
    drift, drift_rms = _rel(ora_bf16.hidden, f64.hidden, rms)
    indep, indep_rms = _rel(ind_hidden, f64.hidden, rms)
    cross, _ = _rel(ind_hidden, ora_bf16.hidden, rms)
    # bf16 storage alone already exceeds the stated bound at this depth ...
    assert drift > STATED, f"drift {drift:.4f}"
    assert indep > STATED, f"independent {indep:.4f}"
    # ... an independent bf16 evaluation is about as far away, and about that far from the oracle's bf16 mode
    assert 0.5 * drift <= indep <= 2.0 * drift, (indep, drift)
    assert cross >= 0.5 * drift, (cross, drift)
    # the allowance the GPU tests use covers it, for the max-abs and the RMS of the error
    assert indep <= STATED + 2.0 * drift
    assert indep_rms <= STATED + 2.0 * drift_rms
    # likewise for the confidences
    crms = float(np.sqrt(np.mean(f64.conf.reshape(-1) ** 2)))
    c_drift, c_drift_rms = _rel(ora_bf16.conf.reshape(-1), f64.conf.reshape(-1), crms)
    c_ind, c_ind_rms = _rel(ind_conf, f64.conf.reshape(-1), crms)
    assert c_ind <= STATED + 2.0 * c_drift and c_ind_rms <= STATED + 2.0 * c_drift_rms


def test_shallow_model_meets_the_stated_bound_without_allowance():
    """The reduced bf16 shape (4 layers, hidden 512): an independent bf16 evaluation is within 2e-2 x RMS of
    float64 in hidden states, importance, cache entries and confidences, with no allowance."""
    case = fs.make_case("small_bf16")
    f64, _, ind_hidden, ind_conf, _ = _evaluations(case)
    ind = dense_block_forward(case.shape, case.model, case.batch, storage="bf16", accum="f32", round_probs=True)
    for name, got, want in (("hidden", ind_hidden, f64.hidden), ("conf", ind_conf, f64.conf.reshape(-1)),
                            ("importance", ind["colsum"].numpy(), f64.importance),
                            ("ibc", ind["kv"].numpy(), f64.ibc)):
        scale = float(np.sqrt(np.mean(want ** 2)))
        err, _ = _rel(got, want, scale)
        assert err <= STATED, f"{name}: {err:.4f} of RMS"


@pytest.mark.parametrize("name", ["small_bf16", "small_bf16_g4"])
def test_a_one_in_a_thousand_logit_gate_is_finer_than_bf16_resolves(name):
    """Decoded ids are compared at a logit gate derived from the hidden-state tolerance (2e-2 x sqrt(D) x
    RMS(W_lm), about 9e-3 here), not at 1e-3: on the reduced shallow shapes an independent bf16 evaluation
    already moves logits by more than twice 1e-3 -- enough to swap two logits 1e-3 apart -- and the top
    logit of more than a tenth of the rows by more than 1e-3, while staying inside the derived gate."""
    case = fs.make_case(name)
    N, B = case.work.n_requests, case.work.block
    z64 = dense_block_forward(case.shape, case.model, case.batch)["logits"].reshape(N * B, -1).numpy()
    _, _, _, _, z = _evaluations(case)
    dz = np.abs(z - z64)
    top = z64.argmax(1)
    top_err = dz[np.arange(len(top)), top]
    gate = STATED * math.sqrt(case.shape.hidden) * float(case.model["lm_head"].float().pow(2).mean().sqrt())
    assert dz.max() > 2e-3, dz.max()
    assert (top_err > 1e-3).mean() > 0.1, (top_err > 1e-3).mean()
    assert dz.max() < gate, (dz.max(), gate)
