"""The allocation-free LM-head confidence entry point against focus_step's own confidences.

focus_lm_head_conf_noalloc serves callers that may not allocate device memory (a thread recording a
CUDA graph, a fixed-budget serving loop, a plug-in inside a framework that owns the device memory).
It keeps its intermediate data in a fixed array inside the library, shared by every call.  This test
calls it through the C ABI twice in a row -- all kept rows, then a shorter prefix of them, so stale
contents of the shared array would show -- and checks both results against the conf / top id that
focus_step computed for the same rows, and the first one also against the float64 oracle's final norm,
LM head and max-softmax on those rows.  This file is collected last on purpose.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import focus_synth as fs

pytestmark = pytest.mark.gpu


def _p(t):
    return C.c_void_p(t.data_ptr())


def test_lm_head_conf_without_allocation_matches_focus_step():
    from decodability_aware_token_b200 import FocusContext, StepParams, _abi
    lib = _abi.load()
    case = fs.make_case("small_bf16")
    w, shp = case.work, case.shape
    dev = torch.device("cuda:0")
    model = {k: ([t.to(dev) for t in v] if isinstance(v, list) else v.to(dev)) for k, v in case.model.items()}
    batch = {k: v.to(dev).clone() for k, v in case.batch.items()}
    with FocusContext(shp, model, max_requests=w.n_requests, max_block=w.block, max_keep=w.k_max,
                      max_pages_per_req=case.max_pages_per_req) as ctx:
        out = ctx.step(batch, StepParams(w.tau, w.k_min, w.k_max, w.conf_threshold))
        torch.cuda.synchronize()
    kc = out.keep_count.cpu().tolist()
    R = int(out.row_offsets[-1])
    assert R > 1
    hidden = out.hidden[:R].contiguous()
    ref_conf = torch.cat([out.conf[b, : kc[b]] for b in range(len(kc))]).cpu().numpy()
    ref_top = torch.cat([out.top_id[b, : kc[b]] for b in range(len(kc))]).cpu().numpy()

    conf = torch.full((R,), -1.0, dtype=torch.float32, device=dev)
    top = torch.full((R,), -7, dtype=torch.int32, device=dev)
    stream = C.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    frac = 2e-2   # the bf16 tolerance of the parity tests: max-abs <= frac x RMS
    first = None
    for rows in (R, max(1, R // 2)):
        conf.fill_(-1.0)
        top.fill_(-7)
        rc = lib.focus_lm_head_conf_noalloc(_p(hidden), rows, shp.hidden, _p(model["final_norm"]),
                                            _p(model["lm_head"]), shp.vocab, shp.rms_eps, _p(conf), _p(top), stream)
        assert rc == _abi.FOCUS_OK, rc
        torch.cuda.synchronize()
        got_c, got_t = conf.cpu().numpy(), top.cpu().numpy()
        want = ref_conf[:rows]
        assert np.all(np.isfinite(got_c[:rows]))
        assert np.abs(got_c[:rows] - want).max() <= frac * np.sqrt(np.mean(want ** 2))
        np.testing.assert_array_equal(got_t[:rows], ref_top[:rows])
        assert np.all(got_c[rows:] == -1.0) and np.all(got_t[rows:] == -7)   # nothing written past `rows`
        if first is None:
            first = (got_c.copy(), got_t.copy())

    # the first call against the oracle (float64 norm, logits, max-softmax, lowest id among the maxima):
    # confidences within 2e-2 x RMS, top ids equal wherever the oracle's top-1 margin exceeds the logit
    # error that tolerance allows (2e-2 x sqrt(D) x RMS of the LM-head weights), else within it
    from oracle import focus_oracle as fo
    h64 = hidden.cpu().double().numpy()
    g64, w64 = fo._f64(case.model["final_norm"]), fo._f64(case.model["lm_head"])
    c64, t64, _, margin = fo.lm_head_conf(h64, g64, w64, shp.rms_eps)
    got_c, got_t = first
    assert np.abs(got_c - c64).max() <= frac * np.sqrt(np.mean(c64 ** 2))
    gate = frac * np.sqrt(shp.hidden) * float(np.sqrt(np.mean(w64 ** 2)))
    z = fo.rms_norm(h64, g64, shp.rms_eps) @ w64.T
    for r in range(R):
        if got_t[r] != t64[r]:
            assert margin[r] <= gate and z[r, t64[r]] - z[r, got_t[r]] <= gate, (r, got_t[r], t64[r], margin[r])

    # sizes beyond the fixed array are refused before anything is launched
    rc = lib.focus_lm_head_conf_noalloc(_p(hidden), 257, shp.hidden, _p(model["final_norm"]), _p(model["lm_head"]),
                                        shp.vocab, shp.rms_eps, _p(conf), _p(top), stream)
    assert rc == _abi.FOCUS_ERR_LIMITS
