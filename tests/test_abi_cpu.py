"""The C-ABI library loads and exports every symbol include/focus.h declares; host-only checks (no GPU)."""
import ctypes as C
import os
import re

import pytest

from decodability_aware_token_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "focus.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(focus_\w+)\s*\(", src, flags=re.M)))


def test_header_declarations_match_binding():
    assert _declared() == sorted(_abi.EXPORTED)


def test_library_exports_every_declared_symbol():
    lib = _abi.load()
    for name in _declared():
        assert hasattr(lib, name), name


def test_status_strings():
    lib = _abi.load()
    codes = [0, -1, -2, -3, -4, -5, -6, -7]
    strs = [lib.focus_status_string(c).decode() for c in codes]
    assert len(set(strs)) == len(codes) and all(strs)
    assert lib.focus_status_string(-99).decode() == "unknown status"


def _cfg(**over):
    base = dict(n_layers=4, hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64, ffn=1024, vocab=1000, rms_eps=1e-6,
                rope_theta=1e4, dtype=_abi.FOCUS_DTYPE_F32)
    base.update(over)
    return _abi.ModelCfg(**base)


def test_workspace_bytes_and_argument_checks():
    lib = _abi.load()
    lim = _abi.Limits(8, 32, 8, 16)
    n1 = lib.focus_workspace_bytes(C.byref(_cfg()), C.byref(lim))
    n2 = lib.focus_workspace_bytes(C.byref(_cfg()), C.byref(_abi.Limits(16, 32, 8, 16)))
    assert 0 < n1 < n2
    assert lib.focus_workspace_bytes(C.byref(_cfg(n_layers=1)), C.byref(lim)) == 0
    assert lib.focus_workspace_bytes(C.byref(_cfg()), C.byref(_abi.Limits(8, 65, 8, 16))) == 0
    assert lib.focus_workspace_bytes(C.byref(_cfg()), C.byref(_abi.Limits(8, 32, 33, 16))) == 0


@pytest.mark.parametrize("over,code", [
    (dict(n_layers=1), _abi.FOCUS_ERR_INVALID_ARG),
    (dict(n_q_heads=3), _abi.FOCUS_ERR_INVALID_ARG),
    (dict(head_dim=96), _abi.FOCUS_ERR_UNSUPPORTED),
    (dict(head_dim=64, dtype=_abi.FOCUS_DTYPE_BF16), _abi.FOCUS_ERR_UNSUPPORTED),
    (dict(hidden=200), _abi.FOCUS_ERR_UNSUPPORTED),
    (dict(dtype=7), _abi.FOCUS_ERR_INVALID_ARG),
])
def test_init_rejects_bad_models_before_touching_the_device(over, code):
    lib = _abi.load()
    ctx = C.c_void_p(1)
    w = _abi.Weights()
    rc = lib.focus_init(C.byref(_cfg(**over)), C.byref(w), C.byref(_abi.Limits(8, 32, 8, 16)), C.byref(ctx))
    assert rc == code and not ctx.value


def test_init_rejects_missing_weights():
    lib = _abi.load()
    ctx = C.c_void_p()
    assert lib.focus_init(C.byref(_cfg()), C.byref(_abi.Weights()), C.byref(_abi.Limits(8, 32, 8, 16)),
                          C.byref(ctx)) == _abi.FOCUS_ERR_INVALID_ARG
    assert lib.focus_init(None, None, None, None) == _abi.FOCUS_ERR_INVALID_ARG


def test_null_handles_are_safe():
    lib = _abi.load()
    assert lib.focus_destroy(None) == 0
    assert lib.focus_get_device_error(None, None) == _abi.FOCUS_ERR_INVALID_ARG
    assert lib.focus_step(None, None, None, None, None) == _abi.FOCUS_ERR_INVALID_ARG


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(_abi, "_lib", None)
    monkeypatch.setattr(_abi, "LIB_PATH", str(tmp_path / "libfocus.so"))
    with pytest.raises(ImportError):
        _abi.load()


def test_null_handles_of_the_block_loop_and_profiling_are_safe():
    lib = _abi.load()
    assert lib.focus_commit_block(None, None, None) == _abi.FOCUS_ERR_INVALID_ARG
    assert lib.focus_decode_block(None, None, None, 4, None, None, None) == _abi.FOCUS_ERR_INVALID_ARG
    assert lib.focus_last_step_launches(None) == -1
    assert lib.focus_profile_begin(None, 0, 1) == _abi.FOCUS_ERR_INVALID_ARG
    assert lib.focus_profile_end(None, None, None) == _abi.FOCUS_ERR_INVALID_ARG
    assert lib.focus_probe_wait_timeout(None, None) == _abi.FOCUS_ERR_INVALID_ARG


# the allocation-free LM head checks its arguments and limits before any device call; the dummy pointers
# below are never dereferenced on these paths
_P = C.c_void_p(4096)


@pytest.mark.parametrize("rows,dim,vocab,eps,code", [
    (-1, 2048, 1000, 1e-6, _abi.FOCUS_ERR_INVALID_ARG),
    (4, 0, 1000, 1e-6, _abi.FOCUS_ERR_INVALID_ARG),
    (4, 2048, 0, 1e-6, _abi.FOCUS_ERR_INVALID_ARG),
    (4, 2048, 1000, float("nan"), _abi.FOCUS_ERR_INVALID_ARG),
    (257, 2048, 1000, 1e-6, _abi.FOCUS_ERR_LIMITS),
    (4, 4224, 1000, 1e-6, _abi.FOCUS_ERR_LIMITS),
    (4, 2048, 163841, 1e-6, _abi.FOCUS_ERR_LIMITS),
    (4, 200, 1000, 1e-6, _abi.FOCUS_ERR_UNSUPPORTED),
    (0, 2048, 1000, 1e-6, _abi.FOCUS_OK),
])
def test_lm_head_noalloc_checks_before_the_device(rows, dim, vocab, eps, code):
    lib = _abi.load()
    assert lib.focus_lm_head_conf_noalloc(_P, rows, dim, _P, _P, vocab, eps, _P, _P, None) == code


@pytest.mark.parametrize("which,offset", [(0, 8), (0, 4), (1, 2), (2, 8), (3, 2), (4, 1)])
def test_lm_head_noalloc_rejects_misaligned_buffers(which, offset):
    """hidden 16-byte, final_norm 8-byte, lm_head 16-byte, conf / top_id 4-byte aligned (a torch view with an
    element offset would otherwise fault on the device); refused before any device call."""
    lib = _abi.load()
    ptrs = [C.c_void_p(4096) for _ in range(5)]
    ptrs[which] = C.c_void_p(4096 + offset)
    h, nrm, w, conf, top = ptrs
    assert lib.focus_lm_head_conf_noalloc(h, 4, 2048, nrm, w, 1000, 1e-6, conf, top, None) == \
        _abi.FOCUS_ERR_INVALID_ARG


def test_lm_head_noalloc_rejects_null_buffers():
    lib = _abi.load()
    for i in range(5):
        ptrs = [_P] * 5
        ptrs[i] = None
        h, nrm, w, conf, top = ptrs
        assert lib.focus_lm_head_conf_noalloc(h, 4, 2048, nrm, w, 1000, 1e-6, conf, top, None) == \
            _abi.FOCUS_ERR_INVALID_ARG
