"""FOCUS focused denoising step on NVIDIA B200 -- Python binding of libfocus.so.

This module only marshals arguments (torch tensors -> device pointers) for the C ABI declared in
include/focus.h; every step of the computation runs in the library's CUDA kernels.  If the library is
missing, importing the step API raises ImportError: there is no fallback path.
"""
from __future__ import annotations

import ctypes as C
import dataclasses
import math
from typing import Optional

import torch

from . import _abi

__all__ = ["FocusContext", "StepParams", "StepOutputs", "FocusError", "status_string", "library_path"]

library_path = _abi.LIB_PATH


class FocusError(RuntimeError):
    def __init__(self, code: int, where: str = ""):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} ({code})")


def status_string(code: int) -> str:
    return _abi.load().focus_status_string(int(code)).decode()


def _check(rc: int, where: str):
    if rc != _abi.FOCUS_OK:
        raise FocusError(rc, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else C.c_void_p(t.data_ptr())


def _need(t: torch.Tensor, name: str, dtype, device, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if t.device != device:
        raise ValueError(f"{name}: on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")


@dataclasses.dataclass
class StepParams:
    tau: float = 0.0
    k_min: int = 1
    k_max: int = 8
    conf_threshold: float = 0.9
    alpha: float = 1.0
    forced_keep_frac: float = -1.0
    forced_keep_idx: Optional[torch.Tensor] = None     # [N, max_keep] int32, ascending
    forced_keep_count: Optional[torch.Tensor] = None   # [N] int32

    def k_cap(self, block: int, max_keep: int) -> int:
        if self.forced_keep_idx is not None:
            return min(max_keep, block)
        if self.forced_keep_frac >= 0:
            return min(block, math.ceil(float(torch.tensor(self.forced_keep_frac, dtype=torch.float32)) * block))
        return self.k_max


@dataclasses.dataclass
class StepOutputs:
    keep_count: torch.Tensor       # [N] int32
    retained_idx: torch.Tensor     # [N, max_keep] int32
    row_offsets: torch.Tensor      # [N + 1] int32
    decoded_ids: torch.Tensor      # [N, B] int32
    conf: torch.Tensor             # [N, max_keep] float32
    top_id: torch.Tensor           # [N, max_keep] int32
    importance: Optional[torch.Tensor] = None   # [2, N, B] float32
    hidden: Optional[torch.Tensor] = None       # [N * max_keep, D] float32

    @classmethod
    def alloc(cls, n: int, block: int, max_keep: int, hidden_dim: int, device, importance=True, hidden=True,
              pin_memory=False):
        dev = torch.device(device)
        kw = dict(device=dev)
        if dev.type == "cpu" and pin_memory:
            kw["pin_memory"] = True
        i32 = dict(dtype=torch.int32, **kw)
        return cls(torch.zeros(n, **i32), torch.zeros(n, max_keep, **i32), torch.zeros(n + 1, **i32),
                   torch.zeros(n, block, **i32), torch.zeros(n, max_keep, dtype=torch.float32, **kw),
                   torch.zeros(n, max_keep, **i32),
                   torch.zeros(2, n, block, dtype=torch.float32, **kw) if importance else None,
                   torch.zeros(n * max_keep, hidden_dim, dtype=torch.float32, **kw) if hidden else None)

    def tensors(self):
        return {f.name: getattr(self, f.name) for f in dataclasses.fields(self)}


class FocusContext:
    """A model's weights bound to a workspace sized by the limits; `step` runs one focused step."""

    def __init__(self, shape, model: dict, *, max_requests: int, max_block: int, max_keep: int,
                 max_pages_per_req: int):
        self._lib = _abi.load()
        self._ctx = C.c_void_p()
        self.shape = shape
        self.dtype = torch.bfloat16 if shape.dtype == "bf16" else torch.float32
        self.device = model["embed"].device
        if self.device.type != "cuda":
            raise ValueError("weights must be CUDA tensors")
        L, D, F, V = shape.n_layers, shape.hidden, shape.ffn, shape.vocab
        Hq, Hkv, d = shape.n_q_heads, shape.n_kv_heads, shape.head_dim
        dt, dev = self.dtype, self.device
        _need(model["embed"], "embed", dt, dev, (V, D))
        _need(model["final_norm"], "final_norm", dt, dev, (D,))
        _need(model["lm_head"], "lm_head", dt, dev, (V, D))
        shapes = {"wqkv": ((Hq + 2 * Hkv) * d, D), "wo": (D, Hq * d), "wgate": (F, D), "wup": (F, D),
                  "wdown": (D, F), "attn_norm": (D,), "mlp_norm": (D,)}
        arrays = {}
        for key, shp in shapes.items():
            if len(model[key]) != L:
                raise ValueError(f"{key}: expected {L} layers")
            for l, t in enumerate(model[key]):
                _need(t, f"{key}[{l}]", dt, dev, shp)
            arrays[key] = (C.c_void_p * L)(*[t.data_ptr() for t in model[key]])
        self._model = model          # the library borrows these: keep them alive
        self._arrays = arrays
        self.cfg = _abi.ModelCfg(L, D, Hq, Hkv, d, F, V, shape.rms_eps, shape.rope_theta,
                                 _abi.FOCUS_DTYPE_BF16 if dt == torch.bfloat16 else _abi.FOCUS_DTYPE_F32)
        w = _abi.Weights(model["embed"].data_ptr(), model["final_norm"].data_ptr(), model["lm_head"].data_ptr(),
                         *[C.cast(arrays[k], C.POINTER(C.c_void_p)) for k in shapes])
        self.limits = _abi.Limits(max_requests, max_block, max_keep, max_pages_per_req)
        with torch.cuda.device(dev):
            _check(self._lib.focus_init(C.byref(self.cfg), C.byref(w), C.byref(self.limits), C.byref(self._ctx)),
                   "focus_init")

    @property
    def max_keep(self) -> int:
        return self.limits.max_keep

    def workspace_bytes(self) -> int:
        return int(self._lib.focus_workspace_bytes(C.byref(self.cfg), C.byref(self.limits)))

    def alloc_outputs(self, n: int, block: int, importance=True, hidden=True) -> StepOutputs:
        return StepOutputs.alloc(n, block, self.max_keep, self.shape.hidden, self.device, importance, hidden)

    def _marshal(self, batch: dict, params: StepParams, out: StepOutputs):
        dev, dt = self.device, self.dtype
        tok = batch["block_tokens"]
        N, B = tok.shape
        pool = batch["kv_pool"]
        L, Hkv, d = self.shape.n_layers, self.shape.n_kv_heads, self.shape.head_dim
        _need(tok, "block_tokens", torch.int32, dev)
        _need(batch["mask"], "mask", torch.uint8, dev, (N, B))
        _need(batch["prefix_len"], "prefix_len", torch.int32, dev, (N,))
        _need(batch["page_table"], "page_table", torch.int32, dev, (N, self.limits.max_pages_per_req))
        _need(pool, "kv_pool", dt, dev)
        if pool.dim() != 6 or tuple(pool.shape[1:4]) != (L, 2, Hkv) or pool.shape[5] != d:
            raise ValueError(f"kv_pool: shape {tuple(pool.shape)}, expected [pages, {L}, 2, {Hkv}, S, {d}]")
        _need(batch["ibc"], "ibc", dt, dev, (N, L, 2, Hkv, B, d))
        mk = self.max_keep
        _need(out.keep_count, "keep_count", torch.int32, dev, (N,))
        _need(out.retained_idx, "retained_idx", torch.int32, dev, (N, mk))
        _need(out.row_offsets, "row_offsets", torch.int32, dev, (N + 1,))
        _need(out.decoded_ids, "decoded_ids", torch.int32, dev, (N, B))
        _need(out.conf, "conf", torch.float32, dev, (N, mk))
        _need(out.top_id, "top_id", torch.int32, dev, (N, mk))
        if out.importance is not None:
            _need(out.importance, "importance", torch.float32, dev, (2, N, B))
        if out.hidden is not None:
            _need(out.hidden, "hidden", torch.float32, dev)
            if out.hidden.shape[0] < N * mk or out.hidden.shape[1] != self.shape.hidden:
                raise ValueError("hidden: expected at least [N * max_keep, D] float32")
        if params.forced_keep_idx is not None:
            _need(params.forced_keep_idx, "forced_keep_idx", torch.int32, dev, (N, mk))
            _need(params.forced_keep_count, "forced_keep_count", torch.int32, dev, (N,))
        cb = _abi.Batch(N, B, pool.shape[4], pool.shape[0], _ptr(tok), _ptr(batch["mask"]), _ptr(batch["prefix_len"]),
                        _ptr(batch["page_table"]), _ptr(pool), _ptr(batch["ibc"]))
        cp = _abi.Params(params.tau, params.alpha, params.conf_threshold, params.forced_keep_frac, params.k_min,
                         params.k_max, _ptr(params.forced_keep_idx), _ptr(params.forced_keep_count))
        co = _abi.StepOut(_ptr(out.keep_count), _ptr(out.retained_idx), _ptr(out.row_offsets), _ptr(out.decoded_ids),
                          _ptr(out.conf), _ptr(out.top_id), _ptr(out.importance), _ptr(out.hidden))
        return cb, cp, co

    def step(self, batch: dict, params: StepParams, out: Optional[StepOutputs] = None,
             stream: Optional[torch.cuda.Stream] = None) -> StepOutputs:
        """Enqueue one focused step on `stream` (default: torch's current stream). Asynchronous."""
        N, B = batch["block_tokens"].shape
        if out is None:
            out = self.alloc_outputs(N, B)
        cb, cp, co = self._marshal(batch, params, out)
        with torch.cuda.device(self.device):
            s = stream if stream is not None else torch.cuda.current_stream(self.device)
            _check(self._lib.focus_step(self._ctx, C.byref(cb), C.byref(cp), C.byref(co), C.c_void_p(s.cuda_stream)),
                   "focus_step")
        return out

    def commit_block(self, batch: dict, stream: Optional[torch.cuda.Stream] = None) -> None:
        """Copy the block's K/V (batch["ibc"]) into the prefix pages at positions P_b .. P_b + B - 1 and
        add B to batch["prefix_len"] (both in place; the page table must map those positions)."""
        N, B = batch["block_tokens"].shape
        cb, _, _ = self._marshal(batch, StepParams(), self.alloc_outputs(N, B))
        with torch.cuda.device(self.device):
            s = stream if stream is not None else torch.cuda.current_stream(self.device)
            _check(self._lib.focus_commit_block(self._ctx, C.byref(cb), C.c_void_p(s.cuda_stream)), "focus_commit_block")

    def decode_block(self, batch: dict, params: StepParams, max_steps: Optional[int] = None,
                     out: Optional[StepOutputs] = None, stream: Optional[torch.cuda.Stream] = None):
        """Decode the block to completion (dense first step, focused steps, dense refresh) and commit it;
        returns (outputs of the last call, number of decoding steps).  Synchronises after every step."""
        N, B = batch["block_tokens"].shape
        if out is None:
            out = self.alloc_outputs(N, B)
        cb, cp, co = self._marshal(batch, params, out)
        steps = C.c_int32(0)
        with torch.cuda.device(self.device):
            s = stream if stream is not None else torch.cuda.current_stream(self.device)
            _check(self._lib.focus_decode_block(self._ctx, C.byref(cb), C.byref(cp), int(max_steps or B), C.byref(co),
                                                C.byref(steps), C.c_void_p(s.cuda_stream)), "focus_decode_block")
        return out, int(steps.value)

    def probe_wait_timeout(self, stream: Optional[torch.cuda.Stream] = None) -> None:
        """Enqueue the failure-path probe: a bounded pipeline wait that nothing satisfies gives up after
        about a second and flags FOCUS_DEVERR_TIMEOUT (read it with device_error)."""
        with torch.cuda.device(self.device):
            s = stream if stream is not None else torch.cuda.current_stream(self.device)
            _check(self._lib.focus_probe_wait_timeout(self._ctx, C.c_void_p(s.cuda_stream)), "focus_probe_wait_timeout")

    def last_step_launches(self) -> int:
        """Kernels the most recent step enqueued."""
        return int(self._lib.focus_last_step_launches(self._ctx))

    def profile_begin(self, kernel_class: str, max_launches: int = 1 << 16):
        """Record CUDA events around every launch of `kernel_class` (see _abi.KERNEL_CLASSES) from now on."""
        _check(self._lib.focus_profile_begin(self._ctx, _abi.KERNEL_CLASSES.index(kernel_class), max_launches),
               "focus_profile_begin")

    def profile_end(self):
        """-> (summed device milliseconds, number of timed launches)."""
        ms, n = C.c_float(0), C.c_int32(0)
        _check(self._lib.focus_profile_end(self._ctx, C.byref(ms), C.byref(n)), "focus_profile_end")
        return float(ms.value), int(n.value)

    def device_error(self):
        """Synchronise, read and clear the device error word -> (status code, FOCUS_DEVERR_* bits)."""
        bits = C.c_int32(0)
        rc = self._lib.focus_get_device_error(self._ctx, C.byref(bits))
        return rc, bits.value

    def close(self):
        if getattr(self, "_ctx", None) is not None and self._ctx.value:
            _check(self._lib.focus_destroy(self._ctx), "focus_destroy")
            self._ctx = C.c_void_p()

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
