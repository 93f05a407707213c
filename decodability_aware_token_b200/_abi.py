"""ctypes mirror of include/focus.h (argument marshalling only)."""
import ctypes as C
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfocus.so")

FOCUS_OK = 0
FOCUS_ERR_INVALID_ARG = -1
FOCUS_ERR_LIMITS = -2
FOCUS_ERR_CUDA = -3
FOCUS_ERR_TIMEOUT = -4
FOCUS_ERR_DEVICE_BOUNDS = -5
FOCUS_ERR_UNSUPPORTED = -6
FOCUS_ERR_NO_MEMORY = -7

FOCUS_DEVERR_TOKEN_ID = 0x1
FOCUS_DEVERR_PAGE_ID = 0x2
FOCUS_DEVERR_PREFIX = 0x4
FOCUS_DEVERR_TIMEOUT = 0x8
FOCUS_DEVERR_FORCED_SET = 0x10

FOCUS_DTYPE_F32 = 0
FOCUS_DTYPE_BF16 = 1

# every symbol include/focus.h declares (checked by the CPU tests)
EXPORTED = ("focus_init", "focus_step", "focus_destroy", "focus_status_string", "focus_get_device_error",
            "focus_workspace_bytes", "focus_last_step_launches", "focus_profile_begin", "focus_profile_end",
            "focus_lm_head_conf_noalloc", "focus_commit_block", "focus_decode_block", "focus_probe_wait_timeout")

KERNEL_CLASSES = ("embed_norm", "qkv_finalize", "attn_score", "attn_ragged", "row_norm", "select", "decode",
                  "gemm_full_qkv", "gemm_full_o", "gemm_full_gateup", "gemm_full_down",
                  "gemm_qkv", "gemm_o", "gemm_gateup", "gemm_down", "gemm_lmhead")


class ModelCfg(C.Structure):
    _fields_ = [("n_layers", C.c_int32), ("hidden", C.c_int32), ("n_q_heads", C.c_int32), ("n_kv_heads", C.c_int32),
                ("head_dim", C.c_int32), ("ffn", C.c_int32), ("vocab", C.c_int32), ("rms_eps", C.c_float),
                ("rope_theta", C.c_float), ("dtype", C.c_int32)]


class Weights(C.Structure):
    _fields_ = [("embed", C.c_void_p), ("final_norm", C.c_void_p), ("lm_head", C.c_void_p),
                ("wqkv", C.POINTER(C.c_void_p)), ("wo", C.POINTER(C.c_void_p)), ("wgate", C.POINTER(C.c_void_p)),
                ("wup", C.POINTER(C.c_void_p)), ("wdown", C.POINTER(C.c_void_p)),
                ("attn_norm", C.POINTER(C.c_void_p)), ("mlp_norm", C.POINTER(C.c_void_p))]


class Limits(C.Structure):
    _fields_ = [("max_requests", C.c_int32), ("max_block", C.c_int32), ("max_keep", C.c_int32),
                ("max_pages_per_req", C.c_int32)]


class Batch(C.Structure):
    _fields_ = [("n_requests", C.c_int32), ("block_size", C.c_int32), ("page_size", C.c_int32),
                ("n_pages", C.c_int32), ("block_tokens", C.c_void_p), ("mask", C.c_void_p),
                ("prefix_len", C.c_void_p), ("page_table", C.c_void_p), ("kv_pool", C.c_void_p), ("ibc", C.c_void_p)]


class Params(C.Structure):
    _fields_ = [("tau", C.c_float), ("alpha", C.c_float), ("conf_threshold", C.c_float),
                ("forced_keep_frac", C.c_float), ("k_min", C.c_int32), ("k_max", C.c_int32),
                ("forced_keep_idx", C.c_void_p), ("forced_keep_count", C.c_void_p)]


class StepOut(C.Structure):
    _fields_ = [("keep_count", C.c_void_p), ("retained_idx", C.c_void_p), ("row_offsets", C.c_void_p),
                ("decoded_ids", C.c_void_p), ("conf", C.c_void_p), ("top_id", C.c_void_p),
                ("importance", C.c_void_p), ("hidden", C.c_void_p)]


_lib = None


def load():
    """Load libfocus.so; raises ImportError if it was not built (there is no fallback path)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m decodability_aware_token_b200.build`")
    lib = C.CDLL(LIB_PATH)
    lib.focus_init.argtypes = [C.POINTER(ModelCfg), C.POINTER(Weights), C.POINTER(Limits), C.POINTER(C.c_void_p)]
    lib.focus_init.restype = C.c_int
    lib.focus_step.argtypes = [C.c_void_p, C.POINTER(Batch), C.POINTER(Params), C.POINTER(StepOut), C.c_void_p]
    lib.focus_step.restype = C.c_int
    lib.focus_destroy.argtypes = [C.c_void_p]
    lib.focus_destroy.restype = C.c_int
    lib.focus_status_string.argtypes = [C.c_int]
    lib.focus_status_string.restype = C.c_char_p
    lib.focus_get_device_error.argtypes = [C.c_void_p, C.POINTER(C.c_int32)]
    lib.focus_get_device_error.restype = C.c_int
    lib.focus_workspace_bytes.argtypes = [C.POINTER(ModelCfg), C.POINTER(Limits)]
    lib.focus_workspace_bytes.restype = C.c_size_t
    lib.focus_last_step_launches.argtypes = [C.c_void_p]
    lib.focus_last_step_launches.restype = C.c_int
    lib.focus_profile_begin.argtypes = [C.c_void_p, C.c_int, C.c_int]
    lib.focus_profile_begin.restype = C.c_int
    lib.focus_profile_end.argtypes = [C.c_void_p, C.POINTER(C.c_float), C.POINTER(C.c_int32)]
    lib.focus_profile_end.restype = C.c_int
    lib.focus_lm_head_conf_noalloc.argtypes = [C.c_void_p, C.c_int32, C.c_int32, C.c_void_p, C.c_void_p, C.c_int32,
                                               C.c_float, C.c_void_p, C.c_void_p, C.c_void_p]
    lib.focus_lm_head_conf_noalloc.restype = C.c_int
    lib.focus_probe_wait_timeout.argtypes = [C.c_void_p, C.c_void_p]
    lib.focus_probe_wait_timeout.restype = C.c_int
    lib.focus_commit_block.argtypes = [C.c_void_p, C.POINTER(Batch), C.c_void_p]
    lib.focus_commit_block.restype = C.c_int
    lib.focus_decode_block.argtypes = [C.c_void_p, C.POINTER(Batch), C.POINTER(Params), C.c_int32, C.POINTER(StepOut),
                                       C.POINTER(C.c_int32), C.c_void_p]
    lib.focus_decode_block.restype = C.c_int
    _lib = lib
    return lib
