"""ctypes declarations of the C ABI in include/lr.h (argument marshalling only).

Loading fails loudly when ``liblr_decode.so`` has not been built; there is no
fallback implementation of any call.
"""
from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liblr_decode.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "lr.h")

# lr_status_t
LR_OK, LR_ERR_INVALID_ARG, LR_ERR_UNSUPPORTED, LR_ERR_MISALIGNED, LR_ERR_WORKSPACE, LR_ERR_CUDA, \
    LR_ERR_DEVICE_TIMEOUT = range(7)
# lr_dtype_t
LR_F32, LR_BF16, LR_F16, LR_I8, LR_I32 = range(5)
LR_MAX_GROUP = 4
LR_MAX_CHAIN = 64
LR_KV_ABSORBED, LR_KV_RECONSTRUCT = 0, 1
LR_NOALLOC_SCRATCH_BYTES = 1 << 20
DEVICE_ERR_MBAR, DEVICE_ERR_TMEM, DEVICE_ERR_GRID_WAIT = 1, 2, 3

c_int, c_void_p, c_size_t, c_float = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_float


class FactorDesc(ctypes.Structure):
    _fields_ = [("A", c_void_p), ("B", c_void_p), ("d_in", c_int), ("d_out", c_int), ("rank", c_int),
                ("active_rank", c_int), ("w_dtype", c_int), ("scale_dtype", c_int),
                ("scale_A", c_void_p), ("scale_B", c_void_p)]


class ChainStep(ctypes.Structure):
    _fields_ = [("n", c_int), ("input_step", c_int), ("input_proj", c_int),
                ("proj", FactorDesc * 4), ("y", c_void_p * 4)]


class RankVec(ctypes.Structure):
    _fields_ = [("n", c_int), ("ranks", ctypes.POINTER(c_int))]


class FfnDesc(ctypes.Structure):
    _fields_ = [("hidden", c_int), ("inter", c_int), ("n_lr", c_int), ("rank", c_int), ("scale_dtype", c_int),
                ("A", c_void_p), ("s_A", c_void_p), ("B", c_void_p), ("s_B", c_void_p),
                ("D", c_void_p), ("s_D", c_void_p), ("W_down", c_void_p), ("s_down", c_void_p)]


class LatentKvDesc(ctypes.Structure):
    _fields_ = [("batch", c_int), ("heads", c_int), ("head_dim", c_int), ("rank", c_int), ("max_ctx", c_int),
                ("scale", c_float), ("B_K", c_void_p), ("B_V", c_void_p), ("mode", c_int),
                ("split_tokens", c_int), ("cache_scale_dtype", c_int), ("rope_base", c_float)]


class FlashDesc(ctypes.Structure):
    _fields_ = [("batch", c_int), ("heads", c_int), ("head_dim", c_int), ("max_ctx", c_int), ("scale", c_float),
                ("split_tokens", c_int)]


P = ctypes.POINTER
_SIGNATURES = {
    "lr_linear": (c_int, [P(FactorDesc), c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_size_t, c_void_p]),
    "lr_linear_workspace_size": (c_int, [P(FactorDesc), c_int, c_int, P(c_size_t)]),
    "lr_linear_noalloc": (c_int, [P(FactorDesc), c_void_p, c_int, c_void_p, c_void_p]),
    "lr_linear_chain": (c_int, [P(ChainStep), c_int, c_void_p, c_int, c_void_p, c_size_t, c_void_p]),
    "lr_linear_chain_workspace_size": (c_int, [P(ChainStep), c_int, c_int, P(c_size_t)]),
    "lr_rank_allocate": (c_int, [P(ctypes.c_double), c_int, ctypes.c_double, P(RankVec), P(c_int)]),
    "lr_linear_chain_ranked": (c_int, [P(ChainStep), c_int, P(RankVec), c_void_p, c_int, c_void_p, c_size_t,
                                       c_void_p]),
    "lr_linear_grouped": (c_int, [P(FactorDesc), c_int, c_void_p, c_int, P(c_void_p), c_void_p, c_size_t,
                                  c_void_p]),
    "lr_linear_grouped_workspace_size": (c_int, [P(FactorDesc), c_int, c_int, P(c_size_t)]),
    "lr_dense_linear": (c_int, [c_void_p, c_int, c_void_p, c_int, c_int, c_int, c_void_p, c_int, c_void_p, c_void_p]),
    "lr_swiglu_ffn": (c_int, [P(FfnDesc), c_void_p, c_int, c_void_p, c_void_p, c_size_t, c_void_p]),
    "lr_swiglu_ffn_workspace_size": (c_int, [P(FfnDesc), c_int, P(c_size_t)]),
    "lr_latent_kv_decode": (c_int, [P(LatentKvDesc), c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                    c_size_t, c_void_p]),
    "lr_latent_kv_workspace_size": (c_int, [P(LatentKvDesc), P(c_size_t)]),
    "lr_latent_kv_decode_q8": (c_int, [P(LatentKvDesc), c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                       c_void_p, c_void_p, c_size_t, c_void_p]),
    "lr_latent_kv_append": (c_int, [P(LatentKvDesc), c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p,
                                    c_void_p, c_size_t, c_void_p]),
    "lr_latent_kv_append_workspace_size": (c_int, [P(LatentKvDesc), c_int, P(c_size_t)]),
    "lr_flash_decode": (c_int, [P(FlashDesc), c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                c_void_p]),
    "lr_flash_decode_workspace_size": (c_int, [P(FlashDesc), P(c_size_t)]),
    "lr_quantize_per_token": (c_int, [c_void_p, c_int, c_int, c_void_p, c_void_p, c_void_p]),
    "lr_gemm_s8s32": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_void_p, c_void_p]),
    "lr_workspace_init": (c_int, [c_void_p, c_size_t, c_void_p]),
    "lr_check_device_error": (c_int, [c_void_p, P(c_int)]),
    "lr_set_wait_timeout_us": (c_int, [ctypes.c_uint]),
    "lr_set_tensor_core_min_batch": (c_int, [c_int, c_int]),
    "lr_status_string": (ctypes.c_char_p, [c_int]),
    "lr_version": (c_int, []),
}

_lib = None


def header_functions() -> list[str]:
    """Names of the entry points declared in include/lr.h."""
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:LR_API\s+)?(?:lr_status_t|const char\*|int)\s+(lr_\w+)\s*\(", text, flags=re.M)))


def load():
    """The loaded library (ctypes.CDLL) with every signature declared."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run `python -m decode_lr_linear_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


class LrError(RuntimeError):
    def __init__(self, fn: str, status: int):
        msg = load().lr_status_string(status).decode()
        super().__init__(f"{fn} failed: {msg} (status {status})")
        self.status = status


def check(fn: str, status: int) -> None:
    if status != LR_OK:
        raise LrError(fn, status)
