"""B200 (sm_100a) low-rank decode library: Python binding of include/lr.h.

The compute path is the CUDA shared library ``liblr_decode.so`` (built by
``python -m decode_lr_linear_b200.build``); this package only marshals
arguments.  ``synth`` holds the seeded synthetic-input generators.
"""
from .ops import (  # noqa: F401
    Factor, FfnWeights, LatentKv, ChainStep, workspace, lr_linear_chain, lr_linear_chain_workspace_size,
    lr_linear, lr_linear_workspace_size, lr_linear_grouped, lr_linear_grouped_workspace_size,
    lr_swiglu_ffn, lr_swiglu_ffn_workspace_size, lr_latent_kv_decode, lr_latent_kv_workspace_size,
    lr_quantize_per_token, lr_gemm_s8s32, lr_workspace_init, lr_check_device_error, lr_set_wait_timeout_us,
    lr_rank_allocate, lr_linear_chain_ranked, lr_dense_linear, lr_flash_decode,
    lr_latent_kv_decode_q8, lr_latent_kv_append, lr_latent_kv_append_workspace_size, lr_set_tensor_core_min_batch,
)
from ._lib import LrError, load  # noqa: F401

__all__ = [n for n in dir() if n.startswith("lr_")] + ["Factor", "FfnWeights", "LatentKv", "ChainStep", "workspace",
                                                       "LrError",
                                                       "load"]
