"""B200-native training-free block-sparse "sol-attn" attention.

The compute path is libbsa.so (CUDA, sm_100a) behind the C ABI in
include/bsa.h; this package is its ctypes binding.  Importing it fails if the
library has not been built (``python block_sparse_attention_26_b200/build.py``).
"""
from .binding import (BSA_ERR_CAPACITY, BSA_DENSE_BLOCK, BSA_DENSE_HYBRID, BSA_DENSE_SHORT, BSA_DENSE_WINDOW, BSA_RUN_SPARSE,
                      BSA_DT_BF16, BSA_DT_F32, BSA_SLA, BSA_SOL, BSA_VSA, EXPORTED, LIB_PATH, BsaError,
                      Buffers, bsa_attention, bsa_attention_prepare, bsa_attention_run,
                      bsa_dense_ref_rows, bsa_selftest_bounded_wait, bsa_launch_count, bsa_layer_host, HostLayer,
                      bsa_device_status, bsa_params,
                      bsa_pool, bsa_qkv_pool, bsa_select, bsa_select_static, bsa_workspace_size, dims, lib, make_params, params_for,
                      bsa_policy, bsa_policy_decide, make_policy, run_layer, run_step)

__all__ = ["BSA_ERR_CAPACITY", "BSA_DENSE_BLOCK", "BSA_DENSE_HYBRID", "BSA_DENSE_SHORT", "BSA_DENSE_WINDOW", "BSA_RUN_SPARSE",
           "BSA_DT_BF16", "BSA_DT_F32", "BSA_SLA", "BSA_SOL", "BSA_VSA", "EXPORTED", "LIB_PATH", "BsaError",
           "Buffers", "bsa_attention", "bsa_attention_prepare", "bsa_attention_run",
           "bsa_dense_ref_rows", "bsa_selftest_bounded_wait", "bsa_launch_count", "bsa_layer_host", "HostLayer",
           "bsa_device_status", "bsa_params",
           "bsa_pool", "bsa_qkv_pool", "bsa_select", "bsa_select_static", "bsa_workspace_size", "dims", "lib", "make_params", "params_for",
           "bsa_policy", "bsa_policy_decide", "make_policy", "run_layer", "run_step"]
