"""B200 (sm_100a) MiniMax Sparse Attention forward path and main-branch backward.

The binding (``block_sparse_long_idx_b200.api``) loads libmsa_b200.so on first use of any of its
names, so that the seeded input generators (``block_sparse_long_idx_b200.synth``) import without
the CUDA library. A missing library raises ImportError: there is no fallback path.
"""
_API_NAMES = {
    "lib", "LIB_PATH", "MsaError", "KV2Q", "msa_kv2q_layout", "status_string", "msa_get_device_error",
    "msa_index_topk", "msa_kv2q_layout_get", "msa_build_kv2q", "msa_sparse_prefill_workspace_size",
    "msa_sparse_prefill", "msa_sparse_decode", "SIGNATURES", "KernelTrace", "msa_launch_count", "KERNEL_NAMES",
    "msa_selftest_wait_timeout", "msa_sparse_prefill_varlen", "msa_sparse_backward", "msa_quantize_e4m3",
    "msa_sparse_prefill_fp8", "E4M3Rows",
}


def __getattr__(name):
    if name in _API_NAMES:
        from . import api

        return getattr(api, name)
    raise AttributeError(name)
