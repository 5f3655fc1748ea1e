"""FlashSampling fused matmul-sample (FMMS) for NVIDIA B200 (sm_100a).

The compute path is a C-ABI shared library (``libfmms.so``, declared in
``include/fmms.h``) built from the CUDA sources in ``csrc/``; ``binding``
marshals torch tensors into it.  Importing this package loads neither the
library nor the binding; the first call of a binding function loads the
library and fails loudly if it is missing.
"""
_BINDING_NAMES = ("FmmsError", "fs_sample", "fs_sample_ex", "fs_sample_grouped",
                  "fs_sample_unfused", "fs_sample_host", "fs_workspace_bytes", "fs_device_status",
                  "fs_status_string", "fs_philox4x32_10", "fs_gumbel", "fs_plan_tiles",
                  "library_path", "load_library", "fs_sample_noalloc",
                  "fs_test_stalled_sample", "fs_sample_shard_keys", "fs_keys_to_tokens",
                  "fs_sample_multi", "fs_workspace_bytes_multi", "fs_summarize_group",
                  "fs_merge_groups", "fs_workspace_bytes_summary", "fs_sample_topk",
                  "fs_set_cta_pairs", "fs_set_partial_merge", "fs_plan_tiles_merged")


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
