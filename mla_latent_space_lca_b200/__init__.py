"""B200-native (sm_100a) MLA decode and latent-condensed attention (LCA).

The work runs in liblca_b200.so (hand-written CUDA kernels behind the C ABI
of include/lca.h); this package only marshals PyTorch tensors into it.  The
library is loaded on first use, which raises ImportError if it has not been
built; nothing falls back to another implementation.
"""
from .api import (default_scale, device_status, launch_count, lca_append_token, lca_combine_shards, lca_condense,
                  lca_condense_append, lca_decode, lca_decode_attn, lca_decode_shard, lca_decode_stored,
                  lca_decode_stored_varlen, lca_decode_varlen,
                  lca_prefill_block, mla_decode_attn, num_groups, profile_collect, profile_enable,
                  shard_record_floats, workspace, workspace_bytes)

__all__ = ["default_scale", "device_status", "launch_count", "lca_append_token", "lca_combine_shards", "lca_condense",
           "lca_condense_append", "lca_decode", "lca_decode_attn", "lca_decode_shard", "lca_decode_stored",
           "lca_decode_stored_varlen", "lca_decode_varlen",
           "lca_prefill_block", "mla_decode_attn", "num_groups", "profile_collect", "profile_enable",
           "shard_record_floats", "workspace", "workspace_bytes"]
