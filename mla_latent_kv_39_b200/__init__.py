"""B200 (sm_100a) MLA latent-KV decode: a C-ABI CUDA library and its binding.

``abi`` wraps the five C entry points of ``libmla.so`` (cache append, query
absorption, split-KV decode, split combine, output projection) one to one;
``layer.DecodeLayer`` sequences them for one layer's decode step.
"""

from .abi import (  # noqa: F401
    Cache,
    Config,
    MLAError,
    check_device_error,
    lib,
    mla_absorb_q,
    mla_absorb_q_packed,
    mla_absorb_q_workspace_size,
    mla_cache_append,
    mla_cache_append_workspace_size,
    mla_cache_append_noalloc,
    mla_combine,
    mla_combine_lse,
    mla_cache_dequant_fp8,
    mla_fp8_scratch_bytes,
    fp8_scratch_cache,
    mla_combine_out_proj,
    mla_combine_out_proj_workspace_size,
    mla_decode,
    mla_decode_packed,
    mla_decode_packed_planned,
    mla_decode_plan,
    mla_decode_workspace_size,
    mla_get_device_error,
    mla_kernel_launches,
    mla_merge_shards,
    mla_out_proj,
    mla_out_proj_workspace_size,
    mla_query_packed_bytes,
)
from .layer import DecodeLayer  # noqa: F401
from .shard import ShardPlan, decode_shard, decode_sharded, gather_partials, shard_plan  # noqa: F401
