"""B200 (sm_100a) split-KV grouped-query attention over packed variable-length
sequences (decode and short-query regime).

    from varlen_gqa_split_b200 import Plan
    plan = Plan(B_max, s_max, Hq, Hkv, D, max_q)      # once, outside capture
    out, lse = plan.run(q, k, v, cu_q, cu_k)          # per step, capturable
    out, lse = plan.run_paged(q, k_cache, v_cache, block_table, cu_q, cu_k)   # paged K/V

The compute runs in libvgqa.so (C ABI: include/varlen_gqa.h); this package
only marshals torch tensors into it.
"""
from ._binding import (ATTN_COMBINE_AUTO, ATTN_COMBINE_FUSED, ATTN_COMBINE_KERNEL, ATTN_DEV_ERR_K_TOO_LONG, ATTN_DEV_ERR_OFFSETS, ATTN_DEV_ERR_PAGE, ATTN_DEV_ERR_Q_TOO_LONG,
                       ATTN_DEV_ERR_TIMEOUT, ATTN_VARIANT_AUTO, ATTN_VARIANT_MMA, ATTN_VARIANT_SIMT, ATTN_VARIANT_TC,
                       AttnError, Plan, lib, merge_lse, strerror)

__all__ = ["ATTN_COMBINE_AUTO", "ATTN_COMBINE_FUSED", "ATTN_COMBINE_KERNEL", "Plan", "AttnError", "lib", "merge_lse",
           "strerror", "ATTN_VARIANT_AUTO", "ATTN_VARIANT_SIMT",
           "ATTN_VARIANT_MMA", "ATTN_VARIANT_TC", "ATTN_DEV_ERR_OFFSETS", "ATTN_DEV_ERR_Q_TOO_LONG",
           "ATTN_DEV_ERR_K_TOO_LONG", "ATTN_DEV_ERR_TIMEOUT", "ATTN_DEV_ERR_PAGE"]
