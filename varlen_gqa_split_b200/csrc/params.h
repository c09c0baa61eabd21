// params.h -- launch parameter block shared by host code and kernels (internal).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace vgqa {

// Default upper bound on one bounded wait, in nanoseconds of %globaltimer.
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;

// Everything a split / combine launch needs.  Passed by value.
struct Params {
    const __nv_bfloat16 *q;    // [T_q, Hq, D]
    const __nv_bfloat16 *k;    // [T_kv, Hkv, D], token stride k_stride elements
    const __nv_bfloat16 *v;    // [T_kv, Hkv, D], token stride v_stride elements
    const int32_t *cu_q;       // [B_max + 1]
    const int32_t *cu_k;       // [B_max + 1]
    __nv_bfloat16 *out;        // [T_q, Hq, D]
    float *lse;                // [T_q, Hq]
    float *o_part;             // [B_max, max_q, Hq, nsplit, D]  (nsplit > 1)
    float2 *ml_part;           // [B_max, max_q, Hq, nsplit]     (m, l) base-2
    uint32_t *err;             // sticky ATTN_DEV_ERR_* bits
    uint32_t *ticket;          // [B_max * Hkv * row_tiles] arrival counters (fused merge)
    unsigned long long *claim; // [B_max * Hkv] tile claims of cut units (tensor-core path)
    uint32_t *done;            // [B_max * Hkv] parts written / merges started per cut unit
    int B_max, s_max, Hq, Hkv, D, max_q, G;
    int nsplit;                // chunks per (sequence, KV head)
    int chunk;                 // keys per chunk
    int rows_per_block;        // query rows (G * tokens) per block
    int row_tiles;             // row blocks per KV head
    float scale_log2;          // (1/sqrt(D)) * log2(e)
    int fused;                 // no combine kernel: on the CUDA-core path (nsplit > 1) the last block
                               // of a unit to finish merges it; on the tcgen05 path the block
                               // holding a cut unit's last part does
    int merge_bytes;           // tensor-core path: shared bytes of the merge area
    int ctas_max;              // tensor-core path: blocks of the launch (merge table size)
    int direct;                // warp-MMA path: block c takes unit c whole (no cut units, no merge)
    int dynamic;               // tensor-core path: blocks sharing a cut unit claim its tiles
    int head_first;            // tensor-core path: schedule order for the fused merge (OrderedWalker)
    int done_per_part;         // tensor-core path: releases on `done` per written part
    int share_stride;          // tensor-core path: block b takes share (b * share_stride) mod blocks
    int unit_cost;             // tensor-core path: tiles' worth of fixed cost per unit in the shares
    int qtile;                 // tensor-core path: query tokens per row tile (a unit is (b, hk, row tile))
    int max_rt;                // tensor-core path: row tiles of a sequence at most (counter stride)
    long long k_stride;        // elements between consecutive tokens of k (Hkv * D when packed)
    long long v_stride;        // elements between consecutive tokens of v
    // paged K/V (block_table != null): key j of sequence b sits in page
    // block_table[b * bt_stride + (j >> page_shift)], slot j & (page size - 1)
    const int32_t *block_table;
    int bt_stride;             // entries per sequence row of block_table
    int page_shift;            // log2(page size)
    int num_pages;             // pages in the cache (valid page indexes)
    int page_box;              // keys per TMA load: min(page size, 64)
    long long page_stride;     // elements between consecutive pages of k and v
    int page_rows;             // page_stride / token stride when whole (tensor maps index rows
                               // page * page_rows + slot), else 0 (tensor maps index (slot, page))
    unsigned long long wait_ns; // limit of one bounded wait on another role or block (%globaltimer ns)
    const uint32_t *stall;     // [1] parts every cut unit's merge waits for beyond its own (0 except
                               // under the plan's test hook, whose parts never arrive)
};

}  // namespace vgqa
