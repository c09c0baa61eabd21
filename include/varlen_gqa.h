/*
 * varlen_gqa.h -- C ABI of the B200 (sm_100a) split-KV varlen GQA attention
 * library (libvgqa.so).
 *
 * The library computes grouped-query attention for packed variable-length
 * (THD) batches in the decode and short-query regime:
 *
 *   for each sequence b, query token qi < Lq_b and query head h
 *   (hk = h / G, G = Hq / Hkv, n = clamp(Lk_b - Lq_b + qi + 1, 0, Lk_b)):
 *     s_j = (1/sqrt(D)) q[cu_q[b]+qi, h, :] . k[cu_k[b]+j, hk, :],  j < n
 *     out = softmax(s) V,   lse = ln sum_j exp(s_j)     (natural log)
 *   n = 0 gives out = 0 and lse = -inf.
 *
 * It runs as split-KV flash-decoding: each (sequence, KV head, KV chunk)
 * block emits unnormalised (O, m, l) partials and a log-sum-exp merge
 * produces the output (AstrAI commit log for csrc/kernels/gqa_decode_attn.cu,
 * split-KV commit; magik.net "Wiring Split-K Dispatch into a Custom CUDA
 * Attention Kernel", section "The Message").  The grid and the split count are
 * fixed when the plan is made, from constants only, and the kernels read the
 * exact lengths from device-side cu_seqlens, so a call makes no device-to-host
 * copy, no allocation and no compilation and can be captured once in a CUDA
 * graph and replayed while the lengths change (cudnn-frontend issue #552
 * "frost(sdpa): THD execute host round-trip", section "Proposal to evaluate").
 *
 * Conventions for every entry point:
 *  - Return value: 0 (ATTN_OK) or a negative ATTN_E_* code; attn_strerror()
 *    names it.  On an error return nothing has been launched or changed.
 *  - "device pointer" means memory of the CUDA device that was current when
 *    the plan was made; the caller owns it and keeps it alive until the work
 *    on the stream that uses it has finished.
 *  - stream: a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  All device work of a call is ordered on that stream.
 *  - Calls on one plan must not overlap on the GPU (the plan's scratch is
 *    reused by every call); use one plan per concurrent stream.
 *  - Thread safety: distinct plans may be used from distinct host threads.
 */
#ifndef VARLEN_GQA_H
#define VARLEN_GQA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---------------------------------------------------------------- errors */
#define ATTN_OK 0
#define ATTN_E_INVALID_ARG (-1)   /* a size or count out of range            */
#define ATTN_E_UNSUPPORTED (-2)   /* e.g. head dim not in {64, 128}           */
#define ATTN_E_NULL (-3)          /* a required pointer is NULL               */
#define ATTN_E_ALIGNMENT (-4)     /* a pointer breaks the alignment contract  */
#define ATTN_E_BAD_PLAN (-5)      /* unknown or destroyed plan handle         */
#define ATTN_E_CUDA (-6)          /* a CUDA runtime / driver call failed      */
#define ATTN_E_NOMEM (-7)         /* device allocation failed                 */
#define ATTN_E_DEVICE (-8)        /* current device is not the plan's device  */
#define ATTN_E_NO_DEVICE (-9)     /* no usable sm_100 device                  */
#define ATTN_E_SCRATCH_LIMIT (-10) /* attn_run_noalloc: shape needs more scratch
                                     than ATTN_NOALLOC_SCRATCH_BYTES            */

/* Sticky device-side error bits, read by attn_check_error().  When a
 * sequence trips one, none of its output rows are written. */
#define ATTN_DEV_ERR_OFFSETS 0x1u      /* cu_q / cu_k negative or decreasing  */
#define ATTN_DEV_ERR_Q_TOO_LONG 0x2u   /* Lq_b > max_q of the plan            */
#define ATTN_DEV_ERR_K_TOO_LONG 0x4u   /* Lk_b > s_max of the plan            */
#define ATTN_DEV_ERR_TIMEOUT 0x8u      /* a bounded pipeline wait gave up      */
#define ATTN_DEV_ERR_PAGE 0x10u        /* a block-table entry outside the cache */

/* Kernel variants (attn_overrides.variant / attn_plan_desc.variant). */
#define ATTN_VARIANT_AUTO 0
#define ATTN_VARIANT_SIMT 1   /* CUDA-core path, any row count               */
#define ATTN_VARIANT_MMA 2    /* TMA-fed warp-MMA path, G*max_q <= 16         */
#define ATTN_VARIANT_TC 3     /* TMA-fed tcgen05 path (tensor memory),
                                 G*max_q <= 128                              */

/* How split partials are merged (attn_overrides.combine / attn_plan_desc.combine). */
#define ATTN_COMBINE_AUTO 0
#define ATTN_COMBINE_KERNEL 1  /* a second kernel merges every row                */
#define ATTN_COMBINE_FUSED 2   /* no second kernel: the block holding a cut unit's
                                  last part merges it (tcgen05 path, static
                                  shares only: with deterministic = -1 the plan
                                  fails with ATTN_E_UNSUPPORTED); on the CUDA-core
                                  path the last block of a unit to finish does  */

typedef struct attn_plan_s *attn_plan_t;   /* opaque */

/*
 * Explicit plan choices, for sweeps in tests and benchmarks (the magik.net
 * post tunes its split count through an environment knob, section "Assumptions
 * and Their Validity"; here it is an argument).  Zero in a field keeps the
 * planner's own choice.
 */
typedef struct {
    int nsplit;    /* KV chunks per (sequence, KV head); >= 1                  */
    int block_n;   /* keys per pipeline tile: 64                                */
    int variant;   /* ATTN_VARIANT_*                                            */
    int stages;    /* pipeline depth of the tensor-core path: 2..8              */
    int combine;   /* ATTN_COMBINE_*                                            */
    int ctas;      /* tensor-core path: blocks sharing the tile space; >= 1     */
    int deterministic; /* 1: bitwise-repeatable results (static tile shares);
                          -1: blocks that share a unit balance it between them
                          at run time, results equal within rounding;
                          0: the plan's choice: run-time balancing on the
                          warp-MMA path, static shares on the tcgen05 path
                          (the CUDA-core path is always repeatable)           */
    int wait_limit_us; /* upper bound of one bounded device wait (a pipeline
                          stage, a merge waiting for a unit's parts), in
                          microseconds; 0 keeps the default of 2 s.  A wait
                          that runs out sets ATTN_DEV_ERR_TIMEOUT and its block
                          returns without writing the rows it was to write  */
    int test_stall;    /* test hook, tensor-core paths only: 1 makes the merge
                          of every cut unit wait for one part that is never
                          written, so those waits run out (after
                          wait_limit_us) on the plan's first call, leaving the
                          cut units' rows unwritten; attn_check_error() clears
                          it.  0 in every other use                         */
} attn_overrides;

/* What the planner chose (attn_plan_info). */
typedef struct {
    int B_max, s_max, Hq, Hkv, D, max_q;
    int G;                 /* Hq / Hkv                                          */
    int variant;           /* ATTN_VARIANT_SIMT, _MMA or _TC                    */
    int nsplit;            /* SIMT path: KV chunks per (sequence, KV head); 0 on
                              the tensor-core path, whose split points follow
                              the balanced per-block shares                      */
    int chunk;             /* SIMT path: keys per chunk (multiple of block_n)    */
    int block_n;           /* keys per tile                                      */
    int stages;            /* pipeline stages (tensor-core path)                 */
    int rows_per_block;    /* query rows (G * q tokens) one block handles        */
    int row_tiles;         /* blocks along the row axis per KV head              */
    int grid_x, grid_y, grid_z;   /* split-kernel grid: SIMT (nsplit, Hkv*row_tiles,
                              B_max); tensor-core (ctas, 1, 1)                    */
    int ctas;              /* tensor-core path: persistent blocks (0 on SIMT)    */
    int deterministic;     /* 1 if results are bitwise repeatable for this plan  */
    int combine;           /* ATTN_COMBINE_KERNEL or ATTN_COMBINE_FUSED; 0 when
                              no unit is ever split (one split per unit on the
                              CUDA-core path; on the warp-MMA path, plans of
                              units of <= 128 keys that fit one wave take one
                              block per unit and write every row directly) */
    int combine_blocks;    /* combine-kernel blocks (0 unless a combine kernel runs) */
    int smem_bytes;        /* dynamic shared memory of the split kernel          */
    int num_sms;           /* SM count of the plan's device                      */
    size_t scratch_bytes;  /* device scratch the plan owns (partials)            */
} attn_plan_desc;

/*
 * attn_plan -- size the grid and the split count once, from constants.
 *
 *   B_max  sequences per call (cu arrays hold B_max + 1 entries); >= 1
 *   s_max  largest key length of any sequence; >= 1
 *   Hq, Hkv  query / KV heads, Hq % Hkv == 0
 *   D      head dimension, 64 or 128
 *   max_q  largest query length of any sequence; 1 for decode; >= 1
 *
 * Source: plan-time grid from declared constants, cudnn-frontend issue #552,
 * section "Proposal to evaluate"; split count that fills the device and falls
 * back to a single direct-write pass when B*Hkv already saturates it, AstrAI
 * commit log (split-KV commit); reject an unsupported head dim rather than run
 * a silent fallback, AstrAI commit log (dispatch commit).
 *
 * Queries the current device's SM count, allocates the partials scratch and a
 * device error word with cudaMalloc, and sets kernel attributes: call it
 * outside stream capture.  The softmax scale is 1/sqrt(D) and the causal mask
 * is aligned to each sequence's tail (a no-op when Lq_b = 1).  On success
 * *out holds a new plan, owned by the caller until attn_destroy().
 */
int attn_plan(attn_plan_t *out, int B_max, int s_max, int Hq, int Hkv, int D,
              int max_q);

/* attn_plan with explicit choices; o may be NULL (same as attn_plan). */
int attn_plan_ex(attn_plan_t *out, int B_max, int s_max, int Hq, int Hkv, int D,
                 int max_q, const attn_overrides *o);

/* Fill *desc with the plan's choices.  Host only; never touches the GPU. */
int attn_plan_info(attn_plan_t plan, attn_plan_desc *desc);

/*
 * attn_run -- one attention call, asynchronous on `stream`.
 *
 *   q      device, bf16 [T_q, Hq, D], packed and contiguous, 16-byte aligned;
 *          readable for at least cu_q[B_max] tokens
 *   k, v   device, bf16 [T_kv, Hkv, D], packed and contiguous, 16-byte aligned;
 *          readable for at least cu_k[B_max] tokens
 *   cu_q, cu_k  device, int32, B_max + 1 entries each, 4-byte aligned:
 *          cu[0] >= 0 and non-decreasing; sequence b owns tokens
 *          [cu[b], cu[b+1]).  A batch smaller than B_max repeats its last
 *          offset (zero-length sequences), the form a buffer sized for the
 *          largest batch takes (TransformerEngine PR #24 "Build the attention
 *          padding mask without host syncs", section Changes).
 *   out    device, bf16 [T_q, Hq, D], 16-byte aligned
 *   lse    device, fp32 [T_q, Hq] (natural log of the scaled scores), 4-byte
 *          aligned
 *
 * Only rows covered by cu_q are written.  A sequence with Lk_b = 0 (or a
 * query that sees no key) gets out = 0 and lse = -inf.  The lengths are read
 * on the device; sequences that break the plan's bounds set a sticky bit for
 * attn_check_error() and are left unwritten.
 *
 * The call launches one kernel (two with ATTN_COMBINE_KERNEL) and nothing
 * else: no host sync, no
 * device-to-host copy, no allocation, so it can be captured in a CUDA graph
 * (the captured graph keeps the pointers; replay it with the same buffers,
 * rewriting cu_q / cu_k and the tensors' contents in place).  Host-detectable
 * errors (NULL or misaligned pointers, wrong device, bad plan) return a code
 * and launch nothing.
 */
int attn_run(attn_plan_t plan, const void *q, const void *k, const void *v,
             const int32_t *cu_q, const int32_t *cu_k, void *out, float *lse,
             void *stream);

/*
 * attn_run_strided -- attn_run with K and V as views into larger buffers.
 *
 *   k_token_stride, v_token_stride  elements between consecutive tokens of
 *          k and v; within a token the Hkv heads of D elements stay
 *          contiguous.  Each stride is >= Hkv * D, a multiple of 8 (16-byte
 *          rows) and at most 2^38; otherwise ATTN_E_INVALID_ARG and nothing is
 *          launched.  A fused cache laid out [T, 2, Hkv, D] passes k = base,
 *          v = base + Hkv * D and both strides 2 * Hkv * D.  All other
 *          arguments, the outputs and the error behaviour are those of
 *          attn_run (which is this call with both strides Hkv * D).
 *
 * Source: the declared-stride contract of THD inputs instead of a packed-
 * stride assumption, cudnn-frontend issue #552 "frost(sdpa): THD execute host
 * round-trip", section Related (#538, #539); stride parameters in the split
 * kernel's interface, magik.net "Wiring Split-K Dispatch into a Custom CUDA
 * Attention Kernel", section "The Message".  Not planned separately: one plan
 * serves packed and strided calls.
 */
int attn_run_strided(attn_plan_t plan, const void *q, const void *k, const void *v,
                     const int32_t *cu_q, const int32_t *cu_k, void *out, float *lse,
                     int64_t k_token_stride, int64_t v_token_stride, void *stream);

/*
 * attn_run_paged -- attn_run over a paged K/V cache.
 *
 *   k_cache, v_cache  device, bf16, 16-byte aligned: num_pages pages of
 *          page_size tokens, each token Hkv heads of D contiguous elements.
 *          Token t of page n starts at element n * page_stride +
 *          t * token_stride of its cache.  K and V share the layout; a cache
 *          laid out [pages, 2, page_size, Hkv, D] passes v_cache = k_cache +
 *          page_size * Hkv * D and page_stride = 2 * page_size * Hkv * D.
 *   page_stride, token_stride  elements; multiples of 8 (16-byte rows),
 *          token_stride >= Hkv * D, page_stride >= page_size * token_stride,
 *          both at most 2^38.
 *   page_size  tokens per page: a power of two, 8 <= page_size <= 2^20.
 *   num_pages  pages in each cache, >= 1; num_pages * page_size < 2^31.
 *   block_table  device, int32 [B_max, bt_stride], 4-byte aligned: key j of
 *          sequence b is token j % page_size of page
 *          block_table[b * bt_stride + j / page_size].  Only the entries
 *          covering the sequence's Lk_b keys are read.
 *   bt_stride  entries per sequence row, >= ceil(s_max / page_size).
 *   cu_k   as for attn_run, but only the lengths Lk_b = cu_k[b+1] - cu_k[b]
 *          are used; where the keys sit comes from the block table.
 *
 * The keys past Lk_b in a sequence's last page are never used, whatever they
 * hold (stale or non-finite values included).  A table entry outside
 * [0, num_pages) sets ATTN_DEV_ERR_PAGE; the keys it names read as zeros, so
 * the call stays inside the cache, but that sequence's output is then
 * meaningless.  Bad sizes or strides return ATTN_E_INVALID_ARG and launch
 * nothing.  Everything else (outputs, capture, error behaviour) is as for
 * attn_run.  Not available through attn_run_noalloc.
 *
 * Source: the paged cache in the split kernel's interface (page size and
 * page bytes among its parameters), magik.net "Wiring Split-K Dispatch into
 * a Custom CUDA Attention Kernel", section "The Message: A Read That Reveals
 * the Architecture"; device-side lengths with the padded positions masked,
 * TransformerEngine PR #24, section Changes.
 */
int attn_run_paged(attn_plan_t plan, const void *q, const void *k_cache, const void *v_cache,
                   int64_t page_stride, int64_t token_stride, int page_size, int num_pages,
                   const int32_t *block_table, int bt_stride, const int32_t *cu_q,
                   const int32_t *cu_k, void *out, float *lse, void *stream);

/*
 * attn_merge_lse -- combine n attention results computed over disjoint key
 * ranges of the same queries (context parallelism: each GPU attends over its
 * own stretch of every sequence's keys; after an all-gather of the (out, lse)
 * pairs every GPU merges them).  Asynchronous on `stream`, no sync, no
 * allocation, capturable.
 *
 *   outs   device, bf16 [n_parts, T_q, Hq, D], 16-byte aligned: part r's out
 *   lses   device, fp32 [n_parts, T_q, Hq], 4-byte aligned: part r's lse
 *          (natural log, -inf where the part saw no key)
 *   cu_q   device, int32, B_max + 1 entries: only tokens
 *          [cu_q[0], cu_q[B_max]) are merged and written
 *   out    device, bf16 [T_q, Hq, D]; lse device, fp32 [T_q, Hq]
 *
 * Per row: M = max_r lse_r, w_r = e^(lse_r - M), out = sum_r w_r out_r /
 * sum_r w_r, lse = M + ln sum_r w_r; a row with every lse_r = -inf gets
 * out = 0, lse = -inf.  The tail-aligned causal mask is a no-op at q_len = 1,
 * so decode splits its keys anywhere; with q_len > 1 each part must have
 * applied the mask for its keys' global positions (attn_run does so only for
 * the part that holds the sequence's last keys).  Errors: NULL pointers,
 * misalignment, sizes out of range (n_parts 1..65536, D 64 or 128); nothing
 * is launched then.
 *
 * Source: the log-sum-exp merge of split partials (AstrAI commit log for
 * csrc/kernels/gqa_decode_attn.cu, split-KV commit) and the reduction of the
 * running (m, l, O) state between devices (kernbench2 docs/adr-proposed
 * commit log, GQA entry), here as one all-gather and a local merge.
 */
int attn_merge_lse(int n_parts, const void *outs, const float *lses, int64_t T_q, const int32_t *cu_q,
                   int B_max, int Hq, int D, void *out, float *lse, void *stream);

/*
 * attn_check_error -- synchronise `stream`, then read and clear the plan's
 * sticky device error bits (ATTN_DEV_ERR_*) into *flags.  When a bit was set
 * it also resets the plan's merge tickets, so the plan stays usable after a
 * call that stopped early (for instance one whose bounded waits ran out:
 * ATTN_DEV_ERR_TIMEOUT; see attn_overrides.wait_limit_us).  It also clears
 * the attn_overrides.test_stall hook.  The only entry point that waits for the GPU; do
 * not call it inside stream capture.
 */
int attn_check_error(attn_plan_t plan, void *stream, uint32_t *flags);

/* Free the plan's device memory.  NULL or an unknown handle is ignored.  The
 * caller must make sure no work that uses the plan is still pending. */
void attn_destroy(attn_plan_t plan);

/* Static message for an ATTN_* return code. */
const char *attn_strerror(int code);

/*
 * attn_run_noalloc -- one attention call for callers that cannot allocate
 * device memory.  The pages have no counterpart: this is a convenience of
 * this library.
 *
 * Who needs it: a caller whose host framework owns the device memory budget
 * through its own pool allocator (a raw cudaMalloc by a library escapes the
 * pool's accounting and can fail once the pool holds the device), or a caller
 * on a latency-critical path where cudaMalloc / cudaFree may synchronise the
 * device.  Such callers cannot make a plan, since attn_plan allocates.
 *
 * Arguments: the shape (B_max, s_max, Hq, Hkv, D, max_q; same meaning and
 * limits as attn_plan) followed by the tensors and stream of attn_run (same
 * layout, alignment and ownership rules).  Results match attn_run within the
 * library's tolerance; the CUDA-core split kernel is used for every shape.
 *
 * Scratch: a file-scope device array of ATTN_NOALLOC_SCRATCH_BYTES inside the
 * library, held by every GPU that loads the library until the process exits.
 * A shape whose split partials would not fit is rejected with
 * ATTN_E_SCRATCH_LIMIT and nothing is launched.  The call allocates nothing
 * (no cudaMalloc, no cudaFree, no allocating library routine).
 *
 * The first call on each device looks up the array's device address and sets
 * a kernel attribute; make that first call before any stream capture begins.
 * With CUDA's lazy module loading (the default since CUDA 12.2) the array's
 * device memory is committed at that first call, not when the library is
 * loaded: a caller whose pool allocator reserves the device's memory should
 * make the first call on each device before the pool takes its reservation,
 * or the first call can fail with ATTN_E_CUDA.
 * All calls on a device share the array and leave their contents in it; each
 * call clears the parts that must start at zero on its own stream.  Calls
 * that overlap on the GPU race on the array: order them (one stream, or
 * events).  Device-detected length errors leave those rows unwritten, as in
 * attn_run, but are not reported (there is no plan to read them from).
 */
#define ATTN_NOALLOC_SCRATCH_BYTES (4u << 20)
int attn_run_noalloc(int B_max, int s_max, int Hq, int Hkv, int D, int max_q,
                     const void *q, const void *k, const void *v,
                     const int32_t *cu_q, const int32_t *cu_k, void *out,
                     float *lse, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* VARLEN_GQA_H */
