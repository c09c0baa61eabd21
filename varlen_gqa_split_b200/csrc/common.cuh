// common.cuh -- device-side building blocks shared by the split and combine
// kernels of libvgqa (sm_100a): parameter block, error bits, bounded
// mbarrier waits, TMA tile loads, warp-level tensor-core fragments.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/varlen_gqa.h"
#include "params.h"

namespace vgqa {

// log2(e): scores are kept in base-2 units inside the kernels so the softmax
// uses the SFU's exp2 directly; lse is converted back to natural log at the end.
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Default upper bound on one wait, in nanoseconds of %globaltimer (a plan may
// set another in Params::wait_ns).  A healthy wait lasts microseconds; past
// the bound the kernel records ATTN_DEV_ERR_TIMEOUT and leaves instead of
// spinning forever.  Drains (a block waiting for its own copies in flight
// before it exits) always use this default.
constexpr unsigned long long kWaitLimitNs = kDefaultWaitNs;

// Index of the partial state of query row (b, qi, h) for split z.
__device__ __forceinline__ long long part_index(const Params &p, int b, int qi, int h, int z) {
    return (((long long)b * p.max_q + qi) * p.Hq + h) * p.nsplit + z;
}

// Chunks of a sequence with Lk keys that hold work.  Chunk 0 always counts,
// so a sequence without keys still produces its (empty) partial and, through
// the merge, its defined output (out = 0, lse = -inf).
__device__ __forceinline__ int live_chunks(int Lk, int chunk) {
    return Lk > 0 ? (Lk + chunk - 1) / chunk : 1;
}

// Reads the lengths of sequence b and checks them against the plan.  Returns
// false (and, when `report`, records the reason) if the sequence must be
// skipped.  The same test runs in every kernel that touches the sequence.
// spec: a speculative read made before the kernel has waited for the one it
// depends on (the value may still change); it goes to L2 only, so that no
// line of cu_seqlens stays in L1 for the later, real reads to hit.
__device__ __forceinline__ bool load_lengths(const Params &p, int b, bool report,
                                             int &q0, int &Lq, int &k0, int &Lk, bool spec = false) {
    q0 = spec ? __ldcg(p.cu_q + b) : __ldg(p.cu_q + b);
    const int q1 = spec ? __ldcg(p.cu_q + b + 1) : __ldg(p.cu_q + b + 1);
    k0 = spec ? __ldcg(p.cu_k + b) : __ldg(p.cu_k + b);
    const int k1 = spec ? __ldcg(p.cu_k + b + 1) : __ldg(p.cu_k + b + 1);
    Lq = q1 - q0;
    Lk = k1 - k0;
    uint32_t bad = 0;
    if (q0 < 0 || k0 < 0 || Lq < 0 || Lk < 0) bad |= ATTN_DEV_ERR_OFFSETS;
    else {
        if (Lq > p.max_q) bad |= ATTN_DEV_ERR_Q_TOO_LONG;
        if (Lk > p.s_max) bad |= ATTN_DEV_ERR_K_TOO_LONG;
    }
    if (bad && report) atomicOr(p.err, bad);
    return bad == 0;
}

// Paged K/V: the page holding key j of sequence b, from the block table, in
// two steps so that the table read can overlap a wait: page_entry() issues
// the read, page_checked() validates the value.  An entry outside
// [0, num_pages) raises ATTN_DEV_ERR_PAGE and gives num_pages, a page past
// the cache: tensor-map loads of it fill zeros and the CUDA-core path skips
// it, so a bad table never reads outside the cache.
__device__ __forceinline__ int page_entry(const Params &p, int b, int j) {
    // volatile: stays ahead of the (volatile) barrier wait that follows it,
    // so the read is in flight during the wait
    int pg;
    asm volatile("ld.global.nc.b32 %0, [%1];"
                 : "=r"(pg)
                 : "l"(p.block_table + (long long)b * p.bt_stride + (j >> p.page_shift)));
    return pg;
}
__device__ __forceinline__ int page_checked(const Params &p, int pg) {
    if ((unsigned)pg >= (unsigned)p.num_pages) {
        atomicOr(p.err, ATTN_DEV_ERR_PAGE);
        return p.num_pages;
    }
    return pg;
}
__device__ __forceinline__ int page_of(const Params &p, int b, int j) { return page_checked(p, page_entry(p, b, j)); }

// pull the block-table entries of keys [0, Lk) of sequence b into L2 (one
// prefetch per 128-byte line), so the per-tile reads that follow hit there
// (the caller's lane `first` of `step` lanes takes every step-th line)
__device__ __forceinline__ void prefetch_pages(const Params &p, int b, int Lk, int first = 0, int step = 1) {
    const int32_t *row = p.block_table + (long long)b * p.bt_stride;
    const int n = (Lk + (1 << p.page_shift) - 1) >> p.page_shift;
    for (int i = 32 * first; i < n; i += 32 * step) asm volatile("prefetch.global.L2 [%0];" ::"l"(row + i));
}

constexpr int kMaxPageBoxes = 8;          // paged K/V: boxes per 64-key tile at the smallest page (8 keys)

// ------------------------------------------------------------ small math

__device__ __forceinline__ float ex2(float x) {   // SFU exp2 (ex2(-inf) = +0)
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);   // .x (low half) = lo
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

// make barrier initialisation visible to the async (TMA) proxy
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

// raise the barrier's expected transaction count without arriving (the
// arrival that completes the phase comes later)
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete.  Bounded: returns
// false after limit_ns (the caller then records ATTN_DEV_ERR_TIMEOUT and
// unwinds).
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity,
                                          unsigned long long limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer() - t0 > limit_ns) return false;
    }
    return true;
}

// ------------------------------------------------------------ TMA

// 3-D tiled bulk tensor load into shared memory, completing
// `bar`'s transaction count.  coords: {c0 innermost, c1, c2}.
__device__ __forceinline__ void tma_load_3d(void *smem_dst, const CUtensorMap *map, uint64_t *bar,
                                            int c0, int c1, int c2, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2),
        "l"(policy)
        : "memory");
}

__device__ __forceinline__ void tma_load_4d(void *smem_dst, const CUtensorMap *map, uint64_t *bar,
                                            int c0, int c1, int c2, int c3, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5, %6}], [%2], %7;" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
        "l"(policy)
        : "memory");
}

// L2 prefetch of a tile (no shared memory, no barrier): a hint, and safe at
// any coordinates, since the tensor map bounds what it may touch
__device__ __forceinline__ void tma_prefetch_3d(const CUtensorMap *map, int c0, int c1, int c2) {
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1), "r"(c2)
                 : "memory");
}
__device__ __forceinline__ void tma_prefetch_4d(const CUtensorMap *map, int c0, int c1, int c2, int c3) {
    asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1), "r"(c2), "r"(c3)
                 : "memory");
}

__device__ __forceinline__ void tma_load_5d(void *smem_dst, const CUtensorMap *map, uint64_t *bar,
                                            int c0, int c1, int c2, int c3, int c4, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5, %6, %7}], [%2], %8;" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4),
        "l"(policy)
        : "memory");
}

// 1-D bulk copy global -> shared, completing `bar`'s
// transaction count.  dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void *smem_dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(smem_dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// order this thread's earlier generic-proxy shared-memory accesses before its
// later async-proxy (bulk copy) accesses
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// L2 policy for data read exactly once (the K/V stream)
__device__ __forceinline__ uint64_t l2_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ uint64_t l2_evict_last() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// stores that ask the L2 to keep the line (data read back soon by another block)
__device__ __forceinline__ void st_keep_f4(float4 *ptr, float4 v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(ptr), "f"(v.x), "f"(v.y),
                 "f"(v.z), "f"(v.w), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void st_keep_f2(float2 *ptr, float2 v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v2.f32 [%0], {%1, %2}, %3;" ::"l"(ptr), "f"(v.x), "f"(v.y), "l"(pol)
                 : "memory");
}

// ------------------------------------------------------------ warp MMA

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t &r0, uint32_t &r1,
                                              uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// D = A(16x16, row) * B(16x8, col) + D ; bf16 inputs, fp32 accumulate
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// transpose an 8x8 b16 matrix held as one warp fragment
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// ------------------------------------------------------------ cp.async

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void *src, bool full) {
    // src-size 0 fills the 16 bytes with zeros and reads nothing
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(full ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// atomic add with release (orders this block's earlier writes, made visible to
// this thread by a preceding barrier) and acquire (orders later reads) at GPU
// scope; returns the old value
__device__ __forceinline__ uint32_t atom_add_acq_rel_gpu(uint32_t *p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// atomic add with release at GPU scope (no result)
__device__ __forceinline__ void red_add_release_gpu(uint32_t *p, uint32_t v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// named barrier over `nthreads` threads (a subset of the block)
__device__ __forceinline__ void named_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

}  // namespace vgqa

namespace vgqa {

// ------------------------------------------------------------ fused merge

// Called by every participating thread of a block after it wrote its
// partials.  Each thread fences its own writes, the block synchronises, and
// one thread takes a ticket for the unit; the block that takes the last of
// the n_live tickets returns true (in all its threads) and must merge the
// unit, then reset the ticket.  No block ever waits for another.
__device__ __forceinline__ bool ticket_last(uint32_t *ticket, int n_live, int tid, int nthreads, int bar,
                                            volatile int *flag) {
    __threadfence();
    named_sync(bar, nthreads);
    if (tid == 0) *flag = atomicAdd(ticket, 1u) == (uint32_t)(n_live - 1);
    named_sync(bar, nthreads);
    const bool last = *flag != 0;
    if (last) __threadfence();
    return last;
}

// Log-sum-exp merge of the n_live partials of rows [r_begin, r_begin + nrows)
// of (sequence b, KV head hk), by `nthreads` threads of one block, writing the
// final output and lse.  Partials are read through L2 (ld.global.cg): other
// blocks wrote them.  `ws` is shared scratch of nrows * (n_live + 1) * 8 bytes.
template <int D>
__device__ void merge_unit(const Params &p, int b, int q0, int hk, int r_begin, int nrows, int n_live,
                           void *ws, int tid, int nthreads, int bar) {
    float2 *ml = reinterpret_cast<float2 *>(ws);          // [nrows][n_live] -> (weight, l)
    float2 *rowML = ml + nrows * n_live;                  // [nrows] (M, L)
    const int G = p.G;
    for (int idx = tid; idx < nrows * n_live; idx += nthreads) {
        const int r = idx / n_live, z = idx % n_live;
        const int row = r_begin + r;
        ml[idx] = __ldcg(p.ml_part + part_index(p, b, row / G, hk * G + row % G, z));
    }
    named_sync(bar, nthreads);
    const int warp = tid >> 5, lane = tid & 31;
    for (int r = warp; r < nrows; r += nthreads / 32) {
        float M = -INFINITY;
        for (int z = lane; z < n_live; z += 32) {
            const float2 x = ml[r * n_live + z];
            if (x.y > 0.f) M = fmaxf(M, x.x);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        const float Mref = M == -INFINITY ? 0.f : M;
        float L = 0.f;
        for (int z = lane; z < n_live; z += 32) {
            float2 x = ml[r * n_live + z];
            const float w = x.y > 0.f ? ex2(x.x - Mref) : 0.f;
            L += x.y * w;
            x.x = w;
            ml[r * n_live + z] = x;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
        if (lane == 0) rowML[r] = make_float2(M, L);
    }
    named_sync(bar, nthreads);
    for (int idx = tid; idx < nrows * (D / 4); idx += nthreads) {
        const int r = idx / (D / 4), d4 = (idx % (D / 4)) * 4;
        const int row = r_begin + r;
        const int qi = row / G, h = hk * G + row % G;
        const long long base = part_index(p, b, qi, h, 0);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
        for (int z = 0; z < n_live; ++z) {
            const float w = ml[r * n_live + z].x;
            const float4 x = __ldcg(reinterpret_cast<const float4 *>(p.o_part + (base + z) * D + d4));
            acc.x = fmaf(w, x.x, acc.x);
            acc.y = fmaf(w, x.y, acc.y);
            acc.z = fmaf(w, x.z, acc.z);
            acc.w = fmaf(w, x.w, acc.w);
        }
        const float2 ML = rowML[r];
        const float inv = ML.y > 0.f ? 1.f / ML.y : 0.f;
        const long long tok = q0 + qi;
        uint2 pk;
        pk.x = pack_bf16x2(acc.x * inv, acc.y * inv);
        pk.y = pack_bf16x2(acc.z * inv, acc.w * inv);
        *reinterpret_cast<uint2 *>(p.out + (tok * p.Hq + h) * D + d4) = pk;
        if (d4 == 0) p.lse[tok * p.Hq + h] = ML.y > 0.f ? (ML.x + log2f(ML.y)) * kLn2 : -INFINITY;
    }
}

// shared bytes merge_unit needs
__host__ __device__ constexpr size_t merge_smem_bytes(int nrows, int n_live) {
    return (size_t)nrows * (n_live + 1) * 8;
}

}  // namespace vgqa
