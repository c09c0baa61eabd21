// combine_slots.cu -- log-sum-exp merge of the partials written by the
// persistent tensor-core split kernels (the partial-slot layout of
// schedule.cuh: slot 2c holds block c's first cut unit, slot 2c + 1 its last;
// a slot holds rows_per_block rows of D fp32 values plus (m, l) per row, m in
// base-2 units of the scaled scores).
//
// The merge is the one the split-KV method ends with (magik.net "Wiring
// Split-K Dispatch into a Custom CUDA Attention Kernel", section "The
// Message"; AstrAI commit log, split-KV commit): with M = max m_s over the
// parts that saw keys, L = sum l_s 2^(m_s - M), out = sum O_s 2^(m_s - M) / L
// and lse = (M + log2 L) ln 2; no part with keys gives out = 0, lse = -inf.
//
// One block per partial slot, launched as a programmatic dependent of the
// split kernel.  It recomputes the schedule from cu_seqlens while the split
// kernel runs, waits only for the parts of its own unit, and merges one
// column slice of it: the n blocks of a cut unit merge it together, each
// reading 1/n of the partial data, so the merge is spread over as many SMs as
// wrote it (one SM can pull only a few tens of GB/s from L2, too little to
// merge a unit alone).
#include "common.cuh"
#include "kernels.h"
#include "schedule.cuh"

namespace vgqa {

namespace {

using namespace sched;

// Few-part merge of one unit's rows.  A pair of lanes takes 2 * NC
// consecutive 4-column items of one row (the two lanes alternate, so each
// 32-byte sector is read whole by one load instruction of the pair); the
// unit's groups are split evenly over its nb combine blocks (this is block
// bi), and a pair takes a group per step with every load of it -- the
// row's (m, l) of each part once, and its NC items of each part -- in
// flight at once.
template <int D, int NP, int NC, class WriteRow>
__device__ __forceinline__ void merge_few(const Params &p, const int *slots, int n, long long ROWS, int R, int nb,
                                          int bi, WriteRow &&write_row) {
    constexpr int kG = D / 4 / (2 * NC);            // groups per row
    static_assert(kG >= 1, "a group spans at most a row");
    const int groups = R * kG;
    const int per = (groups + nb - 1) / nb;
    const int g_lo = min(groups, bi * per), g_hi = min(groups, g_lo + per);
    const int side = threadIdx.x & 1;
    for (int gi = g_lo + (int)(threadIdx.x >> 1); gi < g_hi; gi += (int)(blockDim.x >> 1)) {
        const int r = gi / kG, c0 = (gi % kG) * 2 * NC + side;      // this lane's first 4-column item
        float2 ml[NP];
        float4 o[NP][NC];
#pragma unroll
        for (int j = 0; j < NP; ++j) {
            if (j < n) {
                const long long sr = (long long)slots[j] * ROWS + r;
                ml[j] = __ldcg(p.ml_part + sr);
                const float4 *src = reinterpret_cast<const float4 *>(p.o_part + sr * D) + c0;
#pragma unroll
                for (int q = 0; q < NC; ++q) o[j][q] = __ldcg(src + 2 * q);
            }
        }
        float M = -INFINITY;
#pragma unroll
        for (int j = 0; j < NP; ++j)
            if (j < n && ml[j].y > 0.f) M = fmaxf(M, ml[j].x);
        const float Mref = M == -INFINITY ? 0.f : M;
        float L = 0.f;
        float4 acc[NC];
#pragma unroll
        for (int q = 0; q < NC; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int j = 0; j < NP; ++j) {
            if (j < n && ml[j].y > 0.f) {
                const float w = ex2(ml[j].x - Mref);
                L = fmaf(w, ml[j].y, L);
#pragma unroll
                for (int q = 0; q < NC; ++q) {
                    acc[q].x = fmaf(w, o[j][q].x, acc[q].x);
                    acc[q].y = fmaf(w, o[j][q].y, acc[q].y);
                    acc[q].z = fmaf(w, o[j][q].z, acc[q].z);
                    acc[q].w = fmaf(w, o[j][q].w, acc[q].w);
                }
            }
        }
#pragma unroll
        for (int q = 0; q < NC; ++q) write_row(r, 4 * (c0 + 2 * q), M, L, acc[q]);
    }
}

// Combine: block 2c + k merges slice (c - c_first) of the unit block c cut at
// its start (k = 0) or end (k = 1), if any.  The block is launched as a
// programmatic dependent of the split kernel, so it computes the schedule
// while the split kernel streams; it then waits (bounded) only for the n parts
// of its own unit, whose writers each add 1 (release) to the unit's count, so
// a unit is merged as soon as its last part lands rather than when the whole
// split grid ends.  Each slot's slice is cut again into S sub-slices, one per
// block, so that a unit with many rows is merged by n * S blocks.  After
// merging, each of the unit's n * S combine blocks adds 1 to the count again;
// the last one resets it for the next call.
template <int D>
__global__ void __launch_bounds__(128, 4) combine_slots_kernel(const Params p, const int C, const int S) {
    constexpr int kCols = D / 4;
    constexpr int kT = 128;
    constexpr int kBatch = 12;             // loads in flight per thread (register budget)
    constexpr int kFewParts = 4;           // up to this many parts: row-group merge (merge_few)
    extern __shared__ __align__(16) uint8_t csm[];
    __shared__ long long scan[kT / 32];
    __shared__ long long first[3];
    __shared__ int ok_flag;
    const int tid = threadIdx.x;
    const int sub = blockIdx.x % S;
    const int c = (blockIdx.x / S) >> 1, k = (blockIdx.x / S) & 1;
    const long long ROWS = p.rows_per_block;     // rows of one partial slot
    // the next call's split kernel may launch now; it waits for this grid to
    // complete before it reads anything
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    Share sh;
    if (!block_share(p, c, C, tid, kT, false, scan, first, sh)) return;
    SegWalker wk;
    wk.init(p, sh.b_first, sh.pb_first, sh.lo, sh.hi);
    Segment seg;
    wk.next(p, seg);
    if (k == 1) {                                 // the block's last unit, when it has two or more
        int nseg = 1;
        while (wk.next(p, seg)) ++nseg;
        if (nseg == 1) return;
    }
    if (seg.t0 == 0 && seg.t1 == seg.w) return;       // whole unit: written by the split kernel
    const long long T = sh.T;
    const int Ce = sh.Ce;
    const int c_first = block_of(seg.Pu, T, Ce);
    const int n = block_of(seg.Pu + seg.w - 1, T, Ce) - c_first + 1;
    // the row tile's tokens [tq0, tq0 + nq) of the sequence; partial row r is
    // token tq0 + r / G, head r % G of the KV head's group
    const int tq0 = rt_first(seg.s, seg.rt, p.qtile);
    const int nq = seg.s.Lq - seg.rt * p.qtile - tq0;
    const int G = p.G, R = G * nq;
    const int items = R * kCols;
    const int nb = n * S;                          // blocks merging this unit
    const int per = (items + nb - 1) / nb;
    const int it_lo = min(items, ((c - c_first) * S + sub) * per), it_hi = min(items, it_lo + per);
    const long long u = unit_index(p, seg.b, seg.hk, seg.rt);

    int *slots = reinterpret_cast<int *>(csm);                         // [n]
    for (int j = tid; j < n; j += kT) slots[j] = slot_of(c_first + j, seg.Pu, T, Ce);

    // wait for the unit's n parts, each published by done_per_part release
    // adds (the acquire pairs with them); p.stall adds parts that never come
    // (a test hook, 0 otherwise), so that the bounded wait below runs out
    const uint32_t parts_done = (uint32_t)(n * p.done_per_part) + __ldg(p.stall);
    if (tid == 0) {
        int ok = 1;
        if (ld_acquire_gpu(p.done + u) < parts_done) {
            const unsigned long long t0 = globaltimer();
            while (ld_acquire_gpu(p.done + u) < parts_done) {
                if (globaltimer() - t0 > p.wait_ns) {
                    atomicOr(p.err, ATTN_DEV_ERR_TIMEOUT);
                    ok = 0;
                    break;
                }
                __nanosleep(256);
            }
        }
        ok_flag = ok;
        if (ok && c == c_first && sub == 0) p.claim[u] = 0ull;          // claims, next call
    }
    __syncthreads();
    if (!ok_flag) return;

    auto write_row = [&](int r, int d4, float Mt, float Lt, float4 acc) {
        const float inv = Lt > 0.f ? 1.f / Lt : 0.f;
        const int qi = tq0 + r / G, h = seg.hk * G + r % G;
        const long long tok = seg.s.q0 + qi;
        uint2 pk;
        pk.x = pack_bf16x2(acc.x * inv, acc.y * inv);
        pk.y = pack_bf16x2(acc.z * inv, acc.w * inv);
        *reinterpret_cast<uint2 *>(p.out + (tok * p.Hq + h) * D + d4) = pk;
        if (d4 == 0) p.lse[tok * p.Hq + h] = Lt > 0.f ? (Mt + log2f(Lt)) * kLn2 : -INFINITY;
    };
    if (n <= kFewParts) {
        // few parts: a thread merges NC consecutive 4-column items of one row
        // per step, with all their loads (and the row's (m, l) of each part,
        // read once) in flight together: the merge is latency-bound, so the
        // fewer dependent round trips the better
        const int bi = (c - c_first) * S + sub;            // this block among the unit's nb
        if (n <= 2)
            merge_few<D, 2, 8>(p, slots, n, ROWS, R, nb, bi, write_row);
        else
            merge_few<D, kFewParts, 4>(p, slots, n, ROWS, R, nb, bi, write_row);
        __syncthreads();
        if (tid == 0 && atomicAdd(p.done + u, 1u) == parts_done + (uint32_t)(nb - 1)) p.done[u] = 0u;
        return;
    }

    // many parts: two threads per item (row, 4 columns), each merging every
    // other part with a running max, kBatch loads in flight; the pair then
    // combines
    const int n_work = 2 * (it_hi - it_lo);
    for (int base = 0; base < n_work; base += kT) {
        const int w = base + tid;
        const bool valid = w < n_work;
        const int it = it_lo + (valid ? w >> 1 : 0), half = w & 1;
        const int r = it / kCols, d4 = (it % kCols) * 4;
        float M = -INFINITY, L = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (valid) {
            for (int j0 = half; j0 < n; j0 += 2 * kBatch) {
                float2 ml[kBatch];
                float4 o[kBatch];
#pragma unroll
                for (int q = 0; q < kBatch; ++q) {
                    const int j = j0 + 2 * q;
                    if (j < n) {
                        const long long sl = slots[j];
                        ml[q] = __ldcg(p.ml_part + sl * ROWS + r);
                        o[q] = __ldcg(reinterpret_cast<const float4 *>(p.o_part + (sl * ROWS + r) * D + d4));
                    }
                }
#pragma unroll
                for (int q = 0; q < kBatch; ++q) {
                    if (j0 + 2 * q < n && ml[q].y > 0.f) {
                        const float Mn = fmaxf(M, ml[q].x);
                        const float a = ex2(M - Mn), wq = ex2(ml[q].x - Mn);   // ex2(-inf) = 0
                        acc.x = fmaf(acc.x, a, wq * o[q].x);
                        acc.y = fmaf(acc.y, a, wq * o[q].y);
                        acc.z = fmaf(acc.z, a, wq * o[q].z);
                        acc.w = fmaf(acc.w, a, wq * o[q].w);
                        L = fmaf(L, a, wq * ml[q].y);
                        M = Mn;
                    }
                }
            }
        }
        // combine the pair (adjacent lanes)
        const float M2 = __shfl_xor_sync(0xffffffffu, M, 1);
        const float L2 = __shfl_xor_sync(0xffffffffu, L, 1);
        float4 a2;
        a2.x = __shfl_xor_sync(0xffffffffu, acc.x, 1);
        a2.y = __shfl_xor_sync(0xffffffffu, acc.y, 1);
        a2.z = __shfl_xor_sync(0xffffffffu, acc.z, 1);
        a2.w = __shfl_xor_sync(0xffffffffu, acc.w, 1);
        if (valid && half == 0) {
            const float Mt = fmaxf(M, M2);
            const float Mref = Mt == -INFINITY ? 0.f : Mt;
            const float s1 = ex2(M - Mref), s2 = ex2(M2 - Mref);
            write_row(r, d4, Mt, L * s1 + L2 * s2,
                      make_float4(acc.x * s1 + a2.x * s2, acc.y * s1 + a2.y * s2, acc.z * s1 + a2.z * s2,
                                  acc.w * s1 + a2.w * s2));
        }
    }
    __syncthreads();
    // every combine block of the unit has seen its n parts once each of the
    // n * S blocks has added 1 more: the last one resets the count
    if (tid == 0 && atomicAdd(p.done + u, 1u) == parts_done + (uint32_t)(nb - 1)) p.done[u] = 0u;
}



}  // namespace

size_t combine_slots_smem(int ctas) { return (size_t)((ctas + 3) & ~3) * 4; }

cudaError_t combine_slots_prepare(int D, int ctas) {
    void *fn = D == 64 ? reinterpret_cast<void *>(combine_slots_kernel<64>)
                       : reinterpret_cast<void *>(combine_slots_kernel<128>);
    return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)combine_slots_smem(ctas));
}

int combine_slots_split(int rows, int D) {
    // about 2048 (row, 4-column) items per block at most, up to 8 blocks per
    // slot (1024: 1184 blocks on the short-query workload, two waves of 592
    // resident blocks, 47.9 us per call; 2048: 592 blocks, 47.6 us)
    const int items = rows * (D / 4);
    const int S = (items + 2047) / 2048;
    return S < 1 ? 1 : (S > 8 ? 8 : S);
}

cudaError_t launch_combine_slots(const Params &p, int ctas, cudaStream_t stream) {
    // launched as a programmatic dependent: its blocks may start (and compute
    // the schedule) before the split kernel has finished
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    int S = combine_slots_split(p.G * p.max_q, p.D);
    cfg.gridDim = dim3(2 * ctas * S);
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = combine_slots_smem(ctas);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void *fn = p.D == 64 ? reinterpret_cast<void *>(combine_slots_kernel<64>)
                         : reinterpret_cast<void *>(combine_slots_kernel<128>);
    void *args[] = {const_cast<Params *>(&p), &ctas, &S};
    return cudaLaunchKernelExC(&cfg, fn, args);
}

}  // namespace vgqa
