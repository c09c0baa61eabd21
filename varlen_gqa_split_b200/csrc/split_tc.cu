// split_tc.cu -- persistent TMA-fed split-KV kernel on the fifth-generation
// tensor cores (tcgen05, accumulators in tensor memory) for short-query row
// counts: 128 query rows (G heads x 128 / G query tokens) per unit, and
// longer queries as several row tiles of the sequence, each its own unit.
//
// Same schedule as the warp-MMA kernel (schedule.cuh: equal shares of the
// flattened 64-key tiles; by default the shares stay static on this path,
// without run-time claims; cut units are merged by the slot combine kernel,
// or, instantiated with FUSED, by the block holding each one's last part), but
// the G query heads times the q_len query tokens of a unit form the M = 128
// side of real tensor-core tiles (kernbench2 docs/adr-proposed commit log,
// GQA entry: G folded into the matmul M dimension; every K/V byte is read
// once per KV head).  A pipeline stage holds two of the schedule's 64-key
// tiles of one unit (128 keys), so that both products run as wide
// instructions and every barrier round trip is paid once per 128 keys:
//     S [128 rows x 128 keys] = Q [128 x D] . K^T     (tcgen05.mma, Q and S in tensor memory)
//     O [128 rows x D]       += P [128 x 128 keys] . V (P bf16 and O in tensor memory)
// A stage whose second tile is absent (the end of a block's part of a unit)
// runs S with N = 64 and the product over its 64 keys only.
//
// Tensor memory (512 columns): S in two buffers of 128 columns, O (D
// columns), the unit's Q (D / 2 columns of bf16 pairs) and P (64 columns of
// bf16 pairs).  Q is read from tensor memory by the first product, so the
// tensor core reads only K from shared memory for it.
//
// Warp roles (320 threads):
//   warp 9 -- producer (the whole warp walks the schedule in step, each lane
//     issuing one box, lane 0 taking claims and stage bookkeeping): for each
//     unit it loads the unit's Q tile into a ring stage (one TMA box per
//     D-half of G heads x qtile tokens, right-aligned so it ends at the row
//     tile's last query token; rows past the sequence's own tokens are never
//     written), then pairs the unit's K and V tiles into 128-key stages;
//   warp 8, one lane -- MMA issuer: S(j) = Q K_j^T into one of two S
//     buffers, then O += P(j-1) V_{j-1}, so the softmax of stage j overlaps
//     the second product of stage j-1 (a unit's last stage is not held back:
//     its second product follows at once); completion is tracked with
//     tcgen05.commit on mbarriers; the warp also allocates and frees the
//     tensor memory;
//   warps 0-7 -- softmax and epilogue.  Warp w reads tensor-memory lanes
//     32 (w mod 4) .. +31, one query row per thread, and half h = w / 4 of
//     every stage (its 64-key tile h).  The two warps of a row exchange their
//     halves' maxima through shared memory once per stage, so both take the
//     same running max and add into the one O accumulator; each keeps its own
//     running sum.  The scores are masked (keys before the tile's own start
//     when the tile was right-aligned, and keys past Lk - Lq + qi under the
//     tail-aligned causal mask), and P is written as bf16 pairs into tensor
//     memory, from where the second product reads its A operand.  They also
//     copy each unit's Q from its ring stage into tensor memory (each warp its
//     lanes and half of D), ahead of the previous unit's epilogue, and write
//     the epilogue: each warp its half of D.
//
// The running max is rescaled lazily: O in tensor memory is multiplied by
// 2^(m_old - m_new) only when a row's max grows by more than 2^8 (rare after
// the first stage); otherwise the stage's weights are taken relative to the
// stale max, which stays exact in fp32 and keeps P below 2^8 in bf16.  The
// partial (O, m, l) and the final normalisation use whatever reference max
// the row ended with, so the result is the same softmax.
//
// Every wait on an mbarrier is bounded; a wait that gives up records
// ATTN_DEV_ERR_TIMEOUT, raises a block-wide stop flag that the other roles'
// waits also watch, and the block drains its issued tensor-core work before
// freeing the tensor memory and returning.
#include "common.cuh"
#include "kernels.h"
#include "schedule.cuh"
#include "tc.cuh"

namespace vgqa {

namespace {

using namespace sched;

constexpr int kRows = 128;                // MMA M: query rows of a unit
constexpr int kSub = 2;                   // schedule tiles per pipeline stage
constexpr int kStageKeys = kSub * kBN;    // 128 keys
constexpr int kSoftWarps = 8;             // two per tensor-memory lane quarter (tile halves)
constexpr int kMmaWarp = 8;               // sub-partition 0: its rows are the last to hold query rows
constexpr int kProducerWarp = 9;
constexpr int kThreads = 320;
constexpr int kMetaLast = 1;              // stage flag: the block's last stage of the unit
constexpr int kMetaEmpty = 2;             // stage flag: no data, the unit ends here
constexpr int kMetaQ = 4;                 // stage flag: the unit's Q tile
constexpr int kMetaEnd = 8;               // stage flag: no data, the block's work ends here
constexpr int kSegRing = 16;              // unit descriptors in flight (see UnitDesc)
constexpr float kRescaleLog2 = 8.f;       // lazy rescale threshold (base-2 units)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;             // S(j) in [128 (j mod 2), +128)
constexpr uint32_t kColO = 256;           // O, D columns
constexpr uint32_t kColQ = 384;           // Q, D / 2 columns of bf16 pairs
constexpr uint32_t kColP = 448;           // P, 64 columns of bf16 pairs
constexpr size_t kMinSmemBytes = 120 * 1024;

template <int D>
struct TcLayout {
    static constexpr int kHalves = D / 64;                  // 128-byte swizzle atoms per row
    static constexpr int kSubRows = kBN * 128;              // one 64-key tile of one atom column
    static constexpr int kKvRegion = kStageKeys * 128;      // 128 keys x 128 B
    static constexpr int kKvTile = kHalves * kKvRegion;     // K or V of a stage
    static constexpr int kStage = 2 * kKvTile;              // K + V
    static constexpr int kQRegion = kRows * 128;            // 128 rows x 128 B
    static constexpr uint32_t kTileBytes = 2u * kHalves * kSubRows;   // K + V of one 64-key tile
    static constexpr int kOCols = D / 2;                    // O columns per softmax warp
    static constexpr int kQCols = D / 4;                    // Q columns (bf16 pairs) per softmax warp
};

// What the softmax warps need of a unit, written by the producer with the
// unit's Q stage into a ring of kSegRing entries (entry k mod kSegRing for
// the block's k-th unit).  The producer can run at most `stages` stages (<= 8)
// ahead of the softmax warps and every unit takes at least two stages, so an
// entry is rewritten only after the softmax warps have left its unit.
struct UnitDesc {
    int b, hk, rt, role;                  // role 0: the unit is the block's alone; 1, 2: cut (OrderedWalker)
    int q0, Lq, Lk, w;                    // w: the unit's positions in the flattened tile space
    long long Pu;                         // global index of its first position
    long long pad;
};

// packed fp32 pairs (one instruction for two lanes' worth of FMA / add)
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    unsigned long long ra, rb, rc, rd;
    asm("mov.b64 %0, {%1, %2};" : "=l"(ra) : "f"(a.x), "f"(a.y));
    asm("mov.b64 %0, {%1, %2};" : "=l"(rb) : "f"(b.x), "f"(b.y));
    asm("mov.b64 %0, {%1, %2};" : "=l"(rc) : "f"(c.x), "f"(c.y));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(rd) : "l"(ra), "l"(rb), "l"(rc));
    float2 d;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(d.x), "=f"(d.y) : "l"(rd));
    return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
    unsigned long long ra, rb, rd;
    asm("mov.b64 %0, {%1, %2};" : "=l"(ra) : "f"(a.x), "f"(a.y));
    asm("mov.b64 %0, {%1, %2};" : "=l"(rb) : "f"(b.x), "f"(b.y));
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(rd) : "l"(ra), "l"(rb));
    float2 d;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(d.x), "=f"(d.y) : "l"(rd));
    return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// bounded mbarrier wait that also gives up when another role raised the stop flag
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *stop, const Params &p,
                                         unsigned long long factor = 1) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if (*stop) return false;
        if (globaltimer() - t0 > p.wait_ns * factor) {
            atomicOr(p.err, ATTN_DEV_ERR_TIMEOUT);
            *stop = 1;
            return false;
        }
    }
    return true;
}

// PAGED: K and V come from a paged cache (block table); FUSED: the fused
// merge (head-first unit order, the merge after the unit loop).  Separate
// instantiations keep each kernel free of the code it does not run.
template <int D, bool PAGED, bool FUSED>
__global__ void __launch_bounds__(kThreads, 1) split_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                               const __grid_constant__ CUtensorMap tm_k,
                                                               const __grid_constant__ CUtensorMap tm_v,
                                                               const Params p, const int stages) {
    using L = TcLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ring = smem;                                    // [stages][K | V], or a unit's Q tile
    uint64_t *full = reinterpret_cast<uint64_t *>(ring + stages * L::kStage);
    uint64_t *empty = full + stages;
    uint64_t *q_tm = empty + stages;         // the unit's Q is in tensor memory
    uint64_t *q_ack = q_tm + 1;              // the MMA issuer has taken it (Q may be replaced)
    uint64_t *s_full = q_ack + 1;            // [2] S(j) computed (j mod 2)
    uint64_t *s_free = s_full + 2;           // [2] S(j) read by the softmax warps
    uint64_t *p_full = s_free + 2;           // [2] P(j) written
    uint64_t *o_done = p_full + 2;           // [2] O += P(j) V(j) done
    uint64_t *o_free = o_done + 2;           // O read by the epilogue
    uint64_t *xbar = o_free + 1;             // [4] the two warps of a lane quarter exchanged a value
    uint64_t *drain = xbar + 4;              // all issued tensor-core work done
    uint64_t *mg = drain + 1;                // fused merge: the other parts are published ([2]: alignment)
    int4 *meta = reinterpret_cast<int4 *>(mg + 2);                            // [stages]
    UnitDesc *units = reinterpret_cast<UnitDesc *>(meta + stages);           // [kSegRing]
    float *xbuf = reinterpret_cast<float *>(units + kSegRing);               // [2][2 halves][128]
    float2 *mstash = reinterpret_cast<float2 *>(xbuf + 4 * kRows);           // [kSoftWarps * 32] fused merge
    long long *scan = reinterpret_cast<long long *>(mstash + kSoftWarps * 32); // [kThreads / 32]
    long long *first = scan + kThreads / 32;                                 // [3]
    volatile int *stop = reinterpret_cast<volatile int *>(first + 3);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(first + 3) + 1;
    volatile int *mflag = reinterpret_cast<volatile int *>(first + 3) + 2;   // fused merge: 1 parts ready, 2 not

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    // the block's share: consecutive blocks (which the hardware tends to
    // place on neighbouring SMs) take shares far apart, so every unit shared
    // by several blocks gets a mix of SMs rather than one neighbourhood
    const int c = (int)(((long long)blockIdx.x * p.share_stride) % gridDim.x);

    if (tid == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1 + kSoftWarps);   // the MMA issuer (commit or arrival) + each softmax warp
        }
        mbar_init(q_tm, kSoftWarps);
        mbar_init(q_ack, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&s_free[i], kSoftWarps);
            mbar_init(&p_full[i], kSoftWarps);
            mbar_init(&o_done[i], 1);
        }
        mbar_init(o_free, kSoftWarps);
        for (int i = 0; i < 4; ++i) mbar_init(&xbar[i], 2);
        mbar_init(drain, 1);
        mbar_init(mg, 1);
        *stop = 0;
        fence_barrier_init();
    }
    if (tid == kProducerWarp * 32) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    if (warp == kMmaWarp) {
        tc::tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tc::tmem_relinquish();
    }
    // Launched as a programmatic dependent, the block may start while the
    // previous kernel in the stream still runs.  Meanwhile it prefetches its
    // first K/V tiles into L2 under a speculative schedule (the warp-MMA
    // kernel does the same; both are hints that no later write can make
    // stale).  Then it waits for that kernel before the reads that count;
    // only then may this call's combine kernel launch.
    if constexpr (!PAGED) {
        Share sp;
        if (block_share(p, c, gridDim.x, tid, kThreads, false, scan, first, sp, true) && warp == kProducerWarp)
            first_tiles<FUSED>(p, c, sp, kPrefetchBytes / (int)L::kTileBytes, true, [&](const Segment &sg, int t) {
                const int row = sg.s.k0 + min(t * kBN, sg.s.Lk - kBN);
#pragma unroll
                for (int hf = 0; hf < L::kHalves; ++hf) {
                    tma_prefetch_3d(&tm_k, hf * 64, sg.hk, row);
                    tma_prefetch_3d(&tm_v, hf * 64, sg.hk, row);
                }
            });
        __syncthreads();   // scan / first are reused below
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    Share sh;
    const bool has_work = block_share(p, c, gridDim.x, tid, kThreads, c == 0, scan, first, sh);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const int G = p.G, QT = p.qtile;                         // query tokens per row tile

    if (has_work && warp == kProducerWarp) {

        // ---------------------------------------------------------- producer
        // the whole warp walks the schedule in step and each lane loads one
        // box of a tile (a D-half of K or V; up to 32 boxes from small
        // pages), lane 0 doing the rest
        const unsigned wmask = 0xffffffffu;
        const bool leader = lane == 0;
        const uint64_t pol = l2_evict_first();
        const uint32_t q_bytes = (uint32_t)(L::kHalves * G * QT * 128);
        int s = 0, issued = 0;
        uint32_t phase = 0;
        int nseg = 0;                        // units begun
        int nsub = 0;                        // tiles in the open stage (0: none open)
        int ks_a = 0, ks_b = 0;              // key starts of the open stage's tiles
        auto wait_all = [&](uint64_t *bar, uint32_t parity) -> bool {
            return __all_sync(wmask, wait_bar(bar, parity, stop, p));
        };
        auto acquire = [&]() -> bool { return issued < stages || wait_all(&empty[s], phase ^ 1); };
        auto advance = [&]() {
            ++issued;
            if (++s == stages) {
                s = 0;
                phase ^= 1;
            }
        };
        // the open stage is complete: its key starts and flags, then the
        // arrival that lets its phase finish once its bytes have landed
        auto close = [&](bool last) {
            if (leader) {
                meta[s] = make_int4(ks_a, nsub == 2 ? ks_b : -1, last ? kMetaLast : 0, 0);
                mbar_arrive(&full[s]);
            }
            __syncwarp(wmask);
            nsub = 0;
            advance();
        };
        long long mu = -1;                   // fused merge: the unit whose last part this block holds
        uint32_t mneed = 0;                  // its count once every other part is published
        auto begin = [&](const Segment &sg, int role) -> bool {
            if (FUSED && role == 1 && sg.t1 == sg.w) {
                // the other parts publish kSoftWarps release adds each;
                // p.stall adds parts that never come (a test hook, 0
                // otherwise), so that the bounded wait runs out
                mu = unit_index(p, sg.b, sg.hk, sg.rt);
                mneed = (uint32_t)((c - block_of(sg.Pu, sh.T, sh.Ce)) * kSoftWarps) + __ldg(p.stall);
            }
            if constexpr (PAGED) prefetch_pages(p, sg.b, sg.s.Lk, lane, 32);
            if (!acquire()) return false;
            if (leader) {
                UnitDesc &u = units[nseg % kSegRing];
                u.b = sg.b;
                u.hk = sg.hk;
                u.rt = sg.rt;
                u.role = role;
                u.q0 = sg.s.q0;
                u.Lq = sg.s.Lq;
                u.Lk = sg.s.Lk;
                u.w = sg.w;
                u.Pu = sg.Pu;
                meta[s] = make_int4(0, -1, kMetaQ, nseg);
                mbar_arrive_expect_tx(&full[s], q_bytes);
                // the box ends at the row tile's last query token
                const int t_end = sg.s.q0 + sg.s.Lq - sg.rt * QT;
#pragma unroll
                for (int hf = 0; hf < L::kHalves; ++hf)
                    tma_load_3d(ring + s * L::kStage + hf * L::kQRegion, &tm_q, &full[s], hf * 64, sg.hk * G,
                                t_end - QT, pol);
            }
            __syncwarp(wmask);
            advance();
            ++nseg;
            return true;
        };
        // one 64-key tile: the first or the second of a stage
        auto load_tile = [&](const Segment &sg, int tile, bool last) -> bool {
            const int ks = tile * kBN;
            if constexpr (PAGED) {
                // boxes of page_box keys x one D-half, each from its page:
                // lane l loads box l / (2 halves) of K or V; the table reads
                // go out before the stage wait, so they overlap it
                constexpr int kPer = 2 * L::kHalves;                // loads per box of keys
                const int nbox = kBN / p.page_box, bi = lane / kPer, rem = lane % kPer;
                const int tv = rem / L::kHalves, hf = rem % L::kHalves;
                const bool mine = lane < nbox * kPer;
                const int key = ks + bi * p.page_box;
                const bool in = mine && key < sg.s.Lk;
                const int entry = in ? page_entry(p, sg.b, key) : 0;
                if (nsub == 0 && !acquire()) return false;
                if (leader) mbar_expect_tx(&full[s], L::kTileBytes);
                __syncwarp(wmask);
                uint8_t *st = ring + s * L::kStage;
                if (mine) {
                    // a box past the sequence (or a bad entry) reads page
                    // num_pages, outside the map: zeros
                    const int page = in ? page_checked(p, entry) : p.num_pages;
                    const int slot = key & ((1 << p.page_shift) - 1);       // 0 when pages are < 64 keys
                    uint8_t *dst = st + tv * L::kKvTile + hf * L::kKvRegion + nsub * L::kSubRows +
                                   bi * p.page_box * 128;
                    const CUtensorMap *map = tv ? &tm_v : &tm_k;
                    if (p.page_rows)
                        tma_load_3d(dst, map, &full[s], hf * 64, sg.hk, page * p.page_rows + slot, pol);
                    else
                        tma_load_4d(dst, map, &full[s], hf * 64, sg.hk, slot, page, pol);
                }
            } else {
                if (nsub == 0 && !acquire()) return false;
                if (leader) mbar_expect_tx(&full[s], L::kTileBytes);
                __syncwarp(wmask);
                const int row = sg.s.k0 + min(ks, sg.s.Lk - kBN);
                if (lane < 2 * L::kHalves) {                        // lane: (K or V, D-half)
                    const int tv = lane / L::kHalves, hf = lane % L::kHalves;
                    tma_load_3d(ring + s * L::kStage + tv * L::kKvTile + hf * L::kKvRegion + nsub * L::kSubRows,
                                tv ? &tm_v : &tm_k, &full[s], hf * 64, sg.hk, row, pol);
                }
            }
            // in run-time claims the second tile may precede the first
            if (nsub == 0)
                ks_a = ks;
            else
                ks_b = ks;
            if (++nsub == kSub || last) close(last);
            return true;
        };
        auto empty_stage = [&](const Segment &) -> bool {
            if (nsub) close(false);                                 // a half stage of claimed tiles
            if (!acquire()) return false;
            if (leader) {
                meta[s] = make_int4(0, -1, kMetaLast | kMetaEmpty, 0);
                mbar_arrive(&full[s]);
            }
            __syncwarp(wmask);
            advance();
            return true;
        };
        bool fed = feed_tiles<true, FUSED>(p, sh.b_first, sh.pb_first, sh.lo, sh.hi, begin, load_tile, empty_stage);
        if (nsub) close(false);              // only after a stop: no stage stays without its arrival
        // the end of the block's work, for the consumers
        if (fed && (fed = acquire())) {
            if (leader) {
                meta[s] = make_int4(0, -1, kMetaEnd, 0);
                mbar_arrive(&full[s]);
            }
            __syncwarp(wmask);
            advance();
        }
        if (!fed) *stop = 1;
        // Fused merge: with its tiles all issued, the producer waits
        // (bounded) until the other parts of the unit this block merges are
        // published, so that the softmax warps find them ready when they
        // reach its epilogue (the unit is the block's last: head-first
        // order), and resets the unit's count for the next call -- no block
        // adds to it again in this call.  A part that never came leaves the
        // count set and the rows unwritten; attn_check_error then resets it.
        if (mu >= 0) {
            if (lane == 0) {
                int res = fed ? 1 : 2;
                if (fed && ld_acquire_gpu(p.done + mu) < mneed) {
                    const unsigned long long t0 = globaltimer();
                    while (ld_acquire_gpu(p.done + mu) < mneed) {
                        if (*stop) {
                            res = 2;
                            break;
                        }
                        if (globaltimer() - t0 > p.wait_ns) {
                            atomicOr(p.err, ATTN_DEV_ERR_TIMEOUT);
                            res = 2;
                            break;
                        }
                        __nanosleep(128);
                    }
                }
                if (res == 1) p.done[mu] = 0u;
                *mflag = res;
                mbar_arrive(mg);
            }
            __syncwarp();
        }
        // let the loads in flight land before the block can exit (bounded,
        // also after a stop: the copies target this block's shared memory)
        for (int i = 0; i < min(issued, stages); ++i) {
            if (--s < 0) {
                s = stages - 1;
                phase ^= 1;
            }
            mbar_wait(&full[s], phase);
        }
    } else if (has_work && warp == kMmaWarp) {

        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdS2 = tc::idesc_bf16_f32(kRows, kStageKeys, false);
            constexpr uint32_t kIdS1 = tc::idesc_bf16_f32(kRows, kBN, false);
            constexpr uint32_t kIdO = tc::idesc_bf16_f32(kRows, D, true);
            const uint32_t ring0 = smem_u32(ring);
            int j = 0, k = 0, e = 0, s = 0;
            uint32_t sph = 0;                       // ring position and phase
            bool have_prev = false, ok = true;
            int pj = 0, ps = 0, pe = 0, pn = 0;
            bool pfirst = false;
            auto next_stage = [&](int &cs, int4 &mt) -> bool {
                if (!wait_bar(&full[s], sph, stop, p)) return false;
                mt = meta[s];
                cs = s;
                if (++s == stages) {
                    s = 0;
                    sph ^= 1;
                }
                return true;
            };
            // O += P(pj) V(pj) over the stage's pn tiles: waits for the softmax
            // warps' P and, at a unit's first stage, for the epilogue of the
            // previous unit
            auto issue_pv = [&]() -> bool {
                if (!wait_bar(&p_full[pj & 1], (pj >> 1) & 1, stop, p)) return false;
                if (pfirst && pe >= 1 && !wait_bar(o_free, (pe - 1) & 1, stop, p)) return false;
                tc::fence_after_sync();
                const uint64_t v0 = tc::smem_desc_sw128(ring0 + ps * L::kStage + L::kKvTile, L::kKvRegion, 1024);
#pragma unroll
                for (int kk = 0; kk < kStageKeys / 16; ++kk) {
                    if (kk * 16 < pn * kBN)
                        tc::mma_bf16_ts(tmem + kColO, tmem + kColP + kk * 8, v0 + ((kk * 16 * 128) >> 4), kIdO,
                                        !pfirst || kk > 0);
                }
                tc::commit(smem_u32(&empty[ps]));
                tc::commit(smem_u32(&o_done[pj & 1]));
                return true;
            };
            while (ok) {
                // the unit's Q stage (the softmax warps copy it into tensor
                // memory), or the end of the block's work
                int cs;
                int4 mt;
                if (!(ok = next_stage(cs, mt))) break;
                mbar_arrive(&empty[cs]);
                if (mt.z & kMetaEnd) break;
                if (!(ok = wait_bar(q_tm, k & 1, stop, p))) break;
                mbar_arrive(q_ack);
                ++k;
                bool first = true;
                while (true) {
                    if (!(ok = next_stage(cs, mt))) break;
                    if (mt.z & kMetaEmpty) {
                        // the block's part of the unit ends here: flush the
                        // deferred product of its last stage, if any
                        mbar_arrive(&empty[cs]);
                        if (have_prev) {
                            if (!(ok = issue_pv())) break;
                            have_prev = false;
                            ++e;
                        }
                        break;
                    }
                    const int b = j & 1;
                    const int n = mt.y >= 0 ? 2 : 1;
                    if (j >= 2 && !(ok = wait_bar(&s_free[b], ((j - 2) >> 1) & 1, stop, p))) break;
                    tc::fence_after_sync();
                    // descriptors advance by adding (byte offset >> 4) to the
                    // start-address field (shared addresses stay below 2^18)
                    const uint64_t b0 = tc::smem_desc_sw128(ring0 + cs * L::kStage, 16, 1024);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const int hf = kk >> 2, cc = (kk & 3) * 32;
                        tc::mma_bf16_ts(tmem + kColS + b * kStageKeys, tmem + kColQ + kk * 8,
                                        b0 + ((hf * L::kKvRegion + cc) >> 4), n == 2 ? kIdS2 : kIdS1, kk > 0);
                    }
                    tc::commit(smem_u32(&s_full[b]));
                    if (have_prev && !(ok = issue_pv())) break;
                    have_prev = true;
                    pj = j;
                    ps = cs;
                    pn = n;
                    pfirst = first;
                    pe = e;
                    first = false;
                    ++j;
                    if (mt.z & kMetaLast) {
                        // the unit's last product goes out now: the epilogue
                        // waits for it, and the next stage may be several
                        // (empty) units away
                        if (!(ok = issue_pv())) break;
                        have_prev = false;
                        ++e;
                        break;
                    }
                }
            }
            if (ok && have_prev) ok = issue_pv();
            if (!ok) *stop = 1;
            // nothing this thread issued may still run when the memory is freed
            tc::commit(smem_u32(drain));
            mbar_wait(drain, 0);
        }
        __syncwarp();
    } else if (has_work && warp < kSoftWarps) {

        // ---------------------------------------------------------- softmax + epilogue
        const int quarter = warp & 3, half = warp >> 2;
        const int r = quarter * 32 + lane;                   // query row = tensor-memory lane
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const uint32_t col_o = kColO + half * L::kOCols;     // this warp's columns of O
        const float cs = p.scale_log2;
        // every lane waits; the warp goes on only if all of them succeeded,
        // so the warp-collective tensor-memory accesses stay converged
        auto wwait = [&](uint64_t *bar, uint32_t parity) -> bool {
            const bool w = wait_bar(bar, parity, stop, p);
            return __all_sync(0xffffffffu, w);
        };
        int j = 0, s = 0, kq = 0, nx = 0;
        uint32_t sph = 0;                           // ring position and phase
        bool ok = true;
        // exchange one value per row with the other warp of this lane
        // quarter; false if the wait gave up
        auto exchange = [&](float mine, float &theirs) -> bool {
            float *xb = xbuf + (nx & 1) * 2 * kRows;
            xb[half * kRows + r] = mine;
            __syncwarp();
            if (lane == 0) mbar_arrive(&xbar[quarter]);
            if (!wwait(&xbar[quarter], nx & 1)) return false;
            theirs = xb[(half ^ 1) * kRows + r];
            ++nx;
            return true;
        };
        // the next stage is the next unit's Q stage or the end of the work:
        // Q goes to tensor memory (this warp's lanes and half of D), once the
        // MMA issuer has taken the previous unit's Q (whose products have all
        // completed: this warp waited for each).  more: a unit follows.
        auto copy_q = [&](bool &more) -> bool {
            if (!wwait(&full[s], sph)) return false;
            more = !(meta[s].z & kMetaEnd);
            if (!more) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
                if (++s == stages) {
                    s = 0;
                    sph ^= 1;
                }
                return true;
            }
            if (kq >= 1 && !wwait(q_ack, (kq - 1) & 1)) return false;
            tc::fence_after_sync();
            const int d0 = half * (D / 2);                       // first element of this warp's part
            const uint8_t *qrow = ring + s * L::kStage + (d0 / 64) * L::kQRegion + r * 128;
            const int c0 = (d0 % 64) / 8;                        // first 16-byte chunk of it
            if constexpr (L::kQCols == 32) {
                uint32_t qv[32];
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8) {
                    const uint4 x = *reinterpret_cast<const uint4 *>(qrow + (((c0 + c8) ^ (r & 7)) << 4));
                    qv[4 * c8] = x.x;
                    qv[4 * c8 + 1] = x.y;
                    qv[4 * c8 + 2] = x.z;
                    qv[4 * c8 + 3] = x.w;
                }
                tc::st_32x32b_x32(tmem + lane_base + kColQ + half * L::kQCols, qv);
            } else {
                uint32_t qv[16];
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8) {
                    const uint4 x = *reinterpret_cast<const uint4 *>(qrow + (((c0 + c8) ^ (r & 7)) << 4));
                    qv[4 * c8] = x.x;
                    qv[4 * c8 + 1] = x.y;
                    qv[4 * c8 + 2] = x.z;
                    qv[4 * c8 + 3] = x.w;
                }
                tc::st_32x32b_x16(tmem + lane_base + kColQ + half * L::kQCols, qv);
            }
            tc::wait_st();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&empty[s]);
                mbar_arrive(q_tm);
            }
            if (++s == stages) {
                s = 0;
                sph ^= 1;
            }
            ++kq;
            return true;
        };
        bool mpend = false, mhas = false;   // fused merge pending after the loop; its unit has tiles here
        bool more = false;
        ok = copy_q(more);
        while (ok && more) {
            const UnitDesc &u = units[(kq - 1) % kSegRing];      // the unit whose Q was copied last
            const int Lq = u.Lq, Lk = u.Lk;
            const int tq = r / G, g = r - tq * G;
            const int box0 = Lq - (u.rt + 1) * QT;               // the row tile's first token (may be < 0)
            const int qi = tq + box0;                            // this row's query token in the sequence
            const bool valid = tq < QT && qi >= 0;
            const int vis = valid ? Lk - Lq + qi + 1 : 0;        // keys [0, vis) visible (tail-aligned causal)
            // a lane quarter none of whose 32 rows is a query row of this
            // unit only keeps the barrier protocol (its P rows feed O rows
            // nobody reads); both warps of the quarter see the same rows
            const bool act = __any_sync(0xffffffffu, valid);
            float m_used = -INFINITY, l = 0.f;
            bool first = true, has_tiles = false;
            while (true) {
                if (!(ok = wwait(&full[s], sph))) break;
                const int4 mt = meta[s];
                const int ts = s;                                // this stage
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
                if (++s == stages) {
                    s = 0;
                    sph ^= 1;
                }
                if (mt.z & kMetaEmpty) break;
                has_tiles = true;
                const int ks = half ? mt.y : mt.x;               // this warp's tile (< 0: absent)
                if (PAGED && ks >= 0 && ks + kBN > Lk) {
                    // paged tile past the sequence's end: zero its V rows
                    // past Lk (weight 0 times a stale non-finite value would
                    // not be 0) before this warp's P is signalled; the stage
                    // is refilled only after the product that follows
                    const int z0 = Lk - ks;
                    uint8_t *vt = ring + ts * L::kStage + L::kKvTile + half * L::kSubRows;
                    for (int i = lane + quarter * 32; i < (kBN - z0) * L::kHalves * 8; i += 128) {
                        const int rr = z0 + i / (L::kHalves * 8), rest = i % (L::kHalves * 8);
                        *reinterpret_cast<uint4 *>(vt + (rest >> 3) * L::kKvRegion + rr * 128 + (rest & 7) * 16) =
                            make_uint4(0u, 0u, 0u, 0u);
                    }
                    fence_proxy_async();                         // before the tensor core reads V
                }
                const int b = j & 1;
                if (!(ok = wwait(&s_full[b], (j >> 1) & 1))) break;
                if (!act) {
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(&s_free[b]);
                        mbar_arrive(&p_full[b]);
                    }
                    first = false;
                    ++j;
                    if (mt.z & kMetaLast) break;
                    continue;
                }
                tc::fence_after_sync();
                uint32_t sv[2][32];                              // this warp's 64 scores
                if (ks >= 0) {
                    tc::ld_32x32b_x32(tmem + lane_base + kColS + b * kStageKeys + half * kBN, sv[0]);
                    tc::ld_32x32b_x32(tmem + lane_base + kColS + b * kStageKeys + half * kBN + 32, sv[1]);
                    tc::wait_ld();
                }
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s_free[b]);

                // mask and max of this warp's tile.  The scale (> 0) enters in
                // the exp2 argument, so the raw maximum gives the scaled one;
                // a masked score becomes -inf, whose weight is exactly 0.
                float mx = -INFINITY;
                bool whole_rows = true, dead = false;            // dead: this row's weights are all 0
                if (ks >= 0) {
                    const int ls = PAGED ? ks : min(ks, Lk - kBN);      // key of column 0
                    // visible columns [lo_c, lo_c + width); a row past the unit's
                    // query rows sees none
                    const int lo_c = max(ks - ls, 0);
                    const int width = max(min(kBN, vis - ls) - lo_c, 0);
                    float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                    // A row that sees no key of this tile (past the unit's
                    // query rows, or before its causal limit) needs no per-key
                    // mask: its max is -inf and its weights are forced to 0
                    // below -- unless the tile holds keys past the sequence
                    // read from a page's stale slots, whose scores may be
                    // non-finite.  Per-key masking only runs where some row
                    // sees part of the tile (a sequence's last tiles).
                    const bool stale = PAGED && ks + kBN > Lk;
                    whole_rows = __all_sync(0xffffffffu, (lo_c == 0 && width == kBN) || (width == 0 && !stale));
                    if (whole_rows) {
#pragma unroll
                        for (int cc = 0; cc < kBN; cc += 2)
                            mx4[(cc >> 1) & 3] = fmax3(mx4[(cc >> 1) & 3], __uint_as_float(sv[cc >> 5][cc & 31]),
                                                       __uint_as_float(sv[cc >> 5][(cc + 1) & 31]));
                        if (width == 0) mx4[0] = mx4[1] = mx4[2] = mx4[3] = -INFINITY;
                        dead = width == 0;
                    } else {
                        // masked by selection, no branch per key
#pragma unroll
                        for (int cc = 0; cc < kBN; cc += 2) {
                            const bool k0 = (unsigned)(cc - lo_c) < (unsigned)width;
                            const bool k1 = (unsigned)(cc + 1 - lo_c) < (unsigned)width;
                            const uint32_t x0 = k0 ? sv[cc >> 5][cc & 31] : 0xff800000u;   // -inf
                            const uint32_t x1 = k1 ? sv[cc >> 5][(cc + 1) & 31] : 0xff800000u;
                            sv[cc >> 5][cc & 31] = x0;
                            sv[cc >> 5][(cc + 1) & 31] = x1;
                            mx4[(cc >> 1) & 3] = fmax3(mx4[(cc >> 1) & 3], __uint_as_float(x0), __uint_as_float(x1));
                        }
                    }
                    mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * cs;
                }
                float mo;
                if (!(ok = exchange(mx, mo))) break;
                mx = fmaxf(mx, mo);                              // the row's max over the stage
                const bool need = mx > m_used + kRescaleLog2;    // false while the stage has no visible key
                const float m_new = need ? mx : m_used;
                // P(j) replaces P(j-1), and a rescale of O must follow its
                // product: both wait for O += P(j-1) V(j-1)
                bool waited = j == 0;
                if (!first && __any_sync(0xffffffffu, need)) {
                    if (!(ok = wwait(&o_done[(j - 1) & 1], ((j - 1) >> 1) & 1))) break;
                    waited = true;
                    tc::fence_after_sync();
                    const float alpha = need ? ex2(m_used - m_new) : 1.f;
#pragma unroll
                    for (int ch = 0; ch < L::kOCols / 32; ++ch) {
                        uint32_t o[32];
                        tc::ld_32x32b_x32(tmem + lane_base + col_o + ch * 32, o);
                        tc::wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                        tc::st_32x32b_x32(tmem + lane_base + col_o + ch * 32, o);
                    }
                    tc::wait_st();
                }
                if (need) {
                    l *= ex2(m_used - m_new);                     // ex2(-inf) = 0 on the first visible key
                    m_used = m_new;
                }
                if (ks >= 0) {
                    // a dead row's scores may be anything (rows past the
                    // unit's tokens read whatever the Q tile held): its
                    // weights come out as ex2(-inf) = 0 through the scale 0
                    const float nref = dead ? -INFINITY : (m_used == -INFINITY ? 0.f : -m_used);
                    const float csr = dead ? 0.f : cs;
                    uint32_t pk[kBN / 2];
                    float2 l2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                    const float2 cs2 = make_float2(csr, csr), nr2 = make_float2(nref, nref);
#pragma unroll
                    for (int i = 0; i < kBN / 2; ++i) {
                        const float2 x = ffma2(make_float2(__uint_as_float(sv[i >> 4][(2 * i) & 31]),
                                                           __uint_as_float(sv[i >> 4][(2 * i + 1) & 31])),
                                               cs2, nr2);
                        const float2 pp = make_float2(ex2(x.x), ex2(x.y));
                        l2[i & 1] = fadd2(l2[i & 1], pp);
                        pk[i] = pack_bf16x2(pp.x, pp.y);
                    }
                    l += (l2[0].x + l2[0].y) + (l2[1].x + l2[1].y);
                    if (!waited) {
                        if (!(ok = wwait(&o_done[(j - 1) & 1], ((j - 1) >> 1) & 1))) break;
                        tc::fence_after_sync();
                    }
                    tc::st_32x32b_x32(tmem + lane_base + kColP + half * (kBN / 2), pk);
                    tc::wait_st();
                }
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[b]);
                first = false;
                ++j;
                if (mt.z & kMetaLast) break;
            }
            if (!ok) break;

            // the next unit's Q goes to tensor memory now, so that its first
            // product can run during this unit's epilogue
            const int role = u.role, ub = u.b, uhk = u.hk, urt = u.rt, uw = u.w;
            const long long uq0 = u.q0, uPu = u.Pu;
            if (!(ok = copy_q(more))) break;

            // ---------------- epilogue: this block's part of the unit
            float Lt = l, M = m_used;
            if (has_tiles) {
                if (!(ok = wwait(&o_done[(j - 1) & 1], ((j - 1) >> 1) & 1))) break;
                tc::fence_after_sync();
                if (act) {
                    float lo;
                    if (!(ok = exchange(l, lo))) break;
                    Lt = l + lo;
                }
            }
            const bool whole = role == 0;
            const int slot = role == 1 ? 2 * c : 2 * c + 1;
            const int pr = (qi - max(0, box0)) * G + g;         // row within the unit's partial
            const long long tok = uq0 + qi;
            const int h = uhk * G + g;
            const int d0 = half * L::kOCols;                     // this warp's first column of D
            const long long uidx = unit_index(p, ub, uhk, urt);
            if (FUSED && !whole && uPu + uw <= sh.hi) {
                // Fused mode: this block holds the cut unit's last part (its
                // blocks are c_first .. c in share order).  It merges the
                // unit: its own part straight from tensor memory, the others'
                // from their partial slots in block order, so the result does
                // not depend on timing.  The others streamed their parts
                // first (the share's head-first order), so they are normally
                // published long before; the wait for them is bounded.
                // The unit is the block's last (head-first order), so the
                // merge runs after the loop, where the loop's state is dead;
                // this row's (m, l) waits in shared memory.  Nothing waits
                // for the unit's O to be released.
                mstash[tid] = make_float2(M, Lt);
                mpend = true;
                mhas = has_tiles;
                continue;
            }
            const float inv = Lt > 0.f ? 1.f / Lt : 0.f;
            if (has_tiles) {
#pragma unroll
                for (int ch = 0; ch < L::kOCols / 32; ++ch) {
                    if (!act) break;
                    uint32_t o[32];
                    __syncwarp();
                    tc::ld_32x32b_x32(tmem + lane_base + col_o + ch * 32, o);   // warp-collective
                    tc::wait_ld();
                    if (!valid) {
                    } else if (whole) {
                        uint4 *dst = reinterpret_cast<uint4 *>(p.out + (tok * p.Hq + h) * D + d0 + ch * 32);
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            uint4 w;
                            w.x = pack_bf16x2(__uint_as_float(o[8 * q4 + 0]) * inv, __uint_as_float(o[8 * q4 + 1]) * inv);
                            w.y = pack_bf16x2(__uint_as_float(o[8 * q4 + 2]) * inv, __uint_as_float(o[8 * q4 + 3]) * inv);
                            w.z = pack_bf16x2(__uint_as_float(o[8 * q4 + 4]) * inv, __uint_as_float(o[8 * q4 + 5]) * inv);
                            w.w = pack_bf16x2(__uint_as_float(o[8 * q4 + 6]) * inv, __uint_as_float(o[8 * q4 + 7]) * inv);
                            dst[q4] = w;
                        }
                    } else {
                        float4 *dst = reinterpret_cast<float4 *>(p.o_part + ((long long)slot * kRows + pr) * D + d0 +
                                                                 ch * 32);
                        // kept in L2: the unit's merge reads it back soon
                        const uint64_t keep = l2_evict_last();
#pragma unroll
                        for (int q4 = 0; q4 < 8; ++q4)
                            st_keep_f4(dst + q4,
                                       make_float4(__uint_as_float(o[4 * q4]), __uint_as_float(o[4 * q4 + 1]),
                                                   __uint_as_float(o[4 * q4 + 2]), __uint_as_float(o[4 * q4 + 3])),
                                       keep);
                    }
                }
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(o_free);
            } else if (valid && whole) {
                uint4 *dst = reinterpret_cast<uint4 *>(p.out + (tok * p.Hq + h) * D + d0);
#pragma unroll
                for (int q4 = 0; q4 < L::kOCols / 8; ++q4) dst[q4] = make_uint4(0u, 0u, 0u, 0u);
            }
            if (valid) {
                if (whole) {
                    if (half == 0) p.lse[tok * p.Hq + h] = Lt > 0.f ? (M + log2f(Lt)) * kLn2 : -INFINITY;
                } else {
                    // both warps of the row hold the same (m, l)
                    if (half == 0) st_keep_f2(p.ml_part + (long long)slot * kRows + pr, make_float2(M, Lt), l2_evict_last());
                }
            }
            if (whole) continue;
            // publish this warp's rows and columns of the part: the combine
            // kernel, or in fused mode the unit's last block, waits for all
            // kSoftWarps writer warps of each part
            __syncwarp();
            if (lane == 0) red_add_release_gpu(p.done + uidx, 1u);
        }
        if (ok && mpend) {
            // fused merge of the unit whose last part this block holds:
            // the last unit whose Q was copied, this thread's row of it
            const UnitDesc &u = units[(kq - 1) % kSegRing];
            const long long m_uPu = u.Pu;
            const int tq = r / G, g = r - tq * G;
            const int box0 = u.Lq - (u.rt + 1) * QT;
            const int qi = tq + box0;
            const bool m_valid = tq < QT && qi >= 0;
            const bool m_act = __any_sync(0xffffffffu, m_valid);
            const int m_pr = (qi - max(0, box0)) * G + g;
            const long long m_tok = u.q0 + qi;
            const int m_h = u.hk * G + g;
            const float2 st = mstash[tid];
            const float m_M = st.x, m_Lt = st.y;
            const int d0 = half * L::kOCols;                     // this warp's first column of D
            const int c_first = block_of(m_uPu, sh.T, sh.Ce);
            const int npo = c - c_first;                     // the other parts (>= 1)
            const bool own = mhas && m_Lt > 0.f;
            // the producer has seen them published (schedule order makes
            // that early); (up to twice the limit: the producer's own
            // wait may take the whole limit first)
            ok = __all_sync(0xffffffffu, wait_bar(mg, 0, stop, p, 2));
            const bool got = ok && *mflag == 1;
            if (got && m_act) {
                // the first other part's columns and every part's (m, l),
                // all loads in flight at once (one L2 round trip for a
                // unit cut once); a part that saw no key (l = 0) may not
                // have written its O, so its values are never used
                const long long sr0 = (long long)slot_of(c_first, m_uPu, sh.T, sh.Ce) * kRows + m_pr;
                float4 x0[L::kOCols / 4];
                float2 ml0 = make_float2(0.f, 0.f);
                float Mx = own ? m_M : -INFINITY;
                if (m_valid) {
                    ml0 = __ldcg(p.ml_part + sr0);
                    const float4 *src = reinterpret_cast<const float4 *>(p.o_part + sr0 * D + d0);
#pragma unroll
                    for (int q4 = 0; q4 < L::kOCols / 4; ++q4) x0[q4] = __ldcg(src + q4);
#pragma unroll 4
                    for (int i = 1; i < npo; ++i) {
                        const float2 ml =
                            __ldcg(p.ml_part + (long long)slot_of(c_first + i, m_uPu, sh.T, sh.Ce) * kRows + m_pr);
                        if (ml.y > 0.f) Mx = fmaxf(Mx, ml.x);
                    }
                    if (ml0.y > 0.f) Mx = fmaxf(Mx, ml0.x);
                }
                // weights relative to the largest max: own part, then
                // the others in block order
                const float Mref = Mx == -INFINITY ? 0.f : Mx;
                const float so = own ? ex2(m_M - Mref) : 0.f;
                const bool use0 = ml0.y > 0.f;
                const float w0 = use0 ? ex2(ml0.x - Mref) : 0.f;
                float Ltot = (own ? m_Lt * so : 0.f) + (use0 ? ml0.y * w0 : 0.f);
                // (the tensor-memory reads are warp-collective: every lane
                // takes them at the same point, the per-row work follows in
                // a branch of its own)
#pragma unroll
                for (int ch = 0; ch < L::kOCols / 32; ++ch) {
                    float acc[32];
                    if (mhas) {                                      // warp-uniform
                        uint32_t o[32];
                        __syncwarp();
                        tc::ld_32x32b_x32(tmem + lane_base + col_o + ch * 32, o);   // warp-collective
                        tc::wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) acc[i] = own ? __uint_as_float(o[i]) * so : 0.f;
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) acc[i] = 0.f;
                    }
                    if (m_valid) {
                        if (use0) {
#pragma unroll
                            for (int q4 = 0; q4 < 8; ++q4) {
                                const float4 x = x0[ch * 8 + q4];
                                acc[4 * q4] = fmaf(x.x, w0, acc[4 * q4]);
                                acc[4 * q4 + 1] = fmaf(x.y, w0, acc[4 * q4 + 1]);
                                acc[4 * q4 + 2] = fmaf(x.z, w0, acc[4 * q4 + 2]);
                                acc[4 * q4 + 3] = fmaf(x.w, w0, acc[4 * q4 + 3]);
                            }
                        }
                        // a unit cut more than once: its further parts
                        for (int i = 1; i < npo; ++i) {
                            const long long sr = (long long)slot_of(c_first + i, m_uPu, sh.T, sh.Ce) * kRows + m_pr;
                            const float2 ml = __ldcg(p.ml_part + sr);
                            const float4 *src = reinterpret_cast<const float4 *>(p.o_part + sr * D + d0 + ch * 32);
                            float4 x[8];
#pragma unroll
                            for (int q4 = 0; q4 < 8; ++q4) x[q4] = __ldcg(src + q4);
                            if (ml.y > 0.f) {
                                const float ws = ex2(ml.x - Mref);
                                if (ch == 0) Ltot = fmaf(ml.y, ws, Ltot);
#pragma unroll
                                for (int q4 = 0; q4 < 8; ++q4) {
                                    acc[4 * q4] = fmaf(x[q4].x, ws, acc[4 * q4]);
                                    acc[4 * q4 + 1] = fmaf(x[q4].y, ws, acc[4 * q4 + 1]);
                                    acc[4 * q4 + 2] = fmaf(x[q4].z, ws, acc[4 * q4 + 2]);
                                    acc[4 * q4 + 3] = fmaf(x[q4].w, ws, acc[4 * q4 + 3]);
                                }
                            }
                        }
                        // Ltot is complete after the first chunk's pass
                        const float invt = Ltot > 0.f ? 1.f / Ltot : 0.f;
                        uint4 *dst = reinterpret_cast<uint4 *>(p.out + (m_tok * p.Hq + m_h) * D + d0 + ch * 32);
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            uint4 w;
                            w.x = pack_bf16x2(acc[8 * q4 + 0] * invt, acc[8 * q4 + 1] * invt);
                            w.y = pack_bf16x2(acc[8 * q4 + 2] * invt, acc[8 * q4 + 3] * invt);
                            w.z = pack_bf16x2(acc[8 * q4 + 4] * invt, acc[8 * q4 + 5] * invt);
                            w.w = pack_bf16x2(acc[8 * q4 + 6] * invt, acc[8 * q4 + 7] * invt);
                            dst[q4] = w;
                        }
                    }
                    __syncwarp();
                }
                if (m_valid && half == 0) p.lse[m_tok * p.Hq + m_h] = Ltot > 0.f ? (Mref + log2f(Ltot)) * kLn2 : -INFINITY;
            }
        }
        if (!ok) *stop = 1;
    }

    // free the tensor memory once every role is done with it
    tc::fence_before_sync();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

template <int D>
void *tc_kernel_ptr(bool paged, bool fused) {
    if (fused)
        return paged ? reinterpret_cast<void *>(split_tc_kernel<D, true, true>)
                     : reinterpret_cast<void *>(split_tc_kernel<D, false, true>);
    return paged ? reinterpret_cast<void *>(split_tc_kernel<D, true, false>)
                 : reinterpret_cast<void *>(split_tc_kernel<D, false, false>);
}

}  // namespace

size_t tc_stage_bytes(int D) { return D == 64 ? TcLayout<64>::kStage : TcLayout<128>::kStage; }

size_t tc_smem_need(int D, int stages) {
    // 1 KB alignment slack + ring + barriers (full, empty per stage; 19 more)
    // + meta + unit descriptors + exchange buffer + merge stash + scan + (first, T) + stop
    // flag, tmem slot, merge flags
    return 1024 + tc_stage_bytes(D) * stages + (2 * stages + 19) * 8 + stages * 16 + kSegRing * sizeof(UnitDesc) +
           4 * kRows * 4 + kSoftWarps * 32 * 8 + (kThreads / 32 + 3) * 8 + 32;
}

size_t tc_smem_bytes(int D, int stages) {
    // at least half an SM's shared memory, so one block holds an SM and its
    // tensor-memory allocation never waits for another block's
    const size_t need = tc_smem_need(D, stages);
    return need > kMinSmemBytes ? need : kMinSmemBytes;
}

int tc_rows() { return kRows; }
int tc_parts_per_block() { return kSoftWarps; }
// A unit costs about five 64-key tiles' time besides its tiles (its query
// stage, the pipeline drain of its last stage and the epilogue); the shares
// count it so that blocks holding many small units take fewer tiles (short
// query: 47.9 us with 3, 47.4 with 5 or 8).
int tc_unit_cost() { return 5; }

cudaError_t tc_prepare(int D, int stages, int ctas) {
    for (bool paged : {false, true})
        for (bool fused : {false, true}) {
            void *fn = D == 64 ? tc_kernel_ptr<64>(paged, fused) : tc_kernel_ptr<128>(paged, fused);
            const cudaError_t e =
                cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc_smem_bytes(D, stages));
            if (e != cudaSuccess) return e;
        }
    return combine_slots_prepare(D, ctas);
}

cudaError_t launch_split_tc(const Params &p, const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                            const CUtensorMap &tm_v, int stages, int ctas, cudaStream_t stream) {
    // programmatic dependent launches, as for the warp-MMA kernel
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(ctas);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = tc_smem_bytes(p.D, stages);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int st = stages;
    void *args[] = {const_cast<CUtensorMap *>(&tm_q), const_cast<CUtensorMap *>(&tm_k),
                    const_cast<CUtensorMap *>(&tm_v), const_cast<Params *>(&p), &st};
    const bool paged = p.block_table != nullptr;
    const bool fused = p.fused != 0;
    cudaError_t e = cudaLaunchKernelExC(
        &cfg, p.D == 64 ? tc_kernel_ptr<64>(paged, fused) : tc_kernel_ptr<128>(paged, fused), args);
    if (e != cudaSuccess || p.fused) return e;      // fused: cut units are merged by their last block
    return launch_combine_slots(p, ctas, stream);
}

}  // namespace vgqa
