// split_tc.cu -- persistent TMA-fed split-KV kernel on the fifth-generation
// tensor cores (tcgen05, accumulators in tensor memory) for short-query row
// counts: 128 query rows (G heads x 128 / G query tokens) per unit, and
// longer queries as several row tiles of the sequence, each its own unit.
//
// Same schedule as the warp-MMA kernel (schedule.cuh: equal shares of the
// flattened 64-key tiles, cut units merged by the slot combine kernel; by
// default the shares stay static on this path, without run-time claims), but
// the G query heads times the q_len query tokens of a unit form the M = 128
// side of real tensor-core tiles (kernbench2 docs/adr-proposed commit log,
// GQA entry: G folded into the matmul M dimension; every K/V byte is read
// once per KV head):
//     S [128 rows x 64 keys]  = Q [128 x D] . K^T            (tcgen05.mma, S in tensor memory)
//     O [128 rows x D]       += P [128 x 64 keys] . V        (P bf16 and O in tensor memory)
//
// Warp roles (320 threads):
//   warp 9 -- producer (the whole warp walks the schedule in step, each lane
//     issuing one box, lane 0 taking claims and stage bookkeeping): loads each
//     unit's Q tile (one TMA box of G
//     heads x qtile tokens, right-aligned so it ends at the row tile's last
//     query token; rows past the sequence's own tokens are never written)
//     into one of two Q buffers, then streams the unit's K and V tiles into a
//     ring of shared-memory stages exactly like the warp-MMA kernel;
//   warp 8, one lane -- MMA issuer: S(j) = Q K_j^T into one of two S buffers,
//     then O += P(j-1) V_{j-1}, so the softmax of tile j overlaps the second
//     product of tile j-1 (a unit's last tile is not held back: its second
//     product follows at once); completion is tracked with tcgen05.commit on
//     mbarriers; the warp also allocates and frees the tensor memory;
//   warps 0-7 -- softmax and epilogue.  Warp w reads tensor-memory lanes
//     32 (w mod 4) .. +31, one query row per thread, and column half
//     h = w / 4 of every tile (keys 32h .. 32h+31).  Each half runs its own
//     online softmax in base-2 units over its keys and accumulates its own
//     O_h (the product P[:, half h] V[half h] goes to a separate tensor-memory
//     accumulator), so the two warps of a row never synchronise per tile;
//     the epilogue merges the two halves like two split-KV partials.  The
//     scores are masked (keys before the tile's own start when the tile was
//     right-aligned, and keys past Lk - Lq + qi under the tail-aligned causal
//     mask), and P is written as bf16 pairs into one of two P buffers in
//     tensor memory, from where the second product reads its A operand.
//
// The running max is rescaled lazily: O_h in tensor memory is multiplied by
// 2^(m_old - m_new) only when a row's max grows by more than 2^8 (rare after
// the first tile); otherwise the tile's weights are taken relative to the
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
constexpr int kSoftWarps = 8;             // two per tensor-memory lane quarter (column halves)
constexpr int kEpiWarps = 4;              // the half-0 warps write the outputs
constexpr int kMmaWarp = 8;              // sub-partition 0: its rows are the last to hold query rows
constexpr int kProducerWarp = 9;
constexpr int kThreads = 320;
constexpr int kHalfKeys = kBN / 2;
constexpr int kMetaLast = 1;              // stage flag: the block's last tile of the unit
constexpr int kMetaEmpty = 2;             // stage flag: no data, the unit ends here
constexpr float kRescaleLog2 = 8.f;       // lazy rescale threshold (base-2 units)
constexpr uint32_t kTmemCols = 512;       // S [0, 128), O_0 [128, 128 + D), O_1 [256, 256 + D), P [384, 448)
constexpr uint32_t kColS = 0, kColO0 = 128, kColO1 = 256, kColP = 384;
constexpr uint32_t kPCols = kBN / 2;      // bf16 pairs of one P buffer
constexpr size_t kMinSmemBytes = 120 * 1024;

template <int D>
struct TcLayout {
    static constexpr int kHalves = D / 64;                  // 128-byte swizzle atoms per row
    static constexpr int kKvRegion = kBN * 128;             // 64 keys x 128 B
    static constexpr int kKvTile = kHalves * kKvRegion;     // K or V tile
    static constexpr int kStage = 2 * kKvTile;              // K + V
    static constexpr int kQRegion = kRows * 128;            // 128 rows x 128 B
    static constexpr int kQTile = kHalves * kQRegion;
};

// bounded mbarrier wait that also gives up when another role raised the stop flag
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *stop, const Params &p) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if (*stop) return false;
        if (globaltimer() - t0 > p.wait_ns) {
            atomicOr(p.err, ATTN_DEV_ERR_TIMEOUT);
            *stop = 1;
            return false;
        }
    }
    return true;
}

// PAGED: K and V come from a paged cache (block table); a separate
// instantiation keeps the packed kernel free of that code
template <int D, bool PAGED>
__global__ void __launch_bounds__(kThreads, 1) split_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                               const __grid_constant__ CUtensorMap tm_k,
                                                               const __grid_constant__ CUtensorMap tm_v,
                                                               const Params p, const int stages) {
    using L = TcLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ring = smem;                                    // [stages][K tile | V tile]
    uint8_t *qbuf = ring + stages * L::kStage;               // [2][Q tile]
    uint64_t *full = reinterpret_cast<uint64_t *>(qbuf + 2 * L::kQTile);
    uint64_t *empty = full + stages;
    uint64_t *q_full = empty + stages;       // [2] Q tile landed
    uint64_t *q_free = q_full + 2;           // [2] last product reading the Q tile done
    uint64_t *s_full = q_free + 2;           // [2] S(j) computed (j mod 2)
    uint64_t *s_free = s_full + 2;           // [2] S(j) read by the softmax warps
    uint64_t *p_full = s_free + 2;           // [2] P(j) written
    uint64_t *o_done = p_full + 2;           // [2] O += P(j) V(j) done
    uint64_t *o_free = o_done + 2;           // O_0, O_1 read by the epilogue
    uint64_t *xch = o_free + 1;              // half-1 (m, l) of a unit published
    uint64_t *drain = xch + 1;               // all issued tensor-core work done
    int2 *meta = reinterpret_cast<int2 *>(drain + 1);                         // [stages]
    float2 *xml = reinterpret_cast<float2 *>(meta + stages);                 // [128] half-1 (m, l)
    long long *scan = reinterpret_cast<long long *>(xml + kRows);            // [kThreads / 32]
    long long *first = scan + kThreads / 32;                                 // [3]
    volatile int *stop = reinterpret_cast<volatile int *>(first + 3);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(first + 3) + 1;

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    // the block's share: consecutive blocks (which the hardware tends to
    // place on neighbouring SMs) take shares far apart, so every unit shared
    // by several blocks gets a mix of SMs rather than one neighbourhood
    const int c = (int)(((long long)blockIdx.x * p.share_stride) % gridDim.x);

    if (tid == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1 + kSoftWarps);   // the MMA's commit (or arrival) + each softmax warp
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&q_full[i], 1);
            mbar_init(&q_free[i], 1);
            mbar_init(&s_full[i], 1);
            mbar_init(&s_free[i], kSoftWarps);
            mbar_init(&p_full[i], kSoftWarps);
            mbar_init(&o_done[i], 1);
        }
        mbar_init(o_free, kEpiWarps);
        mbar_init(xch, kSoftWarps - kEpiWarps);
        mbar_init(drain, 1);
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
            first_tiles(p, c, sp, kPrefetchBytes / L::kStage, true, [&](const Segment &sg, int t) {
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
        int s = 0, issued = 0, k = 0;
        uint32_t phase = 0;
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
        // the stage's key start and flags, and the bytes its loads bring
        // (before any lane issues one)
        auto open_stage = [&](int ks, bool last) -> uint8_t * {
            if (leader) {
                meta[s] = make_int2(ks, last ? kMetaLast : 0);
                mbar_arrive_expect_tx(&full[s], L::kStage);
            }
            __syncwarp(wmask);
            return ring + s * L::kStage;
        };
        auto begin = [&](const Segment &sg, int) -> bool {
            if constexpr (PAGED) prefetch_pages(p, sg.b, sg.s.Lk, lane, 32);
            const int qb = k & 1;
            if (k >= 2 && !wait_all(&q_free[qb], ((k - 2) >> 1) & 1)) return false;
            if (leader) {
                mbar_arrive_expect_tx(&q_full[qb], q_bytes);
                // the box ends at the row tile's last query token
                const int t_end = sg.s.q0 + sg.s.Lq - sg.rt * QT;
#pragma unroll
                for (int hf = 0; hf < L::kHalves; ++hf)
                    tma_load_3d(qbuf + qb * L::kQTile + hf * L::kQRegion, &tm_q, &q_full[qb], hf * 64, sg.hk * G,
                                t_end - QT, pol);
            }
            ++k;
            return true;
        };
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
                if (!acquire()) return false;
                uint8_t *st = open_stage(ks, last);
                if (mine) {
                    // a box past the sequence (or a bad entry) reads page
                    // num_pages, outside the map: zeros
                    const int page = in ? page_checked(p, entry) : p.num_pages;
                    const int slot = key & ((1 << p.page_shift) - 1);       // 0 when pages are < 64 keys
                    uint8_t *dst = st + tv * L::kKvTile + hf * L::kKvRegion + bi * p.page_box * 128;
                    const CUtensorMap *map = tv ? &tm_v : &tm_k;
                    if (p.page_rows)
                        tma_load_3d(dst, map, &full[s], hf * 64, sg.hk, page * p.page_rows + slot, pol);
                    else
                        tma_load_4d(dst, map, &full[s], hf * 64, sg.hk, slot, page, pol);
                }
                advance();
                return true;
            }
            if (!acquire()) return false;
            const int row = sg.s.k0 + min(ks, sg.s.Lk - kBN);
            uint8_t *st = open_stage(ks, last);
            if (lane < 2 * L::kHalves) {                        // lane: (K or V, D-half)
                const int tv = lane / L::kHalves, hf = lane % L::kHalves;
                tma_load_3d(st + tv * L::kKvTile + hf * L::kKvRegion, tv ? &tm_v : &tm_k, &full[s], hf * 64, sg.hk,
                            row, pol);
            }
            advance();
            return true;
        };
        auto empty_stage = [&](const Segment &) -> bool {
            if (!acquire()) return false;
            if (leader) {
                meta[s] = make_int2(0, kMetaLast | kMetaEmpty);
                mbar_arrive(&full[s]);
            }
            advance();
            return true;
        };
        if (!feed_tiles<true>(p, sh.b_first, sh.pb_first, sh.lo, sh.hi, begin, load_tile, empty_stage)) *stop = 1;
        // let the loads in flight land before the block can exit (bounded,
        // also after a stop: the copies target this block's shared memory)
        for (int i = 0; i < min(issued, stages); ++i) {
            if (--s < 0) {
                s = stages - 1;
                phase ^= 1;
            }
            mbar_wait(&full[s], phase);
        }
        if (k >= 1) mbar_wait(&q_full[(k - 1) & 1], ((k - 1) >> 1) & 1);
        if (k >= 2) mbar_wait(&q_full[k & 1], ((k - 2) >> 1) & 1);
    } else if (has_work && warp == kMmaWarp) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdS = tc::idesc_bf16_f32(kRows, kBN, false);
            constexpr uint32_t kIdO = tc::idesc_bf16_f32(kRows, D, true);
            const uint32_t ring0 = smem_u32(ring), q0 = smem_u32(qbuf);
            int j = 0, k = 0, e = 0, s = 0;
            uint32_t sph = 0;                       // ring position and phase
            bool have_prev = false, ok = true;
            int pj = 0, ps = 0, pe = 0;
            bool pfirst = false;
            // O_h += P(pj)[:, half h] V(pj)[half h]: waits for the softmax
            // warps' P and, at a unit's first tile, for the epilogue of the
            // previous unit
            auto issue_pv = [&]() -> bool {
                if (!wait_bar(&p_full[pj & 1], (pj >> 1) & 1, stop, p)) return false;
                if (pfirst && pe >= 1 && !wait_bar(o_free, (pe - 1) & 1, stop, p)) return false;
                tc::fence_after_sync();
                const uint64_t v0 = tc::smem_desc_sw128(ring0 + ps * L::kStage + L::kKvTile, L::kKvRegion, 1024);
                const uint32_t pa = tmem + kColP + (pj & 1) * kPCols;
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int kk = 0; kk < kHalfKeys / 16; ++kk) {
                        const int key = h * kHalfKeys + kk * 16;
                        tc::mma_bf16_ts(tmem + (h ? kColO1 : kColO0), pa + key / 2, v0 + ((key * 128) >> 4), kIdO,
                                        !pfirst || kk > 0);
                    }
                tc::commit(smem_u32(&empty[ps]));
                tc::commit(smem_u32(&o_done[pj & 1]));
                return true;
            };
            OrderedWalker wk;
            wk.init(p, sh.b_first, sh.pb_first, sh.lo, sh.hi);
            Segment seg;
            int role;
            while (ok && wk.next(p, seg, role)) {
                const int qb = k & 1;
                if (!(ok = wait_bar(&q_full[qb], (k >> 1) & 1, stop, p))) break;
                const uint32_t qa = q0 + qb * L::kQTile;
                bool first = true;
                while (true) {
                    if (!(ok = wait_bar(&full[s], sph, stop, p))) break;
                    const int2 mt = meta[s];
                    const int cs_ = s;
                    if (++s == stages) {
                        s = 0;
                        sph ^= 1;
                    }
                    if (mt.y & kMetaEmpty) {
                        // the block's part of the unit ends here: flush the
                        // deferred product of its last tile, if any, and
                        // free the Q buffer once the products reading it are
                        // done (the commit tracks them)
                        mbar_arrive(&empty[cs_]);
                        if (have_prev) {
                            if (!(ok = issue_pv())) break;
                            have_prev = false;
                            ++e;
                        }
                        tc::commit(smem_u32(&q_free[qb]));
                        break;
                    }
                    const int b = j & 1;
                    if (j >= 2 && !(ok = wait_bar(&s_free[b], ((j - 2) >> 1) & 1, stop, p))) break;
                    tc::fence_after_sync();
                    // descriptors advance by adding (byte offset >> 4) to the
                    // start-address field (shared addresses stay below 2^18)
                    const uint64_t a0 = tc::smem_desc_sw128(qa, 16, 1024);
                    const uint64_t b0 = tc::smem_desc_sw128(ring0 + cs_ * L::kStage, 16, 1024);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const int hf = kk >> 2, cc = (kk & 3) * 32;
                        tc::mma_bf16_ss(tmem + kColS + b * kBN, a0 + ((hf * L::kQRegion + cc) >> 4),
                                        b0 + ((hf * L::kKvRegion + cc) >> 4), kIdS, kk > 0);
                    }
                    tc::commit(smem_u32(&s_full[b]));
                    if (mt.y & kMetaLast) tc::commit(smem_u32(&q_free[qb]));
                    if (have_prev && !(ok = issue_pv())) break;
                    have_prev = true;
                    pj = j;
                    ps = cs_;
                    pfirst = first;
                    pe = e;
                    first = false;
                    ++j;
                    if (mt.y & kMetaLast) {
                        // the unit's last product goes out now: the epilogue
                        // waits for it, and the next tile may be several
                        // (empty) units away
                        if (!(ok = issue_pv())) break;
                        have_prev = false;
                        ++e;
                        break;
                    }
                }
                ++k;
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
        const uint32_t col_o = half ? kColO1 : kColO0;
        const float cs = p.scale_log2;
        // every lane waits; the warp goes on only if all of them succeeded,
        // so the warp-collective tensor-memory accesses stay converged
        auto wwait = [&](uint64_t *bar, uint32_t parity) -> bool {
            const bool w = wait_bar(bar, parity, stop, p);
            return __all_sync(0xffffffffu, w);
        };
        int j = 0, e = 0, s = 0;
        uint32_t sph = 0;                           // ring position and phase
        bool ok = true;
        OrderedWalker wk;
        wk.init(p, sh.b_first, sh.pb_first, sh.lo, sh.hi);
        Segment seg;
        int role;
        while (ok && wk.next(p, seg, role)) {
            const int Lq = seg.s.Lq, Lk = seg.s.Lk;
            const int tq = r / G, g = r - tq * G;
            const int qi = tq + rt_box_start(seg.s, seg.rt, QT); // this row's query token in the sequence
            const bool valid = tq < QT && qi >= 0;
            const int vis = valid ? Lk - Lq + qi + 1 : 0;        // keys [0, vis) visible (tail-aligned causal)
            // a warp none of whose 32 rows is a query row of this unit only
            // keeps the barrier protocol (its P rows feed O rows nobody reads)
            const bool act = __any_sync(0xffffffffu, valid);
            float m_used = -INFINITY, l = 0.f;
            bool first = true, has_tiles = false;
            while (true) {
                if (!(ok = wwait(&full[s], sph))) break;
                const int2 mt = meta[s];
                const int ts = s;                                // this tile's stage
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
                if (++s == stages) {
                    s = 0;
                    sph ^= 1;
                }
                if (mt.y & kMetaEmpty) break;
                has_tiles = true;
                if (PAGED && mt.x + kBN > Lk) {
                    // paged tile past the sequence's end: zero its V rows
                    // past Lk (weight 0 times a stale non-finite value would
                    // not be 0) before this warp's P is signalled; the stage
                    // is refilled only after the product that follows
                    const int z0 = Lk - mt.x;
                    uint8_t *vt = ring + ts * L::kStage + L::kKvTile;
                    for (int i = tid; i < (kBN - z0) * L::kHalves * 8; i += kSoftWarps * 32) {
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
                    if (mt.y & kMetaLast) break;
                    continue;
                }
                tc::fence_after_sync();
                uint32_t sv[kHalfKeys];
                tc::ld_32x32b_x32(tmem + lane_base + kColS + b * kBN + half * kHalfKeys, sv);
                tc::wait_ld();
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s_free[b]);

                // mask and max of this half.  The scale (> 0) enters in the
                // exp2 argument, so the raw maximum gives the scaled one; a
                // masked score becomes -inf, whose weight is exactly 0.
                const int ks = mt.x, ls = PAGED ? ks : min(ks, Lk - kBN);   // key of column 0
                const int c0 = half * kHalfKeys;
                const int lo_c = ks - ls - c0, hi_c = min(kHalfKeys, vis - ls - c0);   // visible [lo_c, hi_c)
                float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                if (__all_sync(0xffffffffu, lo_c <= 0 && hi_c >= kHalfKeys)) {
#pragma unroll
                    for (int cc = 0; cc < kHalfKeys; ++cc) mx4[cc & 3] = fmaxf(mx4[cc & 3], __uint_as_float(sv[cc]));
                } else {
#pragma unroll
                    for (int cc = 0; cc < kHalfKeys; ++cc) {
                        if (cc < lo_c || cc >= hi_c) sv[cc] = 0xff800000u;   // -inf
                        mx4[cc & 3] = fmaxf(mx4[cc & 3], __uint_as_float(sv[cc]));
                    }
                }
                const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * cs;
                const bool need = mx > m_used + kRescaleLog2;    // false while the tile has no visible key
                const float m_new = need ? mx : m_used;
                if (!first && __any_sync(0xffffffffu, need)) {
                    // O_h holds P V of earlier tiles: rescale it once their
                    // products are done
                    if (!(ok = wwait(&o_done[(j - 1) & 1], ((j - 1) >> 1) & 1))) break;
                    tc::fence_after_sync();
                    const float alpha = need ? ex2(m_used - m_new) : 1.f;
#pragma unroll
                    for (int ch = 0; ch < D / 32; ++ch) {
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
                const float nref = m_used == -INFINITY ? 0.f : -m_used;
                uint32_t pk[kHalfKeys / 2];
                float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int i = 0; i < kHalfKeys / 2; ++i) {
                    const float p0 = ex2(fmaf(__uint_as_float(sv[2 * i]), cs, nref));
                    const float p1 = ex2(fmaf(__uint_as_float(sv[2 * i + 1]), cs, nref));
                    l4[i & 3] += p0 + p1;
                    pk[i] = pack_bf16x2(p0, p1);
                }
                l += (l4[0] + l4[1]) + (l4[2] + l4[3]);
                // P buffer j mod 2 was last read by O += P(j-2) V(j-2), which
                // finished before S(j) (issued after it) was signalled
                tc::st_32x32b_x16(tmem + lane_base + kColP + b * kPCols + half * (kHalfKeys / 2), pk);
                tc::wait_st();
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[b]);
                first = false;
                ++j;
                if (mt.y & kMetaLast) break;
            }
            if (!ok) break;

            // ---------------- epilogue: this block's part of the unit
            if (has_tiles) {
                if (!(ok = wwait(&o_done[(j - 1) & 1], ((j - 1) >> 1) & 1))) break;
                tc::fence_after_sync();
                if (half == 1) {
                    // publish this half's (m, l); the half-0 warp merges
                    xml[r] = make_float2(m_used, l);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(xch);
                    ++e;
                    continue;
                }
                if (!(ok = wwait(xch, e & 1))) break;
                ++e;
            } else if (half == 1) {
                continue;
            }
            // half-0 warps: merge the two halves and write
            float s0 = 1.f, s1 = 0.f, M = m_used, Lt = l;
            if (has_tiles) {
                const float2 o1 = xml[r];
                M = fmaxf(m_used, o1.x);
                const float Mref = M == -INFINITY ? 0.f : M;
                s0 = ex2(m_used - Mref);
                s1 = ex2(o1.x - Mref);
                Lt = l * s0 + o1.y * s1;
            }
            const bool whole = role == 0;
            const int slot = role == 1 ? 2 * c : 2 * c + 1;
            const int pr = (qi - rt_first(seg.s, seg.rt, QT)) * G + g;   // row within the unit's partial
            const long long tok = seg.s.q0 + qi;
            const int h = seg.hk * G + g;
            const float inv = Lt > 0.f ? 1.f / Lt : 0.f;
            if (has_tiles) {
#pragma unroll
                for (int ch = 0; ch < D / 32; ++ch) {
                    if (!act) break;
                    uint32_t o0[32], o1[32];
                    __syncwarp();
                    tc::ld_32x32b_x32(tmem + lane_base + kColO0 + ch * 32, o0);   // warp-collective
                    tc::ld_32x32b_x32(tmem + lane_base + kColO1 + ch * 32, o1);
                    tc::wait_ld();
                    float v[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(o0[i]) * s0 + __uint_as_float(o1[i]) * s1;
                    if (!valid) {
                    } else if (whole) {
                        uint4 *dst = reinterpret_cast<uint4 *>(p.out + (tok * p.Hq + h) * D + ch * 32);
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            uint4 w;
                            w.x = pack_bf16x2(v[8 * q4 + 0] * inv, v[8 * q4 + 1] * inv);
                            w.y = pack_bf16x2(v[8 * q4 + 2] * inv, v[8 * q4 + 3] * inv);
                            w.z = pack_bf16x2(v[8 * q4 + 4] * inv, v[8 * q4 + 5] * inv);
                            w.w = pack_bf16x2(v[8 * q4 + 6] * inv, v[8 * q4 + 7] * inv);
                            dst[q4] = w;
                        }
                    } else {
                        float4 *dst = reinterpret_cast<float4 *>(p.o_part + ((long long)slot * kRows + pr) * D + ch * 32);
#pragma unroll
                        for (int q4 = 0; q4 < 8; ++q4)
                            dst[q4] = make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
                    }
                }
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(o_free);
            } else if (valid && whole) {
                uint4 *dst = reinterpret_cast<uint4 *>(p.out + (tok * p.Hq + h) * D);
#pragma unroll
                for (int q4 = 0; q4 < D / 8; ++q4) dst[q4] = make_uint4(0u, 0u, 0u, 0u);
            }
            if (valid) {
                if (whole)
                    p.lse[tok * p.Hq + h] = Lt > 0.f ? (M + log2f(Lt)) * kLn2 : -INFINITY;
                else
                    p.ml_part[(long long)slot * kRows + pr] = make_float2(M, Lt);
            }
            // publish this warp's rows of the part (the combine waits for all
            // kEpiWarps writer warps of each of the unit's n blocks)
            if (!whole) {
                __syncwarp();
                if (lane == 0) red_add_release_gpu(p.done + unit_index(p, seg.b, seg.hk, seg.rt), 1u);
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
void *tc_kernel_ptr(bool paged) {
    return paged ? reinterpret_cast<void *>(split_tc_kernel<D, true>)
                 : reinterpret_cast<void *>(split_tc_kernel<D, false>);
}

}  // namespace

size_t tc_stage_bytes(int D) { return D == 64 ? TcLayout<64>::kStage : TcLayout<128>::kStage; }

size_t tc_smem_need(int D, int stages) {
    const size_t fixed = D == 64 ? 2 * TcLayout<64>::kQTile : 2 * TcLayout<128>::kQTile;
    // 1 KB alignment slack + ring + Q tiles + barriers + meta + half-1 (m, l) + scan +
    // (first, T) + stop flag, tmem slot
    return 1024 + tc_stage_bytes(D) * stages + fixed + (2 * stages + 17) * 8 + stages * 8 + kRows * 8 +
           (kThreads / 32 + 3) * 8 + 16;
}

size_t tc_smem_bytes(int D, int stages) {
    // at least half an SM's shared memory, so one block holds an SM and its
    // tensor-memory allocation never waits for another block's
    const size_t need = tc_smem_need(D, stages);
    return need > kMinSmemBytes ? need : kMinSmemBytes;
}

int tc_rows() { return kRows; }
int tc_parts_per_block() { return kEpiWarps; }
// A unit costs about three tiles' time besides its tiles (the query load, the
// pipeline drain of its last tile and the epilogue), measured on the
// short-query workload; the shares count it so that blocks holding many
// small units take fewer tiles.
int tc_unit_cost() { return 3; }

cudaError_t tc_prepare(int D, int stages, int ctas) {
    for (bool paged : {false, true}) {
        void *fn = D == 64 ? tc_kernel_ptr<64>(paged) : tc_kernel_ptr<128>(paged);
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
    cudaError_t e = cudaLaunchKernelExC(&cfg, p.D == 64 ? tc_kernel_ptr<64>(paged) : tc_kernel_ptr<128>(paged), args);
    if (e != cudaSuccess) return e;
    return launch_combine_slots(p, ctas, stream);
}

}  // namespace vgqa
