// split_mma.cu -- persistent TMA-fed warp-MMA split-KV kernel for
// decode-sized row counts (G * q_len <= 16 query rows per KV head).
//
// The schedule (schedule.cuh): a persistent grid of about one block per SM,
// each taking an equal contiguous share of the flattened 64-key tiles of all
// (sequence, KV head) units; units cut by share boundaries become partials
// that the slot combine kernel (combine_slots.cu) merges.
//
// Split kernel: 4 consumer warps + 1 producer warp per block.
//
// Producer: the whole warp walks the block's units in step (lane 0 takes the
// claims and keeps the stage bookkeeping, each lane issues one box) and
// streams their K and V tiles (64 keys x D, one box per tensor covering every
// D-half) with cp.async.bulk.tensor (this CTA only) into a ring of
// shared-memory stages in the 128-byte swizzled layout, one mbarrier per
// stage, L2 evict-first.  The ring runs across unit boundaries, so the next
// unit's loads are in flight while the current unit finishes.  A tile whose
// keys would run past its sequence is loaded ending at the sequence's last
// key (its start moves back, the extra keys are masked), so no load reads
// past cu_k[b+1]; a start before the buffer is a negative TMA coordinate,
// which the hardware fills with zeros.
//
// Consumers: warp w takes keys 16w .. 16w+15 of every tile and keeps its own
// online-softmax state.  With at most 16 query rows the contraction keeps the
// keys on the MMA's M side:
//     S^T [16 keys x rows] = K [16 keys x D] . Q^T        (mma.sync m16n8k16)
//     O^T [D x rows]      += V^T [D x 16 keys] . P^T      (V^T via ldmatrix.trans)
// P^T moves from the accumulator layout of the first product to the operand
// layout of the second with movmatrix.trans.  The G query heads of the KV
// head (and the query tokens) are the rows, so every K/V byte is read once
// per KV head (kernbench2 docs/adr-proposed commit log, GQA entry).  Q stays
// raw bf16 in registers (prefetched one unit ahead) and the softmax scale
// enters in fp32 inside the exp2 argument.  At the end of a unit the four
// warp states are merged in shared memory and written.
#include "common.cuh"
#include "kernels.h"
#include "schedule.cuh"

namespace vgqa {

namespace {

using namespace sched;

constexpr int kConsumerWarps = 4;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;
static_assert(kThreads / 32 <= 8, "block_share scan scratch holds 8 warps");
constexpr int kBarConsumers = 1;          // named barrier of the consumer warps
constexpr int kMetaLast = 1;              // stage flag: the block's last tile of the unit
constexpr int kMetaEmpty = 2;             // stage flag: no data, the unit ends here

template <int D>
struct MmaLayout {
    static constexpr int kHalves = D / 64;                  // 128-byte swizzle atoms per row
    static constexpr int kRegion = kBN * 128;               // bytes of one atom column
    static constexpr int kTileBytes = kHalves * kRegion;    // K or V tile
    static constexpr int kStageBytes = 2 * kTileBytes;      // K + V
};

// PAGED: K and V come from a paged cache (block table); DIRECT: block c takes
// unit c whole (plans whose units all fit one wave of blocks, no merge).
// Separate instantiations keep each kernel free of the code it does not run.
template <int D, int NT, bool PAGED, bool DIRECT>
__global__ void __launch_bounds__(kThreads, 1) split_mma_kernel(const __grid_constant__ CUtensorMap tm_k,
                                                                const __grid_constant__ CUtensorMap tm_v,
                                                                const Params p, const int stages) {
    using L = MmaLayout<D>;
    constexpr int KS = D / 16;           // k-steps of S^T, m-tiles of O^T
    constexpr int ROWS = 8 * NT;
    constexpr int OLD = D + 4;           // fp32 row stride of the warp-merge buffer

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ring = smem;
    float *ored = reinterpret_cast<float *>(smem + stages * L::kStageBytes);   // warp-merge buffer
    uint64_t *full = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(ored) + p.merge_bytes);
    uint64_t *empty = full + stages;
    int2 *meta = reinterpret_cast<int2 *>(empty + stages);                       // [stages] (key start, flags)
    long long *scan = reinterpret_cast<long long *>(meta + stages + (stages & 1)); // [warps]
    long long *first = scan + 8;                         // b_first, pb_first, T (scan: kThreads / 32 <= 8)
    volatile int *flags = reinterpret_cast<volatile int *>(first + 3);          // failed

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    // the block's share: consecutive blocks (which the hardware tends to
    // place on neighbouring SMs) take shares far apart, so every unit shared
    // by several blocks gets a mix of SMs rather than one neighbourhood
    const int c = (int)(((long long)blockIdx.x * p.share_stride) % gridDim.x);

    if (tid == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        flags[0] = 0;
        fence_barrier_init();
    }
    if (tid == kConsumers) {
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    // Launched as a programmatic dependent, the block may start while the
    // previous kernel in the stream still runs, which leaves the DRAM idle as
    // it ends.  Meanwhile the block computes a speculative schedule from
    // cu_seqlens as they read now (L2-only reads, so no stale line stays in
    // L1) and, if its share starts on a unit shared with other blocks,
    // prefetches its first tiles into L2 (schedule.cuh first_tiles).  Both
    // are hints: the L2 is coherent, so a prefetched line never hides a later
    // write, and the tensor map bounds every prefetch whatever the lengths
    // read.
    if constexpr (!PAGED && !DIRECT) {         // (direct mode: every share is a whole unit, nothing to prefetch)
        Share sp;
        if (block_share(p, c, gridDim.x, tid, kThreads, false, scan, first, sp, true) && warp == kConsumerWarps)
            first_tiles(p, c, sp, kPrefetchBytes / L::kStageBytes, true, [&](const Segment &sg, int t) {
                const int row = sg.s.k0 + min(t * kBN, sg.s.Lk - kBN);
                tma_prefetch_4d(&tm_k, 0, sg.hk, row, 0);
                tma_prefetch_4d(&tm_v, 0, sg.hk, row, 0);
            });
        __syncthreads();   // scan / first are reused below
    }
    // Wait for that kernel (it may write the inputs, and a previous call's
    // combine resets the counters used below) before any read that counts.
    // Only then may this call's combine kernel launch: it relies on the
    // counters being reset.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // ------------------------------------------------------------ schedule
    Share sh;
    if (!(DIRECT ? unit_share(p, c, tid, kThreads, c == 0, scan, first, sh)
                 : block_share(p, c, gridDim.x, tid, kThreads, c == 0, scan, first, sh)))
        return;
    const long long lo = sh.lo, hi = sh.hi;
    const int b_first = sh.b_first;
    const long long pb_first = sh.pb_first;
    __syncthreads();

    // ------------------------------------------------------------ producer
    // Feeds the ring with the block's tiles (schedule.cuh feed_tiles).  Every
    // stage carries its tile's key start and a flag in shared memory; the
    // block's last stage of a unit is flagged (an empty stage carries the
    // flag when the block got no tile of it).  The whole warp walks the
    // schedule in step and each lane loads one box (K or V of a tile, or of
    // a page's keys: a tile from small pages is up to 16 boxes), lane 0
    // doing the rest.
    if (warp == kConsumerWarps) {
        {
            const unsigned wmask = 0xffffffffu;
            const bool leader = lane == 0;
            const uint64_t pol = l2_evict_first();
            int s = 0, issued = 0;
            uint32_t phase = 0;
            // take the next free stage; false if the wait gave up
            auto acquire = [&]() -> bool {
                const bool w = issued < stages || mbar_wait(&empty[s], phase ^ 1, p.wait_ns);
                if (__all_sync(wmask, w)) return true;
                if (leader) atomicOr(p.err, ATTN_DEV_ERR_TIMEOUT);
                return false;
            };
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
                    mbar_arrive_expect_tx(&full[s], L::kStageBytes);
                }
                __syncwarp(wmask);
                return ring + s * L::kStageBytes;
            };
            auto load_tile = [&](const Segment &sg, int tile, bool last) -> bool {
                const int ks = tile * kBN;
                if constexpr (PAGED) {
                    // boxes of page_box keys, each from its page: lane i loads
                    // box i / 2 of K (i even) or V (i odd); the table reads go
                    // out before the stage wait, so they overlap it
                    const int nbox = kBN / p.page_box, bi = lane >> 1;
                    const bool mine = lane < 2 * nbox;
                    const int key = ks + bi * p.page_box;
                    const bool in = mine && key < sg.s.Lk;
                    const int entry = in ? page_entry(p, sg.b, key) : 0;
                    if (!acquire()) return false;
                    uint8_t *st = open_stage(ks, last);
                    if (mine) {
                        // a box past the sequence (or a bad entry) reads page
                        // num_pages, outside the map: zeros
                        const int page = in ? page_checked(p, entry) : p.num_pages;
                        const int slot = key & ((1 << p.page_shift) - 1);   // 0 when pages are < 64 keys
                        // box bi holds its page_box rows of every half:
                        // [half][row][128 B] at bi * page_box * D * 2
                        uint8_t *dst = st + bi * p.page_box * L::kHalves * 128 + (lane & 1) * L::kTileBytes;
                        const CUtensorMap *map = (lane & 1) ? &tm_v : &tm_k;
                        if (p.page_rows)
                            tma_load_4d(dst, map, &full[s], 0, sg.hk, page * p.page_rows + slot, 0, pol);
                        else
                            tma_load_5d(dst, map, &full[s], 0, sg.hk, slot, page, 0, pol);
                    }
                    advance();
                    return true;
                }
                if (!acquire()) return false;
                const int row = sg.s.k0 + min(ks, sg.s.Lk - kBN);
                uint8_t *st = open_stage(ks, last);
                // one box per tensor fills the tile's halves ([half][row][128 B])
                if (lane < 2)
                    tma_load_4d(st + lane * L::kTileBytes, lane ? &tm_v : &tm_k, &full[s], 0, sg.hk, row, 0, pol);
                advance();
                return true;
            };
            auto empty_stage = [&](const Segment &) -> bool {   // end of a unit without a tile
                if (!acquire()) return false;
                if (leader) {
                    meta[s] = make_int2(0, kMetaLast | kMetaEmpty);
                    mbar_arrive(&full[s]);
                }
                advance();
                return true;
            };
            auto begin = [&](const Segment &sg, int) -> bool {
                if constexpr (PAGED) prefetch_pages(p, sg.b, sg.s.Lk, lane, 32);
                return true;
            };
            feed_tiles<true>(p, b_first, pb_first, lo, hi, begin, load_tile, empty_stage);
        }
        return;
    }

    // ------------------------------------------------------------ consumers
    const int grp = lane >> 2, tig = lane & 3;
    const float cs = p.scale_log2;
    const int G = p.G;
    const uint32_t ring_base = smem_u32(ring);
    const int kbase = warp * 16;
    const int mi = lane >> 3;
    const int k_row = kbase + (mi & 1) * 8 + (lane & 7);    // K: matrices (keys lo/hi) x (d lo/hi)
    const int k_cadd = mi >> 1;
    const int v_row = kbase + (mi >> 1) * 8 + (lane & 7);   // V^T: matrices (d lo/hi) x (keys lo/hi)
    const int v_cadd = mi & 1;
    // tile layout: boxes of pb rows (64 packed; the page's keys, when pages
    // are smaller, paged), each [half][row][128 B]: byte offset of row r's
    // first half is (r / pb) * pb * D * 2 + (r % pb) * 128, the next half
    // pb * 128 further; the 128-byte swizzle works on r mod 8 (pb >= 8)
    const int pb = PAGED ? p.page_box : kBN;
    const uint32_t half_stride = (uint32_t)pb * 128;
    auto row_off = [&](int r) -> uint32_t {
        return (uint32_t)((r / pb) * pb * L::kHalves * 128 + (r % pb) * 128);
    };
    const uint32_t k_ro = row_off(k_row), v_ro = row_off(v_row);
    float *ms = ored + kConsumerWarps * ROWS * OLD;           // [4][ROWS]
    float *lsum = ms + kConsumerWarps * ROWS;                  // [4][ROWS]

    // Q^T fragments (B operand of S^T): row n = nt*8 + grp, d = 16ks + 2tig (+8)
    auto load_q = [&](const Segment &sg, uint32_t (&qf)[NT][KS][2]) {
        const int R = G * sg.s.Lq;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int r = nt * 8 + grp;
            const bool ok = r < R;
            const uint32_t *qp = reinterpret_cast<const uint32_t *>(
                p.q + ((long long)(sg.s.q0 + (ok ? r / G : 0)) * p.Hq + sg.hk * G + (ok ? r % G : 0)) * D);
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                qf[nt][ks][0] = ok ? __ldg(qp + (ks * 16 + 2 * tig) / 2) : 0u;
                qf[nt][ks][1] = ok ? __ldg(qp + (ks * 16 + 8 + 2 * tig) / 2) : 0u;
            }
        }
    };

    OrderedWalker<> wk;
    wk.init(p, b_first, pb_first, lo, hi);
    Segment cur, nxt;
    int role_cur, role_nxt;
    wk.next(p, cur, role_cur);
    bool has_nxt = wk.next(p, nxt, role_nxt);
    uint32_t qf[NT][KS][2], qn[NT][KS][2];
    load_q(cur, qf);
    int s = 0;
    uint32_t phase = 0;
    bool ok_run = true;

    while (true) {
        if (has_nxt) load_q(nxt, qn);               // in flight while this unit runs
        const int R = G * cur.s.Lq;
        const int Lk = cur.s.Lk, Lq = cur.s.Lq;

        int vis[NT][2];
        float m[NT][2], l[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int r = nt * 8 + 2 * tig + e;
                vis[nt][e] = r < R ? Lk - Lq + r / G + 1 : 0;
                m[nt][e] = -INFINITY;
                l[nt][e] = 0.f;
            }
        float o[KS][NT][4];
#pragma unroll
        for (int mt = 0; mt < KS; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) o[mt][nt][0] = o[mt][nt][1] = o[mt][nt][2] = o[mt][nt][3] = 0.f;

        while (ok_run) {
            if (!mbar_wait(&full[s], phase, p.wait_ns)) {
                atomicOr(p.err, ATTN_DEV_ERR_TIMEOUT);
                ok_run = false;
                break;
            }
            const int2 mt = meta[s];
            if (mt.y & kMetaEmpty) {                  // the unit ends without a tile here
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
                if (++s == stages) {
                    s = 0;
                    phase ^= 1;
                }
                break;
            }
            const int t0 = mt.x;
            const uint32_t kst = ring_base + s * L::kStageBytes;
            const uint32_t vst = kst + L::kTileBytes;
            // key index of tile row 0: a packed tile past the sequence's end
            // was moved back to end at its last key; a paged tile starts at
            // t0, and its rows past Lk hold whatever the page held
            constexpr bool paged = PAGED;
            const int ls = paged ? t0 : min(t0, Lk - kBN);
            bool zeroed = false;
            if (paged && t0 + kBN > Lk) {
                // zero this warp's V rows past Lk: their weights are 0, but
                // 0 times a stale non-finite value would not be
                const int z0 = max(kbase, Lk - t0);
                uint8_t *vt = ring + s * L::kStageBytes + L::kTileBytes;
                for (int i = lane; i < (kbase + 16 - z0) * L::kHalves * 8; i += 32) {
                    const int r = z0 + i / (L::kHalves * 8), rest = i % (L::kHalves * 8);
                    *reinterpret_cast<uint4 *>(vt + (rest >> 3) * half_stride + row_off(r) + (rest & 7) * 16) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
                zeroed = true;
                __syncwarp();
            }

            // S^T = K Q^T
            float sacc[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                const int hf = ks >> 2, c0 = (ks & 3) * 2;
                uint32_t a0, a1, a2, a3;
                ldsm_x4(kst + hf * half_stride + k_ro + (((c0 + k_cadd) ^ (k_row & 7)) << 4), a0, a1, a2, a3);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(sacc[nt], a0, a1, a2, a3, qf[nt][ks][0], qf[nt][ks][1]);
            }

            // mask, online softmax (rows 2tig+e; keys grp and grp+8 of this warp)
            const int j_lo = ls + kbase + grp;
            const int j_hi = j_lo + 8;
            uint32_t pb[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                float pl[2], ph[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int lim = vis[nt][e];
                    const float x_lo = (j_lo >= t0 && j_lo < lim) ? sacc[nt][e] : -INFINITY;
                    const float x_hi = (j_hi >= t0 && j_hi < lim) ? sacc[nt][2 + e] : -INFINITY;
                    float mx = fmaxf(x_lo, x_hi);
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                    const float m_new = fmaxf(m[nt][e], mx * cs);
                    const float m_ref = m_new == -INFINITY ? 0.f : m_new;
                    const float alpha = ex2(m[nt][e] - m_ref);
                    pl[e] = ex2(fmaf(x_lo, cs, -m_ref));
                    ph[e] = ex2(fmaf(x_hi, cs, -m_ref));
                    l[nt][e] = l[nt][e] * alpha + pl[e] + ph[e];
                    m[nt][e] = m_new;
#pragma unroll
                    for (int mt = 0; mt < KS; ++mt) {
                        o[mt][nt][e] *= alpha;
                        o[mt][nt][2 + e] *= alpha;
                    }
                }
                pb[nt][0] = movmatrix_trans(pack_bf16x2(pl[0], pl[1]));
                pb[nt][1] = movmatrix_trans(pack_bf16x2(ph[0], ph[1]));
            }

            // O^T += V^T P^T
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) {
                const int hf = mt >> 2, c0 = (mt & 3) * 2;
                uint32_t a0, a1, a2, a3;
                ldsm_x4_trans(vst + hf * half_stride + v_ro + (((c0 + v_cadd) ^ (v_row & 7)) << 4), a0, a1, a2, a3);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(o[mt][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
            }

            // the generic-proxy zeroing precedes the stage's next TMA write
            if (zeroed) fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            if (++s == stages) {
                s = 0;
                phase ^= 1;
            }
            if (mt.y & kMetaLast) break;
        }
        if (!ok_run) flags[0] = 1;   // benign race: every writer stores 1

        // ---------------------------------------------------------- end of unit: merge the 4 warps
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float t = l[nt][e];
                t += __shfl_xor_sync(0xffffffffu, t, 4);
                t += __shfl_xor_sync(0xffffffffu, t, 8);
                t += __shfl_xor_sync(0xffffffffu, t, 16);
                l[nt][e] = t;
            }
        if (grp == 0) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    ms[warp * ROWS + nt * 8 + 2 * tig + e] = m[nt][e];
                    lsum[warp * ROWS + nt * 8 + 2 * tig + e] = l[nt][e];
                }
        }
        named_sync(kBarConsumers, kConsumers);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int row = nt * 8 + 2 * tig + e;
                float M = ms[row];
#pragma unroll
                for (int w = 1; w < kConsumerWarps; ++w) M = fmaxf(M, ms[w * ROWS + row]);
                const float sc = ex2(m[nt][e] - (M == -INFINITY ? 0.f : M));
                float *dst = ored + (warp * ROWS + row) * OLD;
#pragma unroll
                for (int mt = 0; mt < KS; ++mt) {
                    dst[mt * 16 + grp] = o[mt][nt][e] * sc;
                    dst[mt * 16 + grp + 8] = o[mt][nt][2 + e] * sc;
                }
            }
        named_sync(kBarConsumers, kConsumers);
        if (flags[0]) break;                       // a wait gave up: leave this unit unwritten

        const bool whole = role_cur == 0;
        const int slot = role_cur == 1 ? 2 * c : 2 * c + 1;
        for (int idx = tid; idx < ROWS * (D / 4); idx += kConsumers) {
            const int row = idx / (D / 4);
            const int d4 = (idx % (D / 4)) * 4;
            if (row >= R) continue;
            float M = ms[row];
#pragma unroll
            for (int w = 1; w < kConsumerWarps; ++w) M = fmaxf(M, ms[w * ROWS + row]);
            const float Mref = M == -INFINITY ? 0.f : M;
            float Lsum = 0.f;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) {
                Lsum += lsum[w * ROWS + row] * ex2(ms[w * ROWS + row] - Mref);
                const float4 x = *reinterpret_cast<const float4 *>(ored + (w * ROWS + row) * OLD + d4);
                acc.x += x.x;
                acc.y += x.y;
                acc.z += x.z;
                acc.w += x.w;
            }
            if (whole) {
                const int qi = row / G, h = cur.hk * G + row % G;
                const long long tok = cur.s.q0 + qi;
                const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
                uint2 packed;
                packed.x = pack_bf16x2(acc.x * inv, acc.y * inv);
                packed.y = pack_bf16x2(acc.z * inv, acc.w * inv);
                *reinterpret_cast<uint2 *>(p.out + (tok * p.Hq + h) * D + d4) = packed;
                if (d4 == 0) p.lse[tok * p.Hq + h] = Lsum > 0.f ? (M + log2f(Lsum)) * kLn2 : -INFINITY;
            } else {
                *reinterpret_cast<float4 *>(p.o_part + ((long long)slot * ROWS + row) * D + d4) = acc;
                if (d4 == 0) p.ml_part[(long long)slot * ROWS + row] = make_float2(M, Lsum);
            }
        }
        named_sync(kBarConsumers, kConsumers);     // warp-merge buffers free for the next unit
        // publish the part: the combine block merging this unit waits for all n
        if (!whole && tid == 0) red_add_release_gpu(p.done + unit_index(p, cur.b, cur.hk, cur.rt), 1u);

        if (!has_nxt) break;
        cur = nxt;
        role_cur = role_nxt;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                qf[nt][ks][0] = qn[nt][ks][0];
                qf[nt][ks][1] = qn[nt][ks][1];
            }
        has_nxt = wk.next(p, nxt, role_nxt);
    }
}

template <int D, int NT>
void *mma_kernel_ptr(bool paged, bool direct) {
    if (direct)
        return paged ? reinterpret_cast<void *>(split_mma_kernel<D, NT, true, true>)
                     : reinterpret_cast<void *>(split_mma_kernel<D, NT, false, true>);
    return paged ? reinterpret_cast<void *>(split_mma_kernel<D, NT, true, false>)
                 : reinterpret_cast<void *>(split_mma_kernel<D, NT, false, false>);
}

void *pick(int D, int NT, bool paged, bool direct) {
    if (D == 64) return NT == 1 ? mma_kernel_ptr<64, 1>(paged, direct) : mma_kernel_ptr<64, 2>(paged, direct);
    return NT == 1 ? mma_kernel_ptr<128, 1>(paged, direct) : mma_kernel_ptr<128, 2>(paged, direct);
}

}  // namespace

size_t mma_stage_bytes(int D) {
    return D == 64 ? MmaLayout<64>::kStageBytes : MmaLayout<128>::kStageBytes;
}

// shared bytes of the warp-merge buffer (per-warp O^T rows, m, l)
size_t mma_merge_bytes(int D, int NT, int /*ctas*/) {
    const size_t rows = 8 * NT;
    const size_t ored = kConsumerWarps * rows * (D + 4) * 4 + 2 * kConsumerWarps * rows * 4;
    return (ored + 15) / 16 * 16;
}

size_t mma_smem_bytes(int D, int NT, int stages, int ctas) {
    // 1 KB alignment slack + ring + merge area + barriers + scan + (first, T) + flags
    return 1024 + mma_stage_bytes(D) * stages + mma_merge_bytes(D, NT, ctas) + 3 * stages * sizeof(uint64_t) +
           (8 + 3) * sizeof(long long) + 16;
}

int mma_block_n() { return kBN; }
int mma_threads() { return kThreads; }

cudaError_t mma_prepare(int D, int NT, int stages, int ctas) {
    for (bool paged : {false, true})
        for (bool direct : {false, true}) {
            const cudaError_t e =
                cudaFuncSetAttribute(pick(D, NT, paged, direct), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)mma_smem_bytes(D, NT, stages, ctas));
            if (e != cudaSuccess) return e;
        }
    return combine_slots_prepare(D, ctas);
}

cudaError_t launch_split_mma(const Params &p, const CUtensorMap &tm_k, const CUtensorMap &tm_v, int NT,
                             int stages, int ctas, cudaStream_t stream) {
    // Both kernels are launched as programmatic dependents of what precedes
    // them in the stream: the split kernel's blocks may become resident and
    // set up while the previous kernel finishes (they wait for it before
    // reading global memory), and the combine kernel's blocks start (and
    // compute the schedule) before the split kernel has finished.
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(ctas);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = mma_smem_bytes(p.D, NT, stages, ctas);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int st = stages;
    void *split_args[] = {const_cast<CUtensorMap *>(&tm_k), const_cast<CUtensorMap *>(&tm_v),
                          const_cast<Params *>(&p), &st};
    cudaError_t e = cudaLaunchKernelExC(&cfg, pick(p.D, NT, p.block_table != nullptr, p.direct != 0), split_args);
    if (e != cudaSuccess || p.direct) return e;            // direct mode: no unit is cut, nothing to merge
    return launch_combine_slots(p, ctas, stream);
}

}  // namespace vgqa
