// split_mma.cu -- persistent TMA-fed tensor-core split-KV kernel for
// decode-sized row counts (G * q_len <= 16 query rows per KV head), and the
// log-sum-exp combine kernel that follows it.
//
// Schedule.  The work is the flattened sequence of 64-key tiles of every unit
// u = (sequence b, KV head hk), in order of b then hk; a unit with queries but
// no keys counts as one (empty) tile so that it still gets its defined output.
// Each of the C blocks (C fixed by the plan, about one per SM) takes the
// contiguous, equal share [c*T/C, (c+1)*T/C) of the T tiles, computed on the
// device from cu_seqlens at the start of every call -- no host round trip and
// no dead blocks, whatever the lengths are.  A unit that lies inside one
// block's share is finished there and written directly; a unit cut by share
// boundaries is split across consecutive blocks, each of which emits one
// unnormalised (O, m, l) partial.  A block emits at most two partials (the
// units cut by its two boundaries), into slots 2c and 2c + 1.  This is split-KV
// flash-decoding with the split points placed where the device can balance
// them (AstrAI commit log for csrc/kernels/gqa_decode_attn.cu, split-KV
// commit; cudnn-frontend issue #552 "frost(sdpa): THD execute host
// round-trip", sections Context and Proposal to evaluate: device lengths, no
// host totals).
//
// Split kernel: 4 consumer warps + 1 producer warp per block.
//
// Producer: one lane walks the block's units and streams their K and V tiles
// (64 keys x D) with cp.async.bulk.tensor (no multicast) into a ring of
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
//
// Combine kernel: one block per partial slot, launched as a programmatic
// dependent of the split kernel.  It recomputes the schedule from cu_seqlens
// while the split kernel runs, waits only for the parts of its own unit, and
// merges one column slice of it: the n blocks of a cut unit merge it
// together, each reading 1/n of the partial data, so the merge is spread over
// as many SMs as wrote it (one SM can pull only a few tens of GB/s from L2,
// too little to merge a unit alone).
#include "common.cuh"
#include "kernels.h"

namespace vgqa {

namespace {

constexpr int kBN = 64;                   // keys per tile
constexpr int kConsumerWarps = 4;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;
constexpr int kBarConsumers = 1;          // named barrier of the consumer warps
constexpr int kClaim = 2;                 // tiles per claim on a shared unit's counter
constexpr int kMetaLast = 1;              // stage flag: the block's last tile of the unit
constexpr int kMetaEmpty = 2;             // stage flag: no data, the unit ends here

template <int D>
struct MmaLayout {
    static constexpr int kHalves = D / 64;                  // 128-byte swizzle atoms per row
    static constexpr int kRegion = kBN * 128;               // bytes of one atom column
    static constexpr int kTileBytes = kHalves * kRegion;    // K or V tile
    static constexpr int kStageBytes = 2 * kTileBytes;      // K + V
};

// byte offset of (row, 16-byte chunk c) inside a 128B-swizzled [rows][128 B] region
__device__ __forceinline__ uint32_t swz(int row, int c) {
    return row * 128 + ((c ^ (row & 7)) << 4);
}

// tiles of one unit of sequence b: 0 if the sequence is skipped (no query
// rows, or lengths outside the plan), else max(1, ceil(Lk / 64))
__device__ __forceinline__ int unit_tiles(int Lq, int Lk, bool ok) {
    if (!ok || Lq <= 0) return 0;
    return Lk > 0 ? (Lk + kBN - 1) / kBN : 1;
}

struct SeqLen {
    int q0, Lq, k0, Lk, tpu;
};

__device__ __forceinline__ SeqLen seq_len(const Params &p, int b, bool report) {
    SeqLen s;
    const bool ok = load_lengths(p, b, report, s.q0, s.Lq, s.k0, s.Lk);
    s.tpu = unit_tiles(s.Lq, s.Lk, ok);
    return s;
}

// One stretch of a unit inside a block's share.
struct Segment {
    int b, hk;
    SeqLen s;
    int t0, t1;           // tiles [t0, t1) of the unit's tpu tiles
    long long Pu;         // global index of the unit's first tile
};

// Walks a block's share [g, hi) of the flattened tile space unit by unit.
struct SegWalker {
    int b, hk;
    SeqLen s;
    long long pb;         // global index of tile 0 of (b, hk = 0)
    long long g, hi;

    __device__ void init(const Params &p, int b_first, long long pb_first, long long lo, long long hi_) {
        b = b_first;
        pb = pb_first;
        s = seq_len(p, b, false);
        hk = (int)((lo - pb) / s.tpu);
        g = lo;
        hi = hi_;
    }

    __device__ bool next(const Params &p, Segment &seg) {
        if (g >= hi) return false;
        const long long Pu = pb + (long long)hk * s.tpu;
        seg.b = b;
        seg.hk = hk;
        seg.s = s;
        seg.Pu = Pu;
        seg.t0 = (int)(g - Pu);
        const long long end = min(hi, Pu + s.tpu);
        seg.t1 = (int)(end - Pu);
        g = end;
        if (g < hi && ++hk == p.Hkv) {
            // next sequence with work; the share ends before the tiles do, so
            // one exists (the bound only guards against reading past cu)
            pb += (long long)p.Hkv * s.tpu;
            hk = 0;
            do {
                if (++b >= p.B_max) {
                    g = hi;
                    break;
                }
                s = seq_len(p, b, false);
            } while (s.tpu == 0);
        }
        return true;
    }
};

// A block's units in processing order: the units that lie inside its share
// (streamed and written by this block alone) first, then the unit cut at the
// share's start (role 1, partial slot 2c), then the unit cut at its end
// (role 2, slot 2c + 1).  Cut units come last so that every block sharing one
// reaches it near the end of its own work, where run-time balancing can even
// out the blocks' finishing times without delaying any block's own units.
struct OrderedWalker {
    SegWalker wk;
    Segment first_cut, last_cut;
    bool has_first, has_last;
    int phase;            // 0: inside units, 1: the start-cut unit, 2: the end-cut unit, 3: done

    __device__ void init(const Params &p, int b_first, long long pb_first, long long lo, long long hi) {
        wk.init(p, b_first, pb_first, lo, hi);
        wk_lo = lo;
        has_first = has_last = false;
        phase = 0;
    }

    // role: 0 = unit inside the share, 1 = cut at the share's start, 2 = cut at its end
    __device__ bool next(const Params &p, Segment &seg, int &role) {
        if (phase == 0) {
            Segment s;
            while (true) {
                const long long g0 = wk.g;
                if (!wk.next(p, s)) break;
                const bool whole = s.t0 == 0 && s.t1 == s.s.tpu;
                if (whole) {
                    seg = s;
                    role = 0;
                    return true;
                }
                if (g0 == wk_lo) {
                    first_cut = s;
                    has_first = true;
                } else {
                    last_cut = s;
                    has_last = true;
                }
            }
            phase = 1;
        }
        if (phase == 1) {
            phase = 2;
            if (has_first) {
                seg = first_cut;
                role = 1;
                return true;
            }
        }
        if (phase == 2) {
            phase = 3;
            if (has_last) {
                seg = last_cut;
                role = 2;
                return true;
            }
        }
        return false;
    }
    long long wk_lo;
};

// block whose share [c*T/C, (c+1)*T/C) holds global tile t
__device__ __forceinline__ int block_of(long long t, long long T, int C) {
    return (int)(((t + 1) * C - 1) / T);
}
__device__ __forceinline__ long long share_start(int c, long long T, int C) {
    return (long long)c * T / C;
}

// Partial slot of block c for the unit whose first tile is Pu: a block's first
// unit uses slot 2c, its last (cut) unit slot 2c + 1.
__device__ __forceinline__ int slot_of(int c, long long Pu, long long T, int C) {
    return share_start(c, T, C) < Pu ? 2 * c + 1 : 2 * c;
}

// The block's share of the flattened tile space, computed by all `nthreads`
// threads of the block from cu_seqlens.  Each thread weighs a contiguous run of
// sequences; a scan of the run totals gives the tile prefix, the total T and
// the share; the thread whose run holds the share's first tile finds its unit.
// scan: 8 long long, first: 3 long long of shared memory.
struct Share {
    long long T, lo, hi, pb_first;
    int Ce, b_first;
};

__device__ bool block_share(const Params &p, int c, int C, int tid, int nthreads, bool report,
                            long long *scan, long long *first, Share &sh) {
    const int warp = tid >> 5, lane = tid & 31;
    const int per = (p.B_max + nthreads - 1) / nthreads;
    const int b_lo = min(p.B_max, tid * per), b_hi = min(p.B_max, b_lo + per);
    long long my = 0;
    for (int b = b_lo; b < b_hi; ++b) my += (long long)p.Hkv * seq_len(p, b, report).tpu;
    long long incl = my;                                    // warp-inclusive scan
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
    }
    if (lane == 31) scan[warp] = incl;
    if (tid == 0) first[0] = -1;
    __syncthreads();
    if (tid == 0) {
        long long run = 0;
        for (int w = 0; w < nthreads / 32; ++w) {
            const long long x = scan[w];
            scan[w] = run;
            run += x;
        }
        first[2] = run;
    }
    __syncthreads();
    sh.T = first[2];
    const long long my_start = incl - my + scan[warp];      // tiles before this thread's run
    // with fewer tiles than blocks only the first T blocks take a share, so
    // that every share between two blocks of a cut unit holds a tile of it
    sh.Ce = (int)min((long long)C, sh.T);
    if (c >= sh.Ce) return false;                           // no tiles for this block
    sh.lo = share_start(c, sh.T, sh.Ce);
    sh.hi = share_start(c + 1, sh.T, sh.Ce);
    long long pb = my_start;
    if (sh.lo >= pb && sh.lo < pb + my) {
        for (int b = b_lo; b < b_hi; ++b) {
            const long long w = (long long)p.Hkv * seq_len(p, b, false).tpu;
            if (sh.lo < pb + w) {
                first[0] = b;
                first[1] = pb;
                break;
            }
            pb += w;
        }
    }
    __syncthreads();
    sh.b_first = (int)first[0];
    sh.pb_first = first[1];
    return sh.b_first >= 0;                                 // always when lo < T
}

template <int D, int NT>
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
    long long *first = scan + 8;                                                 // b_first, pb_first, T
    volatile int *flags = reinterpret_cast<volatile int *>(first + 3);          // failed

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int c = blockIdx.x;

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
    // previous kernel in the stream still runs; everything above touches only
    // this block's shared memory.  Wait for that kernel (it may write the
    // inputs, and a previous call's combine resets the counters used below)
    // before reading any global memory.  Only then may this call's combine
    // kernel launch: it relies on the counters being reset.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // ------------------------------------------------------------ schedule
    Share sh;
    if (!block_share(p, c, gridDim.x, tid, kThreads, c == 0, scan, first, sh)) return;
    const long long lo = sh.lo, hi = sh.hi;
    const int b_first = sh.b_first;
    const long long pb_first = sh.pb_first;
    __syncthreads();

    // ------------------------------------------------------------ producer
    // Units inside this block's share are streamed whole.  A cut unit is
    // shared with the neighbouring block(s): in the run-time balanced mode the
    // blocks sharing it consume it from both ends through one packed counter
    // per unit (front count in the high word, back count in the low word), the
    // block whose static part is the unit's front claiming upward and the
    // others downward, kClaim tiles at a time with one claim in flight ahead
    // of the loads it feeds; each claim gets the part of its range that the
    // counter's old value shows as still free.  In deterministic mode each
    // block streams its static part.  Every stage carries its tile's key start
    // and a flag in shared memory; the block's last stage of a unit is flagged
    // (an empty stage carries the flag when the block got no tile of it).
    if (warp == kConsumerWarps) {
        if (lane == 0) {
            const uint64_t pol = l2_evict_first();
            OrderedWalker wk;
            wk.init(p, b_first, pb_first, lo, hi);
            Segment seg;
            int role;
            int s = 0, issued = 0;
            uint32_t phase = 0;
            bool ok = true;
            // take the next free stage; false if the wait gave up
            auto acquire = [&]() -> bool {
                if (issued >= stages && !mbar_wait(&empty[s], phase ^ 1)) {
                    atomicOr(p.err, ATTN_DEV_ERR_TIMEOUT);
                    return false;
                }
                return true;
            };
            auto advance = [&]() {
                ++issued;
                if (++s == stages) {
                    s = 0;
                    phase ^= 1;
                }
            };
            auto load_tile = [&](const Segment &sg, int tile, bool last) {
                const int ks = tile * kBN;
                const int row = sg.s.k0 + min(ks, sg.s.Lk - kBN);
                meta[s] = make_int2(ks, last ? kMetaLast : 0);
                uint8_t *st = ring + s * L::kStageBytes;
                mbar_arrive_expect_tx(&full[s], L::kStageBytes);
#pragma unroll
                for (int hf = 0; hf < L::kHalves; ++hf)
                    tma_load_3d(st + hf * L::kRegion, &tm_k, &full[s], hf * 64, sg.hk, row, pol);
#pragma unroll
                for (int hf = 0; hf < L::kHalves; ++hf)
                    tma_load_3d(st + L::kTileBytes + hf * L::kRegion, &tm_v, &full[s], hf * 64, sg.hk, row, pol);
            };
            auto empty_stage = [&]() {                 // end of a unit without a tile
                meta[s] = make_int2(0, kMetaLast | kMetaEmpty);
                mbar_arrive(&full[s]);
            };
            while (ok && wk.next(p, seg, role)) {
                const int ntiles = (seg.s.Lk + kBN - 1) / kBN;
                if (role == 0 || !p.dynamic) {
                    const int tb = role == 0 ? 0 : seg.t0, te = role == 0 ? ntiles : min(ntiles, seg.t1);
                    for (int t = tb; t < te; ++t) {
                        if (!(ok = acquire())) break;
                        load_tile(seg, t, t == te - 1);
                        advance();
                    }
                    if (ok && te <= tb) {
                        if (!(ok = acquire())) break;
                        empty_stage();
                        advance();
                    }
                    continue;
                }
                unsigned long long *claim = p.claim + (long long)seg.b * p.Hkv + seg.hk;
                const bool up = seg.t0 == 0;                       // static part at the unit's front
                const unsigned long long inc = up ? ((unsigned long long)kClaim << 32) : (unsigned long long)kClaim;
                auto range = [&](unsigned long long old, int &t_lo, int &t_hi) {
                    const int f = (int)(old >> 32), b = (int)(old & 0xffffffffu);
                    const int free_hi = ntiles - b;
                    if (up) {
                        t_lo = f;
                        t_hi = min(f + kClaim, free_hi);
                    } else {
                        t_hi = free_hi;
                        t_lo = max(free_hi - kClaim, f);
                    }
                };
                int a_lo, a_hi, n_lo, n_hi;
                range(atomicAdd(claim, inc), a_lo, a_hi);
                bool any = false;
                while (ok && a_lo < a_hi) {
                    // next claim in flight, unless this one already reached the far end
                    const bool more = up ? a_hi < ntiles : a_lo > 0;
                    if (more)
                        range(atomicAdd(claim, inc), n_lo, n_hi);
                    else
                        n_lo = n_hi = 0;
                    const bool final_range = !(n_lo < n_hi);
                    for (int i = 0; i < a_hi - a_lo; ++i) {
                        const int t = up ? a_lo + i : a_hi - 1 - i;
                        if (!(ok = acquire())) break;
                        load_tile(seg, t, final_range && i == a_hi - a_lo - 1);
                        advance();
                        any = true;
                    }
                    a_lo = n_lo;
                    a_hi = n_hi;
                }
                if (ok && !any) {
                    if (!(ok = acquire())) break;
                    empty_stage();
                    advance();
                }
            }
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

    OrderedWalker wk;
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
            if (!mbar_wait(&full[s], phase)) {
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
            const int ls = min(t0, Lk - kBN);     // key index of tile row 0

            // S^T = K Q^T
            float sacc[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                const int hf = ks >> 2, c0 = (ks & 3) * 2;
                uint32_t a0, a1, a2, a3;
                ldsm_x4(kst + hf * L::kRegion + swz(k_row, c0 + k_cadd), a0, a1, a2, a3);
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
                ldsm_x4_trans(vst + hf * L::kRegion + swz(v_row, c0 + v_cadd), a0, a1, a2, a3);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(o[mt][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
            }

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
        if (!whole && tid == 0) red_add_release_gpu(p.done + (long long)cur.b * p.Hkv + cur.hk, 1u);

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

// Combine: block 2c + k merges slice (c - c_first) of the unit block c cut at
// its start (k = 0) or end (k = 1), if any.  The block is launched as a
// programmatic dependent of the split kernel, so it computes the schedule
// while the split kernel streams; it then waits (bounded) only for the n parts
// of its own unit, whose writers each add 1 (release) to the unit's count, so
// a unit is merged as soon as its last part lands rather than when the whole
// split grid ends.  After merging, each of the unit's n combine blocks adds 1
// again; the one that brings the count to 2n resets it for the next call.
template <int D, int NT>
__global__ void __launch_bounds__(128, 4) combine_mma_kernel(const Params p, const int C) {
    constexpr int ROWS = 8 * NT;
    constexpr int kCols = D / 4;
    constexpr int kT = 128;
    constexpr int kBatch = 12;             // loads in flight per thread (register budget)
    extern __shared__ __align__(16) uint8_t csm[];
    __shared__ long long scan[8];
    __shared__ long long first[3];
    __shared__ int ok_flag;
    const int tid = threadIdx.x, lane = tid & 31;
    const int c = blockIdx.x >> 1, k = blockIdx.x & 1;
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
    if (seg.t0 == 0 && seg.t1 == seg.s.tpu) return;   // whole unit: written by the split kernel
    const long long T = sh.T;
    const int Ce = sh.Ce;
    const int c_first = block_of(seg.Pu, T, Ce);
    const int n = block_of(seg.Pu + seg.s.tpu - 1, T, Ce) - c_first + 1;
    const int G = p.G, R = G * seg.s.Lq;
    const int items = R * kCols;
    const int per = (items + n - 1) / n;
    const int it_lo = min(items, (c - c_first) * per), it_hi = min(items, it_lo + per);
    const long long u = (long long)seg.b * p.Hkv + seg.hk;

    int *slots = reinterpret_cast<int *>(csm);                         // [n]
    for (int j = tid; j < n; j += kT) slots[j] = slot_of(c_first + j, seg.Pu, T, Ce);

    // wait for the unit's n parts (acquire pairs with the writers' release)
    if (tid == 0) {
        int ok = 1;
        if (ld_acquire_gpu(p.done + u) < (uint32_t)n) {
            const unsigned long long t0 = globaltimer();
            while (ld_acquire_gpu(p.done + u) < (uint32_t)n) {
                if (globaltimer() - t0 > kWaitLimitNs) {
                    atomicOr(p.err, ATTN_DEV_ERR_TIMEOUT);
                    ok = 0;
                    break;
                }
                __nanosleep(256);
            }
        }
        ok_flag = ok;
        if (ok && c == c_first) p.claim[u] = 0ull;                      // claims, next call
    }
    __syncthreads();
    if (!ok_flag) return;

    // two threads per item (row, 4 columns), each merging every other part
    // with a running max, kBatch loads in flight; the pair then combines
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
            const float Lt = L * s1 + L2 * s2;
            const float inv = Lt > 0.f ? 1.f / Lt : 0.f;
            const int qi = r / G, h = seg.hk * G + r % G;
            const long long tok = seg.s.q0 + qi;
            uint2 pk;
            pk.x = pack_bf16x2((acc.x * s1 + a2.x * s2) * inv, (acc.y * s1 + a2.y * s2) * inv);
            pk.y = pack_bf16x2((acc.z * s1 + a2.z * s2) * inv, (acc.w * s1 + a2.w * s2) * inv);
            *reinterpret_cast<uint2 *>(p.out + (tok * p.Hq + h) * D + d4) = pk;
            if (d4 == 0) p.lse[tok * p.Hq + h] = Lt > 0.f ? (Mt + log2f(Lt)) * kLn2 : -INFINITY;
        }
    }
    (void)lane;
    __syncthreads();
    // every combine block of the unit has seen its n parts once the count
    // reaches 2n: the last one resets it
    if (tid == 0 && atomicAdd(p.done + u, 1u) == (uint32_t)(2 * n - 1)) p.done[u] = 0u;
}

size_t combine_mma_smem(int /*NT*/, int ctas) {
    return (size_t)((ctas + 3) & ~3) * 4;
}

template <int D, int NT>
void *mma_kernel_ptr() {
    return reinterpret_cast<void *>(split_mma_kernel<D, NT>);
}

void *pick(int D, int NT) {
    if (D == 64) return NT == 1 ? mma_kernel_ptr<64, 1>() : mma_kernel_ptr<64, 2>();
    return NT == 1 ? mma_kernel_ptr<128, 1>() : mma_kernel_ptr<128, 2>();
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

void *combine_pick(int D, int NT) {
    if (D == 64)
        return NT == 1 ? reinterpret_cast<void *>(combine_mma_kernel<64, 1>)
                       : reinterpret_cast<void *>(combine_mma_kernel<64, 2>);
    return NT == 1 ? reinterpret_cast<void *>(combine_mma_kernel<128, 1>)
                   : reinterpret_cast<void *>(combine_mma_kernel<128, 2>);
}

cudaError_t mma_prepare(int D, int NT, int stages, int ctas) {
    cudaError_t e = cudaFuncSetAttribute(pick(D, NT), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)mma_smem_bytes(D, NT, stages, ctas));
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(combine_pick(D, NT), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)combine_mma_smem(NT, ctas));
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
    cudaError_t e = cudaLaunchKernelExC(&cfg, pick(p.D, NT), split_args);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3(2 * ctas);
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = combine_mma_smem(NT, ctas);
    void *combine_args[] = {const_cast<Params *>(&p), &ctas};
    return cudaLaunchKernelExC(&cfg, combine_pick(p.D, NT), combine_args);
}

}  // namespace vgqa
