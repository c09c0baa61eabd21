// schedule.cuh -- the persistent split-KV schedule shared by the tensor-core
// split kernels and the slot combine kernel (device code, internal).
//
// The work is the flattened sequence of 64-key tiles of every unit
// u = (sequence b, KV head hk, row tile rt), in order of b, hk, rt.  A row tile
// holds p.qtile query tokens (all of a decode sequence's; for long queries
// the tokens are tiled from the sequence's end, so tile rt ends qtile * rt
// tokens before it) and needs the keys its last token sees under the
// tail-aligned causal mask.  A unit whose rows see no key counts as one
// (empty) tile so that it still gets its defined output.
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
#pragma once

#include "common.cuh"

namespace vgqa {
namespace sched {

constexpr int kBN = 64;                   // keys per tile
constexpr int kClaim = 2;                 // tiles per claim on a shared unit's counter
// K/V bytes per block prefetched into L2 before the dependency wait
// (first_tiles; 37 MB over 148 blocks, about what the DRAM delivers while a
// back-to-back predecessor drains: 128 KB gained less, 512 KB lost it all)
constexpr int kPrefetchBytes = 256 * 1024;

struct SeqLen {
    int q0, Lq, k0, Lk;
    int nrt;              // row tiles (0: the sequence is skipped)
    int tpu;              // weighted positions of one KV head: sum over its row tiles of unit_weight
};

// key tiles of row tile rt: ceil(keys its last token sees / 64), 0 if none
__device__ __forceinline__ int rt_tiles(const SeqLen &s, int rt, int qtile) {
    const int vis = s.Lk - rt * qtile;
    return vis > 0 ? (vis + kBN - 1) / kBN : 0;
}

// A unit's weight in the flattened space: its tiles (at least one, the
// empty tile of a unit that sees no key) plus p.unit_cost tiles' worth for
// what a unit costs besides its tiles (the query load, the pipeline drain,
// the epilogue), so that blocks whose shares hold many small units get fewer
// tiles.  A unit's real tile t sits at position unit_cost + t of its range.
__device__ __forceinline__ int unit_weight(const Params &p, int tiles) { return max(tiles, 1) + p.unit_cost; }

__device__ __forceinline__ SeqLen seq_len(const Params &p, int b, bool report, bool spec = false) {
    SeqLen s;
    const bool ok = load_lengths(p, b, report, s.q0, s.Lq, s.k0, s.Lk, spec);
    if (!ok || s.Lq <= 0) {
        s.nrt = s.tpu = 0;
    } else if (s.Lq <= p.qtile) {                 // one row tile: every decode sequence
        s.nrt = 1;
        s.tpu = unit_weight(p, rt_tiles(s, 0, p.qtile));
    } else {
        s.nrt = (s.Lq + p.qtile - 1) / p.qtile;
        s.tpu = 0;
        for (int rt = 0; rt < s.nrt; ++rt) s.tpu += unit_weight(p, rt_tiles(s, rt, p.qtile));
    }
    return s;
}

// One stretch of a unit inside a block's share.
struct Segment {
    int b, hk, rt;
    SeqLen s;
    int nt;               // the unit's key tiles
    int w;                // its weight (positions)
    int t0, t1;           // positions [t0, t1) of the unit's w positions
    long long Pu;         // global index of the unit's first position
};

// counters of unit (b, hk, rt): tile claims, part counts
__device__ __forceinline__ long long unit_index(const Params &p, int b, int hk, int rt) {
    return ((long long)b * p.Hkv + hk) * p.max_rt + rt;
}

// token range [lo, lo + n) of row tile rt, and where its box starts (may be
// before the sequence: those rows do not exist)
__device__ __forceinline__ int rt_box_start(const SeqLen &s, int rt, int qtile) { return s.Lq - (rt + 1) * qtile; }
__device__ __forceinline__ int rt_first(const SeqLen &s, int rt, int qtile) {
    return max(0, rt_box_start(s, rt, qtile));
}

// Walks a block's share [g, hi) of the flattened tile space unit by unit.
struct SegWalker {
    int b, hk, rt;
    SeqLen s;
    int nt, w;            // the current unit's tiles and weight
    long long Pu;         // global index of the current unit's first position
    long long g, hi;
    bool spec;            // speculative reads of cu_seqlens (load_lengths)

    __device__ void set_unit(const Params &p) {
        nt = rt_tiles(s, rt, p.qtile);
        w = unit_weight(p, nt);
    }

    __device__ void init(const Params &p, int b_first, long long pb_first, long long lo, long long hi_,
                         bool spec_ = false) {
        spec = spec_;
        b = b_first;
        s = seq_len(p, b, false, spec);
        hk = (int)((lo - pb_first) / s.tpu);
        Pu = pb_first + (long long)hk * s.tpu;
        rt = 0;
        set_unit(p);
        if (s.nrt > 1) {
            while (Pu + w <= lo) {        // the row tile holding lo
                Pu += w;
                ++rt;
                set_unit(p);
            }
        }
        g = lo;
        hi = hi_;
    }

    __device__ bool next(const Params &p, Segment &seg) {
        if (g >= hi) return false;
        seg.b = b;
        seg.hk = hk;
        seg.rt = rt;
        seg.s = s;
        seg.nt = nt;
        seg.w = w;
        seg.Pu = Pu;
        seg.t0 = (int)(g - Pu);
        const long long end = min(hi, Pu + w);
        seg.t1 = (int)(end - Pu);
        g = end;
        if (g < hi) {
            Pu += w;
            if (++rt == s.nrt) {
                rt = 0;
                if (++hk == p.Hkv) {
                    // next sequence with work; the share ends before the
                    // tiles do, so one exists (the bound only guards against
                    // reading past cu)
                    hk = 0;
                    do {
                        if (++b >= p.B_max) {
                            g = hi;
                            break;
                        }
                        s = seq_len(p, b, false, spec);
                    } while (s.tpu == 0);
                }
            }
            if (g < hi) set_unit(p);
        }
        return true;
    }
};

// A block's units in processing order.  By default: the units that lie
// inside its share (streamed and written by this block alone) first, then
// the unit cut at the share's start (role 1, partial slot 2c), then the unit
// cut at its end (role 2, slot 2c + 1).  Cut units come last so that every
// block sharing one reaches it near the end of its own work, where run-time
// balancing can even out the blocks' finishing times without delaying any
// block's own units.  `head_first` (static shares with the fused merge, in
// which the block holding a cut unit's last part merges it) orders them so
// that a merge seldom waits: the unit cut at the share's end first (a head
// or middle part, which some later block merges), then the block's own
// units, then the unit cut at its start (whose last part this block may
// hold, the other parts having been streamed first by their blocks).
// HF: head-first order compiled in (the tcgen05 kernel with the fused
// merge); the kernels that never use it keep the plain walker.
template <bool HF = false>
struct OrderedWalker {
    SegWalker wk;
    Segment first_cut, last_cut;
    bool has_first, has_last;
    int phase;            // 0: inside units, 1: the start-cut unit, 2: the end-cut unit, 3: done

    __device__ void init(const Params &p, int b_first, long long pb_first, long long lo, long long hi,
                         bool spec = false, bool = false) {
        wk.init(p, b_first, pb_first, lo, hi, spec);
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
                const bool whole = s.t0 == 0 && s.t1 == s.w;
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

template <>
struct OrderedWalker<true> {
    SegWalker wk;
    Segment first_cut, last_cut;
    bool has_first, has_last, hf;
    int phase;            // cuts last: 0 inside units, 1 start cut, 2 end cut, 3 done;
                          // head first: 4 end cut, 0 inside units (skipping the cuts), 1 start cut, 3 done
    long long wk_lo;

    __device__ void init(const Params &p, int b_first, long long pb_first, long long lo, long long hi,
                         bool spec = false, bool head_first = false) {
        wk.init(p, b_first, pb_first, lo, hi, spec);
        wk_lo = lo;
        has_first = has_last = false;
        hf = head_first;
        phase = 0;
        if (hf) {
            // a first pass finds the unit cut at the share's end
            SegWalker w2 = wk;
            Segment s;
            while (true) {
                const long long g0 = w2.g;
                if (!w2.next(p, s)) break;
                if (g0 != wk_lo && !(s.t0 == 0 && s.t1 == s.w)) {
                    last_cut = s;
                    has_last = true;
                }
            }
            phase = 4;
        }
    }

    // role: 0 = unit inside the share, 1 = cut at the share's start, 2 = cut at its end
    __device__ bool next(const Params &p, Segment &seg, int &role) {
        if (phase == 4) {
            phase = 0;
            if (has_last) {
                seg = last_cut;
                role = 2;
                return true;
            }
        }
        if (phase == 0) {
            Segment s;
            while (true) {
                const long long g0 = wk.g;
                if (!wk.next(p, s)) break;
                const bool whole = s.t0 == 0 && s.t1 == s.w;
                if (whole) {
                    seg = s;
                    role = 0;
                    return true;
                }
                if (g0 == wk_lo) {
                    first_cut = s;
                    has_first = true;
                } else if (!hf) {                  // head first: given before
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
            if (has_last && !hf) {
                seg = last_cut;
                role = 2;
                return true;
            }
        }
        return false;
    }
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
struct Share {
    long long T, lo, hi, pb_first;
    int Ce, b_first;
};

// scan: nthreads / 32 long long of shared memory (one per warp); first: 3.
__device__ __forceinline__ bool block_share(const Params &p, int c, int C, int tid, int nthreads, bool report,
                                            long long *scan, long long *first, Share &sh, bool spec = false) {
    const int warp = tid >> 5, lane = tid & 31;
    const int per = (p.B_max + nthreads - 1) / nthreads;
    const int b_lo = min(p.B_max, tid * per), b_hi = min(p.B_max, b_lo + per);
    long long my = 0;
    for (int b = b_lo; b < b_hi; ++b) my += (long long)p.Hkv * seq_len(p, b, report, spec).tpu;
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
        if (b_hi - b_lo == 1) {                              // one sequence per thread: no second read
            first[0] = b_lo;
            first[1] = pb;
        }
        for (int b = b_lo; b_hi - b_lo > 1 && b < b_hi; ++b) {
            const long long w = (long long)p.Hkv * seq_len(p, b, false, spec).tpu;
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

// Direct mode (plans whose units are at most two tiles and at most one per
// SM): block c takes unit c = (b, hk) whole -- sequence b = c / Hkv, one row
// tile -- so no unit is ever cut, every result is written by the split
// kernel and no merge runs.  Same scan as block_share (each thread weighs a
// run of sequences); the thread whose run holds b finds the unit's first
// position.  Returns false for a block without a unit (b past B_max, or a
// sequence without query tokens).
__device__ __forceinline__ bool unit_share(const Params &p, int c, int tid, int nthreads, bool report,
                                           long long *scan, long long *first, Share &sh) {
    const int warp = tid >> 5, lane = tid & 31;
    const int per = (p.B_max + nthreads - 1) / nthreads;
    const int b_lo = min(p.B_max, tid * per), b_hi = min(p.B_max, b_lo + per);
    const int bc = c / p.Hkv, hk = c - bc * p.Hkv;
    long long my = 0, w_c = 0, before_c = 0;                // run weight; unit c's weight; run weight before b_c
    for (int b = b_lo; b < b_hi; ++b) {
        const long long w = (long long)p.Hkv * seq_len(p, b, report).tpu;
        if (b < bc) before_c += w;
        if (b == bc) w_c = w / p.Hkv;
        my += w;
    }
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
    if (bc >= b_lo && bc < b_hi && w_c > 0) {
        first[0] = bc;
        first[1] = incl - my + scan[warp] + before_c;       // tiles before sequence b_c
        scan[0] = w_c;                                      // (every thread has read its scan entry)
    }
    __syncthreads();
    sh.Ce = (int)gridDim.x;
    sh.b_first = (int)first[0];
    sh.pb_first = first[1];
    sh.lo = sh.pb_first + hk * scan[0];
    sh.hi = sh.lo + scan[0];
    return bc < p.B_max && sh.b_first >= 0;
}

// The block's tiles in the order its producer loads them.  For every segment
// of the block (OrderedWalker order) begin(seg, role) runs once, then
// tile(seg, t, last) for each tile t of the unit the block takes -- `last`
// marks the block's final tile of that unit -- or none(seg) if it takes none.
// A unit inside the share, and every unit in deterministic mode, is taken as
// the static share gives it.  In the run-time balanced mode the blocks that
// share a cut unit consume it from both ends through one packed counter per
// unit (front count in the high word, back count in the low word): the block
// whose static part is the unit's front claims upward, the others downward,
// kClaim tiles at a time with one claim in flight ahead of the tiles it feeds;
// each claim gets the part of its range that the counter's old value shows as
// still free.  A block's claimed tiles of a cut unit all go out with `last`
// false, followed by none(seg): consumers finish their part of the unit at
// that empty stage.  A callback returns false to stop the walk (a wait gave up);
// the function then returns false.
// WARP: the whole warp calls it in step (every lane walks the same
// schedule; lane 0 alone takes the claims and the result is broadcast), so
// that the callbacks can spread their work over the lanes.
template <bool WARP = false, bool HF = false, class Begin, class Tile, class None>
__device__ __forceinline__ bool feed_tiles(const Params &p, int b_first, long long pb_first, long long lo,
                                           long long hi, Begin &&begin, Tile &&tile, None &&none) {
    OrderedWalker<HF> wk;
    wk.init(p, b_first, pb_first, lo, hi, false, p.head_first != 0);
    Segment seg;
    int role;
    while (wk.next(p, seg, role)) {
        if (!begin(seg, role)) return false;
        const int ntiles = seg.nt;
        if (role == 0 || !p.dynamic) {
            const int tb = role == 0 ? 0 : max(0, seg.t0 - p.unit_cost);
            const int te = role == 0 ? ntiles : min(ntiles, max(0, seg.t1 - p.unit_cost));
            for (int t = tb; t < te; ++t)
                if (!tile(seg, t, t == te - 1)) return false;
            if (te <= tb && !none(seg)) return false;
            continue;
        }
        unsigned long long *claim = p.claim + unit_index(p, seg.b, seg.hk, seg.rt);
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
        // The next claim goes out when a range starts and is resolved only
        // after that range's tiles have been fed, so the atomic's round trip
        // overlaps them; the tiles therefore cannot be told which one ends
        // the block's part, and an empty terminator stage (none) marks the
        // end instead.
        // a claim's result lives on lane 0 until it is needed (WARP)
        auto take = [&]() -> unsigned long long {
            return (!WARP || (threadIdx.x & 31) == 0) ? atomicAdd(claim, inc) : 0ull;
        };
        auto seen = [&](unsigned long long v) -> unsigned long long {
            if constexpr (WARP) return __shfl_sync(0xffffffffu, v, 0);
            return v;
        };
        int a_lo, a_hi;
        range(seen(take()), a_lo, a_hi);
        while (a_lo < a_hi) {
            const bool more = up ? a_hi < ntiles : a_lo > 0;   // this range did not reach the far end
            unsigned long long pend = 0;
            if (more) pend = take();
            for (int i = 0; i < a_hi - a_lo; ++i)
                if (!tile(seg, up ? a_lo + i : a_hi - 1 - i, false)) return false;
            if (!more) break;
            range(seen(pend), a_lo, a_hi);
        }
        if (!none(seg)) return false;
    }
    return true;
}

// For a speculative L2 prefetch before the kernel's dependency wait: the
// first `budget` tiles the block is likely to load, fn(seg, t) for each,
// spread over the calling warp's lanes (lane i takes tiles i, i + 32, ...) --
// but only for a block whose share holds no whole unit, that is one that
// starts on a unit shared with other blocks (few, long units: long-context
// decode, short-query batches).  A block that starts on units of its own
// prefetches nothing: measured on continuous batching, such prefetches
// slowed the calls by about 1.5%, the previous call's last blocks, which
// wait on DRAM latency, getting slower under the added traffic.
// In the static mode a cut unit starts where feed_tiles starts it.  In the
// run-time balanced mode the block holding the unit's front starts at its
// tile 0; the others claim from the back, and together their first claims
// take the unit's last tiles, so the j-th of them (j >= 1 in share order)
// takes tiles [nt - j * budget, nt - (j - 1) * budget).
template <bool HF = false, class Fn>
__device__ __forceinline__ void first_tiles(const Params &p, int c, const Share &sh, int budget, bool spec,
                                            Fn &&fn) {
    OrderedWalker<HF> wk;
    wk.init(p, sh.b_first, sh.pb_first, sh.lo, sh.hi, spec, p.head_first != 0);
    Segment seg;
    int role;
    const int lane = threadIdx.x & 31;
    int done = 0;
    while (done < budget && wk.next(p, seg, role)) {
        if (role == 0) return;                         // the share starts on a unit of its own
        const int nt = seg.nt;
        int a = 0, dir = 1, cnt;
        if (!p.dynamic) {
            a = max(0, seg.t0 - p.unit_cost);
            cnt = min(nt, max(0, seg.t1 - p.unit_cost)) - a;
        } else if (seg.t0 == 0) {
            cnt = nt;
        } else {
            const int j = c - block_of(seg.Pu, sh.T, sh.Ce);
            const int e = nt - (j - 1) * budget;
            a = e - 1;
            dir = -1;
            cnt = min(e, budget);
        }
        cnt = max(0, min(cnt, budget - done));
        for (int i = lane; i < cnt; i += 32) fn(seg, a + dir * i);
        done += cnt;
    }
}

}  // namespace sched
}  // namespace vgqa
