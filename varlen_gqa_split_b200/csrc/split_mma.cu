// split_mma.cu -- TMA-fed tensor-core split-KV kernel for decode-sized row
// counts (G * q_len <= 16 query rows per KV head).
//
// Block = 4 consumer warps + 1 producer warp; one block per (KV chunk z,
// KV head hk, sequence b).
//
// Producer: one lane streams the chunk's K and V tiles (64 keys x D) with
// cp.async.bulk.tensor (no multicast) into a ring of shared-memory stages in
// the 128-byte swizzled layout, completing an mbarrier per stage; the K/V
// stream carries an L2 evict-first policy since every byte is read once.
//
// Consumers: warp w takes keys 16w .. 16w+15 of every tile and keeps its own
// online-softmax state, so no cross-warp exchange happens inside the loop.
// Because the rows (the G query heads of the KV head, times the query tokens)
// number at most 16, the contraction is done with keys on the MMA's M side:
//     S^T [16 keys x rows] = K [16 keys x D] . Q^T        (m16n8k16, A = K)
//     O^T [D x rows]      += V^T [D x 16 keys] . P^T      (A = V^T via ldmatrix.trans)
// P^T moves from the accumulator layout of the first product to the operand
// layout of the second with movmatrix.trans, without touching shared memory.
// The rows of the group share every K/V byte (the G fold of the kernbench2
// docs/adr-proposed commit log, GQA entry).  Q stays raw bf16 in registers and
// the softmax scale enters in fp32 inside the exp2 argument, so scaling costs
// no precision.
//
// After the chunk the four warp states are merged in shared memory; the block
// writes the normalised output and lse (one chunk per sequence), or
// unnormalised (O, m, l) partials for the combine kernel.
//
// Tail tiles: a tile whose 64 keys would run past the end of the sequence is
// loaded ending at the sequence's last key instead (its start moves back; keys
// before the tile's nominal start are masked), so no load ever reads past
// cu_k[b+1].  A start before the first token of the buffer is a negative TMA
// coordinate, which the hardware fills with zeros.
#include "common.cuh"
#include "kernels.h"

namespace vgqa {

namespace {

constexpr int kBN = 64;                   // keys per tile
constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;

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

template <int D, int NT>
__global__ void __launch_bounds__(kThreads) split_mma_kernel(const __grid_constant__ CUtensorMap tm_k,
                                                             const __grid_constant__ CUtensorMap tm_v,
                                                             const Params p, const int stages) {
    using L = MmaLayout<D>;
    constexpr int KS = D / 16;           // k-steps of S^T, m-tiles of O^T
    constexpr int ROWS = 8 * NT;
    constexpr int OLD = D + 4;           // fp32 row stride of the merge buffer

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + stages * L::kStageBytes);
    uint64_t *empty = full + stages;
    int *failed = reinterpret_cast<int *>(empty + stages);

    const int z = blockIdx.x;
    const int hk = blockIdx.y;
    const int b = blockIdx.z;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;

    int q0, Lq, k0, Lk;
    if (!load_lengths(p, b, z == 0 && hk == 0, q0, Lq, k0, Lk)) return;
    const int G = p.G;
    const int R = G * Lq;                 // <= ROWS by plan
    if (R == 0) return;
    const int c_begin = z * p.chunk;
    const int c_end = min(c_begin + p.chunk, Lk);
    if (p.nsplit > 1 && z >= live_chunks(Lk, p.chunk)) return;   // dead chunk: the merge skips it
    const int kv_lim = min(c_end, Lk - Lq + (R - 1) / G + 1);
    const int n_tiles = kv_lim > c_begin ? (kv_lim - c_begin + kBN - 1) / kBN : 0;

    if (tid == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        *failed = 0;
        fence_barrier_init();
    }
    __syncthreads();

    // ------------------------------------------------------------ producer
    if (warp == kConsumerWarps) {
        if (lane == 0 && n_tiles > 0) {
            prefetch_tensormap(&tm_k);
            prefetch_tensormap(&tm_v);
            const uint64_t pol = l2_evict_first();
            int s = 0;
            uint32_t phase = 0;
            for (int i = 0; i < n_tiles; ++i) {
                if (i >= stages && !mbar_wait(&empty[s], phase ^ 1)) {
                    atomicOr(p.err, ATTN_DEV_ERR_TIMEOUT);
                    break;
                }
                const int t0 = c_begin + i * kBN;
                const int row = k0 + min(t0, Lk - kBN);
                uint8_t *st = smem + s * L::kStageBytes;
                mbar_arrive_expect_tx(&full[s], L::kStageBytes);
#pragma unroll
                for (int hf = 0; hf < L::kHalves; ++hf)
                    tma_load_3d(st + hf * L::kRegion, &tm_k, &full[s], hf * 64, hk, row, pol);
#pragma unroll
                for (int hf = 0; hf < L::kHalves; ++hf)
                    tma_load_3d(st + L::kTileBytes + hf * L::kRegion, &tm_v, &full[s], hf * 64, hk,
                                row, pol);
                if (++s == stages) {
                    s = 0;
                    phase ^= 1;
                }
            }
        }
        return;
    }

    // ------------------------------------------------------------ consumers
    const int grp = lane >> 2, tig = lane & 3;
    const float c = p.scale_log2;

    // Q^T fragments (B operand of S^T): row n = nt*8 + grp, d = 16ks + 2tig (+8)
    uint32_t qf[NT][KS][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int r = nt * 8 + grp;
        const bool ok = r < R;
        const uint32_t *qp = reinterpret_cast<const uint32_t *>(
            p.q + ((long long)(q0 + (ok ? r / G : 0)) * p.Hq + hk * G + (ok ? r % G : 0)) * D);
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            qf[nt][ks][0] = ok ? __ldg(qp + (ks * 16 + 2 * tig) / 2) : 0u;
            qf[nt][ks][1] = ok ? __ldg(qp + (ks * 16 + 8 + 2 * tig) / 2) : 0u;
        }
    }

    // this thread's softmax rows: n = nt*8 + 2tig + e
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

    const uint32_t smem_base = smem_u32(smem);
    const int kbase = warp * 16;
    // ldmatrix lane -> (row, chunk) offsets
    const int mi = lane >> 3;
    const int k_row = kbase + (mi & 1) * 8 + (lane & 7);    // K: matrices (keys lo/hi) x (d lo/hi)
    const int k_cadd = mi >> 1;
    const int v_row = kbase + (mi >> 1) * 8 + (lane & 7);   // V^T: matrices (d lo/hi) x (keys lo/hi)
    const int v_cadd = mi & 1;

    int s = 0;
    uint32_t phase = 0;
    bool ok_run = true;
    for (int i = 0; i < n_tiles; ++i) {
        if (!mbar_wait(&full[s], phase)) {
            atomicOr(p.err, ATTN_DEV_ERR_TIMEOUT);
            ok_run = false;
            break;
        }
        const uint32_t kst = smem_base + s * L::kStageBytes;
        const uint32_t vst = kst + L::kTileBytes;
        const int t0 = c_begin + i * kBN;
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
                const int lim = min(kv_lim, vis[nt][e]);
                const float x_lo = (j_lo >= t0 && j_lo < lim) ? sacc[nt][e] : -INFINITY;
                const float x_hi = (j_hi >= t0 && j_hi < lim) ? sacc[nt][2 + e] : -INFINITY;
                float mx = fmaxf(x_lo, x_hi);
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                const float m_new = fmaxf(m[nt][e], mx * c);
                const float m_ref = m_new == -INFINITY ? 0.f : m_new;
                const float alpha = ex2(m[nt][e] - m_ref);
                pl[e] = ex2(fmaf(x_lo, c, -m_ref));
                ph[e] = ex2(fmaf(x_hi, c, -m_ref));
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
    }
    if (!ok_run) *failed = 1;   // benign race: every writer stores 1

    // ------------------------------------------------------------ merge the 4 warps
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
    named_sync(1, kConsumerWarps * 32);   // all stages consumed: reuse stage memory

    float *ms = reinterpret_cast<float *>(smem);                  // [4][ROWS]
    float *lsum = ms + kConsumerWarps * ROWS;                     // [4][ROWS]
    float *ored = lsum + kConsumerWarps * ROWS;                   // [4][ROWS][OLD]
    if (grp == 0) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                ms[warp * ROWS + nt * 8 + 2 * tig + e] = m[nt][e];
                lsum[warp * ROWS + nt * 8 + 2 * tig + e] = l[nt][e];
            }
    }
    named_sync(1, kConsumerWarps * 32);
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
    named_sync(1, kConsumerWarps * 32);
    if (*failed) return;

    // ------------------------------------------------------------ epilogue
    const int ctid = tid;                  // 0 .. 127
    for (int idx = ctid; idx < ROWS * (D / 4); idx += kConsumerWarps * 32) {
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
        const int qi = row / G, h = hk * G + row % G;
        if (p.nsplit == 1) {
            const long long tok = q0 + qi;
            const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
            uint2 packed;
            packed.x = pack_bf16x2(acc.x * inv, acc.y * inv);
            packed.y = pack_bf16x2(acc.z * inv, acc.w * inv);
            *reinterpret_cast<uint2 *>(p.out + (tok * p.Hq + h) * D + d4) = packed;
            if (d4 == 0) p.lse[tok * p.Hq + h] = Lsum > 0.f ? (M + log2f(Lsum)) * kLn2 : -INFINITY;
        } else {
            const long long pi = part_index(p, b, qi, h, z);
            *reinterpret_cast<float4 *>(p.o_part + pi * D + d4) = acc;
            if (d4 == 0) p.ml_part[pi] = make_float2(M, Lsum);
        }
    }

    // fused merge: the last block of (b, hk) to finish merges every split
    if (p.nsplit > 1 && p.fused) {
        const int n_live = live_chunks(Lk, p.chunk);
        if (ticket_last(p.ticket + (long long)b * p.Hkv + hk, n_live, ctid, kConsumerWarps * 32, 1,
                        failed + 1)) {
            merge_unit<D>(p, b, q0, hk, 0, R, n_live, smem, ctid, kConsumerWarps * 32, 1);
            if (ctid == 0) p.ticket[(long long)b * p.Hkv + hk] = 0u;
        }
    }
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

size_t mma_smem_bytes(int D, int NT, int stages) {
    const size_t stage = D == 64 ? MmaLayout<64>::kStageBytes : MmaLayout<128>::kStageBytes;
    const size_t rows = 8 * NT;
    const size_t merge = 2 * kConsumerWarps * rows * 4 + kConsumerWarps * rows * (D + 4) * 4;
    size_t body = stage * stages;
    if (body < merge) body = merge;
    // 1 KB alignment slack + barriers + flag
    return 1024 + body + 2 * stages * sizeof(uint64_t) + 16;
}

size_t mma_merge_capacity(int D, int stages) {
    return (size_t)stages * (D == 64 ? MmaLayout<64>::kStageBytes : MmaLayout<128>::kStageBytes);
}

int mma_block_n() { return kBN; }
int mma_threads() { return kThreads; }

cudaError_t mma_prepare(int D, int NT, int stages) {
    return cudaFuncSetAttribute(pick(D, NT), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)mma_smem_bytes(D, NT, stages));
}

cudaError_t launch_split_mma(const Params &p, const CUtensorMap &tm_k, const CUtensorMap &tm_v, int NT,
                             int stages, dim3 grid, cudaStream_t stream) {
    const size_t smem = mma_smem_bytes(p.D, NT, stages);
    if (p.D == 64) {
        if (NT == 1)
            split_mma_kernel<64, 1><<<grid, kThreads, smem, stream>>>(tm_k, tm_v, p, stages);
        else
            split_mma_kernel<64, 2><<<grid, kThreads, smem, stream>>>(tm_k, tm_v, p, stages);
    } else {
        if (NT == 1)
            split_mma_kernel<128, 1><<<grid, kThreads, smem, stream>>>(tm_k, tm_v, p, stages);
        else
            split_mma_kernel<128, 2><<<grid, kThreads, smem, stream>>>(tm_k, tm_v, p, stages);
    }
    return cudaGetLastError();
}

}  // namespace vgqa
