// split_simt.cu -- CUDA-core split-KV kernel: any number of query rows.
//
// One block handles (KV chunk z, KV head hk, row tile rt, sequence b).  Its
// rows are r = qi * G + g for the G query heads of KV head hk and the query
// tokens qi of sequence b (the group folded into the row dimension, as in the
// kernbench2 docs/adr-proposed commit log, GQA entry), 16 rows per tile.  The
// block streams its chunk of keys in tiles of 64 through double-buffered
// shared memory (cp.async, 16-byte vectors, rows past the chunk zero-filled)
// and keeps a running (m, l, O) per row (online softmax).  With one chunk per
// sequence it writes the normalised output and lse directly; otherwise it
// writes unnormalised partials for the combine kernel (AstrAI commit log for
// csrc/kernels/gqa_decode_attn.cu, split-KV commit).
//
// Scores live in base-2 units: q is pre-scaled by (1/sqrt(D)) * log2(e) when
// it is staged (fp32, so the pre-scale costs no precision), and the softmax
// uses exp2.
#include "common.cuh"
#include "kernels.h"

namespace vgqa {

namespace {

constexpr int kRows = 16;      // query rows per block
constexpr int kBN = 64;        // keys per tile
constexpr int kThreads = 128;

template <int D>
struct SimtSmem {
    static constexpr int kLd = D + 8;   // bf16 row stride of K/V tiles (bank spread)
    float q[kRows][D];
    __nv_bfloat16 k[2][kBN][kLd];
    __nv_bfloat16 v[2][kBN][kLd];
    float s[kRows][kBN];               // scores, then probabilities
    float m[kRows], l[kRows], alpha[kRows];
    int vis[kRows];                    // keys [0, vis) visible to the row
    int flag;                          // fused-merge ticket result
};

template <int D>
__global__ void __launch_bounds__(kThreads) split_simt_kernel(const Params p) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    SimtSmem<D> &sm = *reinterpret_cast<SimtSmem<D> *>(smem_raw);

    const int z = blockIdx.x;
    const int hk = blockIdx.y / p.row_tiles;
    const int rt = blockIdx.y % p.row_tiles;
    const int b = blockIdx.z;
    const int tid = threadIdx.x;

    int q0, Lq, k0, Lk;
    if (!load_lengths(p, b, z == 0 && blockIdx.y == 0, q0, Lq, k0, Lk)) return;
    const int G = p.G;
    const int R = G * Lq;
    const int r_begin = rt * kRows;
    if (r_begin >= R) return;                       // no query rows here
    const int nrows = min(kRows, R - r_begin);
    const int c_begin = z * p.chunk;
    const int c_end = min(c_begin + p.chunk, Lk);
    if (p.nsplit > 1 && z >= live_chunks(Lk, p.chunk)) return;   // dead chunk: the merge skips it

    // keys any row of this tile may see inside the chunk (tail-aligned causal)
    const int qi_last = (r_begin + nrows - 1) / G;
    const int kv_lim = min(c_end, Lk - Lq + qi_last + 1);
    const int n_tiles = kv_lim > c_begin ? (kv_lim - c_begin + kBN - 1) / kBN : 0;

    // stage q (pre-scaled, fp32) and the per-row state
    for (int idx = tid; idx < kRows * D; idx += kThreads) {
        const int r = idx / D, d = idx % D;
        float val = 0.f;
        if (r < nrows) {
            const int row = r_begin + r;
            const int qi = row / G, g = row % G;
            val = __bfloat162float(p.q[((long long)(q0 + qi) * p.Hq + hk * G + g) * D + d]) *
                  p.scale_log2;
        }
        sm.q[r][d] = val;
    }
    if (tid < kRows) {
        sm.m[tid] = -INFINITY;
        sm.l[tid] = 0.f;
        sm.vis[tid] = tid < nrows ? Lk - Lq + (r_begin + tid) / G + 1 : 0;
    }

    auto issue = [&](int i, int buf) {
        const int t0 = c_begin + i * kBN;
        constexpr int kChunks = D / 8;            // 16-byte pieces per row
        for (int c = tid; c < kBN * kChunks; c += kThreads) {
            const int rr = c / kChunks, ch = c % kChunks;
            const int j = t0 + rr;
            bool ok = j < kv_lim;
            long long ko = 0, vo = 0;                  // element offsets of the key's token
            if (ok && p.block_table) {                 // paged: page from the block table
                const int pg = page_of(p, b, j);
                ok = pg < p.num_pages;
                ko = vo = (long long)pg * p.page_stride + (long long)(j & ((1 << p.page_shift) - 1)) * p.k_stride;
            } else if (ok) {
                ko = (long long)(k0 + j) * p.k_stride;
                vo = (long long)(k0 + j) * p.v_stride;
            }
            const long long hd = (long long)hk * D + ch * 8;
            cp_async_16(smem_u32(&sm.k[buf][rr][ch * 8]), p.k + (ok ? ko + hd : 0), ok);
            cp_async_16(smem_u32(&sm.v[buf][rr][ch * 8]), p.v + (ok ? vo + hd : 0), ok);
        }
        cp_async_commit();
    };

    // thread roles
    const int kk = tid & (kBN - 1);                 // score phase: one key ...
    const int shalf = tid / kBN;                    // ... and 8 rows
    constexpr int kDP = D / 2;                      // PV phase: one d pair ...
    constexpr int kRG = kThreads / kDP;             // ... row groups
    constexpr int kRPG = kRows / kRG;               // rows per group
    const int dp = tid % kDP;
    const int rg = tid / kDP;

    float acc[kRPG][2];
#pragma unroll
    for (int r = 0; r < kRPG; ++r) acc[r][0] = acc[r][1] = 0.f;

    if (n_tiles > 0) issue(0, 0);
    __syncthreads();

    for (int i = 0; i < n_tiles; ++i) {
        const int buf = i & 1;
        if (i + 1 < n_tiles) {
            issue(i + 1, buf ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();

        // ---- scores: thread -> (key kk, rows shalf*8 .. +8)
        {
            const int j = c_begin + i * kBN + kk;
            float sc[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) sc[r] = 0.f;
            const __nv_bfloat16 *krow = &sm.k[buf][kk][0];
#pragma unroll 4
            for (int d = 0; d < D; d += 8) {
                const uint4 kv = *reinterpret_cast<const uint4 *>(krow + d);
                const float kf[8] = {bf16lo(kv.x), bf16hi(kv.x), bf16lo(kv.y), bf16hi(kv.y),
                                     bf16lo(kv.z), bf16hi(kv.z), bf16lo(kv.w), bf16hi(kv.w)};
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    const float4 qa = *reinterpret_cast<const float4 *>(&sm.q[shalf * 8 + r][d]);
                    const float4 qb = *reinterpret_cast<const float4 *>(&sm.q[shalf * 8 + r][d + 4]);
                    sc[r] = fmaf(qa.x, kf[0], sc[r]);
                    sc[r] = fmaf(qa.y, kf[1], sc[r]);
                    sc[r] = fmaf(qa.z, kf[2], sc[r]);
                    sc[r] = fmaf(qa.w, kf[3], sc[r]);
                    sc[r] = fmaf(qb.x, kf[4], sc[r]);
                    sc[r] = fmaf(qb.y, kf[5], sc[r]);
                    sc[r] = fmaf(qb.z, kf[6], sc[r]);
                    sc[r] = fmaf(qb.w, kf[7], sc[r]);
                }
            }
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const int row = shalf * 8 + r;
                const bool ok = row < nrows && j < kv_lim && j < sm.vis[row];
                sm.s[row][kk] = ok ? sc[r] : -INFINITY;
            }
        }
        __syncthreads();

        // ---- online softmax: 8 threads per row, 8 keys each
        {
            const int row = tid >> 3, sub = tid & 7;
            float x[8];
            float mx = -INFINITY;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                x[e] = sm.s[row][sub * 8 + e];
                mx = fmaxf(mx, x[e]);
            }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            const float m_old = sm.m[row];
            const float m_new = fmaxf(m_old, mx);
            const float m_ref = m_new == -INFINITY ? 0.f : m_new;   // keeps -inf - -inf out
            float sum = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float pe = ex2(x[e] - m_ref);
                sm.s[row][sub * 8 + e] = pe;
                sum += pe;
            }
            sum += __shfl_xor_sync(0xffffffffu, sum, 1);
            sum += __shfl_xor_sync(0xffffffffu, sum, 2);
            sum += __shfl_xor_sync(0xffffffffu, sum, 4);
            __syncwarp();
            if (sub == 0) {
                const float a = ex2(m_old - m_ref);
                sm.alpha[row] = a;
                sm.l[row] = sm.l[row] * a + sum;
                sm.m[row] = m_new;
            }
        }
        __syncthreads();

        // ---- O = alpha * O + P V: thread -> (d pair dp, rows rg*kRPG .. +kRPG)
        {
#pragma unroll
            for (int r = 0; r < kRPG; ++r) {
                const float a = sm.alpha[rg * kRPG + r];
                acc[r][0] *= a;
                acc[r][1] *= a;
            }
#pragma unroll 8
            for (int key = 0; key < kBN; ++key) {
                const uint32_t vv = *reinterpret_cast<const uint32_t *>(&sm.v[buf][key][2 * dp]);
                const float v0 = bf16lo(vv), v1 = bf16hi(vv);
#pragma unroll
                for (int r = 0; r < kRPG; ++r) {
                    const float pr = sm.s[rg * kRPG + r][key];
                    acc[r][0] = fmaf(pr, v0, acc[r][0]);
                    acc[r][1] = fmaf(pr, v1, acc[r][1]);
                }
            }
        }
        __syncthreads();
    }

    // ---- epilogue
#pragma unroll
    for (int r = 0; r < kRPG; ++r) {
        const int row = rg * kRPG + r;
        if (row >= nrows) continue;
        const int qrow = r_begin + row;
        const int qi = qrow / G, h = hk * G + qrow % G;
        const float L = sm.l[row], M = sm.m[row];
        if (p.nsplit == 1) {
            const long long tok = q0 + qi;
            const float inv = L > 0.f ? 1.f / L : 0.f;
            *reinterpret_cast<uint32_t *>(p.out + (tok * p.Hq + h) * D + 2 * dp) =
                pack_bf16x2(acc[r][0] * inv, acc[r][1] * inv);
            if (dp == 0) p.lse[tok * p.Hq + h] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
        } else {
            const long long pi = part_index(p, b, qi, h, z);
            *reinterpret_cast<float2 *>(p.o_part + pi * D + 2 * dp) = make_float2(acc[r][0], acc[r][1]);
            if (dp == 0) p.ml_part[pi] = make_float2(M, L);
        }
    }

    // fused merge: the last block of (b, hk, rt) to finish merges every split
    if (p.nsplit > 1 && p.fused) {
        const int n_live = live_chunks(Lk, p.chunk);
        uint32_t *t = p.ticket + ((long long)b * p.Hkv + hk) * p.row_tiles + rt;
        if (ticket_last(t, n_live, tid, kThreads, 0, &sm.flag)) {
            merge_unit<D>(p, b, q0, hk, r_begin, nrows, n_live, &sm.k[0][0][0], tid, kThreads, 0);
            if (tid == 0) *t = 0u;
        }
    }
}

}  // namespace

size_t simt_merge_capacity(int D) {   // shared bytes the fused merge may use
    return D == 64 ? sizeof(SimtSmem<64>::k) : sizeof(SimtSmem<128>::k);
}

size_t simt_smem_bytes(int D) {
    return D == 64 ? sizeof(SimtSmem<64>) : sizeof(SimtSmem<128>);
}

cudaError_t simt_prepare(int D) {
    if (D == 64)
        return cudaFuncSetAttribute(split_simt_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)sizeof(SimtSmem<64>));
    return cudaFuncSetAttribute(split_simt_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)sizeof(SimtSmem<128>));
}

cudaError_t launch_split_simt(const Params &p, dim3 grid, cudaStream_t stream) {
    if (p.D == 64)
        split_simt_kernel<64><<<grid, kThreads, sizeof(SimtSmem<64>), stream>>>(p);
    else
        split_simt_kernel<128><<<grid, kThreads, sizeof(SimtSmem<128>), stream>>>(p);
    return cudaGetLastError();
}

}  // namespace vgqa
