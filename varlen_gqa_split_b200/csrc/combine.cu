// combine.cu -- log-sum-exp merge of split-KV partials.
//
// One warp per query row (b, qi, h).  The live splits of sequence b are
// z < max(1, ceil(Lk_b / chunk)) (the others exited without writing); each left
// (O_z, m_z, l_z), with O_z unnormalised and m_z in base-2 units of the scaled
// scores.  The merge is
//     M = max_z m_z over splits with l_z > 0,   L = sum_z l_z 2^(m_z - M),
//     out = sum_z O_z 2^(m_z - M) / L,          lse = (M + log2 L) ln 2,
// and L = 0 (no visible key) gives out = 0, lse = -inf (AstrAI commit log for
// csrc/kernels/gqa_decode_attn.cu, split-KV commit; magik.net "Wiring Split-K
// Dispatch into a Custom CUDA Attention Kernel", section "The Message").
#include "common.cuh"
#include "kernels.h"

namespace vgqa {

namespace {

constexpr int kWarps = 4;

template <int D>
__global__ void __launch_bounds__(kWarps * 32) combine_kernel(const Params p) {
    constexpr int VEC = D / 32;           // fp32 values per lane (4 or 2)
    const int lane = threadIdx.x & 31;
    const long long gw = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const long long total = (long long)p.B_max * p.max_q * p.Hq;
    if (gw >= total) return;
    const int h = (int)(gw % p.Hq);
    const long long t = gw / p.Hq;
    const int qi = (int)(t % p.max_q);
    const int b = (int)(t / p.max_q);

    int q0, Lq, k0, Lk;
    if (!load_lengths(p, b, false, q0, Lq, k0, Lk)) return;
    if (qi >= Lq) return;
    const int n_live = min(p.nsplit, live_chunks(Lk, p.chunk));
    const long long base = part_index(p, b, qi, h, 0);

    float M = -INFINITY;
    for (int zz = lane; zz < n_live; zz += 32) {
        const float2 ml = p.ml_part[base + zz];
        if (ml.y > 0.f) M = fmaxf(M, ml.x);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float Mref = M == -INFINITY ? 0.f : M;

    float L = 0.f;
    float acc[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
    for (int zz = 0; zz < n_live; ++zz) {
        const float2 ml = p.ml_part[base + zz];
        const float w = ml.y > 0.f ? ex2(ml.x - Mref) : 0.f;
        L += ml.y * w;
        const float *src = p.o_part + (base + zz) * D + lane * VEC;
        if constexpr (VEC == 4) {
            const float4 x = *reinterpret_cast<const float4 *>(src);
            acc[0] = fmaf(w, x.x, acc[0]);
            acc[1] = fmaf(w, x.y, acc[1]);
            acc[2] = fmaf(w, x.z, acc[2]);
            acc[3] = fmaf(w, x.w, acc[3]);
        } else {
            const float2 x = *reinterpret_cast<const float2 *>(src);
            acc[0] = fmaf(w, x.x, acc[0]);
            acc[1] = fmaf(w, x.y, acc[1]);
        }
    }
    const long long tok = q0 + qi;
    const float inv = L > 0.f ? 1.f / L : 0.f;
    __nv_bfloat16 *dst = p.out + (tok * p.Hq + h) * D + lane * VEC;
    if constexpr (VEC == 4) {
        uint2 pk;
        pk.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
        pk.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
        *reinterpret_cast<uint2 *>(dst) = pk;
    } else {
        *reinterpret_cast<uint32_t *>(dst) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    }
    if (lane == 0) p.lse[tok * p.Hq + h] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
}

}  // namespace

int combine_blocks(const Params &p) {
    const long long total = (long long)p.B_max * p.max_q * p.Hq;
    return (int)((total + kWarps - 1) / kWarps);
}

cudaError_t launch_combine(const Params &p, cudaStream_t stream) {
    const int blocks = combine_blocks(p);
    if (p.D == 64)
        combine_kernel<64><<<blocks, kWarps * 32, 0, stream>>>(p);
    else
        combine_kernel<128><<<blocks, kWarps * 32, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace vgqa
