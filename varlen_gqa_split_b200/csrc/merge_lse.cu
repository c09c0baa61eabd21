// merge_lse.cu -- merge of n normalised attention results over disjoint key
// ranges, given as (out_r, lse_r) pairs: the exchange step of context
// parallelism, where each GPU attends over its own stretch of every
// sequence's keys and the results are combined after an all-gather.
//
// One warp per (query token, head) row.  With lse_r the natural-log
// normaliser of part r (-inf for a part that saw no key):
//     M = max_r lse_r,   w_r = e^(lse_r - M),   L = sum_r w_r,
//     out = sum_r w_r out_r / L,   lse = M + ln L,
// and a row no part saw a key for gets out = 0, lse = -inf.  This is the
// log-sum-exp merge of split partials (AstrAI commit log for
// csrc/kernels/gqa_decode_attn.cu, split-KV commit) applied to normalised
// parts, the running (m, l, O) reduction across devices of the kernbench2
// docs/adr-proposed commit log (GQA entry: reduction of the running state
// between devices).  Only tokens [cu_q[0], cu_q[B_max]) are written.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "../../include/varlen_gqa.h"

#define ATTN_EXPORT extern "C" __attribute__((visibility("default")))

namespace vgqa {

namespace {

constexpr int kWarps = 8;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
__global__ void __launch_bounds__(kWarps * 32) merge_lse_kernel(int n, const __nv_bfloat16 *__restrict__ outs,
                                                                const float *__restrict__ lses, long long T_q,
                                                                const int32_t *__restrict__ cu_q, int B_max, int Hq,
                                                                __nv_bfloat16 *__restrict__ out,
                                                                float *__restrict__ lse) {
    constexpr int VEC = D / 32;               // bf16 values per lane: 4 or 2
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);   // token * Hq + h
    const long long t_lo = (long long)__ldg(cu_q) * Hq, t_hi = (long long)__ldg(cu_q + B_max) * Hq;
    const long long part_rows = T_q * Hq;
    if (row < t_lo || row >= t_hi || row >= part_rows) return;

    float M = -INFINITY;
    for (int r = lane; r < n; r += 32) M = fmaxf(M, __ldg(lses + r * part_rows + row));
#pragma unroll
    for (int off = 16; off; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));

    float acc[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) acc[i] = 0.f;
    float L = 0.f;
    if (M != -INFINITY) {
        for (int r = 0; r < n; ++r) {
            const float lr = __ldg(lses + r * part_rows + row);
            if (lr == -INFINITY) continue;               // no key in this part: weight 0, value unused
            const float w = exp2f((lr - M) * kLog2e);
            L += w;
            const __nv_bfloat16 *src = outs + (r * part_rows + row) * D + lane * VEC;
            if constexpr (VEC == 4) {
                const uint2 x = __ldg(reinterpret_cast<const uint2 *>(src));
                const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(&x.x);
                const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&x.y);
                acc[0] = fmaf(w, __low2float(a), acc[0]);
                acc[1] = fmaf(w, __high2float(a), acc[1]);
                acc[2] = fmaf(w, __low2float(b), acc[2]);
                acc[3] = fmaf(w, __high2float(b), acc[3]);
            } else {
                const uint32_t x = __ldg(reinterpret_cast<const uint32_t *>(src));
                const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(&x);
                acc[0] = fmaf(w, __low2float(a), acc[0]);
                acc[1] = fmaf(w, __high2float(a), acc[1]);
            }
        }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    __nv_bfloat16 *dst = out + row * D + lane * VEC;
    if constexpr (VEC == 4) {
        const __nv_bfloat162 a = __floats2bfloat162_rn(acc[0] * inv, acc[1] * inv);
        const __nv_bfloat162 b = __floats2bfloat162_rn(acc[2] * inv, acc[3] * inv);
        uint2 x;
        x.x = *reinterpret_cast<const uint32_t *>(&a);
        x.y = *reinterpret_cast<const uint32_t *>(&b);
        *reinterpret_cast<uint2 *>(dst) = x;
    } else {
        const __nv_bfloat162 a = __floats2bfloat162_rn(acc[0] * inv, acc[1] * inv);
        *reinterpret_cast<__nv_bfloat162 *>(dst) = a;
    }
    if (lane == 0) lse[row] = L > 0.f ? M + logf(L) : -INFINITY;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

}  // namespace vgqa

ATTN_EXPORT int attn_merge_lse(int n_parts, const void *outs, const float *lses, int64_t T_q, const int32_t *cu_q,
                               int B_max, int Hq, int D, void *out, float *lse, void *stream) {
    using namespace vgqa;
    if (!outs || !lses || !cu_q || !out || !lse) return ATTN_E_NULL;
    if (n_parts < 1 || n_parts > 65536 || T_q < 1 || B_max < 1 || Hq < 1) return ATTN_E_INVALID_ARG;
    if (D != 64 && D != 128) return ATTN_E_UNSUPPORTED;
    if ((long long)T_q * Hq > (1ll << 40)) return ATTN_E_INVALID_ARG;
    if (!aligned(outs, 16) || !aligned(out, 16) || !aligned(lses, 4) || !aligned(lse, 4) || !aligned(cu_q, 4))
        return ATTN_E_ALIGNMENT;
    const long long rows = (long long)T_q * Hq;
    const long long blocks = (rows + kWarps - 1) / kWarps;
    if (blocks > 0x7fffffffll) return ATTN_E_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const auto *o = static_cast<const __nv_bfloat16 *>(outs);
    auto *d = static_cast<__nv_bfloat16 *>(out);
    if (D == 128)
        merge_lse_kernel<128><<<(unsigned)blocks, kWarps * 32, 0, s>>>(n_parts, o, lses, T_q, cu_q, B_max, Hq, d, lse);
    else
        merge_lse_kernel<64><<<(unsigned)blocks, kWarps * 32, 0, s>>>(n_parts, o, lses, T_q, cu_q, B_max, Hq, d, lse);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_E_CUDA;
}
