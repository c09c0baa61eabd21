// api.cpp -- the C ABI of libvgqa (declared in include/varlen_gqa.h).
//
// attn_plan fixes everything that shapes the launch -- kernel variant, split
// count, chunk length, grid, scratch -- from constants (B_max, s_max, head
// counts, head dim, max_q, the device's SM count), so attn_run only fills a
// parameter block, encodes two TMA descriptors on the host and launches: no
// device-to-host copy, no allocation, no compilation (cudnn-frontend issue
// #552 "frost(sdpa): THD execute host round-trip", sections Context and
// Proposal to evaluate).
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <mutex>
#include <unordered_set>

#include "../../include/varlen_gqa.h"
#include "kernels.h"
#include "params.h"

#define ATTN_EXPORT extern "C" __attribute__((visibility("default")))

using namespace vgqa;

struct attn_plan_s {
    attn_plan_desc d;
    int device;
    int NT;                    // tensor-core path: row fragments of 8
    float scale_log2;
    void *scratch;             // one allocation: error word, partials
    uint32_t *err;
    uint32_t *ticket;          // fused-merge arrival counters
    size_t ticket_bytes;
    int merge_bytes;           // tensor-core path: shared bytes of the merge area
    int qtile;                 // tensor-core path: query tokens per row tile
    int max_rt;                // tensor-core path: row tiles per sequence at most
    int direct;                // warp-MMA path: one block per unit, no merge
    float *o_part;
    float2 *ml_part;
    unsigned long long wait_ns; // limit of one bounded wait in the kernels
};

namespace {

std::mutex g_mu;
std::unordered_set<attn_plan_s *> g_plans;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bool live(attn_plan_s *p) {
    std::lock_guard<std::mutex> lk(g_mu);
    return g_plans.count(p) != 0;
}

int get_encoder() {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_encode) return ATTN_OK;
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
        return ATTN_E_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    return ATTN_OK;
}

// [T, Hkv, D] bf16, box = 64 elements x 1 head x block_n tokens, 128-byte
// swizzle.  Packed K/V leave the token extent open (2^31 - 1): every load the
// kernel issues ends at or before its sequence's last key (cu_k[b+1] - 1), so
// the real buffer length never enters.  A paged cache passes its row count,
// so a load at row num_pages * page_rows (the kernels' stand-in for a key
// past the sequence or a bad table entry) lies outside and fills zeros.
int encode_kv_map(CUtensorMap *map, const void *base, int Hkv, int D, int block_n, long long token_stride,
                  long long rows = 0x7fffffff) {
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)token_stride * 2};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)block_n};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? ATTN_OK : ATTN_E_CUDA;
}

// Paged cache [pages, page_size, Hkv, D] bf16 with explicit token and page
// strides, box = 64 elements x 1 head x min(page_size, 64) tokens x 1 page,
// 128-byte swizzle.  A load at page index num_pages (the kernels' stand-in
// for a key past the sequence or a bad table entry) lies wholly outside the
// map and is filled with zeros.
int encode_paged_map(CUtensorMap *map, const void *base, int Hkv, int D, int page_size, int num_pages,
                     long long token_stride, long long page_stride) {
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)page_size, (cuuint64_t)num_pages};
    cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)token_stride * 2, (cuuint64_t)page_stride * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)std::min(page_size, 64), 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? ATTN_OK : ATTN_E_CUDA;
}

// The warp-MMA kernel's K/V maps: the same tensors with the D / 64 halves of
// a row as the outermost dimension (stride 128 bytes), so that one box of
// 64 elements x 1 head x box_rows tokens x D / 64 halves fills a tile's
// halves one after the other ([half][row][128 B], 128-byte swizzle) and a
// tile row range takes one load instead of one per half.  Packed or paged
// with pages a whole number of rows apart: {64, Hkv, rows, halves}; other
// paged caches: {64, Hkv, page_size, num_pages, halves}.
int encode_kv_map_halves(CUtensorMap *map, const void *base, int Hkv, int D, int box_rows, long long token_stride,
                         long long rows) {
    const int halves = D / 64;
    cuuint64_t dims[4] = {64, (cuuint64_t)Hkv, (cuuint64_t)rows, (cuuint64_t)halves};
    cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)token_stride * 2, 128};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, (cuuint32_t)halves};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? ATTN_OK : ATTN_E_CUDA;
}

int encode_paged_map_halves(CUtensorMap *map, const void *base, int Hkv, int D, int page_size, int num_pages,
                            long long token_stride, long long page_stride) {
    const int halves = D / 64;
    cuuint64_t dims[5] = {64, (cuuint64_t)Hkv, (cuuint64_t)page_size, (cuuint64_t)num_pages, (cuuint64_t)halves};
    cuuint64_t strides[4] = {(cuuint64_t)D * 2, (cuuint64_t)token_stride * 2, (cuuint64_t)page_stride * 2, 128};
    cuuint32_t box[5] = {64, 1, (cuuint32_t)std::min(page_size, 64), 1, (cuuint32_t)halves};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? ATTN_OK : ATTN_E_CUDA;
}

// [T, Hq, D] bf16, box = 64 elements x G heads x qtile tokens: one unit's
// query rows (token-major, heads inner) as the tcgen05 kernel's A operand.
// Loads are right-aligned to the sequence's last query token, so, as for K/V,
// the token extent is left open.
int encode_q_map(CUtensorMap *map, const void *base, int Hq, int D, int G, int qtile) {
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hq, (cuuint64_t)0x7fffffff};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hq * D * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)G, (cuuint32_t)qtile};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? ATTN_OK : ATTN_E_CUDA;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int gcd(int a, int b) { return b ? gcd(b, a % b) : a; }

// A stride near n / golden ratio that is coprime with n: b -> (b * stride)
// mod n is then a permutation of the blocks that scatters neighbours.
int share_stride(int n) {
    if (n <= 2) return 1;
    for (int s = (int)(n * 0.6180339887) | 1; s > 1; --s)
        if (gcd(s, n) == 1) return s;
    return 1;
}

bool aligned(const void *ptr, size_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

}  // namespace

ATTN_EXPORT const char *attn_strerror(int code) {
    switch (code) {
    case ATTN_OK: return "success";
    case ATTN_E_INVALID_ARG: return "invalid argument (size or count out of range)";
    case ATTN_E_UNSUPPORTED: return "unsupported configuration (head dim must be 64 or 128)";
    case ATTN_E_NULL: return "a required pointer is NULL";
    case ATTN_E_ALIGNMENT: return "a pointer breaks the alignment contract (16 B tensors, 4 B cu/lse)";
    case ATTN_E_BAD_PLAN: return "unknown or destroyed plan";
    case ATTN_E_CUDA: return "a CUDA call failed";
    case ATTN_E_NOMEM: return "device allocation failed";
    case ATTN_E_DEVICE: return "current device differs from the plan's device";
    case ATTN_E_NO_DEVICE: return "no usable sm_100 device";
    case ATTN_E_SCRATCH_LIMIT: return "shape needs more scratch than the fixed no-allocation array holds";
    default: return "unknown error code";
    }
}

ATTN_EXPORT int attn_plan_ex(attn_plan_t *out, int B_max, int s_max, int Hq, int Hkv, int D, int max_q,
                             const attn_overrides *o) {
    if (!out) return ATTN_E_NULL;
    *out = nullptr;
    if (B_max < 1 || B_max > 65535 || s_max < 1 || s_max > (1 << 30) || Hq < 1 || Hkv < 1 ||
        Hq % Hkv != 0 || max_q < 1 || max_q > 65536)
        return ATTN_E_INVALID_ARG;
    if (D != 64 && D != 128) return ATTN_E_UNSUPPORTED;
    const long long rows = (long long)(Hq / Hkv) * max_q;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_E_NO_DEVICE;
    int major = 0, sms = 0, smem_sm = 0, smem_block = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&smem_block, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
        return ATTN_E_NO_DEVICE;
    if (major != 10) return ATTN_E_NO_DEVICE;

    attn_plan_desc d{};
    d.B_max = B_max;
    d.s_max = s_max;
    d.Hq = Hq;
    d.Hkv = Hkv;
    d.D = D;
    d.max_q = max_q;
    d.G = Hq / Hkv;
    d.num_sms = sms;

    // warp-MMA kernel up to 16 query rows per KV head (the rows ride on the
    // MMA's n8 side); tcgen05 kernel beyond, 128 rows (the M = 128 side) per
    // unit and longer queries in row tiles of 128 / G tokens; CUDA cores when
    // a single token's G heads exceed 128 rows
    const int G_ = Hq / Hkv;
    int variant = o && o->variant ? o->variant
                                  : (rows <= 16 ? ATTN_VARIANT_MMA
                                                : (G_ <= tc_rows() ? ATTN_VARIANT_TC : ATTN_VARIANT_SIMT));
    if (variant != ATTN_VARIANT_MMA && variant != ATTN_VARIANT_SIMT && variant != ATTN_VARIANT_TC)
        return ATTN_E_INVALID_ARG;
    if (variant == ATTN_VARIANT_MMA && rows > 16) return ATTN_E_UNSUPPORTED;
    if (variant == ATTN_VARIANT_TC && G_ > tc_rows()) return ATTN_E_UNSUPPORTED;
    if (o && o->block_n && o->block_n != 64) return ATTN_E_UNSUPPORTED;
    if (o && (o->nsplit < 0 || o->stages < 0 || o->ctas < 0)) return ATTN_E_INVALID_ARG;
    if (o && o->combine && o->combine != ATTN_COMBINE_KERNEL && o->combine != ATTN_COMBINE_FUSED)
        return ATTN_E_INVALID_ARG;
    if (o && (o->wait_limit_us < 0 || o->test_stall < 0 || o->test_stall > 1)) return ATTN_E_INVALID_ARG;
    if (o && o->test_stall && variant == ATTN_VARIANT_SIMT) return ATTN_E_UNSUPPORTED;
    d.variant = variant;
    const int tiles_max = (s_max + 63) / 64;

    int NT = 1;
    int qtile = max_q, max_rt = 1;
    size_t n_ticket = 0, n_part = 0, part_rows = 0;
    int merge_bytes = 0;
    bool plan_direct = false;
    if (variant == ATTN_VARIANT_MMA || variant == ATTN_VARIANT_TC) {
        // persistent: about one block per SM, each with a deep load ring; the
        // split points follow the balanced per-block shares (nsplit and chunk
        // do not apply) and the slot-parallel combine kernel merges cut units
        const bool tcv = variant == ATTN_VARIANT_TC;
        if (o && (o->nsplit || (!tcv && o->combine == ATTN_COMBINE_FUSED))) return ATTN_E_UNSUPPORTED;
        NT = rows <= 8 ? 1 : 2;
        d.block_n = mma_block_n();
        if (tcv) {
            qtile = std::min(max_q, tc_rows() / (Hq / Hkv));
            max_rt = (max_q + qtile - 1) / qtile;
        }
        const long long max_tiles = (long long)B_max * Hkv * max_rt * tiles_max;
        long long ctas = o && o->ctas ? o->ctas : sms;
        ctas = std::min<long long>(ctas, std::max(1LL, max_tiles));
        // units of at most two tiles (s_max <= 128 keys): cutting one saves a
        // block at most one tile but adds a merge, so each unit gets its own
        // block (measured on the tiny workload: 14.3 against 16.4 us isolated)
        const long long units = (long long)B_max * Hkv * max_rt;
        if (!(o && o->ctas) && tiles_max <= 2) ctas = std::min<long long>(ctas, std::max(1LL, units));
        // ... and on the warp-MMA path, when those units fit one wave, block c
        // simply takes unit c: no unit is ever cut, so no merge is launched
        // and no schedule is computed speculatively (the direct write of the
        // split-KV method, for the smallest calls)
        const bool direct = !tcv && !(o && o->ctas) && tiles_max <= 2 && units <= sms;
        if (direct) ctas = units;
        ctas = std::min<long long>(ctas, 65535);
        d.ctas = (int)ctas;
        auto smem_of = [&](int st) { return tcv ? tc_smem_need(D, st) : mma_smem_bytes(D, NT, st, d.ctas); };
        const size_t stage_bytes = tcv ? tc_stage_bytes(D) : mma_stage_bytes(D);
        int stages = o && o->stages ? o->stages : (int)((smem_block - smem_of(0)) / stage_bytes);
        stages = std::min(stages, 8);
        if (stages < 2 || smem_of(stages) > (size_t)smem_block) return ATTN_E_INVALID_ARG;
        d.stages = stages;
        d.rows_per_block = tcv ? tc_rows() : 8 * NT;
        d.row_tiles = 1;
        d.smem_bytes = (int)(tcv ? tc_smem_bytes(D, stages) : smem_of(stages));
        merge_bytes = tcv ? 0 : (int)mma_merge_bytes(D, NT, d.ctas);
        d.nsplit = 0;
        d.chunk = 0;
        d.grid_x = d.ctas;
        d.grid_y = 1;
        d.grid_z = 1;
        // static shares unless asked otherwise on the tensor-core path (its
        // run-time claims measured slower: short-query batches 56.0 -> 53.8 us,
        // 16-key pages 64.1 -> 52.6 us, prefill equal), run-time claims on the
        // warp-MMA decode path (long-context 28.6 -> 27.5 us, ragged
        // 183 -> 175 us); the override's sign picks either
        const int det_req = o ? o->deterministic : 0;
        d.deterministic = det_req > 0 ? 1 : det_req < 0 ? 0 : (tcv ? 1 : 0);
        // warp-MMA path: slot-parallel combine kernel, programmatic dependent
        // launch.  tcgen05 path: where queries span several row tiles the
        // block holding each cut unit's last part merges it (no second
        // kernel; causal prefill 186 -> 150 us), which needs static shares;
        // with one row tile per sequence the combine kernel (short query:
        // 46.0 against 47.3 us fused -- a fused merge's reads of the other
        // parts, issued while most blocks still stream, wait about 4 us in
        // the loaded memory system, on the merging block's critical path)
        const int want = o && o->combine ? o->combine
                                         : (tcv && d.deterministic && max_rt > 1 ? ATTN_COMBINE_FUSED
                                                                                  : ATTN_COMBINE_KERNEL);
        d.combine = tcv ? want : (direct ? 0 : ATTN_COMBINE_KERNEL);
        if (d.combine == ATTN_COMBINE_FUSED && !d.deterministic) return ATTN_E_UNSUPPORTED;
        d.combine_blocks = d.combine == ATTN_COMBINE_KERNEL ? 2 * d.ctas * combine_slots_split((Hq / Hkv) * qtile, D) : 0;
        plan_direct = direct;
        // per unit: tile claims (64-bit), parts written
        n_ticket = 3 * (size_t)B_max * Hkv * max_rt;
        n_part = 2 * (size_t)d.ctas;       // two partial slots per block
        part_rows = d.rows_per_block;
        if ((tcv ? tc_prepare(D, stages, d.ctas) : mma_prepare(D, NT, stages, d.ctas)) != cudaSuccess)
            return ATTN_E_CUDA;
    } else {
        if (o && o->ctas) return ATTN_E_UNSUPPORTED;
        d.deterministic = 1;                 // fixed grid, fixed merge order
        d.block_n = kSimtBlockN;
        d.stages = 2;
        d.rows_per_block = kSimtRowsPerBlock;
        d.row_tiles = (int)((rows + kSimtRowsPerBlock - 1) / kSimtRowsPerBlock);
        d.smem_bytes = (int)simt_smem_bytes(D);
        if ((long long)Hkv * d.row_tiles > 65535) return ATTN_E_INVALID_ARG;
        if (simt_prepare(D) != cudaSuccess) return ATTN_E_CUDA;
        // resident blocks per SM, from shared memory (the binding limit here)
        const int per_sm = std::min(4, std::max(1, smem_sm / (d.smem_bytes + 1024)));
        // Split count: fill the device (about per_sm blocks per SM), capped by
        // the tile count; fall back to one direct-write pass when the
        // (sequence, KV head, row tile) units alone already fill it (AstrAI
        // commit log, split-KV commit).
        const long long units = (long long)B_max * Hkv * d.row_tiles;
        const long long target = (long long)sms * per_sm;
        long long ns;
        if (o && o->nsplit)
            ns = o->nsplit;
        else if (units >= target)
            ns = 1;
        else
            ns = (target + units - 1) / units;
        ns = std::max(1LL, std::min<long long>(ns, std::min(tiles_max, 1024)));
        const int tiles_per_chunk = (int)((tiles_max + ns - 1) / ns);
        d.chunk = tiles_per_chunk * d.block_n;
        d.nsplit = (s_max + d.chunk - 1) / d.chunk;
        d.grid_x = d.nsplit;
        d.grid_y = Hkv * d.row_tiles;
        d.grid_z = B_max;
        // partials merged by the last block of each unit (one launch per call)
        // when its shared memory holds the merge tables, else by a second kernel
        if (d.nsplit > 1) {
            const size_t need = (size_t)d.rows_per_block * (d.nsplit + 1) * 8;
            const int want = o && o->combine ? o->combine : ATTN_COMBINE_FUSED;
            d.combine = (want == ATTN_COMBINE_FUSED && need <= simt_merge_capacity(D)) ? ATTN_COMBINE_FUSED
                                                                                      : ATTN_COMBINE_KERNEL;
            n_part = (size_t)B_max * max_q * Hq * d.nsplit;
            part_rows = 1;
            if (d.combine == ATTN_COMBINE_FUSED) n_ticket = (size_t)B_max * Hkv * d.row_tiles;
        }
    }

    // scratch: error word, merge tickets, O partials, (m, l) partials
    const size_t off_t = 256;
    const size_t off_o = align_up(off_t + n_ticket * sizeof(uint32_t), 256);
    const size_t off_ml = align_up(off_o + n_part * part_rows * D * sizeof(float), 256);
    const size_t total = align_up(off_ml + n_part * part_rows * sizeof(float2), 256);
    d.scratch_bytes = total;

    attn_plan_s *p = new (std::nothrow) attn_plan_s{};
    if (!p) return ATTN_E_NOMEM;
    p->d = d;
    p->device = dev;
    p->NT = NT;
    p->merge_bytes = merge_bytes;
    p->qtile = qtile;
    p->max_rt = max_rt;
    p->direct = plan_direct ? 1 : 0;
    p->scale_log2 = (float)((1.0 / std::sqrt((double)D)) * 1.4426950408889634);
    p->wait_ns = o && o->wait_limit_us > 0 ? (unsigned long long)o->wait_limit_us * 1000ull : kDefaultWaitNs;
    if (cudaMalloc(&p->scratch, total) != cudaSuccess) {
        cudaGetLastError();
        delete p;
        return ATTN_E_NOMEM;
    }
    p->err = static_cast<uint32_t *>(p->scratch);
    p->ticket = n_ticket ? reinterpret_cast<uint32_t *>(static_cast<char *>(p->scratch) + off_t) : nullptr;
    p->ticket_bytes = n_ticket * sizeof(uint32_t);
    p->o_part = n_part ? reinterpret_cast<float *>(static_cast<char *>(p->scratch) + off_o) : nullptr;
    p->ml_part = n_part ? reinterpret_cast<float2 *>(static_cast<char *>(p->scratch) + off_ml) : nullptr;
    // error word, then the test hook's stall count (parts that never arrive,
    // cleared by attn_check_error), then the merge counters
    const uint32_t stall = o ? (uint32_t)o->test_stall : 0u;
    if (cudaMemset(p->scratch, 0, off_o) != cudaSuccess ||
        cudaMemcpy(p->err + 1, &stall, sizeof(stall), cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaDeviceSynchronize() != cudaSuccess) {
        cudaFree(p->scratch);
        delete p;
        return ATTN_E_CUDA;
    }
    {
        std::lock_guard<std::mutex> lk(g_mu);
        g_plans.insert(p);
    }
    if (variant == ATTN_VARIANT_MMA || variant == ATTN_VARIANT_TC) {
        int rc = get_encoder();
        if (rc != ATTN_OK) {
            attn_destroy(p);
            return rc;
        }
    }
    if (d.combine == ATTN_COMBINE_KERNEL && variant == ATTN_VARIANT_SIMT) {
        Params tmp{};
        tmp.B_max = B_max;
        tmp.max_q = max_q;
        tmp.Hq = Hq;
        p->d.combine_blocks = combine_blocks(tmp);
    }
    if (std::getenv("VGQA_LOG"))
        std::fprintf(stderr,
                     "[vgqa] plan B_max=%d s_max=%d Hq=%d Hkv=%d D=%d max_q=%d: variant=%d nsplit=%d chunk=%d "
                     "ctas=%d grid=(%d,%d,%d) smem=%d stages=%d combine=%d scratch=%zu\n",
                     B_max, s_max, Hq, Hkv, D, max_q, p->d.variant, p->d.nsplit, p->d.chunk, p->d.ctas,
                     p->d.grid_x, p->d.grid_y, p->d.grid_z, p->d.smem_bytes, p->d.stages, p->d.combine,
                     p->d.scratch_bytes);
    *out = p;
    return ATTN_OK;
}

ATTN_EXPORT int attn_plan(attn_plan_t *out, int B_max, int s_max, int Hq, int Hkv, int D, int max_q) {
    return attn_plan_ex(out, B_max, s_max, Hq, Hkv, D, max_q, nullptr);
}

ATTN_EXPORT int attn_plan_info(attn_plan_t plan, attn_plan_desc *desc) {
    if (!desc) return ATTN_E_NULL;
    if (!plan || !live(plan)) return ATTN_E_BAD_PLAN;
    *desc = plan->d;
    return ATTN_OK;
}

namespace {

// where the keys live when the cache is paged (attn_run_paged)
struct Paging {
    const int32_t *block_table;
    int bt_stride, page_size, num_pages;
    long long page_stride;
};

int log2_exact(long long x) {
    int s = 0;
    while ((1ll << s) < x) ++s;
    return (1ll << s) == x ? s : -1;
}

int run_impl(attn_plan_t plan, const void *q, const void *k, const void *v, const int32_t *cu_q,
             const int32_t *cu_k, void *out, float *lse, long long k_stride, long long v_stride,
             const Paging *pg, void *stream) {
    if (!plan || !live(plan)) return ATTN_E_BAD_PLAN;
    if (!q || !k || !v || !cu_q || !cu_k || !out || !lse) return ATTN_E_NULL;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(lse, 4) ||
        !aligned(cu_q, 4) || !aligned(cu_k, 4))
        return ATTN_E_ALIGNMENT;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_E_CUDA;
    if (dev != plan->device) return ATTN_E_DEVICE;

    const attn_plan_desc &d = plan->d;
    Params p{};
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.k = static_cast<const __nv_bfloat16 *>(k);
    p.v = static_cast<const __nv_bfloat16 *>(v);
    p.cu_q = cu_q;
    p.cu_k = cu_k;
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.lse = lse;
    p.o_part = plan->o_part;
    p.ml_part = plan->ml_part;
    p.err = plan->err;
    p.stall = plan->err + 1;
    p.wait_ns = plan->wait_ns;
    p.B_max = d.B_max;
    p.s_max = d.s_max;
    p.Hq = d.Hq;
    p.Hkv = d.Hkv;
    p.D = d.D;
    p.max_q = d.max_q;
    p.G = d.G;
    p.nsplit = d.nsplit;
    p.chunk = d.chunk;
    p.rows_per_block = d.rows_per_block;
    p.row_tiles = d.row_tiles;
    p.scale_log2 = plan->scale_log2;
    p.k_stride = k_stride;
    p.v_stride = v_stride;
    if (pg) {
        p.block_table = pg->block_table;
        p.bt_stride = pg->bt_stride;
        p.page_shift = log2_exact(pg->page_size);
        p.num_pages = pg->num_pages;
        p.page_box = std::min(pg->page_size, 64);
        p.page_stride = pg->page_stride;
        // pages a whole number of token rows apart: one row index per key,
        // page * page_rows + slot, into a 3-D map of all the cache's rows
        if (pg->page_stride % k_stride == 0 && (long long)pg->num_pages * (pg->page_stride / k_stride) < (1ll << 31))
            p.page_rows = (int)(pg->page_stride / k_stride);
    }
    p.ticket = plan->ticket;
    p.claim = reinterpret_cast<unsigned long long *>(plan->ticket);
    p.done = plan->ticket + 2 * (size_t)d.B_max * d.Hkv * plan->max_rt;
    p.fused = d.combine == ATTN_COMBINE_FUSED;
    p.merge_bytes = plan->merge_bytes;
    p.ctas_max = d.ctas;
    p.share_stride = share_stride(d.ctas);
    const bool persistent = d.variant == ATTN_VARIANT_MMA || d.variant == ATTN_VARIANT_TC;
    p.dynamic = persistent && !d.deterministic;
    p.head_first = d.variant == ATTN_VARIANT_TC && p.fused;
    p.done_per_part = d.variant == ATTN_VARIANT_TC ? tc_parts_per_block() : 1;
    p.unit_cost = d.variant == ATTN_VARIANT_TC ? tc_unit_cost() : 0;
    p.qtile = plan->qtile;
    p.max_rt = plan->max_rt;
    p.direct = plan->direct;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const dim3 grid(d.grid_x, d.grid_y, d.grid_z);
    // K and V tensor maps of the TMA-fed kernels
    auto kv_maps = [&](CUtensorMap &tm_k, CUtensorMap &tm_v) -> bool {
        if (pg && p.page_rows) {
            const long long rows = (long long)pg->num_pages * p.page_rows;
            const int box = std::min(pg->page_size, 64);
            return encode_kv_map(&tm_k, k, d.Hkv, d.D, box, k_stride, rows) == ATTN_OK &&
                   encode_kv_map(&tm_v, v, d.Hkv, d.D, box, v_stride, rows) == ATTN_OK;
        }
        if (pg)
            return encode_paged_map(&tm_k, k, d.Hkv, d.D, pg->page_size, pg->num_pages, k_stride,
                                    pg->page_stride) == ATTN_OK &&
                   encode_paged_map(&tm_v, v, d.Hkv, d.D, pg->page_size, pg->num_pages, v_stride,
                                    pg->page_stride) == ATTN_OK;
        return encode_kv_map(&tm_k, k, d.Hkv, d.D, d.block_n, k_stride) == ATTN_OK &&
               encode_kv_map(&tm_v, v, d.Hkv, d.D, d.block_n, v_stride) == ATTN_OK;
    };
    cudaError_t e;
    if (d.variant == ATTN_VARIANT_MMA) {
        CUtensorMap tm_k, tm_v;
        bool ok;
        if (pg && !p.page_rows)
            ok = encode_paged_map_halves(&tm_k, k, d.Hkv, d.D, pg->page_size, pg->num_pages, k_stride,
                                         pg->page_stride) == ATTN_OK &&
                 encode_paged_map_halves(&tm_v, v, d.Hkv, d.D, pg->page_size, pg->num_pages, v_stride,
                                         pg->page_stride) == ATTN_OK;
        else {
            const long long rows = pg ? (long long)pg->num_pages * p.page_rows : 0x7fffffffll;
            const int box = pg ? std::min(pg->page_size, 64) : d.block_n;
            ok = encode_kv_map_halves(&tm_k, k, d.Hkv, d.D, box, k_stride, rows) == ATTN_OK &&
                 encode_kv_map_halves(&tm_v, v, d.Hkv, d.D, box, v_stride, rows) == ATTN_OK;
        }
        if (!ok) return ATTN_E_CUDA;
        e = launch_split_mma(p, tm_k, tm_v, plan->NT, d.stages, d.ctas, s);
    } else if (d.variant == ATTN_VARIANT_TC) {
        CUtensorMap tm_q, tm_k, tm_v;
        if (encode_q_map(&tm_q, q, d.Hq, d.D, d.G, plan->qtile) != ATTN_OK || !kv_maps(tm_k, tm_v))
            return ATTN_E_CUDA;
        e = launch_split_tc(p, tm_q, tm_k, tm_v, d.stages, d.ctas, s);
    } else {
        e = launch_split_simt(p, grid, s);
    }
    if (e != cudaSuccess) return ATTN_E_CUDA;
    if (d.combine == ATTN_COMBINE_KERNEL && d.variant == ATTN_VARIANT_SIMT) {
        e = launch_combine(p, s);
        if (e != cudaSuccess) return ATTN_E_CUDA;
    }
    return ATTN_OK;
}

}  // namespace

ATTN_EXPORT int attn_run(attn_plan_t plan, const void *q, const void *k, const void *v, const int32_t *cu_q,
                         const int32_t *cu_k, void *out, float *lse, void *stream) {
    if (!plan || !live(plan)) return ATTN_E_BAD_PLAN;
    const long long packed = (long long)plan->d.Hkv * plan->d.D;
    return run_impl(plan, q, k, v, cu_q, cu_k, out, lse, packed, packed, nullptr, stream);
}

ATTN_EXPORT int attn_run_strided(attn_plan_t plan, const void *q, const void *k, const void *v,
                                 const int32_t *cu_q, const int32_t *cu_k, void *out, float *lse,
                                 int64_t k_token_stride, int64_t v_token_stride, void *stream) {
    if (!plan || !live(plan)) return ATTN_E_BAD_PLAN;
    const long long packed = (long long)plan->d.Hkv * plan->d.D;
    // a token's heads stay contiguous; the token stride keeps 16-byte
    // alignment (the tensor-map rule) and fits the tensor map's range
    for (long long st : {(long long)k_token_stride, (long long)v_token_stride})
        if (st < packed || st % 8 != 0 || st > (1ll << 38)) return ATTN_E_INVALID_ARG;
    return run_impl(plan, q, k, v, cu_q, cu_k, out, lse, k_token_stride, v_token_stride, nullptr, stream);
}

ATTN_EXPORT int attn_run_paged(attn_plan_t plan, const void *q, const void *k_cache, const void *v_cache,
                               int64_t page_stride, int64_t token_stride, int page_size, int num_pages,
                               const int32_t *block_table, int bt_stride, const int32_t *cu_q,
                               const int32_t *cu_k, void *out, float *lse, void *stream) {
    if (!plan || !live(plan)) return ATTN_E_BAD_PLAN;
    if (!block_table) return ATTN_E_NULL;
    if (!aligned(block_table, 4)) return ATTN_E_ALIGNMENT;
    const attn_plan_desc &d = plan->d;
    const long long packed = (long long)d.Hkv * d.D;
    // power-of-two pages of at least 8 tokens: a tile of 64 keys then covers
    // whole pages or lies inside one, and each TMA box starts on a 1 KB
    // boundary of the 128-byte swizzle pattern
    const int shift = log2_exact(page_size);
    if (page_size < 8 || page_size > (1 << 20) || shift < 0 || num_pages < 1 ||
        (long long)num_pages * page_size >= (1ll << 31))
        return ATTN_E_INVALID_ARG;
    if (token_stride < packed || token_stride % 8 != 0 || token_stride > (1ll << 38) || page_stride % 8 != 0 ||
        page_stride < (long long)page_size * token_stride || page_stride > (1ll << 38))
        return ATTN_E_INVALID_ARG;
    if (bt_stride < (d.s_max + page_size - 1) / page_size) return ATTN_E_INVALID_ARG;
    const Paging pg{block_table, bt_stride, page_size, num_pages, page_stride};
    return run_impl(plan, q, k_cache, v_cache, cu_q, cu_k, out, lse, token_stride, token_stride, &pg, stream);
}

ATTN_EXPORT int attn_check_error(attn_plan_t plan, void *stream, uint32_t *flags) {
    if (!flags) return ATTN_E_NULL;
    *flags = 0;
    if (!plan || !live(plan)) return ATTN_E_BAD_PLAN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t h = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess) return ATTN_E_CUDA;
    if (cudaMemcpy(&h, plan->err, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return ATTN_E_CUDA;
    // the error word and the test hook's stall count
    if (cudaMemset(plan->err, 0, 2 * sizeof(uint32_t)) != cudaSuccess) return ATTN_E_CUDA;
    // a call that stopped early may have left merge tickets part-counted
    if (h && plan->ticket_bytes && cudaMemset(plan->ticket, 0, plan->ticket_bytes) != cudaSuccess)
        return ATTN_E_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return ATTN_E_CUDA;
    *flags = h;
    return ATTN_OK;
}

ATTN_EXPORT void attn_destroy(attn_plan_t plan) {
    if (!plan) return;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!g_plans.erase(plan)) return;
    }
    int prev = -1;
    cudaGetDevice(&prev);
    if (prev != plan->device) cudaSetDevice(plan->device);
    cudaFree(plan->scratch);
    if (prev >= 0 && prev != plan->device) cudaSetDevice(prev);
    delete plan;
}
