// noalloc.cu -- attn_run_noalloc: one attention call that allocates nothing.
//
// Some callers cannot call cudaMalloc.  A host framework that owns the whole
// device memory budget through its own pool allocator must not have a library
// grab memory behind the pool's back (the raw allocation escapes the pool's
// accounting and can fail once the pool has reserved the device), and a
// latency-critical path cannot afford cudaMalloc/cudaFree, which may
// synchronise the device.  Such callers cannot create a plan, because
// attn_plan allocates the plan's scratch.
//
// This entry point takes the shape with every call, makes the same kind of
// choices the planner makes, and runs the CUDA-core split kernel with its
// scratch (split partials, merge tickets, error word) taken from one
// file-scope device array of kNoallocScratchBytes.  That array is part of the
// library image: every GPU that loads the library holds it until the process
// exits.  A call that would need more scratch than the array holds is
// rejected with ATTN_E_SCRATCH_LIMIT before anything is launched.
//
// The array's name in host code is only a host-side stand-in for the device
// symbol, so the host never passes it to a kernel: the first call on each
// device looks up the device address with cudaGetSymbolAddress (with that
// device current) and caches it.  That first call also sets the kernel's
// shared-memory attribute, so make it before any stream capture begins.  Under
// lazy module loading (CUDA's default since 12.2) the array's memory is
// committed on that first call, so a caller whose pool reserves the device
// should make it before the pool does.
//
// Every call on a device shares the one array and leaves its contents
// behind; each call clears the error word and the merge tickets (the parts
// that must start at zero) on its stream before launching.  Calls that
// overlap on the GPU (for example on two streams without ordering between
// them) race on the array: order them on one stream or with events.
#include <cmath>
#include <mutex>

#include "../../include/varlen_gqa.h"
#include "kernels.h"
#include "params.h"

#define ATTN_EXPORT extern "C" __attribute__((visibility("default")))

namespace vgqa {
namespace {

constexpr size_t kNoallocScratchBytes = ATTN_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

struct DeviceSetup {
    bool ready = false;
    unsigned char *scratch = nullptr;   // device address of g_noalloc_scratch
    int sms = 0;
    int smem_per_sm = 0;
    bool prepared[2] = {false, false};  // kernel attribute set for D = 64 / 128
};

std::mutex g_setup_mu;
DeviceSetup g_setup[kMaxDevices];

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Once per device, with that device current: resolve the scratch array's
// device address and read the SM count.  Returns ATTN_OK or an error code.
int setup_device(int dev, int D, DeviceSetup &out) {
    std::lock_guard<std::mutex> lk(g_setup_mu);
    DeviceSetup &s = g_setup[dev];
    if (!s.ready) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) {
            cudaGetLastError();
            return ATTN_E_CUDA;
        }
        int major = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&s.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&s.smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) !=
                cudaSuccess)
            return ATTN_E_NO_DEVICE;
        if (major != 10) return ATTN_E_NO_DEVICE;
        s.scratch = static_cast<unsigned char *>(ptr);
        s.ready = true;
    }
    const int di = D == 64 ? 0 : 1;
    if (!s.prepared[di]) {
        if (simt_prepare(D) != cudaSuccess) return ATTN_E_CUDA;
        s.prepared[di] = true;
    }
    out = s;
    return ATTN_OK;
}

bool is_aligned(const void *ptr, size_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

}  // namespace
}  // namespace vgqa

using namespace vgqa;

ATTN_EXPORT int attn_run_noalloc(int B_max, int s_max, int Hq, int Hkv, int D, int max_q, const void *q,
                                 const void *k, const void *v, const int32_t *cu_q, const int32_t *cu_k,
                                 void *out, float *lse, void *stream) {
    if (B_max < 1 || B_max > 65535 || s_max < 1 || s_max > (1 << 30) || Hq < 1 || Hkv < 1 ||
        Hq % Hkv != 0 || max_q < 1 || max_q > 65536)
        return ATTN_E_INVALID_ARG;
    if (D != 64 && D != 128) return ATTN_E_UNSUPPORTED;
    if (!q || !k || !v || !cu_q || !cu_k || !out || !lse) return ATTN_E_NULL;
    if (!is_aligned(q, 16) || !is_aligned(k, 16) || !is_aligned(v, 16) || !is_aligned(out, 16) ||
        !is_aligned(lse, 4) || !is_aligned(cu_q, 4) || !is_aligned(cu_k, 4))
        return ATTN_E_ALIGNMENT;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_E_NO_DEVICE;
    if (dev < 0 || dev >= kMaxDevices) return ATTN_E_DEVICE;
    DeviceSetup s;
    int rc = setup_device(dev, D, s);
    if (rc != ATTN_OK) return rc;

    // split count: fill the device with about as many blocks as fit at once,
    // one direct-write pass when the units alone already do
    const long long G = Hq / Hkv;
    const long long rows = G * max_q;
    const int row_tiles = (int)((rows + kSimtRowsPerBlock - 1) / kSimtRowsPerBlock);
    if ((long long)Hkv * row_tiles > 65535) return ATTN_E_INVALID_ARG;
    const int smem = (int)simt_smem_bytes(D);
    int per_sm = s.smem_per_sm / (smem + 1024);
    per_sm = per_sm < 1 ? 1 : (per_sm > 4 ? 4 : per_sm);
    const long long units = (long long)B_max * Hkv * row_tiles;
    const long long target = (long long)s.sms * per_sm;
    const int tiles_max = (s_max + kSimtBlockN - 1) / kSimtBlockN;
    long long ns = units >= target ? 1 : (target + units - 1) / units;
    if (ns > tiles_max) ns = tiles_max;
    if (ns > 1024) ns = 1024;
    // the fused merge keeps one (weight, l) pair per split and row in shared memory
    while (ns > 1 && (size_t)kSimtRowsPerBlock * (ns + 1) * 8 > simt_merge_capacity(D)) --ns;
    const int chunk = (int)((tiles_max + ns - 1) / ns) * kSimtBlockN;
    const int nsplit = (s_max + chunk - 1) / chunk;

    // scratch layout: error word | merge tickets | O partials | (m, l) partials
    const size_t n_part = nsplit > 1 ? (size_t)B_max * max_q * Hq * nsplit : 0;
    const size_t n_ticket = nsplit > 1 ? (size_t)units : 0;
    const size_t off_t = 256;
    const size_t off_o = round_up(off_t + n_ticket * sizeof(uint32_t), 256);
    const size_t off_ml = round_up(off_o + n_part * D * sizeof(float), 256);
    const size_t total = round_up(off_ml + n_part * sizeof(float2), 256);
    if (total > kNoallocScratchBytes) return ATTN_E_SCRATCH_LIMIT;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the error word and the tickets must start at zero for this call
    if (cudaMemsetAsync(s.scratch, 0, off_o, st) != cudaSuccess) return ATTN_E_CUDA;

    Params p{};
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.k = static_cast<const __nv_bfloat16 *>(k);
    p.v = static_cast<const __nv_bfloat16 *>(v);
    p.cu_q = cu_q;
    p.cu_k = cu_k;
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.lse = lse;
    p.err = reinterpret_cast<uint32_t *>(s.scratch);
    p.wait_ns = kDefaultWaitNs;
    p.ticket = n_ticket ? reinterpret_cast<uint32_t *>(s.scratch + off_t) : nullptr;
    p.o_part = n_part ? reinterpret_cast<float *>(s.scratch + off_o) : nullptr;
    p.ml_part = n_part ? reinterpret_cast<float2 *>(s.scratch + off_ml) : nullptr;
    p.B_max = B_max;
    p.s_max = s_max;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.D = D;
    p.max_q = max_q;
    p.G = (int)G;
    p.nsplit = nsplit;
    p.chunk = chunk;
    p.rows_per_block = kSimtRowsPerBlock;
    p.row_tiles = row_tiles;
    p.scale_log2 = (float)((1.0 / std::sqrt((double)D)) * 1.4426950408889634);
    p.k_stride = p.v_stride = (long long)Hkv * D;
    p.fused = nsplit > 1;
    const dim3 grid(nsplit, Hkv * row_tiles, B_max);
    if (launch_split_simt(p, grid, st) != cudaSuccess) return ATTN_E_CUDA;
    return ATTN_OK;
}
