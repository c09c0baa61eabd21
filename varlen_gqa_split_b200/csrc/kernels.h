// kernels.h -- host-side launchers of libvgqa's kernels (internal).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>

namespace vgqa {

struct Params;

// CUDA-core split kernel (any row count), 16 query rows per block
size_t simt_smem_bytes(int D);
size_t simt_merge_capacity(int D);
cudaError_t simt_prepare(int D);
cudaError_t launch_split_simt(const Params &p, dim3 grid, cudaStream_t stream);
constexpr int kSimtRowsPerBlock = 16;
constexpr int kSimtBlockN = 64;

// Persistent TMA-fed tensor-core split kernel, NT = ceil(G * max_q / 8) in
// {1, 2}, `ctas` blocks sharing the flattened tile space
size_t mma_stage_bytes(int D);
size_t mma_merge_bytes(int D, int NT, int ctas);
size_t mma_smem_bytes(int D, int NT, int stages, int ctas);
int mma_block_n();
int mma_threads();
cudaError_t mma_prepare(int D, int NT, int stages, int ctas);
cudaError_t launch_split_mma(const Params &p, const CUtensorMap &tm_k, const CUtensorMap &tm_v, int NT,
                             int stages, int ctas, cudaStream_t stream);

// Persistent TMA-fed tcgen05 split kernel (accumulators in tensor memory),
// up to tc_rows() query rows per KV head
size_t tc_stage_bytes(int D);
size_t tc_smem_need(int D, int stages);    // bytes the layout uses
size_t tc_smem_bytes(int D, int stages);   // bytes requested at launch (>= half an SM)
int tc_rows();
int tc_parts_per_block();
int tc_unit_cost();                        // fixed cost of a unit, in tiles, for the shares
cudaError_t tc_prepare(int D, int stages, int ctas);
cudaError_t launch_split_tc(const Params &p, const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                            const CUtensorMap &tm_v, int stages, int ctas, cudaStream_t stream);

// log-sum-exp merge of the persistent kernels' partial slots (2 * ctas
// blocks, launched as a programmatic dependent of the split kernel)
size_t combine_slots_smem(int ctas);
int combine_slots_split(int rows, int D);   // blocks per partial slot (S)
cudaError_t combine_slots_prepare(int D, int ctas);
cudaError_t launch_combine_slots(const Params &p, int ctas, cudaStream_t stream);

// log-sum-exp merge of the CUDA-core kernel's dense [.., nsplit] partials
int combine_blocks(const Params &p);
cudaError_t launch_combine(const Params &p, cudaStream_t stream);

}  // namespace vgqa
