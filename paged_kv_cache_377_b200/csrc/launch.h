// launch.h -- host-side entry points of the kernels (internal to libpagedkv.so).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "decode_common.cuh"

namespace pkv {

// kMathFp8: tensor-core (f16 mma.sync) math over e4m3 pools with per-head
// scales; chosen by the fp8 entry points, not by the math option.
// kMathTensorCoreGroups: kMathTensorCore plus the prefix units of prefix
// groups; chosen for a launch that has groups (a kernel of its own, so that
// launches without groups keep the leaner register allocation).
enum DecodeMath { kMathCudaCore = 1, kMathTensorCore = 2, kMathFp8 = 3, kMathTensorCoreGroups = 4 };

// True when the (head_dim, block_size, padded group, math) combination is compiled in.
bool decode_variant_exists(int head_dim, int block_size, int group_pad, int math);

// Shared-memory bytes per CTA of a decode variant (num_stages = stages per consumer warp).
size_t decode_smem_bytes(int head_dim, int block_size, int group_pad, int group, int math, int num_stages,
                         int num_seqs, int pack);

// Sets the variant's dynamic shared-memory limit (once per device) and returns
// how many CTAs of it fit on one SM.
cudaError_t decode_prepare(int head_dim, int block_size, int group_pad, int math, size_t smem_bytes,
                           int *ctas_per_sm);

cudaError_t decode_launch(int head_dim, int block_size, int group_pad, int math, const CUtensorMap &tm_k,
                          const CUtensorMap &tm_v, const DecodeArgs &args, int grid, size_t smem_bytes,
                          cudaStream_t stream);


cudaError_t append_launch(const void *k, const void *v, void *k_cache, void *v_cache, const int64_t *slot_mapping,
                          int num_tokens, int num_kv_heads, int head_dim, int block_size, int num_blocks,
                          int32_t *status, cudaStream_t stream);

// Multi-query paged attention (prefill.cu).
struct PrefillArgs {
    void *out;                    // bf16 [T][Hq][D]
    const void *q;                // bf16 [T][Hq][D]
    const int32_t *block_tables;  // [S][MB]
    const int32_t *context_lens;  // [S]
    const int32_t *query_start;   // [S + 1]
    int32_t *status;
    int num_seqs, num_tokens, num_q_heads, num_kv_heads, group, max_blocks_per_seq, num_blocks, max_query_len;
    float scale_log2;
};

size_t prefill_smem_bytes(int head_dim, int block_size, int max_blocks_per_seq);
cudaError_t prefill_launch(int head_dim, int block_size, const CUtensorMap &tm_k, const CUtensorMap &tm_v,
                           const PrefillArgs &args, int tiles, size_t smem_bytes, cudaStream_t stream);
int prefill_rows_per_cta();

size_t prefill_tc_smem_bytes(int head_dim, int max_blocks_per_seq);
cudaError_t prefill_tc_launch(int head_dim, int block_size, const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                              const CUtensorMap &tm_v, const PrefillArgs &args, int tiles, size_t smem_bytes,
                              cudaStream_t stream);
int prefill_tc_rows_per_cta();

cudaError_t append_fp8_launch(const void *k, const void *v, void *k_cache, void *v_cache, const int64_t *slot_mapping,
                              const float *k_scale, const float *v_scale, int num_tokens, int num_kv_heads,
                              int head_dim, int block_size, int num_blocks, int32_t *status, cudaStream_t stream);

cudaError_t block_copy_launch(void *k_cache, void *v_cache, const int32_t *src, const int32_t *dst,
                              int num_copies, int block_size, int num_kv_heads, int row_bytes, int num_blocks,
                              int32_t *status, cudaStream_t stream);

cudaError_t validate_launch(const int32_t *block_tables, const int32_t *context_lens, int num_seqs,
                            int max_blocks_per_seq, int block_size, int num_blocks, int32_t *status,
                            cudaStream_t stream);

// Launches a kernel whose bounded wait must give up (see selftest.cu).
cudaError_t selftest_bounded_wait_launch(int32_t *status, cudaStream_t stream);

}  // namespace pkv
