// append.cu -- slot-mapped KV-cache append and the device table check.
//
// The append writes each decode step's new key and value into its slot of the
// paged pool (runbyai.xyz post 449, sections 1-2: every step computes and
// caches the new token's key and value; "Deep Dive into vLLM", section 2.1:
// the slot lies in a physical block reached through the block table). Token i
// goes to physical block slot / block_size, offset slot % block_size; a
// negative slot is padding and writes nothing.
#include "device_utils.cuh"
#include "launch.h"

namespace pkv {
namespace {

// One thread per 16 bytes of one (token, kv head) row, for K and V: a warp
// copies two whole 256-byte rows of head_dim 128 (or four of 64), so both the
// loads and the stores are full 32-byte sectors.
__global__ void __launch_bounds__(256)
    kv_append_kernel(const uint4 *__restrict__ k, const uint4 *__restrict__ v, uint4 *__restrict__ k_cache,
                     uint4 *__restrict__ v_cache, const int64_t *__restrict__ slot_mapping, int num_tokens,
                     int num_kv_heads, int chunks_per_row, int block_size, int num_blocks, int32_t *status) {
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t rows = static_cast<int64_t>(num_tokens) * num_kv_heads;
    if (idx >= rows * chunks_per_row) return;
    const int64_t row = idx / chunks_per_row;  // token * num_kv_heads + head
    const int c = static_cast<int>(idx - row * chunks_per_row);
    const int64_t i = row / num_kv_heads;
    const int h = static_cast<int>(row - i * num_kv_heads);
    const int64_t slot = __ldg(slot_mapping + i);
    if (slot < 0) return;
    if (slot >= static_cast<int64_t>(num_blocks) * block_size) {
        if (status && h == 0 && c == 0) atomicOr(status, PKV_STATUS_BAD_SLOT);
        return;
    }
    const int64_t p = slot / block_size;
    const int64_t off = slot - p * block_size;
    const int64_t dst = ((p * block_size + off) * num_kv_heads + h) * chunks_per_row + c;
    const int64_t src = row * chunks_per_row + c;
    k_cache[dst] = __ldg(k + src);
    v_cache[dst] = __ldg(v + src);
}

// The append into e4m3 pools: one thread per 16 codes of one (token, kv head)
// row, K and V; each code is e4m3(rn, satfinite)(x / scale[h]) of its bf16
// source x, the division in fp32.
__global__ void __launch_bounds__(256)
    kv_append_fp8_kernel(const uint4 *__restrict__ k, const uint4 *__restrict__ v, uint4 *__restrict__ k_cache,
                         uint4 *__restrict__ v_cache, const int64_t *__restrict__ slot_mapping,
                         const float *__restrict__ k_scale, const float *__restrict__ v_scale, int num_tokens,
                         int num_kv_heads, int chunks_per_row, int block_size, int num_blocks, int32_t *status) {
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t rows = static_cast<int64_t>(num_tokens) * num_kv_heads;
    if (idx >= rows * chunks_per_row) return;
    const int64_t row = idx / chunks_per_row;  // token * num_kv_heads + head
    const int c = static_cast<int>(idx - row * chunks_per_row);
    const int64_t i = row / num_kv_heads;
    const int h = static_cast<int>(row - i * num_kv_heads);
    const int64_t slot = __ldg(slot_mapping + i);
    if (slot < 0) return;
    if (slot >= static_cast<int64_t>(num_blocks) * block_size) {
        if (status && h == 0 && c == 0) atomicOr(status, PKV_STATUS_BAD_SLOT);
        return;
    }
    const int64_t dst = (slot * num_kv_heads + h) * chunks_per_row + c;  // 16 codes per chunk
    const int64_t src = (row * chunks_per_row + c) * 2;                  // 16 bf16 = two uint4
    k_cache[dst] = quantize16_e4m3(__ldg(k + src), __ldg(k + src + 1), __ldg(k_scale + h));
    v_cache[dst] = quantize16_e4m3(__ldg(v + src), __ldg(v + src + 1), __ldg(v_scale + h));
}

// One thread per (sequence, logical block) entry the sequence needs.
__global__ void __launch_bounds__(256)
    validate_kernel(const int32_t *__restrict__ block_tables, const int32_t *__restrict__ context_lens, int num_seqs,
                    int max_blocks_per_seq, int block_size, int num_blocks, int32_t *status) {
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= static_cast<int64_t>(num_seqs) * max_blocks_per_seq) return;
    const int s = static_cast<int>(idx / max_blocks_per_seq);
    const int b = static_cast<int>(idx - static_cast<int64_t>(s) * max_blocks_per_seq);
    const int64_t cap = static_cast<int64_t>(max_blocks_per_seq) * block_size;
    int L = __ldg(context_lens + s);
    if (L < 0 || L > cap) {
        if (b == 0) atomicOr(status, PKV_STATUS_BAD_CONTEXT_LEN);
        L = L < 0 ? 0 : static_cast<int>(cap);
    }
    if (static_cast<int64_t>(b) * block_size >= L) return;
    const int p = __ldg(block_tables + idx);
    if (p < 0 || p >= num_blocks) atomicOr(status, PKV_STATUS_BAD_BLOCK_ID);
}

// Copy-on-write block copies: whole blocks (bs rows of Hkv * D bf16, K and V)
// from src[c] to dst[c]; one grid-stride pass over 16-byte elements. A copy
// with an id outside [0, num_blocks) is skipped and flagged.
__global__ void block_copy_kernel(uint4 *__restrict__ k_cache, uint4 *__restrict__ v_cache,
                                  const int32_t *__restrict__ src, const int32_t *__restrict__ dst, int num_copies,
                                  int64_t per_block, int num_blocks, int32_t *status) {
    const int64_t total = static_cast<int64_t>(num_copies) * 2 * per_block;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
        const int64_t c = i / (2 * per_block), r = i % (2 * per_block);
        const int kv = static_cast<int>(r / per_block);
        const int64_t e = r % per_block;
        const int32_t s = __ldg(src + c), d = __ldg(dst + c);
        if (s < 0 || s >= num_blocks || d < 0 || d >= num_blocks) {
            if (e == 0 && kv == 0 && status) atomicOr(status, PKV_STATUS_BAD_BLOCK_ID);
            continue;
        }
        uint4 *pool = kv ? v_cache : k_cache;
        pool[d * per_block + e] = pool[s * per_block + e];
    }
}

}  // namespace

cudaError_t block_copy_launch(void *k_cache, void *v_cache, const int32_t *src, const int32_t *dst,
                              int num_copies, int block_size, int num_kv_heads, int row_bytes, int num_blocks,
                              int32_t *status, cudaStream_t stream) {
    const int64_t per_block = static_cast<int64_t>(block_size) * num_kv_heads * row_bytes / 16;  // 16-byte elements
    const int64_t total = static_cast<int64_t>(num_copies) * 2 * per_block;
    if (total == 0) return cudaSuccess;
    int64_t grid = (total + 255) / 256;
    if (grid > 148 * 16) grid = 148 * 16;
    block_copy_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(
        static_cast<uint4 *>(k_cache), static_cast<uint4 *>(v_cache), src, dst, num_copies, per_block, num_blocks,
        status);
    return cudaGetLastError();
}

cudaError_t append_fp8_launch(const void *k, const void *v, void *k_cache, void *v_cache, const int64_t *slot_mapping,
                              const float *k_scale, const float *v_scale, int num_tokens, int num_kv_heads,
                              int head_dim, int block_size, int num_blocks, int32_t *status, cudaStream_t stream) {
    const int chunks = head_dim / 16;
    const int64_t total = static_cast<int64_t>(num_tokens) * num_kv_heads * chunks;
    if (total == 0) return cudaSuccess;
    const int64_t grid = (total + 255) / 256;
    if (grid > 0x7fffffff) return cudaErrorInvalidValue;
    kv_append_fp8_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(
        static_cast<const uint4 *>(k), static_cast<const uint4 *>(v), static_cast<uint4 *>(k_cache),
        static_cast<uint4 *>(v_cache), slot_mapping, k_scale, v_scale, num_tokens, num_kv_heads, chunks, block_size,
        num_blocks, status);
    return cudaGetLastError();
}

cudaError_t append_launch(const void *k, const void *v, void *k_cache, void *v_cache, const int64_t *slot_mapping,
                          int num_tokens, int num_kv_heads, int head_dim, int block_size, int num_blocks,
                          int32_t *status, cudaStream_t stream) {
    const int chunks = head_dim / 8;
    const int64_t total = static_cast<int64_t>(num_tokens) * num_kv_heads * chunks;
    if (total == 0) return cudaSuccess;
    const int64_t grid = (total + 255) / 256;
    if (grid > 0x7fffffff) return cudaErrorInvalidValue;
    kv_append_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(
        static_cast<const uint4 *>(k), static_cast<const uint4 *>(v), static_cast<uint4 *>(k_cache),
        static_cast<uint4 *>(v_cache), slot_mapping, num_tokens, num_kv_heads, chunks, block_size, num_blocks,
        status);
    return cudaGetLastError();
}

cudaError_t validate_launch(const int32_t *block_tables, const int32_t *context_lens, int num_seqs,
                            int max_blocks_per_seq, int block_size, int num_blocks, int32_t *status,
                            cudaStream_t stream) {
    const int64_t total = static_cast<int64_t>(num_seqs) * max_blocks_per_seq;
    if (total == 0) return cudaSuccess;
    const int64_t grid = (total + 255) / 256;
    if (grid > 0x7fffffff) return cudaErrorInvalidValue;
    validate_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(block_tables, context_lens, num_seqs,
                                                                      max_blocks_per_seq, block_size, num_blocks,
                                                                      status);
    return cudaGetLastError();
}

}  // namespace pkv
