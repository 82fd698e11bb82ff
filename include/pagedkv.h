/*
 * pagedkv.h -- C ABI of the paged KV-cache decode library (libpagedkv.so).
 *
 * The operation: single-query attention for a batch of decoding sequences
 * whose keys and values live in fixed-size blocks scattered through one
 * preallocated pool, reached through a per-sequence block table.
 *   - "vLLM Fundamentals: Paged Attention and Batching", section "Paged
 *     Attention": the KV cache is split into blocks that are not contiguous,
 *     each sequence gets a block table, and the paged kernel follows the table
 *     to gather the blocks; section "Just a python process": the pool is one
 *     large tensor allocated once, and the engine packs the block tables into
 *     tensors and sends them to the GPU at every step.
 *   - "Deep Dive into vLLM: PagedAttention & High-Performance Inference",
 *     section 2.1: logical blocks map to physical blocks through the table.
 *   - runbyai.xyz post 449, section 1: a decode step reads the keys and values
 *     of all previous tokens, and is limited by memory bandwidth.
 *
 * Conventions for every call:
 *   - Pointers named d_* or documented as "device" are device pointers owned by
 *     the caller; the library never allocates, frees or keeps any memory.
 *   - Tensors are dense, row-major, in the layouts given below. bf16 tensors
 *     (k, v, q, out, caches) must be 16-byte aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream). Calls only enqueue work; nothing is synchronised unless stated.
 *   - Return value: PKV_OK (0) or a negative PKV_ERR_* code; pkv_last_error()
 *     then gives a message (thread-local, valid until the next call on that
 *     thread). Argument checks run before any CUDA call, so a rejected call
 *     enqueues nothing.
 *   - Problems that only the device can see (a table entry outside the pool, a
 *     context length past the table, a slot past the pool, a bounded wait that
 *     ran out) never trap: the kernels skip the bad access and OR a
 *     PKV_STATUS_* bit into a device status word the caller can read.
 *
 * Readings where the pages are silent: the attention is softmax(scale*q.K^T).V
 * over all context_lens[s] tokens of sequence s (no mask inside the context);
 * query head j reads kv head floor(j / (num_q_heads / num_kv_heads)); the pool
 * layout is [num_blocks][block_size][num_kv_heads][head_dim]; the slot of a
 * token is physical_block * block_size + offset_in_block.
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PKV_OK 0
#define PKV_ERR_INVALID_ARGUMENT (-1) /* null pointer, bad size, misaligned pointer, small workspace */
#define PKV_ERR_UNSUPPORTED (-2)      /* head_dim, block_size or head grouping not compiled in */
#define PKV_ERR_CUDA (-3)             /* a CUDA runtime call or a launch failed */
#define PKV_ERR_OUT_OF_BLOCKS (-4)    /* the block manager has too few free blocks; nothing changed */

/* Bits of the device status word (sticky: kernels only OR bits in). */
#define PKV_STATUS_BAD_BLOCK_ID 1     /* a needed table entry is outside [0, num_blocks); that block is skipped */
#define PKV_STATUS_BAD_CONTEXT_LEN 2  /* context_lens[s] < 0 or > max_blocks_per_seq * block_size; clamped */
#define PKV_STATUS_WAIT_TIMEOUT 4     /* a bounded wait inside a kernel gave up; outputs are not valid */
#define PKV_STATUS_BAD_SLOT 8         /* an append slot is >= num_blocks * block_size; that token is skipped */
#define PKV_STATUS_BAD_PREFIX_GROUP 16 /* a prefix-group member's table differs from the group's shared blocks */

/* Supported shapes of the decode kernels. */
#define PKV_MAX_GROUP 8               /* num_q_heads / num_kv_heads <= 8 */

/*
 * Tuning knobs of paged_attn_decode_ex. Zero in any field means "default".
 *   num_ctas          CTAs of the persistent decode grid (1..1024); default:
 *                     every CTA that fits on the device at once, or fewer for
 *                     a batch whose weight -- bounded by num_seqs x kv heads x
 *                     (max_blocks_per_seq tiles + piece cost), the lengths
 *                     being on the device -- gives a CTA under 8 tiles. The
 *                     KV blocks of a launch are split evenly over the CTAs, so
 *                     this also sets how finely long contexts are split.
 *   num_stages        shared-memory stages (one KV tile each) per warp (1..4; a
 *                     CTA has 4 warps); default: 1 on tensor cores, about 64 KB
 *                     of KV blocks per CTA on CUDA cores.
 *   ctas_per_sm       resident CTAs per SM of the default grid; default: the
 *                     occupancy limit.
 *   math              0 = default (2), 1 = fp32 CUDA cores, 2 = bf16 tensor cores
 *                     (mma.sync m16n8k16, fp32 accumulate; probabilities rounded
 *                     to bf16 for the P.V product).
 *   l2_prefetch       KV blocks each warp prefetches into L2 ahead of the ones
 *                     it loads into shared memory (1..32); -1 or 0 (default) =
 *                     none (on B200 every distance measured slower).
 *   piece_cost        extra weight, in KV blocks, that every non-empty (sequence,
 *                     kv head) segment adds when the batch is split between CTAs,
 *                     standing for a piece's fixed cost (1..64); -1 = none;
 *                     default 8, 16 where a kv head serves more than 4 query
 *                     heads (24 on e4m3 pools), 12 on e4m3 pools and with head
 *                     packing. Keeps CTAs that get many short contexts from
 *                     finishing last.
 *   head_pack         0 = default (2 where possible), 1 = off, 2 = read kv heads
 *                     2h and 2h + 1 together as one head of twice the head_dim
 *                     (the pool's [bs][Hkv][D] rows are the same bytes as
 *                     [bs][Hkv/2][2D]), so that each token row of a read is
 *                     256 contiguous bytes instead of 128. Possible on tensor
 *                     cores with head_dim 64, an even num_kv_heads and a group
 *                     of at most 4 (on e4m3 pools also with head_dim 128, see
 *                     paged_attn_decode_fp8); asking for 2 elsewhere returns
 *                     PKV_ERR_UNSUPPORTED.
 *   tile_tokens       token rows per shared-memory tile: 0 = default (16), 16, or
 *                     32 (block_size 32 only). With 16, a 32-token block is read
 *                     as two tiles of 16 rows, so that the stages of a CTA are as
 *                     small as for 16-token blocks and twice as many CTAs fit on
 *                     an SM; more than block_size returns PKV_ERR_INVALID_ARGUMENT.
 *                     The result does not depend on it beyond rounding order.
 *   prefix_groups     see pkv_prefix_groups above (NULL: none).
 *   prefix_tiles      16-row tiles of a shared prefix that one CTA streams before
 *                     storing its partials (1..4096); default: the CTAs are
 *                     split between the shared prefixes and the rest in
 *                     proportion to their work (the rest bounded by
 *                     max_blocks_per_seq, the lengths being on the device).
 *                     Raised as needed to fit the workspace and leave a CTA
 *                     to the rest.
 */
/*
 * Prefix groups: runs of consecutive sequences of a batch whose block tables
 * start with the same physical blocks -- a shared system prompt, or the
 * parallel samples and beam candidates of one prompt, which share the blocks
 * of their common tokens ("Deep Dive into vLLM", section 2.2, Flexible
 * Sharing; runbyai.xyz post 449, section 3). Group g is sequences begin[g] ..
 * end[g] - 1 (at least two), whose tables agree on entries 0 .. blocks[g] - 1;
 * groups are disjoint and in increasing order (begin[g + 1] >= end[g]). Given as pkv_decode_options.prefix_groups, the decode reads
 * those shared blocks once per group and kv head for all the group's query
 * rows (up to 64 rows per CTA) instead of once per sequence, and merges them
 * with each sequence's own blocks by the log-sum-exp identity; the result is
 * the same attention (up to rounding order). A member whose context ends
 * inside the shared blocks attends only to its own tokens.
 * The kernel checks that each member's table entries equal the group's first
 * sequence's (for the tokens the member attends) and sets
 * PKV_STATUS_BAD_PREFIX_GROUP otherwise (that member's output is then wrong).
 * Used with bf16 pools on tensor cores (math 0 or 2) with 16-row tiles; head
 * packing is not applied to a batch with groups. At most PKV_MAX_PREFIX_GROUPS
 * groups per 2048 sequences; groups beyond that, groups a 2048-sequence launch
 * boundary leaves with one member, and batches whose workspace has no room
 * for the group partials are decoded without the grouping (same results).
 * A launch with groups is cooperative (cudaLaunchCooperativeKernel: its CTAs
 * wait, bounded, for one another's pieces of the shared-prefix segments they
 * merge), so num_ctas is reduced to the CTAs that fit on the device at once.
 */
#define PKV_MAX_PREFIX_GROUPS 16
typedef struct pkv_prefix_groups {
    int num_groups;
    const int32_t *begin;   /* host [num_groups]: first sequence of each group */
    const int32_t *end;     /* host [num_groups]: one past its last; begin + 2 <= end <= next begin, <= num_seqs */
    const int32_t *blocks;  /* host [num_groups]: shared leading table entries, 1 .. max_blocks_per_seq */
} pkv_prefix_groups;

typedef struct pkv_decode_options {
    int num_ctas;
    int num_stages;
    int ctas_per_sm;
    int math;
    int l2_prefetch;
    int piece_cost;
    int head_pack;
    int tile_tokens;
    const pkv_prefix_groups *prefix_groups;  /* NULL: none */
    int prefix_tiles;
} pkv_decode_options;

/*
 * Finds prefix groups in host copies of a batch's tables (for example the
 * rows pkv_bm_pack produced): maximal runs, scanned from the first sequence,
 * of at least two consecutive sequences whose tables agree on at least
 * min_blocks leading entries that every member's context covers; blocks[g] is
 * the run's longest such agreement. Writes at most max_groups groups into
 * begin[], end[], blocks[] and sets *num_groups. Host only; returns PKV_OK or
 * PKV_ERR_INVALID_ARGUMENT.
 */
int pkv_find_prefix_groups(const int32_t *block_tables, const int32_t *context_lens, int num_seqs,
                           int max_blocks_per_seq, int block_size, int min_blocks, int32_t *begin, int32_t *end,
                           int32_t *blocks, int max_groups, int *num_groups);

/*
 * Bytes of device workspace paged_attn_decode needs for this shape
 * (host-only; returns PKV_OK and sets *bytes).
 * Layout: [0, 256) header whose first int32 is the device status word, and
 * whose bytes [8, 20) count the decode launches made with the workspace (each
 * launch advances the count at its end, so every launch -- each replay of a
 * captured CUDA graph too -- has an epoch of its own); one counter per
 * (sequence, kv head) of a launch, tagged with that epoch, so the workspace
 * never needs clearing (zero it whole or not at all: zeroing the launch count
 * alone would let old counters be read as new); fp32 partial outputs and
 * log2-sum-exp values of the context pieces that CTA boundaries cut. At most
 * 2048 sequences go in one launch; longer batches reuse the workspace launch
 * after launch.
 */
int pkv_decode_workspace_bytes(int num_seqs, int num_q_heads, int head_dim, size_t *bytes);

/*
 * Paged decode attention (one query token per sequence).
 *
 * out           device bf16 [num_seqs][num_q_heads][head_dim]   (written)
 * q             device bf16 [num_seqs][num_q_heads][head_dim]
 * k_cache       device bf16 [num_blocks][block_size][num_kv_heads][head_dim]
 * v_cache       device bf16, same layout as k_cache
 * block_tables  device int32 [num_seqs][max_blocks_per_seq]; entry b of row s is
 *               the physical block of logical block b of sequence s. Only
 *               entries b < ceil(context_lens[s] / block_size) are read.
 * context_lens  device int32 [num_seqs]; 0 gives an all-zero output row.
 * scale         multiplies q.k before the softmax (e.g. 1/sqrt(head_dim)).
 * workspace     device, at least pkv_decode_workspace_bytes() bytes, 256-byte
 *               aligned; its status word is ORed, never cleared, by this call.
 *
 * Supported: head_dim in {64, 128}; block_size in {16, 32}; num_q_heads a
 * multiple of num_kv_heads with a ratio <= PKV_MAX_GROUP; num_blocks *
 * block_size < 2^31. Any num_seqs >= 0 (0 is a no-op).
 * Per call (and per 2048 sequences): one persistent decode kernel whose CTAs
 * each take an equal share of the batch's KV blocks (weighted per context
 * piece); a context split between CTAs is merged (log-sum-exp) by the CTA that
 * stores its last piece. For a given device, options and batch shape (the
 * default grid depends on num_seqs and max_blocks_per_seq), results are
 * bitwise reproducible and depend only on the logical order of tokens, not on
 * where their blocks sit in the pool.
 */
int paged_attn_decode(void *out, const void *q, const void *k_cache, const void *v_cache,
                      const int32_t *block_tables, const int32_t *context_lens,
                      int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                      int block_size, float scale, int max_blocks_per_seq, int num_blocks,
                      void *workspace, size_t workspace_bytes, void *stream);

/* paged_attn_decode with tuning knobs (opts may be NULL = all defaults). */
int paged_attn_decode_ex(void *out, const void *q, const void *k_cache, const void *v_cache,
                         const int32_t *block_tables, const int32_t *context_lens,
                         int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                         int block_size, float scale, int max_blocks_per_seq, int num_blocks,
                         void *workspace, size_t workspace_bytes, const pkv_decode_options *opts,
                         void *stream);

/*
 * Multi-query paged attention: chunked prefill and mixed batches ("vLLM
 * Fundamentals", section "Continuous Batching": long prefills are cut into
 * chunks under a token budget and batched with decodes). Sequence s brings
 * n_s = query_start[s + 1] - query_start[s] query tokens, the LAST n_s of its
 * context_lens[s] tokens, whose keys and values are already in the pool
 * (kv_cache_append). Query i of sequence s sits at position
 * p = context_lens[s] - n_s + i and attends causally to positions 0 .. p:
 *   out[query_start[s] + i][j] = softmax_t<=p(scale q.K_t) . V_t, kv head j / G.
 * A decode step is the case n_s = 1.
 *
 * out, q        device bf16 [num_tokens][num_q_heads][head_dim]
 * query_start   device int32 [num_seqs + 1]: 0, then non-decreasing, ending at
 *               num_tokens; every n_s <= context_lens[s] and <= max_query_len
 *               (host int: the largest n_s, which sizes the grid)
 * d_status      device int32 status word (required): a sequence whose
 *               query_start / context length is inconsistent is skipped and sets
 *               PKV_STATUS_BAD_CONTEXT_LEN; a bad table entry sets
 *               PKV_STATUS_BAD_BLOCK_ID (that block is skipped).
 * The rest as paged_attn_decode. Supported: head_dim 64 / 128, block_size
 * 16 / 32, group <= 8, num_seqs and num_kv_heads <= 65535, and a block table
 * row (max_blocks_per_seq * 4 bytes) that fits shared memory next to the
 * kernel's tiles. One launch; no workspace.
 * Kernel: paged_attn_prefill_ex with kernel 0 -- the tcgen05 kernel when the
 * group num_q_heads / num_kv_heads is 1, 2, 4 or 8 and its shared memory
 * (about 100 KB + max_blocks_per_seq * 4 bytes) fits, else the mma.sync
 * kernel: a CTA per (64 rows of (query token, group head), sequence, kv head)
 * streams the K/V blocks its rows need (TMA tile copies, 2-stage ring) and
 * computes S = Q K^T, a causal online softmax and O += P V (mma.sync
 * m16n8k16 bf16, fp32 accumulate; P rounded to bf16).
 */
int paged_attn_prefill(void *out, const void *q, const void *k_cache, const void *v_cache,
                       const int32_t *block_tables, const int32_t *context_lens, const int32_t *query_start,
                       int num_seqs, int num_tokens, int max_query_len, int num_q_heads, int num_kv_heads,
                       int head_dim, int block_size, float scale, int max_blocks_per_seq, int num_blocks,
                       int32_t *d_status, void *stream);

/*
 * paged_attn_prefill with a choice of kernel: 0 = default (tcgen05 where it
 * applies, else mma.sync), 1 = the mma.sync kernel, 2 = the tcgen05 kernel
 * (PKV_ERR_UNSUPPORTED unless num_q_heads / num_kv_heads is 1, 2, 4 or 8 and
 * its shared memory fits); another value returns PKV_ERR_INVALID_ARGUMENT.
 * The tcgen05 kernel: a CTA per 128 rows of (query token, group head) of a
 * sequence and kv head, two CTAs per SM (about 100 KB of shared memory and
 * 256 tensor-memory columns each); S = Q K^T and O += P V on tcgen05.mma with
 * fp32 accumulators in tensor memory (P rounded to bf16, the softmax sums in
 * fp32), Q and the K/V blocks staged by TMA, one thread per query row for
 * the causal online softmax. Every wait inside it is bounded (1 s): one that
 * gives up sets PKV_STATUS_WAIT_TIMEOUT in d_status and the CTA drains its
 * copies and MMAs and frees its tensor memory before it exits.
 */
int paged_attn_prefill_ex(void *out, const void *q, const void *k_cache, const void *v_cache,
                          const int32_t *block_tables, const int32_t *context_lens, const int32_t *query_start,
                          int num_seqs, int num_tokens, int max_query_len, int num_q_heads, int num_kv_heads,
                          int head_dim, int block_size, float scale, int max_blocks_per_seq, int num_blocks,
                          int32_t *d_status, int kernel, void *stream);

/*
 * FP8 KV cache. The pools hold e4m3 codes (1 sign, 4 exponent bits with bias
 * 7, 3 mantissa bits; 0x7f / 0xff are NaN), laid out like the bf16 pools,
 * [num_blocks][block_size][num_kv_heads][head_dim] bytes, with one fp32 scale
 * per kv head for K (k_scale, device [num_kv_heads]) and one for V: element d
 * of head h stands for e4m3(code) * scale[h]. This halves the bytes a decode
 * reads (runbyai post 449, section 5, names quantization among the means for
 * long contexts; the format and the per-head scales are this library's).
 *
 * kv_cache_append_fp8: like kv_cache_append, storing for each element x of
 * token i, head h the e4m3 code nearest to the fp32 quotient x / scale[h]
 * (ties to an even mantissa), saturated to +-448. head_dim must be a
 * multiple of 16.
 *
 * paged_attn_decode_fp8 / paged_attn_decode_append_fp8: paged_attn_decode_ex /
 * paged_attn_decode_append over e4m3 pools (same arguments plus the scales).
 * The codes are widened exactly to f16 and multiplied on tensor cores
 * (mma.sync f16, fp32 accumulation); q is rounded to f16 after scaling each
 * query row by a power of two that puts its largest magnitude in [2^14,
 * 2^15); probabilities are rounded to f16. Supported: head_dim 128, or 64
 * with head packing (an even num_kv_heads and num_q_heads / num_kv_heads <=
 * 4, so that every row read is 128 bytes); block_size 16 or 32; opts->math 0
 * or 2 (1 returns PKV_ERR_UNSUPPORTED). Default ring: about 8 KB of blocks
 * in flight per warp -- 1 stage when kv heads are read in pairs (rows of 256
 * codes, the default for head_dim 128), else 2.
 */
int kv_cache_append_fp8(const void *k, const void *v, void *k_cache, void *v_cache, const int64_t *slot_mapping,
                        const float *k_scale, const float *v_scale, int num_tokens, int num_kv_heads, int head_dim,
                        int block_size, int num_blocks, int32_t *d_status, void *stream);

int paged_attn_decode_fp8(void *out, const void *q, const void *k_cache, const void *v_cache, const float *k_scale,
                          const float *v_scale, const int32_t *block_tables, const int32_t *context_lens,
                          int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size, float scale,
                          int max_blocks_per_seq, int num_blocks, void *workspace, size_t workspace_bytes,
                          const pkv_decode_options *opts, void *stream);

int paged_attn_decode_append_fp8(void *out, const void *q, const void *k_new, const void *v_new,
                                 const int64_t *slot_mapping, void *k_cache, void *v_cache, const float *k_scale,
                                 const float *v_scale, const int32_t *block_tables, const int32_t *context_lens,
                                 int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                 float scale, int max_blocks_per_seq, int num_blocks, void *workspace,
                                 size_t workspace_bytes, const pkv_decode_options *opts, void *stream);

/*
 * One whole decode step in one launch: kv_cache_append of the step's token of
 * every sequence, then paged_attn_decode over contexts that include it (the
 * decode step of "Deep Dive into vLLM", section 2: each generated token's key
 * and value are cached, and attention reads all cached tokens).
 *
 * Same arguments as paged_attn_decode_ex, plus
 * k_new, v_new   device bf16 [num_seqs][num_kv_heads][head_dim]: the step's key
 *                and value of each sequence (16-byte aligned).
 * slot_mapping   device int64 [num_seqs]: slot of sequence s's new token, which
 *                must be the slot of its last position L_s - 1, i.e.
 *                block_tables[s][(L_s - 1) / block_size] * block_size +
 *                (L_s - 1) % block_size; < 0 = no append for s (attention then
 *                reads position L_s - 1 from the pool as it is).
 * k_cache, v_cache are written (the appended rows).
 *
 * Results (out and the pools) are bit-identical to kv_cache_append followed
 * by paged_attn_decode_ex with the same options. The warp that computes the
 * block holding position L_s - 1 takes the new rows from k_new / v_new into
 * its staged copy of the block and writes them to the pool, so the append
 * costs no launch and no extra read. A slot that is >= 0 but not the last
 * position (or, for L_s = 0, not inside the pool) is not written and sets
 * PKV_STATUS_BAD_SLOT in the workspace status word. The caller guarantees,
 * as with any append, that no other sequence of the batch reads a slot that
 * is being written (copy-on-write of shared blocks is the caller's).
 */
int paged_attn_decode_append(void *out, const void *q, const void *k_new, const void *v_new,
                             const int64_t *slot_mapping, void *k_cache, void *v_cache,
                             const int32_t *block_tables, const int32_t *context_lens, int num_seqs,
                             int num_q_heads, int num_kv_heads, int head_dim, int block_size, float scale,
                             int max_blocks_per_seq, int num_blocks, void *workspace, size_t workspace_bytes,
                             const pkv_decode_options *opts, void *stream);

/*
 * paged_attn_decode for callers that cannot allocate device memory. The pages
 * have no counterpart to this call.
 *
 * Who needs it: a caller that owns no device allocator of its own -- for
 * example an engine that, as the pages describe for vLLM, handed all GPU
 * memory left after the weights to one preallocated KV pool, or a plugin host
 * that exposes no allocation hook -- cannot provide the workspace that
 * paged_attn_decode asks for. This call takes the same inputs and output but
 * no workspace: its scratch is a static device array of
 * PKV_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads the
 * library holds until the process exits. It calls no cudaMalloc, cudaFree or
 * other allocating routine.
 *
 * Limits and rules:
 *   - Batches whose workspace (pkv_decode_workspace_bytes) exceeds
 *     PKV_NOALLOC_SCRATCH_BYTES are rejected with
 *     PKV_ERR_INVALID_ARGUMENT and a message giving both sizes.
 *   - The first call on a device looks up the scratch's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture begins. The address is kept for the life of
 *     the process: after cudaDeviceReset, or anything else that destroys the
 *     device's primary context, do not call this entry point again in that
 *     process (it would hand the kernels the old context's address).
 *   - All calls share the one scratch, which keeps the last call's contents.
 *     Calls that overlap on the GPU (different streams, no ordering between
 *     them) race on it and give wrong results: order them.
 *   - d_status: device int32 or NULL. If given, it is overwritten (not ORed)
 *     with this call's PKV_STATUS_* bits once the call's kernels finish.
 * Results are identical to paged_attn_decode with the default options.
 */
#define PKV_NOALLOC_SCRATCH_BYTES (64u << 20)
int paged_attn_decode_noalloc(void *out, const void *q, const void *k_cache, const void *v_cache,
                              const int32_t *block_tables, const int32_t *context_lens,
                              int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                              int block_size, float scale, int max_blocks_per_seq, int num_blocks,
                              int32_t *d_status, void *stream);

/*
 * Slot-mapped cache append: for every token i with slot_mapping[i] >= 0 and
 * every kv head h, copies k[i][h][:] to k_cache[slot / block_size]
 * [slot % block_size][h][:] and v[i][h][:] likewise (runbyai.xyz post 449,
 * sections 1-2: each step computes and caches the new token's key and value).
 *
 * k, v          device bf16 [num_tokens][num_kv_heads][head_dim]
 * k_cache/v_cache device bf16 [num_blocks][block_size][num_kv_heads][head_dim] (updated in place)
 * slot_mapping  device int64 [num_tokens]; < 0 means "no write" (padding)
 * d_status      device int32 status word, or NULL; gets PKV_STATUS_BAD_SLOT for
 *               a slot >= num_blocks * block_size (that token is skipped)
 *
 * head_dim must be a multiple of 8. Bit-exact copy. Two tokens with the same
 * slot race (either may win); the caller keeps slots distinct within a call.
 */
int kv_cache_append(const void *k, const void *v, void *k_cache, void *v_cache,
                    const int64_t *slot_mapping, int num_tokens, int num_kv_heads, int head_dim,
                    int block_size, int num_blocks, int32_t *d_status, void *stream);

/*
 * Device check of a batch's tables: ORs PKV_STATUS_BAD_CONTEXT_LEN for any
 * context length outside [0, max_blocks_per_seq * block_size] and
 * PKV_STATUS_BAD_BLOCK_ID for any needed entry outside [0, num_blocks) into
 * *d_status. Never traps; enqueues one small kernel.
 */
int pkv_validate(const int32_t *block_tables, const int32_t *context_lens, int num_seqs,
                 int max_blocks_per_seq, int block_size, int num_blocks, int32_t *d_status,
                 void *stream);

/*
 * Copies the device status word to *status (host) after synchronising `stream`,
 * and zeroes it when clear != 0. For paged_attn_decode the word is the first
 * int32 of the workspace.
 */
int pkv_read_status(int32_t *d_status, int32_t *status, int clear, void *stream);

/*
 * Self-test of the kernels' failure path: enqueues one kernel that waits on an
 * mbarrier nothing ever arrives at. The bounded wait gives up after about one
 * second and ORs PKV_STATUS_WAIT_TIMEOUT into *d_status (device int32); the
 * kernel then returns normally and the context stays usable. Bit 0x40000000
 * is set instead if the wait wrongly succeeded.
 */
int pkv_selftest_bounded_wait(int32_t *d_status, void *stream);

/*
 * Copy-on-write block copies: for c < num_copies, physical block dst[c] of
 * both pools becomes a copy of block src[c] (block_size rows of num_kv_heads *
 * head_dim elements of elem_bytes bytes: 2 for bf16 pools, 1 for e4m3 pools;
 * a row must be a multiple of 16 bytes). src, dst: device int32 [num_copies] (from
 * pkv_bm_take_copies). The copies must not chain (no dst is another copy's
 * src); the block manager never produces such a list. An id outside
 * [0, num_blocks) skips that copy and ORs PKV_STATUS_BAD_BLOCK_ID into
 * *d_status (device int32, may be NULL). Runs on `stream`; issue it before any
 * other write of the pools in the same step.
 */
int kv_block_copy(void *k_cache, void *v_cache, const int32_t *src, const int32_t *dst, int num_copies,
                  int num_kv_heads, int head_dim, int elem_bytes, int block_size, int num_blocks, int32_t *d_status,
                  void *stream);

/*
 * Host-side block manager of one KV pool (no CUDA calls; thread-safe).
 *
 * It follows the block-table scheme of "Deep Dive into vLLM" (section 2.1:
 * logical blocks map to physical blocks through a per-sequence block table;
 * section 2.2: blocks are allocated only when tokens are stored, and the
 * sequences of parallel sampling or beam search share their prompt's blocks,
 * copy-on-write like an OS) and runbyai post 449 (section 3: prompts that
 * start alike share those blocks; section 4: a finished sequence's blocks are
 * freed at once for new sequences). Each physical block has a reference
 * count; a block is free exactly when the count is 0 (LIFO free list, block 0
 * handed out first). Sequence ids are any int64 the caller chooses.
 *
 * A decode step with the manager: pkv_bm_append for every running sequence
 * (each gives the slot of its new token, the slot of its last position),
 * pkv_bm_take_copies, kv_block_copy of those copies, pkv_bm_pack of the running
 * sequences' tables and lengths, then paged_attn_decode_append with the slots.
 * Fork only between steps (after the step that wrote the parent's last token);
 * pkv_bm_fork refuses while copies are pending.
 *
 * Errors: PKV_ERR_INVALID_ARGUMENT (unknown or reused id, bad sizes) and
 * PKV_ERR_OUT_OF_BLOCKS leave the manager unchanged; pkv_bm_last_error()
 * gives the message.
 */
typedef struct pkv_block_manager pkv_block_manager;

/* A manager of num_blocks free blocks of block_size tokens; NULL if either is <= 0. */
pkv_block_manager *pkv_bm_create(int num_blocks, int block_size);
void pkv_bm_destroy(pkv_block_manager *bm);

/* Free blocks, or a negative error code. */
int pkv_bm_num_free(const pkv_block_manager *bm);

/* References to `block` (sequences holding it + pending copies reading it). */
int pkv_bm_refcount(const pkv_block_manager *bm, int block);

/*
 * A new sequence holding num_tokens tokens (its prompt). With prefix_seq >= 0,
 * its first prefix_tokens tokens are those of sequence prefix_seq: the whole
 * blocks among them (prefix_tokens / block_size blocks) are shared, not
 * copied. slots (host int64 [num_tokens], may be NULL) receives each token's
 * slot for writing the prompt with kv_cache_append, -1 for the shared tokens
 * (already in the pool).
 */
int pkv_bm_add(pkv_block_manager *bm, int64_t seq_id, int64_t num_tokens, int64_t prefix_seq,
               int64_t prefix_tokens, int64_t *slots);

/* Sequence `child` shares every block of `parent` (same tokens). */
int pkv_bm_fork(pkv_block_manager *bm, int64_t parent, int64_t child);

/*
 * Reserves the next position of the sequence for one new token; *slot = its
 * slot. A full last block (or none) takes a fresh block; a last block that
 * has room but is shared is first copied to a fresh block (copy-on-write: the
 * copy is queued for pkv_bm_take_copies).
 */
int pkv_bm_append(pkv_block_manager *bm, int64_t seq_id, int64_t *slot);

/* The sequence leaves: each of its blocks loses a reference. */
int pkv_bm_free(pkv_block_manager *bm, int64_t seq_id);

/* Copies queued since the last call (0 if none). */
int pkv_bm_pending_copies(const pkv_block_manager *bm);

/*
 * Moves the queued copies, in queue order, into src / dst (host int32
 * [capacity]) and returns how many; fails, taking none, if there are more
 * than `capacity`. A queued copy holds a reference on its source block until
 * it is taken, so the source cannot be reused before the copy is issued.
 */
int pkv_bm_take_copies(pkv_block_manager *bm, int32_t *src, int32_t *dst, int capacity);

/* *len = the sequence's token count. */
int pkv_bm_seq_len(const pkv_block_manager *bm, int64_t seq_id, int64_t *len);

/*
 * The step's inputs for sequences seq_ids[0 .. num_seqs): block_tables (host
 * int32 [num_seqs][max_blocks_per_seq], padded with -1) and context_lens (host
 * int32 [num_seqs]), as paged_attn_decode takes them.
 */
int pkv_bm_pack(const pkv_block_manager *bm, const int64_t *seq_ids, int num_seqs, int max_blocks_per_seq,
                int32_t *block_tables, int32_t *context_lens);

/* Message of the last failed block-manager call on this thread. */
const char *pkv_bm_last_error(void);

/* Message of the last failed call on this thread ("" if none). */
const char *pkv_last_error(void);

/* Library version string. */
const char *pkv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H */
