// api.cu -- the C ABI of libpagedkv.so (declared in include/pagedkv.h).
//
// Every entry point checks its arguments on the host before any CUDA call,
// then enqueues kernels on the caller's stream. The library allocates nothing
// and keeps no per-call state: the KV pool, the tables and the workspace are
// the caller's ("vLLM Fundamentals: Paged Attention and Batching", section
// "Just a python process": one large pool tensor allocated once by the engine;
// the engine sends the packed block tables to the GPU at every step).
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "launch.h"
#include "pagedkv.h"

namespace {

thread_local char g_err[512] = "";

int fail(int code, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return code;
}

int ok() {
    g_err[0] = '\0';
    return PKV_OK;
}

int cuda_fail(cudaError_t e, const char *what) {
    return fail(PKV_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int group_pad(int g) { return g <= 1 ? 1 : g <= 2 ? 2 : g <= 4 ? 4 : 8; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Tensor map over a pool [num_blocks][bs][Hkv][D] of `es`-byte elements (bf16:
// 2, e4m3 codes: 1) seen as 4D (128/es, D*es/128, Hkv, num_blocks*bs),
// innermost first; one box = one 128-byte column slice of `rows` consecutive
// token rows (a whole block, or a 16-row half of a 32-token block) of one kv
// head: (128/es, 1, 1, rows), 128-byte swizzled in shared memory (a tile is
// D*es/128 such [rows][128 B] slices).
int make_pool_map(CUtensorMap *map, const void *pool, int num_blocks, int bs, int hkv, int d, int es = 2,
                  int rows = 0) {
    if (rows == 0) rows = bs;
    auto fn = encode_fn();
    if (!fn) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const cuuint64_t inner = 128 / es;
    cuuint64_t dims[4] = {inner, static_cast<cuuint64_t>(d) * es / 128, static_cast<cuuint64_t>(hkv),
                          static_cast<cuuint64_t>(num_blocks) * bs};
    cuuint64_t strides[3] = {128, static_cast<cuuint64_t>(d) * es, static_cast<cuuint64_t>(hkv) * d * es};
    cuuint32_t box[4] = {static_cast<cuuint32_t>(inner), 1, 1, static_cast<cuuint32_t>(rows)};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, es == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                    const_cast<void *>(pool), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return PKV_OK;
}

// Tensor map over the queries q [T][Hkv][G][D] bf16 seen as 5D (64, D/64, G,
// Hkv, T): one box = one 64-column slice of 128 / G query tokens x G heads,
// i.e. 128 rows (token, head) of 128 bytes, 128-byte swizzled.
int make_query_map(CUtensorMap *map, const void *q, int num_tokens, int hkv, int group, int d) {
    auto fn = encode_fn();
    if (!fn) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    cuuint64_t dims[5] = {64, static_cast<cuuint64_t>(d / 64), static_cast<cuuint64_t>(group),
                          static_cast<cuuint64_t>(hkv), static_cast<cuuint64_t>(num_tokens)};
    cuuint64_t strides[4] = {128, static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(group) * d * 2,
                             static_cast<cuuint64_t>(hkv) * group * d * 2};
    cuuint32_t box[5] = {64, 1, static_cast<cuuint32_t>(group), 1, static_cast<cuuint32_t>(128 / group)};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(q), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled (queries) failed (%d)", static_cast<int>(r));
    return PKV_OK;
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    static std::mutex mu;
    static std::vector<int> cache;
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= static_cast<int>(cache.size())) cache.resize(dev + 1, 0);
    if (cache[dev] == 0 && cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
        cache[dev] = n;
    return cache[dev];
}

// Workspace layout: [0, 256) header (status word at 0; the launch epoch at 8
// and the CTAs started at 16, advanced by the kernels) | per-segment piece
// counters [S_chunk * Hkv <= S_chunk * Hq] uint64 | fp32 partial outputs [rows][D] | fp32 log2-sum-exp [rows],
// rows = (S_chunk + kMaxCtas) * Hq bounds the pieces' rows of one launch
// (pieces <= S_chunk * Hkv + C, each with G <= Hq rows).
struct WorkspaceLayout {
    size_t seg_count, o_part, lse_part, total;
};

WorkspaceLayout workspace_layout(int num_seqs, int num_q_heads, int head_dim) {
    const int64_t sc = num_seqs < pkv::kMaxSeqsPerLaunch ? num_seqs : pkv::kMaxSeqsPerLaunch;
    const int64_t rows = (sc + pkv::kMaxCtas) * num_q_heads;
    WorkspaceLayout w;
    w.seg_count = pkv::kWorkspaceHeaderBytes;
    w.o_part = w.seg_count + (sc * num_q_heads * 8 + 255) / 256 * 256;
    w.lse_part = w.o_part + rows * head_dim * 4;
    w.total = w.lse_part + (rows * 4 + 255) / 256 * 256;
    return w;
}

// Stages per warp: one for the tensor-core path (more resident CTAs beat a
// deeper ring: 4 CTAs of 4 warps per SM with 8 KB blocks); about 64 KB of
// blocks in flight per CTA for the CUDA-core path, which fits fewer CTAs.
constexpr int kDefaultL2Prefetch = 0;  // measured on the Llama-shaped batch: any prefetch distance was slower
// Weight of a piece's fixed cost, in 16-row tiles. With 16-row tiles and one
// barrier per stage, 8 beat 4 on every batch (same box: Llama-shaped 364.8 ->
// 355.0 us, OPT-shaped 43.9 -> 42.5, skewed 139.6 -> 132.2, e4m3 308.7 -> 296.0).
// A piece's merge grows with the query heads per kv head: with more than 4,
// 16 (Qwen-shaped, 7 per kv head: 42.6 -> 40.8 us; 8 -> 16 on the Llama-shaped
// batch, 4 per kv head: 354.9 -> 357.5). e4m3 pools: 12 (after the bit-placement
// conversion: Llama-shaped 265.5 -> 260.6 us, OPT-shaped 40.6 -> 38.3, skewed
// 119.0 -> 119.8).
// Head-packed bf16 pools (head_dim 64 in pairs): 12 (after the plain-add
// count-in, OPT-shaped 41.0 -> 39.0 us at 12, 40.3 at 16; 12 instead of 8 cost
// the Llama-shaped batch 2 us and the skewed one 1 us).
constexpr int kDefaultPieceCost = 8;
constexpr int kDefaultPieceCostWideGroup = 16;
constexpr int kDefaultPieceCostFp8 = 12;
constexpr int kDefaultPieceCostPacked = 12;
// e4m3 pools with more than 4 query heads per kv head: 24 (Qwen-shaped, 7 per
// kv head: 47.2 us at 12, 46.5 at 16, 45.1 at 24).
constexpr int kDefaultPieceCostFp8WideGroup = 24;
// Least weight (tiles, piece cost included) per CTA of a default grid. With
// many pieces of one context counted in by a plain add, 8 beat 16 on every
// small batch (same box: tiny 16.4 -> 12.3 us, one 2,048-token context 24.6
// -> 22.5, 4 x 512 24.6 -> 20.5, 8 x 1,024 Qwen-shaped 26.6 -> 24.6); 4 and 2
// were slower on the Qwen- and OPT-shaped ones.
constexpr int kMinCtaWeight = 8;

// Work of one shared-prefix tile (64 query rows) against one suffix tile (the G
// rows of one sequence), for splitting the CTAs between the two: the prefix
// tile does about 64 / G times the math but reads the same bytes, mostly from L2.
constexpr int kPrefixTileCost = 3;

// The prefix units of one launch (sequences s0 .. s0 + sc - 1): the groups of
// the caller's descriptor that have at least two members in the launch, as
// kernel parameters. Leaves a.num_groups = 0 when grouping does not apply.
// The CTAs are split between prefix units and suffixes in proportion to their
// work: the prefix tiles, and at most max_blocks_per_seq * sub tiles per
// sequence (less each group's shared ones) for the suffixes -- the host knows
// the table width, not the context lengths. tiles_per_piece > 0 sets the
// tiles of one unit instead.
void plan_prefix_groups(const pkv_prefix_groups *pg, int s0, int sc, int hkv, int group, int sub, int ctas,
                        int max_blocks_per_seq, int tiles_per_piece, pkv::DecodeArgs &a) {
    a.num_groups = 0;
    a.prefix_ctas = 0;
    a.tiles_per_piece = 1;
    a.prefix_np = 0;
    a.pre_base = 0;
    if (!pg || pg->num_groups <= 0 || ctas < 2) return;
    int n = 0, max_tiles = 0;
    long long prefix_work = 0, suffix_bound = static_cast<long long>(sc) * max_blocks_per_seq * sub;
    for (int g = 0; g < pg->num_groups && n < pkv::kMaxPrefixGroups; ++g) {
        const int lo = pg->begin[g] > s0 ? pg->begin[g] : s0;
        const int hi = pg->end[g] < s0 + sc ? pg->end[g] : s0 + sc;
        if (hi - lo < 2) continue;
        a.grp_begin[n] = lo - s0;
        a.grp_end[n] = hi - s0;
        a.grp_tiles[n] = pg->blocks[g] * sub;
        if (a.grp_tiles[n] > max_tiles) max_tiles = a.grp_tiles[n];
        const int per = pkv::kPrefixRows / group;  // members whose rows fit one unit
        const int row_tiles = (hi - lo + per - 1) / per;
        a.grp_row_tiles[n] = row_tiles;
        a.grp_members[n] = (hi - lo + row_tiles - 1) / row_tiles;  // spread evenly over the row tiles
        prefix_work += static_cast<long long>(row_tiles) * a.grp_tiles[n];
        suffix_bound -= static_cast<long long>(hi - lo) * a.grp_tiles[n];
        ++n;
    }
    if (n == 0) return;
    // Partial rows: the workspace holds (S + 1024) * Hq rows; the suffix pieces
    // take bases below sc * Hkv + ctas, the prefix pieces sc * Hkv * np after them.
    const long long room = 1024LL * hkv - ctas;
    const long long np_max = room / (static_cast<long long>(sc) * hkv);
    if (np_max < 1) return;
    int tpp = tiles_per_piece;
    if (tpp <= 0) {
        // units in proportion to the prefix's share of the work (at least one CTA each way)
        const double share = static_cast<double>(kPrefixTileCost * prefix_work) /
                             static_cast<double>(kPrefixTileCost * prefix_work + (suffix_bound > 0 ? suffix_bound : 0));
        long long target = static_cast<long long>(share * ctas);
        if (target < 1) target = 1;
        if (target > ctas - 1) target = ctas - 1;
        const long long unit_tiles = static_cast<long long>(hkv) * prefix_work;  // (head, row tile, tile) triples
        tpp = static_cast<int>((unit_tiles + target - 1) / target);
        if (tpp < 1) tpp = 1;
    }
    if ((max_tiles + tpp - 1) / tpp > np_max) tpp = static_cast<int>((max_tiles + np_max - 1) / np_max);
    long long units = 0;
    for (;;) {
        units = 0;
        for (int g = 0; g < n; ++g)
            units += static_cast<long long>(hkv) * a.grp_row_tiles[g] * ((a.grp_tiles[g] + tpp - 1) / tpp);
        if (units <= ctas - 1 || tpp >= max_tiles) break;
        ++tpp;  // rounding up the pieces made too many units
    }
    if (units > ctas - 1) return;  // no CTA would be left for the suffixes
    a.num_groups = n;
    a.tiles_per_piece = tpp;
    int np = 0;
    long long u = 0;
    for (int g = 0; g < n; ++g) {
        a.grp_unit0[g] = static_cast<int>(u);
        const int pieces = (a.grp_tiles[g] + tpp - 1) / tpp;
        if (pieces > np) np = pieces;
        u += static_cast<long long>(hkv) * a.grp_row_tiles[g] * pieces;
    }
    a.grp_unit0[n] = static_cast<int>(u);
    a.prefix_ctas = static_cast<int>(u);
    a.prefix_np = np;
    a.pre_base = sc * hkv + ctas;
}

int default_stages(int head_dim, int block_size, int math) {
    if (math == pkv::kMathTensorCore) return 1;
    if (math == pkv::kMathFp8) return head_dim == 256 ? 1 : 2;  // about 8 KB of blocks in flight per warp
    const int stage_bytes = 2 * block_size * head_dim * 2;
    int r = (64 * 1024) / (pkv::kConsumerWarps * stage_bytes);
    return r < 1 ? 1 : r > pkv::kMaxStagesPerWarp ? pkv::kMaxStagesPerWarp : r;
}

}  // namespace

extern "C" {

const char *pkv_last_error(void) { return g_err; }

const char *pkv_version(void) { return "pagedkv 0.1 (sm_100a)"; }

int pkv_decode_workspace_bytes(int num_seqs, int num_q_heads, int head_dim, size_t *bytes) {
    if (!bytes) return fail(PKV_ERR_INVALID_ARGUMENT, "bytes is NULL");
    if (num_seqs < 0 || num_q_heads <= 0 || head_dim <= 0)
        return fail(PKV_ERR_INVALID_ARGUMENT, "num_seqs must be >= 0, num_q_heads and head_dim > 0");
    *bytes = workspace_layout(num_seqs, num_q_heads, head_dim).total;
    return ok();
}

}  // extern "C"

namespace {

// Decode, optionally with the fused append (k_new, v_new, slots all non-NULL),
// over bf16 pools or, with k_scale / v_scale non-NULL, e4m3 pools.
int decode_impl(void *out, const void *q, const void *k_new, const void *v_new, const int64_t *slots,
                const void *k_cache, const void *v_cache, const float *k_scale, const float *v_scale,
                const int32_t *block_tables, const int32_t *context_lens,
                int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size, float scale,
                int max_blocks_per_seq, int num_blocks, void *workspace, size_t workspace_bytes,
                const pkv_decode_options *opts, void *stream) {
    if (num_seqs < 0) return fail(PKV_ERR_INVALID_ARGUMENT, "num_seqs < 0");
    const bool fp8 = k_scale != nullptr || v_scale != nullptr;
    if (fp8 && (!k_scale || !v_scale)) return fail(PKV_ERR_INVALID_ARGUMENT, "k_scale and v_scale must not be NULL");
    if (fp8 && (!aligned(k_scale, 4) || !aligned(v_scale, 4)))
        return fail(PKV_ERR_INVALID_ARGUMENT, "k_scale and v_scale must be 4-byte aligned");
    const bool fused = slots != nullptr;
    if (fused && (!k_new || !v_new)) return fail(PKV_ERR_INVALID_ARGUMENT, "k_new and v_new must not be NULL");
    if (fused && (!aligned(k_new, 16) || !aligned(v_new, 16)))
        return fail(PKV_ERR_INVALID_ARGUMENT, "k_new and v_new must be 16-byte aligned");
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !workspace)
        return fail(PKV_ERR_INVALID_ARGUMENT, "a required pointer is NULL");
    if (num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || max_blocks_per_seq <= 0 ||
        num_blocks <= 0)
        return fail(PKV_ERR_INVALID_ARGUMENT, "head counts, head_dim, block_size, max_blocks_per_seq and "
                                              "num_blocks must be positive");
    if (num_q_heads % num_kv_heads != 0)
        return fail(PKV_ERR_INVALID_ARGUMENT, "num_q_heads %d is not a multiple of num_kv_heads %d", num_q_heads,
                    num_kv_heads);
    if (!std::isfinite(scale)) return fail(PKV_ERR_INVALID_ARGUMENT, "scale is not finite");
    const int group = num_q_heads / num_kv_heads;
    if (head_dim != 64 && head_dim != 128)
        return fail(PKV_ERR_UNSUPPORTED, "head_dim %d not supported (64 or 128)", head_dim);
    if (block_size != 16 && block_size != 32)
        return fail(PKV_ERR_UNSUPPORTED, "block_size %d not supported (16 or 32)", block_size);
    if (group > PKV_MAX_GROUP)
        return fail(PKV_ERR_UNSUPPORTED, "num_q_heads / num_kv_heads = %d exceeds %d", group, PKV_MAX_GROUP);
    if (static_cast<int64_t>(num_blocks) * block_size > 0x7fffffff ||
        static_cast<int64_t>(max_blocks_per_seq) * block_size > 0x7fffffff)
        return fail(PKV_ERR_INVALID_ARGUMENT, "pool or table too large: blocks * block_size must be < 2^31");
    if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(workspace, 256))
        return fail(PKV_ERR_INVALID_ARGUMENT,
                    "out, q, k_cache and v_cache must be 16-byte aligned and workspace 256-byte aligned");
    pkv_decode_options o = {0, 0, 0, 0, 0, 0, 0, 0, nullptr, 0};
    if (opts) o = *opts;
    if (o.num_ctas < 0 || o.num_stages < 0 || o.ctas_per_sm < 0 || o.math < 0 || o.math > 2 ||
        o.l2_prefetch < -1 || o.l2_prefetch > 32 || o.piece_cost < -1 || o.piece_cost > 64 || o.head_pack < 0 ||
        o.head_pack > 2 || (o.tile_tokens != 0 && o.tile_tokens != 16 && o.tile_tokens != 32) || o.prefix_tiles < 0 ||
        o.prefix_tiles > 4096)
        return fail(PKV_ERR_INVALID_ARGUMENT, "negative or unknown option");
    if (o.tile_tokens > block_size)
        return fail(PKV_ERR_INVALID_ARGUMENT, "tile_tokens %d exceeds block_size %d", o.tile_tokens, block_size);
    if (o.num_ctas > pkv::kMaxCtas)
        return fail(PKV_ERR_INVALID_ARGUMENT, "num_ctas %d exceeds %d", o.num_ctas, pkv::kMaxCtas);
    if (static_cast<int64_t>(num_kv_heads) * (max_blocks_per_seq + 64) * pkv::kMaxSeqsPerLaunch > 0x7fffffff)
        return fail(PKV_ERR_INVALID_ARGUMENT, "num_kv_heads * max_blocks_per_seq too large");
    if (fp8 && o.math == pkv::kMathCudaCore)
        return fail(PKV_ERR_UNSUPPORTED, "e4m3 pools are decoded on tensor cores only (math 0 or 2)");
    const int math = fp8 ? pkv::kMathFp8 : o.math ? o.math : pkv::kMathTensorCore;
    const pkv_prefix_groups *pg = o.prefix_groups;
    if (pg && pg->num_groups < 0) return fail(PKV_ERR_INVALID_ARGUMENT, "prefix_groups.num_groups < 0");
    if (pg && pg->num_groups > 0) {
        if (!pg->begin || !pg->end || !pg->blocks)
            return fail(PKV_ERR_INVALID_ARGUMENT, "prefix_groups arrays are NULL");
        for (int g = 0; g < pg->num_groups; ++g) {
            if (pg->begin[g] < (g ? pg->end[g - 1] : 0) || pg->end[g] < pg->begin[g] + 2 || pg->end[g] > num_seqs)
                return fail(PKV_ERR_INVALID_ARGUMENT,
                            "prefix group %d [%d, %d): groups need two or more members, in order, within num_seqs", g,
                            pg->begin[g], pg->end[g]);
            if (pg->blocks[g] < 1 || pg->blocks[g] > max_blocks_per_seq)
                return fail(PKV_ERR_INVALID_ARGUMENT, "prefix_groups.blocks[%d] = %d outside [1, %d]", g,
                            pg->blocks[g], max_blocks_per_seq);
        }
        if (math != pkv::kMathTensorCore)
            return fail(PKV_ERR_UNSUPPORTED, "prefix groups need bf16 pools on tensor cores (math 0 or 2)");
        if (o.head_pack == 2) return fail(PKV_ERR_UNSUPPORTED, "prefix groups are decoded without head packing");
        if (o.tile_tokens == 32) return fail(PKV_ERR_UNSUPPORTED, "prefix groups are read in 16-row tiles");
    } else {
        pg = nullptr;
    }
    // Head packing: kv heads 2h, 2h + 1 of head_dim 64 read as one head of 128
    // (256-byte rows instead of 128-byte ones; for e4m3 pools, 128-byte rows
    // instead of 64-byte ones); the kernel then sees half the kv heads, twice
    // the head_dim and twice the group.
    // For e4m3 pools head_dim 128 packs too: rows of 256 codes.
    const bool can_pack = math != pkv::kMathCudaCore && (head_dim == 64 || (fp8 && head_dim == 128)) &&
                          num_kv_heads % 2 == 0 && 2 * group <= PKV_MAX_GROUP;
    if (o.head_pack == 2 && !can_pack)
        return fail(PKV_ERR_UNSUPPORTED, "head_pack 2 needs tensor-core math, head_dim 64 (or 128 for e4m3 pools), an "
                                         "even num_kv_heads and num_q_heads / num_kv_heads <= %d", PKV_MAX_GROUP / 2);
    const int pack = o.head_pack == 1 || pg ? 1 : can_pack ? 2 : 1;
    if (fp8 && head_dim == 64 && pack != 2)
        return fail(PKV_ERR_UNSUPPORTED, "e4m3 pools need head_dim 128, or head_dim 64 with head packing (an even "
                                         "num_kv_heads and num_q_heads / num_kv_heads <= %d)", PKV_MAX_GROUP / 2);
    const int kd = head_dim * pack, khkv = num_kv_heads / pack, kgroup = group * pack;  // as the kernel sees them
    // Tiles of 16 token rows by default: a 32-token block is read as two tiles,
    // so that a CTA's stages are as small as for 16-token blocks and as many
    // CTAs fit on an SM.
    const int tile = o.tile_tokens ? o.tile_tokens : 16;
    const int ns = o.num_stages ? o.num_stages : default_stages(kd, tile, math);
    if (ns < 1 || ns > pkv::kMaxStagesPerWarp)
        return fail(PKV_ERR_INVALID_ARGUMENT, "num_stages %d outside [1, %d]", ns, pkv::kMaxStagesPerWarp);
    const int gp = group_pad(kgroup);
    if (!pkv::decode_variant_exists(kd, tile, gp, math))
        return fail(PKV_ERR_UNSUPPORTED, "no kernel for head_dim %d, block_size %d, group %d, math %d", head_dim,
                    block_size, group, math);
    const WorkspaceLayout wl = workspace_layout(num_seqs, num_q_heads, head_dim);
    const size_t need = wl.total;
    int rc = PKV_OK;
    if (workspace_bytes < need)
        return fail(PKV_ERR_INVALID_ARGUMENT, "workspace_bytes %zu < required %zu", workspace_bytes, need);
    if (num_seqs == 0) return ok();

    CUtensorMap tm_k, tm_v;
    const int es = fp8 ? 1 : 2;
    if ((rc = make_pool_map(&tm_k, k_cache, num_blocks, block_size, khkv, kd, es, tile)) != PKV_OK) return rc;
    if ((rc = make_pool_map(&tm_v, v_cache, num_blocks, block_size, khkv, kd, es, tile)) != PKV_OK) return rc;

    uint8_t *ws = static_cast<uint8_t *>(workspace);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int sms = sm_count();
    if (sms <= 0) return fail(PKV_ERR_CUDA, "no CUDA device");

    // Sequences go in launches of at most kMaxSeqsPerLaunch (their tables live
    // in shared memory); launches run in stream order and reuse the workspace.
    for (int s0 = 0; s0 < num_seqs; s0 += pkv::kMaxSeqsPerLaunch) {
        const int sc = num_seqs - s0 < pkv::kMaxSeqsPerLaunch ? num_seqs - s0 : pkv::kMaxSeqsPerLaunch;
        // a launch that may have prefix groups is sized for the kernel with the
        // prefix units (its shared memory can be larger)
        bool may_group = false;
        for (int g = 0; pg && g < pg->num_groups; ++g) {
            const int lo = pg->begin[g] > s0 ? pg->begin[g] : s0;
            const int hi = pg->end[g] < s0 + sc ? pg->end[g] : s0 + sc;
            may_group |= hi - lo >= 2;
        }
        const int gmath = may_group ? pkv::kMathTensorCoreGroups : math;
        const size_t smem = pkv::decode_smem_bytes(kd, tile, gp, kgroup, gmath, ns, sc, pack);
        int per_sm = 0;
        cudaError_t e = pkv::decode_prepare(kd, tile, gp, gmath, smem, &per_sm);
        if (e != cudaSuccess) return cuda_fail(e, "decode kernel setup");
        if (per_sm <= 0) return fail(PKV_ERR_INVALID_ARGUMENT, "shared memory %zu bytes per CTA does not fit", smem);
        const int resident = sms * per_sm;  // CTAs that fit on the device at once
        if (o.ctas_per_sm > 0 && o.ctas_per_sm < per_sm) per_sm = o.ctas_per_sm;
        int grid = o.num_ctas > 0 ? o.num_ctas : sms * per_sm;
        if (grid > pkv::kMaxCtas) grid = pkv::kMaxCtas;
        const int pcost_default = fp8 ? (group > 4 ? kDefaultPieceCostFp8WideGroup : kDefaultPieceCostFp8)
                                  : group > 4 ? kDefaultPieceCostWideGroup
                                  : pack == 2 ? kDefaultPieceCostPacked
                                              : kDefaultPieceCost;
        const int pcost = o.piece_cost > 0 ? o.piece_cost : o.piece_cost == 0 ? pcost_default : 0;
        // A batch too small to give every CTA kMinCtaWeight tiles of weight runs
        // on fewer CTAs (the weight is bounded from above by the table width:
        // the lengths stay on the device). A CTA's warps take several tiles at
        // once, so smaller pieces finish no sooner, and every cut costs a merge.
        if (o.num_ctas <= 0 && !may_group) {
            const long long wmax = static_cast<long long>(khkv) * sc *
                                   (static_cast<long long>(max_blocks_per_seq) * (block_size / tile) + pcost);
            const long long want = (wmax + kMinCtaWeight - 1) / kMinCtaWeight;
            if (want < grid) grid = want < 1 ? 1 : static_cast<int>(want);
        }
        // the kernel with prefix units is launched cooperatively (its CTAs wait
        // for one another's pieces): no more CTAs than fit at once
        if (may_group && grid > resident) grid = resident;
        pkv::DecodeArgs a{};
        a.out = static_cast<__nv_bfloat16 *>(out) + static_cast<size_t>(s0) * num_q_heads * head_dim;
        a.q = static_cast<const __nv_bfloat16 *>(q) + static_cast<size_t>(s0) * num_q_heads * head_dim;
        a.block_tables = block_tables + static_cast<size_t>(s0) * max_blocks_per_seq;
        a.context_lens = context_lens + s0;
        a.o_part = reinterpret_cast<float *>(ws + wl.o_part);
        a.lse_part = reinterpret_cast<float *>(ws + wl.lse_part);
        a.seg_count = reinterpret_cast<unsigned long long *>(ws + wl.seg_count);
        a.launch_epoch = reinterpret_cast<unsigned long long *>(ws + pkv::kLaunchCounterOffset);
        a.ctas_started = reinterpret_cast<unsigned int *>(ws + pkv::kLaunchCounterOffset + 8);
        a.status = reinterpret_cast<int32_t *>(ws);
        a.num_seqs = sc;
        a.num_q_heads = num_q_heads;
        a.num_kv_heads = khkv;
        a.group = kgroup;
        a.pack = pack;
        a.sub = block_size / tile;
        a.max_blocks_per_seq = max_blocks_per_seq;
        a.num_blocks = num_blocks;
        a.num_stages = ns;
        a.prefetch = o.l2_prefetch > 0 ? o.l2_prefetch : o.l2_prefetch == 0 ? kDefaultL2Prefetch : 0;
        a.piece_cost = pcost;
        a.scale_log2 = scale * 1.4426950408889634f;
        plan_prefix_groups(may_group ? pg : nullptr, s0, sc, khkv, kgroup, a.sub, grid, max_blocks_per_seq,
                           o.prefix_tiles, a);
        // a launch whose groups were planned runs the kernel with the prefix
        // units; one whose groups were dropped runs the plain kernel in the
        // same shared memory and grid
        const int kmath = a.num_groups > 0 ? pkv::kMathTensorCoreGroups : math;
        if (kmath != gmath) {
            int per_sm_b = 0;
            e = pkv::decode_prepare(kd, tile, gp, kmath, smem, &per_sm_b);
            if (e != cudaSuccess) return cuda_fail(e, "decode kernel setup");
            if (per_sm_b < per_sm) return fail(PKV_ERR_CUDA, "the decode kernel fits fewer CTAs per SM");
        }
        if (fused) {
            const size_t row = static_cast<size_t>(num_kv_heads) * head_dim;  // elements per token
            a.k_new = static_cast<const __nv_bfloat16 *>(k_new) + static_cast<size_t>(s0) * row;
            a.v_new = static_cast<const __nv_bfloat16 *>(v_new) + static_cast<size_t>(s0) * row;
            a.slots = slots + s0;
            a.k_cache = const_cast<void *>(k_cache);
            a.v_cache = const_cast<void *>(v_cache);
        }
        a.k_scale = k_scale;
        a.v_scale = v_scale;
        e = pkv::decode_launch(kd, tile, gp, kmath, tm_k, tm_v, a, grid, smem, st);
        if (e != cudaSuccess) return cuda_fail(e, "decode kernel launch");
    }
    return ok();
}

}  // namespace

extern "C" {

int paged_attn_decode_ex(void *out, const void *q, const void *k_cache, const void *v_cache,
                         const int32_t *block_tables, const int32_t *context_lens, int num_seqs, int num_q_heads,
                         int num_kv_heads, int head_dim, int block_size, float scale, int max_blocks_per_seq,
                         int num_blocks, void *workspace, size_t workspace_bytes, const pkv_decode_options *opts,
                         void *stream) {
    return decode_impl(out, q, nullptr, nullptr, nullptr, k_cache, v_cache, nullptr, nullptr, block_tables,
                       context_lens, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, scale,
                       max_blocks_per_seq, num_blocks, workspace, workspace_bytes, opts, stream);
}

int paged_attn_decode_fp8(void *out, const void *q, const void *k_cache, const void *v_cache, const float *k_scale,
                          const float *v_scale, const int32_t *block_tables, const int32_t *context_lens,
                          int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size, float scale,
                          int max_blocks_per_seq, int num_blocks, void *workspace, size_t workspace_bytes,
                          const pkv_decode_options *opts, void *stream) {
    if (!k_scale || !v_scale) return fail(PKV_ERR_INVALID_ARGUMENT, "k_scale and v_scale must not be NULL");
    return decode_impl(out, q, nullptr, nullptr, nullptr, k_cache, v_cache, k_scale, v_scale, block_tables,
                       context_lens, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, scale,
                       max_blocks_per_seq, num_blocks, workspace, workspace_bytes, opts, stream);
}

int paged_attn_decode_append_fp8(void *out, const void *q, const void *k_new, const void *v_new,
                                 const int64_t *slot_mapping, void *k_cache, void *v_cache, const float *k_scale,
                                 const float *v_scale, const int32_t *block_tables, const int32_t *context_lens,
                                 int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                 float scale, int max_blocks_per_seq, int num_blocks, void *workspace,
                                 size_t workspace_bytes, const pkv_decode_options *opts, void *stream) {
    if (!slot_mapping) return fail(PKV_ERR_INVALID_ARGUMENT, "slot_mapping must not be NULL");
    if (!k_scale || !v_scale) return fail(PKV_ERR_INVALID_ARGUMENT, "k_scale and v_scale must not be NULL");
    return decode_impl(out, q, k_new, v_new, slot_mapping, k_cache, v_cache, k_scale, v_scale, block_tables,
                       context_lens, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, scale,
                       max_blocks_per_seq, num_blocks, workspace, workspace_bytes, opts, stream);
}

int paged_attn_decode_append(void *out, const void *q, const void *k_new, const void *v_new,
                             const int64_t *slot_mapping, void *k_cache, void *v_cache,
                             const int32_t *block_tables, const int32_t *context_lens, int num_seqs, int num_q_heads,
                             int num_kv_heads, int head_dim, int block_size, float scale, int max_blocks_per_seq,
                             int num_blocks, void *workspace, size_t workspace_bytes,
                             const pkv_decode_options *opts, void *stream) {
    if (!slot_mapping) return fail(PKV_ERR_INVALID_ARGUMENT, "slot_mapping must not be NULL");
    return decode_impl(out, q, k_new, v_new, slot_mapping, k_cache, v_cache, nullptr, nullptr, block_tables,
                       context_lens, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, scale,
                       max_blocks_per_seq, num_blocks, workspace, workspace_bytes, opts, stream);
}

int paged_attn_decode(void *out, const void *q, const void *k_cache, const void *v_cache,
                      const int32_t *block_tables, const int32_t *context_lens, int num_seqs, int num_q_heads,
                      int num_kv_heads, int head_dim, int block_size, float scale, int max_blocks_per_seq,
                      int num_blocks, void *workspace, size_t workspace_bytes, void *stream) {
    return paged_attn_decode_ex(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs, num_q_heads,
                                num_kv_heads, head_dim, block_size, scale, max_blocks_per_seq, num_blocks, workspace,
                                workspace_bytes, nullptr, stream);
}

int kv_cache_append(const void *k, const void *v, void *k_cache, void *v_cache, const int64_t *slot_mapping,
                    int num_tokens, int num_kv_heads, int head_dim, int block_size, int num_blocks, int32_t *d_status,
                    void *stream) {
    if (num_tokens < 0) return fail(PKV_ERR_INVALID_ARGUMENT, "num_tokens < 0");
    if (!k || !v || !k_cache || !v_cache || !slot_mapping)
        return fail(PKV_ERR_INVALID_ARGUMENT, "a required pointer is NULL");
    if (num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
        return fail(PKV_ERR_INVALID_ARGUMENT, "num_kv_heads, head_dim, block_size and num_blocks must be positive");
    if (head_dim % 8 != 0) return fail(PKV_ERR_UNSUPPORTED, "head_dim %d is not a multiple of 8", head_dim);
    if (!aligned(k, 16) || !aligned(v, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16))
        return fail(PKV_ERR_INVALID_ARGUMENT, "k, v, k_cache and v_cache must be 16-byte aligned");
    if (d_status && !aligned(d_status, 4)) return fail(PKV_ERR_INVALID_ARGUMENT, "d_status misaligned");
    if (num_tokens == 0) return ok();
    cudaError_t e = pkv::append_launch(k, v, k_cache, v_cache, slot_mapping, num_tokens, num_kv_heads, head_dim,
                                       block_size, num_blocks, d_status, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "append launch");
    return ok();
}

int paged_attn_prefill(void *out, const void *q, const void *k_cache, const void *v_cache,
                       const int32_t *block_tables, const int32_t *context_lens, const int32_t *query_start,
                       int num_seqs, int num_tokens, int max_query_len, int num_q_heads, int num_kv_heads,
                       int head_dim, int block_size, float scale, int max_blocks_per_seq, int num_blocks,
                       int32_t *d_status, void *stream) {
    return paged_attn_prefill_ex(out, q, k_cache, v_cache, block_tables, context_lens, query_start, num_seqs,
                                 num_tokens, max_query_len, num_q_heads, num_kv_heads, head_dim, block_size, scale,
                                 max_blocks_per_seq, num_blocks, d_status, 0, stream);
}

int paged_attn_prefill_ex(void *out, const void *q, const void *k_cache, const void *v_cache,
                          const int32_t *block_tables, const int32_t *context_lens, const int32_t *query_start,
                          int num_seqs, int num_tokens, int max_query_len, int num_q_heads, int num_kv_heads,
                          int head_dim, int block_size, float scale, int max_blocks_per_seq, int num_blocks,
                          int32_t *d_status, int kernel, void *stream) {
    if (kernel < 0 || kernel > 2) return fail(PKV_ERR_INVALID_ARGUMENT, "kernel must be 0, 1 or 2");
    if (num_seqs < 0 || num_tokens < 0 || max_query_len < 0)
        return fail(PKV_ERR_INVALID_ARGUMENT, "num_seqs, num_tokens and max_query_len must be >= 0");
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !query_start || !d_status)
        return fail(PKV_ERR_INVALID_ARGUMENT, "a required pointer is NULL");
    if (num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || max_blocks_per_seq <= 0 ||
        num_blocks <= 0)
        return fail(PKV_ERR_INVALID_ARGUMENT, "head counts, head_dim, block_size, max_blocks_per_seq and "
                                              "num_blocks must be positive");
    if (num_q_heads % num_kv_heads != 0)
        return fail(PKV_ERR_INVALID_ARGUMENT, "num_q_heads %d is not a multiple of num_kv_heads %d", num_q_heads,
                    num_kv_heads);
    if (!std::isfinite(scale)) return fail(PKV_ERR_INVALID_ARGUMENT, "scale is not finite");
    const int group = num_q_heads / num_kv_heads;
    if (head_dim != 64 && head_dim != 128)
        return fail(PKV_ERR_UNSUPPORTED, "head_dim %d not supported (64 or 128)", head_dim);
    if (block_size != 16 && block_size != 32)
        return fail(PKV_ERR_UNSUPPORTED, "block_size %d not supported (16 or 32)", block_size);
    if (group > PKV_MAX_GROUP)
        return fail(PKV_ERR_UNSUPPORTED, "num_q_heads / num_kv_heads = %d exceeds %d", group, PKV_MAX_GROUP);
    if (static_cast<int64_t>(num_blocks) * block_size > 0x7fffffff ||
        static_cast<int64_t>(max_blocks_per_seq) * block_size > 0x7fffffff)
        return fail(PKV_ERR_INVALID_ARGUMENT, "pool or table too large: blocks * block_size must be < 2^31");
    if (num_seqs > 65535 || num_kv_heads > 65535)
        return fail(PKV_ERR_UNSUPPORTED, "at most 65535 sequences and kv heads per call");
    if (static_cast<int64_t>(num_tokens) * num_q_heads * head_dim > (int64_t(1) << 40))
        return fail(PKV_ERR_INVALID_ARGUMENT, "num_tokens too large");
    if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(d_status, 4))
        return fail(PKV_ERR_INVALID_ARGUMENT, "out, q, k_cache and v_cache must be 16-byte aligned");
    // tcgen05 kernel: 128 rows must be whole query tokens (group 1, 2, 4, 8)
    const size_t smem_tc = pkv::prefill_tc_smem_bytes(head_dim, max_blocks_per_seq);
    const bool tc_group = group == 1 || group == 2 || group == 4 || group == 8;
    const bool tc_ok = tc_group && smem_tc <= 227 * 1024;
    if (kernel == 2 && !tc_group)
        return fail(PKV_ERR_UNSUPPORTED, "the tcgen05 kernel needs num_q_heads / num_kv_heads in {1, 2, 4, 8}");
    if (kernel == 2 && !tc_ok)
        return fail(PKV_ERR_UNSUPPORTED, "the tcgen05 kernel needs %zu bytes of shared memory for max_blocks_per_seq %d",
                    smem_tc, max_blocks_per_seq);
    const bool use_tc = kernel == 2 || (kernel == 0 && tc_ok);
    const size_t smem = use_tc ? smem_tc : pkv::prefill_smem_bytes(head_dim, block_size, max_blocks_per_seq);
    if (smem > 227 * 1024)
        return fail(PKV_ERR_UNSUPPORTED, "max_blocks_per_seq %d needs %zu bytes of shared memory", max_blocks_per_seq,
                    smem);
    if (num_seqs == 0 || num_tokens == 0 || max_query_len == 0) return ok();
    const int rows_per_cta = use_tc ? pkv::prefill_tc_rows_per_cta() : pkv::prefill_rows_per_cta();
    const int64_t tiles = (static_cast<int64_t>(max_query_len) * group + rows_per_cta - 1) / rows_per_cta;
    if (tiles > 0x7fffffff) return fail(PKV_ERR_INVALID_ARGUMENT, "max_query_len too large");
    CUtensorMap tm_k, tm_v;
    int rc;
    if ((rc = make_pool_map(&tm_k, k_cache, num_blocks, block_size, num_kv_heads, head_dim)) != PKV_OK) return rc;
    if ((rc = make_pool_map(&tm_v, v_cache, num_blocks, block_size, num_kv_heads, head_dim)) != PKV_OK) return rc;
    pkv::PrefillArgs a{};
    a.out = out;
    a.q = q;
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    a.query_start = query_start;
    a.status = d_status;
    a.num_seqs = num_seqs;
    a.num_tokens = num_tokens;
    a.num_q_heads = num_q_heads;
    a.num_kv_heads = num_kv_heads;
    a.group = group;
    a.max_blocks_per_seq = max_blocks_per_seq;
    a.num_blocks = num_blocks;
    a.max_query_len = max_query_len;
    a.scale_log2 = scale * 1.4426950408889634f;
    cudaError_t e;
    if (use_tc) {
        CUtensorMap tm_q;
        if ((rc = make_query_map(&tm_q, q, num_tokens, num_kv_heads, group, head_dim)) != PKV_OK) return rc;
        e = pkv::prefill_tc_launch(head_dim, block_size, tm_q, tm_k, tm_v, a, static_cast<int>(tiles), smem,
                                   static_cast<cudaStream_t>(stream));
    } else {
        e = pkv::prefill_launch(head_dim, block_size, tm_k, tm_v, a, static_cast<int>(tiles), smem,
                                static_cast<cudaStream_t>(stream));
    }
    if (e != cudaSuccess) return cuda_fail(e, "prefill launch");
    return ok();
}

int kv_cache_append_fp8(const void *k, const void *v, void *k_cache, void *v_cache, const int64_t *slot_mapping,
                        const float *k_scale, const float *v_scale, int num_tokens, int num_kv_heads, int head_dim,
                        int block_size, int num_blocks, int32_t *d_status, void *stream) {
    if (num_tokens < 0) return fail(PKV_ERR_INVALID_ARGUMENT, "num_tokens < 0");
    if (!k || !v || !k_cache || !v_cache || !slot_mapping || !k_scale || !v_scale)
        return fail(PKV_ERR_INVALID_ARGUMENT, "a required pointer is NULL");
    if (num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
        return fail(PKV_ERR_INVALID_ARGUMENT, "num_kv_heads, head_dim, block_size and num_blocks must be positive");
    if (head_dim % 16 != 0) return fail(PKV_ERR_UNSUPPORTED, "head_dim %d is not a multiple of 16", head_dim);
    if (!aligned(k, 16) || !aligned(v, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(k_scale, 4) || !aligned(v_scale, 4))
        return fail(PKV_ERR_INVALID_ARGUMENT, "k, v, k_cache and v_cache must be 16-byte aligned, scales 4-byte");
    if (d_status && !aligned(d_status, 4)) return fail(PKV_ERR_INVALID_ARGUMENT, "d_status misaligned");
    if (num_tokens == 0) return ok();
    cudaError_t e = pkv::append_fp8_launch(k, v, k_cache, v_cache, slot_mapping, k_scale, v_scale, num_tokens,
                                           num_kv_heads, head_dim, block_size, num_blocks, d_status,
                                           static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "append launch");
    return ok();
}

int kv_block_copy(void *k_cache, void *v_cache, const int32_t *src, const int32_t *dst, int num_copies,
                  int num_kv_heads, int head_dim, int elem_bytes, int block_size, int num_blocks, int32_t *d_status,
                  void *stream) {
    if (num_copies < 0) return fail(PKV_ERR_INVALID_ARGUMENT, "num_copies < 0");
    if (!k_cache || !v_cache || (num_copies > 0 && (!src || !dst)))
        return fail(PKV_ERR_INVALID_ARGUMENT, "a required pointer is NULL");
    if (num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
        return fail(PKV_ERR_INVALID_ARGUMENT, "num_kv_heads, head_dim, block_size and num_blocks must be positive");
    if (elem_bytes != 1 && elem_bytes != 2) return fail(PKV_ERR_INVALID_ARGUMENT, "elem_bytes must be 1 or 2");
    if ((head_dim * elem_bytes) % 16 != 0)
        return fail(PKV_ERR_UNSUPPORTED, "a row of head_dim %d is not a multiple of 16 bytes", head_dim);
    if (!aligned(k_cache, 16) || !aligned(v_cache, 16))
        return fail(PKV_ERR_INVALID_ARGUMENT, "k_cache and v_cache must be 16-byte aligned");
    if (d_status && !aligned(d_status, 4)) return fail(PKV_ERR_INVALID_ARGUMENT, "d_status misaligned");
    if (num_copies == 0) return ok();
    cudaError_t e = pkv::block_copy_launch(k_cache, v_cache, src, dst, num_copies, block_size, num_kv_heads,
                                           head_dim * elem_bytes, num_blocks, d_status,
                                           static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "block copy launch");
    return ok();
}

int pkv_validate(const int32_t *block_tables, const int32_t *context_lens, int num_seqs, int max_blocks_per_seq,
                 int block_size, int num_blocks, int32_t *d_status, void *stream) {
    if (num_seqs < 0) return fail(PKV_ERR_INVALID_ARGUMENT, "num_seqs < 0");
    if (!block_tables || !context_lens || !d_status) return fail(PKV_ERR_INVALID_ARGUMENT, "a pointer is NULL");
    if (max_blocks_per_seq <= 0 || block_size <= 0 || num_blocks <= 0)
        return fail(PKV_ERR_INVALID_ARGUMENT, "sizes must be positive");
    if (num_seqs == 0) return ok();
    cudaError_t e = pkv::validate_launch(block_tables, context_lens, num_seqs, max_blocks_per_seq, block_size,
                                         num_blocks, d_status, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "validate launch");
    return ok();
}

int pkv_read_status(int32_t *d_status, int32_t *status, int clear, void *stream) {
    if (!d_status || !status) return fail(PKV_ERR_INVALID_ARGUMENT, "a pointer is NULL");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(status, d_status, sizeof(int32_t), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess && clear) e = cudaMemsetAsync(d_status, 0, sizeof(int32_t), st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "status read");
    return ok();
}

int pkv_selftest_bounded_wait(int32_t *d_status, void *stream) {
    if (!d_status) return fail(PKV_ERR_INVALID_ARGUMENT, "d_status is NULL");
    cudaError_t e = pkv::selftest_bounded_wait_launch(d_status, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
    return ok();
}

}  // extern "C"

// ---------------------------------------------------------------------------
// paged_attn_decode_noalloc: decode for callers that cannot allocate device
// memory. Its scratch (status word + split partials, the layout of the decode
// workspace) is this file-scope device array, sized PKV_NOALLOC_SCRATCH_BYTES;
// every GPU that loads the library holds it until the process exits.
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[PKV_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
std::vector<void *> g_noalloc_ptr;  // device address of g_noalloc_scratch, per device

// In host code g_noalloc_scratch names a host-side stand-in, not device memory:
// the kernels get the address cudaGetSymbolAddress returns for the current
// device, looked up on the first call on that device and cached for the life
// of the process (a device reset, which would move the array, is not followed).
int noalloc_scratch(void **ptr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (dev >= static_cast<int>(g_noalloc_ptr.size())) g_noalloc_ptr.resize(dev + 1, nullptr);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the static decode scratch");
        g_noalloc_ptr[dev] = p;
    }
    *ptr = g_noalloc_ptr[dev];
    return PKV_OK;
}

}  // namespace

extern "C" int paged_attn_decode_noalloc(void *out, const void *q, const void *k_cache, const void *v_cache,
                                         const int32_t *block_tables, const int32_t *context_lens, int num_seqs,
                                         int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                         float scale, int max_blocks_per_seq, int num_blocks, int32_t *d_status,
                                         void *stream) {
    size_t need = 0;
    int rc = pkv_decode_workspace_bytes(num_seqs, num_q_heads, head_dim, &need);
    if (rc != PKV_OK) return rc;
    if (need > PKV_NOALLOC_SCRATCH_BYTES)
        return fail(PKV_ERR_INVALID_ARGUMENT,
                    "this batch needs %zu bytes of decode scratch but the static scratch of "
                    "paged_attn_decode_noalloc holds %u; decode it in smaller batches or use paged_attn_decode "
                    "with a caller-allocated workspace",
                    need, static_cast<unsigned>(PKV_NOALLOC_SCRATCH_BYTES));
    if (d_status && !aligned(d_status, 4)) return fail(PKV_ERR_INVALID_ARGUMENT, "d_status misaligned");
    void *scratch = nullptr;
    if ((rc = noalloc_scratch(&scratch)) != PKV_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // The scratch keeps the previous call's contents: zero its status word so
    // this call reports only its own problems. The launch counter after it
    // and the partials need no clearing (every partial that is read was
    // written earlier in the same call).
    cudaError_t e = cudaMemsetAsync(scratch, 0, sizeof(int32_t), st);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the static scratch's status word");
    rc = paged_attn_decode_ex(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs, num_q_heads,
                              num_kv_heads, head_dim, block_size, scale, max_blocks_per_seq, num_blocks, scratch,
                              PKV_NOALLOC_SCRATCH_BYTES, nullptr, stream);
    if (rc != PKV_OK) return rc;
    if (d_status) {
        e = cudaMemcpyAsync(d_status, scratch, sizeof(int32_t), cudaMemcpyDeviceToDevice, st);
        if (e != cudaSuccess) return cuda_fail(e, "copying the status word");
    }
    return ok();
}
