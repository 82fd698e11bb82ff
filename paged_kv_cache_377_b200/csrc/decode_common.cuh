// decode_common.cuh -- launch-shape constants and the shared-memory layout of the
// paged decode kernel, used by both the kernel and its host launcher.
#pragma once

#include <stdint.h>

namespace pkv {

constexpr int kConsumerWarps = 4;                     // warps of a decode CTA (each loads and computes)
constexpr int kDecodeThreads = 32 * kConsumerWarps;
constexpr int kMaxStages = 16;                        // KV-block stages per CTA (4 warps x up to 4 each)
constexpr int kMaxStagesPerWarp = kMaxStages / kConsumerWarps;
constexpr int kMaxSeqsPerLaunch = 2048;               // per-sequence tables kept in shared memory
constexpr int kMaxCtas = 1024;                        // grid limit; bounds the pieces of a launch
constexpr int kWorkspaceHeaderBytes = 256;
constexpr int kLaunchCounterOffset = 8;               // header bytes [8, 16): launches so far; [16, 20): CTAs started
constexpr int kMaxPrefixGroups = 16;                  // prefix groups per launch (kernel parameters)
constexpr int kPrefixRows = 64;                       // query rows of one prefix unit: 16 per warp

// With pack = 2 the kernel runs on a view of the pool with half the kv heads
// and twice the head_dim: kv heads 2h', 2h' + 1 of head_dim D / 2 are the two
// halves of one 'virtual' head h' of head_dim D, and its 2G query rows are the
// real query heads of both (query row p G + g sees only half p). num_kv_heads,
// group and D below are then the virtual ones; q, out and the partials keep the
// real head_dim D / pack per row.
struct DecodeArgs {
    void *out;                   // bf16 [S][Hq][D / pack]
    const void *q;               // bf16 [S][Hq][D / pack]
    const int32_t *block_tables; // [S][MB]
    const int32_t *context_lens; // [S]
    float *o_part;               // fp32 [piece][G][D / pack], piece = s * Hkv + h + cta
    float *lse_part;             // fp32 [piece][G], log2 domain
    unsigned long long *seg_count;  // [S * Hkv] (launch epoch << 16 | pieces stored), per segment
    // Workspace header words: the launches of this workspace so far (the
    // epoch that tags the counters) and the CTAs of the current launch that
    // have read it. CTA 0 advances the epoch at its end, once all have, so
    // each launch -- a CUDA graph's replays included -- has its own and the
    // counters never need clearing.
    unsigned long long *launch_epoch;
    unsigned int *ctas_started;
    int32_t *status;             // device status word
    int num_seqs;
    int num_q_heads;
    int num_kv_heads;
    int group;                   // Hq / Hkv
    int max_blocks_per_seq;
    int num_blocks;
    int num_stages;              // ring stages per warp (R); the CTA holds 4R
    int prefetch;                // blocks a warp prefetches into L2 beyond the one it loads (0 = none)
    int piece_cost;              // extra weight, in blocks, of every non-empty segment when splitting work
    int pack;                    // 1, or 2: two real kv heads per virtual head (see above)
    int sub;                     // tiles per pool block: 1, or 2 (a 32-token block read as two 16-token tiles)
    // Fused append (slots != nullptr): the step's new token of sequence s, rows
    // k_new[s][h] / v_new[s][h] ([S][Hkv][D] like a pool row), belongs at
    // slots[s], which must be the slot of position L_s - 1. The warp that
    // computes that block puts the rows into its staged tile (so attention
    // sees them) and writes them to the pool.
    const void *k_new;
    const void *v_new;
    const int64_t *slots;
    void *k_cache;               // pool [NB][BS][Hkv][D] (bf16, or e4m3 codes), written by the fused append
    void *v_cache;
    // e4m3 pools: fp32 scale per REAL kv head (element = e4m3(code) * scale); the
    // fused append stores e4m3(rn, satfinite)(x / scale) computed in fp32.
    const float *k_scale;
    const float *v_scale;
    float scale_log2;            // scale * log2(e): logits are kept in base 2
    // Prefix groups (bf16 pools, pack 1, tensor cores). Group g is the
    // sequences grp_begin[g] .. grp_end[g] - 1 of the launch, whose
    // tables agree on the blocks of their first grp_tiles[g] tiles; those tiles
    // are read once per group by prefix units, the rest of each context (its
    // suffix) as usual. CTAs [0, prefix_ctas) run one prefix unit each: the
    // members of row tile rt (grp_members[g] per row tile) and kv head h against
    // prefix piece tp (tiles_per_piece tiles), unit index grp_unit0[g] + (h *
    // grp_row_tiles[g] + rt) * pieces + tp. Their partials take rows (pre_base +
    // (s * Hkv + h) * prefix_np + tp) * G + g of o_part / lse_part.
    int num_groups;
    int prefix_ctas;
    int tiles_per_piece;
    int prefix_np;
    int pre_base;
    int grp_begin[kMaxPrefixGroups];
    int grp_end[kMaxPrefixGroups];
    int grp_tiles[kMaxPrefixGroups];
    int grp_unit0[kMaxPrefixGroups + 1];
    int grp_members[kMaxPrefixGroups];
    int grp_row_tiles[kMaxPrefixGroups];
};

struct DecodeLayout {
    uint32_t stages, qbuf, pscr, merge_acc, merge_m, merge_l, bars, flags, prefix, wprefix, lens, ptiles, prefix_q,
        total;
};

__host__ __device__ inline uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

// Byte offsets from a 1024-byte aligned base. `total` includes 1024 bytes of
// slack for aligning the dynamic shared-memory base. GP = compile-time padded
// group, G = the actual group (query heads per kv head), tensor_core = the
// mma.sync math path (its probability scratch is bf16 [8][BS] per warp).
// kv_elem_bytes = bytes per pool element; dr = dims per stored q / out row
// (D / pack). groups: the launch has prefix units, whose kPrefixRows query rows
// (bf16 [rows][D], 16-byte chunks XOR-swizzled by row) take the area of the
// query slots, probability scratch and merge area (unused by a prefix unit)
// when it is large enough, else an area of their own at the end.
__host__ __device__ inline DecodeLayout decode_layout(int D, int BS, int GP, int G, bool tensor_core, int num_stages,
                                                      int num_seqs, int kv_elem_bytes, int dr, bool groups = false) {
    DecodeLayout L;
    uint32_t off = 0;
    const uint32_t tile = static_cast<uint32_t>(BS * D * kv_elem_bytes);
    L.stages = off;
    off += static_cast<uint32_t>(num_stages) * 2u * tile;          // [stage][K tile, V tile]
    L.qbuf = off;
    off += 2u * G * dr * 2;                                         // two query slots [G][dr] bf16
    off = align_up(off, 16);
    L.pscr = off;
    off += kConsumerWarps * (tensor_core ? BS * 16 : BS * GP * 8);  // per warp probabilities (16-bit [8][BS] on tensor cores)
    L.merge_acc = off;
    off += kConsumerWarps * G * dr * 4;                             // per warp fp32 [G][dr]
    L.merge_m = off;
    off += kConsumerWarps * G * 4;
    L.merge_l = off;
    off += kConsumerWarps * G * 4;
    off = align_up(off, 8);
    L.bars = off;
    off += (2 * kMaxStages + 3) * 8;                                // full[stage], qfull[2], empty[stage], epoch
    L.flags = off;
    off += (2 * kMaxStages + 1 + 2 * kConsumerWarps + 1 + 4 * 2) * 4;  // stage_bad, abort, scan, merges, stage_blk
    L.prefix = off;
    off += static_cast<uint32_t>(num_seqs + 1) * 4;                 // blocks before each sequence
    L.wprefix = off;
    off += static_cast<uint32_t>(num_seqs + 1) * 4;                 // weighted blocks before each sequence
    L.lens = off;
    off += static_cast<uint32_t>(num_seqs) * 4;                     // clamped context lengths
    L.ptiles = off;
    off += static_cast<uint32_t>(num_seqs) * 4;                     // shared-prefix tiles of each sequence (0: none)
    L.prefix_q = L.qbuf;
    if (groups && L.merge_l + kConsumerWarps * G * 4 - L.qbuf < static_cast<uint32_t>(kPrefixRows * D * 2)) {
        off = align_up(off, 128);
        L.prefix_q = off;
        off += kPrefixRows * D * 2;
    }
    L.total = align_up(off, 16) + 1024;
    return L;
}

}  // namespace pkv
