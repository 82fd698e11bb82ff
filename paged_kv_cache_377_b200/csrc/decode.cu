// decode.cu -- paged decode attention for sm_100a.
//
// What it computes: for every sequence s and query head j, softmax over the
// sequence's L_s cached tokens of scale * q.k, applied to the cached values --
// single-query attention whose keys and values are reached through the
// sequence's block table ("vLLM Fundamentals: Paged Attention and Batching",
// section "Paged Attention": the kernel follows the block table to gather the
// blocks; "Deep Dive into vLLM", section 2.1: logical -> physical blocks).
//
// How (design for B200; the pages describe no kernel):
//   * Work decomposition: the unit is one KV block of one (sequence, kv head)
//     "segment"; segments are ordered (sequence, head) and CTA c of C takes
//     the contiguous range [c B / C, (c + 1) B / C) of the B blocks of the
//     launch, so every CTA gets the same number of blocks (+-1) whatever the
//     length skew. A CTA's range crosses a few segments; each crossing is a
//     "piece". Every CTA rebuilds the per-sequence block prefix sums in shared
//     memory, so no planning kernel and no host/device synchronisation are
//     needed.
//   * Four warps per CTA take the blocks round-robin (block g of the CTA's
//     range goes to warp g % 4). Each warp owns a ring of R shared-memory
//     stages and streams its own blocks into it with TMA (4D tile copies of 64
//     columns, 128-byte swizzle), R blocks ahead of the one it computes and
//     across piece boundaries, completing on mbarriers; block-table entries
//     are looked up 32 blocks at a time, one batch ahead. No warp waits for
//     another to refill its stages, and each waiter sees every phase of its
//     barriers in order. Each warp keeps its own online-softmax state (running max m, running sum l, fp32 accumulator)
//     for all G query heads of the GQA group (Milakov & Gimelshein 2018,
//     "Online normalizer calculation for softmax"). Logits are kept in base 2
//     (scale * log2 e folded in).
//   * Two interchangeable math paths per block: CoreMath (fp32 FMA on CUDA
//     cores, packed f32x2) and MmaMath (bf16 tensor cores, mma.sync m16n8k16
//     with fp32 accumulation: S^T = K.Q^T with the block's tokens as M and the
//     G <= 8 query heads as N, then O^T += V^T.P^T).
//   * At the end of a piece the four warp states are merged in shared memory
//     with the log-sum-exp identity. A piece that is a whole segment writes
//     bf16 output directly; the pieces of a segment cut by CTA boundaries
//     write fp32 partials + log2-sum-exp, and the CTA that stores a segment's
//     last piece (a per-segment counter tagged with the launch's epoch, so it
//     never needs clearing) merges them in CTA order.
// Every reduction order depends only on logical token positions, so results
// are bitwise reproducible and independent of where blocks sit in the pool.
#include <cstdio>
#include <mutex>
#include <set>
#include <tuple>

#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "device_utils.cuh"
#include "launch.h"
#include "mma_utils.cuh"

namespace pkv {
namespace {

// A piece: blocks [b0, b1) of segment (s, h), processed by one CTA. L is the
// context length past the sequence's shared prefix (read by prefix units), so
// that block b of the segment holds positions b BS .. b BS + BS - 1 of those.
struct Piece {
    int s, h, b0, b1, L;
    bool whole;  // the piece is the entire segment (no merge needed)
};

// Walks the pieces of this CTA's block range [x, x1) in order. pre[s] holds
// the blocks of sequences < s; sequence s contributes Hkv segments of
// pre[s + 1] - pre[s] blocks each.
struct PieceIter {
    long long x, x1;
    const int *pre;
    const int *lens;
    const int *ptiles;
    int S, Hkv, BS;

    __device__ __forceinline__ bool next(Piece &pc) {
        if (x >= x1) return false;
        int lo = 0, hi = S - 1;
        while (lo < hi) {  // the sequence holding global block x
            const int mid = (lo + hi + 1) >> 1;
            if (static_cast<long long>(Hkv) * pre[mid] <= x) lo = mid;
            else hi = mid - 1;
        }
        const int n = pre[lo + 1] - pre[lo];
        const long long base = static_cast<long long>(Hkv) * pre[lo];
        const int r = static_cast<int>(x - base);
        const int h = r / n;
        const long long seg_end = base + static_cast<long long>(h + 1) * n;
        const long long end = x1 < seg_end ? x1 : seg_end;
        pc.s = lo;
        pc.h = h;
        pc.b0 = r - h * n;
        pc.b1 = pc.b0 + static_cast<int>(end - x);
        const int t0 = ptiles[lo];
        pc.L = lens[lo] - t0 * BS;
        pc.whole = pc.b0 == 0 && end == seg_end && t0 == 0;  // no prefix pieces to merge with
        x = end;
        return true;
    }
};

// Work is split between CTAs by weight: a non-empty segment of n blocks weighs
// n + piece_cost, its first piece_cost units standing for the fixed cost of a
// piece (query load, merge of the warps' states). CTA c takes the weight range
// [c W / C, (c + 1) W / C); its blocks are the real blocks whose weight
// position falls in that range -- a contiguous range of the launch's blocks.
// pre[s] / wpre[s] = blocks / weight of the sequences before s (per head).
// Returns the number of real blocks whose weight position is below v.
__device__ __forceinline__ long long blocks_below(long long v, const int *pre, const int *wpre, int S, int Hkv,
                                                  int piece_cost) {
    if (v >= static_cast<long long>(Hkv) * wpre[S]) return static_cast<long long>(Hkv) * pre[S];
    int lo = 0, hi = S - 1;
    while (lo < hi) {  // the sequence holding weight position v
        const int mid = (lo + hi + 1) >> 1;
        if (static_cast<long long>(Hkv) * wpre[mid] <= v) lo = mid;
        else hi = mid - 1;
    }
    const int w = wpre[lo + 1] - wpre[lo], n = pre[lo + 1] - pre[lo];
    const long long r = v - static_cast<long long>(Hkv) * wpre[lo];
    const int h = static_cast<int>(r / w), o = static_cast<int>(r - static_cast<long long>(h) * w);
    return static_cast<long long>(Hkv) * pre[lo] + static_cast<long long>(h) * n + max(0, o - piece_cost);
}

__device__ __forceinline__ long long weight_begin(int c, long long W, int C) { return static_cast<long long>(c) * W / C; }

// ------------------------------------------------------------------ CUDA-core math

// Reduce N partial sums across the LPT lanes of a token group (xor masks
// LPT/2 .. 1), halving the values a lane carries at each step: afterwards
// v[0] holds the full sum for query head g_own (see g_own_of()).
template <int N, int LPT>
__device__ __forceinline__ void transpose_reduce(float (&v)[N], int lane) {
    static_assert(N <= LPT, "more values than lanes");
    int mask = LPT / 2;
#pragma unroll
    for (int n = N; n > 1; n >>= 1) {
        const bool upper = (lane & mask) != 0;
#pragma unroll
        for (int i = 0; i < n / 2; ++i) {
            const float send = upper ? v[i] : v[i + n / 2];
            const float keep = upper ? v[i + n / 2] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
        }
        mask >>= 1;
    }
#pragma unroll
    for (; mask >= 1; mask >>= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], mask);
}

template <int N, int LPT>
__device__ __forceinline__ int g_own_of(int lane) {
    int g = 0, mask = LPT / 2;
#pragma unroll
    for (int n = N; n > 1; n >>= 1) {
        if (lane & mask) g += n >> 1;
        mask >>= 1;
    }
    return g;
}

// fp32 math on CUDA cores. A token group of LPT = D/8 lanes covers one row
// (8 dims per lane, one 16-byte chunk); a warp handles 32/LPT tokens per pass.
template <int D, int BS, int GP_>
struct CoreMath {
    static constexpr int GP = GP_;
    static constexpr int LPT = D / 8, TPP = 32 / LPT, NPASS = BS / TPP, LPG = 32 / GP;

    int lane, tg, ch, g_own;
    bool writer;
    float2 *pscr;  // this warp's float2 [BS][GP]: logits, then (p, p)
    float2 q2[GP][4];
    float m_run[GP];
    float l_run;
    float2 acc[GP][4];

    __device__ __forceinline__ void init(int warp, int lane_, uint8_t *base, const DecodeLayout &ly) {
        lane = lane_;
        tg = lane / LPT;
        ch = lane % LPT;
        g_own = g_own_of<GP, LPT>(lane);
        writer = (lane % (LPT / GP)) == 0;
        pscr = reinterpret_cast<float2 *>(base + ly.pscr) + warp * BS * GP;
    }

    // query rows of the GQA group, pre-scaled into base-2 logits
    __device__ __forceinline__ void load_q(uint32_t qslot, int group, float scale_log2, int /*pack: always 1 here*/,
                                           const DecodeArgs & /*a*/, int /*h*/) {
        const uint32_t qa = qslot + ch * 16;
        const float2 sc = make_float2(scale_log2, scale_log2);
#pragma unroll
        for (int g = 0; g < GP; ++g) {
            if (g < group) {
                const uint4 r = lds128(qa + g * D * 2);
                q2[g][0] = fmul2(bf16x2_to_float2(r.x), sc);
                q2[g][1] = fmul2(bf16x2_to_float2(r.y), sc);
                q2[g][2] = fmul2(bf16x2_to_float2(r.z), sc);
                q2[g][3] = fmul2(bf16x2_to_float2(r.w), sc);
            } else {
#pragma unroll
                for (int k = 0; k < 4; ++k) q2[g][k] = make_float2(0.f, 0.f);
            }
        }
    }

    __device__ __forceinline__ void reset() {
        l_run = 0.f;
#pragma unroll
        for (int g = 0; g < GP; ++g) {
            m_run[g] = -INFINITY;
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[g][k] = make_float2(0.f, 0.f);
        }
    }

    // One KV tile in two steps: qk() -- logits and the block-wise online-softmax
    // update, leaving the probabilities in the warp's scratch -- reads only the
    // K tile; pv() -- P.V -- only the V tile.
    __device__ __forceinline__ void qk(uint32_t ktile, int valid) {
#pragma unroll
        for (int pass = 0; pass < NPASS; ++pass) {
            const int t = pass * TPP + tg;
            const uint4 kr = lds128(tile_addr<BS>(ktile, t, ch));
            const float2 k0 = bf16x2_to_float2(kr.x), k1 = bf16x2_to_float2(kr.y);
            const float2 k2 = bf16x2_to_float2(kr.z), k3 = bf16x2_to_float2(kr.w);
            float part[GP];
#pragma unroll
            for (int g = 0; g < GP; ++g) {
                float2 s2 = fmul2(q2[g][0], k0);
                s2 = ffma2(q2[g][1], k1, s2);
                s2 = ffma2(q2[g][2], k2, s2);
                s2 = ffma2(q2[g][3], k3, s2);
                part[g] = s2.x + s2.y;
            }
            transpose_reduce<GP, LPT>(part, lane);
            // a token past the context is selected away (its row may hold anything)
            if (writer) pscr[t * GP + g_own].x = (t < valid) ? part[0] : -INFINITY;
        }
        __syncwarp();

        // block max per head, new running max, probabilities, running sum
        const int gs = lane % GP, ts = lane / GP;
        float mx = -INFINITY;
#pragma unroll
        for (int t = ts; t < BS; t += LPG) mx = fmaxf(mx, pscr[t * GP + gs].x);
#pragma unroll
        for (int o = GP; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float m_new[GP];
        bool grew = false;
        float m_own_old = m_run[0], m_own_new = 0.f;
#pragma unroll
        for (int g = 0; g < GP; ++g) {
            m_new[g] = fmaxf(m_run[g], __shfl_sync(0xffffffffu, mx, g));
            grew |= (m_new[g] != m_run[g]);
            if (g == gs) {
                m_own_old = m_run[g];
                m_own_new = m_new[g];
            }
        }
        float psum = 0.f;
#pragma unroll
        for (int t = ts; t < BS; t += LPG) {
            const float p = fast_exp2(pscr[t * GP + gs].x - m_own_new);
            pscr[t * GP + gs] = make_float2(p, p);
            psum += p;
        }
#pragma unroll
        for (int o = GP; o < 32; o <<= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
        l_run = l_run * fast_exp2(m_own_old - m_own_new) + psum;
        if (grew) {  // warp-uniform: m_run is replicated in every lane
#pragma unroll
            for (int g = 0; g < GP; ++g) {
                const float al = fast_exp2(m_run[g] - m_new[g]);
                const float2 a2 = make_float2(al, al);
#pragma unroll
                for (int k = 0; k < 4; ++k) acc[g][k] = fmul2(acc[g][k], a2);
                m_run[g] = m_new[g];
            }
        }
        __syncwarp();
    }

    __device__ __forceinline__ void block(uint32_t ktile, uint32_t vtile, int valid) {
        qk(ktile, valid);
        pv(vtile, valid);
    }

    __device__ __forceinline__ void pv(uint32_t vtile, int valid) {
        // P.V: tokens past the context are skipped, never multiplied by p = 0
#pragma unroll
        for (int pass = 0; pass < NPASS; ++pass) {
            const int t = pass * TPP + tg;
            const uint4 vr = lds128(tile_addr<BS>(vtile, t, ch));
            if (t < valid) {
                const float2 v0 = bf16x2_to_float2(vr.x), v1 = bf16x2_to_float2(vr.y);
                const float2 v2 = bf16x2_to_float2(vr.z), v3 = bf16x2_to_float2(vr.w);
#pragma unroll
                for (int g = 0; g < GP; ++g) {
                    const float2 p = pscr[t * GP + g];
                    acc[g][0] = ffma2(p, v0, acc[g][0]);
                    acc[g][1] = ffma2(p, v1, acc[g][1]);
                    acc[g][2] = ffma2(p, v2, acc[g][2]);
                    acc[g][3] = ffma2(p, v3, acc[g][3]);
                }
            }
        }
        __syncwarp();
    }

    // This warp's (m, l, acc) into the merge area ([warp][G][D], [warp][G]).
    __device__ __forceinline__ void export_state(float *merge_acc, float *merge_m, float *merge_l, int warp, int G,
                                                 int /*pack: always 1 here*/) {
        // token groups of a warp share m_run: their accumulators just add
#pragma unroll
        for (int o = LPT; o < 32; o <<= 1)
#pragma unroll
            for (int g = 0; g < GP; ++g)
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    acc[g][k].x += __shfl_xor_sync(0xffffffffu, acc[g][k].x, o);
                    acc[g][k].y += __shfl_xor_sync(0xffffffffu, acc[g][k].y, o);
                }
        if (tg == 0) {
#pragma unroll
            for (int g = 0; g < GP; ++g) {
                if (g < G) {
                    float4 *dst = reinterpret_cast<float4 *>(merge_acc + (warp * G + g) * D + ch * 8);
                    dst[0] = make_float4(acc[g][0].x, acc[g][0].y, acc[g][1].x, acc[g][1].y);
                    dst[1] = make_float4(acc[g][2].x, acc[g][2].y, acc[g][3].x, acc[g][3].y);
                }
            }
        }
        if (lane == 0) {
#pragma unroll
            for (int g = 0; g < GP; ++g)
                if (g < G) merge_m[warp * G + g] = m_run[g];
        }
        if (lane < G) merge_l[warp * G + lane] = l_run;
    }
};

// ------------------------------------------------------------------ tensor-core math

// bf16 tensor-core math (mma.sync m16n8k16, fp32 accumulate). Per block:
//   S^T[t][g] = K[t][:] . q[g][:]   tokens t as M (16 per tile), heads g as N = 8
//   O^T[d][g] += V[t][d] . P[g][t]  dims d as M (16 per tile), tokens as K
// Lane l holds S^T/O^T elements of rows l/4 and l/4 + 8 and of heads
// g0 = 2 (l % 4), g1 = g0 + 1, so the online-softmax state of a lane is the
// running max and (partial) sum of its two heads.
template <int D, int BS>
struct MmaMath {
    static constexpr int GP = 8;
    static constexpr int KST = D / 16;  // k-steps of q.K
    static constexpr int TT = BS / 16;  // token tiles per block
    static constexpr int DT = D / 16;   // dim tiles of P.V

    int lane;
    uint32_t pscr;  // this warp's bf16 P[GP][BS] (shared address)
    float scale_log2;
    uint32_t qb[KST][2];  // B fragments of q
    float acc[DT][4];     // O^T fragments
    float m0, m1, l0, l1;

    __device__ __forceinline__ void init(int warp, int lane_, uint8_t *base, const DecodeLayout &ly) {
        lane = lane_;
        pscr = smem_u32(base + ly.pscr) + warp * (GP * BS * 2);
    }

    // B fragment (k = dim, n = head): two consecutive dims of q[l/4]; heads past the group are 0.
    // With pack = 2 the slot holds rows of D / 2 dims and query row g is
    // placed in half g / (group / 2) of the virtual head, zeros in the other.
    __device__ __forceinline__ void load_q(uint32_t qslot, int group, float sl2, int pack, const DecodeArgs & /*a*/,
                                           int /*h*/) {
        scale_log2 = sl2;
        const int g = lane >> 2, k2 = (lane & 3) * 2;
        const int half = pack == 2 ? g / (group >> 1) : 0;
        const int dr = D / pack;  // dims per stored row
#pragma unroll
        for (int kk = 0; kk < KST; ++kk) {
            const bool mine = g < group && (pack == 1 || kk / (KST / 2) == half);
            const int col = 16 * kk - half * dr;
            qb[kk][0] = mine ? lds32(qslot + (g * dr + col + k2) * 2) : 0u;
            qb[kk][1] = mine ? lds32(qslot + (g * dr + col + 8 + k2) * 2) : 0u;
        }
    }

    __device__ __forceinline__ void reset() {
        m0 = m1 = -INFINITY;
        l0 = l1 = 0.f;
#pragma unroll
        for (int dt = 0; dt < DT; ++dt)
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[dt][k] = 0.f;
    }

    // One KV tile in two steps: qk() reads only the K tile (logits, online-softmax
    // update, P into the warp's scratch), pv() only the V tile.
    __device__ __forceinline__ void qk(uint32_t ktile, int valid) {
        const int mi = lane >> 3, r = lane & 7;
        const int tr = lane >> 2;  // fragment row of this lane
        // S^T = K . Q^T; ldmatrix x4 gives the A fragment (rows t, cols d) of one k-step
        // two accumulators per tile (even / odd k-steps) halve the dependent mma chain
        float s[TT][4], s2[TT][4];
#pragma unroll
        for (int mt = 0; mt < TT; ++mt) {
#pragma unroll
            for (int k = 0; k < 4; ++k) s[mt][k] = s2[mt][k] = 0.f;
#pragma unroll
            for (int kk = 0; kk < KST; ++kk) {
                uint32_t a[4];
                ldsm_x4(a, tile_addr<BS>(ktile, 16 * mt + r + 8 * (mi & 1), 2 * kk + (mi >> 1)));
                mma_16816((kk & 1) ? s2[mt] : s[mt], a, qb[kk][0], qb[kk][1]);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) s[mt][k] += s2[mt][k];
        }
        // base-2 logits; tokens past the context are selected away (their rows may hold anything)
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int mt = 0; mt < TT; ++mt) {
            const int t0 = 16 * mt + tr, t1 = t0 + 8;
            s[mt][0] = t0 < valid ? s[mt][0] * scale_log2 : -INFINITY;
            s[mt][1] = t0 < valid ? s[mt][1] * scale_log2 : -INFINITY;
            s[mt][2] = t1 < valid ? s[mt][2] * scale_log2 : -INFINITY;
            s[mt][3] = t1 < valid ? s[mt][3] * scale_log2 : -INFINITY;
            mx0 = fmaxf(mx0, fmaxf(s[mt][0], s[mt][2]));
            mx1 = fmaxf(mx1, fmaxf(s[mt][1], s[mt][3]));
        }
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
        }
        const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
        const float a0 = fast_exp2(m0 - n0), a1 = fast_exp2(m1 - n1);
        // probabilities, rounded to bf16 for the P.V product; the sums take the
        // rounded values so numerator and denominator see the same weights
        const int g0 = 2 * (lane & 3);
        float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
        for (int mt = 0; mt < TT; ++mt) {
            const int t0 = 16 * mt + tr;
            const __nv_bfloat16 p0 = __float2bfloat16_rn(fast_exp2(s[mt][0] - n0));
            const __nv_bfloat16 p1 = __float2bfloat16_rn(fast_exp2(s[mt][1] - n1));
            const __nv_bfloat16 p2 = __float2bfloat16_rn(fast_exp2(s[mt][2] - n0));
            const __nv_bfloat16 p3 = __float2bfloat16_rn(fast_exp2(s[mt][3] - n1));
            ps0 += __bfloat162float(p0) + __bfloat162float(p2);
            ps1 += __bfloat162float(p1) + __bfloat162float(p3);
            sts16(pscr + (g0 * BS + t0) * 2, __bfloat16_as_ushort(p0));
            sts16(pscr + ((g0 + 1) * BS + t0) * 2, __bfloat16_as_ushort(p1));
            sts16(pscr + (g0 * BS + t0 + 8) * 2, __bfloat16_as_ushort(p2));
            sts16(pscr + ((g0 + 1) * BS + t0 + 8) * 2, __bfloat16_as_ushort(p3));
        }
        l0 = l0 * a0 + ps0;
        l1 = l1 * a1 + ps1;
        if (__any_sync(0xffffffffu, n0 != m0 || n1 != m1)) {
#pragma unroll
            for (int dt = 0; dt < DT; ++dt) {
                acc[dt][0] *= a0;
                acc[dt][1] *= a1;
                acc[dt][2] *= a0;
                acc[dt][3] *= a1;
            }
        }
        m0 = n0;
        m1 = n1;
        __syncwarp();
    }

    __device__ __forceinline__ void block(uint32_t ktile, uint32_t vtile, int valid) {
        qk(ktile, valid);
        pv(vtile, valid);
    }

    __device__ __forceinline__ void pv(uint32_t vtile, int valid) {
        const int mi = lane >> 3, r = lane & 7;
        // O^T += V^T . P^T; ldmatrix x4 .trans gives the A fragment (rows d, cols t)
#pragma unroll
        for (int ks = 0; ks < TT; ++ks) {
            const uint32_t pb = pscr + ((lane >> 2) * BS + 16 * ks + 2 * (lane & 3)) * 2;
            const uint32_t b0 = lds32(pb), b1 = lds32(pb + 16);
            // V rows past the context may hold NaN: zero them in the fragments
            uint32_t keep_lo = 0xffffffffu, keep_hi = 0xffffffffu;
            if (valid < BS) {
                const int t = 16 * ks + 2 * (lane & 3);
                keep_lo = (t < valid ? 0x0000ffffu : 0u) | (t + 1 < valid ? 0xffff0000u : 0u);
                keep_hi = (t + 8 < valid ? 0x0000ffffu : 0u) | (t + 9 < valid ? 0xffff0000u : 0u);
            }
            if (valid < BS) {  // the segment's last block only
#pragma unroll
                for (int dt = 0; dt < DT; ++dt) {
                    uint32_t a[4];
                    ldsm_x4_trans(a, tile_addr<BS>(vtile, 16 * ks + r + 8 * (mi >> 1), 2 * dt + (mi & 1)));
                    a[0] &= keep_lo;
                    a[1] &= keep_lo;
                    a[2] &= keep_hi;
                    a[3] &= keep_hi;
                    mma_16816(acc[dt], a, b0, b1);
                }
            } else {
#pragma unroll
                for (int dt = 0; dt < DT; ++dt) {
                    uint32_t a[4];
                    ldsm_x4_trans(a, tile_addr<BS>(vtile, 16 * ks + r + 8 * (mi >> 1), 2 * dt + (mi & 1)));
                    mma_16816(acc[dt], a, b0, b1);
                }
            }
        }
        __syncwarp();  // P scratch is rewritten by the next block
    }

    __device__ __forceinline__ void export_state(float *merge_acc, float *merge_m, float *merge_l, int warp, int G,
                                                 int pack) {
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            l0 += __shfl_xor_sync(0xffffffffu, l0, o);
            l1 += __shfl_xor_sync(0xffffffffu, l1, o);
        }
        const int g0 = 2 * (lane & 3), dr = lane >> 2;
        if (lane < 4) {
            if (g0 < G) {
                merge_m[warp * G + g0] = m0;
                merge_l[warp * G + g0] = l0;
            }
            if (g0 + 1 < G) {
                merge_m[warp * G + g0 + 1] = m1;
                merge_l[warp * G + g0 + 1] = l1;
            }
        }
        // rows of D / pack floats: with pack = 2 a column keeps only its own half
        const int DR = D / pack;
        const int h0 = pack == 2 ? g0 / (G >> 1) : 0, h1 = pack == 2 ? (g0 + 1) / (G >> 1) : 0;
        float *r0 = merge_acc + (warp * G + g0) * DR - h0 * DR;
        float *r1 = merge_acc + (warp * G + g0 + 1) * DR - h1 * DR;
#pragma unroll
        for (int dt = 0; dt < DT; ++dt) {
            const int half = (16 * dt) / DR;  // all 16 dims of a tile lie in one half
            if (g0 < G && half == h0) {
                r0[16 * dt + dr] = acc[dt][0];
                r0[16 * dt + dr + 8] = acc[dt][2];
            }
            if (g0 + 1 < G && half == h1) {
                r1[16 * dt + dr] = acc[dt][1];
                r1[16 * dt + dr + 8] = acc[dt][3];
            }
        }
    }
};

// ------------------------------------------------------------------ e4m3 tensor-core math

// d += a (16x16 f16, row) * b (16x8 f16, col), fp32 accumulate.
__device__ __forceinline__ void mma_16816_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Two e4m3 codes of w -- the bytes SEL places in bytes 0 and 2 (SEL's other
// nibbles are 4: zero bytes) -- as an f16x2 of each code's value times 2^-8,
// exactly: the code's magnitude bits (exponent, then mantissa) move to bits
// 7..13 of the f16 and its sign to bit 15; an f16 with exponent field e and
// mantissa m is then 2^(e-15) (1 + m/8), the code's 2^(e-7) (1 + m/8) times
// 2^-8, and the subnormal codes land on the f16 subnormals the same way. The
// sign moves one place up by adding the sign bit to itself. Exact for every
// finite code; the two NaN codes become +-480 x 2^-8 (the kernel only meets
// them in rows it masks). Integer adds and a shift, instead of a conversion
// instruction that occupies the ALU pipe four times as long.
template <uint32_t SEL>
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2_lo8(uint32_t w) {
    const uint32_t t = __byte_perm(w, 0u, SEL);
    return (t + (t & 0x00800080u)) << 7;
}

__device__ __forceinline__ uint32_t f16x2_bits(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// Tensor-core math over e4m3 pools, f16 products with fp32 accumulation. A
// tile holds BS rows of 128 * HP one-byte codes (128-byte swizzled slices):
// HP = 1 -- one virtual head of 128 dims (head_dim 128, or two heads of 64
// packed as in MmaMath); HP = 2 -- two real heads of 128 side by side
// (256-byte rows read from the pool), each query column using only its own
// head's slice.
//   S^T[t][g] = K[t][:] . q[g][:]   as in MmaMath, but ldmatrix gives a lane
//     four consecutive codes of a row, so inside each 16-dim chunk the k index
//     runs over dims in the order (4l, 4l+1 | 4l+2, 4l+3) and q's B fragments
//     are built in the same order; with HP = 2 a column's B fragment is zero
//     on the other head's chunks;
//   O^T[d][g] += V[t][d] . P[g][t]  ldmatrix .trans gives a lane two 2-code
//     columns of two token rows; one byte permute splits them into (dim 2r,
//     tokens) and (dim 2r+1, tokens), so fragment rows r and r + 8 of a dim
//     tile are dims 2r and 2r+1. With HP = 2 each dim tile is multiplied
//     twice, by each head's slice with P zeroed outside that head's columns,
//     so the accumulators hold every column's own 128 dims.
// q is converted to f16 after scaling its row by a power of two that puts
// the row's largest magnitude in [2^14, 2^15) (no overflow, bf16's 8
// significant bits kept); the power of two, the head's K scale and the
// softmax scale fold into one per-column logit multiplier. P is rounded to
// f16. The head's V scale multiplies the accumulators at export.
template <int BS, int HP>
struct Fp8Math {
    static constexpr int D = 128 * HP;  // codes per tile row (the kernel's head_dim)
    static constexpr int GP = 8;
    static constexpr int TT = BS / 16;
    static constexpr int DT = 8;        // dim tiles of the accumulators (128 dims)

    int lane;
    int my_half;          // HP = 2: the head (0/1) of this lane's B-fragment column lane / 4
    bool c1_head0, c1_head1;  // HP = 2: the heads of this lane's two accumulator columns are 1
    uint32_t pscr;        // this warp's f16 P[GP][BS] (shared address)
    uint32_t qb[8][2];    // f16 B fragments of q (row-scaled, chunk-permuted), 8 chunks of 16 dims
    float mult0, mult1;   // base-2 logit multiplier of this lane's two columns
    const float *vsc0, *vsc1;  // V scale of this lane's two columns (read at export)
    float acc[DT][4];     // O^T fragments (rows: dims 2r, 2r+1 of each tile)
    float m0, m1, l0, l1;

    __device__ __forceinline__ void init(int warp, int lane_, uint8_t *base, const DecodeLayout &ly) {
        lane = lane_;
        pscr = smem_u32(base + ly.pscr) + warp * (GP * BS * 2);
    }

    // q rows are bf16 of D / pack dims. HP = 1, pack = 2: row g lies in half
    // g / (group / 2) of the 128 dims. HP = 2 (pack = 2): row g is 128 dims of
    // head g / (group / 2).
    __device__ __forceinline__ void load_q(uint32_t qslot, int group, float sl2, int pack, const DecodeArgs &a,
                                           int h) {
        const int g = lane >> 2, t = lane & 3;
        const int half = pack == 2 ? g / (group >> 1) : 0;
        const int dr = D / pack;
        my_half = HP == 2 ? half : 0;
        float v[8][4];
        float mx = 0.f;
#pragma unroll
        for (int kc = 0; kc < 8; ++kc) {
            bool mine;
            int col;
            if constexpr (HP == 2) {
                mine = g < group;
                col = 16 * kc;
            } else {
                mine = g < group && (pack == 1 || kc / 4 == half);
                col = 16 * kc - half * dr;
            }
            const uint32_t lo = mine ? lds32(qslot + (g * dr + col + 4 * t) * 2) : 0u;
            const uint32_t hi = mine ? lds32(qslot + (g * dr + col + 4 * t + 2) * 2) : 0u;
            const float2 f0 = bf16x2_to_float2(lo), f1 = bf16x2_to_float2(hi);
            v[kc][0] = f0.x;
            v[kc][1] = f0.y;
            v[kc][2] = f1.x;
            v[kc][3] = f1.y;
            mx = fmaxf(mx, fmaxf(fmaxf(fabsf(f0.x), fabsf(f0.y)), fmaxf(fabsf(f1.x), fabsf(f1.y))));
        }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        // power of two 2^(eb - 127) with the row max in [2^14, 2^15); its inverse is exact too
        const int e = static_cast<int>((__float_as_uint(mx) >> 23) & 0xffu);  // biased exponent of the max
        const int eb = mx > 0.f ? min(max(127 + 14 - (e - 127), 1), 253) : 127;
        const float ps = __uint_as_float(static_cast<uint32_t>(eb) << 23);
        const float inv_ps = __uint_as_float(static_cast<uint32_t>(254 - eb) << 23);
#pragma unroll
        for (int kc = 0; kc < 8; ++kc) {
            qb[kc][0] = f16x2_bits(v[kc][0] * ps, v[kc][1] * ps);
            qb[kc][1] = f16x2_bits(v[kc][2] * ps, v[kc][3] * ps);
        }
        const int n0 = 2 * t, n1 = n0 + 1;
        const float ip0 = __shfl_sync(0xffffffffu, inv_ps, 4 * n0), ip1 = __shfl_sync(0xffffffffu, inv_ps, 4 * n1);
        const int hg = pack == 2 ? (group >> 1) : group;  // query rows per real head
        const int h0 = pack * h + (n0 < group ? n0 / hg : 0), h1 = pack * h + (n1 < group ? n1 / hg : 0);
        // x 2^8: the K codes enter the products as f16 of value code x 2^-8
        c1_head0 = HP == 2 && n0 < group && n0 / hg == 1;
        c1_head1 = HP == 2 && n1 < group && n1 / hg == 1;
        mult0 = n0 < group ? sl2 * __ldg(a.k_scale + h0) * ip0 * 256.f : 0.f;
        mult1 = n1 < group ? sl2 * __ldg(a.k_scale + h1) * ip1 * 256.f : 0.f;
        vsc0 = a.v_scale + h0;
        vsc1 = a.v_scale + h1;
    }

    __device__ __forceinline__ void reset() {
        m0 = m1 = -INFINITY;
        l0 = l1 = 0.f;
#pragma unroll
        for (int dt = 0; dt < DT; ++dt)
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[dt][k] = 0.f;
    }

    // One KV tile in two steps, as in MmaMath: qk() reads only the K tile, pv() only the V tile.
    __device__ __forceinline__ void qk(uint32_t ktile, int valid) {
        const int mi = lane >> 3, r = lane & 7;
        const int tr = lane >> 2;
        // S^T = K . Q^T; one ldmatrix x4 covers tokens 0-15 of two 16-dim chunks
        float s[TT][4], s2[TT][4];
#pragma unroll
        for (int mt = 0; mt < TT; ++mt) {
#pragma unroll
            for (int k = 0; k < 4; ++k) s[mt][k] = s2[mt][k] = 0.f;
            if constexpr (HP == 1) {
                // chunks 2kp, 2kp + 1 into two independent chains
#pragma unroll
                for (int kp = 0; kp < 4; ++kp) {
                    uint32_t x[4];
                    ldsm_x4(x, tile_addr<BS>(ktile, 16 * mt + r + 8 * (mi & 1), 2 * kp + (mi >> 1)));
                    // codes as f16 x 2^-8 (the logit multiplier holds the 2^8)
                    const uint32_t a0[4] = {e4m3x2_to_f16x2_lo8<0x4140>(x[0]), e4m3x2_to_f16x2_lo8<0x4140>(x[1]),
                                            e4m3x2_to_f16x2_lo8<0x4342>(x[0]), e4m3x2_to_f16x2_lo8<0x4342>(x[1])};
                    mma_16816_f16(s[mt], a0, qb[2 * kp][0], qb[2 * kp][1]);
                    const uint32_t a1[4] = {e4m3x2_to_f16x2_lo8<0x4140>(x[2]), e4m3x2_to_f16x2_lo8<0x4140>(x[3]),
                                            e4m3x2_to_f16x2_lo8<0x4342>(x[2]), e4m3x2_to_f16x2_lo8<0x4342>(x[3])};
                    mma_16816_f16(s2[mt], a1, qb[2 * kp + 1][0], qb[2 * kp + 1][1]);
                }
#pragma unroll
                for (int k = 0; k < 4; ++k) s[mt][k] += s2[mt][k];
            } else {
                // Two heads per row: head 0's 128 dims accumulate in s, head 1's in
                // s2, every column against both (each lane's q fragment holds its
                // own head's q), and each column keeps its own head's chain -- no
                // per-lane masking of the q fragments. The heads alternate: two
                // independent chains.
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int kp = (j >> 1) + 4 * (j & 1);  // 0, 4, 1, 5, ...: head j & 1
                    const int qc = (2 * kp) % 8;
                    uint32_t x[4];
                    ldsm_x4(x, tile_addr<BS>(ktile, 16 * mt + r + 8 * (mi & 1), 2 * kp + (mi >> 1)));
                    // codes as f16 x 2^-8 (the logit multiplier holds the 2^8)
                    const uint32_t a0[4] = {e4m3x2_to_f16x2_lo8<0x4140>(x[0]), e4m3x2_to_f16x2_lo8<0x4140>(x[1]),
                                            e4m3x2_to_f16x2_lo8<0x4342>(x[0]), e4m3x2_to_f16x2_lo8<0x4342>(x[1])};
                    const uint32_t a1[4] = {e4m3x2_to_f16x2_lo8<0x4140>(x[2]), e4m3x2_to_f16x2_lo8<0x4140>(x[3]),
                                            e4m3x2_to_f16x2_lo8<0x4342>(x[2]), e4m3x2_to_f16x2_lo8<0x4342>(x[3])};
                    auto step = [&](float (&acc_h)[4]) {
                        mma_16816_f16(acc_h, a0, qb[qc][0], qb[qc][1]);
                        mma_16816_f16(acc_h, a1, qb[qc + 1][0], qb[qc + 1][1]);
                    };
                    if (j & 1) step(s2[mt]);
                    else step(s[mt]);
                }
                s[mt][0] = c1_head0 ? s2[mt][0] : s[mt][0];
                s[mt][1] = c1_head1 ? s2[mt][1] : s[mt][1];
                s[mt][2] = c1_head0 ? s2[mt][2] : s[mt][2];
                s[mt][3] = c1_head1 ? s2[mt][3] : s[mt][3];
            }
        }
        // base-2 logits; tokens past the context are selected away (their rows may hold NaN codes)
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int mt = 0; mt < TT; ++mt) {
            const int t0 = 16 * mt + tr, t1 = t0 + 8;
            s[mt][0] = t0 < valid ? s[mt][0] * mult0 : -INFINITY;
            s[mt][1] = t0 < valid ? s[mt][1] * mult1 : -INFINITY;
            s[mt][2] = t1 < valid ? s[mt][2] * mult0 : -INFINITY;
            s[mt][3] = t1 < valid ? s[mt][3] * mult1 : -INFINITY;
            mx0 = fmaxf(mx0, fmaxf(s[mt][0], s[mt][2]));
            mx1 = fmaxf(mx1, fmaxf(s[mt][1], s[mt][3]));
        }
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
        }
        const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
        const float a0 = fast_exp2(m0 - n0), a1 = fast_exp2(m1 - n1);
        // probabilities rounded to f16 for the P.V product; the sums take the rounded values
        const int g0 = 2 * (lane & 3);
        float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
        for (int mt = 0; mt < TT; ++mt) {
            const int t0 = 16 * mt + tr;
            const __half p0 = __float2half_rn(fast_exp2(s[mt][0] - n0));
            const __half p1 = __float2half_rn(fast_exp2(s[mt][1] - n1));
            const __half p2 = __float2half_rn(fast_exp2(s[mt][2] - n0));
            const __half p3 = __float2half_rn(fast_exp2(s[mt][3] - n1));
            ps0 += __half2float(p0) + __half2float(p2);
            ps1 += __half2float(p1) + __half2float(p3);
            sts16(pscr + (g0 * BS + t0) * 2, __half_as_ushort(p0));
            sts16(pscr + ((g0 + 1) * BS + t0) * 2, __half_as_ushort(p1));
            sts16(pscr + (g0 * BS + t0 + 8) * 2, __half_as_ushort(p2));
            sts16(pscr + ((g0 + 1) * BS + t0 + 8) * 2, __half_as_ushort(p3));
        }
        l0 = l0 * a0 + ps0;
        l1 = l1 * a1 + ps1;
        if (__any_sync(0xffffffffu, n0 != m0 || n1 != m1)) {
#pragma unroll
            for (int dt = 0; dt < DT; ++dt) {
                acc[dt][0] *= a0;
                acc[dt][1] *= a1;
                acc[dt][2] *= a0;
                acc[dt][3] *= a1;
            }
        }
        m0 = n0;
        m1 = n1;
        __syncwarp();
    }

    __device__ __forceinline__ void block(uint32_t ktile, uint32_t vtile, int valid) {
        qk(ktile, valid);
        pv(vtile, valid);
    }

    __device__ __forceinline__ void pv(uint32_t vtile, int valid) {
        const int mi = lane >> 3, r = lane & 7;
        // O^T += V^T . P^T; one ldmatrix x4 .trans covers tokens 0-15 of two dim tiles
#pragma unroll
        for (int ks = 0; ks < TT; ++ks) {
            const uint32_t pb = pscr + ((lane >> 2) * BS + 16 * ks + 2 * (lane & 3)) * 2;
            const uint32_t b0 = lds32(pb), b1 = lds32(pb + 16);
            // V rows past the context may hold NaN codes: zero them in the fragments
            uint32_t keep_lo = 0xffffffffu, keep_hi = 0xffffffffu;
            if (valid < BS) {
                const int t = 16 * ks + 2 * (lane & 3);
                keep_lo = (t < valid ? 0x0000ffffu : 0u) | (t + 1 < valid ? 0xffff0000u : 0u);
                keep_hi = (t + 8 < valid ? 0x0000ffffu : 0u) | (t + 9 < valid ? 0xffff0000u : 0u);
            }
#pragma unroll
            for (int hs = 0; hs < HP; ++hs) {
                // head slice hs; with HP = 2 only the columns of head hs take it
                const bool on = HP == 1 || my_half == hs;
                const uint32_t c0 = on ? b0 : 0u, c1 = on ? b1 : 0u;
                // the masks matter in the segment's last block only
                const uint32_t klo = valid < BS ? keep_lo : 0xffffffffu, khi = valid < BS ? keep_hi : 0xffffffffu;
#pragma unroll
                for (int dp = 0; dp < DT / 2; ++dp) {
                    uint32_t x[4];
                    ldsm_x4_trans(x, tile_addr<BS>(vtile, 16 * ks + r + 8 * (mi & 1), 8 * hs + 2 * dp + (mi >> 1)));
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        // x[2j]: tokens 0-7 of tile 2dp + j, x[2j + 1]: tokens 8-15; bytes
                        // (t, 2r) (t, 2r+1) (t+1, 2r) (t+1, 2r+1) -> (t, 2r) (t+1, 2r) | (t, 2r+1) (t+1, 2r+1),
                        // as f16 x 2^-8 (the V scale holds the 2^8)
                        uint32_t av[4] = {e4m3x2_to_f16x2_lo8<0x4240>(x[2 * j]), e4m3x2_to_f16x2_lo8<0x4341>(x[2 * j]),
                                          e4m3x2_to_f16x2_lo8<0x4240>(x[2 * j + 1]),
                                          e4m3x2_to_f16x2_lo8<0x4341>(x[2 * j + 1])};
                        if (valid < BS) {
                            av[0] &= klo;
                            av[1] &= klo;
                            av[2] &= khi;
                            av[3] &= khi;
                        }
                        mma_16816_f16(acc[2 * dp + j], av, c0, c1);
                    }
                }
            }
        }
        __syncwarp();  // P scratch is rewritten by the next block
    }

    // Rows of D / pack floats: HP = 2 -- the column's own 128 dims; HP = 1 with
    // pack = 2 -- the column's own half of the 128.
    __device__ __forceinline__ void export_state(float *merge_acc, float *merge_m, float *merge_l, int warp, int G,
                                                 int pack) {
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            l0 += __shfl_xor_sync(0xffffffffu, l0, o);
            l1 += __shfl_xor_sync(0xffffffffu, l1, o);
        }
        const int g0 = 2 * (lane & 3), dr = lane >> 2;
        if (lane < 4) {
            if (g0 < G) {
                merge_m[warp * G + g0] = m0;
                merge_l[warp * G + g0] = l0;
            }
            if (g0 + 1 < G) {
                merge_m[warp * G + g0 + 1] = m1;
                merge_l[warp * G + g0 + 1] = l1;
            }
        }
        const int DR = D / pack;
        const int h0 = HP == 1 && pack == 2 ? g0 / (G >> 1) : 0, h1 = HP == 1 && pack == 2 ? (g0 + 1) / (G >> 1) : 0;
        float *r0 = merge_acc + (warp * G + g0) * DR - h0 * DR;
        float *r1 = merge_acc + (warp * G + g0 + 1) * DR - h1 * DR;
        // x 2^8: the V codes enter the products as f16 of value code x 2^-8
        const float vs0 = g0 < G ? __ldg(vsc0) * 256.f : 0.f, vs1 = g0 + 1 < G ? __ldg(vsc1) * 256.f : 0.f;
#pragma unroll
        for (int dt = 0; dt < DT; ++dt) {
            const int half = HP == 1 ? (16 * dt) / DR : 0;
            if (g0 < G && half == h0) {
                r0[16 * dt + 2 * dr] = acc[dt][0] * vs0;
                r0[16 * dt + 2 * dr + 1] = acc[dt][2] * vs0;
            }
            if (g0 + 1 < G && half == h1) {
                r1[16 * dt + 2 * dr] = acc[dt][1] * vs1;
                r1[16 * dt + 2 * dr + 1] = acc[dt][3] * vs1;
            }
        }
    }
};

// ------------------------------------------------------------------ pipeline

struct Smem {
    uint8_t *base;
    uint64_t *full, *qfull;  // per stage: its K and V tiles landed; query slots
    volatile int *stage_bad;
    int *stage_blk;  // [kMaxStages] first pool row of the tile whose copy the stage holds
    volatile int *abort_flag;
    volatile int *merge_flag;  // [1 + 2 * 2]: how many segments this CTA completed (<= 2), then
                               // (s, h) of each
    int *scan;
    int *prefix;
    int *wprefix;
    int *lens;
    int *ptiles;     // [S] shared-prefix tiles of each sequence (0: not in a prefix group)
    uint64_t *empty;  // prefix units: all four warps are done with a stage
    volatile unsigned long long *epoch;  // this launch's epoch (read from the workspace header)
};

// The CTAs holding pieces of segment (s, h). CTA c covers weight positions
// [c W / C, (c + 1) W / C), so position v lies in CTA ((v + 1) C - 1) / W; the
// segment's real blocks sit at positions v_first .. v_first + n - 1. With
// W >= C no CTA range is empty and the pieces are held by CTAs c0 .. c0 +
// npieces - 1; with W < C every range holds at most one position, so each of
// the n blocks is a piece of its own, in CTA ((v_first + i + 1) C - 1) / W.
struct SegmentSpan {
    long long v_first;
    int c0, npieces;
};

__device__ __forceinline__ SegmentSpan segment_span(int s, int h, const Smem &sm, int Hkv, long long W, int C,
                                                    int pcost) {
    SegmentSpan sp;
    const int n = sm.prefix[s + 1] - sm.prefix[s];
    sp.v_first = static_cast<long long>(Hkv) * sm.wprefix[s] + static_cast<long long>(h) * (n + pcost) + pcost;
    sp.c0 = static_cast<int>(((sp.v_first + 1) * C - 1) / W);
    sp.npieces = W >= C ? static_cast<int>(((sp.v_first + n) * C - 1) / W) - sp.c0 + 1 : n;
    return sp;
}

// The CTA holding piece i of a segment.
__device__ __forceinline__ int piece_cta(const SegmentSpan &sp, int i, long long W, int C) {
    return W >= C ? sp.c0 + i : static_cast<int>(((sp.v_first + i + 1) * C - 1) / W);
}

// Prefix pieces of sequence s that hold some of its tokens: the prefix units
// of its group whose tiles start below its length.
__device__ __forceinline__ int live_prefix_pieces(int s, const Smem &sm, int BS, int tiles_per_piece) {
    const int pt = sm.ptiles[s], L = sm.lens[s];
    if (pt == 0 || L == 0) return 0;
    const int t = min((L + BS - 1) / BS, pt);
    return (t + tiles_per_piece - 1) / tiles_per_piece;
}

// Pieces segment (s, h) is merged from: its live prefix pieces, then the
// suffix pieces the CTA split gives it (none when the suffix is empty).
__device__ __forceinline__ int segment_pieces(int s, int h, const Smem &sm, int Hkv, long long W, int C, int pcost,
                                              int BS, int tiles_per_piece, SegmentSpan *sp_out) {
    SegmentSpan sp{0, 0, 0};
    if (sm.prefix[s + 1] > sm.prefix[s]) sp = segment_span(s, h, sm, Hkv, W, C, pcost);
    if (sp_out) *sp_out = sp;
    return live_prefix_pieces(s, sm, BS, tiles_per_piece) + sp.npieces;
}

// The partial-row bases of segment (s, h)'s pieces, prefix pieces first:
// operator()(i) is piece i's base (its partial rows are base * G + g).
struct PieceBases {
    SegmentSpan sp;
    long long W;
    int C, npre, seg, pre;  // pre: base of the segment's first prefix piece
    __device__ __forceinline__ int operator()(int i) const {
        return i < npre ? pre + i : seg + piece_cta(sp, i - npre, W, C);
    }
};

// Pieces of segment (s, h) and where their partials are (returns the count).
__device__ __forceinline__ int piece_bases(const DecodeArgs &a, int s, int h, const Smem &sm, long long W, int C,
                                           int pcost, int BS, PieceBases &pb) {
    const int n = segment_pieces(s, h, sm, a.num_kv_heads, W, C, pcost, BS, a.tiles_per_piece, &pb.sp);
    pb.W = W;
    pb.C = C;
    pb.npre = n - pb.sp.npieces;
    pb.seg = s * a.num_kv_heads + h;
    pb.pre = a.pre_base + pb.seg * a.prefix_np;
    return n;
}

// Counts a piece in on its segment's counter (launch epoch << 16 | pieces
// counted) and returns the counter after it. A counter an older launch left
// restarts at 1 through a CAS; once it carries this launch's epoch it keeps it
// for the rest of the launch, so later pieces take a plain add -- no retries
// when the many pieces of a long context arrive together. guess: a recent read
// of the counter.
__device__ __forceinline__ unsigned long long count_piece_in(unsigned long long *cnt, unsigned long long ep,
                                                              unsigned long long guess) {
    unsigned long long old = guess;
    for (;;) {
        if ((old >> 16) == ep) return atomicAdd(cnt, 1ull) + 1ull;
        const unsigned long long prev = atomicCAS(cnt, old, (ep << 16) | 1ull);
        if (prev == old) return (ep << 16) | 1ull;
        old = prev;
    }
}

// Merge of the pieces of segment (s, h) whose partials sit at rows
// base(i) * G + g, i < npieces (log-sum-exp identity): out = sum_c 2^(lse_c - M)
// o_c / sum_c 2^(lse_c - M), with a running maximum. The pieces are dealt to J
// interleaved subsets (i = j, j + J, j + 2J, ...): J, a power of two up to 32,
// spreads a long merge over the threads that a small output leaves idle. Thread
// ctid merges subset ctid mod J of the 4-dim elements ctid / J + k * (threads /
// J), k < kE, with the loads of kAhead pieces of each in flight; the J threads
// of an element (consecutive lanes) then combine in a butterfly and the
// element's subset-0 thread stores it, so the result depends on npieces and G
// only. Partials written by other SMs are read past L1.
// Elements a thread merges: the G x D / 4 float4 columns over the CTA's threads (G <= 8).
template <int D>
constexpr int merge_elems() { return (8 * (D / 4) + kConsumerWarps * 32 - 1) / (kConsumerWarps * 32); }

// a (running state) absorbs b: both log2-sum-exp states of the same element
__device__ __forceinline__ void lse_absorb(float &Ma, float &da, float4 &aa, float Mb, float db, const float4 &ab) {
    if (!(Mb > -INFINITY)) return;  // b holds no piece
    const float Mn = fmaxf(Ma, Mb);
    const float r = fast_exp2(Ma - Mn), w = fast_exp2(Mb - Mn);
    da = da * r + db * w;
    aa.x = aa.x * r + ab.x * w;
    aa.y = aa.y * r + ab.y * w;
    aa.z = aa.z * r + ab.z * w;
    aa.w = aa.w * r + ab.w * w;
    Ma = Mn;
}

template <int D, int kAhead = (8 / merge_elems<D>() > 0 ? 8 / merge_elems<D>() : 1), class Base>
__device__ __forceinline__ void merge_pieces(const DecodeArgs &a, const Base &base, int npieces, int s, int h,
                                             int ctid) {
    constexpr int kE = merge_elems<D>();
    constexpr int kThreads = kConsumerWarps * 32;
    const int G = a.group;
    const int DR = D / a.pack;
    const int E = G * (D / 4);  // float4 elements of the segment's output rows
    int J = 1;
    while (2 * J * E <= kE * kThreads && 2 * J <= npieces && 2 * J <= 32) J *= 2;
    const int j = ctid & (J - 1);  // this thread's subset of the pieces
    const int per = kThreads / J;  // threads per subset
    int eg[kE], ecol[kE];
    float M[kE], den[kE];
    float4 acc[kE];
#pragma unroll
    for (int k = 0; k < kE; ++k) {
        const int e = ctid / J + k * per;
        eg[k] = e / (D / 4);
        ecol[k] = (e % (D / 4)) * 4 - (a.pack == 2 ? eg[k] / (G >> 1) : 0) * DR;
        if (e >= E || ecol[k] < 0 || ecol[k] >= DR) ecol[k] = -1;  // none, or the other half of a packed head
        M[k] = -INFINITY;
        den[k] = 0.f;
        acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    // every element's loads of kAhead pieces are in flight together
    for (int ib = j; ib < npieces; ib += kAhead * J) {
        float lse[kAhead][kE];
        float4 o[kAhead][kE];
#pragma unroll
        for (int i = 0; i < kAhead; ++i) {
            const int pi = ib + i * J;
            const size_t pb = pi < npieces ? static_cast<size_t>(base(pi)) : 0;
#pragma unroll
            for (int k = 0; k < kE; ++k) {
                lse[i][k] = -INFINITY;
                if (pi < npieces && ecol[k] >= 0) {
                    const size_t pr = pb * G + eg[k];
                    lse[i][k] = __ldcg(a.lse_part + pr);
                    o[i][k] = __ldcg(reinterpret_cast<const float4 *>(a.o_part + pr * DR + ecol[k]));
                }
            }
        }
#pragma unroll
        for (int i = 0; i < kAhead; ++i)
#pragma unroll
            for (int k = 0; k < kE; ++k) lse_absorb(M[k], den[k], acc[k], lse[i][k], 1.f, o[i][k]);
    }
    // the J subsets of each element: a butterfly over the J consecutive lanes
    for (int off = 1; off < J; off <<= 1) {
#pragma unroll
        for (int k = 0; k < kE; ++k) {
            const float Mb = __shfl_xor_sync(0xffffffffu, M[k], off), db = __shfl_xor_sync(0xffffffffu, den[k], off);
            float4 ab;
            ab.x = __shfl_xor_sync(0xffffffffu, acc[k].x, off);
            ab.y = __shfl_xor_sync(0xffffffffu, acc[k].y, off);
            ab.z = __shfl_xor_sync(0xffffffffu, acc[k].z, off);
            ab.w = __shfl_xor_sync(0xffffffffu, acc[k].w, off);
            lse_absorb(M[k], den[k], acc[k], Mb, db, ab);
        }
    }
    if (j != 0) return;
#pragma unroll
    for (int k = 0; k < kE; ++k) {
        if (ecol[k] < 0) continue;
        const size_t row = static_cast<size_t>(s) * a.num_q_heads + static_cast<size_t>(h) * G + eg[k];
        const float inv = 1.f / den[k];
        __nv_bfloat162 *dst =
            reinterpret_cast<__nv_bfloat162 *>(static_cast<__nv_bfloat16 *>(a.out) + row * DR + ecol[k]);
        dst[0] = __floats2bfloat162_rn(acc[k].x * inv, acc[k].y * inv);
        dst[1] = __floats2bfloat162_rn(acc[k].z * inv, acc[k].w * inv);
    }
}

// One decode warp. Warp w owns the blocks x0 + w + 4k (k = 0, 1, ...) of the
// CTA's range and a ring of R shared-memory stages (stage w + 4 (k % R)). It
// issues the TMA copies of its own blocks R ahead of the one it computes --
// block k + R goes into the stage block k just freed -- so it waits on no other
// warp to refill its ring -- and prefetches its blocks a further `prefetch`
// ahead into L2, so that those copies are served from L2 and more HBM reads are
// in flight than the ring can hold. Block-table entries of its next 32 blocks
// are looked up one batch ahead. Warp 0 also bulk-copies the query rows of the piece after
// next. All four warps meet at the end of every piece to merge their states.
template <int D, int BS, class Math, int ES, bool GROUPS>
__device__ __forceinline__ void decode_warp(const CUtensorMap *tm_k, const CUtensorMap *tm_v, const DecodeArgs &a,
                                            const Smem &sm, const DecodeLayout &ly, PieceIter pieces, long long x0,
                                            long long x1, long long W, int pcost, int warp, int lane) {
    static_assert(ES == 1 || ES == 2, "pool element bytes");
    constexpr uint32_t kTile = BS * D * ES;   // bytes of one K (or V) tile
    constexpr uint32_t kHalf = BS * 128;      // one TMA copy: BS rows of 128 bytes
    constexpr int kCopies = D * ES / 128;     // copies per tile
    const int R = a.num_stages;
    const int G = a.group;
    const int DR = D / a.pack;  // dims per row of q, out and the partials
    const uint32_t qbytes = static_cast<uint32_t>(G * DR * 2);
    const uint32_t sbase = smem_u32(sm.base);
    float *merge_acc = reinterpret_cast<float *>(sm.base + ly.merge_acc);
    float *merge_m = reinterpret_cast<float *>(sm.base + ly.merge_m);
    float *merge_l = reinterpret_cast<float *>(sm.base + ly.merge_l);
    const int ctid = warp * 32 + lane;

    // ---- issue side: this warp's blocks k = 0 .. nk-1 are global blocks x0 + warp + 4k
    const long long span = x1 - x0;
    const int nk = span > warp ? static_cast<int>((span - warp + kConsumerWarps - 1) / kConsumerWarps) : 0;
    // Tile j of a segment is rows [j % sub * BS, +BS) of the pool block in table
    // entry j / sub; a tile is addressed by its first pool row, -1 if the table
    // entry is not a block of the pool.
    const int sub_shift = a.sub == 2 ? 1 : 0;
    auto lookup = [&](int kb, int &p, int &h) {  // lane j: tile kb + j -> (first pool row or -1, kv head)
        p = 0;
        h = 0;
        const int k = kb + lane;
        if (k < nk) {
            const long long x = x0 + warp + static_cast<long long>(kConsumerWarps) * k;
            int lo = 0, hi = a.num_seqs - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (static_cast<long long>(a.num_kv_heads) * sm.prefix[mid] <= x) lo = mid;
                else hi = mid - 1;
            }
            const int n = sm.prefix[lo + 1] - sm.prefix[lo];
            const int r = static_cast<int>(x - static_cast<long long>(a.num_kv_heads) * sm.prefix[lo]);
            h = r / n;
            const int j = r - h * n + (GROUPS ? sm.ptiles[lo] : 0);  // logical tile of the context
            const int pb = __ldg(a.block_tables + static_cast<size_t>(lo) * a.max_blocks_per_seq + (j >> sub_shift));
            p = (pb < 0 || pb >= a.num_blocks) ? -1 : ((pb << sub_shift) + (j & (a.sub - 1))) * BS;
        }
    };
    int bat_k = 0, bat_p, bat_h, nxt_p, nxt_h;
    lookup(0, bat_p, bat_h);
    lookup(32, nxt_p, nxt_h);
    uint32_t inflight = 0, inflight_par = 0;  // stages whose copy this warp issued and has not yet seen land
    // Block k goes to stage warp + 4 (k % R) with phase parity (k / R) & 1, so
    // block k + R reuses block k's stage with the other parity. (Refilling the
    // K tile as soon as q.K is done, on a barrier of its own, measured slower:
    // the wait between q.K and P.V keeps the compiler from overlapping them.)
    auto issue = [&](int k, int stage, uint32_t par) {  // warp-uniform; k increases call after call
        if (k >= nk) return;
        if (k - bat_k >= 32) {
            bat_k += 32;
            bat_p = nxt_p;
            bat_h = nxt_h;
            lookup(bat_k + 32, nxt_p, nxt_h);
        }
        const int p = __shfl_sync(0xffffffffu, bat_p, k - bat_k);
        const int h = __shfl_sync(0xffffffffu, bat_h, k - bat_k);
        if (a.prefetch > 0) {  // this warp's block k + prefetch, from the current or the next batch (<= 32 ahead)
            const int kp = k + a.prefetch, jp = kp - bat_k;
            const int pp_a = __shfl_sync(0xffffffffu, bat_p, jp & 31), pp_b = __shfl_sync(0xffffffffu, nxt_p, jp & 31);
            const int hp_a = __shfl_sync(0xffffffffu, bat_h, jp & 31), hp_b = __shfl_sync(0xffffffffu, nxt_h, jp & 31);
            const int pp = jp < 32 ? pp_a : pp_b, hp = jp < 32 ? hp_a : hp_b;
            if (lane == 0 && kp < nk && pp >= 0 && !*sm.abort_flag) {
#pragma unroll
                for (int half = 0; half < kCopies; ++half) {
                    tma_prefetch_l2_4d(tm_k, 0, half, hp, pp);
                    tma_prefetch_l2_4d(tm_v, 0, half, hp, pp);
                }
            }
        }
        if (lane == 0 && !*sm.abort_flag) {
            const bool bad = p < 0;
            sm.stage_bad[stage] = bad ? 1 : 0;
            sm.stage_blk[stage] = p;
            if (bad) {
                atomicOr(a.status, PKV_STATUS_BAD_BLOCK_ID);
                mbar_arrive(&sm.full[stage]);
            } else {
                // The stage's previous contents were read with ldmatrix / ld.shared whose
                // results this warp has already consumed, so the copy cannot overtake them.
                uint8_t *dst = sm.base + ly.stages + static_cast<uint32_t>(stage) * 2u * kTile;
                mbar_arrive_expect_tx(&sm.full[stage], 2u * kTile);
#pragma unroll
                for (int half = 0; half < kCopies; ++half) {
                    tma_load_4d(dst + half * kHalf, tm_k, &sm.full[stage], 0, half, h, p);
                    tma_load_4d(dst + kTile + half * kHalf, tm_v, &sm.full[stage], 0, half, h, p);
                }
                inflight |= 1u << stage;
                inflight_par = (inflight_par & ~(1u << stage)) | (par << stage);
            }
        }
    };
    for (int k = 0; k < R; ++k) issue(k, warp + kConsumerWarps * k, 0u);

    // ---- query rows: warp 0 copies piece n + 1's rows while piece n is computed
    uint32_t q_issued = 0, q_issued_par = 0;
    PieceIter ahead = pieces;
    Piece pa{};
    auto issue_q = [&](int n) {  // piece n's rows into slot n % 2 (ahead has just returned piece n)
        if (warp == 0 && lane == 0 && !*sm.abort_flag) {
            const int slot = n & 1;
            const __nv_bfloat16 *src = static_cast<const __nv_bfloat16 *>(a.q) +
                                       (static_cast<size_t>(pa.s) * a.num_q_heads + static_cast<size_t>(pa.h) * G) * DR;
            mbar_arrive_expect_tx(&sm.qfull[slot], qbytes);
            bulk_load(sm.base + ly.qbuf + slot * qbytes, src, qbytes, &sm.qfull[slot]);
            q_issued |= 1u << slot;
            q_issued_par = (q_issued_par & ~(1u << slot)) | ((static_cast<uint32_t>(n >> 1) & 1u) << slot);
        }
    };
    int n_ahead = 0;
    if (ahead.next(pa)) issue_q(n_ahead++);
    if (ahead.next(pa)) issue_q(n_ahead++);

    // ---- compute side
    Math math;
    math.init(warp, lane, sm.base, ly);
    int k = 0, gb_base = 0, npiece = 0, ring = 0;
    uint32_t rphase = 0;
    Piece pc;
    while (pieces.next(pc)) {
        const int slot = npiece & 1;
        if (npiece >= 1 && ahead.next(pa)) issue_q(n_ahead++);  // every warp has read slot (npiece + 1) % 2
        mbar_wait_bounded(&sm.qfull[slot], static_cast<uint32_t>(npiece >> 1) & 1u, sm.abort_flag, a.status);
        math.load_q(sbase + ly.qbuf + slot * qbytes, G, a.scale_log2, a.pack, a, pc.h);
        math.reset();
        ++npiece;

        const int nblk = pc.b1 - pc.b0;
        for (int i = (warp - gb_base % kConsumerWarps + kConsumerWarps) % kConsumerWarps; i < nblk;
             i += kConsumerWarps, ++k) {
            const int stage = warp + kConsumerWarps * ring;
            const uint32_t par = rphase;
            if (++ring == R) {
                ring = 0;
                rphase ^= 1u;
            }
            // Fused append: the block holding position L - 1 takes the step's new
            // row (fetched while the block's copy is in flight; lanes < kChunks
            // the K row, the next kChunks lanes the V row, 16 stored bytes each).
            constexpr int kChunks = D * ES / 16;  // 16-byte chunks of a stored row
            constexpr int kElems = 16 / ES;       // elements per chunk
            const int bi = pc.b0 + i;             // block of the segment
            const bool tail = a.slots != nullptr && (bi + 1) * BS >= pc.L;
            long long slot = -1;
            auto patch_src = [&]() {  // this lane's chunk of the new row (bf16 source)
                return reinterpret_cast<const uint4 *>(
                    static_cast<const __nv_bfloat16 *>(lane < kChunks ? a.k_new : a.v_new) +
                    (static_cast<size_t>(pc.s) * a.num_kv_heads + pc.h) * D + (lane % kChunks) * kElems);
            };
            uint4 patch = make_uint4(0u, 0u, 0u, 0u);  // bf16 pools: loaded while the copy is in flight
            if (tail) {
                slot = __ldg(a.slots + pc.s);
                if (ES == 2 && slot >= 0 && lane < 2 * kChunks) patch = __ldg(patch_src());
            }
            const int valid = min(BS, pc.L - bi * BS);
            const uint32_t ktile = sbase + ly.stages + static_cast<uint32_t>(stage) * 2u * kTile;
            // this lane's chunk of the new row goes into the staged tile and the pool
            auto put_row = [&](long long want, int t) {
                const int c = lane % kChunks;
                uint4 row;
                if constexpr (ES == 2) {
                    row = patch;
                } else {  // quantize: element d of real head r -> e4m3(x / scale[r])
                    const int real = pc.h * a.pack + (c * kElems) / (D / a.pack);
                    const float sc = __ldg((lane < kChunks ? a.k_scale : a.v_scale) + real);
                    const uint4 *src = patch_src();
                    row = quantize16_e4m3(__ldg(src), __ldg(src + 1), sc);
                }
                sts128(tile_addr<BS>(lane < kChunks ? ktile : ktile + kTile, t, c), row);
                *reinterpret_cast<uint4 *>(static_cast<uint8_t *>(lane < kChunks ? a.k_cache : a.v_cache) +
                                           ((static_cast<size_t>(want) * a.num_kv_heads + pc.h) * D) * ES + c * 16) =
                    row;
                fence_proxy_async_shared();  // before a later copy overwrites the tile
            };
            if (mbar_wait_bounded(&sm.full[stage], par, sm.abort_flag, a.status)) inflight &= ~(1u << stage);
            if (!sm.stage_bad[stage] && !*sm.abort_flag) {
                if (tail && slot >= 0) {
                    const long long want = static_cast<long long>(sm.stage_blk[stage]) + (valid - 1);  // row of L - 1
                    if (slot == want) {
                        if (lane < 2 * kChunks) put_row(want, valid - 1);
                        __syncwarp();
                    } else if (lane == 0) {
                        atomicOr(a.status, PKV_STATUS_BAD_SLOT);  // not the last position: not appended
                    }
                }
                math.block(ktile, ktile + kTile, valid);
            }
            __syncwarp();
            issue(k + R, stage, par ^ 1u);  // the stage just freed takes this warp's block k + R
        }
        gb_base += nblk;

        math.export_state(merge_acc, merge_m, merge_l, warp, G, a.pack);
        named_barrier_sync(1, kConsumerWarps * 32);

        // merge the warps' states (log-sum-exp identity) and store
        const size_t seg = static_cast<size_t>(pc.s) * a.num_kv_heads + pc.h;
        for (int e = ctid; e < G * D / 2; e += kConsumerWarps * 32) {
            const int g = e / (D / 2), d = (e % (D / 2)) * 2;
            const int col = d - (a.pack == 2 ? g / (G >> 1) : 0) * DR;  // dim within the stored row
            if (col < 0 || col >= DR) continue;  // the other half of a packed virtual head
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, merge_m[w * G + g]);
            float ls = 0.f, a0 = 0.f, a1 = 0.f;
            if (M != -INFINITY) {
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w) {
                    const float f = fast_exp2(merge_m[w * G + g] - M);
                    const float2 av = *reinterpret_cast<const float2 *>(merge_acc + (w * G + g) * DR + col);
                    ls += merge_l[w * G + g] * f;
                    a0 += av.x * f;
                    a1 += av.y * f;
                }
            }
            const float o0 = ls > 0.f ? a0 / ls : 0.f;
            const float o1 = ls > 0.f ? a1 / ls : 0.f;
            if (pc.whole) {
                const size_t row = static_cast<size_t>(pc.s) * a.num_q_heads + static_cast<size_t>(pc.h) * G + g;
                *reinterpret_cast<__nv_bfloat162 *>(static_cast<__nv_bfloat16 *>(a.out) + row * DR + col) =
                    __floats2bfloat162_rn(o0, o1);
            } else {
                // piece (segment + CTA), row g; CTAs are numbered after the prefix units
                const size_t pr = (seg + blockIdx.x - a.prefix_ctas) * G + g;
                *reinterpret_cast<float2 *>(a.o_part + pr * DR + col) = make_float2(o0, o1);
                if (col == 0) a.lse_part[pr] = ls > 0.f ? M + __log2f(ls) : -INFINITY;
            }
        }
        if (!pc.whole) {
            // A segment cut between CTAs: count this CTA's piece in; the CTA that
            // stores the segment's last piece merges them all.
            // Thread 0 reads the counter while the partials drain (the count-in's
            // first guess; a stale one costs a retry) and counts the segment's
            // pieces meanwhile.
            unsigned long long guess = 0;
            int total = 0;
            if (ctid == 0) {
                guess = *reinterpret_cast<volatile unsigned long long *>(a.seg_count + seg);
                total = segment_pieces(pc.s, pc.h, sm, a.num_kv_heads, W, gridDim.x - a.prefix_ctas, pcost, BS,
                                       a.tiles_per_piece, nullptr);
            }
            __threadfence();
            named_barrier_sync(1, kConsumerWarps * 32);
            if (ctid == 0) {
                unsigned long long *cnt = a.seg_count + seg;
                const unsigned long long ep = *sm.epoch;
                const unsigned long long now = count_piece_in(cnt, ep, guess);
                const int pending = sm.merge_flag[0];
                // (a shared-prefix segment is merged by its designated CTA,
                // merge_grouped_segments, whoever completes it)
                const bool designated = GROUPS && sm.ptiles[pc.s] > 0;
                if (static_cast<int>(now & 0xffffull) == total && !designated) {
                    if (pending < 2) {  // never more than two (below)
                        volatile int *m = sm.merge_flag + 1 + 2 * pending;
                        m[0] = pc.s;
                        m[1] = pc.h;
                        sm.merge_flag[0] = pending + 1;
                    }
                }
            }
        }
        named_barrier_sync(1, kConsumerWarps * 32);
    }
    // Leave no copy in flight into shared memory when the CTA exits (only
    // possible after a wait gave up).
    if (lane == 0) {
        for (int st = 0; st < kMaxStages; ++st)
            if ((inflight >> st) & 1u) mbar_wait_drain(&sm.full[st], (inflight_par >> st) & 1u, a.status);
        // the last copy into each query slot: landed already unless a wait gave up
        if (warp == 0)
            for (int slot = 0; slot < 2; ++slot)
                if ((q_issued >> slot) & 1u) mbar_wait_drain(&sm.qfull[slot], (q_issued_par >> slot) & 1u, a.status);
    }
    // The merges this CTA completes run after its last piece, when the loop's
    // state is dead (a CTA's range cuts at most two segments: its first and
    // its last piece; all pieces between are whole).
    // (none after a wait gave up: a copy may still be landing in the stage buffers).
    // The barrier makes every warp's drain complete and the flags final and
    // the same for all threads.
    named_barrier_sync(1, kConsumerWarps * 32);
    const int pending = *sm.abort_flag ? 0 : sm.merge_flag[0];
    for (int i = 0; i < pending; ++i) {
        const volatile int *m = sm.merge_flag + 1 + 2 * i;
        const int s = m[0], h = m[1];
        __threadfence();
        // the grid's total weight, reloaded rather than kept live across the loop
        const long long Wt = static_cast<long long>(a.num_kv_heads) * sm.wprefix[a.num_seqs];
        PieceBases pb;
        const int n = piece_bases(a, s, h, sm, Wt, gridDim.x - a.prefix_ctas, pcost, BS, pb);
        merge_pieces<D>(a, pb, n, s, h, ctid);
    }
}


// ------------------------------------------------------------------ shared prefixes

// One prefix unit: the query rows of up to kPrefixRows (sequence, q head)
// pairs -- the G rows of each member of one row tile of a prefix group, for
// kv head h -- against tiles [t0, t1) of the group's shared prefix, which are
// read once for all of them. Sharing a physical block is the same as owning
// a copy of it ("Deep Dive into vLLM", section 2.2; runbyai post 449, section
// 3), so a block read here serves every member. Flash-attention style on
// mma.sync: warp w takes rows 16 w .. 16 w + 15 as M (q staged once in shared
// memory, read by ldmatrix), a tile's 16 tokens as N (S = Q K^T), then P as
// the A operand of O += P V; the four warps consume one CTA-wide ring of K/V
// tiles that warp 0 refills. Each row leaves an fp32 partial and its
// log2-sum-exp; the last piece of a segment to be stored merges the segment
// (prefix pieces first, then the suffix pieces).
template <int D>
__device__ __forceinline__ void prefix_unit(const CUtensorMap *tm_k, const CUtensorMap *tm_v, const DecodeArgs &a,
                                            const Smem &sm, const DecodeLayout &ly, long long W, int C, int pcost,
                                            int warp, int lane) {
    constexpr int BS = 16;
    constexpr int KST = D / 16;             // k-steps of q.K
    constexpr int NT = D / 8;               // 8-dim n-tiles of P.V
    constexpr int QC = D / 8;               // 16-byte chunks of a q row
    constexpr uint32_t kTile = BS * D * 2;  // bytes of one K (or V) tile
    constexpr uint32_t kHalf = BS * 128;    // one TMA copy: 16 rows of 128 bytes
    constexpr int kCopies = D * 2 / 128;
    const int G = a.group, Hkv = a.num_kv_heads;
    const int ctid = warp * 32 + lane;
    const int NST = kConsumerWarps * a.num_stages;  // the CTA's stages, one ring

    // ---- which unit: group g, kv head h, row tile rt, prefix piece tp
    const int u = blockIdx.x;
    int g = 0;
    while (g + 1 < a.num_groups && a.grp_unit0[g + 1] <= u) ++g;
    const int T = a.grp_tiles[g];
    const int np = (T + a.tiles_per_piece - 1) / a.tiles_per_piece;
    const int v = u - a.grp_unit0[g];
    const int tp = v % np, rt = (v / np) % a.grp_row_tiles[g], h = v / np / a.grp_row_tiles[g];
    const int m0 = a.grp_begin[g] + rt * a.grp_members[g];
    const int m1 = min(a.grp_end[g], m0 + a.grp_members[g]);
    const int rows = (m1 - m0) * G;
    const int t0 = tp * a.tiles_per_piece;
    int lim_max = 0;  // prefix tokens any member attends to
    for (int m = m0; m < m1; ++m) lim_max = max(lim_max, min(sm.lens[m], T * BS));
    const int t1 = min(min(T, t0 + a.tiles_per_piece), (lim_max + BS - 1) / BS);
    const int ntiles = max(0, t1 - t0);

    // ---- the ring: tile j of the piece goes to stage j % NST, K and V on one barrier
    const int *ltab = a.block_tables + static_cast<size_t>(a.grp_begin[g]) * a.max_blocks_per_seq;
    const int sub_shift = a.sub == 2 ? 1 : 0;
    uint32_t inflight = 0, inflight_par = 0;  // producer (warp 0, lane 0): copies not yet seen landing
    auto issue_tile = [&](int j) {
        const int st = j % NST;
        const uint32_t par = static_cast<uint32_t>(j / NST) & 1u;
        const int tile = t0 + j;
        const int pb = __ldg(ltab + (tile >> sub_shift));
        if (*sm.abort_flag) return;
        if (pb < 0 || pb >= a.num_blocks) {
            atomicOr(a.status, PKV_STATUS_BAD_BLOCK_ID);
            sm.stage_bad[st] = 1;
            mbar_arrive(&sm.full[st]);
            return;
        }
        sm.stage_bad[st] = 0;
        const int prow = ((pb << sub_shift) + (tile & (a.sub - 1))) * BS;  // first pool row of the tile
        uint8_t *dst = sm.base + ly.stages + static_cast<uint32_t>(st) * 2u * kTile;
        mbar_arrive_expect_tx(&sm.full[st], 2u * kTile);
#pragma unroll
        for (int c = 0; c < kCopies; ++c) {
            tma_load_4d(dst + c * kHalf, tm_k, &sm.full[st], 0, c, h, prow);
            tma_load_4d(dst + kTile + c * kHalf, tm_v, &sm.full[st], 0, c, h, prow);
        }
        inflight |= 1u << st;
        inflight_par = (inflight_par & ~(1u << st)) | (par << st);
    };
    if (warp == 0 && lane == 0)
        for (int j = 0; j < min(NST, ntiles); ++j) issue_tile(j);

    // ---- q rows of the unit into shared memory, bf16 [kPrefixRows][D]; chunk c
    // of row R at chunk (c & ~7) | ((c ^ R) & 7), so that ldmatrix's 8 rows of one
    // chunk hit 8 distinct bank groups (padding rows are zeros)
    uint8_t *qs = sm.base + ly.prefix_q;
    const uint32_t qs_addr = smem_u32(qs);
    for (int e = ctid; e < kPrefixRows * QC; e += kConsumerWarps * 32) {
        const int R = e / QC, c = e % QC;
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (R < rows)
            val = __ldg(reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(a.q) +
                                                        (static_cast<size_t>(m0 + R / G) * a.num_q_heads + h * G +
                                                         R % G) * D) + c);
        *reinterpret_cast<uint4 *>(qs + R * (D * 2) + (((c & ~7) | ((c ^ R) & 7)) << 4)) = val;
    }
    named_barrier_sync(1, kConsumerWarps * 32);  // q staged

    // ---- this lane's two rows: fragment rows lane/4 and lane/4 + 8 of the warp,
    // i.e. unit rows R = 16 warp + lane/4 + 8 k: member R / G, q head h G + R % G
    const int tq = lane & 3;
    int row_lim[2];  // prefix tokens the row attends (0: none, or a padding row)
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int R = 16 * warp + (lane >> 2) + 8 * k;
        row_lim[k] = R < rows ? min(sm.lens[m0 + R / G], T * BS) : 0;
    }
    // ldmatrix rows of the q A fragments: matrix lane / 8 = (rows +0 / +8, chunk +0 / +1)
    const int qrow = 16 * warp + (lane & 7) + 8 * ((lane >> 3) & 1), qch = lane >> 4;

    float acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[n][k] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    const int mi = lane >> 3, r8 = lane & 7;
    const uint32_t sbase = smem_u32(sm.base) + ly.stages;

    for (int j = 0; j < ntiles; ++j) {
        const int st = j % NST;
        const uint32_t par = static_cast<uint32_t>(j / NST) & 1u;
        const uint32_t ktile = sbase + static_cast<uint32_t>(st) * 2u * kTile, vtile = ktile + kTile;
        const int tok0 = (t0 + j) * BS;  // context position of the tile's first row
        if (mbar_wait_bounded(&sm.full[st], par, sm.abort_flag, a.status) && warp == 0 && lane == 0)
            inflight &= ~(1u << st);
        const bool live = !sm.stage_bad[st] && !*sm.abort_flag;
        float sc[2][4], sc2[2][4];  // S for tokens 0-7 and 8-15: (row r: 2 tq, 2 tq + 1), (row r + 8: same)
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int k = 0; k < 4; ++k) sc[n][k] = sc2[n][k] = 0.f;
        if (live) {
#pragma unroll
            for (int kk = 0; kk < KST; ++kk) {
                uint32_t qa[4], b[4];
                const int c = 2 * kk + qch;
                ldsm_x4(qa, qs_addr + qrow * (D * 2) + (((c & ~7) | ((c ^ qrow) & 7)) << 4));
                // B fragments (k = dims, n = tokens) of tokens 0-7 and 8-15
                ldsm_x4(b, tile_addr<BS>(ktile, 8 * (mi >> 1) + r8, 2 * kk + (mi & 1)));
                // even and odd k-steps accumulate apart: four independent chains
                mma_16816((kk & 1) ? sc2[0] : sc[0], qa, b[0], b[1]);
                mma_16816((kk & 1) ? sc2[1] : sc[1], qa, b[2], b[3]);
            }
#pragma unroll
            for (int n = 0; n < 2; ++n)
#pragma unroll
                for (int k = 0; k < 4; ++k) sc[n][k] += sc2[n][k];
        }
        // base-2 logits; tokens a row does not attend are selected away
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int rr = k >> 1, t = tok0 + 8 * n + 2 * tq + (k & 1);
                sc[n][k] = (live && t < row_lim[rr]) ? sc[n][k] * a.scale_log2 : -INFINITY;
                mx[rr] = fmaxf(mx[rr], sc[n][k]);
            }
        float alpha[2], mref[2];
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            mx[rr] = fmaxf(mx[rr], __shfl_xor_sync(0xffffffffu, mx[rr], 1));
            mx[rr] = fmaxf(mx[rr], __shfl_xor_sync(0xffffffffu, mx[rr], 2));
            const float mn = fmaxf(m_run[rr], mx[rr]);
            mref[rr] = mn == -INFINITY ? 0.f : mn;  // a row with nothing attended yet: every p is 0
            alpha[rr] = fast_exp2(m_run[rr] - mref[rr]);
            m_run[rr] = mn;
        }
        // probabilities in bf16 (the sums take the rounded values), as the A operand of P.V
        uint32_t pa[4];
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const __nv_bfloat162 p2 = __floats2bfloat162_rn(fast_exp2(sc[n][2 * rr] - mref[rr]),
                                                               fast_exp2(sc[n][2 * rr + 1] - mref[rr]));
                const float2 pf = __bfloat1622float2(p2);
                l_run[rr] = l_run[rr] * (n == 0 ? alpha[rr] : 1.f) + pf.x + pf.y;
                pa[2 * n + rr] = *reinterpret_cast<const uint32_t *>(&p2);
            }
        if (__any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f)) {  // some row's maximum grew
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                acc[n][0] *= alpha[0];
                acc[n][1] *= alpha[0];
                acc[n][2] *= alpha[1];
                acc[n][3] *= alpha[1];
            }
        }
        if (live) {
            // V rows no row of the unit attends may hold anything: zero them in the fragments
            const int vmax = lim_max - tok0;
            uint32_t keep_lo = 0xffffffffu, keep_hi = 0xffffffffu;  // tokens 2 tq, 2 tq + 1 and + 8
            if (vmax < BS) {
                keep_lo = (2 * tq < vmax ? 0x0000ffffu : 0u) | (2 * tq + 1 < vmax ? 0xffff0000u : 0u);
                keep_hi = (2 * tq + 8 < vmax ? 0x0000ffffu : 0u) | (2 * tq + 9 < vmax ? 0xffff0000u : 0u);
            }
#pragma unroll
            for (int dp = 0; dp < NT / 2; ++dp) {
                uint32_t b[4];  // B fragments (k = tokens, n = dims) of dims 16 dp .. +7 and +8 .. +15
                ldsm_x4_trans(b, tile_addr<BS>(vtile, 8 * (mi & 1) + r8, 2 * dp + (mi >> 1)));
                b[0] &= keep_lo;
                b[1] &= keep_hi;
                b[2] &= keep_lo;
                b[3] &= keep_hi;
                mma_16816(acc[2 * dp], pa, b[0], b[1]);
                mma_16816(acc[2 * dp + 1], pa, b[2], b[3]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[st]);
        // warp 0 refills the stage of the previous tile once every warp is done with it
        if (warp == 0 && lane == 0 && j >= 1 && j - 1 + NST < ntiles) {
            const int jp = j - 1;
            if (mbar_wait_bounded(&sm.empty[jp % NST], static_cast<uint32_t>(jp / NST) & 1u, sm.abort_flag, a.status))
                issue_tile(jp + NST);
        }
        __syncwarp();
    }
    // with no copy in flight (possible only after a wait gave up) the stages are free
    if (warp == 0 && lane == 0)
        for (int st = 0; st < kMaxStages; ++st)
            if ((inflight >> st) & 1u) mbar_wait_drain(&sm.full[st], (inflight_par >> st) & 1u, a.status);
    named_barrier_sync(1, kConsumerWarps * 32);
    if (*sm.abort_flag || ntiles == 0) return;

    // ---- each member's table must hold the group's blocks wherever this piece
    // covers tokens the member attends (a caller's wrong grouping is reported);
    // checked after the tiles, with independent loads and one flag per thread
    {
        const int b0 = t0 >> sub_shift, nb = ((t1 - 1) >> sub_shift) - b0 + 1;
        bool bad = false;
#pragma unroll 4
        for (int e = ctid; e < (m1 - m0) * nb; e += kConsumerWarps * 32) {
            const int m = m0 + e / nb, b = b0 + e % nb;
            const int att = (min(sm.lens[m], T * BS) + BS - 1) / BS;  // tiles the member attends
            const int mine = __ldg(a.block_tables + static_cast<size_t>(m) * a.max_blocks_per_seq + b);
            bad |= (b << sub_shift) < att && mine != __ldg(ltab + b);
        }
        if (bad) atomicOr(a.status, PKV_STATUS_BAD_PREFIX_GROUP);
    }

    // ---- this piece's partial of every row that attends some of its tokens
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
        l_run[rr] += __shfl_xor_sync(0xffffffffu, l_run[rr], 1);
        l_run[rr] += __shfl_xor_sync(0xffffffffu, l_run[rr], 2);
    }
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
        if (row_lim[rr] <= t0 * BS) continue;  // attends none of this piece (or a padding row)
        const int R = 16 * warp + (lane >> 2) + 8 * rr;
        const int sq = m0 + R / G, gq = R % G;
        const size_t pr = static_cast<size_t>(a.pre_base + (sq * Hkv + h) * a.prefix_np + tp) * G + gq;
        const float inv = 1.f / l_run[rr];
        float *dst = a.o_part + pr * D + 2 * tq;
#pragma unroll
        for (int n = 0; n < NT; ++n)
            *reinterpret_cast<float2 *>(dst + 8 * n) = make_float2(acc[n][2 * rr] * inv, acc[n][2 * rr + 1] * inv);
        if (tq == 0) a.lse_part[pr] = m_run[rr] + __log2f(l_run[rr]);
    }

    // ---- count the piece in on each member's segment (its designated CTA
    // merges the segment once every piece is in: merge_grouped_segments); the
    // counters are read while the partials drain, the CAS's first guesses
    unsigned long long guess = 0;
    if (ctid < m1 - m0)
        guess = *reinterpret_cast<volatile unsigned long long *>(a.seg_count + static_cast<size_t>(m0 + ctid) * Hkv + h);
    __threadfence();
    named_barrier_sync(1, kConsumerWarps * 32);
    if (ctid < m1 - m0) {
        const int s = m0 + ctid;
        if (min(sm.lens[s], T * BS) > t0 * BS) {
            unsigned long long *cnt = a.seg_count + static_cast<size_t>(s) * Hkv + h;
            const unsigned long long ep = *sm.epoch;
            count_piece_in(cnt, ep, guess);
        }
    }
}

// The merges of the shared-prefix segments, spread over the grid: segment k
// of the launch's grouped segments (members in order, kv heads inner) is
// merged by CTA k mod gridDim.x once all its pieces are in. The last piece
// to arrive would otherwise merge them, and a prefix unit is the last for
// up to all the members of its row tile (a per-warp trace: one unit spent
// 119 us merging 16 segments while most CTAs were done). Every CTA runs this
// after its own work; the launch is cooperative, so all CTAs are resident
// and a CTA waiting for a segment never holds a slot the segment's pieces
// need. The wait is bounded: past it the status word and the abort flag are
// set and the segment is left unmerged.
template <int D>
__device__ __forceinline__ void merge_grouped_segments(const DecodeArgs &a, const Smem &sm, int C, int pcost, int BS,
                                                       int ctid) {
    const int Hkv = a.num_kv_heads;
    int ng = 0;
    for (int g = 0; g < a.num_groups; ++g) ng += (a.grp_end[g] - a.grp_begin[g]) * Hkv;
    const long long W = static_cast<long long>(Hkv) * sm.wprefix[a.num_seqs];
    for (int k = blockIdx.x; k < ng; k += gridDim.x) {
        int g = 0, r = k;  // member r / Hkv of group g, kv head r % Hkv
        while (r >= (a.grp_end[g] - a.grp_begin[g]) * Hkv) {
            r -= (a.grp_end[g] - a.grp_begin[g]) * Hkv;
            ++g;
        }
        const int s = a.grp_begin[g] + r / Hkv, h = r % Hkv;
        PieceBases pb;
        const int n = piece_bases(a, s, h, sm, W, C, pcost, BS, pb);
        if (n == 0) continue;  // no context: a zero row, written by the prologue
        // wait (bounded) until every piece is counted in; one thread polls
        if (ctid == 0) {
            const volatile unsigned long long *cnt = a.seg_count + static_cast<size_t>(s) * Hkv + h;
            const unsigned long long want = (*sm.epoch << 16) | static_cast<unsigned long long>(n);
            const uint64_t t_start = globaltimer_ns();
            while (*cnt != want) {
                if (*sm.abort_flag || globaltimer_ns() - t_start > kWaitLimitNs) {
                    *sm.abort_flag = 1;
                    atomicOr(a.status, PKV_STATUS_WAIT_TIMEOUT);
                    break;
                }
                __nanosleep(200);
            }
        }
        named_barrier_sync(1, kConsumerWarps * 32);
        if (*sm.abort_flag) return;
        __threadfence();
        merge_pieces<D>(a, pb, n, s, h, ctid);
    }
}

// The end of this CTA's part of the launch. CTA 0 advances the workspace's
// epoch for the next launch once every CTA of this one has started (each
// counted itself after reading the epoch; by CTA 0's end they all have, so
// the bounded wait is a formality) and resets the count. The next launch
// starts after this one has ended, so it needs no fence.
__device__ __forceinline__ void finish_launch(const DecodeArgs &a, const Smem &sm, int tid) {
    if (blockIdx.x != 0 || tid != 0) return;
    const volatile unsigned int *started = a.ctas_started;
    const uint64_t t0 = globaltimer_ns();
    while (*started < gridDim.x) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) {  // left for the next launch's counters to restart
            atomicOr(a.status, PKV_STATUS_WAIT_TIMEOUT);
            return;
        }
        __nanosleep(100);
    }
    *reinterpret_cast<volatile unsigned int *>(a.ctas_started) = 0u;
    *reinterpret_cast<volatile unsigned long long *>(a.launch_epoch) = (*sm.epoch + 1) & ((1ull << 48) - 1);
}

// The tensor-core path fits 128 registers per thread, so 4 CTAs (16 warps)
// share an SM; the CUDA-core path keeps its larger per-thread state.
template <int D, int BS, int GP, int MATH>
// Two-head e4m3 tiles (D = 256) take ~58 KB of shared memory: 3 CTAs per SM,
// which leaves them ~170 registers per thread.
__global__ void __launch_bounds__(kDecodeThreads, MATH == kMathCudaCore ? 1 : (MATH == kMathFp8 && D == 256) ? 3 : 4)
    paged_decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const DecodeArgs a) {
    static_assert(D == 64 || D == 128 || (D == 256 && MATH == kMathFp8), "head_dim");
    static_assert(BS == 16 || BS == 32, "block_size");
    static_assert(GP == 1 || GP == 2 || GP == 4 || GP == 8, "group");
    static_assert(MATH == kMathCudaCore || GP == 8, "the tensor-core path pads the group to 8");
    constexpr bool GROUPS = MATH == kMathTensorCoreGroups;
    extern __shared__ uint8_t smem_raw[];
    constexpr int ES = MATH == kMathFp8 ? 1 : 2;  // bytes per pool element
    const DecodeLayout ly = decode_layout(D, BS, GP, a.group, MATH != kMathCudaCore, kConsumerWarps * a.num_stages,
                                          a.num_seqs, ES, D / a.pack, MATH == kMathTensorCoreGroups);
    Smem sm;
    sm.base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    sm.full = reinterpret_cast<uint64_t *>(sm.base + ly.bars);
    sm.qfull = sm.full + kMaxStages;
    sm.stage_bad = reinterpret_cast<volatile int *>(sm.base + ly.flags);
    sm.abort_flag = sm.stage_bad + kMaxStages;
    sm.scan = reinterpret_cast<int *>(sm.base + ly.flags) + kMaxStages + 1;
    sm.merge_flag = reinterpret_cast<volatile int *>(sm.scan + 2 * kConsumerWarps);
    sm.stage_blk = const_cast<int *>(sm.merge_flag) + 1 + 4 * 2;
    sm.prefix = reinterpret_cast<int *>(sm.base + ly.prefix);
    sm.wprefix = reinterpret_cast<int *>(sm.base + ly.wprefix);
    sm.lens = reinterpret_cast<int *>(sm.base + ly.lens);
    sm.ptiles = reinterpret_cast<int *>(sm.base + ly.ptiles);
    sm.empty = sm.qfull + 2;
    sm.epoch = reinterpret_cast<volatile unsigned long long *>(sm.empty + kMaxStages);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int i = 0; i < kConsumerWarps * a.num_stages; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], kConsumerWarps);
            sm.stage_bad[i] = 0;
        }
        for (int i = 0; i < 2; ++i) mbar_init(&sm.qfull[i], 1);
        *sm.abort_flag = 0;
        sm.merge_flag[0] = 0;
        fence_mbar_init();
    }
    // The workspace's launch count (the previous launch advanced it): loaded
    // now, stored for the CTA's threads after the prologue's own loads.
    unsigned long long launch_epoch = 0;
    if (tid == 0) launch_epoch = *reinterpret_cast<volatile unsigned long long *>(a.launch_epoch);
    if (tid == 32) {
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    // The table entries of the first copies are read once the prologue has
    // split the work; meanwhile warp 2 brings this CTA's share of the launch's
    // block tables into L2 (a hint: line by line, inside the array), so those
    // reads hit L2 rather than HBM.
    if (warp == 2) {
        const size_t bytes = static_cast<size_t>(a.num_seqs) * a.max_blocks_per_seq * sizeof(int32_t);
        const size_t per = (bytes + gridDim.x - 1) / gridDim.x;
        const size_t end = min(bytes, (blockIdx.x + 1) * per);
        const char *tables = reinterpret_cast<const char *>(a.block_tables);
        for (size_t off = blockIdx.x * per + lane * 128; off < end; off += 32 * 128)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(tables + off));
    }

    // prefix[s] = blocks of sequences < s (clamped lengths), wprefix[s] = their
    // weight (blocks + piece_cost per non-empty sequence); lens[s] = clamped
    // length; ptiles[s] = tiles of its group's shared prefix, which prefix units
    // read (its blocks here are those of the rest, the suffix)
    const int S = a.num_seqs;
    const int cap = a.max_blocks_per_seq * BS * a.sub;
    const int pcost = min(max(a.piece_cost, 0), 64);  // validated on the host; a bad value moves no index
    const int per = (S + kDecodeThreads - 1) / kDecodeThreads;
    const int lo = min(S, tid * per), hi = min(S, lo + per);
    int mine = 0, mine_w = 0;
    for (int s = lo; s < hi; ++s) {
        int L = __ldg(a.context_lens + s);
        if (L < 0 || L > cap) {
            if (blockIdx.x == 0) atomicOr(a.status, PKV_STATUS_BAD_CONTEXT_LEN);
            L = min(max(L, 0), cap);
        }
        sm.lens[s] = L;
        int pt = 0;
        for (int gi = 0; gi < a.num_groups; ++gi)
            if (s >= a.grp_begin[gi] && s < a.grp_end[gi]) pt = a.grp_tiles[gi];
        sm.ptiles[s] = pt;
        // the fused append writes position L - 1 from the suffix: none inside a shared prefix
        if (pt > 0 && a.slots != nullptr && L > 0 && L <= pt * BS && blockIdx.x == 0 && __ldg(a.slots + s) >= 0)
            atomicOr(a.status, PKV_STATUS_BAD_SLOT);
        const int n = max(0, (L + BS - 1) / BS - pt);
        mine += n;
        mine_w += n > 0 ? n + pcost : 0;
    }
    int incl = mine, incl_w = mine_w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        const int yw = __shfl_up_sync(0xffffffffu, incl_w, o);
        if (lane >= o) {
            incl += y;
            incl_w += yw;
        }
    }
    if (lane == 31) {
        sm.scan[warp] = incl;
        sm.scan[4 + warp] = incl_w;
    }
    __syncthreads();
    int run = incl - mine, run_w = incl_w - mine_w;
    for (int w = 0; w < warp; ++w) {
        run += sm.scan[w];
        run_w += sm.scan[4 + w];
    }
    for (int s = lo; s < hi; ++s) {
        sm.prefix[s] = run;
        sm.wprefix[s] = run_w;
        const int n = max(0, (sm.lens[s] + BS - 1) / BS - sm.ptiles[s]);
        run += n;
        run_w += n > 0 ? n + pcost : 0;
    }
    if (tid == 0) {
        int total = 0, total_w = 0;
        for (int w = 0; w < kDecodeThreads / 32; ++w) {
            total += sm.scan[w];
            total_w += sm.scan[4 + w];
        }
        sm.prefix[S] = total;
        sm.wprefix[S] = total_w;
        *sm.epoch = launch_epoch & ((1ull << 48) - 1);
        // this CTA has read the epoch: counted as started (the added value
        // depends on the loaded one -- always 0 + 1 -- so the count cannot be
        // seen before the read is done; nobody waits for it here)
        atomicAdd(a.ctas_started, 1u + static_cast<unsigned>(launch_epoch >> 63));
    }
    __syncthreads();
    // Sequences with no context get all-zero rows (no piece covers them); CTA c
    // takes sequences c, c + C, ... so that no CTA walks the whole batch.
    for (int s = blockIdx.x; s < S; s += gridDim.x)
            if (sm.lens[s] == 0) {
                for (int e = tid; e < a.num_q_heads * (D / a.pack) / 2; e += kDecodeThreads)
                    reinterpret_cast<__nv_bfloat162 *>(static_cast<__nv_bfloat16 *>(a.out) +
                                                       static_cast<size_t>(s) * a.num_q_heads * (D / a.pack))[e] =
                        __floats2bfloat162_rn(0.f, 0.f);
                // fused append of a sequence with no context: no block computes it,
                // so its rows go straight to the pool (if the slot is in it)
                const long long slot = a.slots ? __ldg(a.slots + s) : -1;
                if (slot >= static_cast<long long>(a.num_blocks) * BS * a.sub) {
                    if (tid == 0) atomicOr(a.status, PKV_STATUS_BAD_SLOT);
                } else if (slot >= 0) {
                    const size_t row = static_cast<size_t>(a.num_kv_heads) * D;  // elements of one token's row
                    constexpr int kElems = 16 / ES;                              // elements per stored 16 bytes
                    const int chunks = static_cast<int>(row / kElems);
                    for (int e = tid; e < 2 * chunks; e += kDecodeThreads) {
                        const int kv = e / chunks, c = e % chunks;
                        const uint4 *src = reinterpret_cast<const uint4 *>(
                            static_cast<const __nv_bfloat16 *>(kv ? a.v_new : a.k_new) + s * row + c * kElems);
                        uint4 v;
                        if constexpr (ES == 2) {
                            v = __ldg(src);
                        } else {
                            const int real = (c * kElems) / (D / a.pack);  // real kv head of the chunk
                            v = quantize16_e4m3(__ldg(src), __ldg(src + 1), __ldg((kv ? a.v_scale : a.k_scale) + real));
                        }
                        *reinterpret_cast<uint4 *>(static_cast<uint8_t *>(kv ? a.v_cache : a.k_cache) +
                                                   (static_cast<size_t>(slot) * row) * ES + c * 16) = v;
                    }
                }
            }

    // CTAs [0, prefix_ctas) run the prefix units; the others split the suffix
    // blocks by weight, numbered from 0
    const long long W = static_cast<long long>(a.num_kv_heads) * sm.wprefix[S];
    const int cta = static_cast<int>(blockIdx.x) - a.prefix_ctas, C = static_cast<int>(gridDim.x) - a.prefix_ctas;
    if constexpr (GROUPS) {
        if (cta < 0) {
            prefix_unit<D>(&tm_k, &tm_v, a, sm, ly, W, C, pcost, warp, lane);
            named_barrier_sync(1, kConsumerWarps * 32);
            merge_grouped_segments<D>(a, sm, C, pcost, BS, tid);
            finish_launch(a, sm, tid);
            return;
        }
    }
    const long long x0 = blocks_below(weight_begin(cta, W, C), sm.prefix, sm.wprefix, S, a.num_kv_heads, pcost);
    const long long x1 = blocks_below(weight_begin(cta + 1, W, C), sm.prefix, sm.wprefix, S, a.num_kv_heads, pcost);
    PieceIter pieces;
    pieces.x = x0;
    pieces.x1 = x1;
    pieces.pre = sm.prefix;
    pieces.lens = sm.lens;
    pieces.ptiles = sm.ptiles;
    pieces.BS = BS;
    pieces.S = S;
    pieces.Hkv = a.num_kv_heads;

    if constexpr (MATH == kMathCudaCore) {
        decode_warp<D, BS, CoreMath<D, BS, GP>, 2, false>(&tm_k, &tm_v, a, sm, ly, pieces, x0, x1, W, pcost,
                                                   warp, lane);
    } else if constexpr (MATH == kMathTensorCore || GROUPS) {
        decode_warp<D, BS, MmaMath<D, BS>, 2, GROUPS>(&tm_k, &tm_v, a, sm, ly, pieces, x0, x1, W, pcost, warp,
                                              lane);
        if constexpr (GROUPS) {
            named_barrier_sync(1, kConsumerWarps * 32);
            merge_grouped_segments<D>(a, sm, C, pcost, BS, tid);
        }
    } else {
        static_assert(D == 128 || D == 256, "the e4m3 path reads rows of 128 or 256 codes");
        decode_warp<D, BS, Fp8Math<BS, D / 128>, 1, false>(&tm_k, &tm_v, a, sm, ly, pieces, x0, x1, W, pcost,
                                                    warp, lane);
    }
    finish_launch(a, sm, tid);
}

using KernelFn = void (*)(const CUtensorMap, const CUtensorMap, const DecodeArgs);

// The tensor-core path always pads the group to 8 (one n8 tile).
int effective_group_pad(int group_pad, int math) { return math == kMathCudaCore ? group_pad : 8; }

KernelFn pick(int D, int BS, int GP, int math) {
#define PKV_CASE(d, bs, gp, m) \
    if (D == d && BS == bs && GP == gp && math == m) return paged_decode_kernel<d, bs, gp, m>;
#define PKV_GP(d, bs)                                                                                \
    PKV_CASE(d, bs, 1, kMathCudaCore) PKV_CASE(d, bs, 2, kMathCudaCore) PKV_CASE(d, bs, 4, kMathCudaCore) \
    PKV_CASE(d, bs, 8, kMathCudaCore) PKV_CASE(d, bs, 8, kMathTensorCore)
    PKV_GP(64, 16) PKV_GP(64, 32) PKV_GP(128, 16) PKV_GP(128, 32)
    PKV_CASE(128, 16, 8, kMathFp8) PKV_CASE(128, 32, 8, kMathFp8)
    PKV_CASE(256, 16, 8, kMathFp8) PKV_CASE(256, 32, 8, kMathFp8)
    PKV_CASE(64, 16, 8, kMathTensorCoreGroups) PKV_CASE(128, 16, 8, kMathTensorCoreGroups)
#undef PKV_GP
#undef PKV_CASE
    return nullptr;
}

}  // namespace

bool decode_variant_exists(int head_dim, int block_size, int group_pad, int math) {
    return pick(head_dim, block_size, effective_group_pad(group_pad, math), math) != nullptr;
}

size_t decode_smem_bytes(int head_dim, int block_size, int group_pad, int group, int math, int num_stages,
                         int num_seqs, int pack) {
    return decode_layout(head_dim, block_size, effective_group_pad(group_pad, math), group, math != kMathCudaCore,
                         kConsumerWarps * num_stages, num_seqs, math == kMathFp8 ? 1 : 2, head_dim / pack,
                         math == kMathTensorCoreGroups)
        .total;
}

cudaError_t decode_prepare(int head_dim, int block_size, int group_pad, int math, size_t smem_bytes,
                           int *ctas_per_sm) {
    KernelFn fn = pick(head_dim, block_size, effective_group_pad(group_pad, math), math);
    if (!fn) return cudaErrorInvalidValue;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    static std::mutex mu;
    static std::set<std::tuple<int, KernelFn>> done;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!done.count({dev, fn})) {
            e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
            if (e != cudaSuccess) return e;
            done.insert({dev, fn});
        }
    }
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, fn, kDecodeThreads, smem_bytes);
}

cudaError_t decode_launch(int head_dim, int block_size, int group_pad, int math, const CUtensorMap &tm_k,
                          const CUtensorMap &tm_v, const DecodeArgs &args, int grid, size_t smem_bytes,
                          cudaStream_t stream) {
    KernelFn fn = pick(head_dim, block_size, effective_group_pad(group_pad, math), math);
    if (!fn) return cudaErrorInvalidValue;
    if (math == kMathTensorCoreGroups) {
        // CTAs of this kernel wait for one another's pieces (shared-prefix
        // merges): a cooperative launch keeps them all resident at once
        CUtensorMap k = tm_k, v = tm_v;
        DecodeArgs d = args;
        void *params[] = {&k, &v, &d};
        return cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(fn), dim3(grid), dim3(kDecodeThreads), params,
                                           smem_bytes, stream);
    }
    fn<<<grid, kDecodeThreads, smem_bytes, stream>>>(tm_k, tm_v, args);
    return cudaGetLastError();
}


}  // namespace pkv
