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
//   * Work item = (sequence, kv head, context split of P tokens). A persistent
//     grid of (SMs x resident CTAs) walks the items with a fixed stride; every
//     CTA rebuilds the prefix sum of split counts in shared memory, so no
//     planning kernel and no host/device synchronisation are needed.
//   * One producer warp streams whole KV blocks of the item's kv head into a
//     ring of shared-memory stages with TMA (one 4D tile copy per K or V block,
//     128-byte swizzle), completing on mbarriers. Block-table entries are read
//     32 at a time by the warp's lanes. The producer runs ahead across item
//     boundaries, so HBM stays busy while consumers merge.
//   * Four consumer warps take the blocks round-robin (block g of the CTA's
//     stream goes to warp g % 4) and each warp owns its own ring of R stages,
//     so every waiter sees every phase of its barriers in order (a parity wait
//     can never alias a phase two steps ahead). Each warp keeps its own
//     online-softmax state (running max m, running sum l, fp32 accumulator)
//     for all G query heads of the GQA group (Milakov & Gimelshein 2018,
//     "Online normalizer calculation for softmax"). Logits are kept in base 2
//     (scale * log2 e folded into q).
//   * At the end of an item the four warp states are merged in shared memory
//     with the log-sum-exp identity. Unsplit sequences write bf16 output
//     directly; split ones write fp32 partials + log2-sum-exp, merged by
//     lse_merge_kernel in a fixed split order.
// Every reduction order depends only on logical token positions, so results
// are bitwise reproducible and independent of where blocks sit in the pool.
#include <cstdio>
#include <mutex>
#include <set>
#include <tuple>

#include "device_utils.cuh"
#include "launch.h"

namespace pkv {
namespace {

struct Item {
    int s, split, h, tok0, tok1, b0, b1, n_split;
};

// Item u -> (sequence, split, kv head) through the shared-memory prefix sums.
template <int BS>
__device__ __forceinline__ Item decode_item(int u, const int *prefix, const DecodeArgs &a, int P, int cap) {
    Item it;
    const int v = u / a.num_kv_heads;
    it.h = u - v * a.num_kv_heads;
    int lo = 0, hi = a.num_seqs - 1;
    while (lo < hi) {  // largest s with prefix[s] <= v
        const int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= v) lo = mid;
        else hi = mid - 1;
    }
    it.s = lo;
    it.split = v - prefix[lo];
    it.n_split = prefix[lo + 1] - prefix[lo];
    int L = __ldg(a.context_lens + lo);
    L = min(max(L, 0), cap);
    it.tok0 = it.split * P;
    it.tok1 = min(L, it.tok0 + P);
    it.b0 = it.tok0 / BS;
    it.b1 = (it.tok1 > it.tok0) ? (it.tok1 + BS - 1) / BS : it.b0;
    return it;
}

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

// Shared address of 16-byte chunk `ch` of row t of a TMA tile loaded with
// SWIZZLE_128B: a row of D bf16 is D/64 lines of 128 bytes, and the chunk
// index inside a line is XORed with the line index mod 8.
template <int D>
__device__ __forceinline__ uint32_t tile_chunk_addr(uint32_t tile, int t, int ch) {
    const uint32_t line = static_cast<uint32_t>(t * (D / 64) + (ch >> 3));
    return tile + line * 128u + ((static_cast<uint32_t>(ch & 7) ^ (line & 7u)) << 4);
}

// One KV block on CUDA cores: logits, block-wise online-softmax update, P.V.
template <int D, int BS, int GP>
__device__ __forceinline__ void block_cuda_core(uint32_t ktile, uint32_t vtile, int valid, const float2 (&q2)[GP][4],
                                                float (&m_run)[GP], float &l_run, float2 (&acc)[GP][4],
                                                float2 *pscr, int tg, int ch, int lane, int g_own, bool writer) {
    constexpr int LPT = D / 8, TPP = 32 / LPT, NPASS = BS / TPP, LPG = 32 / GP;

    // logits: the LPT lanes of a token group each hold 8 dims of the row
#pragma unroll
    for (int pass = 0; pass < NPASS; ++pass) {
        const int t = pass * TPP + tg;
        const uint4 kr = lds128(tile_chunk_addr<D>(ktile, t, ch));
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

    // P.V: tokens past the context are skipped, never multiplied by p = 0
#pragma unroll
    for (int pass = 0; pass < NPASS; ++pass) {
        const int t = pass * TPP + tg;
        const uint4 vr = lds128(tile_chunk_addr<D>(vtile, t, ch));
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

struct Smem {
    uint8_t *base;
    uint64_t *full, *empty, *qfull, *qempty;
    volatile int *stage_bad;
    volatile int *abort_flag;
    int *scan;
    int *prefix;
};

template <int D, int BS, int GP>
__device__ __forceinline__ void producer_warp(const CUtensorMap *tm_k, const CUtensorMap *tm_v, const DecodeArgs &a,
                                              const Smem &sm, const DecodeLayout &ly, int total_items, int lane) {
    constexpr uint32_t kTile = BS * D * 2;
    const int R = a.num_stages;  // stages per consumer warp
    const int P = a.partition_blocks * BS, cap = a.max_blocks_per_seq * BS;
    const uint32_t qbytes = static_cast<uint32_t>(a.group * D * 2);
    int qslot = 0, gb = 0;
    uint32_t qphase = 0;
    uint32_t issued = 0, issued_par = 0, q_issued = 0, q_issued_par = 0;  // copies possibly in flight

    for (int u = blockIdx.x; u < total_items; u += gridDim.x) {
        const Item it = decode_item<BS>(u, sm.prefix, a, P, cap);
        if (lane == 0) {
            if (mbar_wait_bounded(&sm.qempty[qslot], qphase ^ 1u, sm.abort_flag, a.status) && !*sm.abort_flag) {
                const __nv_bfloat16 *src = static_cast<const __nv_bfloat16 *>(a.q) +
                                           (static_cast<size_t>(it.s) * a.num_q_heads +
                                            static_cast<size_t>(it.h) * a.group) * D;
                mbar_arrive_expect_tx(&sm.qfull[qslot], qbytes);
                bulk_load(sm.base + ly.qbuf + qslot * (GP * D * 2), src, qbytes, &sm.qfull[qslot]);
                q_issued |= 1u << qslot;
                q_issued_par = (q_issued_par & ~(1u << qslot)) | (qphase << qslot);
            }
        }
        if (++qslot == 2) {
            qslot = 0;
            qphase ^= 1u;
        }
        const int32_t *row = a.block_tables + static_cast<size_t>(it.s) * a.max_blocks_per_seq;
        for (int bb = it.b0; bb < it.b1; bb += 32) {
            const int b = bb + lane;
            const int p = (b < it.b1) ? __ldg(row + b) : 0;
            const int n = min(32, it.b1 - bb);
            for (int i = 0; i < n; ++i, ++gb) {
                const int pi = __shfl_sync(0xffffffffu, p, i);
                if (lane == 0) {
                    // block gb belongs to consumer warp gb % 4, slot (gb / 4) % R of its ring
                    const int k = gb >> 2;
                    const int stage = (gb & 3) + kConsumerWarps * (k % R);
                    const uint32_t phase = static_cast<uint32_t>(k / R) & 1u;
                    if (mbar_wait_bounded(&sm.empty[stage], phase ^ 1u, sm.abort_flag, a.status) &&
                        !*sm.abort_flag) {
                        // every earlier copy into this stage has been consumed, hence landed
                        issued &= ~(1u << stage);
                        const bool bad = pi < 0 || pi >= a.num_blocks;
                        sm.stage_bad[stage] = bad ? 1 : 0;
                        if (bad) {
                            atomicOr(a.status, PKV_STATUS_BAD_BLOCK_ID);
                            mbar_arrive(&sm.full[stage]);
                        } else {
                            uint8_t *dst = sm.base + ly.stages + static_cast<uint32_t>(stage) * 2u * kTile;
                            mbar_arrive_expect_tx(&sm.full[stage], 2u * kTile);
                            tma_load_4d(dst, tm_k, &sm.full[stage], 0, 0, it.h, pi * BS);
                            tma_load_4d(dst + kTile, tm_v, &sm.full[stage], 0, 0, it.h, pi * BS);
                            issued |= 1u << stage;
                            issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
                        }
                    }
                }
            }
        }
    }
    // Leave no copy in flight into shared memory when the CTA exits.
    if (lane == 0) {
        for (int st = 0; st < kConsumerWarps * R; ++st)
            if ((issued >> st) & 1u) mbar_wait_drain(&sm.full[st], (issued_par >> st) & 1u, a.status);
        for (int qs = 0; qs < 2; ++qs)
            if ((q_issued >> qs) & 1u) mbar_wait_drain(&sm.qfull[qs], (q_issued_par >> qs) & 1u, a.status);
    }
}

template <int D, int BS, int GP>
__device__ __forceinline__ void consumer_warps(const DecodeArgs &a, const Smem &sm, const DecodeLayout &ly,
                                               int total_items, int warp, int lane) {
    constexpr int LPT = D / 8;
    constexpr uint32_t kTile = BS * D * 2;
    const int R = a.num_stages;  // this warp's ring: stages warp, warp + 4, ..., warp + 4 (R - 1)
    const int P = a.partition_blocks * BS, cap = a.max_blocks_per_seq * BS;
    const int tg = lane / LPT, ch = lane % LPT;
    const int g_own = g_own_of<GP, LPT>(lane);
    const bool writer = (lane % (LPT / GP)) == 0;
    const uint32_t sbase = smem_u32(sm.base);
    float2 *pscr = reinterpret_cast<float2 *>(sm.base + ly.pscr) + warp * BS * GP;
    float *merge_acc = reinterpret_cast<float *>(sm.base + ly.merge_acc);
    float *merge_m = reinterpret_cast<float *>(sm.base + ly.merge_m);
    float *merge_l = reinterpret_cast<float *>(sm.base + ly.merge_l);
    const int ctid = warp * 32 + lane;
    int qslot = 0, gb_base = 0, ring = 0;
    uint32_t qphase = 0, rphase = 0;

    for (int u = blockIdx.x; u < total_items; u += gridDim.x) {
        const Item it = decode_item<BS>(u, sm.prefix, a, P, cap);
        const int nblk = it.b1 - it.b0;

        // query rows of the GQA group, pre-scaled into base-2 logits
        float2 q2[GP][4];
        mbar_wait_bounded(&sm.qfull[qslot], qphase, sm.abort_flag, a.status);
        {
            const uint32_t qa = sbase + ly.qbuf + qslot * (GP * D * 2) + ch * 16;
            const float2 sc = make_float2(a.scale_log2, a.scale_log2);
#pragma unroll
            for (int g = 0; g < GP; ++g) {
                if (g < a.group) {
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
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.qempty[qslot]);
        if (++qslot == 2) {
            qslot = 0;
            qphase ^= 1u;
        }

        float m_run[GP];
        float l_run = 0.f;
        float2 acc[GP][4];
#pragma unroll
        for (int g = 0; g < GP; ++g) {
            m_run[g] = -INFINITY;
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[g][k] = make_float2(0.f, 0.f);
        }

        // this warp's blocks of the item: item-local i with (gb_base + i) % 4 == warp
        for (int i = (warp - gb_base % kConsumerWarps + kConsumerWarps) % kConsumerWarps; i < nblk;
             i += kConsumerWarps) {
            const int stage = warp + kConsumerWarps * ring;
            const uint32_t par = rphase;
            if (++ring == R) {
                ring = 0;
                rphase ^= 1u;
            }
            mbar_wait_bounded(&sm.full[stage], par, sm.abort_flag, a.status);
            if (!sm.stage_bad[stage] && !*sm.abort_flag) {
                const int valid = min(BS, it.tok1 - (it.b0 + i) * BS);
                const uint32_t ktile = sbase + ly.stages + static_cast<uint32_t>(stage) * 2u * kTile;
                block_cuda_core<D, BS, GP>(ktile, ktile + kTile, valid, q2, m_run, l_run, acc, pscr, tg, ch, lane,
                                           g_own, writer);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[stage]);
        }
        gb_base += nblk;

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
                float4 *dst = reinterpret_cast<float4 *>(merge_acc + (warp * GP + g) * D + ch * 8);
                dst[0] = make_float4(acc[g][0].x, acc[g][0].y, acc[g][1].x, acc[g][1].y);
                dst[1] = make_float4(acc[g][2].x, acc[g][2].y, acc[g][3].x, acc[g][3].y);
            }
        }
        if (lane == 0) {
#pragma unroll
            for (int g = 0; g < GP; ++g) merge_m[warp * GP + g] = m_run[g];
        }
        if (lane < GP) merge_l[warp * GP + lane] = l_run;
        named_barrier_sync(1, kConsumerWarps * 32);

        // merge the warps' states (log-sum-exp identity) and store
        const int G = a.group;
        const bool split_mode = it.n_split > 1;
        for (int e = ctid; e < G * D / 2; e += kConsumerWarps * 32) {
            const int g = e / (D / 2), d = (e % (D / 2)) * 2;
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, merge_m[w * GP + g]);
            float ls = 0.f, a0 = 0.f, a1 = 0.f;
            if (M != -INFINITY) {
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w) {
                    const float f = fast_exp2(merge_m[w * GP + g] - M);
                    const float2 av = *reinterpret_cast<const float2 *>(merge_acc + (w * GP + g) * D + d);
                    ls += merge_l[w * GP + g] * f;
                    a0 += av.x * f;
                    a1 += av.y * f;
                }
            }
            const float o0 = ls > 0.f ? a0 / ls : 0.f;
            const float o1 = ls > 0.f ? a1 / ls : 0.f;
            const size_t row = static_cast<size_t>(it.s) * a.num_q_heads + static_cast<size_t>(it.h) * G + g;
            if (!split_mode) {
                *reinterpret_cast<__nv_bfloat162 *>(static_cast<__nv_bfloat16 *>(a.out) + row * D + d) =
                    __floats2bfloat162_rn(o0, o1);
            } else {
                const size_t pr = row * a.n_split + it.split;
                *reinterpret_cast<float2 *>(a.o_part + pr * D + d) = make_float2(o0, o1);
                if (d == 0) a.lse_part[pr] = ls > 0.f ? M + __log2f(ls) : -INFINITY;
            }
        }
        named_barrier_sync(1, kConsumerWarps * 32);
    }
}

template <int D, int BS, int GP>
__global__ void __launch_bounds__(kDecodeThreads)
    paged_decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const DecodeArgs a) {
    static_assert(D == 64 || D == 128, "head_dim");
    static_assert(BS == 16 || BS == 32, "block_size");
    static_assert(GP == 1 || GP == 2 || GP == 4 || GP == 8, "group");
    extern __shared__ uint8_t smem_raw[];
    const DecodeLayout ly = decode_layout(D, BS, GP, kConsumerWarps * a.num_stages, a.num_seqs);
    Smem sm;
    sm.base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    sm.full = reinterpret_cast<uint64_t *>(sm.base + ly.bars);
    sm.empty = sm.full + kMaxStages;
    sm.qfull = sm.empty + kMaxStages;
    sm.qempty = sm.qfull + 2;
    sm.stage_bad = reinterpret_cast<volatile int *>(sm.base + ly.flags);
    sm.abort_flag = sm.stage_bad + kMaxStages;
    sm.scan = reinterpret_cast<int *>(sm.base + ly.flags) + kMaxStages + 1;
    sm.prefix = reinterpret_cast<int *>(sm.base + ly.prefix);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int i = 0; i < kConsumerWarps * a.num_stages; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], 1);
            sm.stage_bad[i] = 0;
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.qfull[i], 1);
            mbar_init(&sm.qempty[i], kConsumerWarps);
        }
        *sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kConsumerWarps && lane == 0) {
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }

    // prefix[s] = number of (split) items of sequences < s; every sequence has >= 1
    const int S = a.num_seqs;
    const int P = a.partition_blocks * BS, cap = a.max_blocks_per_seq * BS;
    const int per = (S + kDecodeThreads - 1) / kDecodeThreads;
    const int lo = min(S, tid * per), hi = min(S, lo + per);
    int mine = 0;
    for (int s = lo; s < hi; ++s) {
        int L = __ldg(a.context_lens + s);
        if (L < 0 || L > cap) {
            if (blockIdx.x == 0) atomicOr(a.status, PKV_STATUS_BAD_CONTEXT_LEN);
            L = min(max(L, 0), cap);
        }
        mine += L > 0 ? (L + P - 1) / P : 1;
    }
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) sm.scan[warp] = incl;
    __syncthreads();
    int run = incl - mine;
    for (int w = 0; w < warp; ++w) run += sm.scan[w];
    for (int s = lo; s < hi; ++s) {
        sm.prefix[s] = run;
        int L = min(max(__ldg(a.context_lens + s), 0), cap);
        run += L > 0 ? (L + P - 1) / P : 1;
    }
    if (tid == 0) {
        int total = 0;
        for (int w = 0; w < kDecodeThreads / 32; ++w) total += sm.scan[w];
        sm.prefix[S] = total;
    }
    __syncthreads();
    const int total_items = sm.prefix[S] * a.num_kv_heads;

    if (warp == kConsumerWarps) {
        producer_warp<D, BS, GP>(&tm_k, &tm_v, a, sm, ly, total_items, lane);
    } else {
        consumer_warps<D, BS, GP>(a, sm, ly, total_items, warp, lane);
    }
}

// Merge of split partial results: out = sum_p 2^(lse_p - M) o_p / sum_p 2^(lse_p - M),
// p = 0 .. n_split(s) - 1 in order. One warp per (sequence, query head).
template <int D>
__global__ void __launch_bounds__(256) lse_merge_kernel(const DecodeArgs a, int BS) {
    constexpr int PER = D / 32;
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= a.num_seqs * a.num_q_heads) return;
    const int s = row / a.num_q_heads;
    const int P = a.partition_blocks * BS, cap = a.max_blocks_per_seq * BS;
    const int L = min(max(__ldg(a.context_lens + s), 0), cap);
    const int n = (L + P - 1) / P;
    if (n <= 1) return;  // written directly by the decode kernel
    const float *lse = a.lse_part + static_cast<size_t>(row) * a.n_split;
    float M = -INFINITY;
    for (int p = lane; p < n; p += 32) M = fmaxf(M, lse[p]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float den = 0.f;
    for (int p = lane; p < n; p += 32) den += fast_exp2(lse[p] - M);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    float acc[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] = 0.f;
    const float *op = a.o_part + static_cast<size_t>(row) * a.n_split * D + lane * PER;
    for (int p = 0; p < n; ++p) {
        const float w = fast_exp2(lse[p] - M);
#pragma unroll
        for (int i = 0; i < PER; ++i) acc[i] += w * op[static_cast<size_t>(p) * D + i];
    }
    __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(a.out) + static_cast<size_t>(row) * D + lane * PER;
#pragma unroll
    for (int i = 0; i < PER; i += 2)
        *reinterpret_cast<__nv_bfloat162 *>(out + i) = __floats2bfloat162_rn(acc[i] / den, acc[i + 1] / den);
}

using KernelFn = void (*)(const CUtensorMap, const CUtensorMap, const DecodeArgs);

KernelFn pick(int D, int BS, int GP, int math) {
    if (math != kMathCudaCore) return nullptr;
#define PKV_CASE(d, bs, gp) \
    if (D == d && BS == bs && GP == gp) return paged_decode_kernel<d, bs, gp>;
#define PKV_GP(d, bs) PKV_CASE(d, bs, 1) PKV_CASE(d, bs, 2) PKV_CASE(d, bs, 4) PKV_CASE(d, bs, 8)
    PKV_GP(64, 16) PKV_GP(64, 32) PKV_GP(128, 16) PKV_GP(128, 32)
#undef PKV_GP
#undef PKV_CASE
    return nullptr;
}

}  // namespace

bool decode_variant_exists(int head_dim, int block_size, int group_pad, int math) {
    return pick(head_dim, block_size, group_pad, math) != nullptr;
}

size_t decode_smem_bytes(int head_dim, int block_size, int group_pad, int math, int num_stages, int num_seqs) {
    (void)math;
    return decode_layout(head_dim, block_size, group_pad, kConsumerWarps * num_stages, num_seqs).total;
}

cudaError_t decode_prepare(int head_dim, int block_size, int group_pad, int math, size_t smem_bytes,
                           int *ctas_per_sm) {
    KernelFn fn = pick(head_dim, block_size, group_pad, math);
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
    KernelFn fn = pick(head_dim, block_size, group_pad, math);
    if (!fn) return cudaErrorInvalidValue;
    fn<<<grid, kDecodeThreads, smem_bytes, stream>>>(tm_k, tm_v, args);
    return cudaGetLastError();
}

cudaError_t lse_merge_launch(int head_dim, int block_size, const DecodeArgs &args, cudaStream_t stream) {
    const int rows = args.num_seqs * args.num_q_heads;
    const int grid = (rows + 7) / 8;
    if (grid == 0) return cudaSuccess;
    if (head_dim == 64) lse_merge_kernel<64><<<grid, 256, 0, stream>>>(args, block_size);
    else lse_merge_kernel<128><<<grid, 256, 0, stream>>>(args, block_size);
    return cudaGetLastError();
}

}  // namespace pkv
