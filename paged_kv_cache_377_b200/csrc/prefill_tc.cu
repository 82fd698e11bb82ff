// prefill_tc.cu -- multi-query paged attention on the 5th-generation tensor
// cores (tcgen05.mma, accumulators in tensor memory).
//
// Same operation as prefill.cu (chunked prefill / mixed batches: query i of a
// sequence's n-token chunk attends causally to positions 0 .. L - n + i).
// One CTA per (128 rows of (query token, group head), sequence, kv head):
//   - TMA loads the CTA's 128 query rows once (a 5D box over q viewed as
//     [T][Hkv][G][D]) and streams the context through a 2-stage ring of 64
//     tokens (64 / BS paged blocks) of K and V, 128-byte swizzled tiles;
//   - one thread issues S = Q K^T (M 128, N 64, K = head_dim in steps of 16)
//     into tensor memory and commits it to an mbarrier;
//   - each of the 128 threads owns one query row (one tensor-memory lane):
//     it loads its 64 logits, masks the positions its query may not see,
//     updates its running maximum and sum, writes its row of P in bf16 to
//     shared memory (the operand layout), and rescales its row of O in tensor
//     memory when its maximum has grown by more than 2^8 since the last
//     rescale (otherwise the stale maximum stays the reference: every P is
//     then < 2^8 and the result is the same);
//   - the thread issues O += P V (M 128, N = head_dim, K 64 tokens; V read as
//     an N-major operand straight from its TMA tile) and commits it.
// All waits are bounded (1 s); a wait that gives up flags the status word,
// the CTA drains what it issued and frees its tensor memory.
#include <cuda_bf16.h>

#include "device_utils.cuh"
#include "launch.h"

namespace pkv {
namespace {

constexpr int kTcThreads = 128;
constexpr int kTcRows = 128;    // query rows per CTA (= tensor-memory lanes)
constexpr int kTcTokens = 64;   // context tokens per iteration
// Tensor-memory columns: S takes 64, O head_dim; allocations are powers of two.
__host__ __device__ constexpr uint32_t tmem_cols(int D) { return D == 64 ? 128u : 256u; }

__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    // UMMA shared-memory matrix descriptor: start, leading / stride byte offsets
    // (16-byte units), version 1, 128-byte swizzle.
    return static_cast<uint64_t>((addr >> 4) & 0x3fffu) | (static_cast<uint64_t>((lbo >> 4) & 0x3fffu) << 16) |
           (static_cast<uint64_t>((sbo >> 4) & 0x3fffu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor: bf16 x bf16 -> fp32, A K-major, B K- or N-major.
__host__ __device__ constexpr uint32_t instr_desc(int M, int N, bool b_n_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((b_n_major ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void umma(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}" ::"r"(tmem_d),
        "l"(da), "l"(db), "r"(idesc), "r"(accumulate), "r"(0u)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's lane (warp-collective: the
// warp reconverges first).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    __syncwarp();
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
        "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
          "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
    __syncwarp();
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
        "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
        "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
        "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
        "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
        "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])),
        "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
        "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])),
        "r"(__float_as_uint(v[23])), "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])),
        "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])),
        "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 5D TMA tile load (no multicast).
__device__ __forceinline__ void tma_load_5d(void *dst, const CUtensorMap *map, uint64_t *bar, int c0, int c1, int c2,
                                            int c3, int c4) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(smem_u32(bar))
        : "memory");
}

template <int D, int BS>
__global__ void __launch_bounds__(kTcThreads, 1)
    paged_prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, const PrefillArgs a) {
    static_assert(D == 64 || D == 128, "head_dim");
    static_assert(BS == 16 || BS == 32, "block_size");
    constexpr int HALVES = D / 64;                        // 128-byte column slices of a row
    constexpr uint32_t kHalfKV = kTcTokens * 128;         // one slice of 64 tokens
    constexpr uint32_t kTileKV = HALVES * kHalfKV;        // K (or V) of one stage
    constexpr uint32_t kQHalf = kTcRows * 128;
    constexpr int BPI = kTcTokens / BS;                   // paged blocks per iteration

    const int tile = blockIdx.x, s = blockIdx.y, h = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5;

    const int q0 = __ldg(a.query_start + s), q1 = __ldg(a.query_start + s + 1);
    const int n = q1 - q0;
    const int L = __ldg(a.context_lens + s);
    if (n < 0 || q0 < 0 || q1 > a.num_tokens || n > L || L > a.max_blocks_per_seq * BS ||
        n > a.max_query_len) {
        if (tile == 0 && h == 0 && tid == 0) atomicOr(a.status, PKV_STATUS_BAD_CONTEXT_LEN);
        return;
    }
    const int G = a.group;  // 1, 2, 4 or 8: 128 rows are 128 / G whole query tokens
    const int rows = n * G;
    const int row0 = tile * kTcRows;
    if (row0 >= rows) return;
    const int i0 = row0 / G;  // first query token of the tile
    const int last_query = (min(row0 + kTcRows, rows) - 1) / G;
    const int ntok = L - n + last_query + 1;              // positions 0 .. p of the last row
    const int nit = (ntok + kTcTokens - 1) / kTcTokens;   // iterations of 64 tokens

    // ---- shared memory: Q | stage 0 K, V | stage 1 K, V | P | table | barriers
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sq = base;
    uint8_t *skv = sq + HALVES * kQHalf;
    uint8_t *sp = skv + 2 * 2 * kTileKV;
    int *table = reinterpret_cast<int *>(sp + kTcRows * 128);
    uint64_t *bars = reinterpret_cast<uint64_t *>(table + ((a.max_blocks_per_seq + 3) & ~3));
    uint64_t *q_full = bars, *kv_full = bars + 1, *s_full = bars + 3, *pv_done = bars + 4;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 6);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *stage_bad = abort_flag + 1;  // [2]

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(tmem_cols(D)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
        tc_fence_before();
    }
    if (tid == 32) {
        mbar_init(q_full, 1);
        mbar_init(&kv_full[0], 1);
        mbar_init(&kv_full[1], 1);
        mbar_init(s_full, 1);
        mbar_init(pv_done, 1);
        *abort_flag = 0;
        stage_bad[0] = stage_bad[1] = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    for (int b = tid; b < nit * BPI && b < a.max_blocks_per_seq; b += kTcThreads)
        table[b] = __ldg(a.block_tables + static_cast<size_t>(s) * a.max_blocks_per_seq + b);
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const uint32_t t_s = tbase, t_o = tbase + 64;  // S: columns 0-63, O: 64 .. 64 + D

    // ---- producer: thread 0 issues every copy and MMA
    uint32_t kv_issued = 0, kv_par = 0;  // stages with a K/V copy in flight, and its phase
    int s_commits = 0, pv_commits = 0;    // MMA batches committed to s_full / pv_done
    auto issue_kv = [&](int it) {
        const int st = it & 1;
        uint8_t *kdst = skv + st * 2 * kTileKV, *vdst = kdst + kTileKV;
        int bad = 0;
        uint32_t bytes = 0;
        for (int j = 0; j < BPI; ++j) {
            const int b = it * BPI + j;
            if (b * BS >= ntok) break;
            const int p = table[b];
            if (p < 0 || p >= a.num_blocks) {
                bad = 1;
                continue;
            }
            bytes += 2u * HALVES * BS * 128;
        }
        stage_bad[st] = bad;
        if (bad) atomicOr(a.status, PKV_STATUS_BAD_BLOCK_ID);
        mbar_arrive_expect_tx(&kv_full[st], bytes);
        for (int j = 0; j < BPI; ++j) {
            const int b = it * BPI + j;
            if (b * BS >= ntok) break;
            const int p = table[b];
            if (p < 0 || p >= a.num_blocks) continue;
#pragma unroll
            for (int hf = 0; hf < HALVES; ++hf) {
                tma_load_4d(kdst + hf * kHalfKV + j * BS * 128, &tm_k, &kv_full[st], 0, hf, h, p * BS);
                tma_load_4d(vdst + hf * kHalfKV + j * BS * 128, &tm_v, &kv_full[st], 0, hf, h, p * BS);
            }
        }
        kv_issued |= 1u << st;
        kv_par = (kv_par & ~(1u << st)) | ((static_cast<uint32_t>(it >> 1) & 1u) << st);
    };
    if (tid == 0) {
        mbar_arrive_expect_tx(q_full, HALVES * kQHalf);
#pragma unroll
        for (int hf = 0; hf < HALVES; ++hf)
            tma_load_5d(sq + hf * kQHalf, &tm_q, q_full, 0, hf, 0, h, q0 + i0);
        issue_kv(0);
        if (nit > 1) issue_kv(1);
    }

    // ---- this thread's query row
    const int r = tid;                                  // tensor-memory lane / row of the tile
    const int row = row0 + r;
    const bool live = row < rows;
    const int qi = min(row, rows - 1) / G;              // query token of the row
    const int p_row = L - n + qi;                       // last position it may see
    const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
    float m_ref = -INFINITY, l_run = 0.f;
    bool ok = mbar_wait_bounded(q_full, 0, abort_flag, a.status);
    uint32_t s_par = 0, pv_par = 0;

    for (int it = 0; it < nit; ++it) {
        const int st = it & 1;
        const uint32_t kbase = smem_u32(skv + st * 2 * kTileKV), vbase = kbase + kTileKV;
        // S = Q K^T (thread 0), once this stage has landed
        if (tid == 0 && ok && !*abort_flag) {
            if (mbar_wait_bounded(&kv_full[st], (kv_par >> st) & 1u, abort_flag, a.status)) {
                kv_issued &= ~(1u << st);
                tc_fence_after();
#pragma unroll
                for (int hf = 0; hf < HALVES; ++hf)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma(t_s, smem_desc(smem_u32(sq) + hf * kQHalf + kk * 32, 16, 1024),
                             smem_desc(kbase + hf * kHalfKV + kk * 32, 16, 1024), instr_desc(128, 64, false),
                             (hf | kk) != 0);
                umma_commit(s_full);
                ++s_commits;
            }
        }
        ok = ok && mbar_wait_bounded(s_full, s_par, abort_flag, a.status);
        s_par ^= 1u;
        tc_fence_after();
        // softmax over this row's 64 logits
        float x[64];
        {
            float t0[32], t1[32];
            tmem_ld32(t_s + lane_addr, t0);
            tmem_ld32(t_s + lane_addr + 32, t1);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                x[i] = t0[i];
                x[32 + i] = t1[i];
            }
        }
        float mx = -INFINITY;
#pragma unroll
        for (int t = 0; t < 64; ++t) {
            const int pos = it * kTcTokens + t;
            x[t] = pos <= p_row ? x[t] * a.scale_log2 : -INFINITY;
            mx = fmaxf(mx, x[t]);
        }
        // the reference maximum moves only when it would be exceeded by more than 2^8
        float m_new = m_ref;
        if (mx > m_ref + 8.f) m_new = mx;
        const float alpha = fast_exp2(m_ref - m_new);  // 0 on the first update
        // O += P V of the previous iteration must be done before O is rescaled or P rewritten
        if (it > 0) {
            ok = ok && mbar_wait_bounded(pv_done, pv_par, abort_flag, a.status);
            pv_par ^= 1u;
            tc_fence_after();
            // this row's O in tensor memory times alpha; tcgen05.ld / st are
            // warp-collective, so the whole warp takes the branch together
            if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
                for (int cb = 0; cb < D / 32; ++cb) {
                    float o[32];
                    tmem_ld32(t_o + lane_addr + cb * 32, o);
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] *= alpha;
                    tmem_st32(t_o + lane_addr + cb * 32, o);
                }
            }
        }
        // P in bf16, written in the 128-byte swizzled operand layout (row r, 8 chunks)
        float ps = 0.f;
        uint8_t *prow = sp + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const __nv_bfloat162 v2 =
                    __floats2bfloat162_rn(fast_exp2(x[8 * c + 2 * e] - m_new), fast_exp2(x[8 * c + 2 * e + 1] - m_new));
                ps += __low2float(v2) + __high2float(v2);
                w[e] = *reinterpret_cast<const uint32_t *>(&v2);
            }
            *reinterpret_cast<uint4 *>(prow + ((c ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        l_run = l_run * alpha + ps;
        m_ref = m_new;
        // V rows past the tile's last position (past the context, or in blocks
        // not loaded) may hold anything: zero them so that P = 0 there
        // multiplies zeros
        if (it == nit - 1 && ok) {
            const int valid = ntok - it * kTcTokens;  // tokens of this iteration the tile may see
            for (int e = tid; e < HALVES * kTcTokens * 8; e += kTcThreads) {
                const int hf = e / (kTcTokens * 8), t = (e / 8) % kTcTokens, c = e % 8;
                if (t >= valid)
                    *reinterpret_cast<uint4 *>(skv + st * 2 * kTileKV + kTileKV + hf * kHalfKV + t * 128 +
                                               ((c ^ (t & 7)) << 4)) = make_uint4(0u, 0u, 0u, 0u);
            }
        }
        fence_proxy_async_shared();  // P and the zeroed V rows, before the MMA reads them
        tc_fence_before();
        __syncthreads();
        // O += P V (thread 0), then refill this stage two iterations ahead
        if (tid == 0 && ok && !*abort_flag) {
            tc_fence_after();
            if (!stage_bad[st]) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma(t_o, smem_desc(smem_u32(sp) + kk * 32, 16, 1024),
                         smem_desc(vbase + kk * 16 * 128, kHalfKV, 1024), instr_desc(128, D, true),
                         (it | kk) != 0);
            }
            umma_commit(pv_done);
            ++pv_commits;
            if (it + 2 < nit) {
                // the stage is free once this MMA has read it
                if (mbar_wait_bounded(pv_done, pv_par, abort_flag, a.status)) issue_kv(it + 2);
            }
        }
    }
    // the last O += P V
    if (nit > 0) {
        ok = ok && mbar_wait_bounded(pv_done, pv_par, abort_flag, a.status);
        tc_fence_after();
    }
    // drain copies and MMAs still in flight (only after a wait gave up): a
    // commit's arrival covers every MMA the thread issued before it
    if (tid == 0) {
        for (int st = 0; st < 2; ++st)
            if ((kv_issued >> st) & 1u) mbar_wait_drain(&kv_full[st], (kv_par >> st) & 1u, a.status);
        if (s_commits > 0) mbar_wait_drain(s_full, static_cast<uint32_t>(s_commits - 1) & 1u, a.status);
        if (pv_commits > 0) mbar_wait_drain(pv_done, static_cast<uint32_t>(pv_commits - 1) & 1u, a.status);
    }

    // ---- normalise and store this row (every lane reads its lane of O: the
    // tensor-memory load is warp-collective; only real rows are stored)
    const bool store = ok && !*abort_flag && live;
    const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
    __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(a.out) +
                         (static_cast<size_t>(q0 + qi) * a.num_q_heads + h * G + min(row, rows - 1) % G) * D;
#pragma unroll
    for (int cb = 0; cb < D / 32; ++cb) {
        float o[32];
        tmem_ld32(t_o + lane_addr + cb * 32, o);
        if (store) {
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
                uint4 v;
                const __nv_bfloat162 a0 = __floats2bfloat162_rn(o[i] * inv, o[i + 1] * inv);
                const __nv_bfloat162 a1 = __floats2bfloat162_rn(o[i + 2] * inv, o[i + 3] * inv);
                const __nv_bfloat162 a2 = __floats2bfloat162_rn(o[i + 4] * inv, o[i + 5] * inv);
                const __nv_bfloat162 a3 = __floats2bfloat162_rn(o[i + 6] * inv, o[i + 7] * inv);
                v.x = *reinterpret_cast<const uint32_t *>(&a0);
                v.y = *reinterpret_cast<const uint32_t *>(&a1);
                v.z = *reinterpret_cast<const uint32_t *>(&a2);
                v.w = *reinterpret_cast<const uint32_t *>(&a3);
                *reinterpret_cast<uint4 *>(dst + cb * 32 + i) = v;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tbase), "r"(tmem_cols(D)));
    }
}

using PrefillTcFn = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const PrefillArgs);

PrefillTcFn pick_tc(int D, int BS) {
    if (D == 64 && BS == 16) return paged_prefill_tc_kernel<64, 16>;
    if (D == 64 && BS == 32) return paged_prefill_tc_kernel<64, 32>;
    if (D == 128 && BS == 16) return paged_prefill_tc_kernel<128, 16>;
    if (D == 128 && BS == 32) return paged_prefill_tc_kernel<128, 32>;
    return nullptr;
}

}  // namespace

size_t prefill_tc_smem_bytes(int head_dim, int max_blocks_per_seq) {
    const size_t halves = head_dim / 64;
    return halves * kTcRows * 128 + 2 * 2 * halves * kTcTokens * 128 + kTcRows * 128 +
           static_cast<size_t>((max_blocks_per_seq + 3) & ~3) * 4 + 6 * 8 + 32 + 1024;
}

cudaError_t prefill_tc_launch(int head_dim, int block_size, const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                              const CUtensorMap &tm_v, const PrefillArgs &args, int tiles, size_t smem_bytes,
                              cudaStream_t stream) {
    PrefillTcFn fn = pick_tc(head_dim, block_size);
    if (!fn) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_bytes));
    if (e != cudaSuccess) return e;
    const dim3 grid(static_cast<unsigned>(tiles), static_cast<unsigned>(args.num_seqs),
                    static_cast<unsigned>(args.num_kv_heads));
    fn<<<grid, kTcThreads, smem_bytes, stream>>>(tm_q, tm_k, tm_v, args);
    return cudaGetLastError();
}

int prefill_tc_rows_per_cta() { return kTcRows; }

}  // namespace pkv
