// prefill.cu -- multi-query paged attention: chunked prefill and mixed batches.
//
// "vLLM Fundamentals: Paged Attention and Batching", section "Continuous
// Batching": long prefills are cut into chunks under a per-step token budget
// and batched with decodes, each request processing some number of tokens per
// step. Sequence s brings n_s query tokens, the last n_s of its L_s tokens
// (already appended to the paged pool); query i sits at position
// p = L_s - n_s + i and attends causally to positions 0 .. p. Decode is n_s = 1.
//
// This is the mma.sync kernel: the fallback of paged_attn_prefill for groups
// the tcgen05 kernel (prefill_tc.cu) cannot tile (other than 1, 2, 4, 8) and
// for block tables too long for its shared memory, and kernel 1 of
// paged_attn_prefill_ex.
//
// Structure: one CTA per (64-row tile, sequence, kv head); a row is a (query
// token, group head) pair, row = i * G + g, so the GQA group shares every K/V
// tile. 4 warps x 16 rows. The CTA streams the blocks its last row needs
// through a 2-stage ring of TMA tile copies (the decode kernel's tensor maps
// and 128-byte swizzled tiles), each completing on an mbarrier with a bounded
// wait; all warps compute on a stage, meet at a barrier, and thread 0 refills
// it two blocks ahead. Per block and warp (mma.sync m16n8k16 bf16, fp32
// accumulate, FlashAttention-2 style): S = Q K^T with the warp's Q fragments in
// registers and K as the B operand by ldmatrix, causal mask, online softmax in
// base 2, P converted in registers into the A operand of O += P V with V as
// the B operand by ldmatrix .trans.
#include <cuda_bf16.h>

#include "device_utils.cuh"
#include "launch.h"
#include "mma_utils.cuh"

namespace pkv {
namespace {

constexpr int kPrefillWarps = 4;
constexpr int kPrefillThreads = kPrefillWarps * 32;
constexpr int kRowsPerCta = kPrefillWarps * 16;
constexpr int kPrefillStages = 2;

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}

template <int D, int BS>
__global__ void __launch_bounds__(kPrefillThreads, 2)
    paged_prefill_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                         const PrefillArgs a) {
    static_assert(D == 64 || D == 128, "head_dim");
    static_assert(BS == 16 || BS == 32, "block_size");
    constexpr uint32_t kTile = BS * D * 2;
    constexpr uint32_t kHalf = BS * 128;
    constexpr int KS = D / 16;  // k-steps of Q K^T
    constexpr int NT = BS / 8;  // token tiles of S
    constexpr int DN = D / 8;   // dim tiles of O

    const int tile = blockIdx.x, s = blockIdx.y, h = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // ---- the sequence: its chunk of queries and its causal extent (uniform per CTA)
    const int q0 = __ldg(a.query_start + s), q1 = __ldg(a.query_start + s + 1);
    const int n = q1 - q0;
    const int L = __ldg(a.context_lens + s);
    if (n < 0 || q0 < 0 || q1 > a.num_tokens || n > L || L > a.max_blocks_per_seq * BS ||
        n > a.max_query_len) {
        if (tile == 0 && h == 0 && tid == 0) atomicOr(a.status, PKV_STATUS_BAD_CONTEXT_LEN);
        return;
    }
    const int G = a.group;
    const int rows = n * G;
    const int row0 = tile * kRowsPerCta;
    if (row0 >= rows) return;
    const int last_query = (min(row0 + kRowsPerCta, rows) - 1) / G;
    const int nb = (L - n + last_query) / BS + 1;  // blocks holding positions 0 .. p of the last row

    // ---- shared memory: [stage][K, V] tiles | table row | barriers and flags
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    int *table = reinterpret_cast<int *>(base + kPrefillStages * 2 * kTile);
    uint64_t *full = reinterpret_cast<uint64_t *>(base + kPrefillStages * 2 * kTile +
                                                  ((a.max_blocks_per_seq * 4 + 15) / 16) * 16);
    volatile int *stage_bad = reinterpret_cast<volatile int *>(full + kPrefillStages);
    volatile int *abort_flag = stage_bad + kPrefillStages;

    if (tid == 0) {
        for (int i = 0; i < kPrefillStages; ++i) {
            mbar_init(&full[i], 1);
            stage_bad[i] = 0;
        }
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    for (int b = tid; b < nb; b += kPrefillThreads) {
        const int p = __ldg(a.block_tables + static_cast<size_t>(s) * a.max_blocks_per_seq + b);
        table[b] = p;
    }
    __syncthreads();

    const uint32_t sbase = smem_u32(base);
    uint32_t inflight = 0, inflight_par = 0;  // thread 0: stages with a copy not yet seen landing
    auto issue = [&](int b) {                 // thread 0: block b into stage b % 2
        const int st = b % kPrefillStages;
        const int p = table[b];
        const bool bad = p < 0 || p >= a.num_blocks;
        stage_bad[st] = bad ? 1 : 0;
        if (bad) {
            atomicOr(a.status, PKV_STATUS_BAD_BLOCK_ID);
            mbar_arrive(&full[st]);
            return;
        }
        uint8_t *dst = base + static_cast<uint32_t>(st) * 2u * kTile;
        mbar_arrive_expect_tx(&full[st], 2u * kTile);
#pragma unroll
        for (int half = 0; half < D / 64; ++half) {
            tma_load_4d(dst + half * kHalf, &tm_k, &full[st], 0, half, h, p * BS);
            tma_load_4d(dst + kTile + half * kHalf, &tm_v, &full[st], 0, half, h, p * BS);
        }
        inflight |= 1u << st;
        inflight_par = (inflight_par & ~(1u << st)) | ((static_cast<uint32_t>(b / kPrefillStages) & 1u) << st);
    };
    if (tid == 0) {
        issue(0);
        if (nb > 1) issue(1);
    }

    // ---- this warp's 16 rows: Q fragments (A operand) and causal positions
    const int gl = lane >> 2, t4 = lane & 3;
    const int r_lo = min(row0 + warp * 16 + gl, rows - 1), r_hi = min(row0 + warp * 16 + gl + 8, rows - 1);
    const bool st_lo = row0 + warp * 16 + gl < rows, st_hi = row0 + warp * 16 + gl + 8 < rows;
    const int i_lo = r_lo / G, i_hi = r_hi / G;
    const int p_lo = L - n + i_lo, p_hi = L - n + i_hi;
    const size_t qrow_lo = (static_cast<size_t>(q0 + i_lo) * a.num_q_heads + h * G + r_lo % G) * D;
    const size_t qrow_hi = (static_cast<size_t>(q0 + i_hi) * a.num_q_heads + h * G + r_hi % G) * D;
    const uint32_t *qw = reinterpret_cast<const uint32_t *>(a.q);
    uint32_t qa[KS][4];
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
        qa[ks][0] = __ldg(qw + (qrow_lo + 16 * ks + 2 * t4) / 2);
        qa[ks][1] = __ldg(qw + (qrow_hi + 16 * ks + 2 * t4) / 2);
        qa[ks][2] = __ldg(qw + (qrow_lo + 16 * ks + 8 + 2 * t4) / 2);
        qa[ks][3] = __ldg(qw + (qrow_hi + 16 * ks + 8 + 2 * t4) / 2);
    }
    float o[DN][4];
#pragma unroll
    for (int dn = 0; dn < DN; ++dn)
#pragma unroll
        for (int k = 0; k < 4; ++k) o[dn][k] = 0.f;
    float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;

    for (int b = 0; b < nb; ++b) {
        const int st = b % kPrefillStages;
        const uint32_t par = static_cast<uint32_t>(b / kPrefillStages) & 1u;
        const bool landed = mbar_wait_bounded(&full[st], par, abort_flag, a.status);
        if (tid == 0 && landed) inflight &= ~(1u << st);
        if (landed && !stage_bad[st] && !*abort_flag) {
            const uint32_t ktile = sbase + static_cast<uint32_t>(st) * 2u * kTile, vtile = ktile + kTile;
            // S = Q K^T: ldmatrix of 8 token rows x 4 chunks gives the B fragments of two k-steps
            float sc[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                for (int k = 0; k < 4; ++k) sc[nt][k] = 0.f;
#pragma unroll
                for (int kq = 0; kq < D / 32; ++kq) {
                    uint32_t r[4];
                    ldsm_x4(r, tile_addr<BS>(ktile, 8 * nt + (lane & 7), 4 * kq + (lane >> 3)));
                    mma_16816(sc[nt], qa[2 * kq], r[0], r[1]);
                    mma_16816(sc[nt], qa[2 * kq + 1], r[2], r[3]);
                }
            }
            // base-2 logits with the causal mask (positions past a row's own are -inf)
            float mx_lo = -INFINITY, mx_hi = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int tp = b * BS + 8 * nt + 2 * t4;
                sc[nt][0] = tp <= p_lo ? sc[nt][0] * a.scale_log2 : -INFINITY;
                sc[nt][1] = tp + 1 <= p_lo ? sc[nt][1] * a.scale_log2 : -INFINITY;
                sc[nt][2] = tp <= p_hi ? sc[nt][2] * a.scale_log2 : -INFINITY;
                sc[nt][3] = tp + 1 <= p_hi ? sc[nt][3] * a.scale_log2 : -INFINITY;
                mx_lo = fmaxf(mx_lo, fmaxf(sc[nt][0], sc[nt][1]));
                mx_hi = fmaxf(mx_hi, fmaxf(sc[nt][2], sc[nt][3]));
            }
            mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 1));
            mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 2));
            mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 1));
            mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 2));
            // block 0 always holds position 0 <= p, so every row's maximum is finite from there on
            const float n_lo = fmaxf(m_lo, mx_lo), n_hi = fmaxf(m_hi, mx_hi);
            const float al_lo = fast_exp2(m_lo - n_lo), al_hi = fast_exp2(m_hi - n_hi);
            m_lo = n_lo;
            m_hi = n_hi;
            // P in bf16 (sums over the rounded values), straight into A fragments
            uint32_t pa[NT / 2][4];
            float ps_lo = 0.f, ps_hi = 0.f;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const __nv_bfloat162 lo = __floats2bfloat162_rn(fast_exp2(sc[nt][0] - n_lo), fast_exp2(sc[nt][1] - n_lo));
                const __nv_bfloat162 hi = __floats2bfloat162_rn(fast_exp2(sc[nt][2] - n_hi), fast_exp2(sc[nt][3] - n_hi));
                ps_lo += __low2float(lo) + __high2float(lo);
                ps_hi += __low2float(hi) + __high2float(hi);
                pa[nt / 2][(nt & 1) * 2 + 0] = *reinterpret_cast<const uint32_t *>(&lo);
                pa[nt / 2][(nt & 1) * 2 + 1] = *reinterpret_cast<const uint32_t *>(&hi);
            }
            l_lo = l_lo * al_lo + ps_lo;
            l_hi = l_hi * al_hi + ps_hi;
#pragma unroll
            for (int dn = 0; dn < DN; ++dn) {
                o[dn][0] *= al_lo;
                o[dn][1] *= al_lo;
                o[dn][2] *= al_hi;
                o[dn][3] *= al_hi;
            }
            // O += P V; V rows past the context may hold anything: zero them in the fragments
            const int valid = L - b * BS;
#pragma unroll
            for (int kt = 0; kt < BS / 16; ++kt) {
                uint32_t keep_lo = 0xffffffffu, keep_hi = 0xffffffffu;
                if (valid < BS) {
                    const int t = 16 * kt + 2 * t4;
                    keep_lo = (t < valid ? 0x0000ffffu : 0u) | (t + 1 < valid ? 0xffff0000u : 0u);
                    keep_hi = (t + 8 < valid ? 0x0000ffffu : 0u) | (t + 9 < valid ? 0xffff0000u : 0u);
                }
#pragma unroll
                for (int dp = 0; dp < DN / 2; ++dp) {
                    uint32_t r[4];
                    ldsm_x4_trans(r, tile_addr<BS>(vtile, 16 * kt + (lane & 7) + 8 * ((lane >> 3) & 1),
                                                   2 * dp + (lane >> 4)));
                    mma_16816(o[2 * dp], pa[kt], r[0] & keep_lo, r[1] & keep_hi);
                    mma_16816(o[2 * dp + 1], pa[kt], r[2] & keep_lo, r[3] & keep_hi);
                }
            }
        }
        __syncthreads();  // every warp is done with stage st
        if (tid == 0 && b + kPrefillStages < nb && !*abort_flag) issue(b + kPrefillStages);
    }
    // leave no copy in flight when the CTA exits (only possible after a wait gave up)
    if (tid == 0)
        for (int st = 0; st < kPrefillStages; ++st)
            if ((inflight >> st) & 1u) mbar_wait_drain(&full[st], (inflight_par >> st) & 1u, a.status);
    if (*abort_flag) return;

    // ---- normalise and store this warp's rows
    l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 1);
    l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 2);
    l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 1);
    l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 2);
    const float inv_lo = l_lo > 0.f ? 1.f / l_lo : 0.f, inv_hi = l_hi > 0.f ? 1.f / l_hi : 0.f;
    uint32_t *ow = reinterpret_cast<uint32_t *>(a.out);
#pragma unroll
    for (int dn = 0; dn < DN; ++dn) {
        if (st_lo) ow[(qrow_lo + 8 * dn + 2 * t4) / 2] = pack_bf16x2(o[dn][0] * inv_lo, o[dn][1] * inv_lo);
        if (st_hi) ow[(qrow_hi + 8 * dn + 2 * t4) / 2] = pack_bf16x2(o[dn][2] * inv_hi, o[dn][3] * inv_hi);
    }
}

using PrefillFn = void (*)(const CUtensorMap, const CUtensorMap, const PrefillArgs);

PrefillFn pick_prefill(int D, int BS) {
    if (D == 64 && BS == 16) return paged_prefill_kernel<64, 16>;
    if (D == 64 && BS == 32) return paged_prefill_kernel<64, 32>;
    if (D == 128 && BS == 16) return paged_prefill_kernel<128, 16>;
    if (D == 128 && BS == 32) return paged_prefill_kernel<128, 32>;
    return nullptr;
}

}  // namespace

size_t prefill_smem_bytes(int head_dim, int block_size, int max_blocks_per_seq) {
    return static_cast<size_t>(kPrefillStages) * 2 * block_size * head_dim * 2 +
           static_cast<size_t>((max_blocks_per_seq * 4 + 15) / 16) * 16 + kPrefillStages * 8 + 64 + 1024;
}

cudaError_t prefill_launch(int head_dim, int block_size, const CUtensorMap &tm_k, const CUtensorMap &tm_v,
                           const PrefillArgs &args, int tiles, size_t smem_bytes, cudaStream_t stream) {
    PrefillFn fn = pick_prefill(head_dim, block_size);
    if (!fn) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_bytes));
    if (e != cudaSuccess) return e;
    const dim3 grid(static_cast<unsigned>(tiles), static_cast<unsigned>(args.num_seqs),
                    static_cast<unsigned>(args.num_kv_heads));
    fn<<<grid, kPrefillThreads, smem_bytes, stream>>>(tm_k, tm_v, args);
    return cudaGetLastError();
}

int prefill_rows_per_cta() { return kRowsPerCta; }

}  // namespace pkv
