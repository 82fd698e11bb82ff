// prefill_tc.cu -- multi-query paged attention on the 5th-generation tensor
// cores (tcgen05.mma, accumulators in tensor memory).
//
// Same operation as prefill.cu (chunked prefill / mixed batches: query i of a
// sequence's n-token chunk attends causally to positions 0 .. L - n + i).
// One CTA per (128 rows of (query token, group head), sequence, kv head), two
// CTAs per SM (256 tensor-memory columns each), seven warps; launched with the
// row tiles that see the most context first:
//   - warps 4 and 6 issue the TMA copies: warp 4 the CTA's 128 query rows once
//     (a 5D box over q viewed as [T][Hkv][G][D]) and the K tiles, warp 6 the V
//     tiles, of the context in iterations of 64 tokens (64 / BS paged blocks)
//     through separate 2-stage rings (128-byte swizzled tiles; one lane per
//     block slice). Each blocks on the MMA that frees its next stage and is
//     woken when it completes, so K and V refills never queue behind each
//     other and start as soon as a stage is free (one warp polling both
//     rings issued them ~1.5 us late: a %globaltimer trace);
//   - warp 5 (an elected lane) issues the MMAs: S = Q K^T (M 128, N 64, K =
//     head_dim in steps of 16) into one of two tensor-memory buffers, and
//     O += P V (M 128, N = head_dim, K 64; P read from tensor memory, V as an
//     N-major operand straight from its TMA tile). S of the next iteration
//     runs on the tensor cores while the softmax of this one runs;
//   - warps 0-3: thread r owns query row r (tensor-memory lane r): it loads its
//     64 logits in one tensor-memory load, masks the positions its query may
//     not see, updates its running maximum and sum, writes its row of P in
//     bf16 over the S buffer, and rescales its row of O in tensor memory when
//     its maximum has grown by more than 2^8 since the last rescale
//     (otherwise the stale maximum stays the reference: every P is then < 2^8
//     and the result is the same).
// All waits are bounded (1 s); a wait that gives up flags the status word,
// the CTA drains what it issued and frees its tensor memory.
#include <cuda_bf16.h>

#include "device_utils.cuh"
#include "launch.h"

namespace pkv {
namespace {

constexpr int kSoftmaxThreads = 128;  // warps 0-3: one query row (tensor-memory lane) each
constexpr int kTcThreads = 224;       // + warp 4: Q and K copies, warp 5: MMAs, warp 6: V copies
constexpr int kTcBarriers = 12;
constexpr int kTcRows = 128;          // query rows per CTA (= tensor-memory lanes)
constexpr int kTcTokens = 64;   // context tokens per iteration
// Tensor-memory columns: two S / P buffers of 64 and O (head_dim); allocations
// are powers of two, so both head sizes take 256 (two CTAs fill an SM's 512).
__host__ __device__ constexpr uint32_t tmem_cols(int) { return 256u; }

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

// 64 consecutive fp32 columns of this thread's lane in one load and one wait
// (warp-collective).
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&v)[64]) {
    __syncwarp();
    uint32_t r[64];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
}

// Largest of three (sm_100 three-input max.f32).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Packed fp32 add of both halves (sm_100 f32x2).
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\t"
        "mov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\t"
        "mov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// One lane of the warp (the same one every time), chosen by elect.sync.
__device__ __forceinline__ bool elect_one() {
    uint32_t pred;
    asm volatile(
        "{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(pred));
    return pred != 0;
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

// 16 consecutive 32-bit columns of this thread's lane (warp-collective).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
    __syncwarp();
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

// O += P V with P (A, M x K, K-major) in tensor memory.
__device__ __forceinline__ void umma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t db, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %5, %5, %5}, p;\n\t}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(db), "r"(idesc), "r"(accumulate), "r"(0u)
        : "memory");
}

// A bounded wait whose outcome is the same for the whole warp (tensor-memory
// loads and stores that follow are warp-collective).
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort, int32_t *status) {
    const bool got = mbar_wait_bounded(bar, parity, abort, status);
    return __all_sync(0xffffffffu, got);
}

template <int D, int BS>
__global__ void __launch_bounds__(kTcThreads, 2)
    paged_prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, const PrefillArgs a) {
    static_assert(D == 64 || D == 128, "head_dim");
    static_assert(BS == 16 || BS == 32, "block_size");
    constexpr int HALVES = D / 64;                        // 128-byte column slices of a row
    constexpr uint32_t kHalfKV = kTcTokens * 128;         // one slice of 64 tokens
    constexpr uint32_t kTileKV = HALVES * kHalfKV;        // K (or V) of one stage
    constexpr uint32_t kQHalf = kTcRows * 128;
    constexpr int BPI = kTcTokens / BS;                   // paged blocks per iteration

    // later row tiles see more context (more iterations): they go first
    const int tile = gridDim.x - 1 - blockIdx.x, s = blockIdx.y, h = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

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
    const int nit = (ntok + kTcTokens - 1) / kTcTokens;   // iterations of 64 tokens (>= 1)

    // ---- shared memory: Q | K stages 0, 1 | V stages 0, 1 | barriers | table
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sq = base;
    uint8_t *sk = sq + HALVES * kQHalf;   // [2][kTileKV]
    uint8_t *sv = sk + 2 * kTileKV;       // [2][kTileKV]
    uint64_t *bars = reinterpret_cast<uint64_t *>(sv + 2 * kTileKV);
    // Barriers, each with one phase per use of its stage or buffer b = it & 1:
    //   s_full[b]  S(it) is in tensor memory (and K stage b may be refilled);
    //   p_ready[b] the 128 softmax threads wrote P(it) over it;
    //   pv_free[b] O += P(it) V(it) is done (V stage b may be refilled, S / P
    //              buffer b may take S(it + 2), O may be rescaled).
    // A softmax warp that needs no rescale may run one iteration ahead of the
    // others, never two (S(it + 2) waits for P(it) V(it)), so no wait on these
    // is two phases behind or ahead of its barrier. A warp that has finished
    // its loop may be: the final O is signalled on a barrier of its own, o_full.
    uint64_t *q_full = bars, *k_full = bars + 1, *v_full = bars + 3, *s_full = bars + 5, *p_ready = bars + 7,
             *pv_free = bars + 9, *o_full = bars + 11;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kTcBarriers);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *table = reinterpret_cast<int *>(bars + kTcBarriers + 1);

    if (warp == 5) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(tmem_cols(D)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
        tc_fence_before();
    } else if (warp == 4 && lane == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&v_full[i], 1);
            mbar_init(&pv_free[i], 1);
            mbar_init(&s_full[i], 1);
            mbar_init(&p_ready[i], kSoftmaxThreads);
        }
        mbar_init(o_full, 1);
        *abort_flag = 0;
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
    // tensor memory: S / P buffers at columns 0 and 64, O at 128 .. 128 + D
    const uint32_t t_o = tbase + 128;

    if (warp == 4 || warp == 6) {
        // ---------------- load warps (4: Q and K, 6: V); lane j copies one
        // 128-byte column slice of one paged block
        const bool is_v = warp == 6;
        int use0 = -1, use1 = -1;  // last use of each stage issued
        const int jb = lane / HALVES, hf = lane % HALVES;
        auto issue = [&](int it) {
            const int st = it & 1;
            uint64_t *bar = is_v ? &v_full[st] : &k_full[st];
            const int b = it * BPI + jb;
            bool mine = lane < BPI * HALVES && b * BS < ntok;
            int p = 0;
            if (mine) {
                p = table[b];
                if (p < 0 || p >= a.num_blocks) {
                    if (!is_v && hf == 0) atomicOr(a.status, PKV_STATUS_BAD_BLOCK_ID);
                    mine = false;
                }
            }
            const unsigned m = __ballot_sync(0xffffffffu, mine);
            if (lane == 0) mbar_arrive_expect_tx(bar, static_cast<uint32_t>(__popc(m)) * BS * 128u);
            __syncwarp();
            if (mine)
                tma_load_4d((is_v ? sv : sk) + st * kTileKV + hf * kHalfKV + jb * BS * 128, is_v ? &tm_v : &tm_k, bar,
                            0, hf, h, p * BS);
            (st ? use1 : use0) = it >> 1;
        };
        if (!is_v && lane == 0) {
            mbar_arrive_expect_tx(q_full, HALVES * kQHalf);
#pragma unroll
            for (int q = 0; q < HALVES; ++q) tma_load_5d(sq + q * kQHalf, &tm_q, q_full, 0, q, 0, h, q0 + i0);
        }
        issue(0);
        if (nit > 1) issue(1);
        // K(it) once S(it - 2) is done (its stage is free), V(it) once
        // P(it - 2) V(it - 2) is done; bounded like every wait. Neither barrier
        // can run two phases ahead: S(it) needs K(it), P(it) V(it) needs V(it).
        bool ok = true;
        for (int nx = 2; nx < nit; ++nx) {
            uint64_t *freed = is_v ? &pv_free[nx & 1] : &s_full[nx & 1];
            if (!(ok = warp_wait(freed, static_cast<uint32_t>((nx - 2) >> 1) & 1u, abort_flag, a.status))) break;
            issue(nx);
        }
        // copies still in flight (only after a wait gave up) land before exit
        if (!ok || *abort_flag) {
            if (!is_v) mbar_wait_drain(q_full, 0, a.status);
            uint64_t *full = is_v ? v_full : k_full;
            if (use0 >= 0) mbar_wait_drain(&full[0], static_cast<uint32_t>(use0) & 1u, a.status);
            if (use1 >= 0) mbar_wait_drain(&full[1], static_cast<uint32_t>(use1) & 1u, a.status);
        }
        __syncwarp();
    } else if (warp == 5) {
        // ---------------- MMA warp (one elected lane issues; the operands are
        // computed by the whole warp, outside the branch)
        const bool leader = elect_one();
        bool o_committed = false;  // o_full committed (after the last P V, or by the drain)
        // descriptors of stage / buffer 0; the start address (16-byte units)
        // is the low field, so an offset is added to the descriptor itself
        const uint64_t dq = smem_desc(smem_u32(sq), 16, 1024);
        const uint64_t dk = smem_desc(smem_u32(sk), 16, 1024);
        const uint64_t dv = smem_desc(smem_u32(sv), kHalfKV, 1024);
        auto issue_s = [&](int it) {  // S(it) = Q K(it)^T into buffer it & 1
            const int b = it & 1;
            const uint64_t dkb = dk + ((b * kTileKV) >> 4);
            const uint32_t ts = tbase + 64 * b;
            if (leader) {
#pragma unroll
                for (int hf = 0; hf < HALVES; ++hf)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma(ts, dq + ((hf * kQHalf + kk * 32) >> 4), dkb + ((hf * kHalfKV + kk * 32) >> 4),
                             instr_desc(128, 64, false), (hf | kk) != 0);
                umma_commit(&s_full[b]);
            }
        };
        bool ok = warp_wait(q_full, 0, abort_flag, a.status);
        ok = ok && warp_wait(&k_full[0], 0, abort_flag, a.status);
        if (ok) {
            tc_fence_after();
            issue_s(0);
        }
        for (int it = 0; ok && it < nit; ++it) {
            const int b = it & 1, nb = b ^ 1;
            if (it + 1 < nit) {
                // S(it + 1) into the other buffer, which held P(it - 1)
                if (!(ok = warp_wait(&k_full[nb], static_cast<uint32_t>((it + 1) >> 1) & 1u, abort_flag, a.status)))
                    break;
                if (it >= 1 &&
                    !(ok = warp_wait(&pv_free[nb], static_cast<uint32_t>((it - 1) >> 1) & 1u, abort_flag, a.status)))
                    break;
                tc_fence_after();
                issue_s(it + 1);
            }
            // O += P(it) V(it), once the softmax warps have written P(it)
            if (!(ok = warp_wait(&v_full[b], static_cast<uint32_t>(it >> 1) & 1u, abort_flag, a.status))) break;
            if (!(ok = warp_wait(&p_ready[b], static_cast<uint32_t>(it >> 1) & 1u, abort_flag, a.status))) break;
            tc_fence_after();
            const uint64_t dvb = dv + ((b * kTileKV) >> 4);
            const uint32_t tp = tbase + 64 * b;
            if (leader) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_ts(t_o, tp + kk * 8, dvb + ((kk * 16 * 128) >> 4), instr_desc(128, D, true), (it | kk) != 0);
                umma_commit(&pv_free[b]);
                if (it == nit - 1) umma_commit(o_full);
            }
            if (it == nit - 1) o_committed = true;
        }
        // MMAs still in flight (only after a wait gave up) finish before the
        // tensor memory is freed: a commit's arrival covers every MMA issued
        // before it, and o_full has a single phase, so its wait cannot alias
        if (!o_committed && leader) umma_commit(o_full);
        __syncwarp();
        mbar_wait_drain(o_full, 0, a.status);
        __syncwarp();
    } else {
        // ---------------- softmax warps: thread r owns query row r (tensor-memory lane r)
        const int r = tid;
        const int row = row0 + r;
        const bool live = row < rows;
        const int qi = min(row, rows - 1) / G;              // query token of the row
        const int p_row = L - n + qi;                       // last position it may see
        const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
        float m_ref = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int it = 0; it < nit; ++it) {
            const int b = it & 1;
            const uint32_t t_s = tbase + 64 * b + lane_addr;
            if (!(ok = warp_wait(&s_full[b], static_cast<uint32_t>(it >> 1) & 1u, abort_flag, a.status))) break;
            tc_fence_after();
            float x[64];
            tmem_ld64(t_s, x);
            // x c with c < 0 is (-x)(-c): work with a positive factor
            if (a.scale_log2 < 0.f) {
#pragma unroll
                for (int t = 0; t < 64; ++t) x[t] = -x[t];
            }
            // positions past this row's last one exist only near the end
            if (it * kTcTokens + kTcTokens - 1 > p_row) {
#pragma unroll
                for (int t = 0; t < 64; ++t)
                    if (it * kTcTokens + t > p_row) x[t] = -INFINITY;
            }
            // maximum of the logits (before the positive factor): three-input
            // max, four independent chains
            float mx;
            {
                float m4[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
                for (int t = 4; t < 60; t += 8) {  // x[4 .. 59]
#pragma unroll
                    for (int e = 0; e < 4; ++e) m4[e] = fmax3(m4[e], x[t + e], x[t + 4 + e]);
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) m4[e] = fmaxf(m4[e], x[60 + e]);  // x[60 .. 63]
                mx = fmax3(fmaxf(m4[0], m4[1]), m4[2], m4[3]);
            }
            // log2-domain maximum; the reference moves only when it would be
            // exceeded by more than 2^8
            const float c = fabsf(a.scale_log2);
            float m_new = m_ref;
            if (mx * c > m_ref + 8.f) m_new = mx * c;
            const float alpha = fast_exp2(m_ref - m_new);  // 0 on the first update
            // P = 2^(x c - m) in bf16 over this buffer's first 32 columns (two
            // values per column); x c - m and the fp32 row sum on packed pairs
            const float2 cc = make_float2(c, c), nm = make_float2(-m_new, -m_new);
            float2 ps2a = make_float2(0.f, 0.f), ps2b = make_float2(0.f, 0.f);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t w[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int t = 32 * half + 2 * e;
                    const float2 arg = ffma2(make_float2(x[t], x[t + 1]), cc, nm);
                    const float2 pr = make_float2(fast_exp2(arg.x), fast_exp2(arg.y));
                    if (e & 1)
                        ps2b = fadd2(ps2b, pr);
                    else
                        ps2a = fadd2(ps2a, pr);
                    const __nv_bfloat162 v2 = __floats2bfloat162_rn(pr.x, pr.y);
                    w[e] = *reinterpret_cast<const uint32_t *>(&v2);
                }
                tmem_st16(t_s + 16 * half, w);
            }
            const float ps0 = ps2a.x + ps2b.x, ps1 = ps2a.y + ps2b.y;
            const float ps = ps0 + ps1;
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            l_run = l_run * alpha + ps;
            m_ref = m_new;
            // a warp whose maximum moved rescales its rows of O, once
            // O += P(it - 1) V(it - 1) is done; otherwise it does not wait: the
            // MMAs issued by one thread run in order, so P(it) V(it) may be
            // issued behind P(it - 1) V(it - 1) straight away
            if (it > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
                if (!(ok = warp_wait(&pv_free[b ^ 1], static_cast<uint32_t>((it - 1) >> 1) & 1u, abort_flag, a.status)))
                    break;
                tc_fence_after();
#pragma unroll
                for (int cb = 0; cb < D / 32; ++cb) {
                    float o[32];
                    tmem_ld32(t_o + lane_addr + cb * 32, o);
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] *= alpha;
                    tmem_st32(t_o + lane_addr + cb * 32, o);
                }
            }
            // V rows past the tile's last position (past the context, or in
            // blocks not loaded) may hold anything: zero them so that P = 0
            // there multiplies zeros
            if (it == nit - 1) {
                if (!(ok = warp_wait(&v_full[b], static_cast<uint32_t>(it >> 1) & 1u, abort_flag, a.status))) break;
                const int valid = ntok - it * kTcTokens;
                uint8_t *vt = sv + b * kTileKV;
                for (int e = tid; e < HALVES * kTcTokens * 8; e += kSoftmaxThreads) {
                    const int hf = e / (kTcTokens * 8), t = (e / 8) % kTcTokens, c = e % 8;
                    if (t >= valid)
                        *reinterpret_cast<uint4 *>(vt + hf * kHalfKV + t * 128 + ((c ^ (t & 7)) << 4)) =
                            make_uint4(0u, 0u, 0u, 0u);
                }
                fence_proxy_async_shared();
            }
            tc_fence_before();
            mbar_arrive(&p_ready[b]);
        }
        if (ok) {
            ok = warp_wait(o_full, 0, abort_flag, a.status);
            tc_fence_after();
        }
        // normalise and store this row (every lane reads its lane of O: the
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
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
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
    const size_t bytes = halves * kTcRows * 128 + 2 * 2 * halves * kTcTokens * 128 + (kTcBarriers + 1) * 8 +
                         static_cast<size_t>(max_blocks_per_seq) * 4 + 1024;
    // at most two CTAs per SM: their tensor memory (256 columns each) fills the SM's 512
    return bytes < 80 * 1024 ? 80 * 1024 : bytes;
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
