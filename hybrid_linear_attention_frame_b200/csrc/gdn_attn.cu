// Chunk-causal softmax attention with a rolling KV cache: the softmax layers of
// SANA-WM's hybrid stack (sglang cookbook SANA-WM page, section 1 architecture
// table, "softmax every 4 blocks"; pipeline-configuration table: blocks of
// num_frame_per_block = 3 latent frames, num_cached_blocks = 2, sink_size = 1
// frame).  Over a whole sequence, per batch entry and head,
//
//   o_t = sum_{s in K(t)} softmax_s(q_t . k_s / sqrt(d_k)) v_s,
//   K(t) = [0, sink) U [max(0, b - cached) * block, min(T, (b + 1) * block)),  b = t / block,
//
// the sink frames, the cached blocks and the whole current block.
//
// One CTA of 544 threads per (128 queries, head, batch entry); threads r, r + 128,
// r + 256 and r + 384 share query row r (TMEM lane r), each taking 32 of a tile's keys
// and a quarter of the output columns.  For each key tile of 128 tokens:
//   S = Q K^T on the tensor cores into TMEM (two buffers: the next tile's S runs
//     while this tile's softmax does),
//   the softmax in registers against a lazily moved reference maximum (it moves
//     only when a score exceeds it by more than 2^8, so the accumulator is rarely
//     rescaled; the final division by the running sum makes the result exact
//     whatever reference was used), the row's maximum exchanged once per tile,
//   P in bf16 pairs into TMEM (two buffers), O += P V on the tensor cores into TMEM
//     with P as the A operand.
// K tiles are triple-buffered and V tiles double-buffered, loaded by TMA (128-byte
// swizzle, rows past the end of the sequence read as zeros and are masked).
// Warp 16 issues the copies and the MMAs; warps 0-15 only run the softmax, and the two
// sides meet at mbarriers: S ready / S read, P written / P V done.  Every wait is
// bounded.
#include "gdn_common.cuh"
#include "gdn_sm100.cuh"

namespace gdn {
namespace attn {

using namespace sm100;

constexpr int kBM = 128;                       // queries per CTA
constexpr int kBN = 128;                       // keys per tile
constexpr int kParts = 4;                      // softmax threads per query row (four softmax warps
                                               // per sub-partition hide more of its latency than two)
constexpr int kSoftThreads = kParts * kBM;     // softmax warps 0 .. 4 kParts - 1
constexpr int kProducerWarp = kSoftThreads / 32;   // copies and MMAs
constexpr int kThreads = kSoftThreads + 32;
constexpr int kKeysPer = kBN / kParts;         // keys of a tile per softmax thread
static_assert(kKeysPer % 32 == 0, "whole 16-column P stores");
constexpr uint32_t kBox = 128u * 128u;         // one 64-column SW128 box of 128 rows: 16 KB
constexpr uint32_t kOp = 2u * kBox;            // a 128 x (d <= 128) operand: two boxes
constexpr int kKStages = 3, kVStages = 2;
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kOp;
constexpr uint32_t kOffV = kOffK + kKStages * kOp;
constexpr uint32_t kOffBar = kOffV + kVStages * kOp;
enum : uint32_t { kBarQ = 0, kBarK = 1, kBarV = kBarK + kKStages, kBarS = kBarV + kVStages,
                  kBarPV = kBarS + 2,        // [2] P V of the tile that used P buffer b done
                  kBarSFree = kBarPV + 2,   // [2] the softmax warps have read a score buffer (one arrival each)
                  // [2] P buffer b written and O rescaled (one arrival per softmax warp).  Per
                  // buffer: the softmax can finish tile j + 1 before the issuing warp looks for
                  // tile j, but not tile j + 2 (its P waits for P V(j), issued after that look)
                  kBarPFull = kBarSFree + 2,
                  kNumBars = kBarPFull + 2 };
__host__ __device__ constexpr uint32_t bar_count(uint32_t i) {
    return (i >= kBarSFree && i < kBarPFull + 2) ? (uint32_t)(kSoftThreads / 32) : 1u;
}
constexpr uint32_t kOffAbort = kOffBar + 8u * kNumBars;
constexpr uint32_t kOffTmemSlot = kOffAbort + 8u;
constexpr uint32_t kOffX = kOffTmemSlot + 16u;                 // one float per softmax thread: the row parts' exchange
constexpr uint32_t kSmemBytes = kOffX + 4u * kSoftThreads + 1024u; // + slack for 1024-byte alignment
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kOffK % 1024 == 0 && kOffV % 1024 == 0, "SW128 tiles need 1024-B alignment");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;                  // two 128-column score buffers
constexpr uint32_t kColO = 256;                // the d_v-column output accumulator
constexpr uint32_t kColP = 384;                // two 64-column P buffers: bf16 pairs, the A operand of P V
constexpr float kMoveRef = 8.0f;               // log2 units: p stays below 2^8
constexpr uint32_t kBarGroup = 1;              // named barrier of the softmax warps

constexpr uint32_t kIdS = idesc_bf16(128, 128, false, false);

struct AttnArgs {
    void* out;
    int B, H, T, dk, dv;
    int block_len, cached, sink_len;
    float scale_log2;                          // log2(e) / sqrt(d_k)
    uint64_t wait_limit_ns;
};

__device__ __forceinline__ bool group_all(uint32_t id, uint32_t n, bool v) {
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\t"
                 "setp.ne.u32 p, %3, 0;\n\t"
                 "bar.red.and.pred q, %1, %2, p;\n\t"
                 "selp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r) : "r"(id), "r"(n), "r"(v ? 1u : 0u) : "memory");
    return r != 0;
}

// 2^x (the hardware's approximate exponential; 2^-inf = 0)
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}


// A three-input maximum, and pairs of f32 packed in 64-bit registers for the paired FMA and
// add (one instruction does the work of two): they trim the softmax's instruction count.
__device__ __forceinline__ float max3f(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}
__device__ __forceinline__ uint64_t f2pack(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void f2unpack(uint64_t r, float& a, float& b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32"
                 " [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
                 :: "r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])),
                    "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])),
                    "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
                    "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
                    "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
                    "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15]))
                 : "memory");
}

__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t* v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32"
                 " [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
                 :: "r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]),
                    "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
                    "r"(v[15])
                 : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint64_t kmaj(uint32_t addr) { return smem_desc(addr, 16, 1024, kSwizzle128); }

// Start of the 16-wide K step `ks` of a K-major operand whose K axis (<= 128) is
// split into two 64-column boxes.
__device__ __forceinline__ uint32_t kstep(uint32_t op, int ks) {
    return op + (ks >= 4 ? kBox : 0u) + (uint32_t)(ks & 3) * 32u;
}

// S[128 x 128] = Q K^T, K axis d_k
__device__ __forceinline__ void issue_s(uint32_t q, uint32_t k, uint32_t d, int nks) {
#pragma unroll 1
    for (int ks = 0; ks < nks; ++ks) mma_bf16_warp(d, kmaj(kstep(q, ks)), kmaj(kstep(k, ks)), kIdS, ks > 0);
}

// One tcgen05 MMA whose A operand is in TMEM (row m in lane m, a bf16 pair per column).
__device__ __forceinline__ void mma_bf16_tmem_a_warp(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                                     uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p, e;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "elect.sync _|e, 0xffffffff;\n\t"
                 "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
                 :: "r"(d_tmem), "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
                 : "memory");
}

// O[128 x d_v] (+)= P V, K axis = the 128 keys: P from TMEM (16 keys = 8 columns per
// step), V read MN-major from shared memory (rows = keys).
__device__ __forceinline__ void issue_pv(uint32_t p_tmem, uint32_t v, uint32_t d, uint32_t idpv, bool acc) {
#pragma unroll
    for (int ks = 0; ks < kBN / 16; ++ks)
        mma_bf16_tmem_a_warp(d, p_tmem + 8u * (uint32_t)ks, smem_desc(v + (uint32_t)ks * 2048u, kBox, 1024, kSwizzle128),
                             idpv, (acc || ks > 0) ? 1u : 0u);
}

__global__ void __launch_bounds__(kThreads, 1)
chunk_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const AttnArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gb = smem_raw + (base - raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.y, bb = blockIdx.z;
    const int T = a.T, bl = a.block_len;
    const int t0 = blockIdx.x * kBM;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gb + kOffAbort);
    auto bar = [&](uint32_t i) { return base + kOffBar + 8u * i; };
    const uint64_t lim = a.wait_limit_ns;

    // ---- the key tiles this CTA visits: the union of its rows' key sets ----
    const int tl = min(T, t0 + kBM) - 1;
    const int w_lo = max(0, t0 / bl - a.cached) * bl;
    const int w_hi = min(T, (tl / bl + 1) * bl);
    const int sink = min(a.sink_len, T);
    const bool split = w_lo > sink;                 // sink and window are separate ranges
    const int nA = split ? (sink + kBN - 1) / kBN : 0;
    const int startB = split ? w_lo : 0;
    const int n = nA + (w_hi - startB + kBN - 1) / kBN;
    auto tile_start = [&](int j) { return j < nA ? kBN * j : startB + kBN * (j - nA); };

    // ---- this thread's query row, its part of the keys and its row's key set ----
    const int row = tid & (kBM - 1), part = (tid / kBM) % kParts;   // (softmax threads)
    const int t = t0 + row;
    const int te = min(t, T - 1);
    const int ws = max(0, te / bl - a.cached) * bl;
    const int we = min(T, (te / bl + 1) * bl);

    if (warp == 0) {
        tmem_alloc(base + kOffTmemSlot, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 32) {
        for (uint32_t i = 0; i < kNumBars; ++i) mbar_init(bar(i), bar_count(i));
        fence_mbar_init();
        *abort_flag = 0;
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gb + kOffTmemSlot);
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);   // warp w reads lanes 32 (w % 4) ..
    float* xchg = reinterpret_cast<float*>(gb + kOffX);
    const int nco = a.dv / 16, c_lo = part * nco / kParts, c_hi = (part + 1) * nco / kParts;
    const uint32_t idpv = idesc_bf16(128, a.dv, false, true);
    const int nks = a.dk / 16;

    if (warp == kProducerWarp) {
        // ======================= copies and MMAs =======================
        // issued / waited counts (uniform within the warp) for the drain on the way out
        int k_issued = 0, k_waited = 0, v_issued = 0, v_waited = 0, s_issued = 0, s_waited = 0;
        int pv_issued = 0, pv_waited = 0;
        bool q_pending = false, ok = true;
        auto load_k = [&](int j) {
            if (lane == 0) {
                const uint32_t b = bar(kBarK + j % kKStages), dst = base + kOffK + (uint32_t)(j % kKStages) * kOp;
                mbar_arrive_expect_tx(b, kOp);
                tma_load_4d(dst, &tm_k, b, 0, h, tile_start(j), bb);
                tma_load_4d(dst + kBox, &tm_k, b, 64, h, tile_start(j), bb);
            }
            __syncwarp();
            k_issued = j + 1;
        };
        auto load_v = [&](int j) {
            if (lane == 0) {
                const uint32_t b = bar(kBarV + j % kVStages), dst = base + kOffV + (uint32_t)(j % kVStages) * kOp;
                mbar_arrive_expect_tx(b, kOp);
                tma_load_4d(dst, &tm_v, b, 0, h, tile_start(j), bb);
                tma_load_4d(dst + kBox, &tm_v, b, 64, h, tile_start(j), bb);
            }
            __syncwarp();
            v_issued = j + 1;
        };
        // S of tile j into score buffer j & 1, once its K tile has landed
        auto start_s = [&](int j) -> bool {
            const bool got = mbar_wait(bar(kBarK + j % kKStages), (uint32_t)((j / kKStages) & 1), abort_flag, lim, 21);
            if (!__all_sync(0xffffffffu, got)) return false;      // the MMA issue below is warp-collective
            k_waited = j + 1;
            tc_fence_after();
            issue_s(base + kOffQ, base + kOffK + (uint32_t)(j % kKStages) * kOp, tmem + kColS + 128u * (j & 1), nks);
            mma_commit_warp(bar(kBarS + (j & 1)));
            s_issued = j + 1;
            return true;
        };
        if (lane == 0) {
            mbar_arrive_expect_tx(bar(kBarQ), kOp);
            tma_load_4d(base + kOffQ, &tm_q, bar(kBarQ), 0, h, t0, bb);
            tma_load_4d(base + kOffQ + kBox, &tm_q, bar(kBarQ), 64, h, t0, bb);
        }
        __syncwarp();
        q_pending = true;
        for (int j = 0; j < min(n, kKStages); ++j) load_k(j);
        for (int j = 0; j < min(n, kVStages); ++j) load_v(j);
        ok = __all_sync(0xffffffffu, mbar_wait(bar(kBarQ), 0, abort_flag, lim, 20));
        if (ok) q_pending = false;
        ok = ok && start_s(0);
        for (int j = 0; ok && j < n; ++j) {
            // the next tile's S, once the softmax has read the buffer it goes into (tile j - 1's)
            if (j + 1 < n) {
                if (j >= 1)
                    ok = __all_sync(0xffffffffu, mbar_wait(bar(kBarSFree + ((j + 1) & 1)), (uint32_t)(((j - 1) >> 1) & 1),
                                                           abort_flag, lim, 26));
                ok = ok && start_s(j + 1);
            }
            // tile j's K slot takes tile j + 3 once S(j) is done
            if (ok && j + kKStages < n) {
                ok = __all_sync(0xffffffffu, mbar_wait(bar(kBarS + (j & 1)), (uint32_t)((j >> 1) & 1), abort_flag, lim, 27));
                if (ok) {
                    s_waited = j + 1;
                    load_k(j + kKStages);
                }
            }
            // V slot of tile j - 1 takes tile j + 1 once P V(j - 1) is done
            if (ok && j >= 1 && j + 1 < n) {
                ok = __all_sync(0xffffffffu, mbar_wait(bar(kBarPV + ((j - 1) & 1)), (uint32_t)(((j - 1) >> 1) & 1),
                                                       abort_flag, lim, 28));
                if (ok) {
                    pv_waited = j;
                    load_v(j + 1);
                }
            }
            // P V(j): P written by the softmax (and O rescaled), V landed
            ok = ok && __all_sync(0xffffffffu, mbar_wait(bar(kBarPFull + (j & 1)), (uint32_t)((j >> 1) & 1), abort_flag,
                                                         lim, 29));
            ok = ok && __all_sync(0xffffffffu, mbar_wait(bar(kBarV + j % kVStages), (uint32_t)((j / kVStages) & 1),
                                                         abort_flag, lim, 24));
            if (ok) {
                v_waited = j + 1;
                tc_fence_after();
                issue_pv(tmem + kColP + 64u * (uint32_t)(j & 1), base + kOffV + (uint32_t)(j % kVStages) * kOp,
                         tmem + kColO, idpv, j > 0);
                mma_commit_warp(bar(kBarPV + (j & 1)));
                pv_issued = j + 1;
            }
        }
        if (!ok && lane == 0) {
            // copies and MMAs still in flight land before shared memory and TMEM go away
            if (q_pending) drain_wait(bar(kBarQ), 0);
            for (int j = k_waited; j < k_issued; ++j) drain_wait(bar(kBarK + j % kKStages), (uint32_t)((j / kKStages) & 1));
            for (int j = v_waited; j < v_issued; ++j) drain_wait(bar(kBarV + j % kVStages), (uint32_t)((j / kVStages) & 1));
            for (int j = s_waited; j < s_issued; ++j) drain_wait(bar(kBarS + (j & 1)), (uint32_t)((j >> 1) & 1));
            for (int j = pv_waited; j < pv_issued; ++j) drain_wait(bar(kBarPV + (j & 1)), (uint32_t)((j >> 1) & 1));
        }
        __syncwarp();
    } else {
        // ======================= softmax (warps 0-7) =======================
        // Threads leave the loop only together, after a vote (bar.red), so the
        // exchange barrier is never left half-arrived.
        bool alive = true, ok = true;
        float m_ref = -INFINITY, l = 0.0f;
        for (int j = 0; j < n; ++j) {
            // (the vote on this wait rides on the maximum's exchange barrier below; a thread
            // whose wait gave up reads scores that are not ready, and the vote then ends the loop)
            ok = mbar_wait(bar(kBarS + (j & 1)), (uint32_t)((j >> 1) & 1), abort_flag, lim, 22);
            tc_fence_after();
            const int s0 = tile_start(j) + kKeysPer * part;      // this thread's first key
            const bool sink_tile = j < nA;
            float x[kKeysPer];
#pragma unroll
            for (int c = 0; c < kKeysPer / 16; ++c)
                tmem_ld16(lane_base + kColS + 128u * (j & 1) + (uint32_t)(kKeysPer * part) + 16u * c,
                          *reinterpret_cast<float(*)[16]>(&x[16 * c]));
            // Are all of this thread's keys inside its row's key set?  (Then no per-key mask.)
            bool full;
            if (sink_tile) full = s0 + kKeysPer <= sink;
            else if (split) full = s0 >= ws && s0 + kKeysPer <= we;
            else full = (ws <= sink) ? (s0 + kKeysPer <= max(sink, we))
                                     : (s0 + kKeysPer <= sink || (s0 >= ws && s0 + kKeysPer <= we));
            tmem_wait_ld();
            // this warp is done with the score buffer: the producer may issue tile j + 2 into it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kBarSFree + (j & 1)));
            if (!full) {
#pragma unroll
                for (int i = 0; i < kKeysPer; ++i) {
                    const int s = s0 + i;
                    const bool valid = sink_tile ? (s < sink)
                                                 : (s < T && ((!split && s < sink) || (s >= ws && s < we)));
                    x[i] = valid ? x[i] : -INFINITY;
                }
            }
            // maximum of the raw scores (the scale is positive) over both halves of the row
            float mx[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
            for (int q = 0; q < (kKeysPer - 4) / 2; ++q) mx[q & 3] = max3f(mx[q & 3], x[4 + 2 * q], x[5 + 2 * q]);
            xchg[tid] = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
            if (!group_all(kBarGroup, kSoftThreads, ok)) { alive = false; break; }
            float mrow = xchg[row];
#pragma unroll
            for (int q = 1; q < kParts; ++q) mrow = fmaxf(mrow, xchg[row + kBM * q]);
            const float mt = mrow * a.scale_log2;
            const bool move = mt > m_ref + kMoveRef;   // the same decision in both threads of the row
            float alpha = 1.0f;
            if (move) {
                alpha = ex2(m_ref - mt);
                m_ref = mt;
            }
            const float neg_mr = (m_ref == -INFINITY) ? 0.0f : -m_ref;
            const uint64_t sc2 = f2pack(a.scale_log2, a.scale_log2), nm2 = f2pack(neg_mr, neg_mr);
            uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};        // (+0, +0) pairs
            uint32_t pk[kKeysPer / 2];
#pragma unroll
            for (int i = 0; i < kKeysPer / 2; ++i) {
                float t0, t1;
                f2unpack(fma2(f2pack(x[2 * i], x[2 * i + 1]), sc2, nm2), t0, t1);
                const float p0 = ex2(t0), p1 = ex2(t1);
                acc[i & 3] = add2(acc[i & 3], f2pack(p0, p1));
                pk[i] = pack_bf16x2(p0, p1);
            }
            float sm[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) f2unpack(acc[e], sm[2 * e], sm[2 * e + 1]);
            const float sum = ((sm[0] + sm[1]) + (sm[2] + sm[3])) + ((sm[4] + sm[5]) + (sm[6] + sm[7]));
            l = l * alpha + sum;
            // ---- P buffer j & 1 was used by tile j - 2: its P V must be done; a rescale of O
            // needs the previous P V (tile j - 1) done as well (P V's complete in order) ----
            const bool any_move = __any_sync(0xffffffffu, move && j > 0);
            const int wait_for = any_move ? j - 1 : j - 2;         // (uniform within the warp)
            ok = (wait_for < 0) ||
                 mbar_wait(bar(kBarPV + (wait_for & 1)), (uint32_t)((wait_for >> 1) & 1), abort_flag, lim, 23);
            // (every softmax thread votes here on every tile, whatever it waited for)
            if (!group_all(kBarGroup, kSoftThreads, ok)) { alive = false; break; }
            tc_fence_after();
            // TMEM loads and stores are warp-collective: the whole warp rescales when any
            // of its rows moved its reference (the others with alpha = 1)
            if (any_move) {
                const float f = (move && j > 0) ? alpha : 1.0f;
#pragma unroll 1
                for (int c = c_lo; c < c_hi; ++c) {
                    float o[16];
                    tmem_ld16(lane_base + kColO + 16u * c, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) o[e] *= f;
                    tmem_st16(lane_base + kColO + 16u * c, o);
                }
            }
            // ---- this thread's keys of the P row (bf16 pairs) into TMEM: columns
            // kKeysPer/2 part .. of P buffer j & 1 ----
            {
                const uint32_t pt = lane_base + kColP + 64u * (uint32_t)(j & 1) + (uint32_t)(kKeysPer / 2 * part);
#pragma unroll
                for (int c = 0; c < kKeysPer / 32; ++c) tmem_st16u(pt + 16u * c, &pk[16 * c]);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kBarPFull + (j & 1)));
        }

        // ---- epilogue: wait for the last P V, O / l to bf16 ----
        if (alive) {
            ok = mbar_wait(bar(kBarPV + ((n - 1) & 1)), (uint32_t)(((n - 1) >> 1) & 1), abort_flag, lim, 25);
            alive = group_all(kBarGroup, kSoftThreads, ok);
            if (alive) {
                tc_fence_after();
                xchg[tid] = l;                       // the row sum is the sum of its parts
                named_bar_sync(kBarGroup, kSoftThreads);
                float lrow = 0.0f;
#pragma unroll
                for (int q = 0; q < kParts; ++q) lrow += xchg[row + kBM * q];
                const float inv = 1.0f / lrow;
                __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.out) +
                                      (((size_t)bb * T + (size_t)t) * a.H + h) * (size_t)a.dv;
#pragma unroll 1
                for (int c = c_lo; c < c_hi; ++c) {
                    float o[16];
                    tmem_ld16(lane_base + kColO + 16u * c, o);
                    tmem_wait_ld();
                    if (t < T) {
                        uint4* dst = reinterpret_cast<uint4*>(orow + 16 * c);
                        dst[0] = make_uint4(pack_bf16x2(o[0] * inv, o[1] * inv), pack_bf16x2(o[2] * inv, o[3] * inv),
                                            pack_bf16x2(o[4] * inv, o[5] * inv), pack_bf16x2(o[6] * inv, o[7] * inv));
                        dst[1] = make_uint4(pack_bf16x2(o[8] * inv, o[9] * inv), pack_bf16x2(o[10] * inv, o[11] * inv),
                                            pack_bf16x2(o[12] * inv, o[13] * inv),
                                            pack_bf16x2(o[14] * inv, o[15] * inv));
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace attn

namespace {

// 4-D bf16 map over a [B, T, H, inner] tensor, box {64, 1, 128, 1}, 128-byte swizzle.
bool make_map_rows128(CUtensorMap* map, const void* ptr, int inner, int H, int T, int B)
{
    PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)inner, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)inner * 2, (cuuint64_t)H * inner * 2, (cuuint64_t)T * H * inner * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)attn::kBN, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool attn_supported(int dk, int dv)
{
    // both 64-column boxes of every operand lie partly inside the tensor
    return dk % 16 == 0 && dk > 64 && dk <= 128 && dv % 16 == 0 && dv > 64 && dv <= 128;
}

cudaError_t launch_attn(const void* q, const void* k, const void* v, void* out, int B, int H, int T, int dk,
                        int dv, int block_len, int cached, int sink_len, cudaStream_t stream)
{
    if (!attn_supported(dk, dv) || T < 1) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv;
    if (!make_map_rows128(&mq, q, dk, H, T, B) || !make_map_rows128(&mk, k, dk, H, T, B) ||
        !make_map_rows128(&mv, v, dv, H, T, B))
        return cudaErrorInvalidValue;
    // the dynamic shared memory limit is a per-device setting of the current context: set it on
    // every call (cheap), so that every device and a context re-created after a reset get it
    cudaError_t e = cudaFuncSetAttribute(attn::chunk_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)attn::kSmemBytes);
    if (e != cudaSuccess) return e;
    attn::AttnArgs a;
    a.out = out;
    a.B = B; a.H = H; a.T = T; a.dk = dk; a.dv = dv;
    a.block_len = block_len; a.cached = cached; a.sink_len = sink_len;
    a.scale_log2 = 1.4426950408889634f / sqrtf((float)dk);
    a.wait_limit_ns = g_wait_limit_ns;
    dim3 grid((unsigned)((T + attn::kBM - 1) / attn::kBM), (unsigned)H, (unsigned)B);
    attn::chunk_attn_kernel<<<grid, attn::kThreads, attn::kSmemBytes, stream>>>(mq, mk, mv, a);
    return cudaGetLastError();
}

}  // namespace gdn
