// Tensor-core chunked GDN forward for sm_100a with the state-independent work
// of every chunk done ONCE per head and shared through an L2-resident ring.
//
// A head's d_k x d_v state is split into d_v / 16 column blocks, one CTA each
// (a "group" of CTAs per head).  The per-chunk work splits in two halves
// (notation of gdn_common.cuh):
//
//   prep  (depends on the chunk's inputs only)
//     gates, [K;Q][K;Q]^T on the tensor cores, norms, A and P with the decay,
//     T = (I+A)^{-1} diag(beta) (CUDA cores + mma.sync), W = T diag(e^G/|k|) K
//     and U = T V for all d_v columns (tensor cores)
//   chain (depends on the state; sequential over chunks)
//     [Q;W] S, E = U - W S, K^T diag(e^{G_L-G}/|k|) E and P E, the state update
//     and the output O = diag(e^G/|q|) Q S + P E.
//
// Prep of chunk n is done by CTA n mod (d_v/16) of the group, which writes the
// chunk's record (W and P as ready-made 128-byte-swizzled operand images, U in
// 16-column slices, the per-token scalars) into ring slot n mod kRing and then
// publishes it with a GPU-scope release store.  Every CTA of the group runs the
// chain for its own 16 columns over all chunks, from two shared-memory slots,
// each filled in two parts: loader A acquires the ready flags and copies part A
// (the chunk's q tiles by TMA, the W image by bulk copy) as soon as MMA1 two
// chunks back has read the slot; loader B copies part B (k tiles, P, the U
// slice, the scalars) once the chunk two back is done with entirely, then
// reports the ring slot consumed (so the chain warps never wait on a fence).
// A producer re-fills a ring slot only after every CTA of the group has
// consumed it.  Each wait depends only on chunks with a smaller index, and the launch is
// cooperative (all CTAs resident), so the protocol cannot deadlock; every wait
// is bounded all the same and gives up with GDN_ERR_TIMEOUT.
//
// Groups are persistent: group g serves chains g, g + G, g + 2G, ... back to
// back, numbering their chunks consecutively.
//
// Warp roles inside a CTA: warps 0-3 run the state chain, warps 4-11 the prep
// of this CTA's share of the chunks, warps 12-13 the intra-chunk product P E
// and the output, warps 14 and 15 load the two parts of the chain's slots.
#include <cudaTypedefs.h>

#include <atomic>

#include "gdn_common.cuh"
#include "gdn_status.cuh"
#include "gdn_sm100.cuh"

namespace gdn {
namespace ring {

using namespace sm100;
using tc::kC;
using tc::kXS;

constexpr int kVB = 16;                // state columns per CTA
constexpr int kThreads = 512;          // 16 warps
constexpr int kChainThreads = 128;     // warps 0-3: the state chain
constexpr int kPrepThreads = 256;      // warps 4-11: prep of this CTA's share of the chunks
constexpr int kOutWarp0 = 12;          // warps 12, 13: P E and the output (TMEM lanes 0-63)
constexpr int kLoaderA = 14;           // warp 14: part A of the chain's slots (q and W tiles)
constexpr int kLoaderB = 15;           // warp 15: part B (k tile, P, U, scalars)
// named barriers (3 is the UT inverse's)
constexpr uint32_t kBarChain = 1, kBarPrep = 2, kBarPrepHi = 4, kBarOut = 6;
constexpr int kRing = 16;              // record slots per group
constexpr uint32_t kTmemCols = 512;

// TMEM columns
constexpr uint32_t kColG = 0;          // [K;Q][K;Q]^T     128 (prep)
constexpr uint32_t kColW = 128;        // [T';T] K         128 (prep; lanes 0-63 = W)
constexpr uint32_t kColU = 256;        // [T';T] V         128 (prep; lanes 64-127 = U)
constexpr uint32_t kColQW = 384;       // [Q;W] S          4 x 16 (chain, by chunk mod 4)
constexpr uint32_t kColS = 448;        // K^T E'           16     (chain)
constexpr uint32_t kColPE = 464;       // [P;X] E          2 x 16 (output warps, by chunk parity)

// ---- record (global memory, one per ring slot) ----
constexpr uint32_t kRecW = 0;          // W image: d-columns 0-63 | 64-127, 8 KB each (SW128)
constexpr uint32_t kRecP = 16384;      // P image, 8 KB (SW128)
constexpr uint32_t kRecU = 24576;      // U: per 16-column block [4][64][4] fp32 (4 KB)
__host__ __device__ constexpr uint32_t rec_sc(int dv) { return kRecU + (uint32_t)(dv / 16) * 4096u; }
__host__ __device__ constexpr uint32_t rec_bytes(int dv) { return rec_sc(dv) + 1024u; }
constexpr uint32_t kScCopy = 528;      // GQ[64], DL[64], e^{G_L}, padding
enum : uint32_t { RS_GQ = 0, RS_DL = 64, RS_GL = 128 };

// ---- flags (start of the workspace) ----
// word 0: abort; then per group: ready[kRing], consumed[8] (uint64 each)
constexpr uint32_t kGroupFlags = kRing + 8;
__host__ __device__ constexpr size_t flags_bytes(int G) {
    return ((size_t)(1 + G * kGroupFlags) * 8 + 4095) / 4096 * 4096;
}

// ---- shared memory (from a 1024-aligned base) ----
// chain slot: Q0 | W0 | Q1 | W1 | K0 | K1 | P | U | scalars
constexpr uint32_t kTile = 8192;
constexpr uint32_t cQ0 = 0, cW0 = 8192, cQ1 = 16384, cW1 = 24576, cK0 = 32768, cK1 = 40960;
constexpr uint32_t cP = 49152, cU = 57344, cSc = 61440;
constexpr uint32_t kCSlot = 62464;
constexpr uint32_t kCHalfQ = cQ1 - cQ0;            // [Q;W] of d-columns 64-127
constexpr uint32_t kCHalfK = cK1 - cK0;            // LBO of K^T (MN-major)
// prep area: K0 | Q0 | K1 | Q1 | V0 | V1, then T' | T, AXI, scalars
constexpr uint32_t kOffPrep = 2 * kCSlot;
constexpr uint32_t pK0 = 0, pQ0 = 8192, pK1 = 16384, pQ1 = 24576, pV0 = 32768, pV1 = 40960;
constexpr uint32_t kPHalf = pK1 - pK0;
constexpr uint32_t kOffTp = kOffPrep + 49152;
constexpr uint32_t kOffT = kOffTp + kTile;
constexpr uint32_t kOffAXI = kOffT + kTile;
constexpr uint32_t kScFloats = 13 * 64 + 16;
constexpr uint32_t kOffSc = kOffAXI + 64 * kXS * 4;   // prep scalars, 2 buffers (chunk parity)
constexpr uint32_t kOffSB = ((kOffSc + 2 * kScFloats * 4 + 255) / 256) * 256;   // S bf16, SW32
constexpr uint32_t kOffEB = kOffSB + 128 * 32;     // E  bf16, SW32, 2 buffers (chunk parity)
constexpr uint32_t kOffEP = kOffEB + 2 * 64 * 32;  // E' bf16, SW32, 2 buffers
constexpr uint32_t kOffBar = kOffEP + 2 * 64 * 32;
// mbarriers.  A chain slot is filled in two parts: A = Q and W (read by MMA1 only, so
// released as soon as MMA1 completes) and B = K, P, U and the scalars.
//   fullA[2], fullB[2], freeA[2], freeB[2] (chain ring), ptma, g1, wu (prep), m1,
//   m2s (K^T E'), m2p (P E), eready[2] (E of a slot's chunk is in shared memory and
//   K^T E' has been issued)
// (Loader A tells loader B how many records it has acquired through a monotonic
// counter, not an mbarrier: A may run two chunks ahead of B, and an mbarrier
// phase that advances twice between two looks of its waiter is ambiguous.)
constexpr uint32_t kBarFullA = 0, kBarFullB = 2, kBarFreeA = 4, kBarFreeB = 6, kBarPTma = 8, kBarG1 = 9,
                   kBarWU = 10, kBarM1 = 11, kBarM2S = 12, kBarM2P = 13, kBarEReady = 14, kNumBars = 16;
constexpr uint32_t kFreeBArrivals = 3;  // chain thread 0, one lane of each output warp
constexpr uint32_t kBytesA = 4 * 8192;                          // Q0, Q1, W0, W1
constexpr uint32_t kBytesB = 2 * 8192 + 8192 + 4096 + 528;      // K0, K1, P, U slice, scalars
constexpr uint32_t kOffTmemSlot = kOffBar + kNumBars * 8;
constexpr uint32_t kOffAbort = kOffTmemSlot + 4;
constexpr uint32_t kOffRecOk = kOffAbort + 4;      // records acquired by loader A (monotonic)
constexpr uint32_t kSmemUsed = kOffRecOk + 4;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;

// prep scalar table (floats)
enum : uint32_t {
    SC_G = 0, SC_BETA = 64, SC_RK = 128, SC_RQ = 192, SC_GQ = 256, SC_GAM = 320, SC_DL = 384,
    SC_EXR = 448, SC_EXC = 512, SC_BGK = 768, SC_MISC = 832,
};

static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kCSlot % 1024 == 0 && kOffPrep % 1024 == 0 && kOffTp % 1024 == 0, "SW128 alignment");
static_assert(4 * tc::kMS * 32 * 4 <= kTile, "solve scratch fits in the T tile");
// P E reads a 128-row A operand from P; rows 64-127 (never read back) must stay in shared memory
static_assert(kCSlot + cP + 2 * kTile <= kSmemUsed, "P operand over-read stays inside the allocation");

constexpr uint32_t kIdG1 = idesc_bf16(128, 128, false, false);
constexpr uint32_t kIdM1 = idesc_bf16(128, 16, false, true);
constexpr uint32_t kIdM2S = idesc_bf16(128, 16, true, true);
constexpr uint32_t kIdM2P = idesc_bf16(128, 16, false, true);

struct RingArgs {
    FwdParams p;
    uint8_t* ws;             // workspace: flags, then G * kRing records
    int G;                   // groups (persistent)
    int ncb;                 // CTAs per group = d_v / 16
    uint64_t wait_limit_ns;
};

__device__ __forceinline__ uint64_t kmaj128(uint32_t addr) { return smem_desc(addr, 16, 1024, kSwizzle128); }
__device__ __forceinline__ uint64_t mnmaj128(uint32_t addr, uint32_t lbo) { return smem_desc(addr, lbo, 1024, kSwizzle128); }
__device__ __forceinline__ uint64_t mnmaj32(uint32_t addr) { return smem_desc(addr, 256, 256, kSwizzle32); }

// K step `ks` (16 elements) of a K-major operand whose d axis is split into two
// SW128 column groups `half` bytes apart.
__device__ __forceinline__ uint32_t dstep(uint32_t tile, int ks, uint32_t half) {
    return tile + (ks >= 4 ? half : 0u) + (uint32_t)(ks & 3) * 32u;
}

__device__ __forceinline__ uint32_t tmem_lane(uint32_t tmem, int quarter) {
    return tmem + ((uint32_t)(32 * quarter) << 16);
}

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }

__device__ __forceinline__ float softplus_fast(float x) {
    return fmaxf(x, 0.0f) + __logf(1.0f + __expf(-fabsf(x)));
}
__device__ __forceinline__ float sigmoid_fast(float x) {
    return __fdividef(1.0f, 1.0f + __expf(-x));
}

// Group-local barrier that also returns the AND of `v` over the group.
__device__ __forceinline__ bool group_all(uint32_t id, uint32_t n, bool v) {
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\t"
                 "setp.ne.u32 p, %3, 0;\n\t"
                 "bar.red.and.pred q, %1, %2, p;\n\t"
                 "selp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r) : "r"(id), "r"(n), "r"(v ? 1u : 0u) : "memory");
    return r != 0;
}

// Row `row` of a 16-column bf16 tile in the SW32 layout.
__device__ __forceinline__ void store_row16_sw32(uint32_t tile, uint32_t row, const float (&x)[16]) {
    st_shared_v4(tile + sw32_chunk_offset(row, 0), pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                 pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
    st_shared_v4(tile + sw32_chunk_offset(row, 1), pack_bf16x2(x[8], x[9]), pack_bf16x2(x[10], x[11]),
                 pack_bf16x2(x[12], x[13]), pack_bf16x2(x[14], x[15]));
}

__device__ __forceinline__ void store8_sw128(uint32_t tile, uint32_t row, uint32_t col, const float* x) {
    st_shared_v4(tile + sw128_offset(row, col), pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                 pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
}

// 8 consecutive columns of row `row` of a SW128 image in global memory.
__device__ __forceinline__ void gstore8_sw128(uint8_t* img, uint32_t row, uint32_t col, const float* x) {
    st_global_v4(img + sw128_offset(row, col), pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                 pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
}

// Spin (bounded) until *flag >= want.  Gives up, raising both abort words and
// recording `code`, after `limit_ns` or as soon as an abort word is raised.
__device__ __noinline__ bool wait_flag(const uint64_t* flag, uint64_t want, volatile int* abort_cta,
                                       uint64_t* abort_glob, uint64_t limit_ns, int code) {
    if (ld_acquire_u64(flag) >= want) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        __nanosleep(32);
        if (ld_acquire_u64(flag) >= want) return true;
        if ((it & 15u) == 0) {
            if (*abort_cta || *reinterpret_cast<volatile uint64_t*>(abort_glob) != 0) {
                *abort_cta = 1;
                return false;
            }
            if (globaltimer_ns() - t0 > limit_ns) {
                *abort_cta = 1;
                *reinterpret_cast<volatile uint64_t*>(abort_glob) = 1;
                atomicCAS(&g_device_status, 0, code);
                return false;
            }
        }
    }
}

// Spin (bounded) until the shared-memory counter at `addr` reaches `want`.
__device__ __noinline__ bool wait_counter(uint32_t addr, uint32_t want, volatile int* abort_cta, uint64_t limit_ns,
                                          int code) {
    if (ld_acquire_cta_shared(addr) >= want) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        __nanosleep(32);
        if (ld_acquire_cta_shared(addr) >= want) return true;
        if ((it & 15u) == 0) {
            if (*abort_cta) return false;
            if (globaltimer_ns() - t0 > limit_ns) {
                *abort_cta = 1;
                atomicCAS(&g_device_status, 0, code);
                return false;
            }
        }
    }
}

// The whole warp waits (bounded) until flags[v] >= want for every v < nflags, one
// flag per lane, and returns in `known` the smallest value it saw (flags only
// grow, so a later, smaller `want` needs no new reads).
__device__ __forceinline__ bool wait_flags_warp(const uint64_t* flags, int nflags, uint64_t want, uint64_t& known,
                                                volatile int* abort_cta, uint64_t* abort_glob, uint64_t limit_ns,
                                                int code) {
    const int lane = threadIdx.x & 31;
    bool ok = true;
    uint64_t seen = ~0ull;
    if (lane < nflags) {
        seen = ld_acquire_u64(flags + lane);
        if (seen < want) {
            ok = wait_flag(flags + lane, want, abort_cta, abort_glob, limit_ns, code);
            seen = want;
        }
    }
    ok = __all_sync(0xffffffffu, ok);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const uint64_t o = __shfl_xor_sync(0xffffffffu, seen, off);
        seen = o < seen ? o : seen;
    }
    known = seen;
    return ok;
}

// Where a chunk of group g lives: chain x = (b, h), chunk c of that chain and
// its valid length L.  Chunks of a group are numbered chain after chain, so a
// cursor advances by a fixed stride without per-chunk divisions.
struct Item {
    int x, b, h, c, L;
};
__device__ __forceinline__ void item_set(Item& it, const FwdParams& p, int x, int c) {
    it.x = x;
    it.b = x / p.H;
    it.h = x - it.b * p.H;
    it.c = c;
    it.L = min(kC, p.T - c * kC);
}
// chunk n of group g (one division, for the start of a cursor)
__device__ __forceinline__ Item item_at(const FwdParams& p, int g, int G, int ntk, int n) {
    Item it;
    const int k = n / ntk;
    item_set(it, p, g + k * G, n - k * ntk);
    return it;
}
// advance by `step` chunks
__device__ __forceinline__ void item_advance(Item& it, const FwdParams& p, int G, int ntk, int step) {
    int c = it.c + step, x = it.x;
    if (c >= ntk) {
        while (c >= ntk) { c -= ntk; x += G; }
        item_set(it, p, x, c);
    } else {
        it.c = c;
        it.L = min(kC, p.T - c * kC);
    }
}


// Gates (G, beta) and decay tables of chunk jt into `scx`, run by the 128 prep
// threads of warps pw 4-7 (out of line: it has two call sites).
__device__ __noinline__ void prep_gates_tables(const FwdParams& p, const Item& jt, float* scx, int pw, int lane,
                                               int pt) {
    const int L = jt.L;
    if (pw == 4) {
        const int i0 = 2 * lane, i1 = i0 + 1, t0 = jt.c * kC + i0;
        float g0 = 0.0f, g1 = 0.0f, r0 = 0.0f, r1 = 0.0f;
        if (i0 < L) {
            g0 = __ldg(p.gate + ((size_t)jt.b * p.F + t0 / p.frame_len) * p.H + jt.h);
            r0 = __ldg(p.beta + ((size_t)jt.b * p.T + t0) * p.H + jt.h);
        }
        if (i1 < L) {
            g1 = __ldg(p.gate + ((size_t)jt.b * p.F + (t0 + 1) / p.frame_len) * p.H + jt.h);
            r1 = __ldg(p.beta + ((size_t)jt.b * p.T + t0 + 1) * p.H + jt.h);
        }
        const float la0 = (i0 < L && gate_applies(p, t0)) ? -softplus_fast(g0) : 0.0f;
        const float la1 = (i1 < L && gate_applies(p, t0 + 1)) ? -softplus_fast(g1) : 0.0f;
        float x = la0 + la1;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y;
        }
        scx[SC_G + i0] = x - la1;
        scx[SC_G + i1] = x;
        scx[SC_BETA + i0] = (i0 < L) ? sigmoid_fast(r0) : 0.0f;
        scx[SC_BETA + i1] = (i1 < L) ? sigmoid_fast(r1) : 0.0f;
    }
    named_bar_sync(kBarPrepHi, 128);
    const float GL = scx[SC_G + L - 1];
    for (int idx = pt - 128; idx < 256; idx += 128) {
        if (idx < 64) {
            const int i = idx;
            const float Gi = scx[SC_G + i];
            scx[SC_GAM + i] = __expf(Gi);
            scx[SC_DL + i] = (i < L) ? __expf(GL - Gi) : 0.0f;     // times 1/|k_i| later
            scx[SC_EXR + i] = (i >= 16) ? __expf(Gi - scx[SC_G + 16 * (i >> 4) - 1]) : 1.0f;
            if (i == 0) scx[SC_MISC] = __expf(GL);
        } else {
            const int bi = 1 + (idx - 64) / 64, j = idx & 63;
            scx[SC_EXC + 64 * bi + j] = (j < 16 * bi) ? __expf(scx[SC_G + 16 * bi - 1] - scx[SC_G + j]) : 0.0f;
        }
    }
}

// ---------------------------------------------------------------- MMA issue (one warp)

// prep: [K;Q][K;Q]^T (M = N = 128, K = d_k)
// (K loops are unrolled to their maximum with a warp-uniform guard, so that the
// descriptors are a base plus compile-time offsets)
__device__ __forceinline__ void issue_g1(uint32_t prep, uint32_t tmem, int nks) {
    for (int ks = 0; ks < nks; ++ks) {
        const uint64_t a = kmaj128(dstep(prep + pK0, ks, kPHalf));
        mma_bf16_warp(tmem + kColG, a, a, kIdG1, ks > 0);
    }
}

// prep: [T';T] K (N = d_k) and [T';T] V (N = d_v), K = 64 tokens
__device__ __forceinline__ void issue_wu(uint32_t prep, uint32_t tp, uint32_t tmem, int dk, int dv) {
    const uint32_t idw = idesc_bf16(128, dk, false, true);
    const uint32_t idu = idesc_bf16(128, dv, false, true);
#pragma unroll
    for (int ks = 0; ks < kC / 16; ++ks) {
        const uint64_t a = kmaj128(tp + (uint32_t)ks * 32u);
        mma_bf16_warp(tmem + kColW, a, mnmaj128(prep + pK0 + (uint32_t)ks * 2048u, kPHalf), idw, ks > 0);
        mma_bf16_warp(tmem + kColU, a, mnmaj128(prep + pV0 + (uint32_t)ks * 2048u, pV1 - pV0), idu, ks > 0);
    }
}

// chain: [Q;W] S (M = 128, N = 16, K = d_k) into accumulator buffer qb.  Four buffers:
// MMA1 of chunk n + 4 can only start after the output warps released chunk n's slot.
__device__ __forceinline__ void issue_m1(uint32_t slot, uint32_t sb, uint32_t tmem, int nks, int qb) {
#pragma unroll
    for (int ks = 0; ks < 8; ++ks)
        if (ks < nks)
            mma_bf16_warp(tmem + kColQW + 16u * qb, kmaj128(dstep(slot + cQ0, ks, kCHalfQ)),
                          mnmaj32(sb + (uint32_t)ks * 512u), kIdM1, ks > 0);
}

// chain: K^T E' (M = 128 over d_k), K = 64 tokens: the state increment
__device__ __forceinline__ void issue_m2s(uint32_t slot, uint32_t ep, uint32_t tmem) {
#pragma unroll
    for (int ks = 0; ks < kC / 16; ++ks)
        mma_bf16_warp(tmem + kColS, mnmaj128(slot + cK0 + (uint32_t)ks * 2048u, kCHalfK),
                      mnmaj32(ep + (uint32_t)ks * 512u), kIdM2S, ks > 0);
}

// chain: [P;X] E (rows 0-63 used), K = 64 tokens: the intra-chunk part of the output
__device__ __forceinline__ void issue_m2p(uint32_t slot, uint32_t eb, uint32_t tmem, int s) {
#pragma unroll
    for (int ks = 0; ks < kC / 16; ++ks)
        mma_bf16_warp(tmem + kColPE + 16u * s, kmaj128(slot + cP + (uint32_t)ks * 32u),
                      mnmaj32(eb + (uint32_t)ks * 512u), kIdM2P, ks > 0);
}

// ---------------------------------------------------------------- the kernel

__global__ void __launch_bounds__(kThreads, 1)
gdn_ring_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const RingArgs args)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gb = smem_raw + (base - raw);
    const FwdParams& p = args.p;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, qtr = warp & 3;
    const int vb = blockIdx.x, g = blockIdx.y, G = args.G, ncb = args.ncb;
    const int dk = p.dk, dv = p.dv, nks = dk / 16;
    const int ntk = (p.T + kC - 1) / kC;
    const int nchains = (p.B * p.H - g + G - 1) / G;
    const int total = nchains * ntk;                  // chunks served by this group
    const uint32_t recb = rec_bytes(dv);
    uint64_t* abort_glob = reinterpret_cast<uint64_t*>(args.ws);
    uint64_t* ready = abort_glob + 1 + (size_t)g * kGroupFlags;
    uint64_t* consumed = ready + kRing;
    uint8_t* recs = args.ws + flags_bytes(G) + (size_t)g * kRing * recb;

    float* AXI = reinterpret_cast<float*>(gb + kOffAXI);
    float* MSf = reinterpret_cast<float*>(gb + kOffT);
    float* sc0 = reinterpret_cast<float*>(gb + kOffSc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gb + kOffAbort);
    const uint32_t bars = base + kOffBar;
    auto bar = [&](uint32_t i) { return bars + 8u * i; };
    const uint32_t sbt = base + kOffSB, ebt = base + kOffEB, ept = base + kOffEP;
    const uint32_t prep = base + kOffPrep;
    const uint64_t lim = args.wait_limit_ns;

    if (warp == 0) {
        tmem_alloc(base + kOffTmemSlot, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 32) {
        for (uint32_t i = 0; i < kNumBars; ++i)
            mbar_init(bar(i), (i == kBarFreeB || i == kBarFreeB + 1) ? kFreeBArrivals : 1u);
        fence_mbar_init();
        *abort_flag = 0;
        *reinterpret_cast<volatile uint32_t*>(gb + kOffRecOk) = 0u;
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gb + kOffTmemSlot);

    if (warp < 4) {
        // ======================= chain (warps 0-3) =======================
        // Per chunk n (slot and accumulator parity s = n & 1): MMA1 [Q;W] S ->
        // E = U - W S (warps 2-3) -> K^T E' -> S update.  P E and the output are
        // left to the output warps (eready[s] hands E over).
        float S[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) S[j] = 0.0f;
        bool ok = true;
        int pending = -1;                      // barrier of an MMA group not yet waited for
        Item it = item_at(p, g, G, ntk, 0);
        for (int n = 0; n < total; ++n, item_advance(it, p, G, ntk, 1)) {
            const int s = n & 1;
            const uint32_t slot = base + (uint32_t)s * kCSlot;
            const float* csc = reinterpret_cast<const float*>(gb + (uint32_t)s * kCSlot + cSc);
            const float* cu = reinterpret_cast<const float*>(gb + (uint32_t)s * kCSlot + cU);
            const uint32_t eb = ebt + (uint32_t)s * 2048u, ep = ept + (uint32_t)s * 2048u;
            if (it.c == 0) {
                // first chunk of a chain: its initial state (this thread owns row tid)
                const size_t sbase = ((size_t)it.b * p.H + it.h) * (size_t)dk * dv + (size_t)vb * kVB;
#pragma unroll
                for (int j = 0; j < 16; ++j) S[j] = 0.0f;
                if (p.state_in && tid < dk) {
                    const float4* si = reinterpret_cast<const float4*>(p.state_in + sbase + (size_t)tid * dv);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float4 v4 = si[j];
                        S[4 * j] = v4.x; S[4 * j + 1] = v4.y; S[4 * j + 2] = v4.z; S[4 * j + 3] = v4.w;
                    }
                }
                if (tid < dk) store_row16_sw32(sbt, (uint32_t)tid, S);
                fence_proxy_async_smem();
                tc_fence_before();
                named_bar_sync(kBarChain, kChainThreads);
            }
            ok = mbar_wait(bar(kBarFullA + s), (uint32_t)((n >> 1) & 1), abort_flag, lim, 11);
            if (!group_all(kBarChain, kChainThreads, ok)) { ok = false; break; }
            tc_fence_after();
            if (warp == 0) {
                issue_m1(slot, sbt, tmem, nks, n & 3);
                mma_commit_warp(bar(kBarM1));
                mma_commit_warp(bar(kBarFreeA + s));   // Q and W of the slot: read once MMA1 is done
            }
            pending = kBarM1;
            ok = mbar_wait(bar(kBarM1), (uint32_t)(n & 1), abort_flag, lim, 4);
            ok = ok && mbar_wait(bar(kBarFullB + s), (uint32_t)((n >> 1) & 1), abort_flag, lim, 15);
            if (!group_all(kBarChain, kChainThreads, ok)) { ok = false; break; }
            pending = -1;
            tc_fence_after();
            if (qtr >= 2) {
                const int i = 32 * (qtr - 2) + lane;
                float v[16], u[16];
                tmem_ld16(tmem_lane(tmem, qtr) + kColQW + 16u * (uint32_t)(n & 3), v);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 u4 = ld4(cu + q * 256 + i * 4);
                    u[4 * q] = u4.x; u[4 * q + 1] = u4.y; u[4 * q + 2] = u4.z; u[4 * q + 3] = u4.w;
                }
                const float d = csc[RS_DL + i];
                tmem_wait_ld();
                float e[16], e2[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    e[j] = u[j] - v[j];
                    e2[j] = e[j] * d;
                }
                store_row16_sw32(eb, (uint32_t)i, e);
                store_row16_sw32(ep, (uint32_t)i, e2);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(kBarChain, kChainThreads);
            if (warp == 0) {
                tc_fence_after();
                issue_m2s(slot, ep, tmem);
                mma_commit_warp(bar(kBarM2S));
                tc_fence_before();
                if (elect_one()) mbar_arrive(bar(kBarEReady + s));
                __syncwarp();
            }
            pending = kBarM2S;
            ok = mbar_wait(bar(kBarM2S), (uint32_t)(n & 1), abort_flag, lim, 5);
            if (!group_all(kBarChain, kChainThreads, ok)) { ok = false; break; }
            pending = -1;
            tc_fence_after();
            {
                float v[16];
                tmem_ld16(tmem_lane(tmem, qtr) + kColS, v);
                const float gL = csc[RS_GL];
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) S[j] = fmaf(gL, S[j], v[j]);
                if (tid < dk) store_row16_sw32(sbt, (uint32_t)tid, S);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(kBarChain, kChainThreads);
            if (tid == 0) mbar_arrive(bar(kBarFreeB + s));   // U, scalars and K of the slot are done with
            if (it.c == ntk - 1 && p.state_out && tid < dk) {
                // last chunk of the chain: the final state
                const size_t sbase = ((size_t)it.b * p.H + it.h) * (size_t)dk * dv + (size_t)vb * kVB;
                float4* so = reinterpret_cast<float4*>(p.state_out + sbase + (size_t)tid * dv);
#pragma unroll
                for (int j = 0; j < 4; ++j) so[j] = make_float4(S[4 * j], S[4 * j + 1], S[4 * j + 2], S[4 * j + 3]);
            }
        }
        if (!ok && pending >= 0) {
            // MMAs possibly still in flight must finish before TMEM is released
            drain_wait(bar((uint32_t)pending), 0);
            drain_wait(bar((uint32_t)pending), 1);
        }
    } else if (warp < 12) {
        // ======================= prep (warps 4-11) =======================
        // Chunks vb, vb + ncb, vb + 2 ncb, ... of the group.  Overlapped with the
        // current chunk: the next chunk's tiles (fetched once WU has consumed the
        // current ones), its Gram matrices (started when the current record is
        // handed to the publisher) and its gates and decay tables (computed by
        // warps 8-11 while warps 4-7 run the UT inverse).
        const int pt = tid - kChainThreads;   // 0..255
        const int pw = warp - 4;              // 0..7
        bool ok = true;
        int mma_pending = -1;                 // barrier of an MMA group not yet waited for
        int ptma_issued = 0, ptma_waited = 0;
        uint64_t cons_known = 0;              // all CTAs of the group have consumed this many chunks
        auto issue_prep_tma = [&](const Item& jt) {
            const uint32_t pb = bar(kBarPTma);
            const int t0 = jt.c * kC;
            mbar_arrive_expect_tx(pb, 6 * kTile);
            tma_load_4d(prep + pK0, &tm_k, pb, 0, jt.h, t0, jt.b);
            tma_load_4d(prep + pQ0, &tm_q, pb, 0, jt.h, t0, jt.b);
            tma_load_4d(prep + pK1, &tm_k, pb, 64, jt.h, t0, jt.b);
            tma_load_4d(prep + pQ1, &tm_q, pb, 64, jt.h, t0, jt.b);
            tma_load_4d(prep + pV0, &tm_v, pb, 0, jt.h, t0, jt.b);
            tma_load_4d(prep + pV1, &tm_v, pb, 64, jt.h, t0, jt.b);
        };
        // Gram matrices of the chunk whose tiles are in flight (warp pw 4)
        auto start_g1 = [&](int mm) -> bool {
            if (!mbar_wait(bar(kBarPTma), (uint32_t)(mm & 1), abort_flag, lim, 1)) return false;
            tc_fence_after();
            issue_g1(prep, tmem, nks);
            mma_commit_warp(bar(kBarG1));
            return true;
        };
        auto gates_tables = [&](const Item& jt, float* scx) { prep_gates_tables(p, jt, scx, pw, lane, pt); };
        Item it{0, 0, 0, 0, 0};
        if (vb < total) {
            it = item_at(p, g, G, ntk, vb);
            if (pw == 4) {
                if (elect_one()) issue_prep_tma(it);
                __syncwarp();
                ptma_issued = 1;
                ok = start_g1(0);
                if (ok) ptma_waited = 1;
            }
            if (pw >= 4) gates_tables(it, sc0);
            mma_pending = ok ? (int)kBarG1 : -1;
        }
        int m = 0;
        for (int n = vb; n < total; n += ncb, ++m) {
            float* sc = sc0 + (m & 1) * kScFloats;
            float* scn = sc0 + ((m + 1) & 1) * kScFloats;
            uint8_t* rec = recs + (size_t)(n % kRing) * recb;
            Item nx = it;
            item_advance(nx, p, G, ntk, ncb);
            const bool has_next = n + ncb < total;
            // ---- the ring slot must have been consumed by every CTA of the group ----
            bool got = ok;
            if (pw == 0 && n >= kRing && cons_known < (uint64_t)(n - kRing + 1))
                got = wait_flags_warp(consumed, ncb, (uint64_t)(n - kRing + 1), cons_known, abort_flag, abort_glob,
                                      lim, 14) && ok;
            // ---- [K;Q][K;Q]^T (started earlier); gates and tables are in sc ----
            ok = got && mbar_wait(bar(kBarG1), (uint32_t)(m & 1), abort_flag, lim, 2);
            if (!group_all(kBarPrep, kPrepThreads, ok)) { ok = false; break; }
            mma_pending = -1;
            tc_fence_after();
            const uint32_t tg = tmem + kColG;
            // ---- norms from the Gram diagonal: |k_i|^2 (lanes 0-63), |q_i|^2 (lanes 64-127) ----
            if (pw < 4) {
                float v[32];
                tmem_ld16(tmem_lane(tg, qtr) + 32u * qtr, *reinterpret_cast<float(*)[16]>(&v[0]));
                tmem_ld16(tmem_lane(tg, qtr) + 32u * qtr + 16u, *reinterpret_cast<float(*)[16]>(&v[16]));
                tmem_wait_ld();
                float d = 0.0f;
#pragma unroll
                for (int j = 0; j < 32; ++j) d = (j == lane) ? v[j] : d;
                const float r = rsqrtf(d + kNormEps);
                const int i = 32 * (qtr & 1) + lane;
                if (qtr < 2) {
                    sc[SC_RK + i] = r;
                    sc[SC_DL + i] *= r;
                    sc[SC_BGK + i] = sc[SC_BETA + i] * sc[SC_GAM + i] * r;
                } else {
                    sc[SC_RQ + i] = r;
                    sc[SC_GQ + i] = r * sc[SC_GAM + i];
                }
            }
            named_bar_sync(kBarPrep, kPrepThreads);
            // ---- A (fp32, transposed into AXI) and P (bf16 image in the record) ----
            if ((qtr & 1) == 0 && (pw >> 2) == 1) {
                // rows 0-31 x columns 32-63 lie above the diagonal: A has nothing there, P is zero
                if (qtr == 2) {
                    const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int g8 = 0; g8 < 4; ++g8) gstore8_sw128(rec + kRecP, (uint32_t)lane, (uint32_t)(32 + 8 * g8), z);
                }
            } else {
                const int ch = pw >> 2;
                const int i = 32 * (qtr & 1) + lane;
                const int bi = i >> 4;
                const float Gi = sc[SC_G + i], exr = sc[SC_EXR + i];
                const float ri = (qtr < 2) ? sc[SC_BETA + i] * sc[SC_RK + i] : sc[SC_RQ + i];
#pragma unroll 1
                for (int hh = 0; hh < 2; ++hh) {
                    const int j0 = 32 * ch + 16 * hh;
                    float v[16], val[16];
                    tmem_ld16(tmem_lane(tg, qtr) + (uint32_t)j0, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const float4 a = ld4(sc + SC_G + j0 + 4 * q4);
                        const float4 r4 = ld4(sc + SC_RK + j0 + 4 * q4);
                        const float4 e4 = ld4(sc + SC_EXC + 64 * bi + j0 + 4 * q4);
                        const float gj[4] = {a.x, a.y, a.z, a.w};
                        const float rkj[4] = {r4.x, r4.y, r4.z, r4.w};
                        const float ex[4] = {e4.x, e4.y, e4.z, e4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int jj = 4 * q4 + e, j = j0 + jj;
                            const float dec = ((j >> 4) == bi) ? __expf(Gi - gj[e]) : exr * ex[e];
                            const bool keep = (qtr < 2) ? (j < i) : (j <= i);
                            val[jj] = keep ? ri * rkj[e] * v[jj] * dec : 0.0f;
                        }
                    }
                    if (qtr < 2) {
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj)
                            if (j0 + jj < i) AXI[(j0 + jj) * kXS + i] = val[jj];
                    } else {
                        gstore8_sw128(rec + kRecP, (uint32_t)i, (uint32_t)j0, &val[0]);
                        gstore8_sw128(rec + kRecP, (uint32_t)i, (uint32_t)j0 + 8, &val[8]);
                    }
                }
            }
            tc_fence_before();
            named_bar_sync(kBarPrep, kPrepThreads);
            if (pw < 4) {
                // ---- T = (I + A)^{-1} diag(beta), T' = T diag(e^G / |k|) ----
                tc::unit_lower_inverse_64(AXI, MSf, pt);
                const int i = pt >> 1, j0 = 32 * (pt & 1);
#pragma unroll 1
                for (int q = 0; q < 2; ++q) {
                    const int jb = j0 + 16 * q;
                    float tv[16], tpv[16];
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const float4 x4 = ld4(AXI + i * kXS + jb + 4 * q4);
                        const float4 b4 = ld4(sc + SC_BETA + jb + 4 * q4);
                        const float4 f4 = ld4(sc + SC_BGK + jb + 4 * q4);
                        const float xs[4] = {x4.x, x4.y, x4.z, x4.w};
                        const float bs[4] = {b4.x, b4.y, b4.z, b4.w};
                        const float fs[4] = {f4.x, f4.y, f4.z, f4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float x = (jb + 4 * q4 + e <= i) ? xs[e] : 0.0f;
                            tv[4 * q4 + e] = x * bs[e];
                            tpv[4 * q4 + e] = x * fs[e];
                        }
                    }
                    store8_sw128(base + kOffT, (uint32_t)i, (uint32_t)jb, &tv[0]);
                    store8_sw128(base + kOffT, (uint32_t)i, (uint32_t)jb + 8, &tv[8]);
                    store8_sw128(base + kOffTp, (uint32_t)i, (uint32_t)jb, &tpv[0]);
                    store8_sw128(base + kOffTp, (uint32_t)i, (uint32_t)jb + 8, &tpv[8]);
                }
            } else {
                // ---- the chain's per-token scalars into the record; next chunk's gates ----
                float* rs = reinterpret_cast<float*>(rec + rec_sc(dv));
                const int j = pt - 128;
                if (j < 64) {
                    rs[RS_GQ + j] = sc[SC_GQ + j];
                    rs[RS_DL + j] = sc[SC_DL + j];
                } else if (j < 68) {
                    rs[RS_GL + (j - 64)] = (j == 64) ? sc[SC_MISC] : 0.0f;
                }
                if (has_next) gates_tables(nx, scn);
            }
            fence_proxy_async_smem();
            named_bar_sync(kBarPrep, kPrepThreads);
            if (pw == 0) {
                tc_fence_after();
                issue_wu(prep, base + kOffTp, tmem, dk, dv);
                mma_commit_warp(bar(kBarWU));
            }
            mma_pending = kBarWU;
            ok = mbar_wait(bar(kBarWU), (uint32_t)(m & 1), abort_flag, lim, 3);
            if (!group_all(kBarPrep, kPrepThreads, ok)) { ok = false; break; }
            mma_pending = -1;
            tc_fence_after();
            // the prep tiles are free: fetch the next chunk's
            if (pw == 4 && has_next) {
                if (elect_one()) {
                    fence_proxy_async_smem();
                    issue_prep_tma(nx);
                }
                __syncwarp();
                ptma_issued = m + 2;
            }
            // ---- W (TMEM lanes 0-63) and U (lanes 64-127) into the record ----
            {
                const int half = pw >> 2;
                const bool wpart = qtr < 2;
                const int i = wpart ? 32 * qtr + lane : 32 * (qtr - 2) + lane;
                const int ncol = wpart ? dk : dv;
                const uint32_t col0 = (wpart ? kColW : kColU) + 64u * (uint32_t)half;
#pragma unroll 1
                for (int q2 = 0; q2 < 4; q2 += 2) {
                    float v[2][16];
#pragma unroll
                    for (int q = 0; q < 2; ++q)
                        if (64 * half + 16 * (q2 + q) < ncol)
                            tmem_ld16(tmem_lane(tmem, qtr) + col0 + 16u * (q2 + q), v[q]);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int cb = 64 * half + 16 * (q2 + q);
                        if (cb >= ncol) continue;
                        if (wpart) {
                            uint8_t* img = rec + kRecW + (half ? kTile : 0u);
                            gstore8_sw128(img, (uint32_t)i, (uint32_t)(16 * (q2 + q)), &v[q][0]);
                            gstore8_sw128(img, (uint32_t)i, (uint32_t)(16 * (q2 + q) + 8), &v[q][8]);
                        } else {
                            uint8_t* dst = rec + kRecU + (uint32_t)(cb / 16) * 4096u + (uint32_t)i * 16u;
#pragma unroll
                            for (int r = 0; r < 4; ++r)
                                st_global_v4(dst + r * 1024, __float_as_uint(v[q][4 * r]),
                                             __float_as_uint(v[q][4 * r + 1]), __float_as_uint(v[q][4 * r + 2]),
                                             __float_as_uint(v[q][4 * r + 3]));
                        }
                    }
                }
            }
            tc_fence_before();
            if (!group_all(kBarPrep, kPrepThreads, ok)) { ok = false; break; }
            if (pt == 0) {
                // publish: the barrier orders every prep thread's record writes before this
                // thread's release; the proxy fence orders them before the consumers' bulk
                // copies (async proxy)
                fence_proxy_async_global();
                st_release_u64(ready + (n % kRing), (uint64_t)n + 1);
            }
            if (has_next) {
                // next chunk's Gram matrices while its record slot is awaited
                if (pw == 4) {
                    ok = start_g1(m + 1);
                    if (ok) ptma_waited = m + 2;
                }
                mma_pending = ok ? (int)kBarG1 : -1;
            }
            it = nx;
        }
        if (!ok) {
            if (pw == 4) {
                if (ptma_issued > ptma_waited) drain_wait(bar(kBarPTma), (uint32_t)((ptma_issued - 1) & 1));
                if (mma_pending >= 0) drain_wait(bar((uint32_t)mma_pending), (uint32_t)(m & 1));
            }
        }
    } else if (warp < kLoaderA) {
        // ======================= output (warps 12, 13: TMEM lanes 0-63) =======================
        // For chunk n: P E (issued once the chain has written E and issued K^T E'),
        // then O = diag(e^G/|q|) Q S + P E for rows 32*qtr + lane.
        bool ok = true, m2p_pending = false;
        Item it = item_at(p, g, G, ntk, 0);
        const int i = 32 * qtr + lane;
        for (int n = 0; n < total; ++n, item_advance(it, p, G, ntk, 1)) {
            const int s = n & 1;
            const uint32_t slot = base + (uint32_t)s * kCSlot;
            const float* csc = reinterpret_cast<const float*>(gb + (uint32_t)s * kCSlot + cSc);
            ok = mbar_wait(bar(kBarEReady + s), (uint32_t)((n >> 1) & 1), abort_flag, lim, 7);
            if (!group_all(kBarOut, 64, ok)) { ok = false; break; }
            tc_fence_after();
            const float gq = csc[RS_GQ + i];
            if (warp == kOutWarp0) {
                issue_m2p(slot, ebt + (uint32_t)s * 2048u, tmem, s);
                mma_commit_warp(bar(kBarM2P));
            }
            m2p_pending = true;
            ok = mbar_wait(bar(kBarM2P), (uint32_t)(n & 1), abort_flag, lim, 6);
            if (!group_all(kBarOut, 64, ok)) { ok = false; break; }
            m2p_pending = false;
            tc_fence_after();
            float qs[16], pe[16];
            tmem_ld16(tmem_lane(tmem, qtr) + kColQW + 16u * (uint32_t)(n & 3), qs);
            tmem_ld16(tmem_lane(tmem, qtr) + kColPE + 16u * (uint32_t)s, pe);
            tmem_wait_ld();
            if (i < it.L && p.out) {
                uint32_t w[8];
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    w[j] = pack_bf16x2(fmaf(gq, qs[2 * j], pe[2 * j]), fmaf(gq, qs[2 * j + 1], pe[2 * j + 1]));
                __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) +
                                   (((size_t)it.b * p.T + (size_t)it.c * kC + i) * p.H + it.h) * dv +
                                   (size_t)vb * kVB;
                uint4* o4 = reinterpret_cast<uint4*>(o);
                o4[0] = make_uint4(w[0], w[1], w[2], w[3]);
                o4[1] = make_uint4(w[4], w[5], w[6], w[7]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kBarFreeB + s));   // P, E and this chunk's TMEM are done with
        }
        if (!ok && m2p_pending && warp == kOutWarp0) {
            drain_wait(bar(kBarM2P), 0);
            drain_wait(bar(kBarM2P), 1);
        }
    } else if (warp == kLoaderA) {
        // ======================= loader A (warp 14): q and W tiles =======================
        // Part A of chunk n goes into slot s once MMA1 of chunk n - 2 has read the
        // slot's part A, so it runs about two chunks ahead of the chain.  Ready flags
        // are polled 16 chunks at a time (one L2 round trip and one proxy fence per
        // batch while the prep is ahead), then loader B is told the record is ready.
        bool ok = true;
        int issued = 0, ready_upto = 0;
        Item it = item_at(p, g, G, ntk, 0);
        for (int n = 0; n < total; ++n, item_advance(it, p, G, ntk, 1)) {
            const int s = n & 1;
            if (n >= ready_upto) {
                const int j = n + lane;
                bool rdy = true;
                if (lane == 0) {
                    rdy = wait_flag(ready + (n % kRing), (uint64_t)n + 1, abort_flag, abort_glob, lim, 13);
                } else if (lane < kRing && j < total) {
                    rdy = ld_acquire_u64(ready + (j % kRing)) >= (uint64_t)j + 1;
                } else {
                    rdy = false;
                }
                if (!__shfl_sync(0xffffffffu, rdy ? 1 : 0, 0)) { ok = false; break; }
                // chunks n .. n + run - 1 are ready (run >= 1: lanes in order up to the first not ready)
                const uint32_t notready = __ballot_sync(0xffffffffu, !rdy);
                ready_upto = n + (notready ? __ffs(notready) - 1 : 32);
                __syncwarp();                 // orders every lane's acquire before lane 0's copies
                fence_proxy_async_global();
            }
            if (n >= 2) {
                ok = mbar_wait(bar(kBarFreeA + s), (uint32_t)(((n >> 1) - 1) & 1), abort_flag, lim, 12);
                if (!ok) break;
            }
            if (lane == 0) {
                const uint8_t* rec = recs + (size_t)(n % kRing) * recb;
                const uint32_t slot = base + (uint32_t)s * kCSlot;
                const uint32_t fa = bar(kBarFullA + s);
                const int t0 = it.c * kC;
                mbar_arrive_expect_tx(fa, kBytesA);
                bulk_load(slot + cW0, rec + kRecW, kTile, fa);
                bulk_load(slot + cW1, rec + kRecW + kTile, kTile, fa);
                tma_load_4d(slot + cQ0, &tm_q, fa, 0, it.h, t0, it.b);
                tma_load_4d(slot + cQ1, &tm_q, fa, 64, it.h, t0, it.b);
                st_release_cta_shared(base + kOffRecOk, (uint32_t)(n + 1));
            }
            __syncwarp();
            issued = n + 1;
        }
        if (!ok && lane == 0) {
            // copies still in flight must land before shared memory goes away
            for (int n = max(0, issued - 2); n < issued; ++n)
                drain_wait(bar(kBarFullA + (n & 1)), (uint32_t)((n >> 1) & 1));
        }
        __syncwarp();
    } else {
        // ======================= loader B (warp 15): k tile, P, U, scalars =======================
        // Part B of chunk n goes into slot s once chunk n - 2 is done with entirely (chain
        // and output warps).  Then chunks 0 .. n - 2 count as consumed for the producers.
        bool ok = true;
        int issued = 0;
        Item it = item_at(p, g, G, ntk, 0);
        for (int n = 0; n < total; ++n, item_advance(it, p, G, ntk, 1)) {
            const int s = n & 1;
            ok = wait_counter(base + kOffRecOk, (uint32_t)(n + 1), abort_flag, lim, 16);
            if (ok && n >= 2) ok = mbar_wait(bar(kBarFreeB + s), (uint32_t)(((n >> 1) - 1) & 1), abort_flag, lim, 12);
            if (!ok) break;
            if (lane == 0) {
                fence_proxy_async_global();
                const uint8_t* rec = recs + (size_t)(n % kRing) * recb;
                const uint32_t slot = base + (uint32_t)s * kCSlot;
                const uint32_t fbb = bar(kBarFullB + s);
                const int t0 = it.c * kC;
                mbar_arrive_expect_tx(fbb, kBytesB);
                tma_load_4d(slot + cK0, &tm_k, fbb, 0, it.h, t0, it.b);
                tma_load_4d(slot + cK1, &tm_k, fbb, 64, it.h, t0, it.b);
                bulk_load(slot + cP, rec + kRecP, kTile, fbb);
                bulk_load(slot + cU, rec + kRecU + (uint32_t)vb * 4096u, 4096u, fbb);
                bulk_load(slot + cSc, rec + rec_sc(dv), kScCopy, fbb);
                if (n >= 2 && ((n & 1) == 0 || n + 1 == total)) {
                    // chunk n - 2 is done with, and its bulk copies had landed long before
                    st_release_u64(consumed + vb, (uint64_t)(n - 1));
                }
            }
            __syncwarp();
            issued = n + 1;
        }
        if (!ok && lane == 0) {
            for (int n = max(0, issued - 2); n < issued; ++n)
                drain_wait(bar(kBarFullB + (n & 1)), (uint32_t)((n >> 1) & 1));
        }
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace ring

// ---------------------------------------------------------------- host side

bool ring_supported(int dk, int dv, int chunk_len)
{
    // d > 64 keeps both 64-column TMA boxes of q, k and v partly inside the tensor
    return chunk_len == ring::kC && dk % 16 == 0 && dk > 64 && dk <= 128 && dv % 16 == 0 && dv > 64 &&
           dv <= 128;
}

// Number of persistent groups (heads in flight) for B*H chains on the current
// device: every CTA of the cooperative grid must be resident at once.
cudaError_t ring_groups(int BH, int dv, int* groups)
{
    // the dynamic shared memory limit is a per-device setting of the current context: set it on
    // every call (cheap), so that every device and a context re-created after a reset get it
    cudaError_t e = cudaFuncSetAttribute(ring::gdn_ring_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)ring::kSmemBytes);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0, per_sm = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, ring::gdn_ring_kernel, ring::kThreads,
                                                          ring::kSmemBytes);
    if (e != cudaSuccess) return e;
    const int ncb = dv / ring::kVB;
    const int cap = (sms * per_sm) / ncb;
    *groups = BH < cap ? BH : cap;
    return *groups >= 1 ? cudaSuccess : cudaErrorInvalidConfiguration;
}

size_t ring_workspace_bytes(int G, int dv)
{
    return ring::flags_bytes(G) + (size_t)G * ring::kRing * ring::rec_bytes(dv);
}

// ---- static scratch (the allocation-free entry point) ----
// One file-scope device array serves every call of gdn_forward_static_ws in the
// process on a given device: 24 MiB covers the ring of any supported size on a
// device of up to 160 SMs (the largest need, d_v = 80 on 148 SMs, is 21.4 MB).
constexpr size_t kStaticScratchBytes = 24ull << 20;
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

// Address of the static scratch on the current device, looked up once per
// device (the first call on a device must not be inside a stream capture).
// The cache is an atomic per device, so that threads making their first call
// at the same time store the same value without a data race.  A device reset
// (cudaDeviceReset) unloads the module: the cached address is then stale.
cudaError_t static_scratch(void** ptr, size_t* bytes)
{
    constexpr int kMaxDevices = 64;
    static std::atomic<void*> addr[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    void* a = addr[dev].load(std::memory_order_acquire);
    if (!a) {
        e = cudaGetSymbolAddress(&a, g_static_scratch);
        if (e != cudaSuccess) return e;
        addr[dev].store(a, std::memory_order_release);
    }
    *ptr = a;
    *bytes = kStaticScratchBytes;
    return cudaSuccess;
}

cudaError_t launch_ring(const FwdParams& p, void* ws, size_t ws_bytes, cudaStream_t stream)
{
    if (!ring_supported(p.dk, p.dv, ring::kC) || p.T < 1) return cudaErrorInvalidValue;
    int G = 0;
    cudaError_t e = ring_groups(p.B * p.H, p.dv, &G);
    if (e != cudaSuccess) return e;
    if (ws_bytes < ring_workspace_bytes(G, p.dv)) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, p.q, p.dk, p.H, p.T, p.B, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mk, p.k, p.dk, p.H, p.T, p.B, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mv, p.v, p.dv, p.H, p.T, p.B, 64, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    // the flags start from zero on every call; the records need no clearing
    e = cudaMemsetAsync(ws, 0, ring::flags_bytes(G), stream);
    if (e != cudaSuccess) return e;
    ring::RingArgs args;
    args.p = p;
    args.ws = static_cast<uint8_t*>(ws);
    args.G = G;
    args.ncb = p.dv / ring::kVB;
    args.wait_limit_ns = g_wait_limit_ns;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)args.ncb, (unsigned)G);
    cfg.blockDim = dim3(ring::kThreads);
    cfg.dynamicSmemBytes = ring::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, ring::gdn_ring_kernel, mq, mk, mv, args);
}

}  // namespace gdn
