// Tensor-core chunked GDN forward for sm_100a: tcgen05 MMAs with TMEM
// accumulators, operands staged in shared memory by TMA, warp-specialised.
//
// One CTA owns one (batch, head) chain and 16 columns of the d_k x d_v state
// (columns evolve independently, so CTAs of a head never communicate).  Per
// chunk of 64 tokens (notation of gdn_common.cuh):
//
//   G1   [K;Q][K;Q]^T         M=128 N=128 K=d_k   raw Gram matrices (diagonal: |k|^2, |q|^2)
//   ---  A, P from G1 with norms and decay, T = (I+A)^{-1} diag(beta)  (CUDA cores)
//   WU   [T';T] K , [T';T] V  M=128 N=d_k / 16, K=64   (T' = T diag(e^G / |k|))
//   MMA1 [Q;W] S              M=128 N=16  K=d_k   -> Q S (raw q) and W S
//   ---  E = U - W S, E' = diag(e^{G_L-G}/|k|) E  (CUDA cores)
//   MMA2 K^T E' and [P;X] E   M=128 N=16  K=64    -> state increment, P E
//   ---  S <- e^{G_L} S + K^T E' (fp32, registers);  O = diag(e^G/|q|) Q S + P E
//
// Every product is one M=128 instruction stream: stacking two 64-row operands
// ([K;Q], [T';T], [Q;W]) fills the 128 TMEM lanes, and each epilogue warp reads
// only the 32 lanes its warp index may access.
//
// Warp roles.  Only the second half (MMA1, E, MMA2, state) depends on the
// state; the first half ("prep") depends on the chunk's inputs alone.  Warps
// 0-3 (chain group) run the state chain of chunk c while warps 4-11 (prep
// group) prepare chunk c+1, so the two halves overlap.  The state lives in
// fp32 registers of the chain group (thread m owns row m); only its bf16 copy
// feeds MMA1.  Each group issues its own MMAs from one warp (warp-uniform
// operands, elected lane) and waits on its own commit barriers.
//
// Hand-offs (mbarriers): tile loads -> prep (tma_full[slot]); prep -> chain
// (ready[stage]); chain -> prep (stage_free[stage], after the chain has read
// the stage's P, U and scalars).  Tile slots are refilled by the chain group
// once MMA2 of the slot's chunk has completed.  Every wait is bounded.
#include <cudaTypedefs.h>

#include "gdn_common.cuh"
#include "gdn_status.cuh"
#include "gdn_sm100.cuh"

namespace gdn {
namespace tc {

using namespace sm100;

constexpr int kC = 64;             // chunk length
constexpr int kVB = 16;            // state columns per CTA
constexpr int kThreads = 384;      // 12 warps; warp w reads TMEM lanes 32*(w%4) ..
constexpr int kChainThreads = 128; // warps 0-3
constexpr int kPrepThreads = 256;  // warps 4-11
constexpr uint32_t kBarChain = 1, kBarPrep = 2, kBarSolve = 3;   // named barrier ids
constexpr int kSolveThreads = 128; // prep warps 4-7 run the UT inverse
constexpr int kSlots = 3;          // tile ring depth
constexpr uint32_t kTmemCols = 512;

// TMEM columns (fp32 accumulators, 128 lanes each)
constexpr uint32_t kColG = 0;      // [K;Q][K;Q]^T    2 x 128 columns (prep, next chunk prefetched)
constexpr uint32_t kColW = 256;    // [T';T]K         up to 128  (prep)
constexpr uint32_t kColU = 384;    // [T';T]V         2 x 16     (prep -> chain)
constexpr uint32_t kColQW = 416;   // [Q;W]S          16         (chain)
constexpr uint32_t kColS = 432;    // K^T E'          16         (chain)
constexpr uint32_t kColPE = 448;   // [P;X]E          2 x 16     (chain)

// Shared memory (bytes from a 1024-aligned base).  A ring slot holds, for
// d-columns 0-63 and 64-127 in turn, three consecutive 8 KB SW128 tiles
// K | Q | W (so that [K;Q] and [Q;W] are 128-row operands), then the V tile.
constexpr uint32_t kTile = 8192;
constexpr uint32_t kOffK = 0, kOffQ = kTile, kOffW = 2 * kTile;
constexpr uint32_t kHalf = 3 * kTile;              // d-columns 64-127
constexpr uint32_t kOffV = 6 * kTile;              // 64 x 16 bf16, SW32
constexpr uint32_t kSlotBytes = 6 * kTile + 2048;  // 51200
// P[0] | P[1] | T' | T, SW128 tiles of 8 KB.  [P[s]; next tile] is the A operand
// of P E (its second half only feeds TMEM lanes nobody reads); [T';T] feeds WU.
constexpr uint32_t kOffPTT = kSlots * kSlotBytes;
constexpr uint32_t kOffTp = kOffPTT + 2 * kTile;
constexpr uint32_t kOffT = kOffPTT + 3 * kTile;
constexpr uint32_t kXS = 68;                        // row stride (floats) of AXI
// AXI, fp32 [64][68]: (I+A)^{-1} in and below the diagonal (row-major), A
// transposed strictly above it: A(i, j), j < i, at AXI[j][i].
constexpr uint32_t kOffAXI = kOffPTT + 4 * kTile;
constexpr uint32_t kMS = 8;                         // per-warp solve scratch [32][8], kept inside T
constexpr uint32_t kScFloats = 13 * 64 + 16;
constexpr uint32_t kOffSc = kOffAXI + 64 * kXS * 4; // scalars[2]
constexpr uint32_t kOffSB = ((kOffSc + 2 * kScFloats * 4 + 255) / 256) * 256;  // S bf16, SW32
constexpr uint32_t kOffEB = kOffSB + 128 * 32;      // E  bf16, SW32, 64 rows
constexpr uint32_t kOffEP = kOffEB + 64 * 32;       // E' bf16
constexpr uint32_t kOffBar = kOffEP + 64 * 32;
// barriers: tma_full[3], ready[2], gates[2], g1[2], wu, m1, m2
constexpr uint32_t kBarTma = 0, kBarReady = 3, kBarGates = 5, kBarG1 = 7, kBarWU = 9, kBarM1 = 10,
                   kBarM2 = 11, kNumBars = 12;
constexpr uint32_t kOffTmemSlot = kOffBar + kNumBars * 8;
constexpr uint32_t kOffAbort = kOffTmemSlot + 4;
constexpr uint32_t kSmemUsed = kOffAbort + 4;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;   // slack for aligning the base

// scalar table offsets (floats) within one stage
enum : uint32_t {
    SC_G = 0,        // cumulative log-gate G_i
    SC_BETA = 64,    // beta_i (0 beyond the chunk's valid length)
    SC_RK = 128,     // 1 / |k_i|
    SC_RQ = 192,     // 1 / |q_i|
    SC_GQ = 256,     // e^{G_i} / |q_i|
    SC_GAM = 320,    // e^{G_i}
    SC_DL = 384,     // e^{G_L - G_i} / |k_i|   (0 beyond the valid length)
    SC_EXR = 448,    // e^{G_i - G_{16 floor(i/16) - 1}}   (i >= 16)
    SC_EXC = 512,    // [4][64]: e^{G_{16 b - 1} - G_j}      (j < 16 b; row 0 unused)
    SC_BGK = 768,    // beta_j e^{G_j} / |k_j|
    SC_MISC = 832,   // [0] = e^{G_L}
};

static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kOffPTT % 1024 == 0 && kSlotBytes % 1024 == 0, "SW128 tiles need 1024-B alignment");
static_assert(4 * kMS * 32 * 4 <= kTile, "solve scratch fits in the T tile");

constexpr uint32_t kIdG1 = idesc_bf16(128, 128, false, false);
constexpr uint32_t kIdU = idesc_bf16(128, 16, false, true);
constexpr uint32_t kIdM1 = idesc_bf16(128, 16, false, true);
constexpr uint32_t kIdM2S = idesc_bf16(128, 16, true, true);
constexpr uint32_t kIdM2P = idesc_bf16(128, 16, false, true);

// ---------------------------------------------------------------- MMA issue (one warp)

__device__ __forceinline__ uint64_t kmaj128(uint32_t addr) { return smem_desc(addr, 16, 1024, kSwizzle128); }
__device__ __forceinline__ uint64_t mnmaj128(uint32_t addr) { return smem_desc(addr, kHalf, 1024, kSwizzle128); }
__device__ __forceinline__ uint64_t mnmaj32(uint32_t addr) { return smem_desc(addr, 256, 256, kSwizzle32); }

// Start address of the 16-wide K step `ks` of a K-major operand whose K axis
// is d (two SW128 column groups kHalf bytes apart).
__device__ __forceinline__ uint32_t dstep(uint32_t tile, int ks) {
    return tile + (ks >= 4 ? kHalf : 0u) + (uint32_t)(ks & 3) * 32u;
}

__device__ __forceinline__ void issue_g1(uint32_t slot, uint32_t tmem, int nks, int buf) {
    for (int ks = 0; ks < nks; ++ks) {
        const uint64_t a = kmaj128(dstep(slot + kOffK, ks));
        mma_bf16_warp(tmem + kColG + 128u * buf, a, a, kIdG1, ks > 0);
    }
}

__device__ __forceinline__ void issue_wu(uint32_t slot, uint32_t base, uint32_t tmem, int dk, int s) {
    const uint32_t idw = idesc_bf16(128, dk, false, true);
#pragma unroll
    for (int ks = 0; ks < kC / 16; ++ks) {
        const uint64_t a = kmaj128(base + kOffTp + (uint32_t)ks * 32u);      // [T';T]
        mma_bf16_warp(tmem + kColW, a, mnmaj128(slot + kOffK + (uint32_t)ks * 2048u), idw, ks > 0);
        mma_bf16_warp(tmem + kColU + 16u * s, a, mnmaj32(slot + kOffV + (uint32_t)ks * 512u), kIdU, ks > 0);
    }
}

__device__ __forceinline__ void issue_m1(uint32_t slot, uint32_t sb, uint32_t tmem, int nks) {
    for (int ks = 0; ks < nks; ++ks)
        mma_bf16_warp(tmem + kColQW, kmaj128(dstep(slot + kOffQ, ks)), mnmaj32(sb + (uint32_t)ks * 512u),
                      kIdM1, ks > 0);
}

__device__ __forceinline__ void issue_m2(uint32_t slot, uint32_t base, uint32_t eb, uint32_t ep,
                                         uint32_t tmem, int s) {
    const uint32_t pa = base + kOffPTT + kTile * (uint32_t)s;
#pragma unroll
    for (int ks = 0; ks < kC / 16; ++ks) {
        mma_bf16_warp(tmem + kColS, mnmaj128(slot + kOffK + (uint32_t)ks * 2048u),
                      mnmaj32(ep + (uint32_t)ks * 512u), kIdM2S, ks > 0);
        mma_bf16_warp(tmem + kColPE + 16u * s, kmaj128(pa + (uint32_t)ks * 32u),
                      mnmaj32(eb + (uint32_t)ks * 512u), kIdM2P, ks > 0);
    }
}

// TMA loads of chunk c (tokens c*64 ..) into a ring slot (one elected lane).
__device__ __forceinline__ void issue_tma(const CUtensorMap* tq, const CUtensorMap* tk,
                                          const CUtensorMap* tv, uint32_t slot, uint32_t bar,
                                          int c, int h, int b, int vb) {
    mbar_arrive_expect_tx(bar, 4 * kTile + 2048);
    const int t0 = c * kC;
    tma_load_4d(slot + kOffK, tk, bar, 0, h, t0, b);
    tma_load_4d(slot + kOffQ, tq, bar, 0, h, t0, b);
    tma_load_4d(slot + kHalf + kOffK, tk, bar, 64, h, t0, b);
    tma_load_4d(slot + kHalf + kOffQ, tq, bar, 64, h, t0, b);
    tma_load_4d(slot + kOffV, tv, bar, vb * kVB, h, t0, b);
}

// ---------------------------------------------------------------- helpers

// Gates with the hardware exp2/log2 approximations (results feed bf16 outputs).
__device__ __forceinline__ float softplus_fast(float x) {
    return fmaxf(x, 0.0f) + __logf(1.0f + __expf(-fabsf(x)));
}
__device__ __forceinline__ float sigmoid_fast(float x) {
    return __fdividef(1.0f, 1.0f + __expf(-x));
}

// Row `row` of a 16-column bf16 tile in the SW32 layout (two 16-byte chunks).
__device__ __forceinline__ void store_row16_sw32(uint32_t tile, uint32_t row, const float (&x)[16]) {
    st_shared_v4(tile + sw32_chunk_offset(row, 0), pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                 pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
    st_shared_v4(tile + sw32_chunk_offset(row, 1), pack_bf16x2(x[8], x[9]), pack_bf16x2(x[10], x[11]),
                 pack_bf16x2(x[12], x[13]), pack_bf16x2(x[14], x[15]));
}

// 8 consecutive columns (col % 8 == 0) of row `row` of a SW128 tile.
__device__ __forceinline__ void store8_sw128(uint32_t tile, uint32_t row, uint32_t col, const float* x) {
    st_shared_v4(tile + sw128_offset(row, col), pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                 pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
}

__device__ __forceinline__ uint32_t tmem_lane(uint32_t tmem, int quarter) {
    return tmem + ((uint32_t)(32 * quarter) << 16);
}

// Sum of squares of the 64 bf16 values of one SW128 tile row (any order).
__device__ __forceinline__ float row_sumsq(const uint8_t* row128) {
    const uint4* r = reinterpret_cast<const uint4*>(row128);
    float s = 0.0f;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint4 u = r[c];
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float lo = __uint_as_float(w[k] << 16), hi = __uint_as_float(w[k] & 0xFFFF0000u);
            s = fmaf(lo, lo, s);
            s = fmaf(hi, hi, s);
        }
    }
    return s;
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

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ void st4(float* p, float a, float b, float c, float d) {
    *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
}

struct TcArgs {
    FwdParams p;
    uint64_t wait_limit_ns;
};

// ---------------------------------------------------------------- UT inverse

// A(i, j) for j < i lives transposed above the diagonal of AXI.
__device__ __forceinline__ float AAt(const float* AXI, int i, int j) { return AXI[j * kXS + i]; }
// (I+A)^{-1}(i, j): row-major in and below the diagonal, zero above it.
__device__ __forceinline__ float XIv(const float* AXI, int i, int j) { return (i >= j) ? AXI[i * kXS + j] : 0.0f; }

__device__ __forceinline__ uint32_t tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

// D (16x8) += A (16x8, row) * B (8x8, col), tf32 inputs, fp32 accumulate.  Lane
// l holds A rows g, g+8 / cols t, t+4; B rows t, t+4 / col g; D rows g, g+8 /
// cols 2t, 2t+1, with g = l / 4, t = l % 4.
__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                                uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
                 "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One 16-row x 8-column tile of  X (rows r0.., K columns c0..) * Y (K rows k0.., 8 columns n0..),
// X and Y given as element functors, K a multiple of 8.
template <int K, typename XF, typename YF>
__device__ __forceinline__ void tile16x8(float (&d)[4], XF X, YF Y, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int kk = 0; kk < K; kk += 8)
        mma_tf32_16x8x8(d, tf32(X(g, kk + t)), tf32(X(g + 8, kk + t)), tf32(X(g, kk + t + 4)),
                        tf32(X(g + 8, kk + t + 4)), tf32(Y(kk + t, g)), tf32(Y(kk + t + 4, g)));
}

// Inverse of the unit lower-triangular 64x64 matrix I + A (A strictly lower,
// stored transposed above the diagonal of AXI) into the lower triangle of AXI,
// by forward substitution on the four 16x16 diagonal blocks (fp32 FMA) and two
// levels of block combination  [[X, 0], [C, Y]]^{-1} = [[X^-1, 0], [-Y^-1 C X^-1, Y^-1]]
// whose products run on the tensor cores (mma.sync, tf32 in, fp32 accumulate).
// Every output 8-column tile of a combination depends on the same columns of
// the intermediate product only, so each warp owns whole column tiles and
// keeps its intermediate in a private scratch (MSw: [32][8] per warp).
// Run by the 128 solve threads (st = 0..127, warp pw = st / 32).
__device__ void unit_lower_inverse_64(float* AXI, float* MS, int st) {
    const int pw = st >> 5, lane = st & 31, g = lane >> 2, t = lane & 3;
    if (st < 64) {
        // column j of the inverse of diagonal block o: right-looking substitution, so
        // that the updates of step m are independent of each other
        const int o = 16 * (st >> 4), j = st & 15;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = (i == j) ? 1.0f : 0.0f;
#pragma unroll
        for (int m = 0; m < 15; ++m)
#pragma unroll
            for (int i = m + 1; i < 16; ++i) x[i] = fmaf(-AAt(AXI, o + i, o + m), x[m], x[i]);
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if (i >= j) AXI[(o + i) * kXS + o + j] = x[i];
    }
    named_bar_sync(kBarSolve, kSolveThreads);
    float* MSw = MS + pw * 32 * kMS;
    // level 1: blocks (1,0) and (3,2): Y = -D_hi^{-1} (A_{hi,lo} D_lo^{-1}); warp -> (pair, 8 columns)
    {
        const int pr = pw >> 1, n0 = 8 * (pw & 1);
        const int hi = 16 * (2 * pr + 1), lo = 16 * (2 * pr);
        float m1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        tile16x8<16>(m1, [&](int r, int k) { return AAt(AXI, hi + r, lo + k); },
                     [&](int k, int n) { return XIv(AXI, lo + k, lo + n0 + n); }, lane);
        MSw[g * kMS + 2 * t] = m1[0];
        MSw[g * kMS + 2 * t + 1] = m1[1];
        MSw[(g + 8) * kMS + 2 * t] = m1[2];
        MSw[(g + 8) * kMS + 2 * t + 1] = m1[3];
        __syncwarp();
        float y[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        tile16x8<16>(y, [&](int r, int k) { return XIv(AXI, hi + r, hi + k); },
                     [&](int k, int n) { return MSw[k * kMS + n]; }, lane);
        AXI[(hi + g) * kXS + lo + n0 + 2 * t] = -y[0];
        AXI[(hi + g) * kXS + lo + n0 + 2 * t + 1] = -y[1];
        AXI[(hi + g + 8) * kXS + lo + n0 + 2 * t] = -y[2];
        AXI[(hi + g + 8) * kXS + lo + n0 + 2 * t + 1] = -y[3];
    }
    named_bar_sync(kBarSolve, kSolveThreads);
    // level 2: block rows 32-63, columns 0-31; warp -> 8 columns
    {
        const int n0 = 8 * pw;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            float m2[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            tile16x8<32>(m2, [&](int r, int k) { return AAt(AXI, 32 + 16 * mt + r, k); },
                         [&](int k, int n) { return XIv(AXI, k, n0 + n); }, lane);
            MSw[(16 * mt + g) * kMS + 2 * t] = m2[0];
            MSw[(16 * mt + g) * kMS + 2 * t + 1] = m2[1];
            MSw[(16 * mt + g + 8) * kMS + 2 * t] = m2[2];
            MSw[(16 * mt + g + 8) * kMS + 2 * t + 1] = m2[3];
        }
        __syncwarp();
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            float y[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            tile16x8<32>(y, [&](int r, int k) { return XIv(AXI, 32 + 16 * mt + r, 32 + k); },
                         [&](int k, int n) { return MSw[k * kMS + n]; }, lane);
            const int r0 = 32 + 16 * mt + g;
            AXI[r0 * kXS + n0 + 2 * t] = -y[0];
            AXI[r0 * kXS + n0 + 2 * t + 1] = -y[1];
            AXI[(r0 + 8) * kXS + n0 + 2 * t] = -y[2];
            AXI[(r0 + 8) * kXS + n0 + 2 * t + 1] = -y[3];
        }
    }
    named_bar_sync(kBarSolve, kSolveThreads);
}

// ---------------------------------------------------------------- the kernel

__global__ void __launch_bounds__(kThreads, 1)
gdn_chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const TcArgs args)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gb = smem_raw + (base - raw);
    const FwdParams& p = args.p;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, qtr = warp & 3;
    const int vb = blockIdx.x, bh = blockIdx.y, b = bh / p.H, h = bh % p.H;
    const int dk = p.dk, dv = p.dv, nks = dk / 16;
    const int ntk = (p.T + kC - 1) / kC;

    float* AXI = reinterpret_cast<float*>(gb + kOffAXI);
    float* MSf = reinterpret_cast<float*>(gb + kOffT);
    float* scal = reinterpret_cast<float*>(gb + kOffSc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gb + kOffAbort);
    const uint32_t bars = base + kOffBar;
    auto bar = [&](uint32_t i) { return bars + 8u * i; };
    const uint32_t sbt = base + kOffSB, ebt = base + kOffEB, ept = base + kOffEP;
    const uint64_t lim = args.wait_limit_ns;
    const size_t sbase = ((size_t)b * p.H + h) * (size_t)dk * dv + (size_t)vb * kVB;

    if (warp == 0) {
        tmem_alloc(base + kOffTmemSlot, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 32) {
        for (uint32_t i = 0; i < kNumBars; ++i) mbar_init(bar(i), 1);
        fence_mbar_init();
        *abort_flag = 0;
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    // chain group: thread m < 128 owns row m of the 16-column state slice
    float S[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) S[j] = 0.0f;
    if (tid < kChainThreads) {
        const int m = tid;
        if (p.state_in && m < dk) {
            const float4* si = reinterpret_cast<const float4*>(p.state_in + sbase + (size_t)m * dv);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float4 v4 = si[j];
                S[4 * j] = v4.x; S[4 * j + 1] = v4.y; S[4 * j + 2] = v4.z; S[4 * j + 3] = v4.w;
            }
        }
        if (m < dk) store_row16_sw32(sbt, (uint32_t)m, S);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gb + kOffTmemSlot);
    int tma_issued = 0;                    // chain warp 0: chunks whose loads were issued
    if (warp == 0) {
        tma_issued = min(ntk, kSlots);
        if (elect_one())
            for (int c = 0; c < tma_issued; ++c)
                issue_tma(&tm_q, &tm_k, &tm_v, base + (uint32_t)c * kSlotBytes, bar(kBarTma + c), c, h, b, vb);
        __syncwarp();
    }

    bool ok = true;
    if (warp < 4) {
        // ======================= chain group =======================
        float QS[16];
        float gq = 0.0f;                       // e^{G_i} / |q_i| of this thread's output row
#pragma unroll
        for (int j = 0; j < 16; ++j) QS[j] = 0.0f;
        // raw gate / beta logits of tokens 2*lane and 2*lane+1 of chunk cc (warp 0)
        auto load_logits = [&](int cc, float& g0, float& g1, float& r0, float& r1) {
            const int t0 = cc * kC + 2 * lane, Lc = min(kC, p.T - cc * kC);
            g0 = g1 = r0 = r1 = 0.0f;
            if (2 * lane < Lc) {
                g0 = __ldg(p.gate + ((size_t)b * p.F + t0 / p.frame_len) * p.H + h);
                r0 = __ldg(p.beta + ((size_t)b * p.T + t0) * p.H + h);
            }
            if (2 * lane + 1 < Lc) {
                g1 = __ldg(p.gate + ((size_t)b * p.F + (t0 + 1) / p.frame_len) * p.H + h);
                r1 = __ldg(p.beta + ((size_t)b * p.T + t0 + 1) * p.H + h);
            }
        };
        float pg0 = 0.0f, pg1 = 0.0f, pb0 = 0.0f, pb1 = 0.0f;
        if (warp == 0 && ntk > 0) load_logits(0, pg0, pg1, pb0, pb1);
        // Gates and decay tables of chunk cc into stage cc & 1 (whose previous chunk
        // the chain has finished), then release them to the prep group.
        auto compute_gates = [&](int cc) {
            float* sc = scal + (cc & 1) * kScFloats;
            const int L = min(kC, p.T - cc * kC);
            if (warp == 0) {
                const int i0 = 2 * lane, i1 = i0 + 1;
                const float g0 = pg0, g1 = pg1, r0 = pb0, r1 = pb1;
                if (cc + 1 < ntk) load_logits(cc + 1, pg0, pg1, pb0, pb1);
                const float la0 = (i0 < L && gate_applies(p, cc * kC + i0)) ? -softplus_fast(g0) : 0.0f;
                const float la1 = (i1 < L && gate_applies(p, cc * kC + i1)) ? -softplus_fast(g1) : 0.0f;
                float x = la0 + la1;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, x, off);
                    if (lane >= off) x += y;
                }
                sc[SC_G + i0] = x - la1;
                sc[SC_G + i1] = x;
                sc[SC_BETA + i0] = (i0 < L) ? sigmoid_fast(r0) : 0.0f;
                sc[SC_BETA + i1] = (i1 < L) ? sigmoid_fast(r1) : 0.0f;
            }
            named_bar_sync(kBarChain, kChainThreads);
            const float GL = sc[SC_G + L - 1];
            if (tid < 64) {
                const int i = tid;
                const float Gi = sc[SC_G + i];
                sc[SC_GAM + i] = __expf(Gi);
                sc[SC_DL + i] = (i < L) ? __expf(GL - Gi) : 0.0f;     // times 1/|k_i| in the prep
                sc[SC_EXR + i] = (i >= 16) ? __expf(Gi - sc[SC_G + 16 * (i >> 4) - 1]) : 1.0f;
                if (i == 0) sc[SC_MISC] = __expf(GL);
            }
            for (int idx = tid; idx < 192; idx += kChainThreads) {
                const int bi = 1 + idx / 64, j = idx & 63;
                sc[SC_EXC + 64 * bi + j] = (j < 16 * bi) ? __expf(sc[SC_G + 16 * bi - 1] - sc[SC_G + j]) : 0.0f;
            }
            named_bar_sync(kBarChain, kChainThreads);
            if (tid == 0) mbar_arrive(bar(kBarGates + (cc & 1)));
        };
        // O = diag(e^G/|q|) Q S + P E for chunk cp (warps 0, 1; rows 32*qtr + lane)
        auto output = [&](int cp) {
            if (qtr >= 2) return;
            const int sp = cp & 1, Lp = min(kC, p.T - cp * kC), i = 32 * qtr + lane;
            float pe[16];
            tmem_ld16(tmem_lane(tmem, qtr) + kColPE + 16u * sp, pe);
            tmem_wait_ld();
            if (i < Lp && p.out) {
                const float sq = gq;
                uint32_t w[8];
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    w[j] = pack_bf16x2(fmaf(sq, QS[2 * j], pe[2 * j]), fmaf(sq, QS[2 * j + 1], pe[2 * j + 1]));
                __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) +
                                   (((size_t)b * p.T + (size_t)cp * kC + i) * p.H + h) * dv + (size_t)vb * kVB;
                uint4* o4 = reinterpret_cast<uint4*>(o);
                o4[0] = make_uint4(w[0], w[1], w[2], w[3]);
                o4[1] = make_uint4(w[4], w[5], w[6], w[7]);
            }
        };
        if (ntk > 0) compute_gates(0);
        int mma_bar = -1;                     // MMA group issued and not yet waited for
        uint32_t mma_par = 0;
        int c = 0;
        for (; c < ntk; ++c) {
            const int s = c & 1;
            const uint32_t slot = base + (uint32_t)(c % kSlots) * kSlotBytes;
            const float* sc = scal + s * kScFloats;
            if (c + 1 < ntk) compute_gates(c + 1);
            ok = mbar_wait(bar(kBarReady + s), (uint32_t)((c >> 1) & 1), abort_flag, lim, 6);
            if (!group_all(kBarChain, kChainThreads, ok)) { ok = false; break; }
            tc_fence_after();
            if (warp == 0) {
                issue_m1(slot, sbt, tmem, nks);
                mma_commit_warp(bar(kBarM1));
            }
            mma_bar = kBarM1;
            mma_par = (uint32_t)(c & 1);
            if (c > 0) output(c - 1);          // previous chunk's output while MMA1 runs
            ok = mbar_wait(bar(kBarM1), (uint32_t)(c & 1), abort_flag, lim, 4);
            if (!group_all(kBarChain, kChainThreads, ok)) { ok = false; break; }
            mma_bar = -1;
            tc_fence_after();
            {
                float v[16];
                tmem_ld16(tmem_lane(tmem, qtr) + kColQW, v);
                if (qtr < 2) {
                    gq = sc[SC_GQ + 32 * qtr + lane];
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) QS[j] = v[j];
                } else {
                    float u[16];
                    tmem_ld16(tmem_lane(tmem, qtr) + kColU + 16u * s, u);
                    tmem_wait_ld();
                    const int i = 32 * (qtr - 2) + lane;
                    const float d = sc[SC_DL + i];
                    float e[16], e2[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        e[j] = u[j] - v[j];
                        e2[j] = e[j] * d;
                    }
                    store_row16_sw32(ebt, (uint32_t)i, e);
                    store_row16_sw32(ept, (uint32_t)i, e2);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(kBarChain, kChainThreads);
            if (warp == 0) {
                tc_fence_after();
                issue_m2(slot, base, ebt, ept, tmem, s);
                mma_commit_warp(bar(kBarM2));
            }
            mma_bar = kBarM2;
            mma_par = (uint32_t)(c & 1);
            ok = mbar_wait(bar(kBarM2), (uint32_t)(c & 1), abort_flag, lim, 5);
            if (!group_all(kBarChain, kChainThreads, ok)) { ok = false; break; }
            mma_bar = -1;
            tc_fence_after();
            {
                const int m = tid;
                float v[16];
                tmem_ld16(tmem_lane(tmem, qtr) + kColS, v);
                tmem_wait_ld();
                const float gL = sc[SC_MISC];
#pragma unroll
                for (int j = 0; j < 16; ++j) S[j] = fmaf(gL, S[j], v[j]);
                if (m < dk) store_row16_sw32(sbt, (uint32_t)m, S);
            }
            // the slot of chunk c is free once MMA2 has read it: refill with chunk c + kSlots
            if (warp == 0 && c + kSlots < ntk) {
                if (elect_one()) {
                    fence_proxy_async_smem();
                    issue_tma(&tm_q, &tm_k, &tm_v, slot, bar(kBarTma + (c % kSlots)), c + kSlots, h, b, vb);
                }
                __syncwarp();
                tma_issued = c + kSlots + 1;
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(kBarChain, kChainThreads);
        }
        if (ok && ntk > 0) output(ntk - 1);
        if (!ok && warp == 0) {
            // drain tile loads and an MMA group still in flight before the shared memory
            // and TMEM go away (bounded)
            if (elect_one()) {
                if (mma_bar >= 0) drain_wait(bar((uint32_t)mma_bar), mma_par);
                for (int cc = max(0, tma_issued - kSlots); cc < tma_issued; ++cc)
                    drain_wait(bar(kBarTma + cc % kSlots), (uint32_t)((cc / kSlots) & 1));
            }
            __syncwarp();
        }
        if (ok && p.state_out && tid < dk) {
            float4* so = reinterpret_cast<float4*>(p.state_out + sbase + (size_t)tid * dv);
#pragma unroll
            for (int j = 0; j < 4; ++j) so[j] = make_float4(S[4 * j], S[4 * j + 1], S[4 * j + 2], S[4 * j + 3]);
        }
    } else {
        // ======================= prep group =======================
        const int pt = tid - kChainThreads;   // 0..255
        const int pw = warp - 4;              // 0..7
        // G1 of chunk cc into accumulator buffer cc & 1, issued by prep warp 4 (not in the solve)
        auto prefetch_g1 = [&](int cc) -> bool {
            const bool got = mbar_wait(bar(kBarTma + (cc % kSlots)), (uint32_t)((cc / kSlots) & 1),
                                       abort_flag, lim, 1);
            if (got) {
                tc_fence_after();
                issue_g1(base + (uint32_t)(cc % kSlots) * kSlotBytes, tmem, nks, cc & 1);
                mma_commit_warp(bar(kBarG1 + (cc & 1)));
            }
            return got;
        };
        bool pre_ok = true;
        int g1_issued = 0, g1_waited = 0;     // chunks whose Gram MMAs were issued / waited for
        int wu_chunk = -1;                    // chunk whose W/U MMAs were issued and not waited for
        if (pw == 4 && ntk > 0) {
            pre_ok = prefetch_g1(0);
            g1_issued = pre_ok ? 1 : 0;
        }
        for (int c = 0; c < ntk; ++c) {
            const int s = c & 1, gbuf = c & 1;
            const uint32_t slot = base + (uint32_t)(c % kSlots) * kSlotBytes;
            float* sc = scal + s * kScFloats;
            ok = pre_ok && mbar_wait(bar(kBarGates + s), (uint32_t)((c >> 1) & 1), abort_flag, lim, 7);
            ok = ok && mbar_wait(bar(kBarTma + (c % kSlots)), (uint32_t)((c / kSlots) & 1), abort_flag, lim, 1);
            ok = ok && mbar_wait(bar(kBarG1 + gbuf), (uint32_t)((c >> 1) & 1), abort_flag, lim, 2);
            if (!group_all(kBarPrep, kPrepThreads, ok)) { ok = false; break; }
            g1_waited = c + 1;
            tc_fence_after();
            const uint32_t tg = tmem + kColG + 128u * gbuf;
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
            // ---- A (fp32, transposed into AXI) and P (bf16 SW128) from the raw Gram matrices ----
            if ((qtr & 1) == 0 && (pw >> 2) == 1) {
                // rows 0-31 x columns 32-63 lie above the diagonal: A has nothing there, P is zero
                if (qtr == 2) {
                    const uint32_t ptile = base + kOffPTT + kTile * (uint32_t)s;
                    const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int g8 = 0; g8 < 4; ++g8) store8_sw128(ptile, (uint32_t)lane, (uint32_t)(32 + 8 * g8), z);
                }
            } else {
                const int ch = pw >> 2;                     // column half: 0-31 or 32-63
                const int i = 32 * (qtr & 1) + lane;        // row within the 64-row matrix
                const int bi = i >> 4;
                const float Gi = sc[SC_G + i], exr = sc[SC_EXR + i];
                const float ri = (qtr < 2) ? sc[SC_BETA + i] * sc[SC_RK + i] : sc[SC_RQ + i];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int j0 = 32 * ch + 16 * hh;
                    float v[16], gj[16], rkj[16], ex[16];
                    tmem_ld16(tmem_lane(tg, qtr) + (uint32_t)j0, v);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const float4 a = ld4(sc + SC_G + j0 + 4 * q4);
                        const float4 r4 = ld4(sc + SC_RK + j0 + 4 * q4);
                        const float4 e4 = ld4(sc + SC_EXC + 64 * bi + j0 + 4 * q4);
                        gj[4 * q4] = a.x; gj[4 * q4 + 1] = a.y; gj[4 * q4 + 2] = a.z; gj[4 * q4 + 3] = a.w;
                        rkj[4 * q4] = r4.x; rkj[4 * q4 + 1] = r4.y; rkj[4 * q4 + 2] = r4.z; rkj[4 * q4 + 3] = r4.w;
                        ex[4 * q4] = e4.x; ex[4 * q4 + 1] = e4.y; ex[4 * q4 + 2] = e4.z; ex[4 * q4 + 3] = e4.w;
                    }
                    tmem_wait_ld();
                    float val[16];
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) {
                        const int j = j0 + jj;
                        const float dec = ((j >> 4) == bi) ? __expf(Gi - gj[jj]) : exr * ex[jj];
                        const bool keep = (qtr < 2) ? (j < i) : (j <= i);
                        val[jj] = keep ? ri * rkj[jj] * v[jj] * dec : 0.0f;
                    }
                    if (qtr < 2) {
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj)
                            if (j0 + jj < i) AXI[(j0 + jj) * kXS + i] = val[jj];
                    } else {
                        const uint32_t ptile = base + kOffPTT + kTile * (uint32_t)s;
                        store8_sw128(ptile, (uint32_t)i, (uint32_t)j0, &val[0]);
                        store8_sw128(ptile, (uint32_t)i, (uint32_t)j0 + 8, &val[8]);
                    }
                }
            }
            tc_fence_before();
            named_bar_sync(kBarPrep, kPrepThreads);
            bool ok2 = true;
            if (pw == 4) {
                // next chunk's Gram matrices run on the tensor cores during this chunk's solve
                if (c + 1 < ntk) {
                    ok2 = prefetch_g1(c + 1);
                    if (ok2) g1_issued = c + 2;
                }
            } else if (pw < 4) {
                // ---- T = (I + A)^{-1} diag(beta), T' = T diag(e^G / |k|) ----
                unit_lower_inverse_64(AXI, MSf, pt);
                const int i = pt >> 1, j0 = 32 * (pt & 1);
#pragma unroll
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
            }
            fence_proxy_async_smem();
            if (!group_all(kBarPrep, kPrepThreads, ok2)) { ok = false; break; }
            if (pw == 0) {
                tc_fence_after();
                issue_wu(slot, base, tmem, dk, s);
                mma_commit_warp(bar(kBarWU));
            }
            wu_chunk = c;
            ok = mbar_wait(bar(kBarWU), (uint32_t)(c & 1), abort_flag, lim, 3);
            if (!group_all(kBarPrep, kPrepThreads, ok)) { ok = false; break; }
            wu_chunk = -1;
            tc_fence_after();
            // ---- W (TMEM lanes 0-63) to smem next to Q ----
            if (qtr < 2) {
                const int i = 32 * qtr + lane;
                const int cbeg = 64 * (pw >> 2);
                for (int cb = cbeg; cb < cbeg + 64 && cb < dk; cb += 16) {
                    float v[16];
                    tmem_ld16(tmem_lane(tmem, qtr) + kColW + (uint32_t)cb, v);
                    tmem_wait_ld();
                    const uint32_t tile = slot + (cb >= 64 ? kHalf : 0u) + kOffW;
                    store8_sw128(tile, (uint32_t)i, (uint32_t)(cb & 63), &v[0]);
                    store8_sw128(tile, (uint32_t)i, (uint32_t)(cb & 63) + 8, &v[8]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(kBarPrep, kPrepThreads);
            if (pt == 0) mbar_arrive(bar(kBarReady + s));
        }
        if (!ok) {
            // Gram MMAs issued and not waited for (chunk cc on buffer cc & 1, its (cc >> 1)-th
            // use), and the W/U group if its wait gave up, must finish before TMEM is freed
            if (pw == 4)
                for (int cc = g1_waited; cc < g1_issued; ++cc)
                    drain_wait(bar(kBarG1 + (cc & 1)), (uint32_t)((cc >> 1) & 1));
            if (pw == 0 && wu_chunk >= 0) drain_wait(bar(kBarWU), (uint32_t)(wu_chunk & 1));
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace tc

// ---------------------------------------------------------------- host side

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// 4-D bf16 map over a [B, T, H, inner] tensor, box {box_inner, 1, 64, 1}.
bool make_map(CUtensorMap* map, const void* base, int inner, int H, int T, int B, int box_inner,
              CUtensorMapSwizzle swz, CUtensorMapL2promotion promo = CU_TENSOR_MAP_L2_PROMOTION_L2_256B)
{
    PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)inner, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)inner * 2, (cuuint64_t)H * inner * 2,
                             (cuuint64_t)T * H * inner * 2};
    cuuint32_t box[4] = {(cuuint32_t)box_inner, 1, (cuuint32_t)tc::kC, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, promo, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;   // 2 s
uint64_t g_wait_limit_ns = kDefaultWaitLimitNs;

}  // namespace

// Bound of every device-side wait of later launches (0 restores the default).
void set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns = ns ? ns : kDefaultWaitLimitNs; }

bool tc_supported(int dk, int dv, int chunk_len)
{
    // d_k > 64 keeps both 64-column TMA boxes of q and k partly inside the tensor
    return chunk_len == tc::kC && dk % 16 == 0 && dk > 64 && dk <= 128 && dv % 16 == 0 && dv <= 128;
}

cudaError_t launch_tc(const FwdParams& p, int chunk_len, cudaStream_t stream)
{
    if (!tc_supported(p.dk, p.dv, chunk_len)) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv;
    const int T = p.T > 0 ? p.T : 1;
    if (!make_map(&mq, p.q, p.dk, p.H, T, p.B, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mk, p.k, p.dk, p.H, T, p.B, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mv, p.v, p.dv, p.H, T, p.B, tc::kVB, CU_TENSOR_MAP_SWIZZLE_32B))
        return cudaErrorInvalidValue;
    // the dynamic shared memory limit is a per-device setting of the current context: set it on
    // every call (cheap), so that every device and a context re-created after a reset get it
    cudaError_t e = cudaFuncSetAttribute(tc::gdn_chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)tc::kSmemBytes);
    if (e != cudaSuccess) return e;
    tc::TcArgs args;
    args.p = p;
    args.wait_limit_ns = g_wait_limit_ns;
    dim3 grid(p.dv / tc::kVB, p.B * p.H);
    tc::gdn_chunk_tc_kernel<<<grid, tc::kThreads, tc::kSmemBytes, stream>>>(mq, mk, mv, args);
    return cudaGetLastError();
}

}  // namespace gdn
