// Tensor-core chunked GDN forward for sm_100a: tcgen05 MMAs with TMEM
// accumulators, operands staged in shared memory by TMA.
//
// One CTA owns one (batch, head) chain and 16 columns of the d_k x d_v state
// (columns evolve independently, so CTAs of a head never communicate).  Per
// chunk of 64 tokens (notation of gdn_common.cuh):
//
//   G1   [K;Q] K^T            M=128 N=64  K=d_k   raw Gram matrices
//   ---  A, P from G1 with norms and decay, T = (I+A)^{-1} diag(beta)  (CUDA cores)
//   WU   [T';T] K , [T';T] V  M=128 N=d_k / 16, K=64   (T' = T diag(e^G / |k|))
//   MMA1 [Q;W] S              M=128 N=16  K=d_k   -> Q S (raw q) and W S
//   ---  E = U - W S, E' = diag(e^{G_L-G}/|k|) E  (CUDA cores)
//   MMA2 K^T E' and [P;T'] E  M=128 N=16  K=64    -> state increment, P E
//   ---  S <- e^{G_L} S + K^T E' (fp32, registers);  O = diag(e^G/|q|) Q S + P E
//
// Every product is one M=128 instruction stream: stacking two 64-row operands
// ([K;Q], [T';T], [Q;W], [P;T']) fills the 128 TMEM lanes, and each epilogue
// warp reads only the 32 lanes its warp index may access.  The state is kept
// in fp32 registers of warps 0-3 (thread m owns row m) for the whole sequence;
// only its bf16 copy feeds MMA1.
#include <cudaTypedefs.h>

#include "gdn_common.cuh"
#include "gdn_status.cuh"
#include "gdn_sm100.cuh"

namespace gdn {
namespace tc {

using namespace sm100;

constexpr int kC = 64;             // chunk length
constexpr int kVB = 16;            // state columns per CTA
constexpr int kThreads = 256;      // 8 warps; warp w reads TMEM lanes 32*(w%4) ..
constexpr int kSlots = 3;          // TMA ring depth (chunks in flight)
constexpr uint32_t kTmemCols = 512;

// TMEM columns (fp32 accumulators, 128 lanes each)
constexpr uint32_t kColG = 0;      // [K;Q]K^T      64 columns
constexpr uint32_t kColW = 64;     // [T';T]K       up to 128 columns
constexpr uint32_t kColU = 192;    // [T';T]V       16
constexpr uint32_t kColQW = 208;   // [Q;W]S        16
constexpr uint32_t kColS = 224;    // K^T E'        16
constexpr uint32_t kColPE = 240;   // [P;T']E       16

// Shared memory (bytes from a 1024-aligned base).  A ring slot holds, for
// d-columns 0-63 and 64-127 in turn, three consecutive 8 KB SW128 tiles
// K | Q | W (so that [K;Q] and [Q;W] are 128-row operands), then the V tile.
constexpr uint32_t kTile = 8192;
constexpr uint32_t kOffK = 0, kOffQ = kTile, kOffW = 2 * kTile;
constexpr uint32_t kHalf = 3 * kTile;             // d-columns 64-127
constexpr uint32_t kOffV = 6 * kTile;             // 64 x 16 bf16, SW32
constexpr uint32_t kSlotBytes = 6 * kTile + 2048;  // 51200
constexpr uint32_t kOffPTT = kSlots * kSlotBytes;  // P | T' | T  (SW128, 8 KB each)
constexpr uint32_t kOffAX = kOffPTT + 3 * kTile;   // fp32 [64][65]: A below, (I+A)^-1 above
constexpr uint32_t kOffMS = kOffAX + 64 * 65 * 4;  // fp32 [32][33] solve scratch
constexpr uint32_t kOffSc = kOffMS + 32 * 33 * 4;  // per-chunk scalars
constexpr uint32_t kScFloats = 11 * 64 + 16;
constexpr uint32_t kOffSB = ((kOffSc + kScFloats * 4 + 255) / 256) * 256;  // S bf16, SW32, 128 rows
constexpr uint32_t kOffEB = kOffSB + 128 * 32;     // E  bf16, SW32, 64 rows
constexpr uint32_t kOffEP = kOffEB + 64 * 32;      // E' bf16
constexpr uint32_t kOffBar = kOffEP + 64 * 32;
constexpr uint32_t kNumBars = kSlots + 4;          // tma_full[3], g1, wu, m1, m2
constexpr uint32_t kOffTmemSlot = kOffBar + kNumBars * 8;
constexpr uint32_t kOffAbort = kOffTmemSlot + 4;
constexpr uint32_t kSmemUsed = kOffAbort + 4;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;  // slack for aligning the base

// scalar table offsets (floats)
enum : uint32_t {
    SC_G = 0,        // cumulative log-gate G_i
    SC_BETA = 64,    // beta_i (0 beyond the chunk's valid length)
    SC_RK = 128,     // 1 / |k_i|
    SC_RQ = 192,     // 1 / |q_i|
    SC_GAM = 256,    // e^{G_i}
    SC_DL = 320,     // e^{G_L - G_i}
    SC_EXR = 384,    // e^{G_i - G_{16 floor(i/16) - 1}}   (i >= 16)
    SC_EXC = 448,    // [4][64]: e^{G_{16 b - 1} - G_j}      (j < 16 b)
    SC_MISC = 704,   // [0] = e^{G_L}
};

static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kOffPTT % 1024 == 0 && kSlotBytes % 1024 == 0, "SW128 tiles need 1024-B alignment");

constexpr uint32_t kIdG1 = idesc_bf16(128, 64, false, false);
constexpr uint32_t kIdU = idesc_bf16(128, 16, false, true);
constexpr uint32_t kIdM1 = idesc_bf16(128, 16, false, true);
constexpr uint32_t kIdM2S = idesc_bf16(128, 16, true, true);
constexpr uint32_t kIdM2P = idesc_bf16(128, 16, false, true);

// ---------------------------------------------------------------- MMA issue (one thread)

__device__ __forceinline__ uint64_t kmaj128(uint32_t addr) { return smem_desc(addr, 16, 1024, kSwizzle128); }
__device__ __forceinline__ uint64_t mnmaj128(uint32_t addr) { return smem_desc(addr, kHalf, 1024, kSwizzle128); }
__device__ __forceinline__ uint64_t mnmaj32(uint32_t addr) { return smem_desc(addr, 256, 256, kSwizzle32); }

// Start address of the 16-wide K step `ks` of a K-major operand whose K axis
// is d (two SW128 column groups kHalf bytes apart).
__device__ __forceinline__ uint32_t dstep(uint32_t tile, int ks) {
    return tile + (ks >= 4 ? kHalf : 0u) + (uint32_t)(ks & 3) * 32u;
}

__device__ __forceinline__ void issue_g1(uint32_t slot, uint32_t tmem, int nks) {
    for (int ks = 0; ks < nks; ++ks) {
        const uint32_t a = dstep(slot + kOffK, ks);
        mma_bf16(tmem + kColG, kmaj128(a), kmaj128(a), kIdG1, ks > 0);
    }
}

__device__ __forceinline__ void issue_wu(uint32_t slot, uint32_t ptt, uint32_t tmem, int dk) {
    const uint32_t idw = idesc_bf16(128, dk, false, true);
    for (int ks = 0; ks < kC / 16; ++ks) {
        const uint64_t a = kmaj128(ptt + kTile + (uint32_t)ks * 32u);      // [T';T]
        mma_bf16(tmem + kColW, a, mnmaj128(slot + kOffK + (uint32_t)ks * 2048u), idw, ks > 0);
        mma_bf16(tmem + kColU, a, mnmaj32(slot + kOffV + (uint32_t)ks * 512u), kIdU, ks > 0);
    }
}

__device__ __forceinline__ void issue_m1(uint32_t slot, uint32_t sb, uint32_t tmem, int nks) {
    for (int ks = 0; ks < nks; ++ks)
        mma_bf16(tmem + kColQW, kmaj128(dstep(slot + kOffQ, ks)), mnmaj32(sb + (uint32_t)ks * 512u),
                 kIdM1, ks > 0);
}

__device__ __forceinline__ void issue_m2(uint32_t slot, uint32_t ptt, uint32_t eb, uint32_t ep,
                                         uint32_t tmem) {
    for (int ks = 0; ks < kC / 16; ++ks) {
        mma_bf16(tmem + kColS, mnmaj128(slot + kOffK + (uint32_t)ks * 2048u),
                 mnmaj32(ep + (uint32_t)ks * 512u), kIdM2S, ks > 0);
        mma_bf16(tmem + kColPE, kmaj128(ptt + (uint32_t)ks * 32u), mnmaj32(eb + (uint32_t)ks * 512u),
                 kIdM2P, ks > 0);
    }
}

// TMA loads of chunk c (tokens c*64 ..) into a ring slot.
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

// ---------------------------------------------------------------- epilogue helpers

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

struct TcArgs {
    FwdParams p;
    uint64_t wait_limit_ns;
};

// (I + A)^{-1} is kept in the upper part of AX: element (i, j), j <= i, at AX[j][i + 1].
__device__ __forceinline__ float& XI(float* AX, int i, int j) { return AX[j * 65 + i + 1]; }
__device__ __forceinline__ float AA(const float* AX, int i, int j) { return AX[i * 65 + j]; }

// Blocked inverse of the unit lower-triangular 64x64 matrix I + A (A strictly
// lower, in AX below the diagonal) by forward substitution on 16x16 diagonal
// blocks and two levels of block combination
//   [[X, 0], [C, Y]]^{-1} = [[X^-1, 0], [-Y^-1 C X^-1, Y^-1]].
// All 256 threads take part; fp32 throughout.
__device__ void unit_lower_inverse_64(float* AX, float* MS, int tid) {
    if (tid < 64) {
        const int o = 16 * (tid >> 4), j = tid & 15;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float acc = (i == j) ? 1.0f : 0.0f;
#pragma unroll
            for (int m = 0; m < i; ++m) acc = fmaf(-AA(AX, o + i, o + m), x[m], acc);
            x[i] = acc;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if (i >= j) XI(AX, o + i, o + j) = x[i];
    }
    __syncthreads();
    // level 1: blocks (1,0) and (3,2)
    for (int idx = tid; idx < 512; idx += kThreads) {
        const int pr = idx >> 8, r = (idx >> 4) & 15, cc = idx & 15;
        const int hi = 16 * (2 * pr + 1), lo = 16 * (2 * pr);
        float acc = 0.0f;
        for (int m = cc; m < 16; ++m) acc = fmaf(AA(AX, hi + r, lo + m), XI(AX, lo + m, lo + cc), acc);
        MS[(16 * pr + r) * 33 + cc] = acc;
    }
    __syncthreads();
    for (int idx = tid; idx < 512; idx += kThreads) {
        const int pr = idx >> 8, r = (idx >> 4) & 15, cc = idx & 15;
        const int hi = 16 * (2 * pr + 1), lo = 16 * (2 * pr);
        float acc = 0.0f;
        for (int m = 0; m <= r; ++m) acc = fmaf(XI(AX, hi + r, hi + m), MS[(16 * pr + m) * 33 + cc], acc);
        XI(AX, hi + r, lo + cc) = -acc;
    }
    __syncthreads();
    // level 2: block rows 32-63, columns 0-31
    for (int idx = tid; idx < 1024; idx += kThreads) {
        const int r = idx >> 5, cc = idx & 31;
        float acc = 0.0f;
        for (int m = cc; m < 32; ++m) acc = fmaf(AA(AX, 32 + r, m), XI(AX, m, cc), acc);
        MS[r * 33 + cc] = acc;
    }
    __syncthreads();
    for (int idx = tid; idx < 1024; idx += kThreads) {
        const int r = idx >> 5, cc = idx & 31;
        float acc = 0.0f;
        for (int m = 0; m <= r; ++m) acc = fmaf(XI(AX, 32 + r, 32 + m), MS[m * 33 + cc], acc);
        XI(AX, 32 + r, cc) = -acc;
    }
    __syncthreads();
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

    float* AX = reinterpret_cast<float*>(gb + kOffAX);
    float* MS = reinterpret_cast<float*>(gb + kOffMS);
    float* sc = reinterpret_cast<float*>(gb + kOffSc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gb + kOffAbort);
    const uint32_t bar0 = base + kOffBar;
    const uint32_t bar_g1 = bar0 + 8u * kSlots, bar_wu = bar_g1 + 8u, bar_m1 = bar_g1 + 16u,
                   bar_m2 = bar_g1 + 24u;
    const uint32_t ptt = base + kOffPTT, sbt = base + kOffSB, ebt = base + kOffEB, ept = base + kOffEP;
    const uint64_t lim = args.wait_limit_ns;
    const size_t sbase = ((size_t)b * p.H + h) * (size_t)dk * dv + (size_t)vb * kVB;

    if (warp == 0) {
        tmem_alloc(base + kOffTmemSlot, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 32) {
        for (uint32_t i = 0; i < kNumBars; ++i) mbar_init(bar0 + 8u * i, 1);
        fence_mbar_init();
        *abort_flag = 0;
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    // state rows: thread m < 128 of warps 0-3 owns row m of the 16-column slice
    float S[16];
    if (tid < 128) {
        const int m = tid;
#pragma unroll
        for (int j = 0; j < 16; ++j)
            S[j] = (p.state_in && m < dk) ? p.state_in[sbase + (size_t)m * dv + j] : 0.0f;
        if (m < dk) store_row16_sw32(sbt, (uint32_t)m, S);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gb + kOffTmemSlot);

    if (tid == 0) {
        for (int c = 0; c < kSlots - 1 && c < ntk; ++c)
            issue_tma(&tm_q, &tm_k, &tm_v, base + (uint32_t)c * kSlotBytes, bar0 + 8u * c, c, h, b, vb);
    }

    float QS[16], Ui[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) { QS[j] = 0.0f; Ui[j] = 0.0f; }
    bool ok = true;
    int c = 0;
    for (; c < ntk; ++c) {
        const int s = c % kSlots;
        const uint32_t slot = base + (uint32_t)s * kSlotBytes;
        const uint8_t* gslot = gb + (size_t)s * kSlotBytes;
        const int c0 = c * kC;
        const int L = min(kC, p.T - c0);
        const uint32_t ph = (uint32_t)(c & 1);

        if (tid == 0 && c + kSlots - 1 < ntk) {
            const int cn = c + kSlots - 1;
            fence_proxy_async_smem();
            issue_tma(&tm_q, &tm_k, &tm_v, base + (uint32_t)(cn % kSlots) * kSlotBytes,
                      bar0 + 8u * (cn % kSlots), cn, h, b, vb);
        }

        // ---- gates: log a per token, inclusive prefix sum over the chunk, beta ----
        if (warp == 0) {
            const int i0 = 2 * lane, i1 = i0 + 1;
            float la0 = 0.0f, la1 = 0.0f, be0 = 0.0f, be1 = 0.0f;
            if (i0 < L) {
                const int t = c0 + i0;
                la0 = -softplus_f(p.gate[((size_t)b * p.F + t / p.frame_len) * p.H + h]);
                be0 = sigmoid_f(p.beta[((size_t)b * p.T + t) * p.H + h]);
            }
            if (i1 < L) {
                const int t = c0 + i1;
                la1 = -softplus_f(p.gate[((size_t)b * p.F + t / p.frame_len) * p.H + h]);
                be1 = sigmoid_f(p.beta[((size_t)b * p.T + t) * p.H + h]);
            }
            float x = la0 + la1;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x, off);
                if (lane >= off) x += y;
            }
            sc[SC_G + i0] = x - la1;
            sc[SC_G + i1] = x;
            sc[SC_BETA + i0] = be0;
            sc[SC_BETA + i1] = be1;
        }

        ok = mbar_wait(bar0 + 8u * s, (uint32_t)((c / kSlots) & 1), abort_flag, lim, 1);
        if (!__syncthreads_and(ok)) break;
        if (tid == 0) {
            tc_fence_after();
            issue_g1(slot, tmem, nks);
            mma_commit(bar_g1);
        }

        // ---- norms (2 threads per row: K rows 0-63, Q rows 64-127) and decay tables ----
        {
            const int r = tid >> 1, half = tid & 1;
            const uint8_t* row = gslot + (half ? kHalf : 0u) + (r < 64 ? kOffK : kOffQ) + (uint32_t)(r & 63) * 128u;
            float ss = row_sumsq(row);
            ss += __shfl_xor_sync(0xffffffffu, ss, 1);
            if (half == 0) sc[(r < 64 ? SC_RK : SC_RQ) + (r & 63)] = 1.0f / sqrtf(ss + kNormEps);
        }
        {
            const float GL = sc[SC_G + L - 1];
            if (tid < 64) {
                const int i = tid;
                const float Gi = sc[SC_G + i];
                sc[SC_GAM + i] = expf(Gi);
                sc[SC_DL + i] = (i < L) ? expf(GL - Gi) : 0.0f;
                sc[SC_EXR + i] = (i >= 16) ? expf(Gi - sc[SC_G + 16 * (i >> 4) - 1]) : 1.0f;
                if (i == 0) sc[SC_MISC] = expf(GL);
            } else {
                const int idx = tid - 64, bi = 1 + idx / 64, j = idx & 63;
                sc[SC_EXC + 64 * bi + j] = (j < 16 * bi) ? expf(sc[SC_G + 16 * bi - 1] - sc[SC_G + j]) : 0.0f;
            }
        }
        __syncthreads();

        // ---- A (fp32, smem) and P (bf16 SW128) from the raw Gram matrices ----
        ok = mbar_wait(bar_g1, ph, abort_flag, lim, 2);
        if (!__syncthreads_and(ok)) break;
        tc_fence_after();
        {
            const int ch = warp >> 2;                   // column half: 0-31 or 32-63
            float v[32];
            tmem_ld16(tmem_lane(tmem, qtr) + kColG + 32u * ch, *reinterpret_cast<float(*)[16]>(&v[0]));
            tmem_ld16(tmem_lane(tmem, qtr) + kColG + 32u * ch + 16u, *reinterpret_cast<float(*)[16]>(&v[16]));
            tmem_wait_ld();
            const int i = 32 * (qtr & 1) + lane;        // row within the 64-row matrix
            const float Gi = sc[SC_G + i], exr = sc[SC_EXR + i];
            const float* exc = sc + SC_EXC + 64 * (i >> 4);
            if (qtr < 2) {
                const float bi = sc[SC_BETA + i] * sc[SC_RK + i];
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    const int j = 32 * ch + jj;
                    float a = 0.0f;
                    if (j < i) {
                        const float dec = ((j >> 4) == (i >> 4)) ? expf(Gi - sc[SC_G + j]) : exr * exc[j];
                        a = bi * sc[SC_RK + j] * v[jj] * dec;
                    }
                    AX[i * 65 + j] = a;
                }
            } else {
                const float ri = sc[SC_RQ + i];
                float pv[32];
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    const int j = 32 * ch + jj;
                    float pp = 0.0f;
                    if (j <= i) {
                        const float dec = ((j >> 4) == (i >> 4)) ? expf(Gi - sc[SC_G + j]) : exr * exc[j];
                        pp = ri * sc[SC_RK + j] * v[jj] * dec;
                    }
                    pv[jj] = pp;
                }
#pragma unroll
                for (int g = 0; g < 4; ++g) store8_sw128(ptt, (uint32_t)i, (uint32_t)(32 * ch + 8 * g), &pv[8 * g]);
            }
        }
        tc_fence_before();
        __syncthreads();

        // ---- T = (I + A)^{-1} diag(beta), T' = T diag(e^G / |k|) ----
        unit_lower_inverse_64(AX, MS, tid);
        {
            const int i = tid >> 2, j0 = 16 * (tid & 3);
            float tv[16], tpv[16];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
                const int j = j0 + jj;
                const float x = (j <= i) ? XI(AX, i, j) * sc[SC_BETA + j] : 0.0f;
                tv[jj] = x;
                tpv[jj] = x * sc[SC_GAM + j] * sc[SC_RK + j];
            }
            store8_sw128(ptt + 2 * kTile, (uint32_t)i, (uint32_t)j0, &tv[0]);
            store8_sw128(ptt + 2 * kTile, (uint32_t)i, (uint32_t)j0 + 8, &tv[8]);
            store8_sw128(ptt + kTile, (uint32_t)i, (uint32_t)j0, &tpv[0]);
            store8_sw128(ptt + kTile, (uint32_t)i, (uint32_t)j0 + 8, &tpv[8]);
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            issue_wu(slot, ptt, tmem, dk);
            mma_commit(bar_wu);
        }
        ok = mbar_wait(bar_wu, ph, abort_flag, lim, 3);
        if (!__syncthreads_and(ok)) break;
        tc_fence_after();

        // ---- W (rows in lanes 0-63) to smem next to Q; U (lanes 64-127) to registers ----
        if (qtr < 2) {
            const int i = 32 * qtr + lane;
            const int cbeg = 64 * (warp >> 2);
            for (int cb = cbeg; cb < cbeg + 64 && cb < dk; cb += 16) {
                float v[16];
                tmem_ld16(tmem_lane(tmem, qtr) + kColW + (uint32_t)cb, v);
                tmem_wait_ld();
                const uint32_t tile = slot + (cb >= 64 ? kHalf : 0u) + kOffW;
                store8_sw128(tile, (uint32_t)i, (uint32_t)(cb & 63), &v[0]);
                store8_sw128(tile, (uint32_t)i, (uint32_t)(cb & 63) + 8, &v[8]);
            }
        } else if (warp < 4) {
            tmem_ld16(tmem_lane(tmem, qtr) + kColU, Ui);
            tmem_wait_ld();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            issue_m1(slot, sbt, tmem, nks);
            mma_commit(bar_m1);
        }
        ok = mbar_wait(bar_m1, ph, abort_flag, lim, 4);
        if (!__syncthreads_and(ok)) break;
        tc_fence_after();

        // ---- E = U - W S and E' (warps 2,3); Q S kept by warps 0,1 ----
        if (warp < 4) {
            float v[16];
            tmem_ld16(tmem_lane(tmem, qtr) + kColQW, v);
            tmem_wait_ld();
            if (qtr < 2) {
#pragma unroll
                for (int j = 0; j < 16; ++j) QS[j] = v[j];
            } else {
                const int i = 32 * (qtr - 2) + lane;
                const float sci = sc[SC_DL + i] * sc[SC_RK + i];
                float e[16], e2[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    e[j] = Ui[j] - v[j];
                    e2[j] = e[j] * sci;
                }
                store_row16_sw32(ebt, (uint32_t)i, e);
                store_row16_sw32(ept, (uint32_t)i, e2);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            issue_m2(slot, ptt, ebt, ept, tmem);
            mma_commit(bar_m2);
        }
        ok = mbar_wait(bar_m2, ph, abort_flag, lim, 5);
        if (!__syncthreads_and(ok)) break;
        tc_fence_after();

        // ---- S <- e^{G_L} S + K^T E' ; O = diag(e^G / |q|) Q S + P E ----
        if (warp < 4) {
            const int m = tid;
            float v[16];
            tmem_ld16(tmem_lane(tmem, qtr) + kColS, v);
            tmem_wait_ld();
            const float gL = sc[SC_MISC];
#pragma unroll
            for (int j = 0; j < 16; ++j) S[j] = fmaf(gL, S[j], v[j]);
            if (m < dk) store_row16_sw32(sbt, (uint32_t)m, S);
            if (qtr < 2) {
                float pe[16];
                tmem_ld16(tmem_lane(tmem, qtr) + kColPE, pe);
                tmem_wait_ld();
                const int i = m;
                if (i < L && p.out) {
                    const float sq = sc[SC_GAM + i] * sc[SC_RQ + i];
                    uint32_t w[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        w[j] = pack_bf16x2(fmaf(sq, QS[2 * j], pe[2 * j]), fmaf(sq, QS[2 * j + 1], pe[2 * j + 1]));
                    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) +
                                       (((size_t)b * p.T + c0 + i) * p.H + h) * dv + (size_t)vb * kVB;
                    uint4* o4 = reinterpret_cast<uint4*>(o);
                    o4[0] = make_uint4(w[0], w[1], w[2], w[3]);
                    o4[1] = make_uint4(w[4], w[5], w[6], w[7]);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
    }

    if (!ok && tid == 0) {
        // A bounded wait gave up.  Before the shared memory goes away, wait (again
        // bounded) for the tile loads still in flight: chunks c .. c + kSlots - 2
        // were issued and not yet consumed.  MMAs issued before the give-up
        // complete on their own within microseconds.
        for (int cc = c; cc < ntk && cc < c + kSlots - 1; ++cc) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(bar0 + 8u * (cc % kSlots), (uint32_t)((cc / kSlots) & 1)) &&
                   globaltimer_ns() - t0 < lim) {
            }
        }
    }
    if (ok && p.state_out && tid < 128 && tid < dk) {
        float4* so = reinterpret_cast<float4*>(p.state_out + sbase + (size_t)tid * dv);
#pragma unroll
        for (int j = 0; j < 4; ++j) so[j] = make_float4(S[4 * j], S[4 * j + 1], S[4 * j + 2], S[4 * j + 3]);
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
              CUtensorMapSwizzle swz)
{
    PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)inner, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)inner * 2, (cuuint64_t)H * inner * 2,
                             (cuuint64_t)T * H * inner * 2};
    cuuint32_t box[4] = {(cuuint32_t)box_inner, 1, (cuuint32_t)tc::kC, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

uint64_t g_wait_limit_ns = 2000000000ull;   // 2 s

}  // namespace

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
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(tc::gdn_chunk_tc_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)tc::kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    tc::TcArgs args;
    args.p = p;
    args.wait_limit_ns = g_wait_limit_ns;
    dim3 grid(p.dv / tc::kVB, p.B * p.H);
    tc::gdn_chunk_tc_kernel<<<grid, tc::kThreads, tc::kSmemBytes, stream>>>(mq, mk, mv, args);
    return cudaGetLastError();
}

}  // namespace gdn
