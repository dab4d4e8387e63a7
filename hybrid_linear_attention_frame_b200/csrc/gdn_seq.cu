// Sequence-parallel chunked GDN forward for sm_100a: every SM runs the whole
// per-chunk pipeline (prep, state chain, output) of its own stretch of chunks,
// for all d_v state columns, with no communication between CTAs.
//
// Work split.  The B*H chains of N_c = ceil(T/64) chunks form one list of
// units (chain-major).  CTA g takes the contiguous units [U g / G, U (g+1) / G):
// at most the tail of one chain, some whole chains and the head of another.
// A stretch that starts inside a chain needs the state entering its first
// chunk.  The recurrence forgets geometrically: the homogeneous part of one
// token step, a_t (I - b_t k^_t k^_t^T), has spectral norm <= a_t (the
// normalised key has |k^| < 1 and b_t lies in (0, 1)), so the state entering
// chunk c0 depends on the state entering an earlier chunk cw only through a
// map of norm <= prod_{t in [64 cw, 64 c0)} a_t.  The CTA therefore starts the
// recurrence from a zero state at the latest chunk cw < c0 at which that
// product of gates has fallen to 2^-48 or below (outputs before c0 are not
// written), or, when the gates never shrink that far, at the chain's first
// chunk from the caller's initial state (then it runs the exact recurrence).
// With the SANA-WM gates (a ~ 0.12 per token) one chunk of warm-up suffices.
//
// Per chunk of 64 tokens (notation of gdn_common.cuh; M = 128 everywhere by
// stacking two 64-row operands, fp32 accumulators in TMEM):
//   prep  Gram  [K;Q][K;Q]^T            -> norms (diagonal), A and P with the decay
//         T = (I+A)^{-1} diag(beta), T' = T diag(e^G/|k|)  (CUDA cores + mma.sync)
//         U = [Z;T] V, then W = [T';Z] K accumulated  -> EQS = [W ; U]
//   chain -W to shared memory beside Q; lanes 0-63 of EQS cleared  -> EQS = [0 ; U]
//         MMA1  [Q;-W] S_bf16 onto EQS   -> [Q S ; E = U - W S]
//         E' = diag(e^{G_L-G}/|k|) E and E in bf16;  Q S scaled by e^G/|q| in TMEM
//         MMA2  K^T E' onto SACC = e^{G_L} S  -> next state (fp32, in TMEM)
//         PE    [P;X] E onto EQS lanes 0-63   -> O = diag(e^G/|q|) Q S + P E
// The state lives in TMEM in fp32 and only its bf16 copy feeds MMA1.  When the
// state is read back, the next chunk's decay e^{G_L} is applied to it, so that
// MMA2 adds onto the already decayed state.
//
// Warp roles (20 warps): 0 loads q and k tiles (TMA), 1 issues the Gram MMAs,
// 2 issues the chain MMAs, 3 issues the W/U MMAs and loads v tiles, 4-11 prep,
// 12-19 chain and output (two warps per TMEM lane quarter, each on half of the
// d_v columns).  Hand-offs are mbarriers; every wait is bounded and
// gives up with GDN_ERR_TIMEOUT.
#include <cooperative_groups.h>
#include <cudaTypedefs.h>

#include "gdn_common.cuh"
#include "gdn_status.cuh"
#include "gdn_sm100.cuh"

namespace gdn {
namespace seq {

using namespace sm100;
using tc::kC;
using tc::kXS;

constexpr int kThreads = 640;
constexpr int kMaxAtoms = 7;                 // d_k, d_v <= 112 (16-column atoms)
constexpr int kWarpLoadKQ = 0, kWarpGram = 1, kWarpChainMma = 2, kWarpWU = 3;
constexpr int kPrepWarp0 = 4, kChainWarp0 = 12;
constexpr int kPrepThreads = 256;
constexpr uint32_t kBarPrep = 1;             // named barrier of the prep warps (3: the UT inverse's)

// product of gates over a warm-up stretch below which the state entering it is dropped: 2^-48
constexpr float kWarmupLogDecay = 48.0f * 0.693147181f;

// TMEM columns (128 lanes each)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColG = 0;                // Gram [K;Q][K;Q]^T (N 128)
constexpr uint32_t kColEQS = 128;            // 2 x 128: [W;U] -> [0;U] -> [QS;E] -> [O;-]
constexpr uint32_t kColSacc = 384;           // state: d_k lanes x d_v columns

// Shared memory (bytes from a 1024-aligned base).  d-indexed tiles are made of
// 16-column atoms in the 32-byte swizzle (a row of an atom is 32 B, 16-byte
// chunk c of row r at c ^ ((r >> 2) & 1)), so d = 112 wastes no space; the
// 64 x 64 token tiles use the 128-byte swizzle.
constexpr uint32_t kAtomKQW = 6144;          // per d_k atom: K rows | Q rows | W rows (64 each)
constexpr uint32_t kAtQ = 2048, kAtW = 4096;
// e4m3 inputs: the k and q rows of an atom (16 bytes each, 64 rows each, so [K;Q] is
// one 128-row K-major operand without swizzle) land in the atom's W slot, which is
// free until the chunk's W is written; the Gram reads them there and they are
// widened to the bf16 K and Q atoms beside it
constexpr uint32_t kAtK8 = kAtW, kAtQ8 = kAtW + 1024;
constexpr uint32_t kStageSc = kMaxAtoms * kAtomKQW;          // chain scalars of the stage
constexpr uint32_t kStageBytes = kStageSc + 2048;
constexpr uint32_t kOffV = 2 * kStageBytes;                  // v tile, d_v atoms of 64 rows
constexpr uint32_t kAtomV = 2048;
constexpr uint32_t kTile = 8192;                             // 64 x 64 bf16, 128-byte swizzle
constexpr uint32_t kOffP = kOffV + kMaxAtoms * kAtomV;       // P[2]; [P;X] reads the next 8 KB
constexpr uint32_t kOffTp = kOffP + 2 * kTile;               // T' | Z | T
constexpr uint32_t kOffZ = kOffTp + kTile;
constexpr uint32_t kOffT = kOffZ + kTile;
constexpr uint32_t kOffS = kOffT + kTile;                    // S bf16, d_v atoms of 112 rows
constexpr uint32_t kAtomS = 112 * 32;
constexpr uint32_t kOffEp = kOffS + kMaxAtoms * kAtomS;      // E' bf16, d_v atoms of 64 rows
constexpr uint32_t kAtomE = 64 * 32;
constexpr uint32_t kOffE = kOffEp + kMaxAtoms * kAtomE;      // E bf16; then the output rows [64][d_v] bf16
constexpr uint32_t kOffAXI = kOffE + kMaxAtoms * kAtomE;     // fp32 [64][kXS]: A / (I+A)^{-1}
constexpr uint32_t kScFloats = 13 * 64 + 16;
constexpr uint32_t kOffSc = kOffAXI + 64 * kXS * 4;          // prep scalar table
constexpr uint32_t kOffMS = kOffSc + kScFloats * 4;         // the UT inverse's scratch
constexpr int kCS = 36;                                      // row stride (floats) of its level-2 product
constexpr uint32_t kMSBytes = 32 * kCS * 4;
constexpr uint32_t kOffBar = kOffMS + kMSBytes;
enum : uint32_t {
    B_FULL = 0,       // [2] q/k tiles of a stage landed and its gates written
    B_SFREE = 2,      // [2] chain MMAs done with a stage (and with its P)
    B_VFULL = 4,      // v tile landed
    B_VFREE = 5,      // U MMA done with the v tile
    B_G1 = 6,         // Gram done
    B_GFREE = 7,      // Gram read by the prep (A and P warp groups)
    B_TREADY = 8,     // T' and T written
    B_WU = 9,         // [2] U and W MMAs of a stage done
    B_READY = 11,     // [2] the prep done with a stage (P, scalars, T read by the U/W MMAs)
    B_EQFREE = 13,    // [2] output read from EQS
    B_SREADY = 15,    // bf16 state written and SACC decayed
    B_M1 = 16,        // MMA1 done
    B_EREADY = 17,    // E' written
    B_PEGO = 18,      // E written and Q S scaled
    B_M2 = 19,        // MMA2 done
    B_PEDONE = 20,    // P E done
    B_OFREE = 21,     // output staging (the E tile) read by its TMA store
    B_OREADY = 22,    // the four output warps' rows staged
    B_WREADY = 23,    // -W written beside Q and EQS lanes 0-63 cleared (four chain warps)
    B_KQ16 = 24,      // [2] e4m3 inputs: K and Q of a stage widened to bf16
    kNumBars = 26,
};
constexpr uint32_t kOffTmemSlot = kOffBar + kNumBars * 8;
constexpr uint32_t kOffAbort = kOffTmemSlot + 4;
constexpr uint32_t kOffWarm = kOffAbort + 4;                 // warm-up start chunk of the first stretch
constexpr uint32_t kSmemUsed = kOffWarm + 4;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;

// prep scalar table (floats)
enum : uint32_t {
    SC_G = 0,        // cumulative log-gate G_i
    SC_BETA = 64,    // beta_i (0 beyond the chunk)
    SC_RK = 128,     // 1 / |k_i|
    SC_RQ = 192,     // 1 / |q_i|
    SC_GAM = 256,    // e^{G_i}
    SC_DL = 320,     // e^{G_L - G_i} (0 beyond the chunk), times 1/|k_i| once the norms are known
    SC_EXR = 384,    // e^{G_i - G_{16 floor(i/16) - 1}}   (i >= 16)
    SC_EXC = 448,    // [4][64]: e^{G_{16 b - 1} - G_j}   (j < 16 b; row 0 unused)
    SC_BGK = 704,    // beta_j e^{G_j} / |k_j|
    SC_MISC = 768,
};
// per-chunk scalars in a stage (floats).  Written by the q/k loader warp: the
// cumulative log-gate G_i, beta_i (both 0 past the chunk's valid length) and the
// chunk's decay e^{G_L}.  Written by the prep: e^G/|q| and e^{G_L-G}/|k|.
enum : uint32_t { CS_GQ = 0, CS_DL = 64, CS_G = 128, CS_BETA = 192, CS_GL = 256 };

static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kOffP % 1024 == 0 && kOffTp % 1024 == 0 && kStageBytes % 1024 == 0, "SW128 alignment");
static_assert(kOffS % 256 == 0 && kOffEp % 256 == 0 && kOffE % 256 == 0 && kOffV % 256 == 0 &&
                  kAtomKQW % 256 == 0 && kAtomS % 256 == 0,
              "SW32 alignment");
static_assert(kOffAXI % 16 == 0 && kOffSc % 16 == 0 && kOffMS % 16 == 0 && kOffBar % 8 == 0, "alignment");
static_assert(4 * tc::kMS * 32 * 4 <= kMSBytes, "level-1 scratch fits");

constexpr uint32_t kIdGram = idesc_bf16(128, 128, false, false);
// kind::f8f6f4 with e4m3 A and B (format code 0 in both fields), fp32 D, both K-major
constexpr uint32_t kIdGram8 = (1u << 4) | ((uint32_t)(128 >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);

__host__ __device__ constexpr uint32_t bar_count(uint32_t i) {
    return (i == B_SREADY || i == B_PEGO) ? 8u
           : (i == B_EREADY || i == B_OREADY || i == B_WREADY) ? 4u
           : (i == B_FULL || i == B_FULL + 1 || i == B_GFREE) ? 2u
                                                               : 1u;
}

// descriptors: K-major / MN-major 32-byte swizzle (8-row groups 256 B apart), K-major 128-byte swizzle
__device__ __forceinline__ uint64_t dk32(uint32_t a) { return smem_desc(a, 16, 256, kSwizzle32); }
__device__ __forceinline__ uint64_t dmn32(uint32_t a, uint32_t lbo) { return smem_desc(a, lbo, 256, kSwizzle32); }
__device__ __forceinline__ uint64_t dk128(uint32_t a) { return smem_desc(a, 16, 1024, kSwizzle128); }

__device__ __forceinline__ uint32_t tlane(uint32_t tmem, int quarter) {
    return tmem + ((uint32_t)(32 * quarter) << 16);
}

// Shared address of the 8 columns [c8, c8 + 8) of row r in a tile of SW32 atoms `lbo` bytes apart.
__device__ __forceinline__ uint32_t sw32_at(uint32_t tile, uint32_t lbo, uint32_t r, uint32_t c8) {
    return tile + (c8 >> 4) * lbo + sw32_chunk_offset(r, (c8 >> 3) & 1u);
}

// ---------------------------------------------------------------- e4m3 inputs
// Every e4m3 value, subnormals included, is a bf16 value, so the widening is exact.
// Two e4m3 values (the low byte is the first) -> a bf16 pair (the first in the low half).
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t pair) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((unsigned short)(pair & 0xFFFFu)));
    float lo, hi;
    asm("cvt.f32.f16 %0, %1;" : "=f"(lo) : "h"((unsigned short)(h2 & 0xFFFFu)));
    asm("cvt.f32.f16 %0, %1;" : "=f"(hi) : "h"((unsigned short)(h2 >> 16)));
    return pack_bf16x2(lo, hi);
}

// 16 e4m3 values (byte j = element j) -> one 16-column bf16 atom row (32 bytes) at
// `row` of the 32-byte-swizzled atom `atom`
__device__ __forceinline__ void widen16_to_atom_row(uint32_t atom, uint32_t row, const uint4& x) {
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        o[2 * i] = e4m3x2_to_bf16x2(w[i]);
        o[2 * i + 1] = e4m3x2_to_bf16x2(w[i] >> 16);
    }
    st_shared_v4(atom + sw32_chunk_offset(row, 0), o[0], o[1], o[2], o[3]);
    st_shared_v4(atom + sw32_chunk_offset(row, 1), o[4], o[5], o[6], o[7]);
}

// One tcgen05 MMA of kind::f8f6f4 (both operands e4m3, K = 32 per instruction).
__device__ __forceinline__ void mma_e4m3_warp(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p, e;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "elect.sync _|e, 0xffffffff;\n\t"
                 "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
                 :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
                 : "memory");
}

__device__ __forceinline__ uint4 ld_shared_u4(uint32_t addr) {
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(addr));
    return r;
}

__device__ __forceinline__ void st_bf16x8(uint32_t addr, const float* x) {
    st_shared_v4(addr, pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                 pack_bf16x2(x[6], x[7]));
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

// Arrive without release semantics: for hand-offs that order nothing but TMEM
// reads already completed (tcgen05.wait::ld), so that the arrive does not wait
// for this thread's global stores in flight.
__device__ __forceinline__ void mbar_arrive_relaxed(uint32_t bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.relaxed.cta.shared::cta.b64 st, [%0];\n\t}"
                 :: "r"(bar) : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Read 16-column pieces [0, n) of this warp's 32 TMEM lanes starting at `taddr`,
// kBatch pieces per wait (so that the load latency is paid once per batch), and
// hand each piece to f(piece, values).  Warp-collective: n must be warp-uniform.
template <int kBatch = 2, typename F>
__device__ __forceinline__ void tmem_pieces(uint32_t taddr, int n, F&& f) {
#pragma unroll 1
    for (int a0 = 0; a0 < n; a0 += kBatch) {
        float v[kBatch][16];
#pragma unroll
        for (int j = 0; j < kBatch; ++j)
            if (a0 + j < n) tmem_ld16(taddr + 16u * (uint32_t)(a0 + j), v[j]);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < kBatch; ++j)
            if (a0 + j < n) f(a0 + j, v[j]);
    }
}

__device__ __forceinline__ float softplus_fast(float x) { return fmaxf(x, 0.0f) + __logf(1.0f + __expf(-fabsf(x))); }
__device__ __forceinline__ float sigmoid_fast(float x) { return __fdividef(1.0f, 1.0f + __expf(-x)); }
__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }

__device__ __forceinline__ bool group_all(uint32_t id, uint32_t n, bool v) {
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\t"
                 "setp.ne.u32 p, %3, 0;\n\t"
                 "bar.red.and.pred q, %1, %2, p;\n\t"
                 "selp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r) : "r"(id), "r"(n), "r"(v ? 1u : 0u) : "memory");
    return r != 0;
}

struct SeqArgs {
    FwdParams p;
    uint64_t wait_limit_ns;
    float v_scale;    // e4m3 inputs: v = v_scale * decode(v8) (1 for bf16 inputs)
    int G;            // CTAs
    int grid_sync;    // state_in aliases state_out: every read of it precedes every write
};

// ---------------------------------------------------------------- work split

// This CTA's stretch [u0, u1) of units x * nc + c, as pieces of consecutive
// chains ("range order"): piece 0 starts at chunk c0 of chain x0, every later
// piece at chunk 0; the last one ends at chunk cl.
struct Plan {
    int nc, x0, c0, np, cl;
    int head_first;   // the last piece starts at chunk 0 and stops inside its chain: run it first
};

__device__ __forceinline__ Plan make_plan(const SeqArgs& a) {
    Plan P;
    const int nc = (a.p.T + kC - 1) / kC;
    const long long U = (long long)a.p.B * a.p.H * nc;
    const long long u0 = U * blockIdx.x / a.G, u1 = U * (blockIdx.x + 1) / a.G;
    P.nc = nc;
    P.x0 = (int)(u0 / nc);
    P.c0 = (int)(u0 - (long long)P.x0 * nc);
    const int xl = (int)((u1 - 1) / nc);
    P.np = xl - P.x0 + 1;
    P.cl = (int)(u1 - 1 - (long long)xl * nc) + 1;
    P.head_first = (P.np > 1 && P.cl < nc) ? 1 : 0;
    return P;
}

struct Piece {
    int b, h, cw, c0, c1;   // chain (b, h); chunks [cw, c1) run, outputs from c0 on
    bool rd, wr;            // starts from state_in / ends the chain and writes state_out
};

// Pieces in processing order: the head of a chain (whose state another CTA
// writes at the chain's end) first, so that every read of an initial state by
// a CTA that does not also write that chain's final state happens at the start.
__device__ __forceinline__ Piece piece_at(const SeqArgs& a, const Plan& P, int k, int warm0) {
    int j = k;
    if (P.head_first) j = (k == 0) ? P.np - 1 : k - 1;
    Piece pc;
    const int x = P.x0 + j;
    pc.b = x / a.p.H;
    pc.h = x - pc.b * a.p.H;
    pc.c0 = (j == 0) ? P.c0 : 0;
    pc.c1 = (j == P.np - 1) ? P.cl : P.nc;
    pc.cw = (j == 0) ? warm0 : 0;
    pc.rd = pc.cw == 0 && a.p.state_in != nullptr;
    pc.wr = pc.c1 == P.nc && a.p.state_out != nullptr;
    return pc;
}

// Cursor over the chunks this CTA runs, in processing order (n counts them).
struct Cursor {
    const SeqArgs* a;
    const Plan* P;
    int warm0, k, c, n;
    Piece pc;
    __device__ __forceinline__ Cursor(const SeqArgs& a_, const Plan& P_, int warm0_)
        : a(&a_), P(&P_), warm0(warm0_), k(0), c(0), n(0) {
        pc = piece_at(*a, *P, 0, warm0);
        c = pc.cw;
    }
    __device__ __forceinline__ bool valid() const { return k < P->np; }
    __device__ __forceinline__ bool first() const { return c == pc.cw; }
    __device__ __forceinline__ bool last() const { return c == pc.c1 - 1; }
    __device__ __forceinline__ int L() const { return min(kC, a->p.T - c * kC); }
    __device__ __forceinline__ void next() {
        ++n;
        if (++c >= pc.c1) {
            if (++k < P->np) {
                pc = piece_at(*a, *P, k, warm0);
                c = pc.cw;
            }
        }
    }
};

// Sum over the tokens of chunk c of chain (b, h) of -log a_t (whole warp; all lanes get it).
__device__ __forceinline__ float chunk_decay(const FwdParams& p, int b, int h, int c, int lane) {
    float s = 0.0f;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int t = c * kC + lane + 32 * r;
        if (t < p.T && gate_applies(p, t))
            s += softplus_fast(__ldg(p.gate + ((size_t)b * p.F + t / p.frame_len) * p.H + h));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    return s;
}

// ---------------------------------------------------------------- the kernel

// ---------------------------------------------------------------- UT inverse

// Two floats -> an f16 pair (the first in the low half).  f16 keeps 10 mantissa bits, as
// tf32 does, and the inverse's entries lie well inside its range.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// D (16x8) += A (16x16, row) * B (16x8, col), f16 inputs, fp32 accumulate.  Lane l
// holds A rows g, g+8 / columns 2t, 2t+1 (a0, a1) and 2t+8, 2t+9 (a2, a3), B rows 2t, 2t+1
// (b0) and 2t+8, 2t+9 (b1) of column g, D rows g, g+8 / columns 2t, 2t+1; g = l / 4, t = l % 4.
__device__ __forceinline__ void mma_f16_16x8x16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                                uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
                 "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One 16-row x 8-column tile of X (16 rows, K columns) * Y (K rows, 8 columns), as element
// functors, K a multiple of 16: half the tensor-core instructions of the tf32 form.
template <int K, typename XF, typename YF>
__device__ __forceinline__ void tile16x8h(float (&d)[4], XF X, YF Y, int lane) {
    const int g = lane >> 2, t = 2 * (lane & 3);
#pragma unroll
    for (int kk = 0; kk < K; kk += 16)
        mma_f16_16x8x16(d, pack_f16x2(X(g, kk + t), X(g, kk + t + 1)), pack_f16x2(X(g + 8, kk + t), X(g + 8, kk + t + 1)),
                        pack_f16x2(X(g, kk + t + 8), X(g, kk + t + 9)),
                        pack_f16x2(X(g + 8, kk + t + 8), X(g + 8, kk + t + 9)),
                        pack_f16x2(Y(kk + t, g), Y(kk + t + 1, g)), pack_f16x2(Y(kk + t + 8, g), Y(kk + t + 9, g)));
}
// (I + A)^{-1} for the 64 x 64 unit lower-triangular I + A (A strictly lower, stored
// transposed above the diagonal of AXI) into the lower triangle of AXI, by block
// combination: [[X, 0], [C, Y]]^{-1} = [[X^-1, 0], [-Y^-1 C X^-1, Y^-1]].
//
// Diagonal 16 x 16 blocks and the first level (16 -> 32) on the four A warps (128
// threads, `st`): forward substitution in fp32, one column per thread, the column of A
// that a step needs read as four 16-byte vectors (it is a row of the transposed
// storage); then the two 16 x 16 combinations on mma.sync (f16 in, fp32 accumulate), one
// 8-column tile per warp.
__device__ __forceinline__ void inverse_levels01(float* AXI, float* MS, int st) {
    using tc::AAt;
    using tc::XIv;
    const int pw = st >> 5, lane = st & 31, g = lane >> 2, t = lane & 3;
    if (st < 64) {
        const int o = 16 * (st >> 4), j = st & 15;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = (i == j) ? 1.0f : 0.0f;
#pragma unroll
        for (int m = 0; m < 15; ++m) {
            const float* arow = AXI + (o + m) * kXS + o;     // A(o + i, o + m) at column o + i
            float a[16];
#pragma unroll
            for (int q4 = (m + 1) / 4; q4 < 4; ++q4) {
                const float4 v = *reinterpret_cast<const float4*>(arow + 4 * q4);
                a[4 * q4] = v.x; a[4 * q4 + 1] = v.y; a[4 * q4 + 2] = v.z; a[4 * q4 + 3] = v.w;
            }
#pragma unroll
            for (int i = m + 1; i < 16; ++i) x[i] = fmaf(-a[i], x[m], x[i]);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if (i >= j) AXI[(o + i) * kXS + o + j] = x[i];
    }
    named_bar_sync(tc::kBarSolve, 128);
    // blocks (1,0) and (3,2): Y = -D_hi^{-1} (A_{hi,lo} D_lo^{-1}); warp -> (pair, 8 columns)
    float* MSw = MS + pw * 32 * tc::kMS;
    const int pr = pw >> 1, n0 = 8 * (pw & 1);
    const int hi = 16 * (2 * pr + 1), lo = 16 * (2 * pr);
    float m1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    tile16x8h<16>(m1, [&](int r, int k) { return AAt(AXI, hi + r, lo + k); },
                  [&](int k, int n) { return XIv(AXI, lo + k, lo + n0 + n); }, lane);
    MSw[g * tc::kMS + 2 * t] = m1[0];
    MSw[g * tc::kMS + 2 * t + 1] = m1[1];
    MSw[(g + 8) * tc::kMS + 2 * t] = m1[2];
    MSw[(g + 8) * tc::kMS + 2 * t + 1] = m1[3];
    __syncwarp();
    float y[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    tile16x8h<16>(y, [&](int r, int k) { return XIv(AXI, hi + r, hi + k); },
                  [&](int k, int n) { return MSw[k * tc::kMS + n]; }, lane);
    AXI[(hi + g) * kXS + lo + n0 + 2 * t] = -y[0];
    AXI[(hi + g) * kXS + lo + n0 + 2 * t + 1] = -y[1];
    AXI[(hi + g + 8) * kXS + lo + n0 + 2 * t] = -y[2];
    AXI[(hi + g + 8) * kXS + lo + n0 + 2 * t + 1] = -y[3];
}

// The second level (32 -> 64) on all eight prep warps (`w` = 0..7): C = A_21 X_11
// (one 16 x 8 tile each), then X_21 = -X_22 C (X_22 lower triangular, so the upper
// row tile needs only the first 16 columns of it).  The caller's barrier over the
// eight warps precedes it (levels 0-1 done) and follows it.
__device__ __forceinline__ void inverse_level2(float* AXI, float* C, int w, int lane, uint32_t bar_id) {
    using tc::AAt;
    using tc::XIv;
    const int g = lane >> 2, t = lane & 3, mt = w >> 2, c0 = 8 * (w & 3);
    float c[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    tile16x8h<32>(c, [&](int r, int k) { return AAt(AXI, 32 + 16 * mt + r, k); },
                  [&](int k, int n) { return XIv(AXI, k, c0 + n); }, lane);
    C[(16 * mt + g) * kCS + c0 + 2 * t] = c[0];
    C[(16 * mt + g) * kCS + c0 + 2 * t + 1] = c[1];
    C[(16 * mt + g + 8) * kCS + c0 + 2 * t] = c[2];
    C[(16 * mt + g + 8) * kCS + c0 + 2 * t + 1] = c[3];
    named_bar_sync(bar_id, kPrepThreads);
    float y[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (mt == 0)
        tile16x8h<16>(y, [&](int r, int k) { return XIv(AXI, 32 + r, 32 + k); },
                      [&](int k, int n) { return C[k * kCS + c0 + n]; }, lane);
    else
        tile16x8h<32>(y, [&](int r, int k) { return XIv(AXI, 48 + r, 32 + k); },
                      [&](int k, int n) { return C[k * kCS + c0 + n]; }, lane);
    const int r0 = 32 + 16 * mt + g;
    AXI[r0 * kXS + c0 + 2 * t] = -y[0];
    AXI[r0 * kXS + c0 + 2 * t + 1] = -y[1];
    AXI[(r0 + 8) * kXS + c0 + 2 * t] = -y[2];
    AXI[(r0 + 8) * kXS + c0 + 2 * t + 1] = -y[3];
}

// kF8: q, k, v given as e4m3 bytes (v scaled by a.v_scale), widened to bf16 on the way in.
template <bool kF8>
__global__ void __launch_bounds__(kThreads, 1)
gdn_seq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o, const SeqArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gb = smem_raw + (base - raw);
    const FwdParams& p = a.p;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, qtr = warp & 3;
    const int dk = p.dk, dv = p.dv, nak = dk / 16, nav = dv / 16;
    const uint64_t lim = a.wait_limit_ns;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gb + kOffAbort);
    auto bar = [&](uint32_t i) { return base + kOffBar + 8u * i; };
    const Plan P = make_plan(a);

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
        if (a.p.out) tma_prefetch_desc(&tm_o);
    }
    if (warp == kWarpWU) {
        // warm-up start of the first piece (see the file comment)
        int cw = P.c0;
        if (P.c0 > 0) {
            const int b = P.x0 / p.H, h = P.x0 - (P.x0 / p.H) * p.H;
            float acc = 0.0f;
            cw = 0;
            for (int c = P.c0 - 1; c >= 0; --c) {
                acc += chunk_decay(p, b, h, c, lane);
                if (acc >= kWarmupLogDecay) {
                    cw = c;
                    break;
                }
            }
        }
        if (lane == 0) *reinterpret_cast<volatile int*>(gb + kOffWarm) = cw;
    }
    // the zero tile Z
    for (int i = tid; i < (int)(kTile / 16); i += kThreads) st_shared_v4(base + kOffZ + 16u * i, 0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gb + kOffTmemSlot);
    const int warm0 = *reinterpret_cast<volatile int*>(gb + kOffWarm);

    // Chain warps: S tile and SACC for the first chunk of a piece (state_in or zero),
    // then SREADY.  SACC holds e^{G_L} S for the chunk about to run.
    // chain warp: TMEM lane quarter q, and the half [a_lo, a_lo + na) of the d_v atoms
    const int cq = warp & 3, chf = (warp - kChainWarp0) >> 2;
    const int c_alo = chf ? (nav + 1) / 2 : 0, c_na = chf ? nav - (nav + 1) / 2 : (nav + 1) / 2;
    auto chain_init = [&](const Piece& pc) {
        const int q = cq, row = 32 * q + lane;
        // (read from the gate logits directly: the first piece is set up before the loaders start)
        const float gl = __expf(-chunk_decay(p, pc.b, pc.h, pc.cw, lane));
        const float* si = (pc.rd && row < dk)
                              ? p.state_in + (((size_t)pc.b * p.H + pc.h) * dk + row) * (size_t)dv
                              : nullptr;
        for (int at = c_alo; at < c_alo + c_na; ++at) {
            float v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = 0.0f;
            if (si) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float4 f = *reinterpret_cast<const float4*>(si + 16 * at + 4 * j);
                    v[4 * j] = f.x; v[4 * j + 1] = f.y; v[4 * j + 2] = f.z; v[4 * j + 3] = f.w;
                }
            }
            if (row < dk) {
                st_bf16x8(sw32_at(base + kOffS, kAtomS, row, 16 * at), v);
                st_bf16x8(sw32_at(base + kOffS, kAtomS, row, 16 * at + 8), v + 8);
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] *= gl;
            tmem_st16(tlane(tmem + kColSacc, q) + 16u * at, v);
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_SREADY));
    };
    if (warp >= kChainWarp0 && P.np > 0) chain_init(piece_at(a, P, 0, warm0));
    if (a.grid_sync) {
        // in-place state: every CTA has read the initial states it needs before any final state is written
        tc_fence_before();
        cooperative_groups::this_grid().sync();
        tc_fence_after();
    }

    if (warp == kWarpLoadKQ) {
        // ======================= q and k tiles (TMA) =======================
        bool ok = true;
        int issued = 0;
        for (Cursor cu(a, P, warm0); cu.valid(); cu.next()) {
            const int n = cu.n, s = n & 1;
            // the chunk's gate and beta logits: the only global loads of a chunk besides the
            // tiles, made by this warp (so that no compute warp waits for them at a barrier)
            // and issued before the wait for the stage, which hides their latency
            const int L = cu.L(), i0 = 2 * lane, t0 = cu.c * kC + i0;
            float g0 = 0.f, g1 = 0.f, r0 = 0.f, r1 = 0.f;
            if (i0 < L) {
                g0 = __ldg(p.gate + ((size_t)cu.pc.b * p.F + t0 / p.frame_len) * p.H + cu.pc.h);
                r0 = __ldg(p.beta + ((size_t)cu.pc.b * p.T + t0) * p.H + cu.pc.h);
            }
            if (i0 + 1 < L) {
                g1 = __ldg(p.gate + ((size_t)cu.pc.b * p.F + (t0 + 1) / p.frame_len) * p.H + cu.pc.h);
                r1 = __ldg(p.beta + ((size_t)cu.pc.b * p.T + t0 + 1) * p.H + cu.pc.h);
            }
            if (n >= 2) {
                ok = __all_sync(0xffffffffu, mbar_wait(bar(B_SFREE + s), (uint32_t)(((n - 2) >> 1) & 1),
                                                       abort_flag, lim, 21));
                if (!ok) break;
            }
            const uint32_t st = base + (uint32_t)s * kStageBytes;
            if (lane == 0) {
                if constexpr (kF8) {
                    const uint32_t fb = bar(B_FULL + s);
                    mbar_arrive_expect_tx(fb, (uint32_t)nak * 2u * 1024u);
                    for (int at = 0; at < nak; ++at) {
                        tma_load_4d(st + (uint32_t)at * kAtomKQW + kAtK8, &tm_k, fb, 16 * at, cu.pc.h, cu.c * kC,
                                    cu.pc.b);
                        tma_load_4d(st + (uint32_t)at * kAtomKQW + kAtQ8, &tm_q, fb, 16 * at, cu.pc.h, cu.c * kC,
                                    cu.pc.b);
                    }
                } else {
                    const uint32_t fb = bar(B_FULL + s);
                    mbar_arrive_expect_tx(fb, (uint32_t)nak * 2u * 2048u);
                    for (int at = 0; at < nak; ++at) {
                        tma_load_4d(st + (uint32_t)at * kAtomKQW, &tm_k, fb, 16 * at, cu.pc.h, cu.c * kC, cu.pc.b);
                        tma_load_4d(st + (uint32_t)at * kAtomKQW + kAtQ, &tm_q, fb, 16 * at, cu.pc.h, cu.c * kC,
                                    cu.pc.b);
                    }
                }
            }
            // G (warp scan of the log-gates), beta and e^{G_L} into the stage
            {
                float* cs = reinterpret_cast<float*>(gb + (uint32_t)s * kStageBytes + kStageSc);
                const float la0 = (i0 < L && gate_applies(p, t0)) ? -softplus_fast(g0) : 0.0f;
                const float la1 = (i0 + 1 < L && gate_applies(p, t0 + 1)) ? -softplus_fast(g1) : 0.0f;
                float x = la0 + la1;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, x, off);
                    if (lane >= off) x += y;
                }
                cs[CS_G + i0] = x - la1;
                cs[CS_G + i0 + 1] = x;
                cs[CS_BETA + i0] = (i0 < L) ? sigmoid_fast(r0) : 0.0f;
                cs[CS_BETA + i0 + 1] = (i0 + 1 < L) ? sigmoid_fast(r1) : 0.0f;
                if (lane == 31) cs[CS_GL] = __expf(x);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_FULL + s));
            issued = n + 1;
        }
        if (!ok && lane == 0) {
            for (int m = max(0, issued - 2); m < issued; ++m)
                drain_wait(bar(B_FULL + (m & 1)), (uint32_t)((m >> 1) & 1));
        }
        __syncwarp();
    } else if (warp == kWarpGram) {
        // ======================= Gram MMAs =======================
        bool ok = true;
        int issued = 0;
        for (Cursor cu(a, P, warm0); cu.valid(); cu.next()) {
            const int n = cu.n, s = n & 1;
            ok = mbar_wait(bar(B_FULL + s), (uint32_t)((n >> 1) & 1), abort_flag, lim, 22);
            if (ok && n > 0) ok = mbar_wait(bar(B_GFREE), (uint32_t)((n - 1) & 1), abort_flag, lim, 23);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            const uint32_t st = base + (uint32_t)s * kStageBytes;
            if constexpr (kF8) {
                // [K;Q] in e4m3 straight from the staging: core matrices of 8 rows x 16 bytes,
                // the next 16 bytes of K one atom further on (an odd last atom pairs with the
                // zero tile), the next 8 rows 128 bytes on
#pragma unroll 1
                for (int at = 0; at < nak; at += 2) {
                    const uint32_t a0 = st + (uint32_t)at * kAtomKQW + kAtK8;
                    const uint32_t lbo = (at + 1 < nak) ? kAtomKQW : base + kOffZ - a0;
                    const uint64_t d = smem_desc(a0, lbo, 128, 0);
                    mma_e4m3_warp(tmem + kColG, d, d, kIdGram8, at > 0);
                }
            } else {
#pragma unroll 1
                for (int at = 0; at < nak; ++at) {
                    const uint64_t d = dk32(st + (uint32_t)at * kAtomKQW);
                    mma_bf16_warp(tmem + kColG, d, d, kIdGram, at > 0);
                }
            }
            mma_commit_warp(bar(B_G1));
            issued = n + 1;
            if constexpr (kF8) {
                // while the Gram reads the e4m3 rows, widen them into the stage's bf16 K and Q
                // atoms for the W, MMA1 and MMA2 products (lanes take consecutive rows of one atom)
#pragma unroll 4
                for (int id = lane; id < 2 * kC * nak; id += 32) {
                    const int isq = id >= kC * nak, rem = isq ? id - kC * nak : id;
                    const uint32_t atom = st + (uint32_t)(rem >> 6) * kAtomKQW, r = (uint32_t)(rem & 63);
                    const uint4 x = ld_shared_u4(atom + (isq ? kAtQ8 : kAtK8) + 16u * r);
                    widen16_to_atom_row(atom + (isq ? kAtQ : 0u), r, x);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_KQ16 + s));
            }
        }
        if (!ok && issued > 0 && lane == 0) drain_wait(bar(B_G1), (uint32_t)((issued - 1) & 1));
        __syncwarp();
    } else if (warp == kWarpWU) {
        // ======================= U and W MMAs; v tiles =======================
        const uint32_t idu = idesc_bf16(128, dv, false, true), idw = idesc_bf16(128, dk, false, true);
        bool ok = true;
        int v_issued = 0, wu_issued = 0;
        Cursor cv(a, P, warm0);
        auto load_v = [&](const Cursor& c) {
            if constexpr (kF8) {
                // e4m3 rows straight from global memory (lanes take consecutive 16-byte
                // pieces of a token's row), widened into the v atoms; 7 loads in flight per lane
                const uint8_t* src = static_cast<const uint8_t*>(p.v) +
                                     (((size_t)c.pc.b * p.T + (size_t)c.c * kC) * p.H + c.pc.h) * (size_t)dv;
                const size_t rs = (size_t)p.H * dv;
                const int L = c.L(), npc = kC * nav;
                for (int b0 = 0; b0 < npc; b0 += 32 * 7) {
                    uint4 x[7];
#pragma unroll
                    for (int j = 0; j < 7; ++j) {
                        const int id = b0 + 32 * j + lane, r = id / nav, at = id - r * nav;
                        x[j] = (id < npc && r < L)
                                   ? __ldg(reinterpret_cast<const uint4*>(src + (size_t)r * rs + 16 * at))
                                   : make_uint4(0u, 0u, 0u, 0u);
                    }
#pragma unroll
                    for (int j = 0; j < 7; ++j) {
                        const int id = b0 + 32 * j + lane, r = id / nav, at = id - r * nav;
                        if (id < npc) widen16_to_atom_row(base + kOffV + (uint32_t)at * kAtomV, (uint32_t)r, x[j]);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_VFULL));
            } else {
                if (lane == 0) {
                    mbar_arrive_expect_tx(bar(B_VFULL), (uint32_t)nav * 2048u);
                    for (int at = 0; at < nav; ++at)
                        tma_load_4d(base + kOffV + (uint32_t)at * kAtomV, &tm_v, bar(B_VFULL), 16 * at, c.pc.h,
                                    c.c * kC, c.pc.b);
                }
                __syncwarp();
            }
        };
        if (cv.valid()) {
            load_v(cv);
            v_issued = 1;
        }
        for (Cursor cu(a, P, warm0); cu.valid(); cu.next()) {
            const int n = cu.n, s = n & 1;
            const uint32_t eqs = tmem + kColEQS + 128u * (uint32_t)s;
            ok = mbar_wait(bar(B_TREADY), (uint32_t)(n & 1), abort_flag, lim, 24);
            ok = ok && mbar_wait(bar(B_VFULL), (uint32_t)(n & 1), abort_flag, lim, 25);
            if constexpr (kF8) ok = ok && mbar_wait(bar(B_KQ16 + s), (uint32_t)((n >> 1) & 1), abort_flag, lim, 27);
            if (ok && n >= 2) ok = mbar_wait(bar(B_EQFREE + s), (uint32_t)(((n - 2) >> 1) & 1), abort_flag, lim, 26);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            const uint32_t st = base + (uint32_t)s * kStageBytes;
#pragma unroll
            for (int ks = 0; ks < kC / 16; ++ks)   // [Z;T] V -> [0 ; U]
                mma_bf16_warp(eqs, dk128(base + kOffZ + 32u * ks), dmn32(base + kOffV + 512u * ks, kAtomV), idu,
                              ks > 0);
#pragma unroll
            for (int ks = 0; ks < kC / 16; ++ks)   // + [T';Z] K -> [W ; U]
                mma_bf16_warp(eqs, dk128(base + kOffTp + 32u * ks), dmn32(st + 512u * ks, kAtomKQW), idw, 1u);
            mma_commit_warp(bar(B_WU + (uint32_t)s));
            mma_commit_warp(bar(B_VFREE));
            wu_issued = n + 1;
            cv.next();
            if (cv.valid()) {
                // the next chunk's v tile, once this U MMA has read the buffer
                ok = __all_sync(0xffffffffu, mbar_wait(bar(B_VFREE), (uint32_t)(n & 1), abort_flag, lim, 27));
                if (!ok) break;
                load_v(cv);
                v_issued = n + 2;
            }
        }
        if (!ok && lane == 0) {
            if (wu_issued > 0)
                drain_wait(bar(B_WU + (uint32_t)((wu_issued - 1) & 1)), (uint32_t)(((wu_issued - 1) >> 1) & 1));
            if (v_issued > wu_issued) drain_wait(bar(B_VFULL), (uint32_t)((v_issued - 1) & 1));
        }
        __syncwarp();
    } else if (warp == kWarpChainMma) {
        // ======================= chain MMAs =======================
        const uint32_t id1 = idesc_bf16(128, dv, false, true), id2 = idesc_bf16(128, dv, true, true);
        bool ok = true;
        int pending = -1, pend_n = 0;
        for (Cursor cu(a, P, warm0); cu.valid(); cu.next()) {
            const int n = cu.n, s = n & 1;
            const uint32_t eqs = tmem + kColEQS + 128u * (uint32_t)s;
            const uint32_t st = base + (uint32_t)s * kStageBytes;
            ok = mbar_wait(bar(B_READY + s), (uint32_t)((n >> 1) & 1), abort_flag, lim, 31);
            ok = ok && mbar_wait(bar(B_WREADY), (uint32_t)(n & 1), abort_flag, lim, 35);
            ok = ok && mbar_wait(bar(B_SREADY), (uint32_t)(n & 1), abort_flag, lim, 32);
            if constexpr (kF8) ok = ok && mbar_wait(bar(B_KQ16 + s), (uint32_t)((n >> 1) & 1), abort_flag, lim, 36);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
#pragma unroll 1
            for (int at = 0; at < nak; ++at)       // [Q;-W] S onto [0 ; U]
                mma_bf16_warp(eqs, dk32(st + (uint32_t)at * kAtomKQW + kAtQ), dmn32(base + kOffS + 512u * at, kAtomS),
                              id1, 1u);
            mma_commit_warp(bar(B_M1));
            pending = B_M1; pend_n = n;
            ok = __all_sync(0xffffffffu, mbar_wait(bar(B_EREADY), (uint32_t)(n & 1), abort_flag, lim, 33));
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < kC / 16; ++ks)    // K^T E' onto e^{G_L} S
                mma_bf16_warp(tmem + kColSacc, dmn32(st + 512u * ks, kAtomKQW), dmn32(base + kOffEp + 512u * ks, kAtomE),
                              id2, 1u);
            mma_commit_warp(bar(B_M2));
            pending = B_M2;
            ok = __all_sync(0xffffffffu, mbar_wait(bar(B_PEGO), (uint32_t)(n & 1), abort_flag, lim, 34));
            if (!ok) break;
            tc_fence_after();
            const uint32_t pa = base + kOffP + kTile * (uint32_t)s;
#pragma unroll
            for (int ks = 0; ks < kC / 16; ++ks)    // [P;X] E onto [(e^G/|q|) Q S ; -]
                mma_bf16_warp(eqs, dk128(pa + 32u * ks), dmn32(base + kOffE + 512u * ks, kAtomE), id1, 1u);
            mma_commit_warp(bar(B_PEDONE));
            mma_commit_warp(bar(B_SFREE + s));
            pending = B_PEDONE;
        }
        if (!ok && pending >= 0 && lane == 0) drain_wait(bar((uint32_t)pending), (uint32_t)(pend_n & 1));
        __syncwarp();
    } else if (warp < kChainWarp0) {
        // ======================= prep (warps 4-11) =======================
        const int pt = tid - kPrepWarp0 * 32, pw = warp - kPrepWarp0;
        float* sc = reinterpret_cast<float*>(gb + kOffSc);
        float* AXI = reinterpret_cast<float*>(gb + kOffAXI);
        float* MSf = reinterpret_cast<float*>(gb + kOffMS);
        const uint32_t tg = tmem + kColG;
        bool ok = true;
        // Per chunk: front (the stage's gates, norms), then A and P from the Gram, the
        // UT inverse and T, T'.
        auto front = [&](const Cursor& cu) -> bool {
            const int n = cu.n, s = n & 1, L = cu.L();
            float* cs = reinterpret_cast<float*>(gb + (uint32_t)s * kStageBytes + kStageSc);
            // ---- the stage's gates written, the Gram done ----
            ok = mbar_wait(bar(B_FULL + s), (uint32_t)((n >> 1) & 1), abort_flag, lim, 43);
            ok = ok && mbar_wait(bar(B_G1), (uint32_t)(n & 1), abort_flag, lim, 41);
            if (!group_all(kBarPrep, kPrepThreads, ok)) return false;
            // ---- G and beta from the stage; the decay tables ----
            {
                const float GL = cs[CS_G + 63];
                const int idx = pt;
                if (idx < 64) {
                    const int i = idx;
                    const float Gi = cs[CS_G + i];
                    sc[SC_G + i] = Gi;
                    sc[SC_BETA + i] = cs[CS_BETA + i];
                    sc[SC_GAM + i] = __expf(Gi);
                    sc[SC_DL + i] = (i < L) ? __expf(GL - Gi) : 0.0f;
                    sc[SC_EXR + i] = (i >= 16) ? __expf(Gi - cs[CS_G + 16 * (i >> 4) - 1]) : 1.0f;
                } else {
                    const int bi = 1 + (idx - 64) / 64, j = idx & 63;
                    sc[SC_EXC + 64 * bi + j] = (j < 16 * bi) ? __expf(cs[CS_G + 16 * bi - 1] - cs[CS_G + j]) : 0.0f;
                }
            }
            named_bar_sync(kBarPrep, kPrepThreads);
            tc_fence_after();
            // ---- norms from the Gram diagonal: |k_i|^2 (lanes 0-63), |q_i|^2 (lanes 64-127) ----
            if (pw < 4) {
                float v[32];
                tmem_ld16(tlane(tg, qtr) + 32u * qtr, *reinterpret_cast<float(*)[16]>(&v[0]));
                tmem_ld16(tlane(tg, qtr) + 32u * qtr + 16u, *reinterpret_cast<float(*)[16]>(&v[16]));
                tmem_wait_ld();
                float d = 0.0f;
#pragma unroll
                for (int j = 0; j < 32; ++j) d = (j == lane) ? v[j] : d;
                const float r = rsqrtf(d + kNormEps);
                const int i = 32 * (qtr & 1) + lane;
                if (qtr < 2) {
                    sc[SC_RK + i] = r;
                    const float dl = sc[SC_DL + i] * r;
                    sc[SC_DL + i] = dl;
                    cs[CS_DL + i] = dl;
                    sc[SC_BGK + i] = sc[SC_BETA + i] * sc[SC_GAM + i] * r;
                } else {
                    sc[SC_RQ + i] = r;
                    cs[CS_GQ + i] = r * sc[SC_GAM + i];
                }
            }
            named_bar_sync(kBarPrep, kPrepThreads);
            return true;
        };
        // A (fp32, transposed above the diagonal of AXI; TMEM lanes 0-63) and P (bf16
        // tile P[s]; lanes 64-127) from the Gram, row i = 32 (qtr & 1) + lane of each warp,
        // one 16-column block j0 = 16 bj at a time.  For a row in a later 16-row block
        // than the columns (bi > bj) the decay factors through the block boundary,
        // e^{G_i - G_j} = e^{G_i - G_{16 bi - 1}} e^{G_{16 bi - 1} - G_j} (both factors <= 1);
        // inside the diagonal block it is one exponential; above it A has nothing and P is 0.
        // Each warp takes two column blocks, chosen so that the costly diagonal blocks of
        // a row group fall on different warps.
        auto gram_epilogue = [&](int s) {
            const uint32_t ptile = base + kOffP + kTile * (uint32_t)s;
            const bool isA = qtr < 2;
            const int i = 32 * (qtr & 1) + lane, bi = i >> 4, ii = i & 15, ch = pw >> 2;
            const int bmax = 2 * (qtr & 1) + 1;       // the warp's rows lie in blocks bmax - 1, bmax
            const float Gi = sc[SC_G + i];
            const float R = isA ? sc[SC_BETA + i] * sc[SC_RK + i] : sc[SC_RQ + i];
            const float RX = R * sc[SC_EXR + i];
#pragma unroll 1
            for (int pc = 0; pc < 2; ++pc) {
                const int bj = pc == 0 ? ch : ((qtr & 1) ? 3 - ch : 2 + ch);
                const int j0 = 16 * bj;
                float v[16];
                if (bj > bmax) {
                    // above the diagonal for every row of the warp
                    if (!isA) {
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj) v[jj] = 0.0f;
                        st_bf16x8(ptile + sw128_offset((uint32_t)i, (uint32_t)j0), &v[0]);
                        st_bf16x8(ptile + sw128_offset((uint32_t)i, (uint32_t)j0 + 8u), &v[8]);
                    }
                    continue;
                }
                tmem_ld16(tlane(tg, qtr) + (uint32_t)j0, v);
                tmem_wait_ld();
                if (bi > bj) {
                    const float* rk = sc + SC_RK + j0;
                    const float* ex = sc + SC_EXC + 64 * bi + j0;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const float4 r4 = ld4(rk + 4 * q4), e4 = ld4(ex + 4 * q4);
                        v[4 * q4] *= RX * (r4.x * e4.x);
                        v[4 * q4 + 1] *= RX * (r4.y * e4.y);
                        v[4 * q4 + 2] *= RX * (r4.z * e4.z);
                        v[4 * q4 + 3] *= RX * (r4.w * e4.w);
                    }
                } else if (bi == bj) {
                    const float* rk = sc + SC_RK + j0;
                    const float* gj = sc + SC_G + j0;
                    const int lim_j = isA ? ii : ii + 1;       // A: j < i, P: j <= i
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const float4 r4 = ld4(rk + 4 * q4), g4 = ld4(gj + 4 * q4);
                        const float rr[4] = {r4.x, r4.y, r4.z, r4.w}, gg[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int jj = 4 * q4 + e;
                            const float x = v[jj] * (R * rr[e]) * __expf(Gi - gg[e]);
                            v[jj] = (jj < lim_j) ? x : 0.0f;
                        }
                    }
                } else {
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) v[jj] = 0.0f;
                }
                if (isA) {
                    if (bi >= bj) {
                        float* dst = AXI + j0 * kXS + i;
                        const int n_st = (bi > bj) ? 16 : ii;
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj)
                            if (jj < n_st) dst[jj * kXS] = v[jj];
                    }
                } else {
                    st_bf16x8(ptile + sw128_offset((uint32_t)i, (uint32_t)j0), &v[0]);
                    st_bf16x8(ptile + sw128_offset((uint32_t)i, (uint32_t)j0 + 8u), &v[8]);
                }
            }
        };
        // The warps on TMEM lanes 0-63 (qtr 0, 1) form A and then invert I + A; the
        // warps on lanes 64-127 form P meanwhile (P is needed only by the chain).  Each
        // group releases its half of the Gram accumulator as soon as it has read it.
        // T and T' are written once the previous chunk's U/W MMAs have read them; the
        // chain warps then take -W out of TMEM, so the prep goes straight on to the
        // next chunk.
        auto inverse_t = [&](int n) -> bool {
            const int s = n & 1;
            gram_epilogue(s);
            tc_fence_before();
            named_bar_sync(kBarPrep, kPrepThreads);      // A and P complete: the Gram is free
            if (pt == 0) {
                mbar_arrive(bar(B_GFREE));
                mbar_arrive(bar(B_GFREE));
            }
            // the diagonal blocks and the first level on the P warps (their schedulers carry
            // less of the chain's work than the A warps')
            if (qtr >= 2) inverse_levels01(AXI, MSf, 32 * ((pw & 1) | ((pw >> 2) << 1)) + lane);
            named_bar_sync(kBarPrep, kPrepThreads);
            inverse_level2(AXI, MSf, pw, lane, kBarPrep);
            bool okw = true;
            if (n > 0) okw = mbar_wait(bar(B_WU + (uint32_t)((n - 1) & 1)), (uint32_t)(((n - 1) >> 1) & 1), abort_flag, lim, 42);
            if (!group_all(kBarPrep, kPrepThreads, okw)) return false;
            // ---- T = (I+A)^{-1} diag(beta), T' = T diag(beta e^G / |k|): bf16 tiles ----
            {
                const int i = pt >> 2, jb = 16 * (pt & 3);
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
                        if constexpr (kF8) tv[4 * q4 + e] *= a.v_scale;     // U = (v_scale T) V8
                        tpv[4 * q4 + e] = x * fs[e];
                    }
                }
                st_bf16x8(base + kOffT + sw128_offset((uint32_t)i, (uint32_t)jb), &tv[0]);
                st_bf16x8(base + kOffT + sw128_offset((uint32_t)i, (uint32_t)jb + 8u), &tv[8]);
                st_bf16x8(base + kOffTp + sw128_offset((uint32_t)i, (uint32_t)jb), &tpv[0]);
                st_bf16x8(base + kOffTp + sw128_offset((uint32_t)i, (uint32_t)jb + 8u), &tpv[8]);
            }
            fence_proxy_async_smem();
            named_bar_sync(kBarPrep, kPrepThreads);
            if (pt == 0) {
                mbar_arrive(bar(B_TREADY));
                mbar_arrive(bar(B_READY + s));
            }
            return true;
        };
        for (Cursor cu(a, P, warm0); ok && cu.valid(); cu.next()) {
            ok = front(cu);
            if (!ok) break;
            ok = inverse_t(cu.n);
        }
    } else {
        // ======================= chain and output (warps 12-19) =======================
        const int q = cq, row = 32 * q + lane;
        const uint32_t a_lo = (uint32_t)c_alo;
        const int na = c_na;
        // the half of the d_k atoms of W this warp takes out of TMEM (lane quarters 0, 1)
        const int k_lo = chf ? (nak + 1) / 2 : 0, k_na = chf ? nak - (nak + 1) / 2 : (nak + 1) / 2;
        bool ok = true;
        for (Cursor cu(a, P, warm0); cu.valid(); cu.next()) {
            const int n = cu.n, s = n & 1, L = cu.L();
            const Piece& pc = cu.pc;
            const bool last = cu.last(), emit = cu.c >= pc.c0;
            if (cu.first() && n > 0) chain_init(pc);
            const uint32_t eqs = tlane(tmem + kColEQS + 128u * (uint32_t)s, q);
            const float* cs = reinterpret_cast<const float*>(gb + (uint32_t)s * kStageBytes + kStageSc);
            ok = mbar_wait(bar(B_READY + s), (uint32_t)((n >> 1) & 1), abort_flag, lim, 51);
            if (q < 2) {
                // U and W done: -W (TMEM lanes 0-63 of EQS) beside Q in the stage, and
                // those lanes cleared, so that MMA1 adds Q S onto zero
                ok = ok && mbar_wait(bar(B_WU + (uint32_t)s), (uint32_t)((n >> 1) & 1), abort_flag, lim, 56);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
                const uint32_t stg = base + (uint32_t)s * kStageBytes;
                tmem_pieces<1>(eqs + 16u * (uint32_t)k_lo, k_na, [&](int j0, float (&v)[16]) {
                    const uint32_t at = (uint32_t)(k_lo + j0);
#pragma unroll
                    for (int j = 0; j < 16; ++j) v[j] = -v[j];
                    const uint32_t wa = stg + at * kAtomKQW + kAtW;
                    st_bf16x8(wa + sw32_chunk_offset((uint32_t)row, 0), &v[0]);
                    st_bf16x8(wa + sw32_chunk_offset((uint32_t)row, 1), &v[8]);
#pragma unroll
                    for (int j = 0; j < 16; ++j) v[j] = 0.0f;
                    tmem_st16(eqs + 16u * at, v);
                });
                tmem_wait_st();
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_WREADY));
            }
            ok = ok && mbar_wait(bar(B_M1), (uint32_t)(n & 1), abort_flag, lim, 52);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            if (q >= 2) {
                // E (TMEM lanes 64-127): E' = diag(e^{G_L-G}/|k|) E for MMA2, then E for P E
                const int i = row - 64;
                const float dl = cs[CS_DL + i];
                tmem_pieces<1>(eqs + 16u * a_lo, na, [&](int j0, float (&v)[16]) {
                    const uint32_t at = a_lo + (uint32_t)j0;
                    float e[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) e[j] = v[j] * dl;
                    st_bf16x8(sw32_at(base + kOffEp, kAtomE, (uint32_t)i, 16u * at), &e[0]);
                    st_bf16x8(sw32_at(base + kOffEp, kAtomE, (uint32_t)i, 16u * at + 8u), &e[8]);
                });
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_EREADY));
                // (the E tile doubles as the previous chunk's output staging: wait for its store)
                if (n > 0 && !__all_sync(0xffffffffu, mbar_wait(bar(B_OFREE), (uint32_t)((n - 1) & 1), abort_flag,
                                                                 lim, 57))) {
                    ok = false;
                    break;
                }
                tmem_pieces<1>(eqs + 16u * a_lo, na, [&](int j0, float (&v)[16]) {
                    const uint32_t at = a_lo + (uint32_t)j0;
                    st_bf16x8(sw32_at(base + kOffE, kAtomE, (uint32_t)i, 16u * at), &v[0]);
                    st_bf16x8(sw32_at(base + kOffE, kAtomE, (uint32_t)i, 16u * at + 8u), &v[8]);
                });
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_PEGO));
            } else {
                // Q S (TMEM lanes 0-63) scaled in place by e^G/|q|; P E is added onto it
                const float gq = cs[CS_GQ + row];
                tmem_pieces<1>(eqs + 16u * a_lo, na, [&](int j0, float (&v)[16]) {
                    const uint32_t at = a_lo + (uint32_t)j0;
#pragma unroll
                    for (int j = 0; j < 16; ++j) v[j] *= gq;
                    tmem_st16(eqs + 16u * at, v);
                });
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_PEGO));
            }
            // ---- next state: bf16 copy for MMA1, decayed fp32 back into SACC ----
            // decay of the next chunk of this piece (its stage's gates), applied to the state
            // when it is read back
            float gl_next = 1.0f;
            if (!last) {
                ok = mbar_wait(bar(B_FULL + ((n + 1) & 1)), (uint32_t)(((n + 1) >> 1) & 1), abort_flag, lim, 55);
                gl_next = reinterpret_cast<const float*>(gb + (uint32_t)((n + 1) & 1) * kStageBytes + kStageSc)[CS_GL];
            }
            ok = ok && mbar_wait(bar(B_M2), (uint32_t)(n & 1), abort_flag, lim, 53);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            {
                const uint32_t sa = tlane(tmem + kColSacc, q);
                float* so = (last && pc.wr && row < dk)
                                ? p.state_out + (((size_t)pc.b * p.H + pc.h) * dk + row) * (size_t)dv
                                : nullptr;
                tmem_pieces<1>(sa + 16u * a_lo, na, [&](int j0, float (&v)[16]) {
                    const uint32_t at = a_lo + (uint32_t)j0;
                    if (so) {
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            *reinterpret_cast<float4*>(so + 16 * at + 4 * j) =
                                make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                    }
                    if (!last) {
                        if (row < dk) {
                            st_bf16x8(sw32_at(base + kOffS, kAtomS, (uint32_t)row, 16u * at), &v[0]);
                            st_bf16x8(sw32_at(base + kOffS, kAtomS, (uint32_t)row, 16u * at + 8u), &v[8]);
                        }
#pragma unroll
                        for (int j = 0; j < 16; ++j) v[j] *= gl_next;
                        tmem_st16(sa + 16u * at, v);
                    }
                });
                if (!last) {
                    tmem_wait_st();
                    fence_proxy_async_smem();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(B_SREADY));
                }
            }
            // ---- output rows (TMEM lanes 0-63): bf16 rows into the E tile, one TMA store ----
            if (q < 2) {
                ok = __all_sync(0xffffffffu, mbar_wait(bar(B_PEDONE), (uint32_t)(n & 1), abort_flag, lim, 54));
                if (!ok) break;
                tc_fence_after();
                const bool store = emit && p.out != nullptr;
                if (store) {
                    const uint32_t orow = base + kOffE + (uint32_t)row * (uint32_t)(2 * dv);
                    tmem_pieces<1>(eqs + 16u * a_lo, na, [&](int j0, float (&v)[16]) {
                        const uint32_t at = a_lo + (uint32_t)j0;
                        st_shared_v4(orow + 32u * at, pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                     pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
                        st_shared_v4(orow + 32u * at + 16u, pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]),
                                     pack_bf16x2(v[12], v[13]), pack_bf16x2(v[14], v[15]));
                    });
                    fence_proxy_async_smem();
                }
                // (an mbarrier rather than a named barrier: a warp that gave up on a wait
                // never arrives, and the storing warp's wait for it is bounded)
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_OREADY));
                if (warp == kChainWarp0) {
                    ok = __all_sync(0xffffffffu, mbar_wait(bar(B_OREADY), (uint32_t)(n & 1), abort_flag, lim, 58));
                    if (!ok) break;
                    if (lane == 0) {
                        if (store) {
                            tma_store_4d(&tm_o, base + kOffE, 0, pc.h, cu.c * kC, pc.b);
                            bulk_commit_group();
                            bulk_wait_group_read0();
                        }
                        mbar_arrive_relaxed(bar(B_OFREE));
                        mbar_arrive_relaxed(bar(B_EQFREE + s));
                    }
                    __syncwarp();
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

}  // namespace seq

// ---------------------------------------------------------------- host side

bool seq_supported(int dk, int dv, int chunk_len)
{
    return chunk_len == seq::kC && dk % 16 == 0 && dv % 16 == 0 && dk >= 16 && dv >= 16 &&
           dk <= 16 * seq::kMaxAtoms && dv <= 16 * seq::kMaxAtoms;
}

namespace {
// e4m3 rows of one head: 4-D view {d, H, T, B} in bytes, 16-byte x 64-token boxes
bool make_map_u8(CUtensorMap* map, const void* base, int inner, int H, int T, int B)
{
    PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)inner, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)inner, (cuuint64_t)H * inner, (cuuint64_t)T * H * inner};
    cuuint32_t box[4] = {16, 1, (cuuint32_t)seq::kC, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace

cudaError_t launch_seq(const FwdParams& p, cudaStream_t stream, bool fp8, float v_scale)
{
    if (!seq_supported(p.dk, p.dv, seq::kC) || p.T < 1) return cudaErrorInvalidValue;
    void (*kern)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, seq::SeqArgs) =
        fp8 ? seq::gdn_seq_kernel<true> : seq::gdn_seq_kernel<false>;
    // the dynamic shared memory limit is a per-device setting of the current context: set it on
    // every call (cheap), so that every device and a context re-created after a reset get it
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)seq::kSmemBytes);
    int dev = 0, sms = 0;
    if (e == cudaSuccess) e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const long long nc = (p.T + seq::kC - 1) / seq::kC;
    const long long U = (long long)p.B * p.H * nc;
    CUtensorMap mq, mk, mv;
    // 32-byte boxes, each read by exactly one CTA: no L2 promotion, so that a box
    // fetches its own sectors only and not the neighbouring heads' bytes
    const CUtensorMapL2promotion promo = CU_TENSOR_MAP_L2_PROMOTION_NONE;
    if (fp8) {
        // e4m3 q and k through TMA (16-byte boxes); v is read by the v loader warp directly
        if (!make_map_u8(&mq, p.q, p.dk, p.H, p.T, p.B) || !make_map_u8(&mk, p.k, p.dk, p.H, p.T, p.B))
            return cudaErrorInvalidValue;
        mv = mq;
    } else if (!make_map(&mq, p.q, p.dk, p.H, p.T, p.B, 16, CU_TENSOR_MAP_SWIZZLE_32B, promo) ||
               !make_map(&mk, p.k, p.dk, p.H, p.T, p.B, 16, CU_TENSOR_MAP_SWIZZLE_32B, promo) ||
               !make_map(&mv, p.v, p.dv, p.H, p.T, p.B, 16, CU_TENSOR_MAP_SWIZZLE_32B, promo)) {
        return cudaErrorInvalidValue;
    }
    CUtensorMap mo;
    // output: whole 64-token rows of d_v per store (no swizzle); the q map stands in when there is no output
    if (p.out ? !make_map(&mo, p.out, p.dv, p.H, p.T, p.B, p.dv, CU_TENSOR_MAP_SWIZZLE_NONE, promo) : (mo = mq, false))
        return cudaErrorInvalidValue;
    seq::SeqArgs args;
    args.p = p;
    args.wait_limit_ns = g_wait_limit_ns;
    args.v_scale = fp8 ? v_scale : 1.0f;
    args.G = (int)(U < sms ? U : sms);
    args.grid_sync = (p.state_in != nullptr && (const void*)p.state_in == (const void*)p.state_out) ? 1 : 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)args.G);
    cfg.blockDim = dim3(seq::kThreads);
    cfg.dynamicSmemBytes = seq::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = args.grid_sync ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, mo, args);
}

}  // namespace gdn
