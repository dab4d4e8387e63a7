// Bidirectional GDN: the forward scan plus the same rule run from the last token
// to the first, both from a zero state, every token keeping its own frame's gate
// (the dense checkpoint's "bidirectional" GDN, sglang cookbook SANA-WM page,
// dense-bidirectional section; the pages do not give the form, this is the
// reading the library implements).
//
// The backward scan reuses the forward kernels unchanged: a copy kernel writes the
// inputs in reverse token order (the gate logit of each token's own frame expanded
// to one value per token, so that the copy runs with frame_len 1), the forward
// kernel runs on the copy, and a combine kernel adds its output, mirrored back, to
// the forward scan's output.  Both helper kernels stream rows of 16-byte vectors
// and are bound by HBM bandwidth.
#include "gdn_common.cuh"

namespace gdn {

// Byte offsets of the sub-buffers of the bidirectional workspace.
struct BidirLayout {
    size_t q, k, v, g, b, o, ring, total;
};

namespace bidir {

constexpr int kThreads = 256;
constexpr int kRowsPerBlock = 4;      // (b, t) rows per block: ~50 KB of traffic per block at d 112

// Row t of batch b of the copies takes token T-1-t.  q and k rows hold nqk16, v rows
// nv16 16-byte vectors; beta has one value per head, the gate one per head and frame.
__global__ void __launch_bounds__(kThreads)
reverse_inputs_kernel(const uint4* __restrict__ q, const uint4* __restrict__ k, const uint4* __restrict__ v,
                      const float* __restrict__ gate, const float* __restrict__ beta,
                      uint4* __restrict__ qr, uint4* __restrict__ kr, uint4* __restrict__ vr,
                      float* __restrict__ gr, float* __restrict__ br,
                      int T, int H, int F, int frame_len, int nqk16, int nv16, long long rows)
{
    for (int rr = 0; rr < kRowsPerBlock; ++rr) {
        const long long row = (long long)blockIdx.x * kRowsPerBlock + rr;
        if (row >= rows) return;
        const long long b = row / T;
        const int t = (int)(row - b * T);
        const int ts = T - 1 - t;
        const long long src = b * T + ts;
        const uint4* qs = q + src * nqk16;
        const uint4* ks = k + src * nqk16;
        const uint4* vs = v + src * nv16;
        uint4* qd = qr + row * nqk16;
        uint4* kd = kr + row * nqk16;
        uint4* vd = vr + row * nv16;
        const int n = nqk16 > nv16 ? nqk16 : nv16;
        for (int i = threadIdx.x; i < n; i += kThreads) {
            uint4 a = make_uint4(0, 0, 0, 0), c = a, e = a;
            if (i < nqk16) { a = __ldg(qs + i); c = __ldg(ks + i); }
            if (i < nv16) e = __ldg(vs + i);
            if (i < nqk16) { qd[i] = a; kd[i] = c; }
            if (i < nv16) vd[i] = e;
        }
        const float* gs = gate + (b * F + ts / frame_len) * H;
        for (int h = threadIdx.x; h < H; h += kThreads) {
            br[row * H + h] = __ldg(beta + src * H + h);
            gr[row * H + h] = __ldg(gs + h);
        }
    }
}

__device__ __forceinline__ uint4 add_vec(uint4 x, uint4 y, const __nv_bfloat16*)
{
    uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w}, r[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xs[j]));
        const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ys[j]));
        const __nv_bfloat162 s = __floats2bfloat162_rn(a.x + c.x, a.y + c.y);
        r[j] = *reinterpret_cast<const uint32_t*>(&s);
    }
    return make_uint4(r[0], r[1], r[2], r[3]);
}

__device__ __forceinline__ uint4 add_vec(uint4 x, uint4 y, const float*)
{
    return make_uint4(__float_as_uint(__uint_as_float(x.x) + __uint_as_float(y.x)),
                      __float_as_uint(__uint_as_float(x.y) + __uint_as_float(y.y)),
                      __float_as_uint(__uint_as_float(x.z) + __uint_as_float(y.z)),
                      __float_as_uint(__uint_as_float(x.w) + __uint_as_float(y.w)));
}

// out[b, t] += back[b, T-1-t] (rows of n16 16-byte vectors, added in fp32).
template <typename IOT>
__global__ void __launch_bounds__(kThreads)
combine_kernel(uint4* __restrict__ out, const uint4* __restrict__ back, int T, int n16, long long rows)
{
    for (int rr = 0; rr < kRowsPerBlock; ++rr) {
        const long long row = (long long)blockIdx.x * kRowsPerBlock + rr;
        if (row >= rows) return;
        const long long b = row / T;
        const int t = (int)(row - b * T);
        const long long src = b * T + (T - 1 - t);
        uint4* o = out + row * n16;
        const uint4* s = back + src * n16;
        for (int i = threadIdx.x; i < n16; i += kThreads)
            o[i] = add_vec(o[i], __ldg(s + i), static_cast<const IOT*>(nullptr));
    }
}

}  // namespace bidir

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Sub-buffers of the bidirectional workspace, in this order: reversed q, k, v,
// per-token gate logits, beta logits, the backward scan's output, then the ring
// workspace of the forward kernels (0 bytes where they take none).
BidirLayout bidir_layout(int B, int H, int T, int dk, int dv, size_t elem, size_t ring_bytes)
{
    const size_t th = (size_t)B * T * H;
    BidirLayout L;
    L.q = 0;
    L.k = L.q + align256(th * dk * elem);
    L.v = L.k + align256(th * dk * elem);
    L.g = L.v + align256(th * dv * elem);
    L.b = L.g + align256(th * sizeof(float));
    L.o = L.b + align256(th * sizeof(float));
    L.ring = L.o + align256(th * dv * elem);
    L.total = L.ring + ring_bytes;
    return L;
}

cudaError_t launch_reverse_inputs(const FwdParams& p, size_t elem, uint8_t* ws, const BidirLayout& L,
                                  cudaStream_t stream)
{
    const long long rows = (long long)p.B * p.T;
    if (rows == 0) return cudaSuccess;
    const int nqk16 = (int)((size_t)p.H * p.dk * elem / 16), nv16 = (int)((size_t)p.H * p.dv * elem / 16);
    const unsigned blocks = (unsigned)((rows + bidir::kRowsPerBlock - 1) / bidir::kRowsPerBlock);
    bidir::reverse_inputs_kernel<<<blocks, bidir::kThreads, 0, stream>>>(
        static_cast<const uint4*>(p.q), static_cast<const uint4*>(p.k), static_cast<const uint4*>(p.v),
        p.gate, p.beta, reinterpret_cast<uint4*>(ws + L.q), reinterpret_cast<uint4*>(ws + L.k),
        reinterpret_cast<uint4*>(ws + L.v), reinterpret_cast<float*>(ws + L.g),
        reinterpret_cast<float*>(ws + L.b), p.T, p.H, p.F, p.frame_len, nqk16, nv16, rows);
    return cudaGetLastError();
}

template <typename IOT>
cudaError_t launch_combine(const FwdParams& p, const uint8_t* ws, const BidirLayout& L, cudaStream_t stream)
{
    const long long rows = (long long)p.B * p.T;
    if (rows == 0) return cudaSuccess;
    const int n16 = (int)((size_t)p.H * p.dv * sizeof(IOT) / 16);
    const unsigned blocks = (unsigned)((rows + bidir::kRowsPerBlock - 1) / bidir::kRowsPerBlock);
    bidir::combine_kernel<IOT><<<blocks, bidir::kThreads, 0, stream>>>(
        static_cast<uint4*>(p.out), reinterpret_cast<const uint4*>(ws + L.o), p.T, n16, rows);
    return cudaGetLastError();
}

template cudaError_t launch_combine<__nv_bfloat16>(const FwdParams&, const uint8_t*, const BidirLayout&,
                                                   cudaStream_t);
template cudaError_t launch_combine<float>(const FwdParams&, const uint8_t*, const BidirLayout&, cudaStream_t);

// The backward scan's parameters: the reversed copies, one gate per token, no state.
FwdParams reversed_params(const FwdParams& p, uint8_t* ws, const BidirLayout& L)
{
    FwdParams r = p;
    r.q = ws + L.q;
    r.k = ws + L.k;
    r.v = ws + L.v;
    r.gate = reinterpret_cast<const float*>(ws + L.g);
    r.beta = reinterpret_cast<const float*>(ws + L.b);
    r.out = ws + L.o;
    r.state_in = nullptr;
    r.state_out = nullptr;
    r.frame_len = 1;
    r.F = p.T;
    r.gate_mode = 0;
    return r;
}

}  // namespace gdn
