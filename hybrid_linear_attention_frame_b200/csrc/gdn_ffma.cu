// Chunked GDN forward on CUDA cores (all float32 FFMA).
//
// This is the float32 reference mode (gdn_forward_f32 / gdn_state_step_f32)
// and the bf16 path for sizes the tensor-core kernel does not cover.  One CTA
// owns one (batch, head) chain and a 32-column slice of d_v: columns of the
// state evolve independently (S_new[:, j] depends only on S[:, j] and V[:, j]),
// so slices need no communication.  The state-independent work of a chunk
// (norms, gates, the decayed Gram matrices, the UT inverse, W) is repeated by
// every slice of a head; that is the price of a kernel without cross-CTA
// traffic, acceptable for a reference path.
//
// Shared memory per CTA (floats, sk = d_k + 1, C = chunk length):
//   Q, K, W [C][sk]   V, U/E [C][33]   S [d_k][33]   A, T, P [C][C+1]
//   G, beta, e^G, e^{G_L - G} [C]
#include "gdn_common.cuh"

namespace gdn {

constexpr int kFfmaThreads = 256;
constexpr int kFfmaVB = 32;          // state columns per CTA
constexpr int kFfmaVS = kFfmaVB + 1; // padded row stride of the column-slice tiles

__host__ __device__ inline size_t ffma_smem_floats(int C, int dk) {
    const int sk = dk + 1;
    return (size_t)3 * C * sk + (size_t)2 * C * kFfmaVS + (size_t)dk * kFfmaVS +
           (size_t)3 * C * (C + 1) + (size_t)4 * C;
}

template <typename IOT, int C>
__global__ void __launch_bounds__(kFfmaThreads)
chunk_ffma_kernel(FwdParams p)
{
    extern __shared__ float smem[];
    const int dk = p.dk, dv = p.dv, sk = dk + 1;
    float* Qs = smem;
    float* Ks = Qs + C * sk;
    float* Ws = Ks + C * sk;
    float* Vs = Ws + C * sk;
    float* Us = Vs + C * kFfmaVS;          // U, then E in place
    float* Ss = Us + C * kFfmaVS;          // state slice [dk][33]
    float* As = Ss + dk * kFfmaVS;
    float* Ts = As + C * (C + 1);
    float* Ps = Ts + C * (C + 1);
    float* Gs = Ps + C * (C + 1);          // cumulative log-gate
    float* Bs = Gs + C;                    // beta
    float* Eg = Bs + C;                    // e^{G_i}
    float* Dl = Eg + C;                    // e^{G_last - G_i}

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.y;
    const int b = bh / p.H, h = bh % p.H;
    const int col0 = blockIdx.x * kFfmaVB;
    const IOT* q = static_cast<const IOT*>(p.q);
    const IOT* k = static_cast<const IOT*>(p.k);
    const IOT* v = static_cast<const IOT*>(p.v);
    IOT* out = static_cast<IOT*>(p.out);
    const size_t sbase = ((size_t)b * p.H + h) * (size_t)dk * dv;

    // initial state slice
    for (int idx = tid; idx < dk * kFfmaVB; idx += kFfmaThreads) {
        const int m = idx / kFfmaVB, j = idx % kFfmaVB, col = col0 + j;
        float s = 0.0f;
        if (p.state_in && col < dv) s = p.state_in[sbase + (size_t)m * dv + col];
        Ss[m * kFfmaVS + j] = s;
    }

    for (int c0 = 0; c0 < p.T; c0 += C) {
        const int L = min(C, p.T - c0);
        __syncthreads();   // previous chunk fully consumed

        // ---- load q, k, v slice, gates and betas (rows >= L are zero) ----
        for (int idx = tid; idx < C * dk; idx += kFfmaThreads) {
            const int i = idx / dk, m = idx % dk;
            float qv = 0.0f, kv = 0.0f;
            if (i < L) {
                const size_t off = (((size_t)b * p.T + c0 + i) * p.H + h) * dk + m;
                qv = to_f32(q[off]);
                kv = to_f32(k[off]);
            }
            Qs[i * sk + m] = qv;
            Ks[i * sk + m] = kv;
        }
        for (int idx = tid; idx < C * kFfmaVB; idx += kFfmaThreads) {
            const int i = idx / kFfmaVB, j = idx % kFfmaVB, col = col0 + j;
            float vv = 0.0f;
            if (i < L && col < dv) vv = to_f32(v[(((size_t)b * p.T + c0 + i) * p.H + h) * dv + col]);
            Vs[i * kFfmaVS + j] = vv;
        }
        if (tid < C) {
            float la = 0.0f, bt = 0.0f;
            if (tid < L) {
                const int t = c0 + tid;
                const float g = p.gate[((size_t)b * p.F + t / p.frame_len) * p.H + h];
                la = gate_applies(p, t) ? -softplus_f(g) : 0.0f;
                bt = sigmoid_f(p.beta[((size_t)b * p.T + t) * p.H + h]);
            }
            Gs[tid] = la;   // log-gate for now; prefix sum below
            Bs[tid] = bt;
        }
        __syncthreads();

        // ---- L2 norms (one warp per row) and the cumulative log-gate ----
        for (int i = warp; i < C; i += kFfmaThreads / 32) {
            float sq = 0.0f, skk = 0.0f;
            for (int m = lane; m < dk; m += 32) {
                const float a = Qs[i * sk + m], c = Ks[i * sk + m];
                sq += a * a;
                skk += c * c;
            }
            for (int o = 16; o > 0; o >>= 1) {
                sq += __shfl_xor_sync(0xffffffffu, sq, o);
                skk += __shfl_xor_sync(0xffffffffu, skk, o);
            }
            const float rq = 1.0f / sqrtf(sq + kNormEps), rk = 1.0f / sqrtf(skk + kNormEps);
            for (int m = lane; m < dk; m += 32) {
                Qs[i * sk + m] *= rq;
                Ks[i * sk + m] *= rk;
            }
        }
        if (tid == 0) {
            float acc = 0.0f;
            for (int i = 0; i < C; ++i) { acc += Gs[i]; Gs[i] = acc; }
        }
        __syncthreads();
        if (tid < C) {
            Eg[tid] = expf(Gs[tid]);
            Dl[tid] = expf(Gs[L - 1] - Gs[tid]);   // rows >= L have k = 0, value unused
        }

        // ---- decayed Gram matrices A (strict) and P (inclusive) ----
        for (int idx = tid; idx < C * C; idx += kFfmaThreads) {
            const int i = idx / C, j = idx % C;
            float a = 0.0f, pp = 0.0f;
            if (j <= i) {
                float dkk = 0.0f, dqk = 0.0f;
                for (int m = 0; m < dk; ++m) {
                    const float kj = Ks[j * sk + m];
                    dkk += Ks[i * sk + m] * kj;
                    dqk += Qs[i * sk + m] * kj;
                }
                const float dec = expf(Gs[i] - Gs[j]);
                if (j < i) a = Bs[i] * dkk * dec;
                pp = dqk * dec;
            }
            As[i * (C + 1) + j] = a;
            Ps[i * (C + 1) + j] = pp;
        }
        __syncthreads();

        // ---- T = (I + A)^{-1} diag(beta): forward substitution, one column per thread ----
        if (tid < C) {
            const int j = tid;
            for (int i = 0; i < C; ++i) {
                float val;
                if (i < j) {
                    val = 0.0f;
                } else if (i == j) {
                    val = Bs[j];
                } else {
                    float s = 0.0f;
                    for (int m = j; m < i; ++m) s += As[i * (C + 1) + m] * Ts[m * (C + 1) + j];
                    val = -s;
                }
                Ts[i * (C + 1) + j] = val;
            }
        }
        __syncthreads();

        // ---- W = T diag(e^G) K and U = T V ----
        for (int idx = tid; idx < C * dk; idx += kFfmaThreads) {
            const int i = idx / dk, m = idx % dk;
            float s = 0.0f;
            for (int j = 0; j <= i; ++j) s += Ts[i * (C + 1) + j] * Eg[j] * Ks[j * sk + m];
            Ws[i * sk + m] = s;
        }
        for (int idx = tid; idx < C * kFfmaVB; idx += kFfmaThreads) {
            const int i = idx / kFfmaVB, jv = idx % kFfmaVB;
            float s = 0.0f;
            for (int j = 0; j <= i; ++j) s += Ts[i * (C + 1) + j] * Vs[j * kFfmaVS + jv];
            Us[i * kFfmaVS + jv] = s;
        }
        __syncthreads();

        // ---- E = U - W S ----
        for (int idx = tid; idx < C * kFfmaVB; idx += kFfmaThreads) {
            const int i = idx / kFfmaVB, jv = idx % kFfmaVB;
            float x = 0.0f;
            for (int m = 0; m < dk; ++m) x += Ws[i * sk + m] * Ss[m * kFfmaVS + jv];
            Us[i * kFfmaVS + jv] -= x;
        }
        __syncthreads();

        // ---- O = diag(e^G) Q S + P E ----
        if (out) {
            for (int idx = tid; idx < C * kFfmaVB; idx += kFfmaThreads) {
                const int i = idx / kFfmaVB, jv = idx % kFfmaVB, col = col0 + jv;
                if (i >= L || col >= dv) continue;
                float x = 0.0f, y = 0.0f;
                for (int m = 0; m < dk; ++m) x += Qs[i * sk + m] * Ss[m * kFfmaVS + jv];
                for (int j = 0; j <= i; ++j) y += Ps[i * (C + 1) + j] * Us[j * kFfmaVS + jv];
                out[(((size_t)b * p.T + c0 + i) * p.H + h) * dv + col] = from_f32<IOT>(Eg[i] * x + y);
            }
        }
        __syncthreads();

        // ---- S <- e^{G_L} S + (diag(e^{G_L - G}) K)^T E ----
        const float gl = Eg[L - 1];
        for (int idx = tid; idx < dk * kFfmaVB; idx += kFfmaThreads) {
            const int m = idx / kFfmaVB, jv = idx % kFfmaVB;
            float s = 0.0f;
            for (int j = 0; j < L; ++j) s += Dl[j] * Ks[j * sk + m] * Us[j * kFfmaVS + jv];
            Ss[m * kFfmaVS + jv] = gl * Ss[m * kFfmaVS + jv] + s;
        }
    }
    __syncthreads();

    if (p.state_out) {
        for (int idx = tid; idx < dk * kFfmaVB; idx += kFfmaThreads) {
            const int m = idx / kFfmaVB, j = idx % kFfmaVB, col = col0 + j;
            if (col < dv) p.state_out[sbase + (size_t)m * dv + col] = Ss[m * kFfmaVS + j];
        }
    }
}

template <typename IOT, int C>
static cudaError_t launch_ffma_c(const FwdParams& p, cudaStream_t stream)
{
    const size_t smem = ffma_smem_floats(C, p.dk) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(chunk_ffma_kernel<IOT, C>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((p.dv + kFfmaVB - 1) / kFfmaVB, p.B * p.H);
    chunk_ffma_kernel<IOT, C><<<grid, kFfmaThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

template <typename IOT>
cudaError_t launch_ffma(const FwdParams& p, int chunk_len, cudaStream_t stream)
{
    switch (chunk_len) {
        case 16: return launch_ffma_c<IOT, 16>(p, stream);
        case 32: return launch_ffma_c<IOT, 32>(p, stream);
        case 64: return launch_ffma_c<IOT, 64>(p, stream);
        default: return cudaErrorInvalidValue;
    }
}

template cudaError_t launch_ffma<float>(const FwdParams&, int, cudaStream_t);
template cudaError_t launch_ffma<__nv_bfloat16>(const FwdParams&, int, cudaStream_t);

}  // namespace gdn
