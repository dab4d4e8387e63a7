// Shared device helpers and launch parameters of the GDN kernels.
//
// The recurrence (fixed in writing for SANA-WM's "frame-wise Gated DeltaNet",
// sglang cookbook SANA-WM page, section 1 architecture table):
//   S_t = a_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,  o_t = S_t^T q_t,
//   q, k L2-normalised (eps 1e-6), beta_t = sigmoid(logit), a = exp(-softplus(logit))
//   per latent frame.
// Chunked (WY / UT) evaluation for a chunk of L tokens with cumulative
// log-gates G_i = sum_{s <= i} log a_s and start state S_0:
//   A_ij = beta_i (k_i . k_j) e^{G_i - G_j} for j < i        (strictly lower)
//   T    = (I + A)^{-1} diag(beta)                           (forward substitution)
//   W    = T diag(e^G) K,  U = T V,  E = U - W S_0
//   O    = diag(e^G) Q S_0 + (Q K^T o e^{G_i - G_j}[j <= i]) E
//   S_L  = e^{G_L} S_0 + (diag(e^{G_L - G}) K)^T E
// Decay factors are always exp of a non-positive number (G is non-increasing),
// so nothing overflows however strong the gates are.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {

constexpr float kNormEps = 1e-6f;

struct FwdParams {
    const void* q;
    const void* k;
    const void* v;
    const float* gate;       // [B, F, H]
    const float* beta;       // [B, T, H]
    const float* state_in;   // [B, H, dk, dv] or null
    float* state_out;        // [B, H, dk, dv] or null
    void* out;               // [B, T, H, dv] or null
    int B, H, T, dk, dv, frame_len, F;
    int gate_mode;           // 0: a frame's gate at each of its tokens; 1: once, at its first token
};

// Does token t of the call take its frame's gate?  Frame f covers tokens
// f*frame_len .. (f+1)*frame_len - 1; gate_mode 0 applies a_f at all of them,
// gate_mode 1 only at the first (the two readings of "frame-wise").
__device__ __forceinline__ bool gate_applies(const FwdParams& p, int t) {
    return p.gate_mode == 0 || (t % p.frame_len) == 0;
}

__device__ __forceinline__ float softplus_f(float x) {
    // log(1 + e^x) = max(x, 0) + log1p(e^{-|x|})
    return fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x)));
}

__device__ __forceinline__ float sigmoid_f(float x) {
    return 1.0f / (1.0f + expf(-x));
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

}  // namespace gdn
