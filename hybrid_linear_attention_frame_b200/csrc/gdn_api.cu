// C ABI of the GDN forward library: argument checks, dispatch, host-buffer entry.
//
// Every entry point validates its arguments before touching CUDA and returns a
// gdn_status; nothing is enqueued on an error.  The library never allocates.
#include <stdint.h>
#include <string.h>

#include "gdn.h"
#include "gdn_common.cuh"

namespace gdn {
template <typename IOT>
cudaError_t launch_ffma(const FwdParams& p, int chunk_len, cudaStream_t stream);
bool tc_supported(int dk, int dv, int chunk_len);
cudaError_t launch_tc(const FwdParams& p, int chunk_len, cudaStream_t stream);
bool ring_supported(int dk, int dv, int chunk_len);
cudaError_t ring_groups(int BH, int dv, int* groups);
size_t ring_workspace_bytes(int G, int dv);
cudaError_t launch_ring(const FwdParams& p, void* ws, size_t ws_bytes, cudaStream_t stream);
bool seq_supported(int dk, int dv, int chunk_len);
cudaError_t launch_seq(const FwdParams& p, cudaStream_t stream, bool fp8, float v_scale);
cudaError_t static_scratch(void** ptr, size_t* bytes);
int read_and_clear_device_status(cudaStream_t stream);
void set_wait_limit_ns(uint64_t ns);
}  // namespace gdn

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb)
{
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t x0 = reinterpret_cast<uintptr_t>(a), y0 = reinterpret_cast<uintptr_t>(b);
    return x0 < y0 + nb && y0 < x0 + na;
}

bool supported_dim(int d) { return d >= 16 && d <= 128 && d % 16 == 0; }

// Checks shared by every entry point.  `need_out` is false for the
// state-only streaming step.
int validate(const void* q, const void* k, const void* v, const float* gate,
             const float* beta, const float* state_in, const float* state_out,
             const void* out, bool need_out, size_t elem,
             int B, int H, int T, int dk, int dv, int frame_len, int chunk_len,
             gdn::FwdParams* p)
{
    if (B < 1 || H < 1 || T < 0 || frame_len < 1) return GDN_ERR_INVALID_ARG;
    if (dk < 1 || dv < 1 || chunk_len < 1) return GDN_ERR_INVALID_ARG;
    if (!supported_dim(dk) || !supported_dim(dv)) return GDN_ERR_UNSUPPORTED;
    if (chunk_len != 16 && chunk_len != 32 && chunk_len != 64) return GDN_ERR_UNSUPPORTED;
    if ((int64_t)B * H > INT32_MAX) return GDN_ERR_UNSUPPORTED;
    if (!q || !k || !v || !gate || !beta) return GDN_ERR_INVALID_ARG;
    if (need_out && !out) return GDN_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16)) return GDN_ERR_INVALID_ARG;
    if (out && !aligned(out, 16)) return GDN_ERR_INVALID_ARG;
    if ((state_in && !aligned(state_in, 16)) || (state_out && !aligned(state_out, 16)))
        return GDN_ERR_INVALID_ARG;
    if (!aligned(gate, 4) || !aligned(beta, 4)) return GDN_ERR_INVALID_ARG;

    const int64_t F = ((int64_t)T + frame_len - 1) / frame_len;
    const size_t nq = (size_t)B * T * H * dk * elem;
    const size_t nv = (size_t)B * T * H * dv * elem;
    const size_t ng = (size_t)B * F * H * sizeof(float);
    const size_t nb = (size_t)B * T * H * sizeof(float);
    const size_t ns = (size_t)B * H * dk * dv * sizeof(float);
    if (out) {
        if (overlaps(out, nv, q, nq) || overlaps(out, nv, k, nq) || overlaps(out, nv, v, nv) ||
            overlaps(out, nv, gate, ng) || overlaps(out, nv, beta, nb) ||
            overlaps(out, nv, state_in, ns) || overlaps(out, nv, state_out, ns))
            return GDN_ERR_INVALID_ARG;
    }
    if (state_out && state_out != state_in) {
        if (overlaps(state_out, ns, q, nq) || overlaps(state_out, ns, k, nq) ||
            overlaps(state_out, ns, v, nv) || overlaps(state_out, ns, gate, ng) ||
            overlaps(state_out, ns, beta, nb) || overlaps(state_out, ns, state_in, ns))
            return GDN_ERR_INVALID_ARG;
    }
    p->q = q; p->k = k; p->v = v; p->gate = gate; p->beta = beta;
    p->state_in = state_in; p->state_out = const_cast<float*>(state_out);
    p->out = const_cast<void*>(out);
    p->B = B; p->H = H; p->T = T; p->dk = dk; p->dv = dv; p->frame_len = frame_len;
    p->F = (int)F;
    p->gate_mode = 0;
    return GDN_OK;
}

int to_status(cudaError_t e) { return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA; }

int run_bf16(const gdn::FwdParams& p, int chunk_len, cudaStream_t stream)
{
    if (p.T > 0 && gdn::seq_supported(p.dk, p.dv, chunk_len)) return to_status(gdn::launch_seq(p, stream, false, 1.0f));
    if (gdn::tc_supported(p.dk, p.dv, chunk_len)) return to_status(gdn::launch_tc(p, chunk_len, stream));
    return to_status(gdn::launch_ffma<__nv_bfloat16>(p, chunk_len, stream));
}

// Does this call take the shared-prep ring kernel (and so need a workspace)?
bool uses_ring(int T, int dk, int dv, int chunk_len) { return T > 0 && gdn::ring_supported(dk, dv, chunk_len); }

int workspace_need(int B, int H, int dv, size_t* need)
{
    int G = 0;
    if (gdn::ring_groups(B * H, dv, &G) != cudaSuccess) return GDN_ERR_CUDA;
    *need = gdn::ring_workspace_bytes(G, dv);
    return GDN_OK;
}

// bf16 forward with a caller-provided workspace: the ring kernel where it
// applies, else the workspace is not touched and the plain path runs.
int run_bf16_ws(const gdn::FwdParams& p, int chunk_len, void* ws, size_t ws_bytes, cudaStream_t stream)
{
    if (!uses_ring(p.T, p.dk, p.dv, chunk_len)) return run_bf16(p, chunk_len, stream);
    size_t need = 0;
    const int st = workspace_need(p.B, p.H, p.dv, &need);
    if (st != GDN_OK) return st;
    if (!ws || !aligned(ws, 256) || ws_bytes < need) return GDN_ERR_INVALID_ARG;
    const int64_t F = ((int64_t)p.T + p.frame_len - 1) / p.frame_len;
    const size_t nq = (size_t)p.B * p.T * p.H * p.dk * 2;
    const size_t nv = (size_t)p.B * p.T * p.H * p.dv * 2;
    const size_t ng = (size_t)p.B * F * p.H * sizeof(float);
    const size_t nb = (size_t)p.B * p.T * p.H * sizeof(float);
    const size_t ns = (size_t)p.B * p.H * p.dk * p.dv * sizeof(float);
    if (overlaps(ws, need, p.q, nq) || overlaps(ws, need, p.k, nq) || overlaps(ws, need, p.v, nv) ||
        overlaps(ws, need, p.gate, ng) || overlaps(ws, need, p.beta, nb) ||
        overlaps(ws, need, p.state_in, ns) || overlaps(ws, need, p.state_out, ns) ||
        overlaps(ws, need, p.out, nv))
        return GDN_ERR_INVALID_ARG;
    return to_status(gdn::launch_ring(p, ws, ws_bytes, stream));
}

// Layout of the bidirectional workspace (elem: 2 for bf16 I/O, 4 for fp32 I/O).
int bidir_need(int B, int H, int T, int dk, int dv, int chunk_len, size_t elem, gdn::BidirLayout* L)
{
    size_t ring = 0;
    // the two scans take the sequence-parallel kernel where it applies (no ring workspace)
    if (elem == 2 && uses_ring(T, dk, dv, chunk_len) && !gdn::seq_supported(dk, dv, chunk_len)) {
        const int st = workspace_need(B, H, dv, &ring);
        if (st != GDN_OK) return st;
    }
    *L = gdn::bidir_layout(B, H, T, dk, dv, elem, ring);
    return GDN_OK;
}

// Forward scan of the caller's inputs into out; backward scan as the forward kernel
// over token-reversed copies in the workspace; then out += mirrored backward output.
int run_bidir(const gdn::FwdParams& p, int chunk_len, size_t elem, void* ws, size_t ws_bytes,
              cudaStream_t stream)
{
    if (p.T == 0) return GDN_OK;
    if ((int64_t)p.H * (p.dk > p.dv ? p.dk : p.dv) * (int64_t)elem / 16 > INT32_MAX ||
        (int64_t)p.B * p.T > 4 * (int64_t)INT32_MAX)
        return GDN_ERR_UNSUPPORTED;
    gdn::BidirLayout L;
    int st = bidir_need(p.B, p.H, p.T, p.dk, p.dv, chunk_len, elem, &L);
    if (st != GDN_OK) return st;
    if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return GDN_ERR_INVALID_ARG;
    const size_t nq = (size_t)p.B * p.T * p.H * p.dk * elem;
    const size_t nv = (size_t)p.B * p.T * p.H * p.dv * elem;
    const size_t ng = (size_t)p.B * p.F * p.H * sizeof(float);
    const size_t nb = (size_t)p.B * p.T * p.H * sizeof(float);
    if (overlaps(ws, L.total, p.q, nq) || overlaps(ws, L.total, p.k, nq) || overlaps(ws, L.total, p.v, nv) ||
        overlaps(ws, L.total, p.gate, ng) || overlaps(ws, L.total, p.beta, nb) ||
        overlaps(ws, L.total, p.out, nv))
        return GDN_ERR_INVALID_ARG;
    uint8_t* w = static_cast<uint8_t*>(ws);
    if (gdn::launch_reverse_inputs(p, elem, w, L, stream) != cudaSuccess) return GDN_ERR_CUDA;
    const gdn::FwdParams r = gdn::reversed_params(p, w, L);
    const size_t ring_bytes = L.total - L.ring;
    if (elem == 2) {
        st = ring_bytes ? run_bf16_ws(p, chunk_len, w + L.ring, ring_bytes, stream) : run_bf16(p, chunk_len, stream);
        if (st == GDN_OK)
            st = ring_bytes ? run_bf16_ws(r, chunk_len, w + L.ring, ring_bytes, stream)
                            : run_bf16(r, chunk_len, stream);
        if (st != GDN_OK) return st;
        return to_status(gdn::launch_combine<__nv_bfloat16>(p, w, L, stream));
    }
    st = to_status(gdn::launch_ffma<float>(p, chunk_len, stream));
    if (st == GDN_OK) st = to_status(gdn::launch_ffma<float>(r, chunk_len, stream));
    if (st != GDN_OK) return st;
    return to_status(gdn::launch_combine<float>(p, w, L, stream));
}

// Segment length (tokens) for a host-buffer call cut into about four pieces along T whose
// copies overlap the computation, or 0 when the call is too small for that to pay.  Pieces
// start at frame boundaries and at chunk boundaries (multiples of lcm(64, frame_len)).
int host_segment_len(int T, int frame_len)
{
    int64_t a = 64, b = frame_len;
    while (b) { const int64_t t = a % b; a = b; b = t; }
    const int64_t unit = 64 / a * (int64_t)frame_len;          // lcm(64, frame_len)
    if (unit > T / 4 || (int64_t)T < 16384) return 0;
    const int64_t seg = ((T / 4 + unit - 1) / unit) * unit;
    return seg < T ? (int)seg : 0;
}

// Host-buffer forward for B = 1 cut along T into segments: segment i's inputs go up on one
// stream, its computation (gdn_forward's kernel on that segment, the state carried on the
// device from the previous segment) runs on the caller's stream, its output comes down on a
// third, so that the copies of neighbouring segments overlap the computation and each other.
// The recurrence is the same (the state entering each segment is the exact state after the
// previous one); only the chunking inside the layer differs from one gdn_forward call.
int forward_host_pipelined(const gdn::FwdParams& p, int seg, const void* h_q, const void* h_k, const void* h_v,
                           const float* h_gate_logit, const float* h_beta_logit, const float* h_state_in,
                           float* h_state_out, void* h_out, int chunk_len, cudaStream_t stream)
{
    const int T = p.T, H = p.H, dk = p.dk, dv = p.dv, fl = p.frame_len;
    const int nseg = (T + seg - 1) / seg;
    const size_t ns = (size_t)H * dk * dv * sizeof(float);
    cudaStream_t s_in = nullptr, s_out = nullptr;
    cudaEvent_t ev[32];
    int nev = 0;
    cudaError_t e = cudaStreamCreateWithFlags(&s_in, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&s_out, cudaStreamNonBlocking);
    while (e == cudaSuccess && nev < 2 * nseg + 1 && nev < 32) {
        e = cudaEventCreateWithFlags(&ev[nev], cudaEventDisableTiming);
        if (e == cudaSuccess) ++nev;
    }
    int st = (e == cudaSuccess && nev == 2 * nseg + 1) ? GDN_OK : GDN_ERR_CUDA;
    // the caller's earlier work on `stream` comes first (the device buffers may be in use)
    if (st == GDN_OK && cudaEventRecord(ev[2 * nseg], stream) != cudaSuccess) st = GDN_ERR_CUDA;
    if (st == GDN_OK && cudaStreamWaitEvent(s_in, ev[2 * nseg], 0) != cudaSuccess) st = GDN_ERR_CUDA;
    for (int i = 0; st == GDN_OK && i < nseg; ++i) {
        const int t0 = i * seg, t1 = min(T, t0 + seg), L = t1 - t0;
        const int f0 = t0 / fl, f1 = (t1 + fl - 1) / fl;
        const size_t oq = (size_t)t0 * H * dk, ov = (size_t)t0 * H * dv, ob = (size_t)t0 * H;
        auto up = [&](void* dst, const void* src, size_t bytes) {
            if (e == cudaSuccess) e = cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, s_in);
        };
        e = cudaSuccess;
        up(static_cast<__nv_bfloat16*>(const_cast<void*>(p.q)) + oq, static_cast<const __nv_bfloat16*>(h_q) + oq,
           (size_t)L * H * dk * 2);
        up(static_cast<__nv_bfloat16*>(const_cast<void*>(p.k)) + oq, static_cast<const __nv_bfloat16*>(h_k) + oq,
           (size_t)L * H * dk * 2);
        up(static_cast<__nv_bfloat16*>(const_cast<void*>(p.v)) + ov, static_cast<const __nv_bfloat16*>(h_v) + ov,
           (size_t)L * H * dv * 2);
        up(const_cast<float*>(p.gate) + (size_t)f0 * H, h_gate_logit + (size_t)f0 * H, (size_t)(f1 - f0) * H * 4);
        up(const_cast<float*>(p.beta) + ob, h_beta_logit + ob, (size_t)L * H * 4);
        if (i == 0 && h_state_in) up(p.state_out, h_state_in, ns);
        if (e == cudaSuccess) e = cudaEventRecord(ev[2 * i], s_in);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, ev[2 * i], 0);
        if (e != cudaSuccess) { st = GDN_ERR_CUDA; break; }
        gdn::FwdParams q = p;
        q.T = L;
        q.F = f1 - f0;
        q.q = static_cast<const __nv_bfloat16*>(p.q) + oq;
        q.k = static_cast<const __nv_bfloat16*>(p.k) + oq;
        q.v = static_cast<const __nv_bfloat16*>(p.v) + ov;
        q.gate = p.gate + (size_t)f0 * H;
        q.beta = p.beta + ob;
        q.out = static_cast<__nv_bfloat16*>(p.out) + ov;
        q.state_in = (i == 0) ? (h_state_in ? p.state_out : nullptr) : p.state_out;   // carried in place
        q.state_out = p.state_out;
        st = run_bf16(q, chunk_len, stream);
        if (st != GDN_OK) break;
        if (cudaEventRecord(ev[2 * i + 1], stream) != cudaSuccess ||
            cudaStreamWaitEvent(s_out, ev[2 * i + 1], 0) != cudaSuccess ||
            cudaMemcpyAsync(static_cast<__nv_bfloat16*>(h_out) + ov, q.out, (size_t)L * H * dv * 2,
                            cudaMemcpyDeviceToHost, s_out) != cudaSuccess)
            st = GDN_ERR_CUDA;
    }
    if (st == GDN_OK && h_state_out &&
        cudaMemcpyAsync(h_state_out, p.state_out, ns, cudaMemcpyDeviceToHost, s_out) != cudaSuccess)
        st = GDN_ERR_CUDA;
    // wait for everything enqueued (also after an error), then release the streams and events
    if (s_out && cudaStreamSynchronize(s_out) != cudaSuccess) st = GDN_ERR_CUDA;
    if (s_in && cudaStreamSynchronize(s_in) != cudaSuccess) st = GDN_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) st = GDN_ERR_CUDA;
    for (int j = 0; j < nev; ++j) cudaEventDestroy(ev[j]);
    if (s_in) cudaStreamDestroy(s_in);
    if (s_out) cudaStreamDestroy(s_out);
    return st;
}

int forward_host(const void* h_q, const void* h_k, const void* h_v,
                     const float* h_gate_logit, const float* h_beta_logit,
                     const float* h_state_in, float* h_state_out, void* h_out,
                     void* d_q, void* d_k, void* d_v,
                     float* d_gate_logit, float* d_beta_logit,
                     float* d_state, void* d_out,
                     int B, int H, int T, int d_k_dim, int d_v_dim,
                     int frame_len, int chunk_len, void* ws, size_t ws_bytes, cudaStream_t stream)
{
    if (!h_q || !h_k || !h_v || !h_gate_logit || !h_beta_logit || !h_out) return GDN_ERR_INVALID_ARG;
    if ((h_state_in || h_state_out) && !d_state) return GDN_ERR_INVALID_ARG;
    gdn::FwdParams p;
    int st = validate(d_q, d_k, d_v, d_gate_logit, d_beta_logit, h_state_in ? d_state : nullptr,
                      d_state, d_out, true, 2, B, H, T, d_k_dim, d_v_dim, frame_len,
                      chunk_len, &p);
    if (st != GDN_OK) return st;
    const int64_t F = ((int64_t)T + frame_len - 1) / frame_len;
    const size_t nq = (size_t)B * T * H * d_k_dim * 2;
    const size_t nv = (size_t)B * T * H * d_v_dim * 2;
    const size_t ng = (size_t)B * F * H * sizeof(float);
    const size_t nb = (size_t)B * T * H * sizeof(float);
    const size_t ns = (size_t)B * H * d_k_dim * d_v_dim * sizeof(float);
    if (!ws && B == 1 && d_state && gdn::seq_supported(d_k_dim, d_v_dim, chunk_len)) {
        const int seg = host_segment_len(T, frame_len);
        if (seg > 0)
            return forward_host_pipelined(p, seg, h_q, h_k, h_v, h_gate_logit, h_beta_logit, h_state_in,
                                          h_state_out, h_out, chunk_len, stream);
    }
    cudaError_t e = cudaSuccess;
    if (e == cudaSuccess) e = cudaMemcpyAsync(d_q, h_q, nq, cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess) e = cudaMemcpyAsync(d_k, h_k, nq, cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess) e = cudaMemcpyAsync(d_v, h_v, nv, cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess) e = cudaMemcpyAsync(d_gate_logit, h_gate_logit, ng, cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess) e = cudaMemcpyAsync(d_beta_logit, h_beta_logit, nb, cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess && h_state_in) e = cudaMemcpyAsync(d_state, h_state_in, ns, cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return GDN_ERR_CUDA;
    st = ws ? run_bf16_ws(p, chunk_len, ws, ws_bytes, stream) : run_bf16(p, chunk_len, stream);
    if (st != GDN_OK) return st;
    e = cudaMemcpyAsync(h_out, d_out, nv, cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess && h_state_out) e = cudaMemcpyAsync(h_state_out, d_state, ns, cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    return to_status(e);
}

}  // namespace

extern "C" {

int gdn_forward(const void* q, const void* k, const void* v,
                const float* gate_logit, const float* beta_logit,
                const float* state_in, float* state_out, void* out,
                int B, int H, int T, int d_k, int d_v,
                int frame_len, int chunk_len, cudaStream_t stream)
{
    gdn::FwdParams p;
    int st = validate(q, k, v, gate_logit, beta_logit, state_in, state_out, out, true, 2,
                      B, H, T, d_k, d_v, frame_len, chunk_len, &p);
    if (st != GDN_OK) return st;
    return run_bf16(p, chunk_len, stream);
}

int gdn_forward_fp8(const void* q8, const void* k8, const void* v8, float v_scale,
                    const float* gate_logit, const float* beta_logit,
                    const float* state_in, float* state_out, void* out,
                    int B, int H, int T, int d_k, int d_v,
                    int frame_len, int chunk_len, cudaStream_t stream)
{
    if (!(v_scale >= 0.0f && v_scale <= 3.4028235e38f)) return GDN_ERR_INVALID_ARG;   // NaN fails too
    gdn::FwdParams p;
    int st = validate(q8, k8, v8, gate_logit, beta_logit, state_in, state_out, out, true, 1,
                      B, H, T, d_k, d_v, frame_len, chunk_len, &p);
    if (st != GDN_OK) return st;
    if (!gdn::seq_supported(d_k, d_v, chunk_len)) return GDN_ERR_UNSUPPORTED;
    // out is bf16 (2 bytes per element, the inputs 1): check it at its own size
    const int64_t F = ((int64_t)T + frame_len - 1) / frame_len;
    const size_t nq = (size_t)B * T * H * d_k, nv = (size_t)B * T * H * d_v, no = 2 * nv;
    const size_t ng = (size_t)B * F * H * sizeof(float), nb = (size_t)B * T * H * sizeof(float);
    const size_t ns = (size_t)B * H * d_k * d_v * sizeof(float);
    if (overlaps(out, no, q8, nq) || overlaps(out, no, k8, nq) || overlaps(out, no, v8, nv) ||
        overlaps(out, no, gate_logit, ng) || overlaps(out, no, beta_logit, nb) ||
        overlaps(out, no, state_in, ns) || overlaps(out, no, state_out, ns))
        return GDN_ERR_INVALID_ARG;
    // no token to read: the state passes through (the element type of q, k, v does not matter)
    if (T == 0) return run_bf16(p, chunk_len, stream);
    return to_status(gdn::launch_seq(p, stream, true, v_scale));
}

int gdn_state_step(const void* q, const void* k, const void* v,
                   const float* gate_logit, const float* beta_logit,
                   float* state, void* out,
                   int B, int H, int T, int d_k, int d_v,
                   int frame_len, int chunk_len, cudaStream_t stream)
{
    if (!state) return GDN_ERR_INVALID_ARG;
    gdn::FwdParams p;
    int st = validate(q, k, v, gate_logit, beta_logit, state, state, out, false, 2,
                      B, H, T, d_k, d_v, frame_len, chunk_len, &p);
    if (st != GDN_OK) return st;
    return run_bf16(p, chunk_len, stream);
}

int gdn_forward_f32(const float* q, const float* k, const float* v,
                    const float* gate_logit, const float* beta_logit,
                    const float* state_in, float* state_out, float* out,
                    int B, int H, int T, int d_k, int d_v,
                    int frame_len, int chunk_len, cudaStream_t stream)
{
    gdn::FwdParams p;
    int st = validate(q, k, v, gate_logit, beta_logit, state_in, state_out, out, true, 4,
                      B, H, T, d_k, d_v, frame_len, chunk_len, &p);
    if (st != GDN_OK) return st;
    return to_status(gdn::launch_ffma<float>(p, chunk_len, stream));
}

int gdn_state_step_f32(const float* q, const float* k, const float* v,
                       const float* gate_logit, const float* beta_logit,
                       float* state, float* out,
                       int B, int H, int T, int d_k, int d_v,
                       int frame_len, int chunk_len, cudaStream_t stream)
{
    if (!state) return GDN_ERR_INVALID_ARG;
    gdn::FwdParams p;
    int st = validate(q, k, v, gate_logit, beta_logit, state, state, out, false, 4,
                      B, H, T, d_k, d_v, frame_len, chunk_len, &p);
    if (st != GDN_OK) return st;
    return to_status(gdn::launch_ffma<float>(p, chunk_len, stream));
}

int gdn_forward_host(const void* h_q, const void* h_k, const void* h_v,
                     const float* h_gate_logit, const float* h_beta_logit,
                     const float* h_state_in, float* h_state_out, void* h_out,
                     void* d_q, void* d_k, void* d_v,
                     float* d_gate_logit, float* d_beta_logit,
                     float* d_state, void* d_out,
                     int B, int H, int T, int d_k_dim, int d_v_dim,
                     int frame_len, int chunk_len, cudaStream_t stream)
{
    return forward_host(h_q, h_k, h_v, h_gate_logit, h_beta_logit, h_state_in, h_state_out, h_out, d_q, d_k,
                        d_v, d_gate_logit, d_beta_logit, d_state, d_out, B, H, T, d_k_dim, d_v_dim, frame_len,
                        chunk_len, nullptr, 0, stream);
}

int gdn_forward_host_ws(const void* h_q, const void* h_k, const void* h_v,
                        const float* h_gate_logit, const float* h_beta_logit,
                        const float* h_state_in, float* h_state_out, void* h_out,
                        void* d_q, void* d_k, void* d_v,
                        float* d_gate_logit, float* d_beta_logit,
                        float* d_state, void* d_out,
                        int B, int H, int T, int d_k_dim, int d_v_dim,
                        int frame_len, int chunk_len, void* workspace, size_t workspace_bytes,
                        cudaStream_t stream)
{
    if (uses_ring(T, d_k_dim, d_v_dim, chunk_len) && !workspace) return GDN_ERR_INVALID_ARG;
    return forward_host(h_q, h_k, h_v, h_gate_logit, h_beta_logit, h_state_in, h_state_out, h_out, d_q, d_k,
                        d_v, d_gate_logit, d_beta_logit, d_state, d_out, B, H, T, d_k_dim, d_v_dim, frame_len,
                        chunk_len, workspace, workspace_bytes, stream);
}

int gdn_forward_gated(const void* q, const void* k, const void* v,
                      const float* gate_logit, const float* beta_logit,
                      const float* state_in, float* state_out, void* out,
                      int B, int H, int T, int d_k, int d_v, int frame_len, int chunk_len,
                      int gate_mode, void* workspace, size_t workspace_bytes, cudaStream_t stream)
{
    if (gate_mode != 0 && gate_mode != 1) return GDN_ERR_INVALID_ARG;
    gdn::FwdParams p;
    int st = validate(q, k, v, gate_logit, beta_logit, state_in, state_out, out, true, 2,
                      B, H, T, d_k, d_v, frame_len, chunk_len, &p);
    if (st != GDN_OK) return st;
    p.gate_mode = gate_mode;
    return workspace ? run_bf16_ws(p, chunk_len, workspace, workspace_bytes, stream)
                     : run_bf16(p, chunk_len, stream);
}

int gdn_forward_gated_f32(const float* q, const float* k, const float* v,
                          const float* gate_logit, const float* beta_logit,
                          const float* state_in, float* state_out, float* out,
                          int B, int H, int T, int d_k, int d_v, int frame_len, int chunk_len,
                          int gate_mode, cudaStream_t stream)
{
    if (gate_mode != 0 && gate_mode != 1) return GDN_ERR_INVALID_ARG;
    gdn::FwdParams p;
    int st = validate(q, k, v, gate_logit, beta_logit, state_in, state_out, out, true, 4,
                      B, H, T, d_k, d_v, frame_len, chunk_len, &p);
    if (st != GDN_OK) return st;
    p.gate_mode = gate_mode;
    return to_status(gdn::launch_ffma<float>(p, chunk_len, stream));
}

int gdn_forward_static_ws(const void* q, const void* k, const void* v,
                          const float* gate_logit, const float* beta_logit,
                          const float* state_in, float* state_out, void* out,
                          int B, int H, int T, int d_k, int d_v,
                          int frame_len, int chunk_len, cudaStream_t stream)
{
    gdn::FwdParams p;
    int st = validate(q, k, v, gate_logit, beta_logit, state_in, state_out, out, true, 2,
                      B, H, T, d_k, d_v, frame_len, chunk_len, &p);
    if (st != GDN_OK) return st;
    if (!uses_ring(T, d_k, d_v, chunk_len)) return run_bf16(p, chunk_len, stream);
    size_t need = 0;
    st = workspace_need(B, H, d_v, &need);
    if (st != GDN_OK) return st;
    void* ws = nullptr;
    size_t ws_bytes = 0;
    if (gdn::static_scratch(&ws, &ws_bytes) != cudaSuccess) return GDN_ERR_CUDA;
    if (need > ws_bytes) return GDN_ERR_UNSUPPORTED;     // more than the static scratch holds
    return to_status(gdn::launch_ring(p, ws, ws_bytes, stream));
}

int gdn_workspace_bytes(int B, int H, int T, int d_k, int d_v, int chunk_len, size_t* bytes)
{
    if (!bytes) return GDN_ERR_INVALID_ARG;
    *bytes = 0;
    if (B < 1 || H < 1 || T < 0 || (int64_t)B * H > INT32_MAX) return GDN_ERR_INVALID_ARG;
    if (!supported_dim(d_k) || !supported_dim(d_v)) return GDN_ERR_UNSUPPORTED;
    if (chunk_len != 16 && chunk_len != 32 && chunk_len != 64) return GDN_ERR_UNSUPPORTED;
    if (!uses_ring(T, d_k, d_v, chunk_len)) return GDN_OK;
    return workspace_need(B, H, d_v, bytes);
}

int gdn_forward_ws(const void* q, const void* k, const void* v,
                   const float* gate_logit, const float* beta_logit,
                   const float* state_in, float* state_out, void* out,
                   int B, int H, int T, int d_k, int d_v,
                   int frame_len, int chunk_len, void* workspace, size_t workspace_bytes,
                   cudaStream_t stream)
{
    gdn::FwdParams p;
    int st = validate(q, k, v, gate_logit, beta_logit, state_in, state_out, out, true, 2,
                      B, H, T, d_k, d_v, frame_len, chunk_len, &p);
    if (st != GDN_OK) return st;
    return run_bf16_ws(p, chunk_len, workspace, workspace_bytes, stream);
}

int gdn_state_step_ws(const void* q, const void* k, const void* v,
                      const float* gate_logit, const float* beta_logit,
                      float* state, void* out,
                      int B, int H, int T, int d_k, int d_v,
                      int frame_len, int chunk_len, void* workspace, size_t workspace_bytes,
                      cudaStream_t stream)
{
    if (!state) return GDN_ERR_INVALID_ARG;
    gdn::FwdParams p;
    int st = validate(q, k, v, gate_logit, beta_logit, state, state, out, false, 2,
                      B, H, T, d_k, d_v, frame_len, chunk_len, &p);
    if (st != GDN_OK) return st;
    return run_bf16_ws(p, chunk_len, workspace, workspace_bytes, stream);
}

int gdn_bidir_workspace_bytes(int B, int H, int T, int d_k, int d_v, int chunk_len, int elem_bytes,
                              size_t* bytes)
{
    if (!bytes) return GDN_ERR_INVALID_ARG;
    *bytes = 0;
    if (elem_bytes != 2 && elem_bytes != 4) return GDN_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || T < 0 || (int64_t)B * H > INT32_MAX) return GDN_ERR_INVALID_ARG;
    if (!supported_dim(d_k) || !supported_dim(d_v)) return GDN_ERR_UNSUPPORTED;
    if (chunk_len != 16 && chunk_len != 32 && chunk_len != 64) return GDN_ERR_UNSUPPORTED;
    if (T == 0) return GDN_OK;
    gdn::BidirLayout L;
    const int st = bidir_need(B, H, T, d_k, d_v, chunk_len, (size_t)elem_bytes, &L);
    if (st == GDN_OK) *bytes = L.total;
    return st;
}

int gdn_forward_bidir(const void* q, const void* k, const void* v,
                      const float* gate_logit, const float* beta_logit, void* out,
                      int B, int H, int T, int d_k, int d_v, int frame_len, int chunk_len,
                      void* workspace, size_t workspace_bytes, cudaStream_t stream)
{
    gdn::FwdParams p;
    int st = validate(q, k, v, gate_logit, beta_logit, nullptr, nullptr, out, true, 2,
                      B, H, T, d_k, d_v, frame_len, chunk_len, &p);
    if (st != GDN_OK) return st;
    return run_bidir(p, chunk_len, 2, workspace, workspace_bytes, stream);
}

int gdn_forward_bidir_f32(const float* q, const float* k, const float* v,
                          const float* gate_logit, const float* beta_logit, float* out,
                          int B, int H, int T, int d_k, int d_v, int frame_len, int chunk_len,
                          void* workspace, size_t workspace_bytes, cudaStream_t stream)
{
    gdn::FwdParams p;
    int st = validate(q, k, v, gate_logit, beta_logit, nullptr, nullptr, out, true, 4,
                      B, H, T, d_k, d_v, frame_len, chunk_len, &p);
    if (st != GDN_OK) return st;
    return run_bidir(p, chunk_len, 4, workspace, workspace_bytes, stream);
}

int gdn_softmax_attention(const void* q, const void* k, const void* v, void* out,
                          int B, int H, int T, int d_k, int d_v,
                          int frame_len, int frames_per_block, int cached_blocks, int sink_frames,
                          cudaStream_t stream)
{
    if (B < 1 || H < 1 || T < 0 || B > 65535 || H > 65535) return GDN_ERR_INVALID_ARG;
    if (frame_len < 1 || frames_per_block < 1 || cached_blocks < 0 || sink_frames < 0) return GDN_ERR_INVALID_ARG;
    if ((int64_t)frame_len * frames_per_block > INT32_MAX / 2 || (int64_t)frame_len * sink_frames > INT32_MAX)
        return GDN_ERR_INVALID_ARG;
    if (!gdn::attn_supported(d_k, d_v)) return GDN_ERR_UNSUPPORTED;
    if ((int64_t)T + 256 > INT32_MAX) return GDN_ERR_UNSUPPORTED;
    if (!q || !k || !v || !out) return GDN_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16)) return GDN_ERR_INVALID_ARG;
    const size_t nq = (size_t)B * T * H * d_k * 2, nv = (size_t)B * T * H * d_v * 2;
    if (overlaps(out, nv, q, nq) || overlaps(out, nv, k, nq) || overlaps(out, nv, v, nv)) return GDN_ERR_INVALID_ARG;
    if (T == 0) return GDN_OK;
    return to_status(gdn::launch_attn(q, k, v, out, B, H, T, d_k, d_v, frame_len * frames_per_block,
                                      cached_blocks, frame_len * sink_frames, stream));
}

const char* gdn_status_string(int status)
{
    switch (status) {
        case GDN_OK: return "ok";
        case GDN_ERR_INVALID_ARG: return "invalid argument (null, misaligned or overlapping pointer, or bad size)";
        case GDN_ERR_UNSUPPORTED: return "unsupported size (d_k, d_v in 16..128 step 16; chunk_len 16, 32 or 64)";
        case GDN_ERR_CUDA: return "CUDA runtime error";
        case GDN_ERR_TIMEOUT: return "a bounded device-side wait timed out";
        default: return "unknown status";
    }
}

int gdn_get_last_device_status(cudaStream_t stream)
{
    return gdn::read_and_clear_device_status(stream);
}

int gdn_set_wait_limit_ns(unsigned long long ns)
{
    gdn::set_wait_limit_ns((uint64_t)ns);
    return GDN_OK;
}

int gdn_bf16_path(int d_k, int d_v, int chunk_len)
{
    if (gdn::seq_supported(d_k, d_v, chunk_len)) return 2;
    return gdn::tc_supported(d_k, d_v, chunk_len) ? 1 : 0;
}

int gdn_version(void) { return 100; }

}  // extern "C"
