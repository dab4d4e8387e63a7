/*
 * gdn.h -- C ABI of the frame-wise Gated DeltaNet (GDN) forward pass on B200.
 *
 * The operation.  SANA-WM's Stage-1 DiT mixes tokens with "frame-wise Gated
 * DeltaNet + softmax every 4 blocks" (sglang cookbook SANA-WM page, section 1,
 * architecture table: 20 heads of head_dim 112) and keeps long causal history
 * as a bounded recurrent state (same page, introduction; d9249 blog, key-idea
 * section).  The pages print no formula, so the recurrence is fixed here.  For
 * every batch entry b and head h independently:
 *
 *     S_t = a_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t
 *
 *   q_t, k_t   L2-normalised per token: x / sqrt(sum_i x_i^2 + 1e-6)
 *   beta_t     sigmoid(beta_logit[b, t, h])                  (one per token)
 *   a_t        exp(-softplus(gate_logit[b, t / frame_len, h])) (one per latent
 *              frame, shared by all frame_len tokens of that frame; token 0 of
 *              a call is the first token of a frame)
 *   S          d_k x d_v float32 state (row index = key dimension), carried
 *              across chunks, frames and calls.
 *
 * The kernels evaluate it chunk by chunk (chunk_len tokens) with the WY / UT
 * form of the delta rule; results equal the token recurrence up to rounding.
 *
 * Layouts (row-major, contiguous, element counts):
 *   q, k        [B, T, H, d_k]     bf16 (gdn_forward / gdn_state_step) or f32 (*_f32)
 *   v, out      [B, T, H, d_v]     same element type as q
 *   gate_logit  [B, ceil(T / frame_len), H]  float32
 *   beta_logit  [B, T, H]          float32
 *   state       [B, H, d_k, d_v]   float32
 *
 * Ownership and memory.  The caller owns every buffer; device pointers must
 * point to device memory of the current device, host pointers (gdn_forward_host
 * only) should be pinned.  The library allocates no memory and keeps no state
 * between calls except one device status word per device.  The *_ws entry
 * points additionally take a caller-owned device workspace (see below).
 *
 * Asynchrony.  Work is enqueued on `stream` (0 = legacy default stream) and
 * the call returns without waiting, except gdn_forward_host, which waits for
 * its own stream.  Argument errors are reported synchronously and enqueue
 * nothing.
 *
 * Supported sizes: B, H >= 1; T >= 0 (T = 0 passes the state through);
 * d_k, d_v in {16, 32, ..., 128}; chunk_len in {16, 32, 64}; frame_len >= 1;
 * B * T * H * max(d_k, d_v) < 2^31 elements per tensor is NOT required (64-bit
 * indexing), but B * H, T and ceil(T / frame_len) must each fit in an int.
 * Every pointer to q, k, v, out and the state must be 16-byte aligned; the
 * logit pointers 4-byte aligned.  `out` must not overlap any input.
 * state_in == state_out is allowed (in-place update).
 *
 * Beyond the forward layer the library also provides, each documented at its
 * declaration: the workspace and allocation-free variants of the forward pass
 * (gdn_forward_ws, gdn_state_step_ws, gdn_forward_host_ws, gdn_forward_static_ws),
 * the other gate placement (gdn_forward_gated*), the bidirectional form of the
 * dense checkpoint (gdn_forward_bidir*), the chunk-causal softmax attention layer
 * with its rolling KV cache (gdn_softmax_attention), and the status and wait-bound
 * controls (gdn_get_last_device_status, gdn_set_wait_limit_ns).
 */
#ifndef GDN_H
#define GDN_H

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = -1,   /* null / misaligned / overlapping pointer, bad size  */
    GDN_ERR_UNSUPPORTED = -2,   /* size outside the supported set above               */
    GDN_ERR_CUDA = -3,          /* a CUDA runtime call or kernel launch failed        */
    GDN_ERR_TIMEOUT = -4        /* a bounded device-side wait gave up (see below)     */
} gdn_status;

/*
 * Forward pass, bf16 q/k/v/out, float32 logits and state.
 *   state_in   may be NULL: zero initial state.
 *   state_out  may be NULL: the final state is not written.
 * Returns a gdn_status.
 *
 * Which kernel runs (gdn_bf16_path reports it).  With chunk_len 64 and
 * d_k, d_v <= 112 (the SANA-WM layer has 112): the sequence-parallel kernel,
 * the fast path, with no workspace.  Every SM runs the whole per-chunk pipeline
 * of its own stretch of the B*H chains' chunks.  A stretch that begins inside a
 * chain starts the recurrence from a zero state at the latest earlier chunk
 * past which the product of the gates a_t has fallen to 2^-48 or below; where
 * the gates never shrink that far, it starts at the chain's first token from
 * state_in.  The state dropped that way is damped by the gates to 2^-48 of its
 * size: a bound, not an estimate, since a token step without its write has
 * spectral norm <= a_t.  So the result equals the recurrence up to rounding.
 * Slowly decaying gates make those warm-ups longer and the call slower, down
 * to one SM per chain when nothing decays.  With d_k or d_v = 128: a kernel
 * with one CTA per 16 state columns of each chain (about 2.5x slower per token
 * at d = 112).  With chunk_len 16 or 32: an FFMA chunked kernel.  When
 * state_in == state_out the launch is cooperative and every initial state is
 * read before any final state is written.
 */
int gdn_forward(const void* q, const void* k, const void* v,
                const float* gate_logit, const float* beta_logit,
                const float* state_in, float* state_out, void* out,
                int B, int H, int T, int d_k, int d_v,
                int frame_len, int chunk_len, cudaStream_t stream);

/*
 * One streaming block (SANA-WM streams 3 latent frames per block: sglang
 * cookbook, section 9 pipeline-config table, num_frame_per_block): advance
 * the state in place over the block's T tokens.  `state` is read and then
 * overwritten (must not be NULL); `out` may be NULL (state-only update).
 */
int gdn_state_step(const void* q, const void* k, const void* v,
                   const float* gate_logit, const float* beta_logit,
                   float* state, void* out,
                   int B, int H, int T, int d_k, int d_v,
                   int frame_len, int chunk_len, cudaStream_t stream);

/* float32 reference mode: same operation, float32 q/k/v/out, all-FFMA math. */
int gdn_forward_f32(const float* q, const float* k, const float* v,
                    const float* gate_logit, const float* beta_logit,
                    const float* state_in, float* state_out, float* out,
                    int B, int H, int T, int d_k, int d_v,
                    int frame_len, int chunk_len, cudaStream_t stream);

int gdn_state_step_f32(const float* q, const float* k, const float* v,
                       const float* gate_logit, const float* beta_logit,
                       float* state, float* out,
                       int B, int H, int T, int d_k, int d_v,
                       int frame_len, int chunk_len, cudaStream_t stream);

/*
 * FP8 input variant (the pages ship fp8 precision modes for Stage-1: FlashDreams
 * SANA-WM streaming runner page, requirements and CLI sections, precision flags;
 * they give no scheme, so the library reads it as follows).  q8, k8, v8 hold OCP
 * e4m3 bytes (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits,
 * subnormals, no infinities, 0x7F / 0xFF NaN) in the layouts of gdn_forward
 * ([B, T, H, d] row-major, one byte per element).  The layer computes
 * gdn_forward on q = e4m3(q8), k = e4m3(k8), v = v_scale * e4m3(v8): q and k
 * need no scale, since their L2 normalisation cancels any positive one; v_scale
 * (finite, >= 0) is one float32 per call.  out (bf16), the logits and the state
 * (float32) are as in gdn_forward, and state_in may alias state_out (a streaming
 * step in place).  Every e4m3 value is exactly a bf16 value, so the kernel widens
 * the tiles to bf16 in shared memory and the arithmetic is that of gdn_forward's
 * sequence-parallel kernel; v_scale is applied to the bf16 T operand of U = T V.
 * The HBM bytes per token and head drop from 900 to 564 at d = 112.
 * Supported: d_k, d_v multiples of 16 in [16, 112], chunk_len 64 (else
 * GDN_ERR_UNSUPPORTED); q8, k8, v8 16-byte aligned.  NaN codes give NaN
 * outputs.  Errors otherwise as gdn_forward; nothing is enqueued on an error.
 */
int gdn_forward_fp8(const void* q8, const void* k8, const void* v8, float v_scale,
                    const float* gate_logit, const float* beta_logit,
                    const float* state_in, float* state_out, void* out,
                    int B, int H, int T, int d_k, int d_v,
                    int frame_len, int chunk_len, cudaStream_t stream);

/*
 * End-to-end call with HOST buffers (bf16 q/k/v/out, float32 logits/state):
 * copies the inputs to the caller's device buffers d_* on `stream`, runs
 * gdn_forward, copies out (and the final state, if h_state_out is not NULL)
 * back, and waits for the stream.  h_state_in / d_state may be NULL together
 * (zero initial state); d_state is also where the final state is produced.
 * With B = 1, d_state given, the sequence-parallel kernel's sizes and T of at
 * least 16,384 tokens and four multiples of lcm(64, frame_len), the call cuts T
 * into about four segments at such boundaries: each segment's inputs go up on an
 * internal stream, its computation (the state carried in d_state) runs on
 * `stream`, its output comes down on another internal stream, so that the copies
 * overlap the computation and each other.  The result is the same recurrence;
 * only the chunking differs from one gdn_forward call (rounding-level
 * differences).  Host buffers should be pinned for the copies to overlap.
 */
int gdn_forward_host(const void* h_q, const void* h_k, const void* h_v,
                     const float* h_gate_logit, const float* h_beta_logit,
                     const float* h_state_in, float* h_state_out, void* h_out,
                     void* d_q, void* d_k, void* d_v,
                     float* d_gate_logit, float* d_beta_logit,
                     float* d_state, void* d_out,
                     int B, int H, int T, int d_k_dim, int d_v_dim,
                     int frame_len, int chunk_len, cudaStream_t stream);

/*
 * Workspace entry points.  The chunked method splits every chunk's work into a
 * state-independent half (gates, norms, the decayed key Gram matrix, the UT
 * inverse T = (I + A)^{-1} diag(beta), W = T diag(e^G) K and U = T V) and the
 * state chain.  These calls keep every chain on its own group of CTAs (one
 * per 16 state columns) over the whole sequence: they run the first half once
 * per chunk and head and hand the results to the
 * CTAs of the head's state chain through a ring of records in `workspace`
 * (a few tens of MB, sized by gdn_workspace_bytes, reused chunk after chunk so
 * that it stays in L2).  Results equal gdn_forward's up to rounding.
 *
 * gdn_workspace_bytes writes to *bytes the workspace size the *_ws calls need
 * for these sizes on the CURRENT device (it depends on the SM count); 0 means
 * the sizes take a path without workspace (d_k or d_v <= 64, chunk_len != 64
 * or T = 0) and `workspace` may then be NULL.  Returns a gdn_status.
 *
 * workspace: device memory of the current device, 256-byte aligned, at least
 * *bytes long, overlapping no other argument.  Its contents need no
 * initialisation and are garbage afterwards.  Calls that share a workspace
 * must not run concurrently (same stream, or ordered by events).  Otherwise
 * the arguments, layouts and errors are those of gdn_forward / gdn_state_step
 * / gdn_forward_host; a too small, misaligned, NULL (when needed) or
 * overlapping workspace gives GDN_ERR_INVALID_ARG.  The kernel is launched
 * cooperatively (all of its CTAs resident at once); while another kernel
 * occupies SMs of the device the launch may fail with GDN_ERR_CUDA.
 */
int gdn_workspace_bytes(int B, int H, int T, int d_k, int d_v, int chunk_len, size_t* bytes);

int gdn_forward_ws(const void* q, const void* k, const void* v,
                   const float* gate_logit, const float* beta_logit,
                   const float* state_in, float* state_out, void* out,
                   int B, int H, int T, int d_k, int d_v,
                   int frame_len, int chunk_len, void* workspace, size_t workspace_bytes,
                   cudaStream_t stream);

int gdn_state_step_ws(const void* q, const void* k, const void* v,
                      const float* gate_logit, const float* beta_logit,
                      float* state, void* out,
                      int B, int H, int T, int d_k, int d_v,
                      int frame_len, int chunk_len, void* workspace, size_t workspace_bytes,
                      cudaStream_t stream);

int gdn_forward_host_ws(const void* h_q, const void* h_k, const void* h_v,
                        const float* h_gate_logit, const float* h_beta_logit,
                        const float* h_state_in, float* h_state_out, void* h_out,
                        void* d_q, void* d_k, void* d_v,
                        float* d_gate_logit, float* d_beta_logit,
                        float* d_state, void* d_out,
                        int B, int H, int T, int d_k_dim, int d_v_dim,
                        int frame_len, int chunk_len, void* workspace, size_t workspace_bytes,
                        cudaStream_t stream);

/*
 * gdn_forward without a caller workspace and without any allocation: the same
 * shared-prep ring kernel as gdn_forward_ws, its ring kept in one static device
 * array of 24 MiB inside the library (enough for every supported size on devices
 * of up to 160 SMs).  The pages describe no such entry point: it exists so that
 * a caller that cannot provide memory (or must not allocate) still gets the
 * fast path.
 *   - Arguments, layouts and errors as gdn_forward; sizes whose ring would not
 *     fit in the static array return GDN_ERR_UNSUPPORTED.  Sizes served without
 *     a workspace (see gdn_workspace_bytes) run the plain path.
 *   - The static array is looked up once per device on the first call, which
 *     must therefore not be made inside a stream capture.
 *   - Every call on a device uses the same array: calls that overlap in time
 *     (other streams, other threads) race and give wrong results; order them.
 *     Its contents persist between calls and mean nothing to the caller.
 */
int gdn_forward_static_ws(const void* q, const void* k, const void* v,
                          const float* gate_logit, const float* beta_logit,
                          const float* state_in, float* state_out, void* out,
                          int B, int H, int T, int d_k, int d_v,
                          int frame_len, int chunk_len, cudaStream_t stream);

/*
 * The other reading of "frame-wise" (gate placement).  gdn_forward applies a
 * frame's gate a_f = exp(-softplus(gate_logit[f])) at every token of frame f
 * (gate_mode 0).  With gate_mode 1 it applies a_f once, at the first token of
 * frame f (t % frame_len == 0; a_t = 1 at the frame's other tokens), i.e. one
 * decay per latent-frame step.  The pages name the layer "frame-wise Gated
 * DeltaNet" (sglang cookbook SANA-WM page, section 1 architecture table) without
 * fixing which; both are offered.
 *   gdn_forward_gated: bf16 as gdn_forward, or as gdn_forward_ws when
 *     `workspace` is not NULL (then sized by gdn_workspace_bytes).
 *   gdn_forward_gated_f32: float32 reference mode as gdn_forward_f32.
 * gate_mode outside {0, 1} gives GDN_ERR_INVALID_ARG; everything else as the
 * entry points named.
 */
int gdn_forward_gated(const void* q, const void* k, const void* v,
                      const float* gate_logit, const float* beta_logit,
                      const float* state_in, float* state_out, void* out,
                      int B, int H, int T, int d_k, int d_v, int frame_len, int chunk_len,
                      int gate_mode, void* workspace, size_t workspace_bytes, cudaStream_t stream);

int gdn_forward_gated_f32(const float* q, const float* k, const float* v,
                          const float* gate_logit, const float* beta_logit,
                          const float* state_in, float* state_out, float* out,
                          int B, int H, int T, int d_k, int d_v, int frame_len, int chunk_len,
                          int gate_mode, cudaStream_t stream);

/*
 * Bidirectional GDN for the dense (whole-clip) checkpoint.  The pages name a
 * "bidirectional" checkpoint with full bidirectional attention over the clip
 * (sglang cookbook SANA-WM page, dense-bidirectional section) but do not give the
 * form; the library reads it as
 *     o_t = S_t^T q_t + R_t^T q_t,
 * S the forward scan of gdn_forward from a zero state, and R the same rule run from
 * the last token to the first from a zero state,
 *     R_t = a_t (I - beta_t k_t k_t^T) R_{t+1} + beta_t k_t v_t^T,  R_T = 0,
 * every token keeping its own q, k, v, beta and its own frame's gate (applied at
 * every token of the frame).  No state goes in or out.
 *
 * Layouts as gdn_forward (no state arguments).  The workspace (device, 256-byte
 * aligned, not overlapping any argument, contents need no initialisation, owned by
 * the caller and busy until the call's work on `stream` completes) holds the
 * token-reversed copies of q, k, v, beta and the per-token gate logits, the backward
 * scan's output and, for the bf16 entry at sizes that the sequence-parallel kernel
 * does not take but the ring kernel of gdn_forward_ws does (d above 112), that
 * ring: gdn_bidir_workspace_bytes gives its size (about 1.5x the bytes of q, k and
 * v; 0 when T = 0).  elem_bytes is 2 for gdn_forward_bidir, 4 for
 * gdn_forward_bidir_f32.
 *
 * Work on `stream`: one copy kernel, the forward kernel twice (gdn_forward's
 * kernel, or the ring kernel of gdn_forward_ws where the workspace holds a ring;
 * the float32 kernel of gdn_forward_f32 for the _f32 entry), one combine kernel.  Rounding (bf16 entry):
 * each scan's output is rounded to bf16, their sum is formed in fp32 and rounded to
 * bf16 again.  Errors: as gdn_forward; a missing, misaligned, small or overlapping
 * workspace gives GDN_ERR_INVALID_ARG; B*T above 4 * INT32_MAX gives
 * GDN_ERR_UNSUPPORTED.  Nothing is enqueued on an error.
 */
int gdn_bidir_workspace_bytes(int B, int H, int T, int d_k, int d_v, int chunk_len, int elem_bytes,
                              size_t* bytes);

int gdn_forward_bidir(const void* q, const void* k, const void* v,
                      const float* gate_logit, const float* beta_logit, void* out,
                      int B, int H, int T, int d_k, int d_v, int frame_len, int chunk_len,
                      void* workspace, size_t workspace_bytes, cudaStream_t stream);

int gdn_forward_bidir_f32(const float* q, const float* k, const float* v,
                          const float* gate_logit, const float* beta_logit, float* out,
                          int B, int H, int T, int d_k, int d_v, int frame_len, int chunk_len,
                          void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Chunk-causal softmax attention with a rolling KV cache: the softmax layers that
 * SANA-WM interleaves with the GDN layers (sglang cookbook SANA-WM page, section 1
 * architecture table, "softmax every 4 blocks"; pipeline-configuration table:
 * num_frame_per_block 3, num_cached_blocks 2, sink_size 1 frame).  Per batch entry
 * and head, over the whole sequence:
 *     o_t = sum_{s in K(t)} softmax_s(q_t . k_s / sqrt(d_k)) v_s,
 *     K(t) = [0, sink_frames * frame_len)
 *            U [max(0, b - cached_blocks) * L, min(T, (b + 1) * L)),
 * L = frames_per_block * frame_len, b = t / L: the sink frames, the cached blocks
 * and the whole current block (causal across blocks, full inside one).  This is
 * what streaming generation computes block by block with the cache.
 *
 * q, k: [B, T, H, d_k] bf16; v, out: [B, T, H, d_v] bf16; device pointers,
 * 16-byte aligned; out must not overlap q, k or v.  d_k, d_v in 80..128, multiples
 * of 16 (GDN_ERR_UNSUPPORTED otherwise); B, H <= 65535.  Scores and the softmax in
 * fp32, P rounded to bf16 for the P V product, output rounded to bf16.  T = 0 does
 * nothing.  One kernel launch on `stream`; no workspace.  Errors as gdn_forward.
 */
int gdn_softmax_attention(const void* q, const void* k, const void* v, void* out,
                          int B, int H, int T, int d_k, int d_v,
                          int frame_len, int frames_per_block, int cached_blocks, int sink_frames,
                          cudaStream_t stream);

/* Human-readable text of a gdn_status value (static storage). */
const char* gdn_status_string(int status);

/*
 * Every wait inside the kernels (on an mbarrier completing a TMA copy or a
 * tensor-core MMA, or on a ring flag written by another CTA) is bounded.  A wait that runs out records GDN_ERR_TIMEOUT in
 * a per-device status word and the kernel stops its work and returns cleanly.
 * This call synchronises `stream`, returns the recorded status (GDN_OK if none)
 * and clears it.
 */
int gdn_get_last_device_status(cudaStream_t stream);

/*
 * Bound, in nanoseconds, of every device-side wait of the launches that follow
 * (process-wide; default 2 s; 0 restores the default).  A bound below what a call
 * legitimately needs makes it give up: the kernel stops its work, leaves its
 * outputs undefined and records GDN_ERR_TIMEOUT for gdn_get_last_device_status;
 * the context stays usable.  Meant for testing that path.  Waits for work that is
 * already in flight when a kernel gives up keep a fixed 2 s bound.  Returns GDN_OK.
 */
int gdn_set_wait_limit_ns(unsigned long long ns);

/* Which kernel gdn_forward / gdn_state_step / gdn_forward_host dispatch to for
 * the given sizes: 0 = FFMA chunked kernel, 1 = tensor-core kernel with one CTA
 * per 16 state columns of each chain, 2 = sequence-parallel tensor-core kernel. */
int gdn_bf16_path(int d_k, int d_v, int chunk_len);

/* Library version, as major * 10000 + minor * 100 + patch. */
int gdn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H */
