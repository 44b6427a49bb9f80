/*
 * deltanet.h - C ABI of the B200 (sm_100a) delta-rule sequence-mixing library.
 *
 * The library computes the innermost layer of a DeltaNet / linear-attention
 * block: the sequence mixing over a per-head Dk x Dv state S, with the q/k/v
 * projections, feature maps of the DeltaNet layer (silu + L2 normalise) and
 * the output projection left to the caller.  Row-vector convention:
 * o_t = q_t S_t, S is Dk x Dv.
 *
 * Sources (web pages on the subject):
 *   [P1] "How a Baseten Engineer Traced 7 Years of Attention Mechanism
 *        Evolution -- From GPT-2 to Kimi K3, in Runable PyTorch" (wpnews.pro)
 *   [P3] "GPT-2 から Kimi K3 まで、AI モデルの進化を解説" (news.ainew.jp)
 *
 * Conventions common to every call
 *   - All tensors are row-major and contiguous.  q, k: (B,H,T,Dk);
 *     v, o: (B,H,T,Dv); beta, alpha: (B,H,T) float32; S0, S_out, S:
 *     (B,H,Dk,Dv) float32 (Dv contiguous); z0, z_out: (B,H,Dk) float32.
 *   - q, k, v and o share one element type, dn_dtype.  State, normaliser,
 *     beta and alpha are always float32.
 *   - Every pointer except `workspace` of the host-side queries is a DEVICE
 *     pointer on the current CUDA device.  The caller owns and allocates every
 *     buffer, including the workspace; the library allocates nothing per call.
 *   - Calls are asynchronous on `cuda_stream` (a cudaStream_t; NULL = legacy
 *     default stream).  DN_OK means "validated and launched".
 *   - Argument validation happens on the host, before any CUDA call; a
 *     rejected call launches nothing and touches no buffer.
 *   - No query scaling (no 1/sqrt(d)), no normalisation of k: the pages' read
 *     "o = q @ S" has no denominator ([P3] "DeltaNet (Fast weight
 *     programmers)").  NaN/Inf inputs propagate as through the recurrence.
 *   - Device-side waits are bounded: a wait that runs out sets a sticky
 *     status word in the workspace (read it with deltanet_get_device_status)
 *     and the kernel returns without trapping.
 */
#ifndef DELTANET_H_
#define DELTANET_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every entry point. */
typedef enum {
    DN_OK = 0,
    DN_ERR_INVALID_ARG = -1,    /* null pointer, negative size, bad aliasing     */
    DN_ERR_UNSUPPORTED = -2,    /* shape / chunk size / dtype not implemented    */
    DN_ERR_ALIGNMENT = -3,      /* q, k, v, o not 16-byte aligned (TMA rule)     */
    DN_ERR_CUDA = -4,           /* a CUDA runtime / driver call failed           */
    DN_ERR_DEVICE_TIMEOUT = -5, /* a bounded device wait ran out (status word)   */
    DN_ERR_WORKSPACE = -6       /* workspace missing or smaller than required    */
} dn_status;

/* Element type of q, k, v and o. */
typedef enum { DN_F32 = 0, DN_BF16 = 1 } dn_dtype;

/*
 * Bytes of device workspace the chunked calls need for this problem: 256 for
 * the sticky device status word and its padding, plus, for bf16 inputs, per
 * (b, h, chunk of C tokens) 4 C^2 + 4 C bytes (16,640 at C = 64, 66,048 at
 * C = 128) for the per-chunk factors T diag(beta), T diag(beta) diag(gamma)
 * (bf16 C x C) and the decay prefix (C floats) that the chunk-parallel
 * pre-pass hands to the chunk kernel.  The workspace must be
 * cleared once with deltanet_workspace_init before its first use; it may then
 * be reused by any number of calls on the same stream.  Returns 0 for sizes
 * the library rejects.
 */
size_t deltanet_workspace_bytes(int B, int H, int T, int Dk, int Dv, int C, dn_dtype dt);

/* Clear the device status word of `workspace` (asynchronous memset). */
int deltanet_workspace_init(void *workspace, size_t ws_bytes, void *cuda_stream);

/*
 * Chunkwise-parallel DeltaNet forward (prefill / training forward).
 *
 * Computes, for every (b,h) sequence and t = 0..T-1, the delta rule of [P3]
 * "DeltaNet (Parallelizing linear transformers with delta rule)" (the direct
 * per-token loop), gated as in [P1]'s Gated DeltaNet paragraph ("decay first,
 * then precise write"):
 *     S'   = alpha_t S_{t-1}                 (alpha_t = 1 when alpha == NULL)
 *     u_t  = beta_t (v_t - k_t S')
 *     S_t  = S' + k_t^T u_t
 *     o_t  = q_t S_t                         (state after the write)
 * It evaluates this in chunks of C tokens with the Householder / WY
 * reparameterisation ([P3] same section; [P1] "split the sequence into chunks
 * of size C ... a Householder transformation reparameterizes the delta
 * updates"): per chunk, T = (I + strict_lower(diag(beta) (K K^T * Gamma)))^-1,
 * U = T diag(beta) (V - diag(gamma) K S), O = diag(gamma) Q S +
 * (tril(Q K^T) * Gamma) U, S <- gamma_C S + (diag(gamma_C/gamma) K)^T U.
 *
 *   q, k       (B,H,T,Dk), v (B,H,T,Dv), element type dt, 16-byte aligned.
 *   beta       (B,H,T) float32 write strengths.
 *   alpha      (B,H,T) float32 decays in [0,1], or NULL for plain DeltaNet.
 *   S0         (B,H,Dk,Dv) float32 initial state, or NULL for zero.
 *   o          (B,H,T,Dv) output, element type dt, 16-byte aligned; must not
 *              overlap any input.
 *   S_out      (B,H,Dk,Dv) float32 final state, or NULL.  May equal S0
 *              (in-place carry); any other overlap is rejected.
 *   Dk, Dv     64 or 128.   C: 64 (bf16 and f32) or 128 (bf16 only);
 *              other values, and f32 with C = 128, give DN_ERR_UNSUPPORTED.
 *   T >= 0; T need not be a multiple of C (the ragged tail is handled
 *   exactly).  T == 0 copies S0 (or zeros) to S_out, for every C and dtype;
 *   q, k, v, beta, alpha and o may then be NULL.  B * H * ceil(T / C) must
 *   not exceed INT_MAX (DN_ERR_UNSUPPORTED otherwise).
 *   workspace  device buffer of deltanet_workspace_bytes(...) bytes.
 * bf16 runs on tcgen05 tensor cores with float32 state and accumulation;
 * f32 runs on CUDA cores in float32 throughout.
 */
int deltanet_chunk_fwd(const void *q, const void *k, const void *v,
                       const float *beta, const float *alpha, const float *S0,
                       void *o, float *S_out,
                       int B, int H, int T, int Dk, int Dv, int C, dn_dtype dt,
                       void *workspace, size_t ws_bytes, void *cuda_stream);

/*
 * Options of the *_ex entry points (bit flags, OR-ed together; 0 gives the
 * plain call).
 *
 * DN_OPT_PRESTEP: the DeltaNet layer's feature maps run inside the call ([P3]
 *   "DeltaNet (Fast weight programmers)", the layer's forward: q and k go
 *   through silu and an L2 normalisation over the head dimension, beta through
 *   a sigmoid).  q and k are then the raw projections and beta holds logits;
 *   per token  q <- silu(q) / max(||silu(q)||_2, 1e-12),  likewise k,
 *   beta <- 1 / (1 + exp(-beta)).  This saves the separate elementwise pass
 *   (and its HBM round trip) over q, k and beta.
 * DN_OPT_GATE_PER_DIM: alpha holds one decay per key dimension, (B,H,T,Dk)
 *   for the chunked call and (B,H,Dk) for the decode step: row i of the state
 *   decays by alpha_t[i] before the delta write ([P1], the KDA paragraph:
 *   scalar gating replaced by per-dimension gating).  alpha must not be NULL.
 * DN_OPT_SEQ_SPLIT (chunked call; ignored by the decode step): permission to
 *   cut each sequence into G segments that run side by side.  The chunk
 *   transition is affine in the state ([P3] "DeltaNet (Parallelizing linear
 *   transformers with delta rule)": a product of generalised Householder
 *   factors plus a write), so segment g >= 1 runs from a zero state next to
 *   its homogeneous chain (v = 0, S0 = I), and the segments are joined after:
 *   entry states Sin[g+1] = A_g Sin[g] + Send_g, outputs O_g += R_g Sin[g].
 *   The result equals the unsplit call up to rounding (R and the entry states
 *   enter one product in bf16).  The library takes G > 1 only for bf16
 *   inputs, C = 64, no other option but DN_OPT_PRESTEP (the pre-pass then
 *   maps q and k once, and both chains read the mapped copies), G <= 16
 *   dividing T, at least 8 chunks
 *   per segment, and few enough heads that both chains of every segment fit
 *   the GPU's SMs at once (B*H*G*(Dk + Dv)/64 <= SM count); among those it
 *   picks the G with the shortest estimated critical path (chunks per
 *   segment, plus about two chunks per segment boundary for the join, plus
 *   a fixed eight), and G = 1 when no split beats the plain call's T/64
 *   chunks.  deltanet_seq_segments gives G.  With G > 1 the workspace
 *   (deltanet_workspace_bytes_ex) adds
 *   B*H*T*Dk bf16 values and four (B*H*G, Dk, Dv | Dk) float32 state arrays,
 *   and the call uses a second stream of the library's own, joined to
 *   cuda_stream by events.
 *
 * Paths: DN_OPT_PRESTEP and DN_OPT_GATE_PER_DIM are built for C = 64 (C = 128
 * gives DN_ERR_UNSUPPORTED; DN_OPT_SEQ_SPLIT alone runs unsplit there).
 * DN_OPT_PRESTEP alone on bf16 inputs runs on the tcgen05 path: the pre-pass
 * maps each chunk's q and k once and writes them to the workspace, where the
 * chunk kernel reads them (the workspace of deltanet_workspace_bytes plus
 * 2 * B*H*T*Dk bf16 values); every
 * other combination (per-dimension decay, float32 inputs) runs on the
 * CUDA-core kernel (float32 arithmetic) and needs only the 256-byte status
 * word.  deltanet_workspace_bytes_ex gives the size for each case.  The
 * decode step takes both options on its usual kernel.  Unknown bits give
 * DN_ERR_INVALID_ARG.
 */
enum {
    DN_OPT_PRESTEP = 1,
    DN_OPT_GATE_PER_DIM = 2,
    DN_OPT_SEQ_SPLIT = 4
};

/* The number of segments G a deltanet_chunk_fwd_ex call with these arguments
 * runs (1: no split), for the current device.  Host only. */
int deltanet_seq_segments(int B, int H, int T, int Dk, int Dv, int C, dn_dtype dt,
                          unsigned int options);

/* The same rule for a GPU with sm_count SMs (1 when sm_count < 1): plans a
 * split for another device, or checks the rule without one.  Host only. */
int deltanet_seq_segments_sm(int B, int H, int T, int Dk, int Dv, int C, dn_dtype dt,
                             unsigned int options, int sm_count);

/* deltanet_workspace_bytes for a deltanet_chunk_fwd_ex call with `options`. */
size_t deltanet_workspace_bytes_ex(int B, int H, int T, int Dk, int Dv, int C, dn_dtype dt,
                                   unsigned int options);

/*
 * deltanet_chunk_fwd with options (see above).  Arguments, layout, ownership,
 * aliasing and status codes as deltanet_chunk_fwd, except: with
 * DN_OPT_PRESTEP q and k are raw projections and beta holds logits; with
 * DN_OPT_GATE_PER_DIM alpha is (B,H,T,Dk) float32 in [0,1].
 */
int deltanet_chunk_fwd_ex(const void *q, const void *k, const void *v,
                          const float *beta, const float *alpha, const float *S0,
                          void *o, float *S_out,
                          int B, int H, int T, int Dk, int Dv, int C, dn_dtype dt,
                          unsigned int options,
                          void *workspace, size_t ws_bytes, void *cuda_stream);

/*
 * One recurrent decode step for a batch of B x H states, updated in place.
 *
 * The case t = 1 of the recurrence above ([P3] "DeltaNet (Fast weight
 * programmers)" with a cached state; [P1] Gated DeltaNet):
 *     r = k S, p = q S (one pass over S)
 *     u = beta (v - alpha r);   o = alpha p + (q . k) u
 *     S <- alpha S + k^T u
 * Each state is read once and written once.
 *   q, k (B,H,Dk); v, o (B,H,Dv): element type dt, 16-byte aligned.
 *   beta (B,H) float32; alpha (B,H) float32 or NULL.
 *   S    (B,H,Dk,Dv) float32, updated in place; 16-byte aligned.
 *   Dk, Dv in {64, 128}.
 * Unlike the chunked calls this one takes no workspace: each CTA reads one
 * state, keeps it in registers between the two reductions and the write, and
 * hands nothing to a later kernel, so there is no scratch to place and no
 * second kernel whose bounded wait could need a status word.
 */
int deltanet_decode_step(const void *q, const void *k, const void *v,
                         const float *beta, const float *alpha, float *S, void *o,
                         int B, int H, int Dk, int Dv, dn_dtype dt, void *cuda_stream);

/*
 * deltanet_decode_step with options (see above): with DN_OPT_PRESTEP q and k
 * are raw projections and beta logits (the maps run in the kernel); with
 * DN_OPT_GATE_PER_DIM alpha is (B,H,Dk): row i of S is scaled by alpha[i]
 * before the read, then u = beta (v - k S'), o = q S' + (q . k) u,
 * S <- S' + k^T u.  Each state is still read once and written once.
 */
int deltanet_decode_step_ex(const void *q, const void *k, const void *v,
                            const float *beta, const float *alpha, float *S, void *o,
                            int B, int H, int Dk, int Dv, dn_dtype dt, unsigned int options,
                            void *cuda_stream);

/*
 * Causal linear attention with the ELU+1 feature map (the additive special
 * case: the delta rule with its read term dropped).
 *
 * [P3] "Linear attention" (cached forward) and [P1] (Q' = ELU(Q)+1,
 * K' = ELU(K)+1): with q' = ELU(q)+1, k' = ELU(k)+1 applied inside,
 *     S_t = S_{t-1} + k'_t^T v_t,   z_t = z_{t-1} + k'_t,
 *     o_t = (q'_t S_t) / (q'_t . z_t)
 * evaluated with the chunked loop of [P3] "DeltaNet (Parallelizing linear
 * transformers with delta rule)": per chunk O = (Q'S + tril(Q'K'^T) V) /
 * (Q'z + tril(Q'K'^T) 1), S += K'^T V, z += K'^T 1.
 *   q, k raw (feature map applied inside); v unmapped.
 *   S0, z0 nullable (zero); S_out, z_out nullable.  S_out may equal S0 and
 *   z_out may equal z0.  C must be 64 (bf16 and f32); C = 128 gives
 *   DN_ERR_UNSUPPORTED before anything is launched.  T == 0 copies S0 and z0
 *   (or zeros) to S_out and z_out.  Other arguments as deltanet_chunk_fwd (no
 *   beta, alpha).
 */
int linear_attn_fwd(const void *q, const void *k, const void *v,
                    const float *S0, const float *z0,
                    void *o, float *S_out, float *z_out,
                    int B, int H, int T, int Dk, int Dv, int C, dn_dtype dt,
                    void *workspace, size_t ws_bytes, void *cuda_stream);

/*
 * Bytes of device workspace deltanet_chunk_bwd needs: the 256-byte status word
 * plus the float32 entry state of every 32-token chunk of every (b, h)
 * (B * H * ceil(T / 32) * Dk * Dv * 4 bytes).  0 for sizes it rejects.
 */
size_t deltanet_chunk_bwd_workspace_bytes(int B, int H, int T, int Dk, int Dv, dn_dtype dt);

/*
 * Gradient of deltanet_chunk_fwd (the backward of a training step).
 *
 * [P3] "DeltaNet (Parallelizing linear transformers with delta rule)" gives
 * the chunkwise form as what makes linear-time training hardware-efficient;
 * this call runs the reverse of that form.  For the loss
 *     L = sum(dO * o) + sum(dS_T * S_T)
 * of the forward with the same q, k, v, beta, alpha, S0, it writes
 *     dq, dk  (B,H,T,Dk) float32      dv (B,H,T,Dv) float32
 *     dbeta   (B,H,T) float32         dlog_alpha (B,H,T) float32 = alpha * dL/dalpha
 *     dS0     (B,H,Dk,Dv) float32 (nullable)
 * dO has the shape and element type of o; dS_T is (B,H,Dk,Dv) float32 or NULL
 * (zero).  dlog_alpha may be NULL; it must be NULL when alpha is NULL.  The
 * decay enters through log(max(alpha, e^-87)), as in the forward.
 * Inputs as deltanet_chunk_fwd (Dk, Dv in {64, 128}, bf16 or f32, any T >= 0;
 * T = 0 copies dS_T, or zeros, to dS0); the float32 buffers need 4-byte
 * alignment; no output may overlap an input or another output.  Arithmetic is
 * float32 on CUDA cores: a forward sweep stores the chunk entry states in the
 * workspace, then a reverse sweep forms the gradients chunk by chunk.  The
 * result is deterministic.
 */
int deltanet_chunk_bwd(const void *q, const void *k, const void *v,
                       const float *beta, const float *alpha, const float *S0,
                       const void *dO, const float *dS_T,
                       float *dq, float *dk, float *dv, float *dbeta, float *dlog_alpha,
                       float *dS0,
                       int B, int H, int T, int Dk, int Dv, dn_dtype dt,
                       void *workspace, size_t ws_bytes, void *cuda_stream);

/*
 * Synchronise `cuda_stream` and read the sticky device status word of
 * `workspace`: DN_OK, or DN_ERR_DEVICE_TIMEOUT if any earlier kernel given
 * this workspace ran out of a bounded wait (results of that call are then
 * undefined).  Clear it with deltanet_workspace_init.
 */
int deltanet_get_device_status(const void *workspace, void *cuda_stream);

/*
 * Self-test of the bounded-wait machinery: launches one CTA that waits on an
 * mbarrier nothing arrives on, for at most `wait_ns` nanoseconds (<= 2e9),
 * then records DN_ERR_DEVICE_TIMEOUT in the workspace status word and exits.
 * Used by tests to show that a wait that runs out ends in a status the host
 * reads, with the context still usable.
 */
int deltanet_selftest_wait_timeout(void *workspace, size_t ws_bytes, long long wait_ns,
                                   void *cuda_stream);

/*
 * deltanet_chunk_fwd without a workspace argument, for callers that cannot
 * allocate device memory where they call the library: code running inside
 * another framework's allocator or memory-pool hooks (a cudaMalloc there would
 * re-enter the allocator), plug-ins or embedded runtimes whose device memory is
 * budgeted up front, and paths that must avoid cudaMalloc because it can
 * synchronise the device.  The pages have no counterpart to this; it only
 * changes where the scratch lives.
 *
 * Arguments, computation, results and status codes are those of
 * deltanet_chunk_fwd.  The scratch (the device status word and, for bf16
 * inputs, the per-chunk factors of the chunked solve) comes from a static
 * device array of 1 MiB inside the library, one per device that loads it,
 * held until the process exits: enough for about 64 (b, h, 64-token chunk)
 * units of bf16 work.  Nothing is allocated: no
 * cudaMalloc, cudaFree or allocating library routine is called.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with the caller's current device, which must be
 *     the device of the pointers and the stream); make that first call before
 *     any stream capture.  The address is kept for the life of the process: a
 *     process that resets the device (cudaDeviceReset) after that first call
 *     must not call this entry point on that device again.
 *   - Each call clears the status word with an asynchronous memset on
 *     `cuda_stream`, then launches the kernel there.  A call rejected by
 *     validation may still have cleared that private word; it touches none of
 *     the caller's buffers.
 *   - All calls on a device share the one array: calls that overlap on the GPU
 *     (for instance on different streams) race on it.  The status word cannot
 *     be read back through this entry point; use deltanet_chunk_fwd with a
 *     caller-owned workspace when bounded-wait timeouts must be observed.
 *   - A problem whose workspace need (deltanet_workspace_bytes) exceeds 1 MiB
 *     is rejected with DN_ERR_WORKSPACE.
 */
int deltanet_chunk_fwd_noalloc(const void *q, const void *k, const void *v,
                               const float *beta, const float *alpha, const float *S0,
                               void *o, float *S_out,
                               int B, int H, int T, int Dk, int Dv, int C, dn_dtype dt,
                               void *cuda_stream);

/*
 * Bytes of DEVICE workspace deltanet_chunk_fwd_host needs: the 256-byte status
 * word, then two staging slots, each holding one group of heads' q, k, v, o,
 * beta, alpha, S0 and S_out plus that group's pre-pass factors (the per-chunk
 * factors of deltanet_workspace_bytes for the group's heads).  The heads are
 * taken in groups of ceil(B*H / 4).  Each region starts on a 256-byte boundary.
 * Returns 0 for sizes the library rejects.
 */
size_t deltanet_host_workspace_bytes(int B, int H, int T, int Dk, int Dv, int C, dn_dtype dt);

/*
 * deltanet_chunk_fwd on HOST buffers: q, k, v, beta, alpha, S0, o and S_out
 * have the shapes, types and meaning of deltanet_chunk_fwd's arguments but
 * live in host memory (no alignment needed).  The heads pass through the
 * device in groups of ceil(B*H / 4): the host-to-device copy of one group,
 * the computation of the group before it and the device-to-host copy of the
 * group before that run at the same time, on three streams the library
 * creates once per device.  Those streams start after the work already queued
 * on cuda_stream, and cuda_stream waits for the last copy back, so the call is
 * asynchronous on cuda_stream like the device entry points: the host buffers
 * must stay valid, and o and S_out must not be read, until cuda_stream has
 * passed this call (cudaStreamSynchronize).  The copies only overlap when the
 * host buffers are page-locked (cudaHostAlloc / cudaHostRegister); pageable
 * memory gives the same results more slowly.
 *
 *   workspace  DEVICE buffer of deltanet_host_workspace_bytes(...) bytes,
 *              16-byte aligned, cleared once with deltanet_workspace_init;
 *              its status word is read with deltanet_get_device_status.
 * Errors as deltanet_chunk_fwd; o must not overlap an input, S_out may equal
 * S0.  Concurrent calls on one device are queued one after the other.
 */
int deltanet_chunk_fwd_host(const void *q, const void *k, const void *v,
                            const float *beta, const float *alpha, const float *S0,
                            void *o, float *S_out,
                            int B, int H, int T, int Dk, int Dv, int C, dn_dtype dt,
                            void *workspace, size_t ws_bytes, void *cuda_stream);

/* Static string for a status code. */
const char *deltanet_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
int deltanet_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DELTANET_H_ */
