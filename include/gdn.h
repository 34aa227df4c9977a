/*
 * gdn.h -- C ABI of the B200 (sm_100a) gated delta rule library, libgdn.so.
 *
 * The operation is the gated delta rule of Gated DeltaNet,
 *
 *     S_t = S_{t-1} ( alpha_t ( I - beta_t k_t k_t^T ) ) + beta_t v_t k_t^T,
 *     o_t = S_t q_t,
 *
 * as stated in "Gated Delta Networks: Improving Mamba2 with Delta Rule"
 * (atlas.scime.ai summary, section "Approach"), computed either chunk by chunk
 * with the gated WY/UT representation that page names ("extended WY/UT
 * chunkwise algorithm"; "Gated DeltaNet: Harmonizing Gating and the Delta Rule
 * for Superior Linear RNNs", section "Hardware-Efficient Training"), or one
 * token at a time for decoding.  The read-out o_t = S_t q_t uses the state after
 * the token's own update (the pages do not write the read-out down).
 *
 * Conventions shared by every entry point
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *    allocates nothing and only enqueues work on `stream` (a cudaStream_t; NULL
 *    means the legacy default stream).  Calls return as soon as the work is
 *    enqueued.  No entry point keeps state between calls, except
 *    gdn_chunk_fwd_noalloc, whose fixed scratch array and cached address are
 *    described at its declaration.
 *  - Layouts are dense row-major (C order), no strides:
 *        q, k      [B, T, H, Dk]     (decode: [B, H, Dk])
 *        v, o      [B, T, H, Dv]     (decode: [B, H, Dv])
 *        log_alpha [B, T, H] float   (decode: [B, H])   log of the gate, <= 0
 *        beta      [B, T, H] float   (decode: [B, H])   write strength
 *        S0, S_T, S [B, H, Dv, Dk] float  -- row i of a head's state is value
 *                                   channel i, contiguous over the key channels.
 *  - q, k, v and o share one element type (`dtype`); the gates and the state
 *    are always float32.  Arithmetic is float32 (tensor-core products take
 *    bf16 operands with float32 accumulation on the bf16 path).
 *  - Every pointer must be 16-byte aligned.
 *  - Errors are reported before anything is launched: GDN_ERR_INVALID_ARG for a
 *    NULL required pointer, a negative size, a misaligned pointer or a short
 *    workspace; GDN_ERR_UNSUPPORTED for sizes outside the limits below;
 *    GDN_ERR_CUDA if a launch fails (the CUDA error is left for the caller to
 *    read with cudaGetLastError / cudaPeekAtLastError).
 */
#ifndef GDN_H
#define GDN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,
    GDN_ERR_UNSUPPORTED = 2,
    GDN_ERR_CUDA = 3
} gdn_status_t;

typedef enum {
    GDN_F32 = 0,   /* q, k, v, o are float32 */
    GDN_BF16 = 1   /* q, k, v, o are bfloat16 */
} gdn_dtype_t;

/* Which kernels a chunkwise forward call with these sizes runs. */
typedef enum {
    GDN_PATH_NONE = 0,     /* empty problem: nothing (or only a state copy) runs */
    GDN_PATH_SIMT = 1,     /* two CUDA-core kernels: chunk preparation, then the
                              sequential state/output pass; needs a workspace */
    GDN_PATH_TCGEN05 = 2   /* bf16, Dk = 128 or 256, chunk 64, Dv a multiple of
                              64: the per-chunk UT transform for all chunks in
                              parallel (into the workspace; at Dk = 256 also the
                              gated Q K^T and W = T diag(beta gamma) K), then one
                              tcgen05 tensor-core kernel for the sequential pass;
                              needs a workspace */
} gdn_path_t;

/* Which tcgen05 variant a gdn_chunk_fwd call with these sizes runs (the pages
 * have no counterpart; all compute the same result up to rounding):
 * 0 = not the tcgen05 path (or invalid sizes), 1 = fused (the sequential kernel
 * forms Q K^T and the WY factors itself; Dk = 128 when the sequential grid of
 * Dv / 64 x H x B CTAs fills most of the GPU), 2 = precomputed (the parallel
 * kernel also forms the gated Q K^T and W per chunk; Dk = 256, and Dk = 128 with
 * fewer than 74 sequential CTAs), 3 = split (precomputed, with each sequence cut
 * into G segments of whole chunks when the sequential grid covers under a quarter
 * of the GPU, Dk = 128 and T a multiple of 64 G: the chunk recurrence is affine in
 * the state, so each segment's map S_end = S_start M + N is formed in parallel, a
 * scan gives every segment's start state, and the segments then run at once).
 * The workspace size depends on it. */
int gdn_chunk_fwd_variant(int B, int T, int H, int Dk, int Dv, int chunk, gdn_dtype_t dtype);

/* Limits: 1 <= Dk <= 256, 1 <= Dv <= 512, chunk in {16, 32, 64}; B, T, H >= 0
 * (a zero size is an empty problem and is not an error); B, H <= 65535 and
 * B * H * (T + 64) <= 2^40 (so that no byte count derived from the sizes can
 * overflow); beyond these GDN_ERR_UNSUPPORTED. */

/*
 * Optional input prologue of the _ex entry points, applied inside the kernels
 * (bit flags, may be combined).  The pages fix neither a normalisation of q and
 * k nor a parameterisation of the gates; these are the plain readings (exact
 * write-over S_t k_t = v_t, the "Critical Insight" section of "Gated DeltaNet:
 * Harmonizing Gating and the Delta Rule ...", holds for unit keys):
 *   GDN_FLAG_L2NORM_QK   q and k are divided by sqrt(|x|^2 + 1e-6), per token
 *                        and head, before use (the caller passes raw q, k);
 *   GDN_FLAG_GATE_LOGITS log_alpha holds a logit x and beta a logit y:
 *                        log alpha = -softplus(x) = -log(1 + e^x), beta = 1 / (1 + e^-y).
 */
typedef enum {
    GDN_FLAG_NONE = 0,
    GDN_FLAG_L2NORM_QK = 1,
    GDN_FLAG_GATE_LOGITS = 2
} gdn_flag_t;

/*
 * Chunkwise forward over a whole sequence (training / prefill form).
 *
 * Each sequence is cut into chunks of `chunk` tokens (the last one may be
 * shorter).  Inside a chunk, with g_r the running sum of log_alpha from the
 * chunk start and Gamma_ri = exp(g_r - g_i) for i <= r:
 *   A    = strictly-lower( diag(beta) (Gamma o K K^T) )        gated Gram matrix
 *   T    = (I + A)^-1                                          UT transform
 *   U    = T diag(beta) ( V - diag(exp g) K S^T )              corrected values
 *   O    = diag(exp g) Q S^T + (Q K^T o Gamma o causal) U     chunk output
 *   S   <- exp(g_n) S + U^T diag(exp(g_n - g)) K               next chunk's state
 * which reproduces the token recurrence exactly up to rounding.
 *
 *   q, k, v, log_alpha, beta : inputs, layouts above (required).
 *   S0  : initial state per head, or NULL for zeros.  May equal S_T.
 *   o   : output [B,T,H,Dv] in `dtype` (required; must not overlap an input).
 *   S_T : final state per head, or NULL if not wanted.
 *   workspace / workspace_bytes : device scratch of at least
 *         gdn_chunk_fwd_workspace_size(...) bytes (NULL/0 when that is 0),
 *         16-byte aligned, overlapping no other argument; its contents on
 *         entry do not matter and are undefined on return.
 */
gdn_status_t gdn_chunk_fwd(const void *q, const void *k, const void *v,
                           const float *log_alpha, const float *beta,
                           const float *S0, void *o, float *S_T,
                           int B, int T, int H, int Dk, int Dv, int chunk,
                           gdn_dtype_t dtype, void *workspace,
                           size_t workspace_bytes, void *stream);

/* Bytes of device workspace gdn_chunk_fwd needs for these sizes (0 for empty
 * problems): on the tensor-core path 16 KiB per 64-token chunk of every
 * (batch, head), on the CUDA-core path (2 chunk^2 + chunk) floats per chunk. */
size_t gdn_chunk_fwd_workspace_size(int B, int T, int H, int Dk, int Dv,
                                    int chunk, gdn_dtype_t dtype);

/*
 * gdn_chunk_fwd with the input prologue selected by `flags` (gdn_flag_t bits;
 * 0 is exactly gdn_chunk_fwd).  q, k, log_alpha and beta are read as the flags
 * say and are not modified.  The workspace must hold
 * gdn_chunk_fwd_workspace_size_ex(..., flags) bytes (the tensor-core path keeps
 * 1/|k| per token there, the CUDA-core path the prepared inputs).  Unknown flag
 * bits: GDN_ERR_INVALID_ARG.
 */
gdn_status_t gdn_chunk_fwd_ex(const void *q, const void *k, const void *v,
                              const float *log_alpha, const float *beta,
                              const float *S0, void *o, float *S_T,
                              int B, int T, int H, int Dk, int Dv, int chunk,
                              gdn_dtype_t dtype, unsigned flags, void *workspace,
                              size_t workspace_bytes, void *stream);
size_t gdn_chunk_fwd_workspace_size_ex(int B, int T, int H, int Dk, int Dv,
                                       int chunk, gdn_dtype_t dtype, unsigned flags);

/* The path gdn_chunk_fwd takes for these sizes (a gdn_path_t), or -1 if the
 * sizes are invalid or unsupported. */
int gdn_chunk_fwd_path(int B, int T, int H, int Dk, int Dv, int chunk,
                       gdn_dtype_t dtype);

/*
 * Chunkwise forward over N variable-length sequences packed along the token
 * dimension without padding (the serving / prefill form; the pages say nothing
 * about batching, this is the plain reading): q, k [total, H, Dk], v and o
 * [total, H, Dv], log_alpha and beta [total, H], with total = cu_seqlens[N].
 * Sequence n is tokens cu_seqlens[n] .. cu_seqlens[n + 1] - 1 and has its own
 * state, S0 and S_T [N, H, Dv, Dk] (NULL S0: zeros; an empty sequence gets
 * S_T = S0).  The offsets (N + 1 ints, starting at 0, non-decreasing) are given
 * twice: `cu_seqlens` in device memory, read by the kernels, and
 * `cu_seqlens_host` in host memory, read before anything is launched for the
 * sizes and the checks; both must hold the same values.  Everything else is as
 * for gdn_chunk_fwd_ex; the workspace must hold
 * gdn_chunk_fwd_varlen_workspace_size(...) bytes.  Bad offsets:
 * GDN_ERR_INVALID_ARG; N above 65535: GDN_ERR_UNSUPPORTED.
 */
gdn_status_t gdn_chunk_fwd_varlen(const void *q, const void *k, const void *v,
                                  const float *log_alpha, const float *beta,
                                  const float *S0, void *o, float *S_T,
                                  const int *cu_seqlens, const int *cu_seqlens_host,
                                  int N, int H, int Dk, int Dv, int chunk,
                                  gdn_dtype_t dtype, unsigned flags, void *workspace,
                                  size_t workspace_bytes, void *stream);
size_t gdn_chunk_fwd_varlen_workspace_size(const int *cu_seqlens_host, int N, int H,
                                           int Dk, int Dv, int chunk, gdn_dtype_t dtype,
                                           unsigned flags);

/*
 * gdn_chunk_fwd without a caller workspace, for callers that cannot allocate
 * device memory (engines that plan all buffers at start-up and forbid
 * allocation later, paths where cudaMalloc's implicit synchronisation is not
 * acceptable, hosts that hand the library no memory).  The pages have no
 * counterpart: this is a property of the library, not of the method.
 *
 * Same arguments and results as gdn_chunk_fwd, minus the workspace.  The
 * scratch is a fixed 8 MiB array inside the library (held on every GPU that
 * loads it until exit).  The size limit is checked first: sizes whose workspace
 * (gdn_chunk_fwd_workspace_size) exceeds 8 MiB return GDN_ERR_UNSUPPORTED with
 * nothing launched and no pointer looked at; the other checks are those of
 * gdn_chunk_fwd.  The first call on a device looks up the array's address
 * (with that device current) and must come before any stream capture; the
 * address is kept for the life of the process, so a cudaDeviceReset makes this
 * entry point unusable on that device until the process restarts.  All calls
 * share the array and it keeps the last call's contents (every path that uses
 * it writes its scratch before reading it): calls whose work overlaps on the
 * GPU race and must be serialised by the caller.  Allocates nothing.
 */
gdn_status_t gdn_chunk_fwd_noalloc(const void *q, const void *k, const void *v,
                                   const float *log_alpha, const float *beta,
                                   const float *S0, void *o, float *S_T,
                                   int B, int T, int H, int Dk, int Dv, int chunk,
                                   gdn_dtype_t dtype, void *stream);

/*
 * One recurrent (decoding) step for every (b, h): the state is read, updated
 * and written back in place, constant memory per head ("Gated DeltaNet-2:
 * Decoupling Erase and Write in Linear Attention", abstract: decoding with
 * constant memory; the rule itself from the "Approach" section cited above):
 *   u = beta (v - alpha S k);   S <- alpha S + u k^T;   o = S q.
 *
 *   q, k [B,H,Dk]; v [B,H,Dv]; log_alpha, beta [B,H]; S [B,H,Dv,Dk] float32
 *   (in place); o [B,H,Dv] in `dtype`.  All required.
 */
gdn_status_t gdn_decode_step(const void *q, const void *k, const void *v,
                             const float *log_alpha, const float *beta,
                             float *S, void *o, int B, int H, int Dk, int Dv,
                             gdn_dtype_t dtype, void *stream);

/* gdn_decode_step with the input prologue selected by `flags` (gdn_flag_t bits,
 * applied in the kernel; 0 is exactly gdn_decode_step). */
gdn_status_t gdn_decode_step_ex(const void *q, const void *k, const void *v,
                                const float *log_alpha, const float *beta,
                                float *S, void *o, int B, int H, int Dk, int Dv,
                                gdn_dtype_t dtype, unsigned flags, void *stream);

/*
 * Chunkwise backward: the gradients of a scalar loss L through gdn_chunk_fwd,
 * given dL/do and dL/dS_T.  The pages name the parallel (chunkwise) training
 * algorithm ("Gated Delta Networks: Improving Mamba2 with Delta Rule", section
 * "Approach"; "Gated DeltaNet: Harmonizing Gating and the Delta Rule ...",
 * section "Hardware-Efficient Training") but print no backward; this is the
 * exact derivative of the forward (plain gates: log_alpha and beta as given,
 * no prologue), computed chunk by chunk through the WY/UT form.
 *
 *   inputs  q, k [B,T,H,Dk], v [B,T,H,Dv] in `dtype`; log_alpha, beta [B,T,H]
 *           float32; S0 [B,H,Dv,Dk] float32 or NULL (zeros) -- as for the forward;
 *           d_o [B,T,H,Dv] in `dtype`; dS_T [B,H,Dv,Dk] float32 or NULL (zeros).
 *   outputs dq, dk [B,T,H,Dk] and dv [B,T,H,Dv] in `dtype`; dlog_alpha, dbeta
 *           [B,T,H] float32; dS0 [B,H,Dv,Dk] float32 or NULL (not written).
 *
 * Two paths (gdn_chunk_bwd_path).  GDN_PATH_TCGEN05 (bf16, Dk = 128, chunk 64,
 * Dv 64 or 128): the forward's chunk tiles (P, T'', W, T) and the state
 * entering every chunk are recomputed on the tensor cores, the state gradient
 * is walked back over the chunks with dS^T in tensor memory, and the per-chunk
 * gradients are tcgen05 products in parallel over the chunks; bf16 operands,
 * float32 accumulation.  GDN_PATH_SIMT otherwise: float32 on the CUDA cores
 * (bf16 inputs widened), the same three steps.  bf16 gradients are rounded
 * once at the end.  The workspace (gdn_chunk_bwd_workspace_size bytes) holds
 * the recomputed tiles and chunk states and the state gradients.  Limits as
 * for the forward plus Dk <= 128 (GDN_ERR_UNSUPPORTED otherwise).  Outputs
 * must not overlap any input or each other; the workspace must not overlap
 * anything.  T = 0 only sets dS0 = dS_T.  Enqueued on `stream`; a bounded
 * wait of the tensor-core kernels that ran out is reported by
 * gdn_check_device_status.
 */
gdn_status_t gdn_chunk_bwd(const void *q, const void *k, const void *v,
                           const float *log_alpha, const float *beta, const float *S0,
                           const void *d_o, const float *dS_T,
                           void *dq, void *dk, void *dv, float *dlog_alpha, float *dbeta,
                           float *dS0, int B, int T, int H, int Dk, int Dv, int chunk,
                           gdn_dtype_t dtype, void *workspace, size_t workspace_bytes,
                           void *stream);
size_t gdn_chunk_bwd_workspace_size(int B, int T, int H, int Dk, int Dv, int chunk,
                                    gdn_dtype_t dtype);
/* Which kernels gdn_chunk_bwd runs for these sizes (gdn_path_t; -1 for invalid
 * or unsupported sizes): GDN_PATH_TCGEN05 for bf16, Dk = 128, chunk 64, Dv 64
 * or 128, else GDN_PATH_SIMT.  The workspace size depends on it. */
int gdn_chunk_bwd_path(int B, int T, int H, int Dk, int Dv, int chunk, gdn_dtype_t dtype);

/*
 * Channel-wise gates.  "Gated DeltaNet-2: Decoupling Erase and Write in Linear
 * Attention" (abstract) gives each key channel its own decay (as KDA does) and
 * splits the scalar beta into a channel-wise erase gate b_t on the key side and
 * a channel-wise write gate w_t on the value side; it reduces to the scalar
 * rule when the three collapse.  The pages give no formula; the reading taken
 * keeps one rank-one edit per token:
 *
 *   S_t = S_{t-1} Diag(alpha_t) (I - (b_t o k_t) k_t^T) + (w_t o v_t) k_t^T,
 *   o_t = S_t q_t,   alpha_t = exp(log_alpha_t) per key channel.
 *
 *   q, k [B,T,H,Dk] and v, o [B,T,H,Dv] in `dtype`; log_alpha and b [B,T,H,Dk]
 *   float32; w [B,T,H,Dv] float32; S0 (or NULL), S_T (or NULL) [B,H,Dv,Dk]
 *   float32, S_T may equal S0.  With log_alpha, b and w constant over their
 *   channels (log alpha, beta, beta) this is gdn_chunk_fwd.
 *
 * Chunkwise on the CUDA cores (float32 arithmetic): the channel-wise decay
 * between two rows of a chunk enters each key product as exp(Lam_r - Lam_i)
 * per channel.  Limits as for gdn_chunk_fwd plus Dk <= 128
 * (GDN_ERR_UNSUPPORTED).  Workspace: gdn_chunk_fwd_cw_workspace_size bytes
 * ((2 C^2 + C Dk) floats per chunk and head).  Enqueued on `stream`.
 */
gdn_status_t gdn_chunk_fwd_cw(const void *q, const void *k, const void *v,
                              const float *log_alpha, const float *b, const float *w,
                              const float *S0, void *o, float *S_T,
                              int B, int T, int H, int Dk, int Dv, int chunk,
                              gdn_dtype_t dtype, void *workspace, size_t workspace_bytes,
                              void *stream);
/* Which kernels gdn_chunk_fwd_cw runs for these sizes (gdn_path_t; -1 for
 * invalid sizes): GDN_PATH_TCGEN05 for bf16, Dk = 128, chunk 64 and Dv a
 * multiple of 64 -- a parallel per-chunk kernel (the channel-wise decays taken
 * through 16-row blocks, the UT transform, W and the decayed operands) and the
 * sequential tcgen05 kernel with a per-key-channel state decay -- else
 * GDN_PATH_SIMT (CUDA cores).  The workspace size depends on it. */
int gdn_chunk_fwd_cw_path(int B, int T, int H, int Dk, int Dv, int chunk, gdn_dtype_t dtype);
size_t gdn_chunk_fwd_cw_workspace_size(int B, int T, int H, int Dk, int Dv, int chunk,
                                       gdn_dtype_t dtype);

/*
 * One recurrent step of the channel-wise rule above for every (b, h), the
 * state updated in place: q, k, log_alpha, b [B,H,Dk]; v, w, o [B,H,Dv];
 * S [B,H,Dv,Dk] float32.  All required; o must not overlap S or an input.
 */
gdn_status_t gdn_decode_step_cw(const void *q, const void *k, const void *v,
                                const float *log_alpha, const float *b, const float *w,
                                float *S, void *o, int B, int H, int Dk, int Dv,
                                gdn_dtype_t dtype, void *stream);

/*
 * Synchronise the current device and report whether a fused tensor-core
 * kernel gave up since the last check: its pipeline waits are bounded (about
 * two seconds each); a CTA that times out stops, records a flag and leaves its
 * outputs incomplete.  Returns GDN_ERR_CUDA if the flag was set (and clears
 * it) or if synchronising failed, GDN_OK otherwise.
 */
gdn_status_t gdn_check_device_status(void);

/*
 * Test hook of that failure detection (the pages have no counterpart).  With
 * `enable` != 0 the sequential tensor-core kernel of every later
 * gdn_chunk_fwd* call on the current device withholds the arrival that
 * publishes its first stage of inputs: every warp's first wait runs out (about
 * two seconds), each CTA records the flag above, stops, drains its copies and
 * frees its tensor memory, and the call's outputs are left incomplete.  Nothing
 * faults and the context stays usable.  enable = 0 restores normal operation.
 * Synchronous; returns GDN_ERR_CUDA if the flag could not be written.
 */
gdn_status_t gdn_debug_withhold_first_arrival(int enable);

/* Static, human-readable name of a status code. */
const char *gdn_status_string(gdn_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H */
