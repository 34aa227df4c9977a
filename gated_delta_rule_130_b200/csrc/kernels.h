// Internal launchers of the library's kernels (host side).  Each enqueues its
// kernels on `st` and returns the launch status; argument checking is done by
// the C-ABI layer before any of these is called.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace gdn {

// Recurrent step over every (b,h): decode.cu.
// (flags: input prologue bits, see common.cuh.)
cudaError_t launch_decode(const void *q, const void *k, const void *v, const float *log_alpha,
                          const float *beta, float *S, void *o, int B, int H, int Dk, int Dv,
                          bool bf16, unsigned flags, cudaStream_t st);

// Input prologue for the CUDA-core path: prologue.cu.  Writes the prepared q, k
// (if L2-normalising) and gates (if given as logits) into `ws` and points `out`
// at the arrays to use (the originals where the flags leave them alone).
struct Prepared {
    const void *q, *k;
    const float *log_alpha, *beta;
};
size_t prologue_bytes(int B, int T, int H, int Dk, bool bf16, unsigned flags);
cudaError_t launch_prologue(const void *q, const void *k, const float *la, const float *be,
                            int B, int T, int H, int Dk, bool bf16, unsigned flags, void *ws,
                            Prepared *out, cudaStream_t st);

// CUDA-core chunkwise forward (any supported size, f32 or bf16): chunk_simt.cu.
size_t simt_workspace_bytes(int B, int T, int H, int chunk);
cudaError_t launch_chunk_simt(const void *q, const void *k, const void *v, const float *log_alpha,
                              const float *beta, const float *S0, void *o, float *S_T, int B,
                              int T, int H, int Dk, int Dv, int chunk, bool bf16, void *workspace,
                              cudaStream_t st);

// The backward's recomputation on the CUDA-core path (chunk_simt.cu): T, P, g
// per chunk into ws_prep ([B,H,NT] x (2 C^2 + C) floats) and the state entering
// every chunk into S_hist ([B,H,NT,Dv,Dk] floats).
// (S_hist == nullptr: T, P, g only.)
cudaError_t launch_bwd_recompute(const void *q, const void *k, const void *v, const float *la,
                                 const float *beta, const float *S0, int B, int T, int H, int Dk,
                                 int Dv, int chunk, bool bf16, float *ws_prep, float *S_hist,
                                 cudaStream_t st);

// CUDA-core chunkwise backward (Dk <= 128): chunk_bwd.cu.  Workspace: the
// recomputed T, P, g, the chunk states and the state gradients.
// bf16 sizes the tensor-core forward takes recompute the chunk states with it
// (its [T'; T''] tiles and a scratch output then also live in the workspace).
bool bwd_supported(int Dk, int chunk);
size_t bwd_workspace_bytes(int B, int T, int H, int Dk, int Dv, int chunk, bool bf16);
cudaError_t launch_chunk_bwd(const void *q, const void *k, const void *v, const float *la,
                             const float *beta, const float *S0, const void *d_o,
                             const float *dS_T, void *dq, void *dk, void *dv, float *dla,
                             float *dbeta, float *dS0, int B, int T, int H, int Dk, int Dv,
                             int chunk, bool bf16, void *workspace, cudaStream_t st);

// Tensor-core chunkwise backward (bf16, Dk = 128, chunk 64, Dv 64 or 128):
// chunk_bwd_tc.cu, reached through launch_chunk_bwd.  Its recompute is the
// precomputed variant (chunk_tc_wide.cu, launch_recompute_bwd): the [P; T''], W
// and T tiles of every chunk, then the state entering every chunk (bf16).
bool bwd_tc_supported(int B, int T, int H, int Dk, int Dv, int chunk, bool bf16);
size_t bwd_tc_workspace_bytes(int B, int T, int H, int Dv);
cudaError_t launch_chunk_bwd_tc(const void *q, const void *k, const void *v, const float *la,
                                const float *beta, const float *S0, const void *d_o,
                                const float *dS_T, void *dq, void *dk, void *dv, float *dla,
                                float *dbeta, float *dS0, int B, int T, int H, int Dv,
                                void *workspace, cudaStream_t st);
cudaError_t launch_recompute_bwd(const void *q, const void *k, const void *v,
                                 const float *log_alpha, const float *beta, const float *S0,
                                 int B, int T, int H, int Dv, void *pt, void *wt, void *tr,
                                 void *S_hist, cudaStream_t st);

// Channel-wise gates (decay per key channel, erase gate b on the key side,
// write gate w on the value side; CUDA cores, Dk <= 128): chunk_cw.cu.
// log alpha and b are [B,T,H,Dk] float32, w is [B,T,H,Dv] float32.
bool cw_supported(int Dk, int chunk);
size_t cw_workspace_bytes(int B, int T, int H, int Dk, int chunk);
cudaError_t launch_chunk_cw(const void *q, const void *k, const void *v, const float *la,
                            const float *bg, const float *wg, const float *S0, void *o, float *S_T,
                            int B, int T, int H, int Dk, int Dv, int chunk, bool bf16,
                            void *workspace, cudaStream_t st);
cudaError_t launch_decode_cw(const void *q, const void *k, const void *v, const float *la,
                             const float *bg, const float *wg, float *S, void *o, int B, int H,
                             int Dk, int Dv, bool bf16, cudaStream_t st);

// tcgen05 chunkwise forward (bf16, chunk 64, Dk = 128 or 256, Dv a multiple of
// 64), in one of two variants chosen inside these calls from the sizes:
//  - fused (chunk_tc.cu, Dk = 128): the parallel kernel writes one bf16
//    [T'; T''] tile (128 x 64) per chunk of every head (and 1/|k| per token
//    with the L2-normalisation flag); the sequential kernel forms Q K^T and the
//    WY factors itself.  Chosen when the sequential grid fills most of the GPU.
//  - precomputed (chunk_tc_wide.cu, Dk = 256 always, Dk = 128 when the
//    sequential grid would leave most SMs idle): the parallel kernel also forms
//    the gated Q K^T and W, writing one bf16 [P; T''] tile (128 x 64) and one
//    bf16 W tile (64 x Dk) per chunk of every head (and 1/|q|, 1/|k| per token
//    with the flag); the sequential kernel keeps only the state-dependent
//    products, a shorter chain per chunk.
bool tc_supported(int B, int T, int H, int Dk, int Dv, int chunk, bool bf16);
bool tc_precomputed(int n_seq, int H, int Dk, int Dv);
size_t tc_workspace_bytes(int B, int T, int H, unsigned flags, int Dk, int Dv);
// The fused variant's workspace (the backward's state recompute uses it).
size_t tc_workspace_bytes_fused(int B, int T, int H, unsigned flags);
// S_hist (optional): the state entering every chunk, [B*H][NT][Dv][Dk] float32.
cudaError_t launch_chunk_tc(const void *q, const void *k, const void *v, const float *log_alpha,
                            const float *beta, const float *S0, void *o, float *S_T, int B, int T,
                            int H, int Dk, int Dv, unsigned flags, void *workspace,
                            cudaStream_t st, float *S_hist = nullptr);
// The same over n_seq sequences packed along the token dimension: fixed length
// T_fixed (cu_seqlens == nullptr) or the device offsets cu_seqlens (n_seq + 1);
// total_chunks = sum of ceil(length / 64).  The workspace then starts with the
// per-sequence chunk offsets (computed on the device).
size_t tc_workspace_bytes_seqs(int n_seq, long long total_chunks, int H, bool varlen,
                               unsigned flags, int Dk, int Dv);
cudaError_t launch_chunk_tc_seqs(const void *q, const void *k, const void *v,
                                 const float *log_alpha, const float *beta, const float *S0,
                                 void *o, float *S_T, int n_seq, int T_fixed, long long total_T,
                                 const int *cu_seqlens, long long total_chunks, int H, int Dk,
                                 int Dv, unsigned flags, void *workspace, cudaStream_t st,
                                 float *S_hist = nullptr);

// Shared by both tcgen05 files (chunk_tc.cu): bytes of the per-sequence chunk
// offsets and launch order at the start of a packed batch's workspace, and the
// one-block kernel that computes them on the device.
size_t tc_offsets_bytes(int n_seq, bool varlen);
cudaError_t launch_seq_schedule(const int *cu_seqlens, int n_seq, int *cu_chunks, int *order,
                                cudaStream_t st);
// The precomputed variant (chunk_tc_wide.cu); reached through the tc_* calls above.
size_t tcw_workspace_bytes_seqs(int n_seq, long long total_chunks, int H, bool varlen,
                                unsigned flags, int Dk);
cudaError_t launch_chunk_tcw_seqs(const void *q, const void *k, const void *v,
                                  const float *log_alpha, const float *beta, const float *S0,
                                  void *o, float *S_T, int n_seq, int T_fixed, long long total_T,
                                  const int *cu_seqlens, long long total_chunks, int H, int Dk,
                                  int Dv, unsigned flags, void *workspace, cudaStream_t st);

// A fixed-length batch whose sequential grid covers under a quarter of the GPU
// (Dk = 128, T a multiple of 64 G) runs split into G segments per sequence
// (chunk_tc_wide.cu; the precomputed variant's kernels, reached through
// launch_chunk_tcw_seqs): tcw_split_segments gives G (1: not split).
int tcw_split_segments(int B, int T, int H, int Dk, int Dv);
size_t tcw_split_workspace_bytes(int B, int T, int H, int Dv, unsigned flags);
cudaError_t launch_chunk_tcw_split(const void *q, const void *k, const void *v,
                                   const float *log_alpha, const float *beta, const float *S0,
                                   void *o, float *S_T, int B, int T, int H, int Dv,
                                   unsigned flags, void *workspace, cudaStream_t st);
// Its small kernels (chunk_split.cu): M[i] = I (128 x 128) for i < n_maps, `rows`
// zero rows of 128 bf16 and the order of pass 1 (every segment but the last of
// each of the B sequences); the scan of the segments' start states.
cudaError_t launch_split_init(float *M, long long n_maps, void *zrow, int rows, int *order, int B,
                              int G, cudaStream_t st);
cudaError_t launch_split_scan(const float *S0, const float *N, const float *M, float *Ss, int B,
                              int G, int H, int Dv, cudaStream_t st);

// The precomputed variant's sequential kernel (Dk = 128) in its channel-wise
// mode: operands Q o exp(Lam), K o exp(Lam_last - Lam), w o V ([B*T, H, D] bf16),
// the [P; T''] and W tiles and exp(Lam_last) per key channel ([tiles][128]
// float32), all from chunk_cw_tc.cu's parallel kernel.
cudaError_t launch_chunk_tcw_seq_cw(const void *qe, const void *kd, const void *vw,
                                    const void *pt, const void *wt, const float *glk,
                                    const float *S0, void *o, float *S_T, int B, int T, int H,
                                    int Dv, cudaStream_t st);

// Channel-wise gates on the tensor cores (bf16, Dk = 128, chunk 64, Dv a
// multiple of 64): chunk_cw_tc.cu.
bool cw_tc_supported(int B, int T, int H, int Dk, int Dv, int chunk, bool bf16);
size_t cw_tc_workspace_bytes(int B, int T, int H, int Dv);
cudaError_t launch_chunk_cw_tc(const void *q, const void *k, const void *v, const float *la,
                               const float *bg, const float *wg, const float *S0, void *o,
                               float *S_T, int B, int T, int H, int Dv, void *workspace,
                               cudaStream_t st);

// Read and clear the flag a fused-kernel CTA sets when one of its bounded waits
// times out (synchronous).
cudaError_t read_and_clear_device_error(unsigned int *flag);
cudaError_t read_and_clear_device_error_wide(unsigned int *flag);  // the Dk = 256 kernel's flag
cudaError_t read_and_clear_device_error_bwd(unsigned int *flag);   // the backward's tcgen05 kernels
// Test hook: the sequential tcgen05 kernel withholds its first stage's arrival
// (every CTA then times out, about two seconds, and sets that flag).
cudaError_t set_withhold_first_arrival(bool on);

}  // namespace gdn
