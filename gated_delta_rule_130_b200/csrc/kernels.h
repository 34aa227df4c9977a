// Internal launchers of the library's kernels (host side).  Each enqueues its
// kernels on `st` and returns the launch status; argument checking is done by
// the C-ABI layer before any of these is called.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace gdn {

// Recurrent step over every (b,h): decode.cu.
cudaError_t launch_decode(const void *q, const void *k, const void *v, const float *log_alpha,
                          const float *beta, float *S, void *o, int B, int H, int Dk, int Dv,
                          bool bf16, cudaStream_t st);

// CUDA-core chunkwise forward (any supported size, f32 or bf16): chunk_simt.cu.
size_t simt_workspace_bytes(int B, int T, int H, int chunk);
cudaError_t launch_chunk_simt(const void *q, const void *k, const void *v, const float *log_alpha,
                              const float *beta, const float *S0, void *o, float *S_T, int B,
                              int T, int H, int Dk, int Dv, int chunk, bool bf16, void *workspace,
                              cudaStream_t st);

// tcgen05 chunkwise forward (bf16, Dk = 128, chunk 64): chunk_tc.cu.  The
// workspace holds one bf16 [T'; T''] tile (128 x 64) per chunk of every head.
bool tc_supported(int B, int T, int H, int Dk, int Dv, int chunk, bool bf16);
size_t tc_workspace_bytes(int B, int T, int H);
cudaError_t launch_chunk_tc(const void *q, const void *k, const void *v, const float *log_alpha,
                            const float *beta, const float *S0, void *o, float *S_T, int B, int T,
                            int H, int Dk, int Dv, void *workspace, cudaStream_t st);

// Read and clear the flag a fused-kernel CTA sets when one of its bounded waits
// times out (synchronous).
cudaError_t read_and_clear_device_error(unsigned int *flag);

}  // namespace gdn
