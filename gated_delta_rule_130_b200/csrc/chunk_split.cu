// The small kernels of a split sequence (chunk_tc_wide.cu, launch_chunk_tcw_split):
// the identity start state of every segment's map and a zero token row, and the
// scan that chains the segments' affine maps into their start states.
//
// The chunk recurrence of "Gated Delta Networks: Improving Mamba2 with Delta Rule"
// (section "Approach"), S <- gamma_last S + U'^T diag(exp(g_last - g)) K with
// U' = U - W S^T, is affine in S: S_next = S (gamma_last I - W^T D K) + U^T D K.
// Over a segment of chunks the map composes to S_end = S_start M + N, so the start
// states of consecutive segments follow from S_start(g + 1) = S_start(g) M_g + N_g.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace gdn {

namespace {

constexpr int DK = 128;         // key width of the split path
constexpr int SCAN_ROWS = 16;   // value rows per CTA of the scan
constexpr int SCAN_THREADS = 256;

// M[i] = I (DK x DK float32) for i < n_maps; zrow[0 .. rows DK) = 0; order[z] for
// z < B (G - 1): the segments b G + g, g < G - 1 (every segment but the last).
__global__ void split_init_kernel(float *__restrict__ M, long long n_maps,
                                  __nv_bfloat16 *__restrict__ zrow, int rows,
                                  int *__restrict__ order, int B, int G) {
    const long long total = n_maps * DK * DK;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int e = (int)(i % (DK * DK));
        M[i] = (e / DK == e % DK) ? 1.f : 0.f;
    }
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < rows * DK; i += gridDim.x * blockDim.x)
        zrow[i] = __float2bfloat16_rn(0.f);
    for (int z = blockIdx.x * blockDim.x + threadIdx.x; z < B * (G - 1); z += gridDim.x * blockDim.x)
        order[z] = (z / (G - 1)) * G + z % (G - 1);
}

// One CTA per (16 value rows, head, sequence).  Arrays of every segment s = b G + g:
// N, Ss [s][H][Dv][DK], M [s][H][DK][DK] (float32).  Ss(b, 0) = S0[b] (or 0),
// Ss(b, g + 1) = Ss(b, g) M(b, g) + N(b, g), float32 throughout.
__global__ void __launch_bounds__(SCAN_THREADS)
split_scan_kernel(const float *__restrict__ S0, const float *__restrict__ N,
                  const float *__restrict__ M, float *__restrict__ Ss, int G, int H, int Dv) {
    extern __shared__ float sm[];
    float *Ms = sm;                 // DK x DK
    float *Sr = Ms + DK * DK;       // SCAN_ROWS x DK, the current start state's rows
    const int tid = threadIdx.x;
    const int r0 = blockIdx.x * SCAN_ROWS, h = blockIdx.y, b = blockIdx.z;
    const auto state = [&](int s) { return ((size_t)s * H + h) * Dv * DK + (size_t)r0 * DK; };
    for (int i = tid; i < SCAN_ROWS * DK; i += SCAN_THREADS) {
        const float x = S0 ? S0[((size_t)b * H + h) * Dv * DK + (size_t)r0 * DK + i] : 0.f;
        Sr[i] = x;
        Ss[state(b * G) + i] = x;
    }
    // thread -> column j, rows rb .. rb + 7
    const int j = tid % DK, rb = (tid / DK) * (SCAN_ROWS / 2);
    for (int g = 0; g + 1 < G; ++g) {
        const int s = b * G + g;
        __syncthreads();  // Sr written, Ms free
        const float4 *src = reinterpret_cast<const float4 *>(M + ((size_t)s * H + h) * DK * DK);
        for (int i = tid; i < DK * DK / 4; i += SCAN_THREADS)
            reinterpret_cast<float4 *>(Ms)[i] = src[i];
        __syncthreads();
        float acc[SCAN_ROWS / 2];
#pragma unroll
        for (int rr = 0; rr < SCAN_ROWS / 2; ++rr) acc[rr] = N[state(s) + (size_t)(rb + rr) * DK + j];
#pragma unroll 4
        for (int m = 0; m < DK; ++m) {
            const float mv = Ms[m * DK + j];
#pragma unroll
            for (int rr = 0; rr < SCAN_ROWS / 2; ++rr) acc[rr] = fmaf(Sr[(rb + rr) * DK + m], mv, acc[rr]);
        }
        __syncthreads();  // every thread has read Sr
#pragma unroll
        for (int rr = 0; rr < SCAN_ROWS / 2; ++rr) {
            Sr[(rb + rr) * DK + j] = acc[rr];
            Ss[state(s + 1) + (size_t)(rb + rr) * DK + j] = acc[rr];
        }
    }
}

}  // namespace

cudaError_t launch_split_init(float *M, long long n_maps, void *zrow, int rows, int *order, int B,
                              int G, cudaStream_t st) {
    split_init_kernel<<<592, 256, 0, st>>>(M, n_maps, static_cast<__nv_bfloat16 *>(zrow), rows,
                                           order, B, G);
    return cudaPeekAtLastError();
}

cudaError_t launch_split_scan(const float *S0, const float *N, const float *M, float *Ss, int B,
                              int G, int H, int Dv, cudaStream_t st) {
    if (Dv % SCAN_ROWS != 0) return cudaErrorInvalidValue;
    const int smem = (DK * DK + SCAN_ROWS * DK) * (int)sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(split_scan_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    split_scan_kernel<<<dim3(Dv / SCAN_ROWS, H, B), SCAN_THREADS, smem, st>>>(S0, N, M, Ss, G, H,
                                                                             Dv);
    return cudaPeekAtLastError();
}

}  // namespace gdn
