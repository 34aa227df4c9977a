// Input prologue for the CUDA-core chunkwise path: one pass that writes the
// prepared inputs into the workspace, which the unchanged path then reads.
//   q_hat, k_hat = x / sqrt(|x|^2 + eps) per token and head (when L2-normalising;
//                  stored in the input element type)
//   log alpha = -softplus(x), beta = sigmoid(y)   (when the gates are logits)
// The tensor-core path and the decode step apply the same prologue inside their
// own kernels instead (scales folded into existing products).
#include "common.cuh"
#include "kernels.h"

namespace gdn {

// One warp per (token, head) row: lanes stride over the Dk channels.
template <typename T>
__global__ void __launch_bounds__(256)
prologue_rows(const T *__restrict__ q, const T *__restrict__ k, const float *__restrict__ la,
              const float *__restrict__ be, T *__restrict__ qn, T *__restrict__ kn,
              float *__restrict__ la_out, float *__restrict__ be_out, long long n_rows, int Dk,
              unsigned flags) {
    const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) / 32;
    const int lane = threadIdx.x % 32;
    if (row >= n_rows) return;  // whole warp leaves together
    if (flags & kFlagL2Norm) {
        const T *qr = q + row * Dk;
        const T *kr = k + row * Dk;
        float q2 = 0.f, k2 = 0.f;
        for (int c = lane; c < Dk; c += 32) {
            const float a = to_f32(qr[c]), b = to_f32(kr[c]);
            q2 += a * a;
            k2 += b * b;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            q2 += __shfl_xor_sync(0xffffffffu, q2, off);
            k2 += __shfl_xor_sync(0xffffffffu, k2, off);
        }
        const float rq = rsqrtf(q2 + kNormEps), rk = rsqrtf(k2 + kNormEps);
        for (int c = lane; c < Dk; c += 32) {
            qn[row * Dk + c] = from_f32<T>(rq * to_f32(qr[c]));
            kn[row * Dk + c] = from_f32<T>(rk * to_f32(kr[c]));
        }
    }
    if ((flags & kFlagGateLogits) && lane == 0) {
        const float2 gp = gate_pair(la[row], be[row], flags);
        la_out[row] = gp.x;
        be_out[row] = gp.y;
    }
}

size_t prologue_bytes(int B, int T, int H, int Dk, bool bf16, unsigned flags) {
    const size_t rows = (size_t)B * T * H, esz = bf16 ? 2 : 4;
    size_t n = 0;
    if (flags & kFlagL2Norm) n += 2 * rows * Dk * esz;
    if (flags & kFlagGateLogits) n += 2 * rows * sizeof(float);
    return (n + 255) & ~size_t(255);
}

cudaError_t launch_prologue(const void *q, const void *k, const float *la, const float *be,
                            int B, int T, int H, int Dk, bool bf16, unsigned flags, void *ws,
                            Prepared *out, cudaStream_t st) {
    const long long rows = (long long)B * T * H;
    const size_t esz = bf16 ? 2 : 4;
    uint8_t *p = static_cast<uint8_t *>(ws);
    out->q = q;
    out->k = k;
    out->log_alpha = la;
    out->beta = be;
    void *qn = nullptr, *kn = nullptr;
    float *la_out = nullptr, *be_out = nullptr;
    if (flags & kFlagL2Norm) {
        qn = p;
        kn = p + rows * Dk * esz;
        p += 2 * rows * Dk * esz;
        out->q = qn;
        out->k = kn;
    }
    if (flags & kFlagGateLogits) {
        la_out = reinterpret_cast<float *>(p);
        be_out = la_out + rows;
        out->log_alpha = la_out;
        out->beta = be_out;
    }
    if (!flags || rows == 0) return cudaSuccess;
    const unsigned blocks = (unsigned)((rows * 32 + 255) / 256);
    if (bf16)
        prologue_rows<__nv_bfloat16><<<blocks, 256, 0, st>>>(
            static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k), la, be,
            static_cast<__nv_bfloat16 *>(qn), static_cast<__nv_bfloat16 *>(kn), la_out, be_out,
            rows, Dk, flags);
    else
        prologue_rows<float><<<blocks, 256, 0, st>>>(
            static_cast<const float *>(q), static_cast<const float *>(k), la, be,
            static_cast<float *>(qn), static_cast<float *>(kn), la_out, be_out, rows, Dk, flags);
    return cudaPeekAtLastError();
}

}  // namespace gdn
