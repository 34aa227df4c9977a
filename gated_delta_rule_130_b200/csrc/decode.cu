// Recurrent (single-token) step of the gated delta rule, state in HBM updated in
// place.  For each head and each value channel i (one row of S):
//     sk = S_i . k,  sq = S_i . q,  kq = k . q
//     u_i = beta (v_i - alpha sk)
//     S_i <- alpha S_i + u_i k            (the rule of "Gated Delta Networks:
//                                          Improving Mamba2 with Delta Rule",
//                                          section "Approach", expanded per row)
//     o_i = S_i(new) . q = alpha sq + u_i kq
// One pass over the state: every byte of S is read once and written once, so
// the step is bound by HBM bandwidth (about one flop per byte).
// With the input prologue (flags), k and q are scaled by 1/sqrt(|x|^2 + eps):
// the norms come from the same reductions as the dot products and the scales
// are folded into sk, sq, kq and the rank-one update; the gates may arrive as
// logits.
#include "common.cuh"
#include "kernels.h"

namespace gdn {

// Vectorised form for Dk = 16 * L: a state row is shared by L lanes (L divides
// 32), each lane owning four float4 of the row.  Lane l of a row holds float4
// number j*L + l (j = 0..3), so each load instruction of a warp reads whole
// consecutive 128-byte lines.
template <typename T, int L>
__global__ void __launch_bounds__(256)
decode_rows_vec(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                const float *__restrict__ log_alpha, const float *__restrict__ beta,
                float *__restrict__ S, T *__restrict__ o, long long n_rows, int Dv,
                unsigned flags) {
    constexpr int DK = 16 * L;
    const long long gt = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long row = gt / L;
    const int lane = (int)(gt % L);
    const bool valid = row < n_rows;
    const long long head = valid ? row / Dv : 0;

    float4 s[4], kk[4], qq[4];
    float4 *srow = reinterpret_cast<float4 *>(S + (valid ? row : 0) * DK);
    const T *kh = k + head * DK;
    const T *qh = q + head * DK;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int f4 = j * L + lane;  // float4 index within the row
        if (valid) {
            s[j] = srow[f4];
            kk[j] = load4(kh + 4 * f4);
            qq[j] = load4(qh + 4 * f4);
        } else {
            s[j] = kk[j] = qq[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    float sk = 0.f, sq = 0.f, kq = 0.f, kk2 = 0.f, qq2 = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        sk += s[j].x * kk[j].x + s[j].y * kk[j].y + s[j].z * kk[j].z + s[j].w * kk[j].w;
        sq += s[j].x * qq[j].x + s[j].y * qq[j].y + s[j].z * qq[j].z + s[j].w * qq[j].w;
        kq += kk[j].x * qq[j].x + kk[j].y * qq[j].y + kk[j].z * qq[j].z + kk[j].w * qq[j].w;
        if (flags & kFlagL2Norm) {
            kk2 += kk[j].x * kk[j].x + kk[j].y * kk[j].y + kk[j].z * kk[j].z + kk[j].w * kk[j].w;
            qq2 += qq[j].x * qq[j].x + qq[j].y * qq[j].y + qq[j].z * qq[j].z + qq[j].w * qq[j].w;
        }
    }
#pragma unroll
    for (int off = L / 2; off > 0; off >>= 1) {
        sk += __shfl_xor_sync(0xffffffffu, sk, off);
        sq += __shfl_xor_sync(0xffffffffu, sq, off);
        kq += __shfl_xor_sync(0xffffffffu, kq, off);
        if (flags & kFlagL2Norm) {
            kk2 += __shfl_xor_sync(0xffffffffu, kk2, off);
            qq2 += __shfl_xor_sync(0xffffffffu, qq2, off);
        }
    }
    if (!valid) return;
    // k_hat = rk k, q_hat = rq q
    const float rk = (flags & kFlagL2Norm) ? rsqrtf(kk2 + kNormEps) : 1.f;
    const float rq = (flags & kFlagL2Norm) ? rsqrtf(qq2 + kNormEps) : 1.f;
    const float2 gp = gate_pair(log_alpha[head], beta[head], flags);
    const float alpha = expf(gp.x);
    const float b = gp.y;
    const int i = (int)(row - head * Dv);
    const float u = b * (to_f32(v[head * Dv + i]) - alpha * rk * sk);
    const float uk = u * rk;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float4 n;
        n.x = alpha * s[j].x + uk * kk[j].x;
        n.y = alpha * s[j].y + uk * kk[j].y;
        n.z = alpha * s[j].z + uk * kk[j].z;
        n.w = alpha * s[j].w + uk * kk[j].w;
        srow[j * L + lane] = n;
    }
    if (lane == 0) o[head * Dv + i] = from_f32<T>(rq * (alpha * sq + uk * kq));
}

// Any Dk: one warp per state row, lanes stride over the key channels.
template <typename T>
__global__ void __launch_bounds__(256)
decode_rows_warp(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                 const float *__restrict__ log_alpha, const float *__restrict__ beta,
                 float *__restrict__ S, T *__restrict__ o, long long n_rows, int Dk, int Dv,
                 unsigned flags) {
    const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) / 32;
    const int lane = threadIdx.x % 32;
    if (row >= n_rows) return;  // whole warp leaves together
    const long long head = row / Dv;
    float *srow = S + row * Dk;
    const T *kh = k + head * Dk;
    const T *qh = q + head * Dk;
    float sk = 0.f, sq = 0.f, kq = 0.f, kk2 = 0.f, qq2 = 0.f;
    for (int c = lane; c < Dk; c += 32) {
        const float s = srow[c], kc = to_f32(kh[c]), qc = to_f32(qh[c]);
        sk += s * kc;
        sq += s * qc;
        kq += kc * qc;
        kk2 += kc * kc;
        qq2 += qc * qc;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        sk += __shfl_xor_sync(0xffffffffu, sk, off);
        sq += __shfl_xor_sync(0xffffffffu, sq, off);
        kq += __shfl_xor_sync(0xffffffffu, kq, off);
        kk2 += __shfl_xor_sync(0xffffffffu, kk2, off);
        qq2 += __shfl_xor_sync(0xffffffffu, qq2, off);
    }
    const float rk = (flags & kFlagL2Norm) ? rsqrtf(kk2 + kNormEps) : 1.f;
    const float rq = (flags & kFlagL2Norm) ? rsqrtf(qq2 + kNormEps) : 1.f;
    const float2 gp = gate_pair(log_alpha[head], beta[head], flags);
    const float alpha = expf(gp.x);
    const int i = (int)(row - head * Dv);
    const float u = gp.y * (to_f32(v[head * Dv + i]) - alpha * rk * sk);
    const float uk = u * rk;
    for (int c = lane; c < Dk; c += 32) srow[c] = alpha * srow[c] + uk * to_f32(kh[c]);
    if (lane == 0) o[head * Dv + i] = from_f32<T>(rq * (alpha * sq + uk * kq));
}

template <typename T>
static cudaError_t launch_decode_t(const void *q, const void *k, const void *v,
                                   const float *la, const float *beta, float *S, void *o,
                                   int B, int H, int Dk, int Dv, unsigned flags,
                                   cudaStream_t st) {
    const long long n_rows = (long long)B * H * Dv;
    const T *qq = static_cast<const T *>(q);
    const T *kk = static_cast<const T *>(k);
    const T *vv = static_cast<const T *>(v);
    T *oo = static_cast<T *>(o);
    const int threads = 256;
    auto blocks_for = [&](long long lanes_per_row) {
        return (unsigned)((n_rows * lanes_per_row + threads - 1) / threads);
    };
    switch (Dk) {
#define GDN_DECODE_VEC(LANES)                                                              \
    case 16 * LANES:                                                                       \
        decode_rows_vec<T, LANES><<<blocks_for(LANES), threads, 0, st>>>(                  \
            qq, kk, vv, la, beta, S, oo, n_rows, Dv, flags);                               \
        break;
        GDN_DECODE_VEC(1)
        GDN_DECODE_VEC(2)
        GDN_DECODE_VEC(4)
        GDN_DECODE_VEC(8)
        GDN_DECODE_VEC(16)
#undef GDN_DECODE_VEC
        default:
            decode_rows_warp<T><<<blocks_for(32), threads, 0, st>>>(qq, kk, vv, la, beta, S, oo,
                                                                  n_rows, Dk, Dv, flags);
    }
    return cudaPeekAtLastError();
}

cudaError_t launch_decode(const void *q, const void *k, const void *v, const float *la,
                          const float *beta, float *S, void *o, int B, int H, int Dk, int Dv,
                          bool bf16, unsigned flags, cudaStream_t st) {
    return bf16 ? launch_decode_t<__nv_bfloat16>(q, k, v, la, beta, S, o, B, H, Dk, Dv, flags, st)
                : launch_decode_t<float>(q, k, v, la, beta, S, o, B, H, Dk, Dv, flags, st);
}

}  // namespace gdn
