// Channel-wise gates (the Gated DeltaNet-2 form of "Gated DeltaNet-2:
// Decoupling Erase and Write in Linear Attention", abstract): a decay per key
// channel, an erase gate on the key side and a write gate on the value side,
//   S_t = S_{t-1} Diag(alpha_t) (I - (b_t o k_t) k_t^T) + (w_t o v_t) k_t^T,  o_t = S_t q_t
// (one rank-one edit per token; the scalar rule when alpha, b and w collapse to
// alpha, beta, beta).  CUDA cores, float32 arithmetic, Dk <= 128.
//
// Chunk algebra (rows r, i of a chunk of C tokens; Lam_r = running sum of
// log alpha_r over the chunk, a vector over the key channels; S the incoming
// state).  The decay between two rows is channel-wise, so it cannot be pulled
// out of the key products as in the scalar case; it enters every product as
// exp(Lam_r - Lam_i) <= 1 per channel (the asymmetric erase factors):
//   A_ri = sum_j b_rj k_rj k_ij exp(Lam_rj - Lam_ij)   (i < r)
//   P_ri = sum_j q_rj k_ij exp(Lam_rj - Lam_ij)        (i <= r)
//   T    = (I + A)^-1,  P' = P T
//   R    = w o V - (b o K o exp(Lam)) S^T
//   U    = T R,   O = (Q o exp(Lam)) S^T + P' R
//   S   <- S Diag(exp(Lam_last)) + U^T (K o exp(Lam_last - Lam))
// Rows past a ragged end are zero tokens (k = q = b = w = 0, log alpha = 0).
//
// Kernels: cw_prep (one CTA per chunk) writes T, P' and Lam; cw_state (one CTA
// per head and 64 value channels) runs the chunks in order with its slice of S
// in shared memory; decode_cw is the single-token step, one warp per state row.
#include "common.cuh"
#include "kernels.h"

namespace gdn {

namespace {

constexpr int kThreads = 256;
// The chunk kernels (prep and the sequential pass) run one CTA per SM; 16 warps
// hide more of their shared-memory latency than 8.
constexpr int kSeqThreads = 512;

__host__ __device__ inline size_t cw_chunk_floats(int C, int Dk) {
    return 2 * (size_t)C * C + (size_t)C * Dk;
}

template <typename T>
__global__ void __launch_bounds__(kSeqThreads)
cw_prep(const T *__restrict__ q, const T *__restrict__ k, const float *__restrict__ la,
        const float *__restrict__ bg, float *__restrict__ ws, int Tlen, int H, int Dk, int C,
        int NT) {
    extern __shared__ float sm[];
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int ldk = Dk + 1;
    float *Ks = sm;                // C x ldk
    float *Qs = Ks + C * ldk;      // C x ldk
    float *BK = Qs + C * ldk;      // C x ldk : b o k
    float *Lm = BK + C * ldk;      // C x ldk : running sum of log alpha
    float *A = Lm + C * ldk;       // C x C
    float *Tm = A + C * C;         // C x C
    float *P = Tm + C * C;         // C x C
    const int t0 = c * C, n = min(C, Tlen - t0);
    const size_t tok = (size_t)b * Tlen + t0;

    for (int idx = threadIdx.x; idx < C * Dk; idx += kSeqThreads) {
        const int r = idx / Dk, j = idx - r * Dk;
        float kv = 0.f, qv = 0.f, bv = 0.f, lv = 0.f;
        if (r < n) {
            const size_t off = ((tok + r) * H + h) * Dk + j;
            kv = to_f32(k[off]);
            qv = to_f32(q[off]);
            bv = bg[off];
            lv = la[off];
        }
        Ks[r * ldk + j] = kv;
        Qs[r * ldk + j] = qv;
        BK[r * ldk + j] = bv * kv;
        Lm[r * ldk + j] = lv;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < Dk; j += kSeqThreads) {  // running sums, one channel per thread
        float acc = 0.f;
        for (int r = 0; r < C; ++r) {
            acc += Lm[r * ldk + j];
            Lm[r * ldk + j] = acc;
        }
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < C * C; idx += kSeqThreads) {
        const int r = idx / C, i = idx - r * C;
        float a = 0.f, p = 0.f;
        if (i <= r) {
            for (int j = 0; j < Dk; ++j) {
                const float e = expf(Lm[r * ldk + j] - Lm[i * ldk + j]) * Ks[i * ldk + j];
                a += BK[r * ldk + j] * e;
                p += Qs[r * ldk + j] * e;
            }
            if (i == r) a = 0.f;
        }
        A[idx] = a;
        P[idx] = p;
    }
    __syncthreads();
    // T = (I + A)^-1 by forward substitution, one column per thread
    for (int j = threadIdx.x; j < C; j += kSeqThreads) {
        for (int r = 0; r < C; ++r) {
            float val = (r == j) ? 1.f : 0.f;
            if (r > j) {
                float acc = 0.f;
                for (int i = j; i < r; ++i) acc += A[r * C + i] * Tm[i * C + j];
                val = -acc;
            }
            Tm[r * C + j] = val;
        }
    }
    __syncthreads();
    float *out = ws + (((size_t)b * H + h) * NT + c) * cw_chunk_floats(C, Dk);
    for (int idx = threadIdx.x; idx < C * C; idx += kSeqThreads) {
        const int r = idx / C, j = idx - r * C;
        float acc = 0.f;  // (P T)[r][j]
        for (int i = j; i <= r; ++i) acc += P[r * C + i] * Tm[i * C + j];
        out[idx] = Tm[idx];
        out[C * C + idx] = acc;
    }
    for (int idx = threadIdx.x; idx < C * Dk; idx += kSeqThreads) {
        const int r = idx / Dk, j = idx - r * Dk;
        out[2 * C * C + idx] = Lm[r * ldk + j];
    }
}

template <typename T, int DVT>
__global__ void __launch_bounds__(kSeqThreads)
cw_state(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
         const float *__restrict__ bg, const float *__restrict__ wg, const float *__restrict__ S0,
         T *__restrict__ o, float *__restrict__ S_T, const float *__restrict__ ws, int Tlen, int H,
         int Dk, int Dv, int C, int NT) {
    extern __shared__ float sm[];
    const int v0 = blockIdx.x * DVT, h = blockIdx.y, b = blockIdx.z;
    const int nv = min(DVT, Dv - v0);
    const int ldk = Dk + 1, ldv = DVT + 1;
    float *Ss = sm;                 // DVT x ldk : this CTA's rows of S
    float *QL = Ss + DVT * ldk;     // C x ldk : q o exp(Lam)
    float *BL = QL + C * ldk;       // C x ldk : b o k o exp(Lam)
    float *KD = BL + C * ldk;       // C x ldk : k o exp(Lam_last - Lam)
    float *Tm = KD + C * ldk;       // C x C
    float *Pp = Tm + C * C;         // C x C : P T
    float *R = Pp + C * C;          // C x ldv
    float *Xq = R + C * ldv;        // C x ldv
    float *Un = Xq + C * ldv;       // C x ldv
    float *ln = Un + C * ldv;       // Dk : exp(Lam_last)
    const size_t head = (size_t)b * H + h;

    for (int idx = threadIdx.x; idx < DVT * Dk; idx += kSeqThreads) {
        const int i = idx / Dk, j = idx - i * Dk;
        Ss[i * ldk + j] = (i < nv && S0) ? S0[(head * Dv + v0 + i) * Dk + j] : 0.f;
    }
    for (int c = 0; c < NT; ++c) {
        const int t0 = c * C, n = min(C, Tlen - t0);
        const size_t tok = (size_t)b * Tlen + t0;
        const float *wsc = ws + (head * NT + c) * cw_chunk_floats(C, Dk);
        const float *Lam = wsc + 2 * C * C;
        __syncthreads();  // the previous chunk has finished with every buffer
        for (int idx = threadIdx.x; idx < C * Dk; idx += kSeqThreads) {
            const int r = idx / Dk, j = idx - r * Dk;
            float kv = 0.f, qv = 0.f, bv = 0.f;
            if (r < n) {
                const size_t off = ((tok + r) * H + h) * Dk + j;
                kv = to_f32(k[off]);
                qv = to_f32(q[off]);
                bv = bg[off];
            }
            const float lr = Lam[idx], ll = Lam[(C - 1) * Dk + j];
            const float er = expf(lr);
            QL[r * ldk + j] = qv * er;
            BL[r * ldk + j] = bv * kv * er;
            KD[r * ldk + j] = kv * expf(ll - lr);
            if (r == 0) ln[j] = expf(ll);
        }
        for (int idx = threadIdx.x; idx < C * C; idx += kSeqThreads) {
            Tm[idx] = wsc[idx];
            Pp[idx] = wsc[C * C + idx];
        }
        __syncthreads();
        // R = w o V - BL S^T,  Xq = QL S^T
        for (int idx = threadIdx.x; idx < C * DVT; idx += kSeqThreads) {
            const int r = idx / DVT, i = idx - r * DVT;
            float xb = 0.f, xq = 0.f;
            for (int j = 0; j < Dk; ++j) {
                const float s = Ss[i * ldk + j];
                xb += BL[r * ldk + j] * s;
                xq += QL[r * ldk + j] * s;
            }
            float wv = 0.f;
            if (r < n && i < nv) {
                const size_t off = ((tok + r) * H + h) * Dv + v0 + i;
                wv = wg[off] * to_f32(v[off]);
            }
            R[r * ldv + i] = wv - xb;
            Xq[r * ldv + i] = xq;
        }
        __syncthreads();
        // U = T R,  O = Xq + P' R
        for (int idx = threadIdx.x; idx < C * DVT; idx += kSeqThreads) {
            const int r = idx / DVT, i = idx - r * DVT;
            float u = 0.f, y = 0.f;
            for (int m = 0; m <= r; ++m) {
                const float rr = R[m * ldv + i];
                u += Tm[r * C + m] * rr;
                y += Pp[r * C + m] * rr;
            }
            Un[r * ldv + i] = u;
            if (r < n && i < nv)
                o[((tok + r) * H + h) * Dv + v0 + i] = from_f32<T>(Xq[r * ldv + i] + y);
        }
        __syncthreads();
        // S <- S Diag(exp(Lam_last)) + U^T KD
        for (int idx = threadIdx.x; idx < DVT * Dk; idx += kSeqThreads) {
            const int i = idx / Dk, j = idx - i * Dk;
            float acc = 0.f;
            for (int r = 0; r < C; ++r) acc += Un[r * ldv + i] * KD[r * ldk + j];
            Ss[i * ldk + j] = ln[j] * Ss[i * ldk + j] + acc;
        }
    }
    __syncthreads();
    if (S_T) {
        for (int idx = threadIdx.x; idx < nv * Dk; idx += kSeqThreads) {
            const int i = idx / Dk, j = idx - i * Dk;
            S_T[(head * Dv + v0 + i) * Dk + j] = Ss[i * ldk + j];
        }
    }
}

// One token for every (b, h): one warp per state row i (Dk channels), lanes
// striding over the channels; the row is read and written once.
template <typename T>
__global__ void __launch_bounds__(kThreads)
decode_cw(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
          const float *__restrict__ la, const float *__restrict__ bg, const float *__restrict__ wg,
          float *__restrict__ S, T *__restrict__ o, long long rows, int Dk, int Dv) {
    const long long row = ((long long)blockIdx.x * kThreads + threadIdx.x) / 32;
    const int lane = threadIdx.x % 32;
    if (row >= rows) return;  // whole warp leaves together
    const long long head = row / Dv;
    const int i = (int)(row - head * Dv);
    float *s = S + row * Dk;
    const T *qh = q + head * Dk, *kh = k + head * Dk;
    const float *lh = la + head * Dk, *bh = bg + head * Dk;
    float e = 0.f;
    for (int j = lane; j < Dk; j += 32) {
        const float d = expf(lh[j]) * s[j];
        s[j] = d;  // decayed, rewritten below
        e += d * bh[j] * to_f32(kh[j]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) e += __shfl_xor_sync(0xffffffffu, e, off);
    const float wv = wg[head * Dv + i] * to_f32(v[head * Dv + i]);
    float acc = 0.f;
    for (int j = lane; j < Dk; j += 32) {
        const float kj = to_f32(kh[j]);
        const float x = s[j] + (wv - e) * kj;
        s[j] = x;
        acc += x * to_f32(qh[j]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) o[row] = from_f32<T>(acc);
}

// The same step with the row in registers: NPL = Dk / 32 consecutive channels
// per lane (16-byte accesses), ROWS rows of one head per warp so that the
// head's gates are loaded once per warp.  The state row is read and written once.
template <typename T, int NPL, int ROWS>
__global__ void __launch_bounds__(kThreads)
decode_cw_vec(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
              const float *__restrict__ la, const float *__restrict__ bg,
              const float *__restrict__ wg, float *__restrict__ S, T *__restrict__ o,
              long long rows, int Dv) {
    constexpr int Dk = 32 * NPL;
    const long long row0 = (((long long)blockIdx.x * kThreads + threadIdx.x) / 32) * ROWS;
    const int lane = threadIdx.x % 32;
    if (row0 >= rows) return;  // whole warp leaves together (rows is a multiple of ROWS)
    const long long head = row0 / Dv;
    const int j0 = lane * NPL;
    float al[NPL], bk[NPL], kk[NPL], qq[NPL];
#pragma unroll
    for (int m = 0; m < NPL; m += 4) {
        const float4 l4 = load4(la + head * Dk + j0 + m), b4 = load4(bg + head * Dk + j0 + m);
        const float4 k4 = load4(k + head * Dk + j0 + m), q4 = load4(q + head * Dk + j0 + m);
        const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, bv[4] = {b4.x, b4.y, b4.z, b4.w};
        const float kv[4] = {k4.x, k4.y, k4.z, k4.w}, qv[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            al[m + u] = expf(lv[u]);
            kk[m + u] = kv[u];
            bk[m + u] = bv[u] * kv[u];
            qq[m + u] = qv[u];
        }
    }
    // o_i = (alpha o S_i + c_i k) . q = (alpha o S_i) . q + c_i (k . q): both of a
    // row's sums come from the row as read, and the rows' reductions interleave
    float kq = 0.f;
#pragma unroll
    for (int m = 0; m < NPL; ++m) kq += kk[m] * qq[m];
    float4 sv[ROWS][NPL / 4];
#pragma unroll
    for (int rr = 0; rr < ROWS; ++rr) {
        const float *s = S + (row0 + rr) * Dk + j0;
#pragma unroll
        for (int m = 0; m < NPL; m += 4) sv[rr][m / 4] = *reinterpret_cast<const float4 *>(s + m);
    }
    float e[ROWS], sq[ROWS];
#pragma unroll
    for (int rr = 0; rr < ROWS; ++rr) {
        e[rr] = 0.f;
        sq[rr] = 0.f;
#pragma unroll
        for (int m = 0; m < NPL; m += 4) {
            const float a[4] = {al[m] * sv[rr][m / 4].x, al[m + 1] * sv[rr][m / 4].y,
                                al[m + 2] * sv[rr][m / 4].z, al[m + 3] * sv[rr][m / 4].w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                e[rr] += a[u] * bk[m + u];
                sq[rr] += a[u] * qq[m + u];
            }
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        kq += __shfl_xor_sync(0xffffffffu, kq, off);
#pragma unroll
        for (int rr = 0; rr < ROWS; ++rr) {
            e[rr] += __shfl_xor_sync(0xffffffffu, e[rr], off);
            sq[rr] += __shfl_xor_sync(0xffffffffu, sq[rr], off);
        }
    }
#pragma unroll
    for (int rr = 0; rr < ROWS; ++rr) {
        const long long row = row0 + rr;
        const int i = (int)(row - head * Dv);
        const float c = wg[head * Dv + i] * to_f32(v[head * Dv + i]) - e[rr];
        float *s = S + row * Dk + j0;
#pragma unroll
        for (int m = 0; m < NPL; m += 4)
            *reinterpret_cast<float4 *>(s + m) =
                make_float4(al[m] * sv[rr][m / 4].x + c * kk[m], al[m + 1] * sv[rr][m / 4].y + c * kk[m + 1],
                            al[m + 2] * sv[rr][m / 4].z + c * kk[m + 2],
                            al[m + 3] * sv[rr][m / 4].w + c * kk[m + 3]);
        if (lane == 0) o[row] = from_f32<T>(sq[rr] + c * kq);
    }
}

template <typename T>
cudaError_t launch_cw_t(const void *q, const void *k, const void *v, const float *la,
                        const float *bg, const float *wg, const float *S0, void *o, float *S_T,
                        int B, int Tlen, int H, int Dk, int Dv, int C, void *workspace,
                        cudaStream_t st) {
    constexpr int DVT = 64;  // one CTA per SM (shared memory): fewer, busier CTAs
    const int NT = (Tlen + C - 1) / C;
    float *ws = static_cast<float *>(workspace);
    const size_t smem_prep = (4 * (size_t)C * (Dk + 1) + 3 * (size_t)C * C) * sizeof(float);
    const size_t smem_state = ((size_t)DVT * (Dk + 1) + 3 * (size_t)C * (Dk + 1) +
                               2 * (size_t)C * C + 3 * (size_t)C * (DVT + 1) + Dk) *
                              sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(cw_prep<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem_prep);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(cw_state<T, DVT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem_state);
    if (e != cudaSuccess) return e;
    cw_prep<T><<<dim3(NT, H, B), kSeqThreads, smem_prep, st>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), la, bg, ws, Tlen, H, Dk, C, NT);
    e = cudaPeekAtLastError();
    if (e != cudaSuccess) return e;
    cw_state<T, DVT><<<dim3((Dv + DVT - 1) / DVT, H, B), kSeqThreads, smem_state, st>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), bg, wg,
        S0, static_cast<T *>(o), S_T, ws, Tlen, H, Dk, Dv, C, NT);
    return cudaPeekAtLastError();
}

}  // namespace

bool cw_supported(int Dk, int chunk) {
    return Dk <= 128 && (chunk == 16 || chunk == 32 || chunk == 64);
}

size_t cw_workspace_bytes(int B, int T, int H, int Dk, int chunk) {
    const size_t NT = ((size_t)T + chunk - 1) / chunk;
    return (size_t)B * H * NT * cw_chunk_floats(chunk, Dk) * sizeof(float);
}

cudaError_t launch_chunk_cw(const void *q, const void *k, const void *v, const float *la,
                            const float *bg, const float *wg, const float *S0, void *o, float *S_T,
                            int B, int T, int H, int Dk, int Dv, int chunk, bool bf16,
                            void *workspace, cudaStream_t st) {
    return bf16 ? launch_cw_t<__nv_bfloat16>(q, k, v, la, bg, wg, S0, o, S_T, B, T, H, Dk, Dv,
                                             chunk, workspace, st)
                : launch_cw_t<float>(q, k, v, la, bg, wg, S0, o, S_T, B, T, H, Dk, Dv, chunk,
                                     workspace, st);
}

cudaError_t launch_decode_cw(const void *q, const void *k, const void *v, const float *la,
                             const float *bg, const float *wg, float *S, void *o, int B, int H,
                             int Dk, int Dv, bool bf16, cudaStream_t st) {
    const long long rows = (long long)B * H * Dv;
    constexpr int ROWS = 4;
    if ((Dk == 128 || Dk == 256) && Dv % ROWS == 0) {
        const long long warps = rows / ROWS;
        const unsigned blocks = (unsigned)((warps * 32 + kThreads - 1) / kThreads);
#define GDN_CW_VEC(TT, NPL)                                                                    \
    decode_cw_vec<TT, NPL, ROWS><<<blocks, kThreads, 0, st>>>(                                  \
        static_cast<const TT *>(q), static_cast<const TT *>(k), static_cast<const TT *>(v), la, \
        bg, wg, S, static_cast<TT *>(o), rows, Dv)
        if (bf16) {
            if (Dk == 128) GDN_CW_VEC(__nv_bfloat16, 4);
            else GDN_CW_VEC(__nv_bfloat16, 8);
        } else {
            if (Dk == 128) GDN_CW_VEC(float, 4);
            else GDN_CW_VEC(float, 8);
        }
#undef GDN_CW_VEC
        return cudaPeekAtLastError();
    }
    const unsigned blocks = (unsigned)((rows * 32 + kThreads - 1) / kThreads);
    if (bf16)
        decode_cw<__nv_bfloat16><<<blocks, kThreads, 0, st>>>(
            static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k),
            static_cast<const __nv_bfloat16 *>(v), la, bg, wg, S,
            static_cast<__nv_bfloat16 *>(o), rows, Dk, Dv);
    else
        decode_cw<float><<<blocks, kThreads, 0, st>>>(
            static_cast<const float *>(q), static_cast<const float *>(k),
            static_cast<const float *>(v), la, bg, wg, S, static_cast<float *>(o), rows, Dk, Dv);
    return cudaPeekAtLastError();
}

}  // namespace gdn
