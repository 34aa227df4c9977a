// CUDA-core chunkwise forward of the gated delta rule, for every supported size
// and both element types (the float32 path, and bf16 sizes the fused tensor-core
// kernel does not take).  Arithmetic is float32 throughout.
//
// Chunk algebra (a chunk of C tokens, rows r; g_r = running sum of log alpha from
// the chunk start; Gamma_ri = exp(g_r - g_i) for i <= r; S the incoming state):
//   A  = strictly-lower( diag(beta) (Gamma o K K^T) )
//   T  = (I + A)^-1                         (the UT transform of the WY form)
//   P  = Q K^T o Gamma o [i <= r],   P' = P T
//   R  = diag(beta) (V - diag(exp g) K S^T)
//   U  = T R                                (corrected values)
//   O  = diag(exp g) Q S^T + P' R
//   S <- exp(g_last) S + U^T diag(exp(g_last - g)) K
// This is the gated WY/UT chunkwise form named in "Gated Delta Networks:
// Improving Mamba2 with Delta Rule" (section "Approach") and "Gated DeltaNet:
// Harmonizing Gating and the Delta Rule ..." (section "Hardware-Efficient
// Training"), written out with the state applied through T instead of through
// separately stored W = T diag(beta exp g) K (so U = T diag(beta) V - W S^T).
// Rows past the end of a ragged last chunk are zero tokens with beta = 0 and
// log alpha = 0, which leaves every quantity of the real rows unchanged.
//
// Two kernels: chunk_prep (one CTA per chunk, all chunks in parallel) writes
// T, P' and g to the workspace; chunk_state (one CTA per head and slice of
// value channels) runs the chunks of its head in order with its slice of S in
// shared memory.
#include "common.cuh"
#include "kernels.h"

namespace gdn {

__host__ __device__ inline size_t per_chunk_floats(int C) { return 2 * (size_t)C * C + C; }

// Both kernels run one CTA per SM (shared memory); 16 warps hide more of their
// shared-memory latency than 8.
constexpr int kSeqThreads = 512;

size_t simt_workspace_bytes(int B, int T, int H, int C) {
    const size_t NT = ((size_t)T + C - 1) / C;
    return (size_t)B * H * NT * per_chunk_floats(C) * sizeof(float);
}

// kPT: write P' = P T (the forward's read-out); else P itself (the backward's).
template <typename T, bool kPT>
__global__ void __launch_bounds__(kSeqThreads)
chunk_prep(const T *__restrict__ q, const T *__restrict__ k, const float *__restrict__ la,
           const float *__restrict__ beta, float *__restrict__ ws, int Tlen, int H, int Dk, int C,
           int NT) {
    extern __shared__ float sm[];
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int ldk = Dk + 1;
    float *Ks = sm;                // C x ldk
    float *Qs = Ks + C * ldk;      // C x ldk
    float *A = Qs + C * ldk;       // C x C
    float *Tm = A + C * C;         // C x C
    float *P = Tm + C * C;         // C x C
    float *g = P + C * C;          // C
    float *bt = g + C;             // C
    const int t0 = c * C;
    const int n = min(C, Tlen - t0);

    for (int idx = threadIdx.x; idx < C * Dk; idx += blockDim.x) {
        const int r = idx / Dk, j = idx - r * Dk;
        float kv = 0.f, qv = 0.f;
        if (r < n) {
            const size_t off = (((size_t)b * Tlen + t0 + r) * H + h) * Dk + j;
            kv = to_f32(k[off]);
            qv = to_f32(q[off]);
        }
        Ks[r * ldk + j] = kv;
        Qs[r * ldk + j] = qv;
    }
    if (threadIdx.x < C) {
        const int r = threadIdx.x;
        const size_t off = ((size_t)b * Tlen + t0 + r) * H + h;
        g[r] = r < n ? la[off] : 0.f;
        bt[r] = r < n ? beta[off] : 0.f;
    }
    __syncthreads();
    if (threadIdx.x == 0) {  // running sum of log alpha within the chunk
        float acc = 0.f;
        for (int r = 0; r < C; ++r) {
            acc += g[r];
            g[r] = acc;
        }
    }
    __syncthreads();

    // gated Gram matrices A (strictly lower) and P (lower, diagonal included)
    for (int idx = threadIdx.x; idx < C * C; idx += blockDim.x) {
        const int r = idx / C, i = idx - r * C;
        float a = 0.f, p = 0.f;
        if (i <= r) {
            float dk = 0.f, dq = 0.f;
            for (int j = 0; j < Dk; ++j) {
                const float ki = Ks[i * ldk + j];
                dk += Ks[r * ldk + j] * ki;
                dq += Qs[r * ldk + j] * ki;
            }
            const float gam = expf(g[r] - g[i]);
            if (i < r) a = bt[r] * gam * dk;
            p = gam * dq;
        }
        A[idx] = a;
        P[idx] = p;
    }
    __syncthreads();

    // T = (I + A)^-1 by forward substitution, one column per thread:
    // T[r][j] = delta_rj - sum_{j <= i < r} A[r][i] T[i][j]
    for (int j = threadIdx.x; j < C; j += blockDim.x) {
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

    float *out = ws + (((size_t)b * H + h) * NT + c) * per_chunk_floats(C);
    for (int idx = threadIdx.x; idx < C * C; idx += blockDim.x) {
        const int r = idx / C, j = idx - r * C;
        float acc = 0.f;  // (P T)[r][j]; both factors lower triangular
        if (kPT)
            for (int i = j; i <= r; ++i) acc += P[r * C + i] * Tm[i * C + j];
        out[idx] = Tm[idx];
        out[C * C + idx] = kPT ? acc : P[idx];
    }
    if (threadIdx.x < C) out[2 * C * C + threadIdx.x] = g[threadIdx.x];
}

template <typename T, int DVT>
__global__ void __launch_bounds__(kSeqThreads)
chunk_state(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
            const float *__restrict__ beta, const float *__restrict__ S0, T *__restrict__ o,
            float *__restrict__ S_T, const float *__restrict__ ws, float *__restrict__ S_hist,
            int Tlen, int H, int Dk, int Dv, int C, int NT) {
    extern __shared__ float sm[];
    const int v0 = blockIdx.x * DVT, h = blockIdx.y, b = blockIdx.z;
    const int nv = min(DVT, Dv - v0);
    const int ldk = Dk + 1, ldv = DVT + 1;
    float *Ss = sm;                   // DVT x ldk : this CTA's rows of S
    float *Ks = Ss + DVT * ldk;       // C x ldk
    float *Qs = Ks + C * ldk;         // C x ldk
    float *Tm = Qs + C * ldk;         // C x C
    float *Pp = Tm + C * C;           // C x C
    float *R = Pp + C * C;            // C x ldv
    float *Xq = R + C * ldv;          // C x ldv
    float *Un = Xq + C * ldv;         // C x ldv
    float *bt = Un + C * ldv;         // C
    float *eg = bt + C;               // C : exp(g_r)
    float *dc = eg + C;               // C : exp(g_last - g_r)
    float *gl = dc + C;               // 1 : exp(g_last)
    const size_t head = (size_t)b * H + h;

    for (int idx = threadIdx.x; idx < DVT * Dk; idx += blockDim.x) {
        const int i = idx / Dk, j = idx - i * Dk;
        Ss[i * ldk + j] = (i < nv && S0) ? S0[(head * Dv + v0 + i) * Dk + j] : 0.f;
    }
    for (int c = 0; c < NT; ++c) {
        const int t0 = c * C, n = min(C, Tlen - t0);
        const float *wsc = ws + (head * NT + c) * per_chunk_floats(C);
        __syncthreads();  // previous chunk has finished with every buffer
        if (S_hist) {     // the state entering chunk c (the backward recomputes it)
            float *dst = S_hist + ((head * NT + c) * Dv + v0) * Dk;
            for (int idx = threadIdx.x; idx < nv * Dk; idx += blockDim.x) {
                const int i = idx / Dk, j = idx - i * Dk;
                dst[idx] = Ss[i * ldk + j];
            }
        }
        for (int idx = threadIdx.x; idx < C * Dk; idx += blockDim.x) {
            const int r = idx / Dk, j = idx - r * Dk;
            float kv = 0.f, qv = 0.f;
            if (r < n) {
                const size_t off = (((size_t)b * Tlen + t0 + r) * H + h) * Dk + j;
                kv = to_f32(k[off]);
                qv = to_f32(q[off]);
            }
            Ks[r * ldk + j] = kv;
            Qs[r * ldk + j] = qv;
        }
        for (int idx = threadIdx.x; idx < C * C; idx += blockDim.x) {
            Tm[idx] = wsc[idx];
            Pp[idx] = wsc[C * C + idx];
        }
        if (threadIdx.x < C) {
            const int r = threadIdx.x;
            const float gr = wsc[2 * C * C + r], glast = wsc[2 * C * C + C - 1];
            bt[r] = r < n ? beta[((size_t)b * Tlen + t0 + r) * H + h] : 0.f;
            eg[r] = expf(gr);
            dc[r] = expf(glast - gr);
            if (r == 0) gl[0] = expf(glast);
        }
        __syncthreads();

        // R = diag(beta)(V - diag(exp g) K S^T),  Xq = diag(exp g) Q S^T
        for (int idx = threadIdx.x; idx < C * DVT; idx += blockDim.x) {
            const int r = idx / DVT, i = idx - r * DVT;
            float xk = 0.f, xq = 0.f;
            for (int j = 0; j < Dk; ++j) {
                const float s = Ss[i * ldk + j];
                xk += Ks[r * ldk + j] * s;
                xq += Qs[r * ldk + j] * s;
            }
            const float vv =
                (r < n && i < nv) ? to_f32(v[(((size_t)b * Tlen + t0 + r) * H + h) * Dv + v0 + i])
                                  : 0.f;
            R[r * ldv + i] = bt[r] * (vv - eg[r] * xk);
            Xq[r * ldv + i] = eg[r] * xq;
        }
        __syncthreads();

        // U = T R,  O = Xq + P' R
        for (int idx = threadIdx.x; idx < C * DVT; idx += blockDim.x) {
            const int r = idx / DVT, i = idx - r * DVT;
            float u = 0.f, y = 0.f;
            for (int m = 0; m <= r; ++m) {
                const float rr = R[m * ldv + i];
                u += Tm[r * C + m] * rr;
                y += Pp[r * C + m] * rr;
            }
            Un[r * ldv + i] = u;
            if (o && r < n && i < nv)
                o[(((size_t)b * Tlen + t0 + r) * H + h) * Dv + v0 + i] =
                    from_f32<T>(Xq[r * ldv + i] + y);
        }
        __syncthreads();

        // S <- exp(g_last) S + U^T diag(exp(g_last - g)) K
        for (int idx = threadIdx.x; idx < DVT * Dk; idx += blockDim.x) {
            const int i = idx / Dk, j = idx - i * Dk;
            float acc = 0.f;
            for (int r = 0; r < C; ++r) acc += Un[r * ldv + i] * dc[r] * Ks[r * ldk + j];
            Ss[i * ldk + j] = gl[0] * Ss[i * ldk + j] + acc;
        }
    }
    __syncthreads();
    if (S_T) {
        for (int idx = threadIdx.x; idx < nv * Dk; idx += blockDim.x) {
            const int i = idx / Dk, j = idx - i * Dk;
            S_T[(head * Dv + v0 + i) * Dk + j] = Ss[i * ldk + j];
        }
    }
}

template <typename T, int DVT>
static cudaError_t launch_simt_t(const void *q, const void *k, const void *v, const float *la,
                                 const float *beta, const float *S0, void *o, float *S_T, int B,
                                 int Tlen, int H, int Dk, int Dv, int C, void *workspace,
                                 cudaStream_t st) {
    const int NT = (Tlen + C - 1) / C;
    float *ws = static_cast<float *>(workspace);
    const size_t smem_prep = (2 * (size_t)C * (Dk + 1) + 3 * (size_t)C * C + 2 * C) * sizeof(float);
    const size_t smem_state = ((size_t)DVT * (Dk + 1) + 2 * (size_t)C * (Dk + 1) +
                               2 * (size_t)C * C + 3 * (size_t)C * (DVT + 1) + 3 * C + 1) *
                              sizeof(float);
    cudaError_t e;
    e = cudaFuncSetAttribute(chunk_prep<T, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem_prep);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(chunk_state<T, DVT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem_state);
    if (e != cudaSuccess) return e;
    chunk_prep<T, true><<<dim3(NT, H, B), kSeqThreads, smem_prep, st>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), la, beta, ws, Tlen, H, Dk, C, NT);
    e = cudaPeekAtLastError();
    if (e != cudaSuccess) return e;
    chunk_state<T, DVT><<<dim3((Dv + DVT - 1) / DVT, H, B), kSeqThreads, smem_state, st>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), beta, S0,
        static_cast<T *>(o), S_T, ws, nullptr, Tlen, H, Dk, Dv, C, NT);
    return cudaPeekAtLastError();
}

// The backward's recomputation: T, P and g of every chunk into ws_prep, and the
// state entering every chunk into S_hist ([B, H, NT, Dv, Dk] float32).
template <typename T, int DVT>
static cudaError_t launch_recompute_t(const void *q, const void *k, const void *v,
                                      const float *la, const float *beta, const float *S0,
                                      int B, int Tlen, int H, int Dk, int Dv, int C,
                                      float *ws_prep, float *S_hist, cudaStream_t st) {
    const int NT = (Tlen + C - 1) / C;
    const size_t smem_prep = (2 * (size_t)C * (Dk + 1) + 3 * (size_t)C * C + 2 * C) * sizeof(float);
    const size_t smem_state = ((size_t)DVT * (Dk + 1) + 2 * (size_t)C * (Dk + 1) +
                               2 * (size_t)C * C + 3 * (size_t)C * (DVT + 1) + 3 * C + 1) *
                              sizeof(float);
    cudaError_t e;
    e = cudaFuncSetAttribute(chunk_prep<T, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem_prep);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(chunk_state<T, DVT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem_state);
    if (e != cudaSuccess) return e;
    chunk_prep<T, false><<<dim3(NT, H, B), kSeqThreads, smem_prep, st>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), la, beta, ws_prep, Tlen, H, Dk, C,
        NT);
    e = cudaPeekAtLastError();
    if (e != cudaSuccess || !S_hist) return e;
    chunk_state<T, DVT><<<dim3((Dv + DVT - 1) / DVT, H, B), kSeqThreads, smem_state, st>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), beta, S0,
        nullptr, nullptr, ws_prep, S_hist, Tlen, H, Dk, Dv, C, NT);
    return cudaPeekAtLastError();
}

cudaError_t launch_bwd_recompute(const void *q, const void *k, const void *v, const float *la,
                                 const float *beta, const float *S0, int B, int T, int H, int Dk,
                                 int Dv, int chunk, bool bf16, float *ws_prep, float *S_hist,
                                 cudaStream_t st) {
    if (Dk > 128)
        return bf16 ? launch_recompute_t<__nv_bfloat16, 16>(q, k, v, la, beta, S0, B, T, H, Dk,
                                                            Dv, chunk, ws_prep, S_hist, st)
                    : launch_recompute_t<float, 16>(q, k, v, la, beta, S0, B, T, H, Dk, Dv, chunk,
                                                    ws_prep, S_hist, st);
    return bf16 ? launch_recompute_t<__nv_bfloat16, 64>(q, k, v, la, beta, S0, B, T, H, Dk, Dv,
                                                        chunk, ws_prep, S_hist, st)
                : launch_recompute_t<float, 64>(q, k, v, la, beta, S0, B, T, H, Dk, Dv, chunk,
                                                ws_prep, S_hist, st);
}

cudaError_t launch_chunk_simt(const void *q, const void *k, const void *v, const float *la,
                              const float *beta, const float *S0, void *o, float *S_T, int B,
                              int T, int H, int Dk, int Dv, int chunk, bool bf16, void *workspace,
                              cudaStream_t st) {
    // 64 value rows per CTA for Dk <= 128 (one CTA per SM by shared memory, about
    // 182 KB at C = 64: fewer, busier CTAs, one wave for B H Dv / 64 <= 148);
    // narrower slices for wide keys keep the footprint under the per-CTA limit
    // (Dk = 256, C = 64: about 195 KB).
    if (Dk > 128)
        return bf16 ? launch_simt_t<__nv_bfloat16, 16>(q, k, v, la, beta, S0, o, S_T, B, T, H, Dk,
                                                       Dv, chunk, workspace, st)
                    : launch_simt_t<float, 16>(q, k, v, la, beta, S0, o, S_T, B, T, H, Dk, Dv,
                                               chunk, workspace, st);
    return bf16 ? launch_simt_t<__nv_bfloat16, 64>(q, k, v, la, beta, S0, o, S_T, B, T, H, Dk, Dv,
                                                   chunk, workspace, st)
                : launch_simt_t<float, 64>(q, k, v, la, beta, S0, o, S_T, B, T, H, Dk, Dv, chunk,
                                           workspace, st);
}

}  // namespace gdn
