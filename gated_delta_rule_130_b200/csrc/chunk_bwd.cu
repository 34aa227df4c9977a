// CUDA-core chunkwise backward of the gated delta rule (Dk <= 128, every chunk
// size of the forward, f32 or bf16 inputs, float32 arithmetic).
//
// The parallel training algorithm of "Gated Delta Networks: Improving Mamba2
// with Delta Rule" (section "Approach") and "Gated DeltaNet: Harmonizing Gating
// and the Delta Rule ..." (section "Hardware-Efficient Training") differentiated
// chunk by chunk.  Per chunk (rows r, i; S the state entering it, S' the state
// leaving it; g, Gamma, A, T, W, U, P as in the forward; D = diag(exp(g_n - g)),
// gamma = exp(g), U' = U - W S^T), with dO and dS' = dL/dS' given:
//
//   dU'  = P^T dO + D K dS'^T               Z  = T^T dU'      dV = diag(beta) Z
//   dS   = gamma_n dS' + dO^T diag(gamma) Q - Z^T diag(beta gamma) K   (to the left)
//   dP   = dO U'^T (lower, diagonal included)
//   dQ   = diag(gamma) dO S + (dP o Gamma) K
//   Y    = T^T dW,  dW = -dU' S
//   dA   = strictly-lower( -(Y W^T + Z U^T) )     (the UT transform's adjoint)
//   E    = diag(beta) (dA o Gamma)
//   dK   = (dP o Gamma)^T Q + D U' dS' + diag(beta gamma) Y + E K + E^T K
//   dbeta_r = gamma_r Y_r.k_r + Z_r.v_r + sum_i dA_ri Gamma_ri k_r.k_i
//   dg   = rows of (diag(gamma) dO S o Q), of dP o P (rows minus columns), of
//          beta gamma (Y o K), of dA o A (rows minus columns), minus D (U' o K dS'^T)
//          row sums, plus gamma_n <dS', S> + sum_r D_r U'_r.(K dS'^T)_r on the
//          last row;  dlog alpha = running sum of dg from the chunk's end.
//
// Three steps: the forward's chunk_prep (T, P, g per chunk) and chunk_state
// (the state entering every chunk) recompute what the forward kept on chip;
// bwd_state walks the chunks of each head backwards with its slice of dS in
// shared memory and records dS' per chunk; bwd_grads then forms every input
// gradient of every chunk in parallel.
#include "common.cuh"
#include "kernels.h"

namespace gdn {

namespace {

// The sequential (chunk-walking) kernels run one CTA per SM; 16 warps hide more
// of their shared-memory latency than 8.
constexpr int kSeqThreads = 512;

// Per (b, h, chunk) floats of the recomputed T, P and g.
__host__ __device__ inline size_t prep_floats(int C) { return 2 * (size_t)C * C + C; }

// dS, walked backwards over the chunks of one head, DVT rows per CTA.
template <typename T, int DVT>
__global__ void __launch_bounds__(kSeqThreads)
bwd_state(const T *__restrict__ q, const T *__restrict__ k, const float *__restrict__ beta,
          const T *__restrict__ d_o, const float *__restrict__ dS_T, float *__restrict__ dS0,
          const float *__restrict__ ws_prep, float *__restrict__ dS_hist, int Tlen, int H, int Dk,
          int Dv, int C, int NT) {
    extern __shared__ float sm[];
    const int v0 = blockIdx.x * DVT, h = blockIdx.y, b = blockIdx.z;
    const int nv = min(DVT, Dv - v0);
    const int ldk = Dk + 1, ldv = DVT + 1;
    float *dS = sm;                 // DVT x ldk
    float *Ks = dS + DVT * ldk;     // C x ldk
    float *Qs = Ks + C * ldk;       // C x ldk
    float *Tm = Qs + C * ldk;       // C x C
    float *Pm = Tm + C * C;         // C x C
    float *dO = Pm + C * C;         // C x ldv
    float *dU = dO + C * ldv;       // C x ldv : dU'
    float *Z = dU + C * ldv;        // C x ldv
    float *bg = Z + C * ldv;        // C : beta exp(g)
    float *eg = bg + C;             // C : exp(g)
    float *dc = eg + C;             // C : exp(g_last - g)
    float *gl = dc + C;             // 1 : exp(g_last)
    const size_t head = (size_t)b * H + h;

    for (int idx = threadIdx.x; idx < DVT * Dk; idx += kSeqThreads) {
        const int i = idx / Dk, j = idx - i * Dk;
        dS[i * ldk + j] = (i < nv && dS_T) ? dS_T[(head * Dv + v0 + i) * Dk + j] : 0.f;
    }
    for (int c = NT - 1; c >= 0; --c) {
        const int t0 = c * C, n = min(C, Tlen - t0);
        const float *wsc = ws_prep + (head * NT + c) * prep_floats(C);
        __syncthreads();
        {   // dS' of this chunk (the gradient of the state it hands on)
            float *dst = dS_hist + ((head * NT + c) * Dv + v0) * Dk;
            for (int idx = threadIdx.x; idx < nv * Dk; idx += kSeqThreads) {
                const int i = idx / Dk, j = idx - i * Dk;
                dst[idx] = dS[i * ldk + j];
            }
        }
        for (int idx = threadIdx.x; idx < C * Dk; idx += kSeqThreads) {
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
        for (int idx = threadIdx.x; idx < C * C; idx += kSeqThreads) {
            Tm[idx] = wsc[idx];
            Pm[idx] = wsc[C * C + idx];
        }
        for (int idx = threadIdx.x; idx < C * DVT; idx += kSeqThreads) {
            const int r = idx / DVT, i = idx - r * DVT;
            dO[r * ldv + i] = (r < n && i < nv)
                                  ? to_f32(d_o[(((size_t)b * Tlen + t0 + r) * H + h) * Dv + v0 + i])
                                  : 0.f;
        }
        if (threadIdx.x < C) {
            const int r = threadIdx.x;
            const float gr = wsc[2 * C * C + r], glast = wsc[2 * C * C + C - 1];
            const float bt = r < n ? beta[((size_t)b * Tlen + t0 + r) * H + h] : 0.f;
            eg[r] = expf(gr);
            bg[r] = bt * eg[r];
            dc[r] = expf(glast - gr);
            if (r == 0) gl[0] = expf(glast);
        }
        __syncthreads();

        // dU' = P^T dO + D K dS^T
        for (int idx = threadIdx.x; idx < C * DVT; idx += kSeqThreads) {
            const int r = idx / DVT, i = idx - r * DVT;
            float a = 0.f, kd = 0.f;
            for (int m = r; m < C; ++m) a += Pm[m * C + r] * dO[m * ldv + i];
            for (int j = 0; j < Dk; ++j) kd += Ks[r * ldk + j] * dS[i * ldk + j];
            dU[r * ldv + i] = a + dc[r] * kd;
        }
        __syncthreads();
        // Z = T^T dU'
        for (int idx = threadIdx.x; idx < C * DVT; idx += kSeqThreads) {
            const int r = idx / DVT, i = idx - r * DVT;
            float a = 0.f;
            for (int m = r; m < C; ++m) a += Tm[m * C + r] * dU[m * ldv + i];
            Z[r * ldv + i] = a;
        }
        __syncthreads();
        // dS <- exp(g_last) dS + dO^T diag(exp g) Q - Z^T diag(beta exp g) K
        for (int idx = threadIdx.x; idx < DVT * Dk; idx += kSeqThreads) {
            const int i = idx / Dk, j = idx - i * Dk;
            float a = 0.f;
            for (int r = 0; r < C; ++r)
                a += dO[r * ldv + i] * eg[r] * Qs[r * ldk + j] - Z[r * ldv + i] * bg[r] * Ks[r * ldk + j];
            dS[i * ldk + j] = gl[0] * dS[i * ldk + j] + a;
        }
    }
    __syncthreads();
    if (dS0) {
        for (int idx = threadIdx.x; idx < nv * Dk; idx += kSeqThreads) {
            const int i = idx / Dk, j = idx - i * Dk;
            dS0[(head * Dv + v0 + i) * Dk + j] = dS[i * ldk + j];
        }
    }
}

template <int DVT>
constexpr size_t bwd_state_smem_floats(int C, int Dk) {
    return (size_t)DVT * (Dk + 1) + 2 * (size_t)C * (Dk + 1) + 2 * (size_t)C * C +
           3 * (size_t)C * (DVT + 1) + 3 * C + 1;
}

constexpr int DVS = 16;        // value channels per pass of bwd_grads
constexpr int kGradThreads = 512;
constexpr int kMaxCols = 16;   // key channels per thread: Dk / (kGradThreads / C) <= 128 / 8
static_assert(kGradThreads / 16 <= 32, "a row's threads share one warp (C >= 16)");

__host__ __device__ constexpr int region_floats(int C, int Dk) {
    return (2 * DVS * (Dk + 1) + 7 * C * (DVS + 1)) > C * (Dk + 1)
               ? 2 * DVS * (Dk + 1) + 7 * C * (DVS + 1)
               : C * (Dk + 1);
}

__host__ __device__ constexpr size_t bwd_grads_smem_floats(int C, int Dk) {
    return 3 * (size_t)C * (Dk + 1) + 2 * (size_t)C * C + 2 * (size_t)C * (C + 1) +
           region_floats(C, Dk) + 8 * (size_t)C + 2;
}

// The t-th element (row-major) of the lower triangle with the diagonal:
// r (r + 1) / 2 <= t < (r + 1) (r + 2) / 2, i = t - r (r + 1) / 2.
__device__ __forceinline__ void lower_incl(int t, int &r, int &i) {
    int rr = (int)((sqrtf(8.f * (float)t + 1.f) - 1.f) * 0.5f);
    while (rr * (rr + 1) / 2 > t) --rr;
    while ((rr + 1) * (rr + 2) / 2 <= t) ++rr;
    r = rr;
    i = t - rr * (rr + 1) / 2;
}

// Every input gradient of one chunk of one head.  The thread layout for the
// C x Dk results: kGradThreads / C consecutive threads share a row, each owning
// the key channels j = sub, sub + kGradThreads / C, ...
template <typename T>
__global__ void __launch_bounds__(kGradThreads)
bwd_grads(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
          const float *__restrict__ beta, const T *__restrict__ d_o,
          const float *__restrict__ ws_prep, const float *__restrict__ S_hist,
          const float *__restrict__ dS_hist, T *__restrict__ dq, T *__restrict__ dk,
          T *__restrict__ dv, float *__restrict__ dla, float *__restrict__ dbeta, int Tlen, int H,
          int Dk, int Dv, int C, int NT) {
    extern __shared__ float sm[];
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const size_t head = (size_t)b * H + h;
    const int t0 = c * C, n = min(C, Tlen - t0);
    const int ldk = Dk + 1, lds = DVS + 1;
    float *Qs = sm;                      // C x ldk
    float *Ks = Qs + C * ldk;            // C x ldk
    float *Ws = Ks + C * ldk;            // C x ldk : W = T diag(beta exp g) K
    float *Tm = Ws + C * ldk;            // C x C
    // P (later E) and dP are read along rows by the threads of several rows at
    // once: a row stride of C + 1 keeps those reads on distinct banks
    const int ldc = C + 1;
    float *Pm = Tm + C * C;              // C x ldc : P, later E
    float *dP = Pm + C * ldc;            // C x ldc : dO U'^T, later (dP o Gamma)
    float *ZU = dP + C * ldc;            // C x C : Z U^T
    float *R = ZU + C * C;               // the value-slice buffers, later dW then Y
    float *gv = R + region_floats(C, Dk);  // C : g
    float *eg = gv + C;                  // C : exp(g)
    float *dc = eg + C;                  // C : exp(g_last - g)
    float *bt = dc + C;                  // C : beta
    float *dbv = bt + C;                 // C : sum_v Z V
    float *hv = dbv + C;                 // C : sum_v U' (K dS'^T)
    float *dg = hv + C;                  // C : dL/dg, then dL/dlog alpha
    float *db = dg + C;                  // C : dL/dbeta (Gram and W terms)
    float *misc = db + C;                // [0] <dS', S>, [1] exp(g_last)
    float *Ss = R;                       // DVS x ldk : rows v0.. of S
    float *dSs = Ss + DVS * ldk;         // DVS x ldk : rows v0.. of dS'
    float *Vs = dSs + DVS * ldk;         // C x lds
    float *dOs = Vs + C * lds;
    float *Us = dOs + C * lds;
    float *Ups = Us + C * lds;           // U'
    float *KdS = Ups + C * lds;          // K dS'^T
    float *dUs = KdS + C * lds;          // dU'
    float *Zs = dUs + C * lds;           // T^T dU'
    const float *wsc = ws_prep + (head * NT + c) * prep_floats(C);
    const float *Sc = S_hist + (head * NT + c) * (size_t)Dv * Dk;
    const float *dSc = dS_hist + (head * NT + c) * (size_t)Dv * Dk;
    const int tid = threadIdx.x;
    const int TPR = kGradThreads / C, row = tid / TPR, sub = tid - row * TPR;
    const size_t tok = (size_t)b * Tlen + t0;  // first token of the chunk

    for (int idx = tid; idx < C * Dk; idx += kGradThreads) {
        const int r = idx / Dk, j = idx - r * Dk;
        float kv = 0.f, qv = 0.f;
        if (r < n) {
            const size_t off = ((tok + r) * H + h) * Dk + j;
            kv = to_f32(k[off]);
            qv = to_f32(q[off]);
        }
        Ks[r * ldk + j] = kv;
        Qs[r * ldk + j] = qv;
    }
    for (int idx = tid; idx < C * C; idx += kGradThreads) {
        const int r = idx / C, i = idx - r * C;
        Tm[idx] = wsc[idx];
        Pm[r * ldc + i] = wsc[C * C + idx];
        dP[r * ldc + i] = 0.f;
        ZU[idx] = 0.f;
    }
    if (tid < C) {
        const float gr = wsc[2 * C * C + tid], glast = wsc[2 * C * C + C - 1];
        gv[tid] = gr;
        eg[tid] = expf(gr);
        dc[tid] = expf(glast - gr);
        bt[tid] = tid < n ? beta[(tok + tid) * H + h] : 0.f;
        dbv[tid] = hv[tid] = dg[tid] = db[tid] = 0.f;
        if (tid == 0) {
            misc[0] = 0.f;
            misc[1] = expf(glast);
        }
    }
    __syncthreads();
    for (int idx = tid; idx < C * Dk; idx += kGradThreads) {
        const int r = idx / Dk, j = idx - r * Dk;
        float a = 0.f;
        for (int m = 0; m <= r; ++m) a += Tm[r * C + m] * bt[m] * eg[m] * Ks[m * ldk + j];
        Ws[r * ldk + j] = a;
    }

    float aQ[kMaxCols], aW[kMaxCols], aK[kMaxCols];
#pragma unroll
    for (int m = 0; m < kMaxCols; ++m) aQ[m] = aW[m] = aK[m] = 0.f;

    for (int v0 = 0; v0 < Dv; v0 += DVS) {
        const int nv = min(DVS, Dv - v0);
        for (int idx = tid; idx < DVS * Dk; idx += kGradThreads) {
            const int i = idx / Dk, j = idx - i * Dk;
            Ss[i * ldk + j] = i < nv ? Sc[(size_t)(v0 + i) * Dk + j] : 0.f;
            dSs[i * ldk + j] = i < nv ? dSc[(size_t)(v0 + i) * Dk + j] : 0.f;
        }
        for (int idx = tid; idx < C * DVS; idx += kGradThreads) {
            const int r = idx / DVS, i = idx - r * DVS;
            const bool in = r < n && i < nv;
            const size_t off = ((tok + r) * H + h) * Dv + v0 + i;
            Vs[r * lds + i] = in ? to_f32(v[off]) : 0.f;
            dOs[r * lds + i] = in ? to_f32(d_o[off]) : 0.f;
        }
        __syncthreads();
        // U = T diag(beta) V,  U' = U - W S^T,  K dS'^T
        for (int idx = tid; idx < C * DVS; idx += kGradThreads) {
            const int r = idx / DVS, i = idx - r * DVS;
            float u = 0.f, w = 0.f, kd = 0.f;
            for (int m = 0; m <= r; ++m) u += Tm[r * C + m] * bt[m] * Vs[m * lds + i];
            for (int j = 0; j < Dk; ++j) {
                w += Ws[r * ldk + j] * Ss[i * ldk + j];
                kd += Ks[r * ldk + j] * dSs[i * ldk + j];
            }
            Us[r * lds + i] = u;
            Ups[r * lds + i] = u - w;
            KdS[r * lds + i] = kd;
        }
        __syncthreads();
        // dU' = P^T dO + D K dS'^T
        for (int idx = tid; idx < C * DVS; idx += kGradThreads) {
            const int r = idx / DVS, i = idx - r * DVS;
            float a = 0.f;
            for (int m = r; m < C; ++m) a += Pm[m * ldc + r] * dOs[m * lds + i];
            dUs[r * lds + i] = a + dc[r] * KdS[r * lds + i];
        }
        __syncthreads();
        // Z = T^T dU',  dV = diag(beta) Z
        for (int idx = tid; idx < C * DVS; idx += kGradThreads) {
            const int r = idx / DVS, i = idx - r * DVS;
            float z = 0.f;
            for (int m = r; m < C; ++m) z += Tm[m * C + r] * dUs[m * lds + i];
            Zs[r * lds + i] = z;
            if (r < n && i < nv) dv[((tok + r) * H + h) * Dv + v0 + i] = from_f32<T>(bt[r] * z);
        }
        __syncthreads();
        // this slice's share of dP = dO U'^T, Z U^T and the row and scalar sums
        for (int t = tid; t < C * (C + 1) / 2; t += kGradThreads) {  // i <= r only
            int r, i;
            lower_incl(t, r, i);
            float a = 0.f, z = 0.f;
            for (int u = 0; u < DVS; ++u) {
                a += dOs[r * lds + u] * Ups[i * lds + u];
                z += Zs[r * lds + u] * Us[i * lds + u];
            }
            dP[r * ldc + i] += a;
            if (i < r) ZU[r * C + i] += z;
        }
        if (tid < C) {
            float a = 0.f, e = 0.f;
            for (int u = 0; u < DVS; ++u) {
                a += Zs[tid * lds + u] * Vs[tid * lds + u];
                e += Ups[tid * lds + u] * KdS[tid * lds + u];
            }
            dbv[tid] += a;
            hv[tid] += e;
        }
        {
            float p = 0.f;
            for (int idx = tid; idx < DVS * Dk; idx += kGradThreads) {
                const int i = idx / Dk, j = idx - i * Dk;
                p += Ss[i * ldk + j] * dSs[i * ldk + j];
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
            if ((tid & 31) == 0) atomicAdd(&misc[0], p);
        }
        // the owner's C x Dk sums: dO S, -dU' S, U' dS'
#pragma unroll
        for (int m = 0; m < kMaxCols; ++m) {
            const int j = sub + TPR * m;
            if (j < Dk) {
                float a = 0.f, w = 0.f, e = 0.f;
                for (int u = 0; u < DVS; ++u) {
                    const float s = Ss[u * ldk + j];
                    a += dOs[row * lds + u] * s;
                    w += dUs[row * lds + u] * s;
                    e += Ups[row * lds + u] * dSs[u * ldk + j];
                }
                aQ[m] += a;
                aW[m] -= w;
                aK[m] += e;
            }
        }
        __syncthreads();
    }

    // dQ1 = diag(exp g) dO S and D U' dS'; the first term of dg; dW into R
    const float egr = eg[row], dcr = dc[row], btr = bt[row];
    float *DW = R;  // C x ldk (the slice buffers are no longer needed)
    float q1 = 0.f;
#pragma unroll
    for (int m = 0; m < kMaxCols; ++m) {
        const int j = sub + TPR * m;
        if (j < Dk) {
            aQ[m] *= egr;
            aK[m] *= dcr;
            q1 += aQ[m] * Qs[row * ldk + j];
            DW[row * ldk + j] = aW[m];
        }
    }
    for (int o = TPR / 2; o > 0; o >>= 1) q1 += __shfl_xor_sync(0xffffffffu, q1, o);
    if (sub == 0) atomicAdd(&dg[row], q1);
    __syncthreads();
    // Y = T^T dW (then kept in R in place of dW)
#pragma unroll
    for (int m = 0; m < kMaxCols; ++m) {
        const int j = sub + TPR * m;
        if (j < Dk) {
            float y = 0.f;
            for (int mm = row; mm < C; ++mm) y += Tm[mm * C + row] * DW[mm * ldk + j];
            aW[m] = y;
        }
    }
    __syncthreads();
#pragma unroll
    for (int m = 0; m < kMaxCols; ++m) {
        const int j = sub + TPR * m;
        if (j < Dk) DW[row * ldk + j] = aW[m];
    }
    // the read-out's gating: dg from dP o P, and dP <- dP o Gamma (i <= r; the
    // upper triangle stays zero and is never read)
    for (int t = tid; t < C * (C + 1) / 2; t += kGradThreads) {
        int r, i;
        lower_incl(t, r, i);
        const float dp = dP[r * ldc + i];
        if (i < r) {
            const float dG = dp * Pm[r * ldc + i];
            atomicAdd(&dg[r], dG);
            atomicAdd(&dg[i], -dG);
        }
        dP[r * ldc + i] = dp * expf(gv[r] - gv[i]);
    }
    __syncthreads();
    // dA = strictly-lower(-(Y W^T + Z U^T)); its dg and dbeta terms; E into Pm
    // (i < r only; Pm keeps P elsewhere, which is never read as E)
    for (int t = tid; t < C * (C - 1) / 2; t += kGradThreads) {
        int r, i;
        lower_incl(t, r, i);
        r += 1;  // the strictly lower pairs of C rows are the pairs i <= r of C - 1 rows
        float yw = 0.f, kk = 0.f;
        for (int j = 0; j < Dk; ++j) {
            yw += DW[r * ldk + j] * Ws[i * ldk + j];
            kk += Ks[r * ldk + j] * Ks[i * ldk + j];
        }
        const float da = -(yw + ZU[r * C + i]);
        const float G = expf(gv[r] - gv[i]);
        const float a = bt[r] * G * kk;  // A[r][i]
        atomicAdd(&dg[r], da * a);
        atomicAdd(&dg[i], -da * a);
        atomicAdd(&db[r], da * G * kk);
        Pm[r * ldc + i] = bt[r] * da * G;
    }
    __syncthreads();
    // dQ = dQ1 + (dP o Gamma) K
    // dK = (dP o Gamma)^T Q + D U' dS' + diag(beta exp g) Y + E K + E^T K
    float yk = 0.f;
    const size_t qk_row = ((tok + row) * H + h) * Dk;
#pragma unroll
    for (int m = 0; m < kMaxCols; ++m) {
        const int j = sub + TPR * m;
        if (j < Dk) {
            const float y = DW[row * ldk + j];
            aK[m] += btr * egr * y;
            yk += y * Ks[row * ldk + j];
        }
    }
    // one pass over the chunk rows i: (dP o Gamma) along this row (dQ) and down
    // this column (dK), E along the row and down the column (dK); each matrix
    // element is loaded once for all of the thread's key channels
    for (int i = 0; i < C; ++i) {
        const float pr = i <= row ? dP[row * ldc + i] : 0.f;
        const float pc = i >= row ? dP[i * ldc + row] : 0.f;
        const float e = (i < row ? Pm[row * ldc + i] : 0.f) + (i > row ? Pm[i * ldc + row] : 0.f);
#pragma unroll
        for (int m = 0; m < kMaxCols; ++m) {
            const int j = sub + TPR * m;
            if (j < Dk) {
                const float kij = Ks[i * ldk + j];
                aQ[m] += pr * kij;
                aK[m] += pc * Qs[i * ldk + j] + e * kij;
            }
        }
    }
    if (row < n) {
#pragma unroll
        for (int m = 0; m < kMaxCols; ++m) {
            const int j = sub + TPR * m;
            if (j < Dk) {
                dq[qk_row + j] = from_f32<T>(aQ[m]);
                dk[qk_row + j] = from_f32<T>(aK[m]);
            }
        }
    }
    for (int o = TPR / 2; o > 0; o >>= 1) yk += __shfl_xor_sync(0xffffffffu, yk, o);
    if (sub == 0) {
        atomicAdd(&db[row], egr * yk);
        atomicAdd(&dg[row], btr * egr * yk);
    }
    __syncthreads();
    // the state's terms of dg, then dlog alpha = running sum from the chunk's end
    if (tid == 0) {
        float s = misc[1] * misc[0];
        for (int r = 0; r < C; ++r) {
            const float hr = dc[r] * hv[r];
            dg[r] -= hr;
            s += hr;
        }
        dg[C - 1] += s;
        float acc = 0.f;
        for (int r = C - 1; r >= 0; --r) {
            acc += dg[r];
            dg[r] = acc;
        }
    }
    __syncthreads();
    if (tid < n) {
        dla[(tok + tid) * H + h] = dg[tid];
        dbeta[(tok + tid) * H + h] = db[tid] + dbv[tid];
    }
}

// Workspace: [T, P, g per chunk | S_hist | dS_hist | (tensor-core recompute:
// its tile workspace | a scratch output)].
size_t base_floats(int B, int T, int H, int Dk, int Dv, int C) {
    const size_t NT = ((size_t)T + C - 1) / C;
    return (size_t)B * H * NT * (prep_floats(C) + 2 * (size_t)Dv * Dk);
}

bool tc_recompute(int B, int T, int H, int Dk, int Dv, int C, bool bf16) {
    return tc_supported(B, T, H, Dk, Dv, C, bf16);
}

template <typename T>
cudaError_t launch_bwd_t(const void *q, const void *k, const void *v, const float *la,
                         const float *beta, const float *S0, const void *d_o, const float *dS_T,
                         void *dq, void *dk, void *dv, float *dla, float *dbeta, float *dS0, int B,
                         int Tlen, int H, int Dk, int Dv, int C, void *workspace,
                         cudaStream_t st) {
    constexpr int DVT = 64;  // one CTA per SM (shared memory): fewer, busier CTAs
    const int NT = (Tlen + C - 1) / C;
    float *ws_prep = static_cast<float *>(workspace);
    float *S_hist = ws_prep + (size_t)B * H * NT * prep_floats(C);
    float *dS_hist = S_hist + (size_t)B * H * NT * Dv * Dk;
    const bool bf16 = sizeof(T) == 2;
    cudaError_t e;
    if (tc_recompute(B, Tlen, H, Dk, Dv, C, bf16)) {
        // T, P, g on the CUDA cores; the chunk states from the tensor-core forward
        uint8_t *tail = reinterpret_cast<uint8_t *>(ws_prep + base_floats(B, Tlen, H, Dk, Dv, C));
        void *o_scratch = tail + ((tc_workspace_bytes_fused(B, Tlen, H, 0) + 255) & ~size_t(255));
        e = launch_bwd_recompute(q, k, v, la, beta, S0, B, Tlen, H, Dk, Dv, C, bf16, ws_prep,
                                 nullptr, st);
        if (e != cudaSuccess) return e;
        e = launch_chunk_tc(q, k, v, la, beta, S0, o_scratch, nullptr, B, Tlen, H, Dk, Dv, 0u,
                            tail, st, S_hist);
    } else {
        e = launch_bwd_recompute(q, k, v, la, beta, S0, B, Tlen, H, Dk, Dv, C, bf16, ws_prep,
                                 S_hist, st);
    }
    if (e != cudaSuccess) return e;
    const size_t smem_s = bwd_state_smem_floats<DVT>(C, Dk) * sizeof(float);
    const size_t smem_g = bwd_grads_smem_floats(C, Dk) * sizeof(float);
    e = cudaFuncSetAttribute(bwd_state<T, DVT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem_s);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(bwd_grads<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem_g);
    if (e != cudaSuccess) return e;
    bwd_state<T, DVT><<<dim3((Dv + DVT - 1) / DVT, H, B), kSeqThreads, smem_s, st>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), beta, static_cast<const T *>(d_o),
        dS_T, dS0, ws_prep, dS_hist, Tlen, H, Dk, Dv, C, NT);
    e = cudaPeekAtLastError();
    if (e != cudaSuccess) return e;
    bwd_grads<T><<<dim3(NT, H, B), kGradThreads, smem_g, st>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), beta,
        static_cast<const T *>(d_o), ws_prep, S_hist, dS_hist, static_cast<T *>(dq),
        static_cast<T *>(dk), static_cast<T *>(dv), dla, dbeta, Tlen, H, Dk, Dv, C, NT);
    return cudaPeekAtLastError();
}

}  // namespace

size_t bwd_workspace_bytes(int B, int T, int H, int Dk, int Dv, int chunk, bool bf16) {
    if (bwd_tc_supported(B, T, H, Dk, Dv, chunk, bf16)) return bwd_tc_workspace_bytes(B, T, H, Dv);
    size_t n = base_floats(B, T, H, Dk, Dv, chunk) * sizeof(float);
    if (tc_recompute(B, T, H, Dk, Dv, chunk, bf16))
        n += ((tc_workspace_bytes_fused(B, T, H, 0) + 255) & ~size_t(255)) +
             (size_t)B * T * H * Dv * sizeof(__nv_bfloat16);
    return n;
}

bool bwd_supported(int Dk, int chunk) {
    return Dk <= 128 && (chunk == 16 || chunk == 32 || chunk == 64) &&
           bwd_grads_smem_floats(chunk, Dk) * sizeof(float) <= 227 * 1024;
}

cudaError_t launch_chunk_bwd(const void *q, const void *k, const void *v, const float *la,
                             const float *beta, const float *S0, const void *d_o,
                             const float *dS_T, void *dq, void *dk, void *dv, float *dla,
                             float *dbeta, float *dS0, int B, int T, int H, int Dk, int Dv,
                             int chunk, bool bf16, void *workspace, cudaStream_t st) {
    if (bwd_tc_supported(B, T, H, Dk, Dv, chunk, bf16))
        return launch_chunk_bwd_tc(q, k, v, la, beta, S0, d_o, dS_T, dq, dk, dv, dla, dbeta, dS0, B,
                                   T, H, Dv, workspace, st);
    return bf16 ? launch_bwd_t<__nv_bfloat16>(q, k, v, la, beta, S0, d_o, dS_T, dq, dk, dv, dla,
                                              dbeta, dS0, B, T, H, Dk, Dv, chunk, workspace, st)
                : launch_bwd_t<float>(q, k, v, la, beta, S0, d_o, dS_T, dq, dk, dv, dla, dbeta,
                                      dS0, B, T, H, Dk, Dv, chunk, workspace, st);
}

}  // namespace gdn
