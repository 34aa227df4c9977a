// Channel-wise gates (the Gated DeltaNet-2 reading, "Gated DeltaNet-2:
// Decoupling Erase and Write in Linear Attention", abstract: a decay per key
// channel, an erase gate on the key side and a write gate on the value side,
// "channel-wise decay absorbed into asymmetric erase factors"),
//   S_t = S_{t-1} Diag(alpha_t) (I - (b_t o k_t) k_t^T) + (w_t o v_t) k_t^T,  o_t = S_t q_t,
// on the tensor cores: bf16 q/k/v/o, Dk = 128, chunk 64, Dv a multiple of 64.
//
// Per chunk (rows r, i; Lam_r the running sum of log alpha over the chunk, per
// key channel; S the incoming state):
//   A_ri = sum_j b_rj k_rj k_ij exp(Lam_rj - Lam_ij)   (i < r),   T = (I + A)^-1
//   P_ri = sum_j q_rj k_ij exp(Lam_rj - Lam_ij)        (i <= r)
//   W    = T (b o K o exp(Lam)),   U = T (w o V),   U' = U - W S^T
//   O    = (Q o exp(Lam)) S^T + P U'
//   S   <- S Diag(exp(Lam_last)) + U'^T (K o exp(Lam_last - Lam))
// which is the shape of the scalar precomputed variant (chunk_tc_wide.cu) with
// Q, K and V replaced by Q o exp(Lam), K o exp(Lam_last - Lam) and w o V and the
// state's decay a vector over the key channels.  Two kernels:
//  1. gdn_ut_cw_kernel, one CTA of 16 warps per (chunk, head, batch), all chunks
//     in parallel.  The decays between rows are channel-wise, so they cannot be
//     taken out of the key products as row and column scales; split the chunk
//     into 16-row blocks:
//       - a block I against an earlier block J factors through the reference
//         row m = 16 I - 1 between them: exp(Lam_r - Lam_i) =
//         exp(Lam_r - Lam_m) exp(Lam_m - Lam_i), both factors <= 1 (no overflow
//         for any decay), so A_IJ = L_I R_I,J^T and P_IJ = M_I R_I,J^T with
//         L_I = b o K_I o 2^(Lam_I - Lam_m), M_I = Q_I o 2^(Lam_I - Lam_m),
//         R = K_J o 2^(Lam_m - Lam_J): bf16 mma.sync products of 16-row blocks
//         (the factorisation is per block pair; 16 rows is below the M = 64 of
//         a tcgen05 product);
//       - inside a diagonal block, rows 8-15 against rows 0-7 factor the same
//         way through the block's row 7 (mma.sync); the two 8 x 8 diagonal
//         sub-blocks are summed directly over the channels in float32, the
//         decay from row i to row r as the product of the consecutive-row
//         decays 2^(Lam_{m+1} - Lam_m) <= 1, four warps per block;
//     then the blocked UT solve, W = T (b o K o 2^Lam) (mma.sync), and the
//     operands of the sequential kernel: [P; T''] (T'' = T with the columns of
//     rows past the end zeroed), W, Q o 2^Lam, K o 2^(Lam_last - Lam), w o V
//     and 2^Lam_last per key channel, into the workspace.
//  2. the precomputed variant's sequential tcgen05 kernel in its channel-wise
//     mode (launch_chunk_tcw_seq_cw in chunk_tc_wide.cu).
// Lam is kept in log2 units (exp2 of the hardware approximation).  Rows past a
// ragged end are zero tokens (k = q = b = w = 0, log alpha = 0).
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tc_common.cuh"

namespace gdn {

// Optional phase timeline of two CTAs of the parallel kernel (chunk 0 and chunk
// 63 of head 8, batch 0) for performance work: build with -DGDN_TRACE; that build
// alone exports gdn_trace_cw_read().
#ifdef GDN_TRACE
__device__ unsigned long long g_trace_cw[2 * 16];
#define TCW(ev)                                                                           \
    do {                                                                                  \
        if (threadIdx.x == 0 && blockIdx.z == 0 &&                                        \
            ((blockIdx.x == 0 && blockIdx.y == 0) || (blockIdx.x == 63 && blockIdx.y == 8))) \
            g_trace_cw[(blockIdx.x == 0 ? 0 : 16) + (ev)] = clock64();                    \
    } while (0)
#else
#define TCW(ev) \
    do {        \
    } while (0)
#endif

namespace cwt {

using namespace sm100;
using tc::C;
using tc::LDA;

constexpr int DK = 128;
constexpr int THREADS = 512;                  // 16 warps
constexpr int LDF = DK + 8;                   // float32 row stride of the per-channel arrays:
                                              // 16-byte rows, conflict-free float2 fragments
constexpr int LDT = C + 8;                    // bf16 row stride of T for the W product
constexpr int SM_K = 0;                       // k (f32, 64 x LDF)
constexpr int SM_Q = SM_K + C * LDF * 4;      // q
constexpr int SM_BK = SM_Q + C * LDF * 4;     // b o k
constexpr int SM_LM = SM_BK + C * LDF * 4;    // Lam log2(e) (running sums per channel)
constexpr int SM_AF = SM_LM + C * LDF * 4;    // A (f32, 64 x LDA); then T as bf16
constexpr int SM_TF = SM_AF + C * LDA * 4;    // T (f32)
constexpr int SM_PF = SM_TF + C * LDA * 4;    // P (f32)
constexpr int NPAIR = 72;                     // (r, i), i <= r, of the two 8 x 8 diagonal sub-blocks
constexpr int SM_DS = SM_PF + C * LDA * 4;    // diagonal blocks: channel quarters 1-3 partial sums
constexpr int SMEM = SM_DS + 4 * 3 * NPAIR * 2 * 4;
constexpr int PT_ELEMS = 2 * C * C, W_ELEMS = C * DK;
constexpr float LOG2E = 1.4426950408889634f;
static_assert(SM_AF % 16 == 0 && SM_TF % 16 == 0 && SM_PF % 16 == 0 && SM_DS % 16 == 0,
              "16-byte aligned buffers");
static_assert(SMEM <= 227 * 1024, "shared memory budget");
static_assert(LDF % 4 == 0 && (C * LDF * 4) % 16 == 0, "16-byte rows of the per-channel arrays");

// channels j, j + 1 (j even) of row r of a per-channel array
__device__ __forceinline__ float2 ld2(const float *a, int r, int j) {
    return *reinterpret_cast<const float2 *>(a + r * LDF + j);
}
// channels j .. j + 3 (j a multiple of 4)
__device__ __forceinline__ float4 ld4(const float *a, int r, int j) {
    return *reinterpret_cast<const float4 *>(a + r * LDF + j);
}

__global__ void __launch_bounds__(THREADS, 1)
gdn_ut_cw_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                 const __nv_bfloat16 *__restrict__ v, const float *__restrict__ la,
                 const float *__restrict__ bg, const float *__restrict__ wg,
                 __nv_bfloat16 *__restrict__ qe, __nv_bfloat16 *__restrict__ kd,
                 __nv_bfloat16 *__restrict__ vw, __nv_bfloat16 *__restrict__ pt,
                 __nv_bfloat16 *__restrict__ wt, float *__restrict__ glk, int T, int H, int Dv) {
    extern __shared__ __align__(16) uint8_t sm[];
    // the sequential kernel that follows may be scheduled now (it waits for this
    // grid's completion before it reads what this kernel writes)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int NT = (T + C - 1) / C;
    const int t0 = c * C, n = min(C, T - t0);
    const size_t tok0 = (size_t)b * T + t0;
    const size_t tile = ((size_t)b * NT + c) * H + h;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    float *KF = reinterpret_cast<float *>(sm + SM_K);
    float *QF = reinterpret_cast<float *>(sm + SM_Q);
    float *BK = reinterpret_cast<float *>(sm + SM_BK);
    float *LM = reinterpret_cast<float *>(sm + SM_LM);
    float *AF = reinterpret_cast<float *>(sm + SM_AF);
    float *TF = reinterpret_cast<float *>(sm + SM_TF);
    float *PF = reinterpret_cast<float *>(sm + SM_PF);
    float *DS = reinterpret_cast<float *>(sm + SM_DS);
    __nv_bfloat16 *TB = reinterpret_cast<__nv_bfloat16 *>(sm + SM_AF);
    TCW(0);

    // q, k, b o k and log alpha of the chunk's rows (zero past the end); thread ->
    // (row r, four groups of 4 channels 4 g8 + 32 u), so that the eight threads of a
    // row store 16-byte groups into eight different bank quads; all sixteen loads
    // are in flight before any is used (one CTA per SM: the loads in flight are
    // what hides the memory latency)
    {
        const int r = tid >> 3, g8 = tid & 7;
        const bool in = r < n;
        const size_t off = ((tok0 + (in ? r : 0)) * H + h) * DK + 4 * g8;
        uint2 k4[4], q4[4];
        float4 b4[4], l4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            k4[u] = in ? *reinterpret_cast<const uint2 *>(k + off + 32 * u) : make_uint2(0u, 0u);
            q4[u] = in ? *reinterpret_cast<const uint2 *>(q + off + 32 * u) : make_uint2(0u, 0u);
            b4[u] = in ? *reinterpret_cast<const float4 *>(bg + off + 32 * u) : make_float4(0.f, 0.f, 0.f, 0.f);
            l4[u] = in ? *reinterpret_cast<const float4 *>(la + off + 32 * u) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = 4 * g8 + 32 * u;
            const float2 k01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&k4[u].x));
            const float2 k23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&k4[u].y));
            const float2 q01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&q4[u].x));
            const float2 q23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&q4[u].y));
            *reinterpret_cast<float4 *>(KF + r * LDF + j) = make_float4(k01.x, k01.y, k23.x, k23.y);
            *reinterpret_cast<float4 *>(QF + r * LDF + j) = make_float4(q01.x, q01.y, q23.x, q23.y);
            *reinterpret_cast<float4 *>(BK + r * LDF + j) =
                make_float4(b4[u].x * k01.x, b4[u].y * k01.y, b4[u].z * k23.x, b4[u].w * k23.y);
            *reinterpret_cast<float4 *>(LM + r * LDF + j) =
                make_float4(l4[u].x * LOG2E, l4[u].y * LOG2E, l4[u].z * LOG2E, l4[u].w * LOG2E);
        }
    }
    // per-channel passes below: thread -> (channel jc, quarter rq of the rows)
    constexpr int RQ = C / 4;                      // rows per quarter
    const int jc = tid & (DK - 1), rq = tid >> 7;
    __syncthreads();
    TCW(1);
    {   // running sums over the rows, per channel: each quarter locally, then the
        // totals of the earlier quarters are added
        float acc = 0.f;
        for (int rr = 0; rr < RQ; ++rr) {
            const int r = rq * RQ + rr;
            acc += LM[r * LDF + jc];
            LM[r * LDF + jc] = acc;
        }
    }
    __syncthreads();
    {
        float base = 0.f;
        for (int qq = 0; qq < rq; ++qq) base += LM[(qq * RQ + RQ - 1) * LDF + jc];
        __syncthreads();
        for (int rr = 0; rr < RQ; ++rr) LM[(rq * RQ + rr) * LDF + jc] += base;
    }
    __syncthreads();
    TCW(2);

    // the two 8 x 8 diagonal sub-blocks of each diagonal 16-block, summed
    // directly: warps 4I .. 4I+3 take block I, each a quarter of the channels.
    // Lane -> sub-block s, the rows rp and 7 - rp of it (rp + 1 and 8 - rp pairs
    // (r, i), i <= r: nine in all) and 8 of the warp's 32 channels (the pairs
    // 8 jb + 2 cs, + 1 for jb < 4: float2 loads whose 8-byte banks differ across a
    // half-warp), so each row's values are loaded once per channel and the
    // columns' values are shared by the two rows; the four lanes of a row pair
    // then add their channel parts.
    {
        const int I = warp >> 2, ch = warp & 3;
        const int sb = lane >> 4, rp = (lane >> 2) & 3, cs = lane & 3;
        const int i0 = 16 * I + 8 * sb;
        const int rA = i0 + rp, rB = i0 + 7 - rp;
        float aA[4] = {}, pA[4] = {}, aB[8] = {}, pB[8] = {};
        // The decay from row i to row r (i <= r) of the sub-block is the product of the
        // decays between consecutive rows, d_m = 2^(Lam_{m+1} - Lam_m) <= 1 for
        // m = i .. r - 1: seven exp2 per channel, no overflow for any decay, and the
        // factors multiply in float32 (a running product down the columns).
        const int b = 7 - rp;  // rB and rA within the sub-block: b and rp
#pragma unroll 2
        for (int jb = 0; jb < 4; ++jb) {
            const int j = 32 * ch + 8 * jb + 2 * cs;
            const float2 bA = ld2(BK, rA, j), bB = ld2(BK, rB, j);
            const float2 qA = ld2(QF, rA, j), qB = ld2(QF, rB, j);
            float2 l[8], kI[8];
#pragma unroll
            for (int ii = 0; ii < 8; ++ii) {
                l[ii] = ld2(LM, i0 + ii, j);
                kI[ii] = ld2(KF, i0 + ii, j);
            }
            float2 d[7];
#pragma unroll
            for (int m = 0; m < 7; ++m)
                d[m] = make_float2(tc::ex2(l[m + 1].x - l[m].x), tc::ex2(l[m + 1].y - l[m].y));
            // row rB: columns ii = b down to 0 (eB = 1 at ii = b, then times d[ii])
            float2 eB = make_float2(1.f, 1.f), eA = make_float2(1.f, 1.f);
#pragma unroll
            for (int ii = 7; ii >= 0; --ii) {
                if (ii < 7 && ii < b) {
                    eB.x *= d[ii].x;
                    eB.y *= d[ii].y;
                }
                const bool kB = ii <= b;
                const float eB0 = kB ? eB.x * kI[ii].x : 0.f, eB1 = kB ? eB.y * kI[ii].y : 0.f;
                aB[ii] = fmaf(bB.y, eB1, fmaf(bB.x, eB0, aB[ii]));
                pB[ii] = fmaf(qB.y, eB1, fmaf(qB.x, eB0, pB[ii]));
                if (ii < 4) {
                    // row rA: columns ii = rp down to 0
                    if (ii < 3 && ii < rp) {
                        eA.x *= d[ii].x;
                        eA.y *= d[ii].y;
                    }
                    const bool kA = ii <= rp;
                    const float eA0 = kA ? eA.x * kI[ii].x : 0.f, eA1 = kA ? eA.y * kI[ii].y : 0.f;
                    aA[ii] = fmaf(bA.y, eA1, fmaf(bA.x, eA0, aA[ii]));
                    pA[ii] = fmaf(qA.y, eA1, fmaf(qA.x, eA0, pA[ii]));
                }
            }
        }
#pragma unroll
        for (int ii = 0; ii < 8; ++ii) {
            aB[ii] += __shfl_xor_sync(0xffffffffu, aB[ii], 1);
            aB[ii] += __shfl_xor_sync(0xffffffffu, aB[ii], 2);
            pB[ii] += __shfl_xor_sync(0xffffffffu, pB[ii], 1);
            pB[ii] += __shfl_xor_sync(0xffffffffu, pB[ii], 2);
        }
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) {
            aA[ii] += __shfl_xor_sync(0xffffffffu, aA[ii], 1);
            aA[ii] += __shfl_xor_sync(0xffffffffu, aA[ii], 2);
            pA[ii] += __shfl_xor_sync(0xffffffffu, pA[ii], 1);
            pA[ii] += __shfl_xor_sync(0xffffffffu, pA[ii], 2);
        }
        // pair slots of this row pair: k < 8 - rp -> (rB, i0 + k), else (rA, i0 + k - (8 - rp))
        float *ds = DS + I * 3 * NPAIR * 2;   // partial sums of channel quarters 1-3
        const int slot0 = (sb * 4 + rp) * 9;
        if (ch > 0 && cs == 0) {
#pragma unroll
            for (int ii = 0; ii < 8; ++ii)
                if (ii <= 7 - rp) {
                    ds[((ch - 1) * NPAIR + slot0 + ii) * 2] = aB[ii];
                    ds[((ch - 1) * NPAIR + slot0 + ii) * 2 + 1] = pB[ii];
                }
#pragma unroll
            for (int ii = 0; ii < 4; ++ii)
                if (ii <= rp) {
                    ds[((ch - 1) * NPAIR + slot0 + 8 - rp + ii) * 2] = aA[ii];
                    ds[((ch - 1) * NPAIR + slot0 + 8 - rp + ii) * 2 + 1] = pA[ii];
                }
        }
        __syncthreads();
        if (ch == 0 && cs == 0) {
#pragma unroll
            for (int ii = 0; ii < 8; ++ii)
                if (ii <= 7 - rp) {
                    float a = aB[ii], pp = pB[ii];
#pragma unroll
                    for (int cq = 0; cq < 3; ++cq) {
                        a += ds[(cq * NPAIR + slot0 + ii) * 2];
                        pp += ds[(cq * NPAIR + slot0 + ii) * 2 + 1];
                    }
                    AF[rB * LDA + i0 + ii] = rB > i0 + ii ? a : 0.f;
                    PF[rB * LDA + i0 + ii] = pp;
                }
#pragma unroll
            for (int ii = 0; ii < 4; ++ii)
                if (ii <= rp) {
                    float a = aA[ii], pp = pA[ii];
#pragma unroll
                    for (int cq = 0; cq < 3; ++cq) {
                        a += ds[(cq * NPAIR + slot0 + 8 - rp + ii) * 2];
                        pp += ds[(cq * NPAIR + slot0 + 8 - rp + ii) * 2 + 1];
                    }
                    AF[rA * LDA + i0 + ii] = rA > i0 + ii ? a : 0.f;
                    PF[rA * LDA + i0 + ii] = pp;
                }
        }
    }
    TCW(3);
    // blocks I > J through the reference row m = 16 I - 1 (warps 0-5, one pair each)
    if (warp < 6) {
        const int I = warp == 0 ? 1 : (warp < 3 ? 2 : 3);
        const int J = warp == 0 ? 0 : (warp < 3 ? warp - 1 : warp - 3);
        const int mref = 16 * I - 1;
        float accA[2][4] = {}, accP[2][4] = {};
#pragma unroll 2
        for (int ks = 0; ks < DK / 16; ++ks) {
            const int j0 = 16 * ks;
            // Lam of the reference row at the fragments' two channel pairs
            const float2 lm[2] = {ld2(LM, mref, j0 + 2 * t), ld2(LM, mref, j0 + 2 * t + 8)};
            uint32_t aL[4], aM[4];
#pragma unroll
            for (int sl = 0; sl < 4; ++sl) {  // a0 (g, 2t) a1 (g+8, 2t) a2 (g, 2t+8) a3 (g+8, 2t+8)
                const int r = 16 * I + g + 8 * (sl & 1), j = j0 + 2 * t + 8 * (sl >> 1);
                const float2 lr = ld2(LM, r, j), bk = ld2(BK, r, j), qf = ld2(QF, r, j);
                const float e0 = tc::ex2(lr.x - lm[sl >> 1].x), e1 = tc::ex2(lr.y - lm[sl >> 1].y);
                aL[sl] = tc::pack_bf16(bk.x * e0, bk.y * e1);
                aM[sl] = tc::pack_bf16(qf.x * e0, qf.y * e1);
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                // B[kk][n] = K_i o 2^(Lam_m - Lam_i) at row i = 16 J + 8 nt + n, channel j0 + kk
                const int i = 16 * J + 8 * nt + g;
                uint32_t bb[2];
#pragma unroll
                for (int hb = 0; hb < 2; ++hb) {
                    const float2 li = ld2(LM, i, j0 + 2 * t + 8 * hb), kf = ld2(KF, i, j0 + 2 * t + 8 * hb);
                    bb[hb] = tc::pack_bf16(kf.x * tc::ex2(lm[hb].x - li.x), kf.y * tc::ex2(lm[hb].y - li.y));
                }
                mma_bf16_16x8x16(accA[nt], aL, bb);
                mma_bf16_16x8x16(accP[nt], aM, bb);
            }
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int col = 16 * J + 8 * nt + 2 * t;
            const int r0 = 16 * I + g, r1 = r0 + 8;
            *reinterpret_cast<float2 *>(AF + r0 * LDA + col) = make_float2(accA[nt][0], accA[nt][1]);
            *reinterpret_cast<float2 *>(AF + r1 * LDA + col) = make_float2(accA[nt][2], accA[nt][3]);
            *reinterpret_cast<float2 *>(PF + r0 * LDA + col) = make_float2(accP[nt][0], accP[nt][1]);
            *reinterpret_cast<float2 *>(PF + r1 * LDA + col) = make_float2(accP[nt][2], accP[nt][3]);
        }
    }
    // rows 8-15 against rows 0-7 of each diagonal block through its row 7 (warps
    // 6-9, one block each): a 16 x 8 product whose rows 0-7 are left zero
    else if (warp < 10) {
        const int I = warp - 6, mref = 16 * I + 7;
        float accA[4] = {}, accP[4] = {};
#pragma unroll 2
        for (int ks = 0; ks < DK / 16; ++ks) {
            const int j0 = 16 * ks;
            const float2 lm[2] = {ld2(LM, mref, j0 + 2 * t), ld2(LM, mref, j0 + 2 * t + 8)};
            uint32_t aL[4] = {0u, 0u, 0u, 0u}, aM[4] = {0u, 0u, 0u, 0u};
#pragma unroll
            for (int sl = 1; sl < 4; sl += 2) {  // a1 (g+8, 2t), a3 (g+8, 2t+8)
                const int r = 16 * I + 8 + g, j = j0 + 2 * t + 8 * (sl >> 1);
                const float2 lr = ld2(LM, r, j), bk = ld2(BK, r, j), qf = ld2(QF, r, j);
                const float e0 = tc::ex2(lr.x - lm[sl >> 1].x), e1 = tc::ex2(lr.y - lm[sl >> 1].y);
                aL[sl] = tc::pack_bf16(bk.x * e0, bk.y * e1);
                aM[sl] = tc::pack_bf16(qf.x * e0, qf.y * e1);
            }
            const int i = 16 * I + g;  // B[kk][n] = K_i o 2^(Lam_m - Lam_i), n = g
            uint32_t bb[2];
#pragma unroll
            for (int hb = 0; hb < 2; ++hb) {
                const float2 li = ld2(LM, i, j0 + 2 * t + 8 * hb), kf = ld2(KF, i, j0 + 2 * t + 8 * hb);
                bb[hb] = tc::pack_bf16(kf.x * tc::ex2(lm[hb].x - li.x), kf.y * tc::ex2(lm[hb].y - li.y));
            }
            mma_bf16_16x8x16(accA, aL, bb);
            mma_bf16_16x8x16(accP, aM, bb);
        }
        const int r1 = 16 * I + 8 + g, col = 16 * I + 2 * t;
        *reinterpret_cast<float2 *>(AF + r1 * LDA + col) = make_float2(accA[2], accA[3]);
        *reinterpret_cast<float2 *>(PF + r1 * LDA + col) = make_float2(accP[2], accP[3]);
    }
    else {
        // w o V (it needs neither A nor P) on the six warps the block products leave
        // idle: item -> (row, 16 consecutive value channels), 16-byte loads
        for (int item = tid - 320; item < C * (Dv / 16); item += THREADS - 320) {
            const int r = item / (Dv / 16), jv0 = 16 * (item % (Dv / 16));
            if (r >= n) break;
            const size_t off = ((tok0 + r) * H + h) * Dv + jv0;
            const uint4 v0 = *reinterpret_cast<const uint4 *>(v + off);
            const uint4 v1 = *reinterpret_cast<const uint4 *>(v + off + 8);
            float4 w4[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) w4[u] = *reinterpret_cast<const float4 *>(wg + off + 4 * u);
            const uint32_t vw_[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            const float wv[16] = {w4[0].x, w4[0].y, w4[0].z, w4[0].w, w4[1].x, w4[1].y, w4[1].z, w4[1].w,
                                  w4[2].x, w4[2].y, w4[2].z, w4[2].w, w4[3].x, w4[3].y, w4[3].z, w4[3].w};
            uint32_t out[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&vw_[e]));
                out[e] = tc::pack_bf16(f.x * wv[2 * e], f.y * wv[2 * e + 1]);
            }
            uint4 *dst = reinterpret_cast<uint4 *>(vw + off);
            dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
            dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
        }
    }
    __syncthreads();  // A and P complete
    TCW(4);

    // T = (I + A)^-1: diagonal blocks by substitution, the rest by block products
    // on warps 0-3 (named barrier 1); meanwhile warps 4-15 write the sequential
    // kernel's token operands Q o 2^Lam and K o 2^(Lam_last - Lam): item -> (row r,
    // 4 channels 4 g8 + 32 u) as in the input phase (16-byte shared-memory reads
    // whose bank quads differ across eight threads, 8-byte stores)
    if (warp < 4) {
        if (tid < C) tc::ut_diag(AF, TF, tid);
        named_barrier(1, 128);
        tc::ut_offdiag4<1>(AF, TF, tid);
    } else {
        for (int item = tid - 128; item < C * 32; item += THREADS - 128) {
            const int r = item >> 5, g8 = item & 7, u = (item >> 3) & 3;
            if (r >= n) break;
            const int j = 4 * g8 + 32 * u;
            const float4 lr = ld4(LM, r, j), ll = ld4(LM, C - 1, j);
            const float4 qf = ld4(QF, r, j), kf = ld4(KF, r, j);
            const size_t off = ((tok0 + r) * H + h) * DK + j;
            *reinterpret_cast<uint2 *>(qe + off) =
                make_uint2(tc::pack_bf16(qf.x * tc::ex2(lr.x), qf.y * tc::ex2(lr.y)),
                           tc::pack_bf16(qf.z * tc::ex2(lr.z), qf.w * tc::ex2(lr.w)));
            *reinterpret_cast<uint2 *>(kd + off) =
                make_uint2(tc::pack_bf16(kf.x * tc::ex2(ll.x - lr.x), kf.y * tc::ex2(ll.y - lr.y)),
                           tc::pack_bf16(kf.z * tc::ex2(ll.z - lr.z), kf.w * tc::ex2(ll.w - lr.w)));
        }
    }
    __syncthreads();
    TCW(5);

    // [P; T''] (T'' = T with zero columns for rows past the end), and T as bf16
    // over the dead A buffer; 8 threads per 128-byte row
    {
        __nv_bfloat16 *dpt = pt + tile * PT_ELEMS;
#pragma unroll
        for (int m = 0; m < PT_ELEMS / 8 / THREADS; ++m) {
            const int idx = tid + THREADS * m;
            const int rt = idx >> 3, i0 = 8 * (idx & 7), r = rt & (C - 1);
            const float *src = (rt < C ? PF : TF) + r * LDA + i0;
            const float4 sa = *reinterpret_cast<const float4 *>(src);
            const float4 sb = *reinterpret_cast<const float4 *>(src + 4);
            const float sv[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = (i0 + e <= r && (rt < C || i0 + e < n)) ? sv[e] : 0.f;
            *reinterpret_cast<uint4 *>(dpt + rt * C + i0) =
                make_uint4(tc::pack_bf16(x[0], x[1]), tc::pack_bf16(x[2], x[3]),
                           tc::pack_bf16(x[4], x[5]), tc::pack_bf16(x[6], x[7]));
            if (rt >= C) {
                float y[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) y[e] = (i0 + e <= r) ? sv[e] : 0.f;
                *reinterpret_cast<uint4 *>(TB + r * LDT + i0) =
                    make_uint4(tc::pack_bf16(y[0], y[1]), tc::pack_bf16(y[2], y[3]),
                               tc::pack_bf16(y[4], y[5]), tc::pack_bf16(y[6], y[7]));
            }
        }
        if (tid < DK) glk[tile * DK + tid] = tc::ex2(LM[(C - 1) * LDF + tid]);
    }
    __syncthreads();
    TCW(6);

    // W = T (b o K o 2^Lam): warp w -> rows 16 (w % 4) .. + 15 (T is lower
    // triangular: chunk rows up to 16 (w % 4) + 15 contribute), channels
    // 32 (w / 4) .. + 31
    {
        const int RB = warp & 3, nh = warp >> 2;
        const int mi = lane >> 3, ri = lane & 7;
        const __nv_bfloat16 *arow = TB + (16 * RB + ri + 8 * (mi & 1)) * LDT + 8 * (mi >> 1);
        float acc[4][4] = {};
        for (int ks = 0; ks <= RB; ++ks) {
            uint32_t a[4];
            ldmatrix_x4(a, arow + 16 * ks);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const int j = 32 * nh + 8 * nt + g;  // B[kk][n] at chunk row 16 ks + kk, channel j
                uint32_t bb[2];
#pragma unroll
                for (int hb = 0; hb < 2; ++hb) {
                    const int i = 16 * ks + 2 * t + 8 * hb;
                    bb[hb] = tc::pack_bf16(BK[i * LDF + j] * tc::ex2(LM[i * LDF + j]),
                                           BK[(i + 1) * LDF + j] * tc::ex2(LM[(i + 1) * LDF + j]));
                }
                mma_bf16_16x8x16(acc[nt], a, bb);
            }
        }
        __nv_bfloat16 *dw = wt + tile * W_ELEMS;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            const int col = 32 * nh + 8 * nt + 2 * t;
            const int r0 = 16 * RB + g;
            *reinterpret_cast<uint32_t *>(dw + r0 * DK + col) = tc::pack_bf16(acc[nt][0], acc[nt][1]);
            *reinterpret_cast<uint32_t *>(dw + (r0 + 8) * DK + col) =
                tc::pack_bf16(acc[nt][2], acc[nt][3]);
        }
    }

    TCW(7);
    TCW(8);
    TCW(9);
}

}  // namespace cwt

#ifdef GDN_TRACE
extern "C" int gdn_trace_cw_read(unsigned long long *dst) {
    return (int)cudaMemcpyFromSymbol(dst, g_trace_cw, sizeof(g_trace_cw));
}
#endif

bool cw_tc_supported(int B, int T, int H, int Dk, int Dv, int chunk, bool bf16) {
    return bf16 && chunk == cwt::C && Dk == cwt::DK && Dv % 64 == 0 && B >= 1 && T >= 1 &&
           H >= 1 && tc::encode_fn() != nullptr;
}

// Workspace: [Q o 2^Lam, K o 2^(Lam_last - Lam): [B*T, H, 128] bf16 each][w o V:
// [B*T, H, Dv] bf16][[P; T''] tiles][W tiles][2^Lam_last per key channel].
size_t cw_tc_workspace_bytes(int B, int T, int H, int Dv) {
    const size_t tok = (size_t)B * T * H;
    const size_t tiles = (size_t)B * ((T + cwt::C - 1) / cwt::C) * H;
    return tok * (2 * cwt::DK + Dv) * sizeof(__nv_bfloat16) +
           tiles * (cwt::PT_ELEMS + cwt::W_ELEMS) * sizeof(__nv_bfloat16) +
           tiles * cwt::DK * sizeof(float);
}

cudaError_t launch_chunk_cw_tc(const void *q, const void *k, const void *v, const float *la,
                               const float *bg, const float *wg, const float *S0, void *o,
                               float *S_T, int B, int T, int H, int Dv, void *workspace,
                               cudaStream_t st) {
    const size_t tok = (size_t)B * T * H;
    const int NT = (T + cwt::C - 1) / cwt::C;
    const size_t tiles = (size_t)B * NT * H;
    auto *qe = static_cast<__nv_bfloat16 *>(workspace);
    __nv_bfloat16 *kd = qe + tok * cwt::DK;
    __nv_bfloat16 *vw = kd + tok * cwt::DK;
    __nv_bfloat16 *pt = vw + tok * Dv;
    __nv_bfloat16 *wt = pt + tiles * cwt::PT_ELEMS;
    float *glk = reinterpret_cast<float *>(wt + tiles * cwt::W_ELEMS);
    cudaError_t e = cudaFuncSetAttribute(cwt::gdn_ut_cw_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, cwt::SMEM);
    if (e != cudaSuccess) return e;
    cwt::gdn_ut_cw_kernel<<<dim3(NT, H, B), cwt::THREADS, cwt::SMEM, st>>>(
        static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k),
        static_cast<const __nv_bfloat16 *>(v), la, bg, wg, qe, kd, vw, pt, wt, glk, T, H, Dv);
    e = cudaPeekAtLastError();
    if (e != cudaSuccess) return e;
    return launch_chunk_tcw_seq_cw(qe, kd, vw, pt, wt, glk, S0, o, S_T, B, T, H, Dv, st);
}

}  // namespace gdn
