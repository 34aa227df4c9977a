// Chunkwise backward of the gated delta rule on sm_100a tensor cores: bf16
// q/k/v/d_o, Dk = 128, chunk C = 64, Dv = 64 or 128; float32 gates, states,
// gradients of the gates and of the state, float32 accumulation in TMEM.
//
// The parallel training algorithm of "Gated Delta Networks: Improving Mamba2
// with Delta Rule" (section "Approach") and "Gated DeltaNet: Harmonizing Gating
// and the Delta Rule ..." (section "Hardware-Efficient Training"), differentiated
// chunk by chunk.  Per chunk (rows r, i; g_r the running sum of log alpha from
// the chunk start, gamma_r = exp(g_r), D_r = exp(g_last - g_r), Gamma_ri =
// exp(g_r - g_i) for i <= r; S the state entering the chunk, dS' the gradient
// of the state leaving it; T = (I + A)^-1, P, W = T diag(beta gamma) K and
// T'' = T diag(beta) as in the forward):
//
//   N   = V + X,  X = -diag(gamma) K S^T,  U' = T'' V + T'' X   (so U' = U - W S^T)
//   dU' = P^T dO + diag(D) K dS'^T,   Z = T^T dU',   dV = diag(beta) Z
//   dS  = gamma_last dS' + dO^T diag(gamma) Q - dU'^T W        (to the left)
//   dP  = lower(dO U'^T),   dQ = diag(gamma) dO S + (dP o Gamma) K
//   dA  = -strictly-lower(Z U'^T),   E = diag(beta) (dA o Gamma)
//   dK  = (dP o Gamma)^T Q + diag(D) U' dS' - diag(beta gamma) Z S + (E + E^T) K
//   dbeta_r = Z_r . N_r + sum_i dA_ri Gamma_ri k_r . k_i
//   dg_r    = gamma_r (dO S)_r . q_r + sum_i (dP o P + dA o A)_ri - sum_m (dP o P + dA o A)_mr
//             + beta_r Z_r . X_r                  (+ gamma_last <dS', S> on the last row)
//   dlog alpha_r = sum_{m >= r} dg_m + sum_{m < r} D_m U'_m . (K dS'^T)_m   (within the chunk)
//
// Two facts shorten the textbook form: U' depends on T only through U' = T M,
// M = diag(beta) N, so the UT transform's adjoint -T^T dT T^T collapses to
// dA = -Z U'^T; and Y = T^T dW with dW = -dU' S is -Z S, so W is needed only by
// the state-gradient chain, where -K^T diag(beta gamma) Z = -W^T dU'.
// dlog alpha is a small difference of large sums where the decays are strong,
// so the terms that cancel exactly are never formed: the row and column sums of
// dP o P and dA o A come from the same float32 products and leave out the
// diagonal (its terms cancel row for column), and the decay D_m of the state
// update enters as the prefix sum above rather than as -D_r U'_r . (K dS'^T)_r
// on every row plus their total on the last one.  X is kept apart from V (its
// own bf16 tile) for the same reason: rounded into N it would vanish where
// gamma is tiny, and with it the term beta_r Z_r . X_r.
//
// Launches (one stream): the precomputed forward's parallel kernel for the
// [P; T''], W and T tiles and its sequential kernel, fed those tiles, for the
// state entering every chunk in bf16 (chunk_tc_wide.cu), then
//  1. gdn_bwd_chain_kernel: one CTA per (sequence, head, 64 value channels)
//     walking the chunks backwards with dS^T (128 keys x 64 values, float32) in
//     tensor memory; per chunk R = K dS'^T (M = 64), dU' = P^T dO + D o R in an
//     epilogue, and dS^T = gamma_last dS'^T + Q^T (gamma o dO) - W^T dU'
//     (M = 128).  It records dS' (bf16) for every chunk and writes dS0.
//  2. gdn_bwd_grads_kernel: one CTA per (chunk, head), all chunks in parallel;
//     twelve groups of tcgen05 products in four dependent phases, epilogues between
//     them (every operand a 128-byte-swizzled bf16 tile in shared memory, every
//     accumulator in TMEM), then dq, dk, dv, dlog alpha and dbeta.
// Rows past the end of a sequence are loaded as zeros (four-dimensional tensor
// maps over [B, T, H, D]) and carry beta = 0, log alpha = 0: they add nothing.
// Every mbarrier wait is bounded (about two seconds); a CTA that times out sets
// an error flag (gdn_check_device_status) and stops.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tc_common.cuh"

namespace gdn {

// Set by a CTA of the backward's tensor-core kernels that gave up waiting.
__device__ unsigned int g_bwd_error = 0;

// Optional phase timeline of two CTAs of the gradient kernel (chunk 0 and chunk
// 63 of head 8, batch 0) for performance work: build with -DGDN_TRACE; that
// build alone exports gdn_trace_bwd_read().  Compiled out otherwise.
#ifdef GDN_TRACE
__device__ unsigned long long g_trace_bwd[2 * 16];
#define TG(ev)                                                                          \
    do {                                                                                \
        if (threadIdx.x == 0 && blockIdx.z == 0 &&                                      \
            ((blockIdx.x == 0 && blockIdx.y == 0) || (blockIdx.x == 63 && blockIdx.y == 8))) \
            g_trace_bwd[(blockIdx.x == 0 ? 0 : 16) + (ev)] = clock64();                 \
    } while (0)
#else
#define TG(ev) \
    do {       \
    } while (0)
#endif

namespace btc {

using namespace sm100;
using tc::C;
using tc::Ctx;

constexpr int DK = 128;
constexpr int DVT = 64;            // value channels per CTA of the chain kernel
constexpr int PANEL = 8192;        // 64 rows x 128 bytes: one swizzled panel of 64 columns
constexpr float LOG2E = 1.4426950408889634f;

// 16 bf16 values of row `row`, columns [16 piece, 16 piece + 16), of a swizzled panel.
__device__ __forceinline__ void load16_bf16(const uint8_t *tile, int row, int piece, float (&v)[16]) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const uint4 u = *reinterpret_cast<const uint4 *>(tile + sw128_offset(row, (2 * piece + k) * 16));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[e]));
            v[8 * k + 2 * e] = f.x;
            v[8 * k + 2 * e + 1] = f.y;
        }
    }
}

__device__ __forceinline__ void store16_global_bf16(__nv_bfloat16 *dst, const float (&v)[16]) {
    uint4 *d = reinterpret_cast<uint4 *>(dst);
    d[0] = make_uint4(tc::pack_bf16(v[0], v[1]), tc::pack_bf16(v[2], v[3]),
                      tc::pack_bf16(v[4], v[5]), tc::pack_bf16(v[6], v[7]));
    d[1] = make_uint4(tc::pack_bf16(v[8], v[9]), tc::pack_bf16(v[10], v[11]),
                      tc::pack_bf16(v[12], v[13]), tc::pack_bf16(v[14], v[15]));
}

// ===================================================== 1. state-gradient chain
namespace chain {

constexpr int NTHREADS = 384;
constexpr int W_TMA = 0, W_MMA = 1, W_OG = 2, W_STATE0 = 4;  // OG: warps 2, 3; state: 4-11
// One stage (two in a ring): K, Q and W as two 64-key panels each, P (rows 0-63
// of the [P; T''] tile), dO (this CTA's 64 value channels), gamma o dO.
constexpr int OFF_K = 0, OFF_Q = 2 * PANEL, OFF_W = 4 * PANEL, OFF_P = 6 * PANEL,
              OFF_DO = 7 * PANEL, OFF_OG = 8 * PANEL;
constexpr int STAGE = 9 * PANEL;
constexpr int TX_BYTES = 8 * PANEL;             // everything but gamma o dO comes by TMA
constexpr int SM_SB = 2 * STAGE;                // dS'^T (bf16): 128 key rows x 64 values
constexpr int SM_DU = SM_SB + 2 * PANEL;        // -dU' (bf16): 64 rows x 64 values
constexpr int SM_GV = SM_DU + PANEL;            // per stage: gamma, D (64 each), gamma_last
constexpr int GV_GAM = 0, GV_DCY = 64, GV_GL = 128, GV_STRIDE = 132;
constexpr int SM_BAR = SM_GV + 2 * GV_STRIDE * 4;
enum {
    B_IN_FULL = 0,    // [2] TMA bytes + the gate vectors
    B_IN_EMPTY = 2,   // [2] the stage's last product completed
    B_OG_FULL = 4,    // [2] gamma o dO written (warps 2, 3)
    B_PD_FULL = 6,    // [2] P^T dO (double-buffered in TMEM)
    B_PD_EMPTY = 8,   // [2] P^T dO read
    B_S_READY = 10,   // dS'^T copied to shared memory, TMEM scaled by gamma_last
    B_R_FULL = 11,    // K dS'^T
    B_U_READY = 12,   // -dU' in shared memory
    B_ST_FULL = 13,   // the state-gradient update completed
    NBAR = 14
};
constexpr int SM_MISC = SM_BAR + NBAR * 8;
constexpr int SMEM_BYTES = SM_MISC + 16 + 1024;
constexpr uint32_t TM_ST = 0, TM_R = 64, TM_PD = 128, TM_COLS = 256;
static_assert(SM_BAR % 8 == 0, "aligned barriers");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");

struct Params {
    const float *log_alpha;
    const float *dS_T;            // [B*H][Dv][Dk] or null
    float *dS0;                   // [B*H][Dv][Dk] or null
    __nv_bfloat16 *dS_hist;       // [B*H][NT][Dv][Dk]: dS' of every chunk
    int T, H, Dv, NT;
};

__global__ void __launch_bounds__(NTHREADS, 1)
gdn_bwd_chain_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_w,
                     const __grid_constant__ CUtensorMap tm_p, const Params p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    Ctx cx;
    cx.base = base;
    cx.bar = reinterpret_cast<uint64_t *>(base + SM_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + SM_MISC);
    cx.abort = reinterpret_cast<volatile uint32_t *>(base + SM_MISC + 4);
    cx.err = &g_bwd_error;
    float *gv_all = reinterpret_cast<float *>(base + SM_GV);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int v0 = blockIdx.x * DVT, h = blockIdx.y, b = blockIdx.z;
    const int T = p.T, H = p.H, NT = p.NT;
    const size_t head = (size_t)b * H + h;

    if (tid == 0) {
        int counts[NBAR];
        for (int i = 0; i < NBAR; ++i) counts[i] = 1;
        counts[B_OG_FULL] = counts[B_OG_FULL + 1] = 2;
        counts[B_PD_EMPTY] = counts[B_PD_EMPTY + 1] = 8;
        counts[B_S_READY] = counts[B_U_READY] = 8;
        for (int i = 0; i < NBAR; ++i) mbar_init(cx.bar + i, counts[i]);
        *cx.abort = 0u;
        fence_mbar_init();
    }
    if (warp == W_MMA) {
        tmem_alloc(tmem_slot, TM_COLS);
        tmem_relinquish();
    }
    if (warp == W_TMA && lane == 0) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_do);
        prefetch_tensormap(&tm_w);
        prefetch_tensormap(&tm_p);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == W_TMA) {
        // --------------------------------- TMA loads + per-chunk gate vectors
        int armed = 0;
        for (int k = 0; k < NT; ++k) {
            const int c = NT - 1 - k, s = k & 1, t0 = c * C;
            float la[2];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int r = lane + 32 * hh;
                la[hh] = t0 + r < T ? p.log_alpha[((size_t)b * T + t0 + r) * H + h] : 0.f;
            }
            if (k >= 2 && !tc::warp_wait(cx, B_IN_EMPTY + s, ((k - 2) >> 1) & 1)) break;
            if (lane == 0) {
                uint8_t *st = base + s * STAGE;
                uint64_t *fb = cx.bar + B_IN_FULL + s;
                const int tile = (b * NT + c) * H + h;
                mbar_expect_tx(fb, TX_BYTES);
#pragma unroll
                for (int kb = 0; kb < 2; ++kb) {
                    tma_load_4d(st + OFF_K + kb * PANEL, &tm_k, fb, kb * 64, h, t0, b);
                    tma_load_4d(st + OFF_Q + kb * PANEL, &tm_q, fb, kb * 64, h, t0, b);
                    tma_load_3d(st + OFF_W + kb * PANEL, &tm_w, fb, kb * 64, 0, tile);
                }
                tma_load_3d(st + OFF_P, &tm_p, fb, 0, 0, tile);
                tma_load_4d(st + OFF_DO, &tm_do, fb, v0, h, t0, b);
            }
            armed = k + 1;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y0 = __shfl_up_sync(0xffffffffu, la[0], off);
                const float y1 = __shfl_up_sync(0xffffffffu, la[1], off);
                if (lane >= off) {
                    la[0] += y0;
                    la[1] += y1;
                }
            }
            la[1] += __shfl_sync(0xffffffffu, la[0], 31);
            const float g0 = la[0] * LOG2E, g1 = la[1] * LOG2E;
            const float glast = __shfl_sync(0xffffffffu, g1, 31);
            float *gv = gv_all + s * GV_STRIDE;
            gv[GV_GAM + lane] = tc::ex2(g0);
            gv[GV_GAM + 32 + lane] = tc::ex2(g1);
            gv[GV_DCY + lane] = tc::ex2(glast - g0);
            gv[GV_DCY + 32 + lane] = tc::ex2(glast - g1);
            if (lane == 0) gv[GV_GL] = tc::ex2(glast);
            __syncwarp();
            if (lane == 0) mbar_arrive(cx.bar + B_IN_FULL + s);
        }
        // never leave with copies in flight
        if (lane == 0) {
            for (int k = armed - 2 < 0 ? 0 : armed - 2; k < armed; ++k) {
                uint64_t *fb = cx.bar + B_IN_FULL + (k & 1);
                const uint64_t t0 = tc::now_ns();
                while (!mbar_try_wait(fb, (k >> 1) & 1) && tc::now_ns() - t0 < tc::kTimeoutNs) {
                }
            }
        }
    } else if (warp == W_MMA) {
        // ------------------------------------------------------------- MMA
        const uint32_t idesc_r = idesc_bf16(64, DVT, false, true);
        const uint32_t idesc_pd = idesc_bf16(64, DVT, true, true);
        const uint32_t idesc_st = idesc_bf16(128, DVT, true, true);
        const uint32_t sb = smem_u32(base + SM_SB), du = smem_u32(base + SM_DU);
        // P^T dO of chunk index kk into TMEM buffer kk & 1: A = P^T (MN-major), B = dO (MN-major)
        const auto issue_pd = [&](int kk, int s) {
            const uint32_t st = smem_u32(base + s * STAGE);
#pragma unroll
            for (int j = 0; j < C / 16; ++j)
                mma_bf16(tmem + TM_PD + 64 * (kk & 1), desc_sw128(st + OFF_P + j * 2048, PANEL, 1024),
                         desc_sw128(st + OFF_DO + j * 2048, PANEL, 1024), idesc_pd, j > 0);
            mma_commit(cx.bar + B_PD_FULL + (kk & 1));
        };
        bool ok = NT > 0 && tc::warp_wait(cx, B_IN_FULL, 0);
        tc_fence_after();
        if (ok && lane == 0) issue_pd(0, 0);
        __syncwarp();
        for (int k = 0; ok && k < NT; ++k) {
            const int s = k & 1;
            const uint32_t st = smem_u32(base + s * STAGE);
            if (!tc::warp_wait(cx, B_IN_FULL + s, (k >> 1) & 1)) break;
            if (!tc::warp_wait(cx, B_S_READY, k & 1)) break;
            tc_fence_after();
            // R = K dS'^T : A = K (K-major, two key panels), B = dS'^T (MN-major)
            if (lane == 0) {
#pragma unroll
                for (int j = 0; j < DK / 16; ++j) {
                    const uint32_t koff = (j >> 2) * PANEL + (j & 3) * 32;
                    mma_bf16(tmem + TM_R, desc_sw128(st + OFF_K + koff, 16, 1024),
                             desc_sw128(sb + j * 2048, PANEL, 1024), idesc_r, j > 0);
                }
                mma_commit(cx.bar + B_R_FULL);
            }
            __syncwarp();
            // dS^T += Q^T (gamma o dO): A = Q^T (MN-major, key panels PANEL apart)
            if (!tc::warp_wait(cx, B_OG_FULL + s, (k >> 1) & 1)) break;
            tc_fence_after();
            if (lane == 0) {
#pragma unroll
                for (int j = 0; j < C / 16; ++j)
                    mma_bf16(tmem + TM_ST, desc_sw128(st + OFF_Q + j * 2048, PANEL, 1024),
                             desc_sw128(st + OFF_OG + j * 2048, PANEL, 1024), idesc_st, 1u);
            }
            __syncwarp();
            // dS^T += W^T (-dU'), then the stage is free
            if (!tc::warp_wait(cx, B_U_READY, k & 1)) break;
            tc_fence_after();
            if (lane == 0) {
#pragma unroll
                for (int j = 0; j < C / 16; ++j)
                    mma_bf16(tmem + TM_ST, desc_sw128(st + OFF_W + j * 2048, PANEL, 1024),
                             desc_sw128(du + j * 2048, PANEL, 1024), idesc_st, 1u);
                mma_commit(cx.bar + B_ST_FULL);
                mma_commit(cx.bar + B_IN_EMPTY + s);
            }
            __syncwarp();
            if (k + 1 < NT) {
                if (!tc::warp_wait(cx, B_IN_FULL + (s ^ 1), ((k + 1) >> 1) & 1)) break;
                if (k + 1 >= 2 &&
                    !tc::warp_wait(cx, B_PD_EMPTY + ((k + 1) & 1), (((k + 1) >> 1) - 1) & 1))
                    break;
                tc_fence_after();
                if (lane == 0) issue_pd(k + 1, s ^ 1);
                __syncwarp();
            }
        }
    } else if (warp < W_STATE0) {
        // --------------------------------------------------- gamma o dO rows
        const int r = 32 * (warp - W_OG) + lane;
        for (int k = 0; k < NT; ++k) {
            const int s = k & 1;
            if (!tc::warp_wait(cx, B_IN_FULL + s, (k >> 1) & 1)) break;
            const float gr = gv_all[s * GV_STRIDE + GV_GAM + r];
            uint8_t *st = base + s * STAGE;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
                const uint32_t off = sw128_offset(r, cc * 16);
                const uint4 u = *reinterpret_cast<const uint4 *>(st + OFF_DO + off);
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
                uint32_t o[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[e]));
                    o[e] = tc::pack_bf16(f.x * gr, f.y * gr);
                }
                *reinterpret_cast<uint4 *>(st + OFF_OG + off) = make_uint4(o[0], o[1], o[2], o[3]);
            }
            fence_async_smem();
            tc::warp_arrive(cx, B_OG_FULL + s);
        }
    } else {
        // ------------------------------------------------------------ STATE
        // 8 warps: warp w reads TMEM lanes 32 (w % 4) .. + 31 (key channel lrow
        // of dS^T; chunk rows 16 (w % 4) .. + 15 of the M = 64 products in its
        // lanes 0-15) and columns 32 hf .. + 31 of the 64 value channels.
        const int q = warp & 3, hf = (warp - W_STATE0) >> 2;
        const int lrow = 32 * q + lane;
        const uint32_t lane_addr = tmem + ((uint32_t)(32 * q) << 16);
        {
            float x[16];
#pragma unroll
            for (int pc = 0; pc < 2; ++pc) {
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    x[j] = p.dS_T ? p.dS_T[(head * p.Dv + v0 + 32 * hf + 16 * pc + j) * DK + lrow] : 0.f;
                tmem_st16(lane_addr + TM_ST + 32 * hf + 16 * pc, x);
            }
            tmem_wait_st();
        }
        bool ok = true;
        for (int k = 0; k < NT; ++k) {
            const int c = NT - 1 - k, s = k & 1;
            if (k >= 1 && !tc::warp_wait(cx, B_ST_FULL, (k - 1) & 1)) {
                ok = false;
                break;
            }
            if (!tc::warp_wait(cx, B_IN_FULL + s, (k >> 1) & 1)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const float *gv = gv_all + s * GV_STRIDE;
            const float gl = gv[GV_GL];
            float x0[16], x1[16];
            tmem_ld16(lane_addr + TM_ST + 32 * hf, x0);
            tmem_ld16(lane_addr + TM_ST + 32 * hf + 16, x1);
            tmem_wait_ld();
            tc::store16_bf16(base + SM_SB, lrow, 2 * hf, x0);
            tc::store16_bf16(base + SM_SB, lrow, 2 * hf + 1, x1);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                x0[j] *= gl;
                x1[j] *= gl;
            }
            tmem_st16(lane_addr + TM_ST + 32 * hf, x0);
            tmem_st16(lane_addr + TM_ST + 32 * hf + 16, x1);
            tmem_wait_st();
            fence_async_smem();
            tc_fence_before();
            tc::warp_arrive(cx, B_S_READY);
            {   // dS' of chunk c for the gradient kernel, [Dv][Dk] bf16, from this
                // thread's own row of the bf16 copy (beside the K dS'^T product)
                auto *dst = reinterpret_cast<unsigned short *>(p.dS_hist) +
                            ((head * NT + c) * p.Dv + v0 + 32 * hf) * DK + lrow;
#pragma unroll
                for (int k8 = 0; k8 < 4; ++k8) {
                    const uint4 u = *reinterpret_cast<const uint4 *>(
                        base + SM_SB + sw128_offset(lrow, (4 * hf + k8) * 16));
                    const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        dst[(size_t)(8 * k8 + e) * DK] = (unsigned short)(e & 1 ? wd[e >> 1] >> 16 : wd[e >> 1] & 0xffffu);
                }
            }
            // -dU' rows = -(P^T dO + D o (K dS'^T))
            if (!tc::warp_wait(cx, B_PD_FULL + s, (k >> 1) & 1) || !tc::warp_wait(cx, B_R_FULL, k & 1)) {
                ok = false;
                break;
            }
            tc_fence_after();
            // chunk row 16 q + l % 16, values 32 hf + 16 (l / 16) .. + 15 (16-lane loads)
            float r0[16], d0[16];
            tmem_ld16x2<16>(lane_addr + TM_R + 32 * hf, r0);
            tmem_ld16x2<16>(lane_addr + TM_PD + 64 * s + 32 * hf, d0);
            tmem_wait_ld();
            {
                const int r = 16 * q + (lane & 15);
                const float dc = gv[GV_DCY + r];
#pragma unroll
                for (int j = 0; j < 16; ++j) d0[j] = -fmaf(dc, r0[j], d0[j]);
                tc::store16_bf16(base + SM_DU, r, 2 * hf + (lane >> 4), d0);
            }
            fence_async_smem();
            tc_fence_before();
            tc::warp_arrive(cx, B_U_READY);
            tc::warp_arrive(cx, B_PD_EMPTY + s);
        }
        // dS0: the gradient of the state entering the first chunk
        if (ok && NT > 0 && tc::warp_wait(cx, B_ST_FULL, (NT - 1) & 1)) {
            tc_fence_after();
            float x0[16], x1[16];
            tmem_ld16(lane_addr + TM_ST + 32 * hf, x0);
            tmem_ld16(lane_addr + TM_ST + 32 * hf + 16, x1);
            tmem_wait_ld();
            if (p.dS0) {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    p.dS0[(head * p.Dv + v0 + 32 * hf + j) * DK + lrow] = x0[j];
                    p.dS0[(head * p.Dv + v0 + 32 * hf + 16 + j) * DK + lrow] = x1[j];
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == W_MMA) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

}  // namespace chain

// ====================================================== 2. per-chunk gradients
namespace grads {

constexpr int NTHREADS = 256;

// Shared memory (bytes; every tile 1024-aligned, 128-byte swizzled, panels of
// 64 columns).  Tiles written by an epilogue reuse the space of tiles whose
// last product has completed.
template <int DV>
struct L {
    static constexpr int VB = DV / 64 * PANEL;           // a 64 x DV tile
    static constexpr int SD_PANEL = 2 * DV * 128;        // per key panel: S rows, then dS' rows
    static constexpr int SM_K = 0, SM_Q = 2 * PANEL, SM_V = 4 * PANEL, SM_DO = SM_V + VB;
    static constexpr int SM_SD = SM_DO + VB;
    static constexpr int SM_P = SM_SD + 2 * SD_PANEL;    // P, T'' (one TMA tile), then T
    static constexpr int SM_T = SM_P + 2 * PANEL;
    static constexpr int SM_N = SM_T + PANEL;            // X = -gamma o (K S^T)
    static constexpr int SM_DU = SM_N + VB;
    static constexpr int SM_UD = SM_DU + VB;
    static constexpr int SM_ZB = SM_UD + VB;
    static constexpr int SM_MISC = SM_ZB + VB;
    static constexpr int SM_OG = SM_N;          // gamma o dO over X (same thread, same piece)
    static constexpr int SM_UT = SM_DU;         // U' over dU' (read by the Z product only)
    static constexpr int SM_ZT = SM_P + PANEL;  // Z over T'' and T
    static constexpr int SM_DP = SM_V;          // dP o Gamma over V
    static constexpr int SM_EE = SM_DU;         // E + E^T over U'
    static constexpr int SM_ES = SM_ZB;         // E^T (row-major scratch) over -beta gamma o Z
    // per-row float arrays in SM_MISC: the gate vectors, then partial sums written
    // with plain stores (no shared-memory atomics): two column halves per row for
    // the row sums, four row quarters per column for the column sums
    enum { F_G2 = 0, F_BE, F_GAM, F_DCY, F_UR = 4, F_ZN = 6, F_ZX = 8, F_XR = 10, F_DG = 12,
           F_QS = 14, F_XC = 16, NF = 20 };
    // [1] gamma_last, [2] [4] the final scans' warp totals, [8 + w] warp w's part of <dS', S>
    static constexpr int SM_SCAL = SM_MISC + NF * 64 * 4;
    static constexpr int SM_BAR = SM_SCAL + 64;
    // [0] TMA  [1] phase A  [2] phase B  [3] phase C: dP, dA'  [4] phase D
    // [5] K K^T  [6] phase C: dQ, dK
    static constexpr int NBAR = 7;
    static constexpr int SMEM_BYTES = SM_BAR + NBAR * 8 + 16 + 1024;
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
    static_assert(VB >= PANEL && SM_SD % 1024 == 0 && SM_MISC % 1024 == 0, "layout");
};
// TMEM columns (512): phase A  [K S^T | K dS'^T] 0..2DV, P^T dO 2DV..3DV, K K^T 448..511;
// phase B  Z 0..DV, U' 2DV..3DV (K dS'^T kept); phase C/D  dP 0..63, dA' 64..127,
// dQ 128..255, dK 256..383.
constexpr uint32_t TM_KK = 448, TM_DP = 0, TM_DA = 64, TM_Q2 = 128, TM_K2 = 256, TM_COLS = 512;

// The state entering each chunk and the gradient of the state leaving it come by
// TMA from [B*H][NT][Dv][Dk] bf16 arrays (tm_sh, tm_dsh: boxes of 64 keys x DV rows).
struct Params {
    const float *log_alpha, *beta;
    __nv_bfloat16 *dq, *dk, *dv;
    float *dla, *dbeta;
    int T, H, NT;
    int pf_stride;  // the SM count: each CTA prefetches into L2 the inputs of CTA + pf_stride
};

template <int DV>
__global__ void __launch_bounds__(NTHREADS, 1)
gdn_bwd_grads_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                     const __grid_constant__ CUtensorMap tm_pt, const __grid_constant__ CUtensorMap tm_t,
                     const __grid_constant__ CUtensorMap tm_sh, const __grid_constant__ CUtensorMap tm_dsh,
                     const Params p) {
    using Ly = L<DV>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    Ctx cx;
    cx.base = base;
    cx.bar = reinterpret_cast<uint64_t *>(base + Ly::SM_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + Ly::SM_BAR + Ly::NBAR * 8);
    cx.abort = reinterpret_cast<volatile uint32_t *>(base + Ly::SM_BAR + Ly::NBAR * 8 + 4);
    cx.err = &g_bwd_error;
    float *fv = reinterpret_cast<float *>(base + Ly::SM_MISC);
    float *g2s = fv + Ly::F_G2 * 64, *bes = fv + Ly::F_BE * 64, *gams = fv + Ly::F_GAM * 64,
          *dcys = fv + Ly::F_DCY * 64;
    float *rs_ur = fv + Ly::F_UR * 64, *rs_zn = fv + Ly::F_ZN * 64, *rs_zx = fv + Ly::F_ZX * 64,
          *rs_x = fv + Ly::F_XR * 64, *cs_x = fv + Ly::F_XC * 64, *rs_dg = fv + Ly::F_DG * 64,
          *rs_qs = fv + Ly::F_QS * 64;  // [hf][64] (cs_x: [quarter][64])
    float *scal = reinterpret_cast<float *>(base + Ly::SM_SCAL);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int T = p.T, H = p.H, NT = p.NT, t0 = c * C;
    const int tile = (b * NT + c) * H + h;
    const int hist = (b * H + h) * NT + c;
    TG(0);

    if (tid == 0) {
        for (int i = 0; i < Ly::NBAR; ++i) mbar_init(cx.bar + i, 1);
        *cx.abort = 0u;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    TG(1);

    const uint32_t sK = smem_u32(base + Ly::SM_K), sQ = smem_u32(base + Ly::SM_Q),
                   sDO = smem_u32(base + Ly::SM_DO), sSD = smem_u32(base + Ly::SM_SD),
                   sP = smem_u32(base + Ly::SM_P), sT = smem_u32(base + Ly::SM_T),
                   sN = smem_u32(base + Ly::SM_N), sDU = smem_u32(base + Ly::SM_DU),
                   sUD = smem_u32(base + Ly::SM_UD), sZB = smem_u32(base + Ly::SM_ZB),
                   sZT = smem_u32(base + Ly::SM_ZT), sDP = smem_u32(base + Ly::SM_DP),
                   sEE = smem_u32(base + Ly::SM_EE), sUT = smem_u32(base + Ly::SM_UT),
                   sOG = smem_u32(base + Ly::SM_OG);
    const auto kdesc = [](uint32_t t, int j) {  // K-major operand, step j of 16 along K
        return desc_sw128(t + (j >> 2) * PANEL + (j & 3) * 32, 16, 1024);
    };

    // warp 1 issues the copies and then, once they have landed, the products of
    // phase A (they do not need the gates), and warp 2 the prefetches, while warp 0
    // loads the gates
    if (tid == 32) {
        uint64_t *fb = cx.bar + 0;
        mbar_arrive_expect_tx(fb, 4 * PANEL + 2 * Ly::VB + 3 * PANEL + 4 * DV * 128);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
            tma_load_4d(base + Ly::SM_K + kb * PANEL, &tm_k, fb, kb * 64, h, t0, b);
            tma_load_4d(base + Ly::SM_Q + kb * PANEL, &tm_q, fb, kb * 64, h, t0, b);
        }
#pragma unroll
        for (int vb = 0; vb < DV / 64; ++vb) {
            tma_load_4d(base + Ly::SM_V + vb * PANEL, &tm_v, fb, vb * 64, h, t0, b);
            tma_load_4d(base + Ly::SM_DO + vb * PANEL, &tm_do, fb, vb * 64, h, t0, b);
        }
        tma_load_3d(base + Ly::SM_P, &tm_pt, fb, 0, 0, tile);
        tma_load_3d(base + Ly::SM_T, &tm_t, fb, 0, 0, tile);
        // [S; dS'] per 64-key panel: S rows 0 .. DV - 1, dS' rows DV .. 2 DV - 1
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
            tma_load_3d(base + Ly::SM_SD + kb * Ly::SD_PANEL, &tm_sh, fb, kb * 64, 0, hist);
            tma_load_3d(base + Ly::SM_SD + kb * Ly::SD_PANEL + DV * 128, &tm_dsh, fb, kb * 64, 0, hist);
        }
        // ---------------- phase A: [K S^T | K dS'^T], P^T dO, K K^T
        const bool landed = tc::wait_bar(cx, 0, 0);
        tc_fence_after();
        if (landed) {
#pragma unroll
            for (int j = 0; j < DK / 16; ++j)
                mma_bf16(tmem, kdesc(sK, j),
                         desc_sw128(sSD + (j >> 2) * Ly::SD_PANEL + (j & 3) * 32, 16, 1024),
                         idesc_bf16(64, 2 * DV, false, false), j > 0);
#pragma unroll
            for (int j = 0; j < C / 16; ++j)
                mma_bf16(tmem + 2 * DV, desc_sw128(sP + j * 2048, PANEL, 1024),
                         desc_sw128(sDO + j * 2048, PANEL, 1024), idesc_bf16(64, DV, true, true), j > 0);
        }
        mma_commit(cx.bar + 1);
        // K K^T is read by epilogue C only
        if (landed) {
#pragma unroll
            for (int j = 0; j < DK / 16; ++j)
                mma_bf16(tmem + TM_KK, kdesc(sK, j), kdesc(sK, j), idesc_bf16(64, 64, false, false), j > 0);
        }
        mma_commit(cx.bar + 5);
    }
    if (warp == 2) {
        // one CTA per SM: the CTA one wave later (linear index + SM count) finds its
        // inputs in L2, their DRAM reads overlapping this CTA's products (the tiles by
        // lane 0, the gates of its rows by every lane)
        const long long lin = blockIdx.x + (long long)NT * (blockIdx.y + (long long)H * blockIdx.z);
        const long long nxt = lin + p.pf_stride;
        if (p.pf_stride > 0 && nxt < (long long)NT * H * gridDim.z) {
            const int c2 = (int)(nxt % NT), h2 = (int)((nxt / NT) % H), b2 = (int)(nxt / ((long long)NT * H));
            const int t2 = c2 * C, tile2 = (b2 * NT + c2) * H + h2, hist2 = (b2 * H + h2) * NT + c2;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int rr = lane + 32 * hh;
                if (t2 + rr < T) {
                    const size_t gi = ((size_t)b2 * T + t2 + rr) * H + h2;
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(p.log_alpha + gi));
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(p.beta + gi));
                }
            }
            if (lane == 0) {
#pragma unroll
            for (int kb = 0; kb < 2; ++kb) {
                tma_prefetch_l2_4d(&tm_k, kb * 64, h2, t2, b2);
                tma_prefetch_l2_4d(&tm_q, kb * 64, h2, t2, b2);
                tma_prefetch_l2_3d(&tm_sh, kb * 64, 0, hist2);
                tma_prefetch_l2_3d(&tm_dsh, kb * 64, 0, hist2);
            }
#pragma unroll
            for (int vb = 0; vb < DV / 64; ++vb) {
                tma_prefetch_l2_4d(&tm_v, vb * 64, h2, t2, b2);
                tma_prefetch_l2_4d(&tm_do, vb * 64, h2, t2, b2);
            }
            tma_prefetch_l2_3d(&tm_pt, 0, 0, tile2);
            tma_prefetch_l2_3d(&tm_t, 0, 0, tile2);
            }
        }
    }
    if (warp == 0) {
        // gates of the chunk's rows lane, lane + 32 (rows past the end: 0)
        float la[2], be[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int r = lane + 32 * hh;
            const bool in = t0 + r < T;
            const size_t gi = ((size_t)b * T + t0 + r) * H + h;
            la[hh] = in ? p.log_alpha[gi] : 0.f;
            be[hh] = in ? p.beta[gi] : 0.f;
        }
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y0 = __shfl_up_sync(0xffffffffu, la[0], off);
            const float y1 = __shfl_up_sync(0xffffffffu, la[1], off);
            if (lane >= off) {
                la[0] += y0;
                la[1] += y1;
            }
        }
        la[1] += __shfl_sync(0xffffffffu, la[0], 31);
        const float glast = __shfl_sync(0xffffffffu, la[1], 31) * LOG2E;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int r = lane + 32 * hh;
            const float g2 = la[hh] * LOG2E;
            g2s[r] = g2;
            bes[r] = be[hh];
            gams[r] = tc::ex2(g2);
            dcys[r] = tc::ex2(glast - g2);
        }
        if (lane == 0) scal[1] = tc::ex2(glast);
    }
    __syncthreads();
    TG(2);

    // epilogue threads: warp w -> chunk row r = 16 (w % 4) + (l % 16), in TMEM lane
    // 32 (w % 4) + l % 16 (M = 64 layout), column half hf = w / 4; the 16-lane loads
    // give lanes 16-31 the second quarter of the warp's columns (sub = 1)
    const int q = warp & 3, hf = warp >> 2, sub = lane >> 4;
    const int r = 16 * q + (lane & 15);
    const uint32_t la_ = tmem + ((uint32_t)(32 * q) << 16);

    TG(3);
    bool ok = tc::warp_wait(cx, 1, 0);
    tc_fence_after();
    TG(4);
    {   // <dS', S> from the two bf16 tiles (same swizzle: element for element at a
        // fixed distance of DV rows), after this thread has seen the copies land
        ok = tc::warp_wait(cx, 0, 0) && ok;
        float dot = 0.f;
        for (int idx = tid; idx < 2 * DV * 8; idx += NTHREADS) {
            const int kb = idx / (DV * 8), o = (idx % (DV * 8)) * 16;
            const uint8_t *pan = base + Ly::SM_SD + kb * Ly::SD_PANEL;
            const uint4 a = *reinterpret_cast<const uint4 *>(pan + o);
            const uint4 d = *reinterpret_cast<const uint4 *>(pan + DV * 128 + o);
            const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, dw[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&aw[e]));
                const float2 fd = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&dw[e]));
                dot = fmaf(fa.x, fd.x, fmaf(fa.y, fd.y, dot));
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
        if (lane == 0) scal[8 + warp] = dot;
    }
    // 16-value pieces per thread: columns c0 = hf DV / 2 + 16 pc (lanes 0-15) and
    // c0 + DV / 4 (lanes 16-31)
    constexpr int NPC = DV / 64;
    constexpr int QV = DV / 4;
    // epilogue A: X = -gamma o (K S^T), dU' = P^T dO + D o (K dS'^T)
#pragma unroll 1
    for (int pc = 0; pc < NPC; ++pc) {
        const int c0 = hf * (DV / 2) + 16 * pc;
        const int i0 = c0 + sub * QV, vp = i0 >> 6, piece = (i0 & 63) >> 4;
        float ks[16], rr[16], pd[16];
        tmem_ld16x2<QV>(la_ + c0, ks);
        tmem_ld16x2<QV>(la_ + DV + c0, rr);
        tmem_ld16x2<QV>(la_ + 2 * DV + c0, pd);
        tmem_wait_ld();
        const float gr = gams[r], dr = dcys[r];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            ks[j] *= -gr;
            pd[j] = fmaf(dr, rr[j], pd[j]);
        }
        tc::store16_bf16(base + Ly::SM_N + vp * PANEL, r, piece, ks);
        tc::store16_bf16(base + Ly::SM_DU + vp * PANEL, r, piece, pd);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    TG(5);
    // ---------------- phase B: U' = T'' V + T'' X, Z = T^T dU'
    if (tid == 0) {
        tc_fence_after();
        if (ok) {
            const uint32_t sV = smem_u32(base + Ly::SM_V);
#pragma unroll
            for (int j = 0; j < C / 16; ++j)
                mma_bf16(tmem + 2 * DV, desc_sw128(sP + PANEL + j * 32, 16, 1024),
                         desc_sw128(sV + j * 2048, PANEL, 1024), idesc_bf16(64, DV, false, true), j > 0);
#pragma unroll
            for (int j = 0; j < C / 16; ++j)
                mma_bf16(tmem + 2 * DV, desc_sw128(sP + PANEL + j * 32, 16, 1024),
                         desc_sw128(sN + j * 2048, PANEL, 1024), idesc_bf16(64, DV, false, true), 1u);
#pragma unroll
            for (int j = 0; j < C / 16; ++j)
                mma_bf16(tmem, desc_sw128(sT + j * 2048, PANEL, 1024),
                         desc_sw128(sDU + j * 2048, PANEL, 1024), idesc_bf16(64, DV, true, true), j > 0);
        }
        mma_commit(cx.bar + 2);
    }
    ok = tc::warp_wait(cx, 2, 0) && ok;
    tc_fence_after();
    TG(6);
    // epilogue B: U', D o U', Z, -beta gamma o Z, dV = beta o Z, gamma o dO (over X,
    // after the thread's own X piece is read), row dots
    {
        const float br = bes[r], gr = gams[r], dr = dcys[r];
        const bool in = t0 + r < T;
        float ur = 0.f, zv = 0.f, zx = 0.f;
#pragma unroll 1
        for (int pc = 0; pc < NPC; ++pc) {
            const int c0 = hf * (DV / 2) + 16 * pc;
            const int i0 = c0 + sub * QV, vp = i0 >> 6, piece = (i0 & 63) >> 4;
            float up[16], rr[16], z[16];
            tmem_ld16x2<QV>(la_ + 2 * DV + c0, up);
            tmem_ld16x2<QV>(la_ + DV + c0, rr);
            tmem_ld16x2<QV>(la_ + c0, z);
            tmem_wait_ld();
            float t[16];
            tc::store16_bf16(base + Ly::SM_UT + vp * PANEL, r, piece, up);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                ur = fmaf(up[j], rr[j], ur);
                t[j] = dr * up[j];
            }
            tc::store16_bf16(base + Ly::SM_UD + vp * PANEL, r, piece, t);
            tc::store16_bf16(base + Ly::SM_ZT + vp * PANEL, r, piece, z);
#pragma unroll
            for (int j = 0; j < 16; ++j) t[j] = -br * gr * z[j];
            tc::store16_bf16(base + Ly::SM_ZB + vp * PANEL, r, piece, t);
            if (in) {
#pragma unroll
                for (int j = 0; j < 16; ++j) t[j] = br * z[j];
                store16_global_bf16(p.dv + (((size_t)b * T + t0 + r) * H + h) * DV + i0, t);
            }
            load16_bf16(base + Ly::SM_N + vp * PANEL, r, piece, t);
#pragma unroll
            for (int j = 0; j < 16; ++j) zx = fmaf(z[j], t[j], zx);
            load16_bf16(base + Ly::SM_V + vp * PANEL, r, piece, t);
#pragma unroll
            for (int j = 0; j < 16; ++j) zv = fmaf(z[j], t[j], zv);
            load16_bf16(base + Ly::SM_DO + vp * PANEL, r, piece, t);
#pragma unroll
            for (int j = 0; j < 16; ++j) t[j] *= gr;
            tc::store16_bf16(base + Ly::SM_OG + vp * PANEL, r, piece, t);
        }
        // the two column quarters of a row (lanes l and l + 16) add up
        ur += __shfl_xor_sync(0xffffffffu, ur, 16);
        zv += __shfl_xor_sync(0xffffffffu, zv, 16);
        zx += __shfl_xor_sync(0xffffffffu, zx, 16);
        if (sub == 0) {
            rs_ur[64 * hf + r] = ur;
            rs_zn[64 * hf + r] = zv + zx;
            rs_zx[64 * hf + r] = zx;
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    TG(7);
    // ---------------- phase C: dP = dO U'^T, dA' = Z U'^T, dQ = (gamma o dO) S,
    //                  dK = (D o U') dS' + (-beta gamma o Z) S
    if (tid == 0) {
        tc_fence_after();
        const uint32_t id64 = idesc_bf16(64, 64, false, false), idk = idesc_bf16(64, DK, false, true);
        if (ok) {
#pragma unroll
            for (int j = 0; j < DV / 16; ++j) {
                mma_bf16(tmem + TM_DP, kdesc(sDO, j), kdesc(sUT, j), id64, j > 0);
                mma_bf16(tmem + TM_DA, kdesc(sZT, j), kdesc(sUT, j), id64, j > 0);
            }
        }
        mma_commit(cx.bar + 3);
        // the wider dQ and dK products run while epilogue C reads dP and dA'
        if (ok) {
#pragma unroll
            for (int j = 0; j < DV / 16; ++j) {
                mma_bf16(tmem + TM_Q2, kdesc(sOG, j), desc_sw128(sSD + j * 2048, Ly::SD_PANEL, 1024), idk,
                         j > 0);
                mma_bf16(tmem + TM_K2, kdesc(sUD, j),
                         desc_sw128(sSD + DV * 128 + j * 2048, Ly::SD_PANEL, 1024), idk, j > 0);
            }
#pragma unroll
            for (int j = 0; j < DV / 16; ++j)
                mma_bf16(tmem + TM_K2, kdesc(sZB, j), desc_sw128(sSD + j * 2048, Ly::SD_PANEL, 1024),
                         idk, 1u);
        }
        mma_commit(cx.bar + 6);
    }
    ok = tc::warp_wait(cx, 3, 0) && ok;
    ok = tc::warp_wait(cx, 5, 0) && ok;
    tc_fence_after();
    TG(8);
    // epilogue C (row r, columns i0 = 32 hf + 16 sub .. + 15 of the 64 x 64 matrices):
    // dP o Gamma (bf16 tile), E^T (row-major scratch), dbeta's and dg's sums, and
    // gamma_r (dO S)_r . q_r from the dQ accumulator before (dP o Gamma) K joins it
    {
        const float br = bes[r], g2r = g2s[r];
        // E^T (row-major scratch): entry (i, r) holds E_ri
        __nv_bfloat16 *est = reinterpret_cast<__nv_bfloat16 *>(base + Ly::SM_ES);
        float xr = 0.f, dgr = 0.f, qs = 0.f;
        const int i0 = 32 * hf + 16 * sub;
        float ev[16];
        {
            float dp[16], da[16], kk[16];
            tmem_ld16x2<16>(la_ + TM_DP + 32 * hf, dp);
            tmem_ld16x2<16>(la_ + TM_DA + 32 * hf, da);
            tmem_ld16x2<16>(la_ + TM_KK + 32 * hf, kk);
            tmem_wait_ld();
            float pv[16];
            load16_bf16(base + Ly::SM_P, r, i0 >> 4, pv);
            float col[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int i = i0 + e;
                const bool low = i <= r, slow = i < r;
                const float G = low ? tc::ex2(g2r - g2s[i]) : 0.f;
                const float dpg = low ? dp[e] * G : 0.f;
                const float dA = slow ? -da[e] : 0.f;
                const float Gk = slow ? G * kk[e] : 0.f;
                const float x = (slow ? dp[e] * pv[e] : 0.f) + dA * br * Gk;
                xr += x;
                dgr = fmaf(dA, Gk, dgr);
                ev[e] = br * dA * G;
                col[e] = x;
                dp[e] = dpg;
            }
            tc::store16_bf16(base + Ly::SM_DP, r, i0 >> 4, dp);
            // column sums over the 16 rows of each half-warp
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                float v = col[e];
                v += __shfl_xor_sync(0xffffffffu, v, 8);
                v += __shfl_xor_sync(0xffffffffu, v, 4);
                v += __shfl_xor_sync(0xffffffffu, v, 2);
                v += __shfl_xor_sync(0xffffffffu, v, 1);
                col[e] = v;
            }
            if ((lane & 15) == 0) {
#pragma unroll
                for (int e = 0; e < 16; ++e) cs_x[64 * q + i0 + e] = col[e];
            }
        }
        TG(13);
        // once the dQ and dK products have completed: E^T over their operand
        // -beta gamma o Z, and gamma_r (dO S)_r . q_r (keys 64 hf + 16 pc in lanes
        // 0-15, + 32 in lanes 16-31)
        ok = tc::warp_wait(cx, 6, 0) && ok;
        tc_fence_after();
#pragma unroll
        for (int e = 0; e < 16; ++e) est[(i0 + e) * C + r] = __float2bfloat16_rn(ev[e]);
#pragma unroll 1
        for (int pc = 0; pc < 2; ++pc) {
            float x[16], qv[16];
            tmem_ld16x2<32>(la_ + TM_Q2 + 64 * hf + 16 * pc, x);
            tmem_wait_ld();
            load16_bf16(base + Ly::SM_Q + hf * PANEL, r, pc + 2 * sub, qv);
#pragma unroll
            for (int j = 0; j < 16; ++j) qs = fmaf(x[j], qv[j], qs);
        }
        xr += __shfl_xor_sync(0xffffffffu, xr, 16);
        dgr += __shfl_xor_sync(0xffffffffu, dgr, 16);
        qs += __shfl_xor_sync(0xffffffffu, qs, 16);
        if (sub == 0) {
            rs_x[64 * hf + r] = xr;
            rs_dg[64 * hf + r] = dgr;
            rs_qs[64 * hf + r] = qs;
        }
        TG(14);
        __syncthreads();  // E^T complete
        TG(15);
        {
            float et[16], ee[16];
            // row r of E^T is column r of E: E_ir for the rows i > r
            const uint4 *src = reinterpret_cast<const uint4 *>(est + r * C + i0);
            const uint4 u0 = src[0], u1 = src[1];
            const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[e]));
                et[2 * e] = f.x;
                et[2 * e + 1] = f.y;
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int i = i0 + e;
                ee[e] = i < r ? ev[e] : (i > r ? et[e] : 0.f);
            }
            tc::store16_bf16(base + Ly::SM_EE, r, i0 >> 4, ee);
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    TG(9);
    // ---------------- phase D: dQ += (dP o Gamma) K, dK += (dP o Gamma)^T Q + (E + E^T) K
    if (tid == 0) {
        tc_fence_after();
        if (ok) {
            const uint32_t idk = idesc_bf16(64, DK, false, true), idt = idesc_bf16(64, DK, true, true);
#pragma unroll
            for (int j = 0; j < C / 16; ++j) {
                mma_bf16(tmem + TM_Q2, desc_sw128(sDP + j * 32, 16, 1024),
                         desc_sw128(sK + j * 2048, PANEL, 1024), idk, 1u);
                mma_bf16(tmem + TM_K2, desc_sw128(sDP + j * 2048, PANEL, 1024),
                         desc_sw128(sQ + j * 2048, PANEL, 1024), idt, 1u);
                mma_bf16(tmem + TM_K2, desc_sw128(sEE + j * 32, 16, 1024),
                         desc_sw128(sK + j * 2048, PANEL, 1024), idk, 1u);
            }
        }
        mma_commit(cx.bar + 4);
    }
    ok = tc::warp_wait(cx, 4, 0) && ok;
    tc_fence_after();
    TG(10);
    // final epilogue: dq, dk (row r, keys 64 hf + 32 sub .. + 31)
    {
        const bool in = t0 + r < T;
#pragma unroll 1
        for (int pc = 0; pc < 2; ++pc) {
            const int c0 = 64 * hf + 16 * pc, k0 = c0 + 32 * sub;
            float dq[16], dk[16];
            tmem_ld16x2<32>(la_ + TM_Q2 + c0, dq);
            tmem_ld16x2<32>(la_ + TM_K2 + c0, dk);
            tmem_wait_ld();
            if (in) {
                const size_t row = (((size_t)b * T + t0 + r) * H + h) * DK + k0;
                store16_global_bf16(p.dq + row, dq);
                store16_global_bf16(p.dk + row, dk);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    TG(11);
    if (tid < C) {
        // dlog alpha_r = (the sum of dg over rows >= r) + (the sum of the state
        // update's decay terms over rows < r); warp 0 holds rows 0-31, warp 1 rows 32-63
        const int rr = tid;
        const float xc = cs_x[rr] + cs_x[64 + rr] + cs_x[128 + rr] + cs_x[192 + rr];
        float dg = rs_qs[rr] + rs_qs[64 + rr] + rs_x[rr] + rs_x[64 + rr] - xc +
                   bes[rr] * (rs_zx[rr] + rs_zx[64 + rr]);
        if (rr == C - 1) {
            float dot = 0.f;
#pragma unroll
            for (int w = 0; w < 8; ++w) dot += scal[8 + w];
            dg += scal[1] * dot;
        }
        // the prefix is an exclusive scan of the shifted terms, never an inclusive
        // sum minus the row's own term (D = 1 on the last row makes that term large)
        const float hterm = dcys[rr] * (rs_ur[rr] + rs_ur[64 + rr]);
        float hp = __shfl_up_sync(0xffffffffu, hterm, 1);
        if (lane == 0) hp = 0.f;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_down_sync(0xffffffffu, dg, off);
            if (lane + off < 32) dg += y;
            const float z = __shfl_up_sync(0xffffffffu, hp, off);
            if (lane >= off) hp += z;
        }
        if (warp == 1 && lane == 0) scal[4] = dg;            // rows 32..63 in total
        if (warp == 0 && lane == 31) scal[2] = hp + hterm;   // rows 0..31 in total
        named_barrier(1, C);
        if (warp == 0) dg += scal[4];
        else hp += scal[2];
        const float dlog = dg + hp;
        if (ok && t0 + rr < T) {
            const size_t gi = ((size_t)b * T + t0 + rr) * H + h;
            p.dla[gi] = dlog;
            p.dbeta[gi] = rs_zn[rr] + rs_zn[64 + rr] + rs_dg[rr] + rs_dg[64 + rr];
        }
    }
    TG(12);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

}  // namespace grads

// [n_tiles, rows, 64] bf16 tile array: box of `box_rows` rows x 64 columns of one
// tile, 128-byte swizzle.
bool make_map_tiles(CUtensorMap *m, const void *ptr, int rows, int box_rows, long long n_tiles) {
    auto enc = tc::encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)C, (cuuint64_t)rows, (cuuint64_t)n_tiles};
    cuuint64_t strides[2] = {(cuuint64_t)C * 2, (cuuint64_t)rows * C * 2};
    cuuint32_t box[3] = {(cuuint32_t)C, (cuuint32_t)box_rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box,
               es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// W tiles [n_tiles, 64, 128] bf16: box of 64 keys x 64 rows.
bool make_map_wt(CUtensorMap *m, const void *ptr, long long n_tiles) {
    auto enc = tc::encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)DK, (cuuint64_t)C, (cuuint64_t)n_tiles};
    cuuint64_t strides[2] = {(cuuint64_t)DK * 2, (cuuint64_t)C * DK * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)C, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box,
               es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct Ws {
    __nv_bfloat16 *pt, *wt, *tr, *S_hist, *dS_hist;
    size_t bytes;
};

inline size_t up256(size_t n) { return (n + 255) & ~size_t(255); }

// Workspace: [P; T''] tiles | W tiles | T tiles | S_hist | dS_hist (both bf16).
Ws carve(void *base, int B, int T, int H, int Dv) {
    const size_t NT = ((size_t)T + C - 1) / C, tiles = (size_t)B * NT * H;
    const size_t states = (size_t)B * H * NT * Dv * DK;
    const size_t sz[5] = {tiles * 2 * C * C * 2, tiles * C * DK * 2, tiles * C * C * 2, states * 2,
                          states * 2};
    uint8_t *p = static_cast<uint8_t *>(base);
    size_t off[5], o = 0;
    for (int i = 0; i < 5; ++i) {
        off[i] = o;
        o += up256(sz[i]);
    }
    Ws w;
    w.pt = reinterpret_cast<__nv_bfloat16 *>(p + off[0]);
    w.wt = reinterpret_cast<__nv_bfloat16 *>(p + off[1]);
    w.tr = reinterpret_cast<__nv_bfloat16 *>(p + off[2]);
    w.S_hist = reinterpret_cast<__nv_bfloat16 *>(p + off[3]);
    w.dS_hist = reinterpret_cast<__nv_bfloat16 *>(p + off[4]);
    w.bytes = o;
    return w;
}

// [n, Dv, 128] bf16 state arrays: box of 64 keys x `rows` value rows of one state.
bool make_map_states(CUtensorMap *m, const void *ptr, int Dv, int rows, long long n) {
    auto enc = tc::encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)DK, (cuuint64_t)Dv, (cuuint64_t)n};
    cuuint64_t strides[2] = {(cuuint64_t)DK * 2, (cuuint64_t)Dv * DK * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box,
               es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DV>
cudaError_t launch_grads(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                         const CUtensorMap &mdo, const CUtensorMap &mpt, const CUtensorMap &mt,
                         const grads::Params &gp, const Ws &w, int B, cudaStream_t st) {
    const long long n_hist = (long long)B * gp.H * gp.NT;
    CUtensorMap msh, mdsh;
    if (!make_map_states(&msh, w.S_hist, DV, DV, n_hist) ||
        !make_map_states(&mdsh, w.dS_hist, DV, DV, n_hist))
        return cudaErrorInvalidValue;
    auto *kern = grads::gdn_bwd_grads_kernel<DV>;
    constexpr int smem = grads::L<DV>::SMEM_BYTES;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<dim3(gp.NT, gp.H, B), grads::NTHREADS, smem, st>>>(mq, mk, mv, mdo, mpt, mt, msh, mdsh, gp);
    return cudaPeekAtLastError();
}

}  // namespace btc

bool bwd_tc_supported(int B, int T, int H, int Dk, int Dv, int chunk, bool bf16) {
    return bf16 && Dk == btc::DK && chunk == tc::C && (Dv == 64 || Dv == 128) &&
           tc_supported(B, T, H, Dk, Dv, chunk, bf16) && tc::encode_fn() != nullptr;
}

size_t bwd_tc_workspace_bytes(int B, int T, int H, int Dv) {
    return btc::carve(nullptr, B, T, H, Dv).bytes;
}

cudaError_t launch_chunk_bwd_tc(const void *q, const void *k, const void *v, const float *la,
                                const float *beta, const float *S0, const void *d_o,
                                const float *dS_T, void *dq, void *dk, void *dv, float *dla,
                                float *dbeta, float *dS0, int B, int T, int H, int Dv,
                                void *workspace, cudaStream_t st) {
    using namespace btc;
    const int NT = (T + C - 1) / C;
    const long long n_tiles = (long long)B * NT * H;
    Ws w = carve(workspace, B, T, H, Dv);
    // recompute: the chunk tiles, then the state entering every chunk
    cudaError_t e = launch_recompute_bwd(q, k, v, la, beta, S0, B, T, H, Dv, w.pt, w.wt, w.tr,
                                         w.S_hist, st);
    if (e != cudaSuccess) return e;
    CUtensorMap mq, mk, mv, mdo, mw, mp, mpt, mt;
    if (!tc::make_map(&mq, q, B, T, H, DK) || !tc::make_map(&mk, k, B, T, H, DK) ||
        !tc::make_map(&mv, v, B, T, H, Dv) || !tc::make_map(&mdo, d_o, B, T, H, Dv) ||
        !make_map_wt(&mw, w.wt, n_tiles) || !make_map_tiles(&mp, w.pt, 2 * C, C, n_tiles) ||
        !make_map_tiles(&mpt, w.pt, 2 * C, 2 * C, n_tiles) ||
        !make_map_tiles(&mt, w.tr, C, C, n_tiles))
        return cudaErrorInvalidValue;
    chain::Params cp;
    cp.log_alpha = la;
    cp.dS_T = dS_T;
    cp.dS0 = dS0;
    cp.dS_hist = w.dS_hist;
    cp.T = T;
    cp.H = H;
    cp.Dv = Dv;
    cp.NT = NT;
    e = cudaFuncSetAttribute(chain::gdn_bwd_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             chain::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    chain::gdn_bwd_chain_kernel<<<dim3(Dv / DVT, H, B), chain::NTHREADS, chain::SMEM_BYTES, st>>>(
        mq, mk, mdo, mw, mp, cp);
    e = cudaPeekAtLastError();
    if (e != cudaSuccess) return e;
    grads::Params gp;
    gp.log_alpha = la;
    gp.beta = beta;
    gp.dq = static_cast<__nv_bfloat16 *>(dq);
    gp.dk = static_cast<__nv_bfloat16 *>(dk);
    gp.dv = static_cast<__nv_bfloat16 *>(dv);
    gp.dla = dla;
    gp.dbeta = dbeta;
    gp.T = T;
    gp.H = H;
    gp.NT = NT;
    {
        int dev = 0, sms = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return cudaErrorUnknown;
        gp.pf_stride = sms;
    }
    return Dv == 128 ? launch_grads<128>(mq, mk, mv, mdo, mpt, mt, gp, w, B, st)
                     : launch_grads<64>(mq, mk, mv, mdo, mpt, mt, gp, w, B, st);
}

#ifdef GDN_TRACE
extern "C" int gdn_trace_bwd_read(unsigned long long *dst) {
    return (int)cudaMemcpyFromSymbol(dst, g_trace_bwd, sizeof(g_trace_bwd));
}
#endif

cudaError_t read_and_clear_device_error_bwd(unsigned int *flag) {
    cudaError_t e = cudaMemcpyFromSymbol(flag, g_bwd_error, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_bwd_error, &zero, sizeof(unsigned int));
}

}  // namespace gdn
