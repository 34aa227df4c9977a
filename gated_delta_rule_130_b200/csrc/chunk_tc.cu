// Fused chunkwise forward of the gated delta rule on sm_100a tensor cores
// (tcgen05 + TMEM + TMA), bf16 q/k/v/o, float32 gates, state and accumulation.
//
// Per chunk of C = 64 tokens (rows r), with g_r the running sum of log alpha
// from the chunk start, gamma_r = exp(g_r), and S the state (Dv x Dk) entering
// the chunk, the gated WY/UT form ("Gated Delta Networks: Improving Mamba2 with
// Delta Rule", section "Approach"; "Gated DeltaNet: Harmonizing Gating and the
// Delta Rule ...", section "Hardware-Efficient Training") is evaluated as
//   A   = strictly-lower( beta_r exp(g_r - g_i) k_r . k_i )         Gram, gated
//   T   = (I + A)^-1                                               UT transform
//   W   = T diag(beta gamma) K,   U = T diag(beta) V                WY factors
//   U'  = U - W S^T                                                corrected values
//   O   = diag(gamma) Q S^T + (Q K^T o exp(g_r - g_i) o [i <= r]) U'
//   S  <- gamma_last S + U'^T diag(exp(g_last - g)) K
// The first four lines do not depend on S and run one chunk ahead of the
// sequential part.
//
// One CTA owns one (batch, head, 64-wide slice of value channels) and walks the
// chunks of that head in order, with its slice of S^T (Dk x 64, float32)
// resident in tensor memory for the whole sequence.  Warp roles:
//   warps 0-3  PREP   gates and cumulative sums, A and P from the Gram matrix,
//                     the UT solve (float32, CUDA cores), W to shared memory
//   warps 4-7  STATE  U' = U - W S^T, the chunk output, the state hand-off
//   warp 8     TMA    K, Q and V tiles into a two-stage ring
//   warp 9     MMA    the sequential products (one elected thread)
//   warp 10    MMA    the chunk-local products (one elected thread)
// Every product is a tcgen05.mma with M = 128 (bf16 operands in 128-byte
// swizzled shared memory, float32 accumulators in TMEM):
//   G  = [K;Q] K^T            (prep)   rows 0-63 K K^T, rows 64-127 Q K^T
//   WU = [T';T''] [K | V]     (prep)   T' = T diag(beta gamma), T'' = T diag(beta);
//                                      W = rows 0-63 x K columns, U = rows 64-127 x V columns
//   X  = [Q;W] S^T            (state)  rows 0-63 Q S^T, rows 64-127 W S^T
//   Y  = [P;*] U'             (state)  rows 0-63 intra-chunk output
//   S^T += K^T diag(exp(g_last - g)) U'   (state; S^T kept pre-scaled by gamma_last)
// Shared-memory stage layout per 64-wide key block: K | Q | W (8 KiB each), so
// that [K;Q] and [Q;W] are contiguous 128-row operands, and the K blocks and the
// V tile sit 24 KiB apart so [K | V] is one MN-major operand of width Dk + 64.
//
// Rows past the end of the sequence are loaded as zeros by TMA and get
// beta = 0, log alpha = 0, which leaves the real rows' results unchanged.
// Every mbarrier wait is bounded (about two seconds); on a timeout the CTA
// records an error flag, stops all roles, waits for its outstanding copies and
// releases its tensor memory.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace gdn {

// Set by a fused-kernel CTA that gave up waiting (read with gdn_check_device_status).
__device__ unsigned int g_tc_error = 0;

namespace tc {

using namespace sm100;

constexpr int C = 64;          // chunk length (tokens)
constexpr int DVT = 64;        // value channels per CTA
constexpr int DK = 128;        // key channels
constexpr int KB = DK / 64;    // 64-wide key blocks
constexpr int NSTAGE = 2;
constexpr int BLK = 8192;      // one 64 x 64 bf16 tile (64 rows of 128 bytes)
constexpr int GRP = 3 * BLK;   // K | Q | W of one key block
constexpr int STAGE = KB * GRP + BLK;
constexpr int OFF_K = 0, OFF_Q = BLK, OFF_W = 2 * BLK, OFF_V = KB * GRP;
constexpr int LDA = 65;        // padded float32 row stride of the solve buffers

// shared-memory map (bytes from the 1024-aligned base)
constexpr int SM_STAGE = 0;
constexpr int SM_SB = NSTAGE * STAGE;          // S^T bf16, DK rows x 128 B (MN-major B)
constexpr int SM_UN = SM_SB + DK * 128;        // U' bf16, 64 rows (MN-major B)
constexpr int SM_UP = SM_UN + BLK;             // diag(exp(g_last - g)) U' bf16
constexpr int SM_PT = SM_UP + BLK;             // P tiles for even / odd chunks
constexpr int SM_TT = SM_PT + 2 * BLK;         // [T'; T''] 128 rows (K-major A)
constexpr int SM_AF = SM_TT + 2 * BLK;         // A, float32 64 x LDA
constexpr int SM_TF = SM_AF + 64 * LDA * 4;    // T, float32 64 x LDA
constexpr int SM_XS = SM_TF + 64 * LDA * 4;    // solve scratch, 3 x 16 x 16 float32
constexpr int SM_GATE = SM_XS + 3 * 256 * 4;   // 2 x {gamma[64], decay[64], gamma_last}
constexpr int GATE_STRIDE = 256;               // floats per parity
constexpr int SM_PG = SM_GATE + 2 * GATE_STRIDE * 4;  // prep-private: g2[64], beta[64], carry
constexpr int SM_BAR = SM_PG + 160 * 4;
constexpr int NBAR = 24;
constexpr int SM_MISC = SM_BAR + NBAR * 8;     // tmem base, abort flag
constexpr int SM_TOTAL = SM_MISC + 16;
constexpr int SMEM_BYTES = SM_TOTAL + 1024;    // + alignment slack
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");

// TMEM columns
constexpr uint32_t TM_ST = 0, TM_X = 64, TM_Y = 128, TM_G = 192, TM_WU = 256;
constexpr uint32_t TM_U = TM_WU + DK;
constexpr uint32_t TM_COLS = 512;

// barrier indices
enum {
    B_IN_FULL = 0,      // [2] TMA -> consumers
    B_IN_EMPTY = 2,     // [2] chain MMA (after the state update) -> TMA
    B_G_FULL = 4,       // prep MMA -> prep
    B_G_EMPTY = 5,      // prep -> prep MMA (128)
    B_TT_FULL = 6,      // prep -> prep MMA (128)
    B_WU_FULL = 7,      // prep MMA -> prep, state
    B_WU_EMPTY = 8,     // prep (64) + state (64) -> prep MMA
    B_PREP_FULL = 9,    // [2] prep -> chain MMA, state (128)
    B_PT_EMPTY = 11,    // [2] chain MMA -> prep
    B_GATE_EMPTY = 13,  // [2] state -> prep (128)
    B_X_FULL = 15,      // chain MMA -> state
    B_U_READY = 16,     // state (64) -> chain MMA
    B_Y_FULL = 17,      // chain MMA -> state
    B_ST_FULL = 18,     // chain MMA -> state
    B_S_READY = 19,     // state (128) -> chain MMA
};

constexpr int NTHREADS = 352;
constexpr uint64_t kTimeoutNs = 2000000000ull;

__device__ __forceinline__ uint64_t now_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

struct Ctx {
    uint8_t *base;
    uint64_t *bar;
    volatile uint32_t *abort;
};

// Bounded wait; false (and the CTA-wide abort flag set) on timeout or abort.
__device__ __noinline__ bool wait_bar(const Ctx &cx, int idx, uint32_t parity) {
    uint64_t *b = cx.bar + idx;
    if (mbar_try_wait(b, parity)) return true;
    const uint64_t t0 = now_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(b, parity)) return true;
        if ((it & 255u) == 0) {
            if (*cx.abort) return false;
            if (now_ns() - t0 > kTimeoutNs) {
                *cx.abort = 1u;
                atomicOr(&g_tc_error, 1u);
                return false;
            }
        }
    }
}

// The same wait made by every lane of a warp, with a warp-uniform result (so a
// timeout never splits a warp in front of a warp-collective tcgen05 access).
__device__ __forceinline__ bool warp_wait(const Ctx &cx, int idx, uint32_t parity) {
    const bool ok = wait_bar(cx, idx, parity);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// Store 64 floats as one 128-byte bf16 row `row` of a 128B-swizzled tile.
__device__ __forceinline__ void store_row_bf16(uint8_t *tile, int row, const float *v) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint4 q;
        q.x = pack_bf16(v[8 * c + 0], v[8 * c + 1]);
        q.y = pack_bf16(v[8 * c + 2], v[8 * c + 3]);
        q.z = pack_bf16(v[8 * c + 4], v[8 * c + 5]);
        q.w = pack_bf16(v[8 * c + 6], v[8 * c + 7]);
        *reinterpret_cast<uint4 *>(tile + sw128_offset(row, c * 16)) = q;
    }
}

// 64 consecutive TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&v)[64]) {
    float *p = v;
#pragma unroll
    for (int j = 0; j < 4; ++j) tmem_ld16(taddr + 16 * j, *reinterpret_cast<float(*)[16]>(p + 16 * j));
    tmem_wait_ld();
}

// T = (I + A)^-1 for the 64 x 64 strictly lower A in AF (float32, stride LDA),
// written to TF (lower triangle and diagonal; the strict upper part is not
// written).  Blocked by 16: the four diagonal blocks by forward substitution,
// then T_IJ = -T_II sum_{J<=K<I} A_IK T_KJ by block diagonals.  Called by the
// 128 prep threads together (t = 0..127); uses named barrier 1.
__device__ __forceinline__ void ut_solve(const float *AF, float *TF, float *XS, int t) {
    if (t < 64) {
        const int I = t >> 4, j = t & 15, o = 16 * I;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < r; ++i) acc += AF[(o + r) * LDA + o + i] * x[i];
            x[r] = (r == j) ? 1.f : ((r < j) ? 0.f : -acc);
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) TF[(o + r) * LDA + o + j] = x[r];
    }
    named_barrier(1, 128);
    const int c = t & 15, rr = t >> 4;  // column c, rows rr and rr + 8 of each block
    for (int d = 1; d <= 3; ++d) {
        const int nb = 4 - d;
        for (int b = 0; b < nb; ++b) {
            const int I = d + b, J = b;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int r = rr + 8 * h;
                float acc = 0.f;
                for (int K = J; K < I; ++K) {
#pragma unroll
                    for (int m = 0; m < 16; ++m)
                        acc += AF[(16 * I + r) * LDA + 16 * K + m] * TF[(16 * K + m) * LDA + 16 * J + c];
                }
                XS[b * 256 + r * 16 + c] = acc;
            }
        }
        named_barrier(1, 128);
        for (int b = 0; b < nb; ++b) {
            const int I = d + b, J = b;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int r = rr + 8 * h;
                float acc = 0.f;
#pragma unroll
                for (int m = 0; m < 16; ++m)
                    acc += TF[(16 * I + r) * LDA + 16 * I + m] * XS[b * 256 + m * 16 + c];
                TF[(16 * I + r) * LDA + 16 * J + c] = -acc;
            }
        }
        named_barrier(1, 128);
    }
}

struct Params {
    const float *log_alpha;
    const float *beta;
    const float *S0;
    __nv_bfloat16 *o;
    float *S_T;
    int T, H, Dv, NT;
};

__global__ void __launch_bounds__(NTHREADS, 1)
gdn_chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    Ctx cx;
    cx.base = base;
    cx.bar = reinterpret_cast<uint64_t *>(base + SM_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + SM_MISC);
    cx.abort = reinterpret_cast<volatile uint32_t *>(base + SM_MISC + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int vt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int v0 = vt * DVT;
    const int T = p.T, H = p.H, NT = p.NT;

    if (tid == 0) {
        const int counts[NBAR] = {1, 1, 1, 1, 1, 128, 128, 1, 128, 128, 128, 1, 1, 128, 128,
                                  1, 64, 1, 1, 128, 1, 1, 1, 1};
        for (int i = 0; i < NBAR; ++i) mbar_init(cx.bar + i, counts[i]);
        *cx.abort = 0u;
        fence_mbar_init();
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, TM_COLS);
        tmem_relinquish();
    }
    if (warp == 8 && lane == 0) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 8) {
        // ------------------------------------------------------------- TMA
        if (lane == 0) {
            int armed = 0;
            for (int c = 0; c < NT; ++c) {
                const int s = c & 1;
                if (c >= 2 && !wait_bar(cx, B_IN_EMPTY + s, ((c - 2) >> 1) & 1)) break;
                uint8_t *st = base + SM_STAGE + s * STAGE;
                mbar_arrive_expect_tx(cx.bar + B_IN_FULL + s, (2 * KB + 1) * BLK);
                const int t0 = c * C;
#pragma unroll
                for (int kb = 0; kb < KB; ++kb) {
                    tma_load_4d(st + kb * GRP + OFF_K, &tm_k, cx.bar + B_IN_FULL + s, kb * 64, h, t0, b);
                    tma_load_4d(st + kb * GRP + OFF_Q, &tm_q, cx.bar + B_IN_FULL + s, kb * 64, h, t0, b);
                }
                tma_load_4d(st + OFF_V, &tm_v, cx.bar + B_IN_FULL + s, v0, h, t0, b);
                armed = c + 1;
            }
            // never leave with copies in flight: wait for the last two stages
            for (int c = armed - 2 < 0 ? 0 : armed - 2; c < armed; ++c) {
                uint64_t *fb = cx.bar + B_IN_FULL + (c & 1);
                const uint64_t t0 = now_ns();
                while (!mbar_try_wait(fb, (c >> 1) & 1) && now_ns() - t0 < kTimeoutNs) {
                }
            }
        }
    } else if (warp == 10) {
        // ------------------------------------------- MMA: chunk-local products
        if (lane == 0) {
            const uint32_t idesc_g = idesc_bf16(128, 64, false, false);
            const uint32_t idesc_wu = idesc_bf16(128, DK + DVT, false, true);
            for (int c = 0; c < NT; ++c) {
                const int s = c & 1;
                const uint32_t st = smem_u32(base + SM_STAGE + s * STAGE);
                if (!wait_bar(cx, B_IN_FULL + s, (c >> 1) & 1)) break;
                if (c >= 1 && !wait_bar(cx, B_G_EMPTY, (c - 1) & 1)) break;
                tc_fence_after();
                // G = [K;Q] K^T : A rows 0-63 = K, 64-127 = Q (K-major); B = K (K-major)
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk) {
                    const uint32_t koff = (kk >> 2) * GRP + (kk & 3) * 32;
                    mma_bf16(tmem + TM_G, desc_sw128(st + OFF_K + koff, 16, 1024),
                             desc_sw128(st + OFF_K + koff, 16, 1024), idesc_g, kk > 0);
                }
                mma_commit(cx.bar + B_G_FULL);
                if (!wait_bar(cx, B_TT_FULL, c & 1)) break;
                if (c >= 1 && !wait_bar(cx, B_WU_EMPTY, (c - 1) & 1)) break;
                tc_fence_after();
                // WU = [T'; T''] [K | V] : A K-major (K = 64 tokens), B MN-major
                const uint32_t tt = smem_u32(base + SM_TT);
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    mma_bf16(tmem + TM_WU, desc_sw128(tt + kk * 32, 16, 1024),
                             desc_sw128(st + OFF_K + kk * 2048, GRP, 1024), idesc_wu, kk > 0);
                mma_commit(cx.bar + B_WU_FULL);
            }
        }
    } else if (warp == 9) {
        // ---------------------------------------------- MMA: sequential chain
        if (lane == 0) {
            const uint32_t idesc_x = idesc_bf16(128, DVT, false, true);
            const uint32_t idesc_y = idesc_bf16(128, DVT, false, true);
            const uint32_t idesc_s = idesc_bf16(128, DVT, true, true);
            const uint32_t sb = smem_u32(base + SM_SB), un = smem_u32(base + SM_UN),
                           up = smem_u32(base + SM_UP);
            for (int c = 0; c < NT; ++c) {
                const int s = c & 1;
                const uint32_t st = smem_u32(base + SM_STAGE + s * STAGE);
                if (!wait_bar(cx, B_IN_FULL + s, (c >> 1) & 1)) break;
                if (!wait_bar(cx, B_PREP_FULL + s, (c >> 1) & 1)) break;
                if (!wait_bar(cx, B_S_READY, c & 1)) break;
                tc_fence_after();
                // X = [Q; W] S^T : A K-major (rows 0-63 Q, 64-127 W), B = S^T MN-major
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk) {
                    const uint32_t koff = (kk >> 2) * GRP + (kk & 3) * 32;
                    mma_bf16(tmem + TM_X, desc_sw128(st + OFF_Q + koff, 16, 1024),
                             desc_sw128(sb + kk * 2048, 16, 1024), idesc_x, kk > 0);
                }
                mma_commit(cx.bar + B_X_FULL);
                if (!wait_bar(cx, B_U_READY, c & 1)) break;
                tc_fence_after();
                // Y = [P; *] U'  (rows 64-127 of the A tile are not used)
                const uint32_t pt = smem_u32(base + SM_PT + s * BLK);
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    mma_bf16(tmem + TM_Y, desc_sw128(pt + kk * 32, 16, 1024),
                             desc_sw128(un + kk * 2048, 16, 1024), idesc_y, kk > 0);
                mma_commit(cx.bar + B_Y_FULL);
                mma_commit(cx.bar + B_PT_EMPTY + s);
                // S^T += K^T (decay U') : A = K^T (MN-major, key blocks GRP apart)
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    mma_bf16(tmem + TM_ST, desc_sw128(st + OFF_K + kk * 2048, GRP, 1024),
                             desc_sw128(up + kk * 2048, 16, 1024), idesc_s, 1u);
                mma_commit(cx.bar + B_ST_FULL);
                mma_commit(cx.bar + B_IN_EMPTY + s);
            }
        }
    } else if (warp < 4) {
        // ------------------------------------------------------------- PREP
        const int t = tid;  // TMEM lane t
        float *AF = reinterpret_cast<float *>(base + SM_AF);
        float *TF = reinterpret_cast<float *>(base + SM_TF);
        float *XS = reinterpret_cast<float *>(base + SM_XS);
        float *g2 = reinterpret_cast<float *>(base + SM_PG);        // g * log2(e)
        float *bt = g2 + 64;                                          // beta
        float *carry = bt + 64;
        const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
        constexpr float LOG2E = 1.4426950408889634f;
        for (int c = 0; c < NT; ++c) {
            const int s = c & 1;
            const int t0 = c * C;
            uint8_t *st = base + SM_STAGE + s * STAGE;
            float *gate = reinterpret_cast<float *>(base + SM_GATE) + s * GATE_STRIDE;
            bool ok = true;  // false once a wait has failed; the CTA is then aborting
            if (c >= 2) ok &= warp_wait(cx, B_GATE_EMPTY + s, ((c - 2) >> 1) & 1);
            // gates: running sum of log alpha within the chunk (rows 0..63)
            if (t < 64) {
                const bool in = t0 + t < T;
                const size_t gi = ((size_t)b * T + t0 + t) * H + h;
                float la = in ? p.log_alpha[gi] : 0.f;
                const float be = in ? p.beta[gi] : 0.f;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, la, off);
                    if (lane >= off) la += y;
                }
                if (t == 31) carry[0] = la;
                bt[t] = be;
                g2[t] = la;  // within-warp prefix; rows 32..63 get the carry below
            }
            named_barrier(1, 128);
            if (t < 64) {
                const float g = g2[t] + (t >= 32 ? carry[0] : 0.f);
                named_barrier(2, 64);
                g2[t] = g * LOG2E;
                named_barrier(2, 64);
                const float glast = g2[63];
                gate[t] = ex2(g2[t]);                  // gamma_r
                gate[64 + t] = ex2(glast - g2[t]);     // exp(g_last - g_r)
                if (t == 0) gate[128] = ex2(glast);    // gamma_last
            }
            named_barrier(1, 128);
            // Gram matrix -> A (rows of K K^T, lanes 0-63) and P (rows of Q K^T, lanes 64-127)
            ok &= warp_wait(cx, B_G_FULL, c & 1);
            tc_fence_after();
            {
                float gv[64];
                tmem_ld64(lane_addr + TM_G, gv);
                tc_fence_before();
                mbar_arrive(cx.bar + B_G_EMPTY);
                if (t < 64) {
                    const int r = t;
                    const float gr = g2[r], br = bt[r];
#pragma unroll
                    for (int i = 0; i < 64; ++i)
                        AF[r * LDA + i] = (i < r) ? br * ex2(gr - g2[i]) * gv[i] : 0.f;
                } else {
                    const int r = t - 64;
                    if (c >= 2) ok &= warp_wait(cx, B_PT_EMPTY + s, ((c - 2) >> 1) & 1);
                    const float gr = g2[r];
#pragma unroll
                    for (int i = 0; i < 64; ++i) gv[i] = (i <= r) ? ex2(gr - g2[i]) * gv[i] : 0.f;
                    store_row_bf16(base + SM_PT + s * BLK, r, gv);
                    fence_async_smem();
                }
            }
            named_barrier(1, 128);
            ut_solve(AF, TF, XS, t);
            // [T'; T''] : row t, T'(r,i) = T(r,i) beta_i gamma_i, T''(r,i) = T(r,i) beta_i
            {
                const int r = t & 63;
                float row[64];
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    const float sc = bt[i] * ((t < 64) ? gate[i] : 1.f);
                    row[i] = (i <= r) ? TF[r * LDA + i] * sc : 0.f;
                }
                store_row_bf16(base + SM_TT, t, row);
                fence_async_smem();
                mbar_arrive(cx.bar + B_TT_FULL);
            }
            // W rows (lanes 0-63) to the stage's W slots
            ok &= warp_wait(cx, B_WU_FULL, c & 1);
            tc_fence_after();
            if (t < 64) {
#pragma unroll
                for (int kb = 0; kb < KB; ++kb) {
                    float w[64];
                    tmem_ld64(lane_addr + TM_WU + 64 * kb, w);
                    store_row_bf16(st + kb * GRP + OFF_W, t, w);
                }
                fence_async_smem();
                tc_fence_before();
                mbar_arrive(cx.bar + B_WU_EMPTY);
            }
            mbar_arrive(cx.bar + B_PREP_FULL + s);
            // leave together: every prep thread sees the same decision
            if (named_barrier_or(1, 128, !ok || *cx.abort)) break;
        }
    } else {
        // ------------------------------------------------------------ STATE
        const int t = tid - 128;  // TMEM lane t: key channel t of S^T; chunk row for X/Y
        const int q = warp & 3;
        const uint32_t lane_addr = tmem + ((uint32_t)(q * 32) << 16);
        uint8_t *sb = base + SM_SB;
        const size_t head = (size_t)b * H + h;
        // initial state: S^T row t = S0[v0 .. v0+63][t]
        {
            float sv[64];
#pragma unroll
            for (int j = 0; j < 64; ++j)
                sv[j] = p.S0 ? p.S0[(head * p.Dv + v0 + j) * DK + t] : 0.f;
            store_row_bf16(sb, t, sv);
            fence_async_smem();
            if (warp_wait(cx, B_PREP_FULL + 0, 0)) {
                const float gl = reinterpret_cast<const float *>(base + SM_GATE)[128];
#pragma unroll
                for (int j = 0; j < 64; ++j) sv[j] *= gl;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    tmem_st16(lane_addr + TM_ST + 16 * j, *reinterpret_cast<float(*)[16]>(sv + 16 * j));
                tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(cx.bar + B_S_READY);
        }
        for (int c = 0; c < NT; ++c) {
            if (__any_sync(0xffffffffu, *cx.abort != 0u)) break;
            const int s = c & 1;
            const int t0 = c * C;
            const float *gate = reinterpret_cast<const float *>(base + SM_GATE) + s * GATE_STRIDE;
            float oq[64];
            if (!warp_wait(cx, B_X_FULL, c & 1)) break;
            tc_fence_after();
            if (t >= 64) {
                // U' = U - W S^T for chunk row r
                const int r = t - 64;
                float x[64], u[64];
                tmem_ld64(lane_addr + TM_X, x);
                tmem_ld64(lane_addr + TM_U, u);
#pragma unroll
                for (int j = 0; j < 64; ++j) u[j] -= x[j];
                store_row_bf16(base + SM_UN, r, u);
                const float dc = gate[64 + r];
#pragma unroll
                for (int j = 0; j < 64; ++j) u[j] *= dc;
                store_row_bf16(base + SM_UP, r, u);
                fence_async_smem();
                tc_fence_before();
                mbar_arrive(cx.bar + B_U_READY);
                mbar_arrive(cx.bar + B_WU_EMPTY);
            } else {
                // inter-chunk part of the output for chunk row t: gamma_t (Q S^T)_t
                tmem_ld64(lane_addr + TM_X, oq);
                const float gr = gate[t];
#pragma unroll
                for (int j = 0; j < 64; ++j) oq[j] *= gr;
                if (!warp_wait(cx, B_Y_FULL, c & 1)) break;
                tc_fence_after();
                float y[64];
                tmem_ld64(lane_addr + TM_Y, y);
                if (t0 + t < T) {
                    __nv_bfloat16 *dst = p.o + (((size_t)b * T + t0 + t) * H + h) * p.Dv + v0;
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) {
                        uint4 qv;
                        qv.x = pack_bf16(oq[8 * cc + 0] + y[8 * cc + 0], oq[8 * cc + 1] + y[8 * cc + 1]);
                        qv.y = pack_bf16(oq[8 * cc + 2] + y[8 * cc + 2], oq[8 * cc + 3] + y[8 * cc + 3]);
                        qv.z = pack_bf16(oq[8 * cc + 4] + y[8 * cc + 4], oq[8 * cc + 5] + y[8 * cc + 5]);
                        qv.w = pack_bf16(oq[8 * cc + 6] + y[8 * cc + 6], oq[8 * cc + 7] + y[8 * cc + 7]);
                        reinterpret_cast<uint4 *>(dst)[cc] = qv;
                    }
                }
            }
            // state hand-off: S^T (already gamma-scaled + update) -> bf16 copy, pre-scale
            if (!warp_wait(cx, B_ST_FULL, c & 1)) break;
            tc_fence_after();
            {
                float sv[64];
                tmem_ld64(lane_addr + TM_ST, sv);
                if (c + 1 < NT) {
                    store_row_bf16(sb, t, sv);
                    fence_async_smem();
                    if (!warp_wait(cx, B_PREP_FULL + (s ^ 1), ((c + 1) >> 1) & 1)) break;
                    const float gl = reinterpret_cast<const float *>(base + SM_GATE)[(s ^ 1) * GATE_STRIDE + 128];
#pragma unroll
                    for (int j = 0; j < 64; ++j) sv[j] *= gl;
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        tmem_st16(lane_addr + TM_ST + 16 * j, *reinterpret_cast<float(*)[16]>(sv + 16 * j));
                    tmem_wait_st();
                } else if (p.S_T) {
#pragma unroll
                    for (int j = 0; j < 64; ++j) p.S_T[(head * p.Dv + v0 + j) * DK + t] = sv[j];
                }
                tc_fence_before();
                mbar_arrive(cx.bar + B_S_READY);
                mbar_arrive(cx.bar + B_GATE_EMPTY + s);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

// ------------------------------------------------------------------- host --
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// [B, T, H, D] bf16, box of 64 channels x 1 head x 64 tokens x 1 batch, 128B swizzle.
bool make_map(CUtensorMap *m, const void *ptr, int B, int T, int H, int D) {
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)T * H * D * 2};
    cuuint32_t box[4] = {64, 1, 64, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(ptr), dims, strides, box,
               es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tc

bool tc_supported(int B, int T, int H, int Dk, int Dv, int chunk, bool bf16) {
    return bf16 && chunk == tc::C && Dk == tc::DK && Dv % tc::DVT == 0 && B >= 1 && T >= 1 &&
           H >= 1 && tc::encode_fn() != nullptr;
}

cudaError_t launch_chunk_tc(const void *q, const void *k, const void *v, const float *log_alpha,
                            const float *beta, const float *S0, void *o, float *S_T, int B, int T,
                            int H, int Dk, int Dv, cudaStream_t st) {
    CUtensorMap mq, mk, mv;
    if (!tc::make_map(&mq, q, B, T, H, Dk) || !tc::make_map(&mk, k, B, T, H, Dk) ||
        !tc::make_map(&mv, v, B, T, H, Dv))
        return cudaErrorInvalidValue;
    tc::Params p;
    p.log_alpha = log_alpha;
    p.beta = beta;
    p.S0 = S0;
    p.o = static_cast<__nv_bfloat16 *>(o);
    p.S_T = S_T;
    p.T = T;
    p.H = H;
    p.Dv = Dv;
    p.NT = (T + tc::C - 1) / tc::C;
    cudaError_t e = cudaFuncSetAttribute(tc::gdn_chunk_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         tc::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    tc::gdn_chunk_tc_kernel<<<dim3(Dv / tc::DVT, H, B), tc::NTHREADS, tc::SMEM_BYTES, st>>>(
        mq, mk, mv, p);
    return cudaPeekAtLastError();
}

cudaError_t read_and_clear_device_error(unsigned int *flag) {
    cudaError_t e = cudaMemcpyFromSymbol(flag, g_tc_error, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_tc_error, &zero, sizeof(unsigned int));
}

}  // namespace gdn
