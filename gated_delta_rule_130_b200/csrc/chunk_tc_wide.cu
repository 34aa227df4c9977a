// Chunkwise forward of the gated delta rule on sm_100a tensor cores for wide
// heads: Dk = 256, Dv any multiple of 64 (the 1.3B-parameter layer shape has
// Dv = 512), bf16 q/k/v/o, float32 gates, state and accumulation.
//
// The chunk algebra is the one of chunk_tc.cu (the gated WY/UT form of "Gated
// Delta Networks: Improving Mamba2 with Delta Rule", section "Approach"; "Gated
// DeltaNet: Harmonizing Gating and the Delta Rule ...", section
// "Hardware-Efficient Training"), per chunk of C = 64 tokens with g_r the
// running sum of log alpha from the chunk start and gamma_r = exp(g_r):
//   A   = strictly-lower( beta_r exp(g_r - g_i) k_r . k_i ),   T = (I + A)^-1
//   P   = Q K^T o exp(g_r - g_i) o [i <= r]
//   W   = T diag(beta gamma) K,   U = T diag(beta) V,   U' = U - W S^T
//   O   = diag(gamma) Q S^T + P U'
//   S  <- gamma_last S + U'^T diag(exp(g_last - g)) K
// At Dk = 256 a chunk's key-side tiles (Q, K and W, 32 KiB each) and a 256-row
// slice of the state leave no room in one SM for chunk_tc.cu's in-kernel Gram
// and WY products next to a two-stage ring, so the key-side work moves to the
// parallel kernel:
//  1. gdn_utw_kernel, one CTA per (chunk, head), all chunks in parallel: the
//     Gram matrix and Q K^T (one tcgen05 product from TMA-loaded tiles), the
//     gating, the blocked UT solve, and W = T diag(beta gamma) K (a second
//     tcgen05 product); it writes the bf16 tiles [P; T''] (128 x 64, T'' =
//     T diag(beta)) and W (64 x 256) of each chunk to the workspace.  None of
//     it depends on the state, and it is formed once per head instead of once
//     per value slice.
//  2. gdn_chunk_tcw_kernel, one CTA per (sequence, head, 64 value channels),
//     walking the chunks in order with S^T (256 x 64, float32, as two 128-lane
//     halves) resident in tensor memory.  Products (tcgen05.mma, M = 128, bf16
//     operands in 128-byte-swizzled shared memory, float32 in TMEM):
//       X     = [Q;W] S^T             rows 0-63 Q S^T, rows 64-127 W S^T (K = 256)
//       U     = [P;T''] V             rows 64-127 U (rows 0-63 unused)     (K = 64)
//       S^T_h += K_h^T diag(exp(g_last - g)) U'   for the key halves h     (K = 64)
//       Y     = [P;T''] U'            rows 0-63 P U', Y preloaded with gamma Q S^T
//     Warp roles: 0 TMA (and gate vectors), 1 the sequential products (TMEM
//     owner), 2 the U product, 4-11 the state warps (U' = U - W S^T, the
//     output, the state hand-off).  [Q;W] and K are single-buffered and
//     refilled as soon as the product that last reads them completes; V,
//     [P;T''] and the gate vectors use a two-stage ring.
// Rows past the end of a sequence are loaded as zeros and get beta = 0 and
// log alpha = 0, which leaves the real rows' results unchanged.  Every mbarrier
// wait is bounded (about two seconds); a CTA that times out sets an error flag
// (gdn_check_device_status), stops, waits for its copies and frees its TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tc_common.cuh"

namespace gdn {

// Set by a CTA of gdn_chunk_tcw_kernel that gave up waiting.
__device__ unsigned int g_tcw_error = 0;

// Optional per-role timeline of the sequential kernel's CTA (0,0,0), chunks
// 0-63, for performance work: build with -DGDN_TRACE; that build alone exports
// gdn_tracew_wide_read() (end of this file).  Compiled out otherwise.
#ifdef GDN_TRACE
__device__ unsigned long long g_trace_wide[64 * 16];
#define TW(c, ev)                                                                       \
    do {                                                                                \
        if ((threadIdx.x & 31) == 0 && blockIdx.x == 0 && blockIdx.y == 0 &&            \
            blockIdx.z == 0 && (c) < 64)                                                \
            g_trace_wide[(c) * 16 + (ev)] = clock64();                                  \
        __syncwarp();                                                                   \
    } while (0)
#else
#define TW(c, ev) \
    do {          \
    } while (0)
#endif

namespace tcw {

using namespace sm100;
using tc::C;
using tc::Ctx;
using tc::LDA;
using tc::Seqs;
using tc::Span;

constexpr int DVT = 64;            // value channels per CTA of the sequential kernel
constexpr float LOG2E = 1.4426950408889634f;

// ------------------------------------------------------------- UT kernel --
// One CTA of 4 warps per (global chunk g, head h).  Outputs at tile index
// g H + h: [P; T''] (128 x 64 bf16, row-major), W (64 x DK bf16, row-major),
// optionally T itself (64 x 64 bf16, row-major, for the backward) and, when
// normalising, 1/|q| and 1/|k| of the chunk's rows (2 x 64 float32).
// The chunk's K and Q rows arrive by TMA (128-byte swizzle), interleaved per
// 64-key block as K | Q so that [K; Q] is one 128-row operand, and both
// products are tcgen05.mma into tensor memory:
//   G = [K; Q] K^T   (M = 128, N = 64; N = 128 with [K; Q]^T when normalising,
//                     whose diagonals give |k|^2 and |q|^2): lanes 0-63 the Gram
//                     matrix, lanes 64-127 Q K^T
//   W = T' K         (M = 64, two products of N = 128 key columns; A = T' from
//                     shared memory, B = K MN-major), after the UT solve
// An M = 64 product puts row m in TMEM lane 32 (m / 16) + m % 16.  At Dk = 256
// two CTAs fit on an SM (105 KiB of shared memory, 256 TMEM columns each), at
// Dk = 128 three (73 KiB, 128 columns).
constexpr int UT_THREADS = 128;
constexpr int SM_KQ = 0;                           // per key block: K (8 KiB), then Q (8 KiB)
constexpr int KQ_BLK = 16384;
constexpr int PT_ELEMS = 2 * C * C;
template <int DK>
struct UtDims {
    static constexpr int KB = DK / 64;                        // 64-key blocks
    static constexpr int SM_AF = SM_KQ + KB * KQ_BLK;         // A (f32, 64 x LDA); then T' (bf16, swizzled)
    static constexpr int SM_TF = SM_AF + C * LDA * 4;         // T (f32, 64 x LDA)
    static constexpr int SM_G = SM_TF + C * LDA * 4;          // 5 x 64 floats of per-row gates and norms
    static constexpr int SM_UBAR = SM_G + 5 * C * 4;          // 3 mbarriers, TMEM base, abort flag
    static constexpr int UT_SMEM = SM_UBAR + 48 + 1024;       // + alignment slack (1024-byte tiles)
    static constexpr uint32_t UT_TM_COLS = DK;                // G (<= 128 columns), then W
    static constexpr int W_ELEMS = C * DK;
    static_assert(SM_AF % 1024 == 0 && SM_TF % 16 == 0 && SM_G % 16 == 0 && SM_UBAR % 8 == 0,
                  "aligned UT buffers");
};

template <int DK, bool kNorm>
__global__ void __launch_bounds__(UT_THREADS, DK == 256 ? 2 : 3)
gdn_utw_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const float *__restrict__ log_alpha, const float *__restrict__ beta,
               __nv_bfloat16 *__restrict__ pt, __nv_bfloat16 *__restrict__ wt,
               __nv_bfloat16 *__restrict__ tr, float *__restrict__ rqk, const Seqs sq, int H,
               unsigned flags) {
    using L = UtDims<DK>;
    constexpr int KB = L::KB, SM_AF = L::SM_AF, SM_TF = L::SM_TF, SM_G = L::SM_G,
                  SM_UBAR = L::SM_UBAR, W_ELEMS = L::W_ELEMS;
    constexpr uint32_t UT_TM_COLS = L::UT_TM_COLS;
    extern __shared__ __align__(1024) uint8_t ut_raw[];
    uint8_t *sm = ut_raw + ((1024u - (smem_u32(ut_raw) & 1023u)) & 1023u);
    // the sequential kernel that follows may be scheduled now (it waits for this
    // grid's completion before it reads the tiles)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int gch = blockIdx.x, h = blockIdx.y;
    const int b = tc::seq_of_chunk(sq, gch);
    const Span sp = tc::seq_span(sq, b);
    const int c = gch - sp.chunk0, T = sp.len, t0 = c * C;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t tile = (size_t)gch * H + h;
    float *AF = reinterpret_cast<float *>(sm + SM_AF);
    float *TF = reinterpret_cast<float *>(sm + SM_TF);
    float *g2s = reinterpret_cast<float *>(sm + SM_G);
    float *bes = g2s + C, *bgs = g2s + 2 * C, *rks = g2s + 3 * C, *rqs = g2s + 4 * C;
    Ctx cx;
    cx.base = sm;
    cx.bar = reinterpret_cast<uint64_t *>(sm + SM_UBAR);  // [0] K, Q landed [1] G done [2] W done
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + SM_UBAR + 24);
    cx.abort = reinterpret_cast<volatile uint32_t *>(sm + SM_UBAR + 28);
    cx.err = &g_tcw_error;

    if (tid == 0) {
        for (int i = 0; i < 3; ++i) mbar_init(cx.bar + i, 1);
        *cx.abort = 0u;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, UT_TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    // K and Q rows of the chunk.  Rows past the end of the sequence (the next
    // sequence's, or TMA's zero fill) get beta = 0 and log alpha = 0: their rows
    // of A and their columns of T', T'' and P vanish, and their rows of P are
    // outputs of tokens that are never stored.  Warp 1 (the MMA issuer, which waits
    // for them) starts the copies, so that warp 0's gate loads start at once.
    if (tid == 32) {
        mbar_arrive_expect_tx(cx.bar + 0, 2 * KB * 8192);
#pragma unroll
        for (int kb = 0; kb < KB; ++kb) {
            tma_load_4d(sm + SM_KQ + kb * KQ_BLK, &tm_k, cx.bar + 0, kb * 64, h, sp.off + t0, 0);
            tma_load_4d(sm + SM_KQ + kb * KQ_BLK + 8192, &tm_q, cx.bar + 0, kb * 64, h,
                        sp.off + t0, 0);
        }
    }
    if (warp == 0) {
        // running sum of log alpha over rows lane and lane + 32, in log2 units
        float la[2], be[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int r = lane + 32 * hh;
            const bool in = t0 + r < T;
            const size_t gi = (size_t)(sp.off + t0 + r) * H + h;
            const float2 gp = in ? gate_pair(log_alpha[gi], beta[gi], flags) : make_float2(0.f, 0.f);
            la[hh] = gp.x;
            be[hh] = gp.y;
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
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const float g2 = la[hh] * LOG2E;
            g2s[lane + 32 * hh] = g2;
            bes[lane + 32 * hh] = be[hh];
            bgs[lane + 32 * hh] = be[hh] * tc::ex2(g2);
        }
    } else if (warp == 1) {
        const bool landed = tc::warp_wait(cx, 0, 0);
        tc_fence_after();
        if (landed && lane == 0) {
            const uint32_t kq = smem_u32(sm + SM_KQ);
            const uint32_t idesc = idesc_bf16(128, kNorm ? 128 : 64, false, false);
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk) {
                const uint32_t off = (kk >> 2) * KQ_BLK + (kk & 3) * 32;
                mma_bf16(tmem, desc_sw128(kq + off, 16, 1024), desc_sw128(kq + off, 16, 1024),
                         idesc, kk > 0);
            }
            mma_commit(cx.bar + 1);
        }
        __syncwarp();
    }
    __syncthreads();  // the gate vectors are written
    // warps 0, 1: Gram row r = 32 w + lane; warps 2, 3: Q K^T row r = 32 (w - 2) + lane
    const bool is_p = warp >= 2;
    const int r = 32 * (warp & 1) + lane;
    float row[C];
    float dg = 0.f;  // |k_r|^2 or |q_r|^2 from the diagonals
    {
        const bool done = tc::warp_wait(cx, 1, 0);
        tc_fence_after();
        if (done) {
#pragma unroll
            for (int pc = 0; pc < C / 16; ++pc) {
                float v[16];
                tmem_ld16(lane_addr + 16 * pc, v);
#pragma unroll
                for (int j = 0; j < 16; ++j) row[16 * pc + j] = v[j];
            }
            if constexpr (kNorm) {
                // Q Q^T (lanes 64-127, columns 64-127) for |q_r|^2
                float v[16];
#pragma unroll
                for (int pc = 0; pc < C / 16; ++pc) {
                    tmem_ld16(lane_addr + 64 + 16 * pc, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) dg = (16 * pc + j == r) ? v[j] : dg;
                }
                if (!is_p) {
#pragma unroll
                    for (int j = 0; j < C; ++j) dg = (j == r) ? row[j] : dg;
                }
            }
            tmem_wait_ld();
        } else {
#pragma unroll
            for (int j = 0; j < C; ++j) row[j] = 0.f;
        }
    }
    tc_fence_before();
    if constexpr (kNorm) {
        const float rn = rsqrtf(fmaxf(dg, 0.f) + kNormEps);
        if (is_p) {
            rqs[r] = rn;
        } else {
            rks[r] = rn;
            bgs[r] *= rn;
        }
        rqk[tile * 2 * C + (is_p ? 0 : C) + r] = rn;
        __syncthreads();
    }
    {
        // A_ri = beta_r exp(g_r - g_i) k_r . k_i  (i < r)      -> A (float32)
        // P_ri = exp(g_r - g_i) q_r . k_i         (i <= r)     -> [P; T''] rows 0-63
        const float grl = g2s[r];
        const float sr = is_p ? (kNorm ? rqs[r] : 1.f) : (kNorm ? bes[r] * rks[r] : bes[r]);
        __nv_bfloat16 *dp = pt + tile * PT_ELEMS + r * C;
#pragma unroll
        for (int i8 = 0; i8 < C / 8; ++i8) {
            float a[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int i = 8 * i8 + e;
                const float s = kNorm ? sr * rks[i] : sr;
                const bool keep = is_p ? (i <= r) : (i < r);
                // exponents are <= 0 where kept (g is non-increasing)
                a[e] = keep ? s * tc::ex2(grl - g2s[i]) * row[i] : 0.f;
            }
            if (is_p) {
                *reinterpret_cast<uint4 *>(dp + 8 * i8) =
                    make_uint4(tc::pack_bf16(a[0], a[1]), tc::pack_bf16(a[2], a[3]),
                               tc::pack_bf16(a[4], a[5]), tc::pack_bf16(a[6], a[7]));
            } else {
                *reinterpret_cast<float4 *>(AF + r * LDA + 8 * i8) = make_float4(a[0], a[1], a[2], a[3]);
                *reinterpret_cast<float4 *>(AF + r * LDA + 8 * i8 + 4) = make_float4(a[4], a[5], a[6], a[7]);
            }
        }
    }
    __syncthreads();  // A complete, G no longer read
    if (tid < C) tc::ut_diag(AF, TF, tid);
    __syncthreads();
    tc::ut_offdiag4(AF, TF, tid);  // ends with a CTA-wide barrier

    // T'' = T diag(beta) -> [P; T''] rows 64-127 (8 threads per 128-byte row), and
    // T' = T diag(beta gamma / |k|) as the swizzled bf16 A operand of W = T' K
    // (over the dead A buffer); both lower triangular
    {
        __nv_bfloat16 *dpt = pt + tile * PT_ELEMS + C * C;
        uint8_t *tp = sm + SM_AF;
#pragma unroll
        for (int m = 0; m < C * C / 8 / UT_THREADS; ++m) {
            const int idx = tid + UT_THREADS * m;
            const int rr = idx >> 3, i0 = 8 * (idx & 7);
            const float4 ta = *reinterpret_cast<const float4 *>(TF + rr * LDA + i0);
            const float4 tb = *reinterpret_cast<const float4 *>(TF + rr * LDA + i0 + 4);
            const float tv[8] = {ta.x, ta.y, ta.z, ta.w, tb.x, tb.y, tb.z, tb.w};
            float x[8], y[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const bool low = i0 + e <= rr;
                x[e] = low ? tv[e] * bes[i0 + e] : 0.f;
                y[e] = low ? tv[e] * bgs[i0 + e] : 0.f;
            }
            *reinterpret_cast<uint4 *>(dpt + rr * C + i0) =
                make_uint4(tc::pack_bf16(x[0], x[1]), tc::pack_bf16(x[2], x[3]),
                           tc::pack_bf16(x[4], x[5]), tc::pack_bf16(x[6], x[7]));
            *reinterpret_cast<uint4 *>(tp + sw128_offset(rr, 2 * i0)) =
                make_uint4(tc::pack_bf16(y[0], y[1]), tc::pack_bf16(y[2], y[3]),
                           tc::pack_bf16(y[4], y[5]), tc::pack_bf16(y[6], y[7]));
            if (tr) {
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = i0 + e <= rr ? tv[e] : 0.f;
                *reinterpret_cast<uint4 *>(tr + tile * C * C + rr * C + i0) =
                    make_uint4(tc::pack_bf16(x[0], x[1]), tc::pack_bf16(x[2], x[3]),
                               tc::pack_bf16(x[4], x[5]), tc::pack_bf16(x[6], x[7]));
            }
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();  // T' is in shared memory for the tensor cores
    if (warp == 1) {
        tc_fence_after();
        if (lane == 0) {
            // W = T' K: A = T' (K-major, 64 rows), B = K (MN-major: 64-key blocks
            // KQ_BLK apart, 16 chunk rows per step), 128 key columns per product
            const uint32_t tp = smem_u32(sm + SM_AF), kq = smem_u32(sm + SM_KQ);
            const uint32_t idesc = idesc_bf16(64, 128, false, true);
#pragma unroll
            for (int nh = 0; nh < DK / 128; ++nh)
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    mma_bf16(tmem + 128 * nh, desc_sw128(tp + kk * 32, 16, 1024),
                             desc_sw128(kq + nh * 2 * KQ_BLK + kk * 2048, KQ_BLK, 1024), idesc,
                             kk > 0);
            mma_commit(cx.bar + 2);
        }
        __syncwarp();
    }
    {
        // W rows: row 16 w + l % 16 in TMEM lane 32 w + l % 16; the 16-lane loads give
        // lanes 0-15 columns 16 pc .. + 15 and lanes 16-31 the next 16
        const bool done = tc::warp_wait(cx, 2, 0);
        tc_fence_after();
        const int wr = 16 * warp + (lane & 15);
        __nv_bfloat16 *dw = wt + tile * W_ELEMS + (size_t)wr * DK + 16 * (lane >> 4);
#pragma unroll 1
        for (int pc = 0; pc < DK / 16; pc += 2) {
            float v0[16];
            tmem_ld16x2<16>(lane_addr + 16 * pc, v0);
            tmem_wait_ld();
            if (done) {
                uint4 *d4 = reinterpret_cast<uint4 *>(dw + 16 * pc);
                d4[0] = make_uint4(tc::pack_bf16(v0[0], v0[1]), tc::pack_bf16(v0[2], v0[3]),
                                   tc::pack_bf16(v0[4], v0[5]), tc::pack_bf16(v0[6], v0[7]));
                d4[1] = make_uint4(tc::pack_bf16(v0[8], v0[9]), tc::pack_bf16(v0[10], v0[11]),
                                   tc::pack_bf16(v0[12], v0[13]), tc::pack_bf16(v0[14], v0[15]));
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, UT_TM_COLS);
    }
}

// ----------------------------------------------------- sequential kernel --
constexpr int BLK = 8192;                       // one 64 x 64 bf16 tile (64 rows of 128 B)
constexpr int VP_STAGE = 3 * BLK;               // V (8 KiB), [P; T''] (16 KiB)
constexpr int GV_GAM = 0;                       // gamma_r (/ |q_r| when normalising)
constexpr int GV_DCY = 64;                      // exp(g_last - g_r) (/ |k_r| when normalising)
constexpr int GV_GL = 128;                      // gamma_last
constexpr int GV_GLK = 256;                     // channel-wise gates: exp(Lam_last) per key channel
constexpr int GV_STRIDE = 512;
constexpr int NBAR = 20;

// Shared memory and TMEM of the sequential kernel for Dk = 128 or 256.  The
// [Q; W] and K tiles have NQ stages: two at Dk = 128, one at Dk = 256 (where
// two would not fit beside the 256-row state copy).
template <int DK>
struct SeqDims {
    static constexpr int KB = DK / 64;          // 64-key blocks
    static constexpr int NH = DK / 128;         // 128-lane halves of S^T
    static constexpr int NQ = DK == 128 ? 2 : 1;
    static constexpr int QW_BYTES = KB * 2 * BLK, K_BYTES = KB * BLK;
    static constexpr int SM_QW = 0;                         // per key block: Q, then W
    static constexpr int SM_KT = SM_QW + NQ * QW_BYTES;     // K, key blocks of 8 KiB
    static constexpr int SM_VP = SM_KT + NQ * K_BYTES;      // 2 stages of V, [P; T'']
    static constexpr int SM_SB = SM_VP + 2 * VP_STAGE;      // S^T bf16: DK rows x 128 B (MN-major B)
    static constexpr int SM_UN = SM_SB + DK * 128;          // U' bf16 (MN-major B)
    static constexpr int SM_UP = SM_UN + BLK;               // diag(exp(g_last - g) / |k|) U' bf16
    static constexpr int SM_GV = SM_UP + BLK;               // gate vectors, 2 stages
    static constexpr int SM_BAR = SM_GV + 2 * GV_STRIDE * 4;
    static constexpr int SM_MISC = SM_BAR + NBAR * 8;       // TMEM base, abort flag
    static constexpr int SMEM_BYTES = SM_MISC + 16 + 1024;  // + alignment slack
    // TMEM columns: S^T (keys 128 h .. in columns 64 h ..), X, U, Y
    static constexpr uint32_t TM_ST = 0, TM_X = 64 * NH, TM_U = TM_X + 64, TM_Y = TM_U + 64;
    static constexpr uint32_t TM_COLS = TM_Y + 64 <= 256 ? 256 : 512;
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
    static_assert(SM_KT % 1024 == 0 && SM_VP % 1024 == 0 && SM_SB % 1024 == 0 &&
                      SM_UN % 1024 == 0 && SM_UP % 1024 == 0 && VP_STAGE % 1024 == 0,
                  "1024-byte aligned swizzled tiles");
};

enum {
    B_QW_FULL = 0,      // [2] TMA: [Q; W] (1 + tx)
    B_QW_EMPTY = 2,     // [2] chain commit after X (1)
    B_K_FULL = 4,       // [2] TMA: K (1 + tx)
    B_K_EMPTY = 6,      // [2] chain commit after the state update (1)
    B_VP_FULL = 8,      // [2] TMA: V, [P; T''] (tx) + gate vectors (1)
    B_VP_EMPTY = 10,    // [2] chain commit after Y (1)
    B_U_FULL = 12,      // U-product commit (1)
    B_U_EMPTY = 13,     // state warps that read U (4)
    B_X_FULL = 14,      // chain commit after X (1)
    B_U_READY = 15,     // state warps: U', decayed U' and the Y preload written (8)
    B_ST_FULL = 16,     // chain commit after the state update (1)
    B_S_READY = 17,     // state warps: S^T hand-off done (8)
    B_Y_FULL = 18,      // chain commit after Y (1)
    B_COUNT = 19
};
static_assert(B_COUNT <= NBAR, "barrier slots");

constexpr int W_TMA = 0, W_CHAIN = 1, W_UMMA = 2;
constexpr int W_STATE0 = 4, NSTATEW = 8;
constexpr int NTHREADS = 32 * (W_STATE0 + NSTATEW);

struct Params {
    const float *log_alpha;
    const float *S0;
    __nv_bfloat16 *o;      // null: the output is not stored (the segment maps of a split sequence)
    float *S_T;
    const float *rqk;      // 1/|q|, 1/|k| per chunk row from the UT kernel (normalising only)
    // Channel-wise gates (chunk_cw_tc.cu): the per-chunk decay per key channel,
    // exp(Lam_last), [tiles][DK] float32.  When set, the Q, K and V operands are
    // already Q o exp(Lam), K o exp(Lam_last - Lam) and w o V, so gamma_r and
    // exp(g_last - g_r) are 1 and the state's decay is this per-key vector
    // (log_alpha is not read).
    const float *glk;
    // optional (fixed-length batches, the backward's recompute): the state entering
    // every chunk, [B*H][NT][Dv][DK] bf16
    __nv_bfloat16 *S_hist;
    // tm_v maps a 64-token zero tensor (V = 0; every later token is out of bounds
    // and loads as zeros): its L2 prefetches are skipped
    bool v_zero;
    Seqs sq;
    int H, Dv;
    unsigned flags;
};

template <int DK, bool kNorm>
__global__ void __launch_bounds__(NTHREADS, 1)
gdn_chunk_tcw_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_w,
                     const __grid_constant__ CUtensorMap tm_pt, const Params p) {
    using L = SeqDims<DK>;
    constexpr int KB = L::KB, NH = L::NH, NQ = L::NQ;
    constexpr int SM_QW = L::SM_QW, SM_KT = L::SM_KT, SM_VP = L::SM_VP, SM_SB = L::SM_SB,
                  SM_UN = L::SM_UN, SM_UP = L::SM_UP, SM_GV = L::SM_GV, SM_BAR = L::SM_BAR,
                  SM_MISC = L::SM_MISC;
    constexpr uint32_t TM_ST = L::TM_ST, TM_X = L::TM_X, TM_U = L::TM_U, TM_Y = L::TM_Y,
                       TM_COLS = L::TM_COLS;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    Ctx cx;
    cx.base = base;
    cx.bar = reinterpret_cast<uint64_t *>(base + SM_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + SM_MISC);
    cx.abort = reinterpret_cast<volatile uint32_t *>(base + SM_MISC + 4);
    cx.err = &g_tcw_error;
    float *gv_all = reinterpret_cast<float *>(base + SM_GV);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int vt = blockIdx.x, h = blockIdx.y;
    const int b = p.sq.order ? p.sq.order[blockIdx.z] : (int)blockIdx.z;
    const int v0 = vt * DVT;
    const int H = p.H;
    const Span sp = tc::seq_span(p.sq, b);
    const int T = sp.len, NT = (T + C - 1) / C;
    const size_t head = (size_t)b * H + h;
    if (NT == 0) {
        if (p.S_T)
            for (int e = threadIdx.x; e < DVT * DK; e += NTHREADS) {
                const size_t idx = head * p.Dv * DK + (size_t)v0 * DK + e;
                p.S_T[idx] = p.S0 ? p.S0[idx] : 0.f;
            }
        return;
    }

    if (tid == 0) {
        int counts[B_COUNT];
        for (int i = 0; i < B_COUNT; ++i) counts[i] = 1;
        counts[B_U_EMPTY] = NSTATEW / 2;
        counts[B_U_READY] = counts[B_S_READY] = NSTATEW;
        for (int i = 0; i < B_COUNT; ++i) mbar_init(cx.bar + i, counts[i]);
        *cx.abort = 0u;
        fence_mbar_init();
    }
    if (warp == W_CHAIN) {
        tmem_alloc(tmem_slot, TM_COLS);
        tmem_relinquish();
    }
    if (warp == W_TMA && lane == 0) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        prefetch_tensormap(&tm_w);
        prefetch_tensormap(&tm_pt);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == W_TMA) {
        // ------------------------------------------------ TMA loads, gate vectors
        float nla[2], nrq[2] = {1.f, 1.f}, nrk[2] = {1.f, 1.f};  // next chunk's gate values
        constexpr int NGL = DK / 32;                               // per-key decays per lane
        float ngl[NGL];
        const bool cw = p.glk != nullptr;
        const auto fetch = [&](int cc) {
            if (cw) {
                const size_t tl = (size_t)(sp.chunk0 + cc) * H + h;
#pragma unroll
                for (int m = 0; m < NGL; ++m) ngl[m] = p.glk[tl * DK + lane + 32 * m];
                return;
            }
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int r = lane + 32 * hh;
                const bool in = cc * C + r < T;
                const size_t gi = (size_t)(sp.off + cc * C + r) * H + h;
                nla[hh] = in ? p.log_alpha[gi] : 0.f;
                if (kNorm) {
                    const size_t tl = (size_t)(sp.chunk0 + cc) * H + h;
                    nrq[hh] = p.rqk[tl * 2 * C + r];
                    nrk[hh] = p.rqk[tl * 2 * C + C + r];
                }
            }
        };
        // the tiles (and the norms) come from the UT kernel launched just before
        // this one (programmatic dependent launch): wait for its completion
        asm volatile("griddepcontrol.wait;" ::: "memory");
        fetch(0);
        int n_vp = 0, n_qw = 0, n_k = 0;  // stages issued
        for (int c = 0; c < NT; ++c) {
            const int s = c & 1, t0 = c * C;
            const int tile = (sp.chunk0 + c) * H + h;
            float la[2] = {0.f, 0.f}, gl2[NGL];
            const float rq2[2] = {nrq[0], nrq[1]}, rk2[2] = {nrk[0], nrk[1]};
#pragma unroll
            for (int m = 0; m < NGL; ++m) gl2[m] = cw ? ngl[m] : 1.f;
            if (!cw) {
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const bool in = t0 + lane + 32 * hh < T;
                    const float x = nla[hh];
                    la[hh] = in ? ((p.flags & kFlagGateLogits) ? neg_softplus(x) : x) : 0.f;
                }
            }
            if (c + 1 < NT) fetch(c + 1);
            // V and [P; T''] of chunk c once the Y product of chunk c - 2 is done
            if (c >= 2 && !tc::warp_wait(cx, B_VP_EMPTY + s, ((c - 2) >> 1) & 1)) break;
            uint8_t *vp = base + SM_VP + s * VP_STAGE;
            if (lane == 0) {
                mbar_expect_tx(cx.bar + B_VP_FULL + s, VP_STAGE);
                tma_load_4d(vp, &tm_v, cx.bar + B_VP_FULL + s, v0, h, sp.off + t0, 0);
                tma_load_3d(vp + BLK, &tm_pt, cx.bar + B_VP_FULL + s, 0, 0, tile);
            }
            TW(c, 0);
            n_vp = c + 1;
            // gate vectors of chunk c (running sums in log2 units; rows past the
            // end carry log alpha = 0)
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
            // (channel-wise gates: la = 0, so gamma and the row decays are 1)
            gv[GV_GAM + lane] = tc::ex2(g0) * rq2[0];
            gv[GV_GAM + 32 + lane] = tc::ex2(g1) * rq2[1];
            gv[GV_DCY + lane] = tc::ex2(glast - g0) * rk2[0];
            gv[GV_DCY + 32 + lane] = tc::ex2(glast - g1) * rk2[1];
            if (lane == 0) gv[GV_GL] = tc::ex2(glast);
#pragma unroll
            for (int m = 0; m < NGL; ++m) gv[GV_GLK + lane + 32 * m] = gl2[m];
            __syncwarp();
            if (lane == 0) mbar_arrive(cx.bar + B_VP_FULL + s);
            // [Q; W] of chunk c once the X product of chunk c - NQ is done
            const int sq = c % NQ, pq = (c / NQ) & 1;
            if (c >= NQ && !tc::warp_wait(cx, B_QW_EMPTY + sq, pq ^ 1)) break;
            if (lane == 0) {
                uint8_t *qwb = base + SM_QW + sq * L::QW_BYTES;
                mbar_arrive_expect_tx(cx.bar + B_QW_FULL + sq, L::QW_BYTES);
#pragma unroll
                for (int kb = 0; kb < KB; ++kb) {
                    tma_load_4d(qwb + kb * 2 * BLK, &tm_q, cx.bar + B_QW_FULL + sq, kb * 64, h,
                                sp.off + t0, 0);
                    tma_load_3d(qwb + kb * 2 * BLK + BLK, &tm_w, cx.bar + B_QW_FULL + sq,
                                kb * 64, 0, tile);
                }
            }
            TW(c, 1);
            n_qw = c + 1;
            // K of chunk c once the state update of chunk c - NQ is done
            if (c >= NQ && !tc::warp_wait(cx, B_K_EMPTY + sq, pq ^ 1)) break;
            if (lane == 0) {
                uint8_t *ktb = base + SM_KT + sq * L::K_BYTES;
                mbar_arrive_expect_tx(cx.bar + B_K_FULL + sq, L::K_BYTES);
#pragma unroll
                for (int kb = 0; kb < KB; ++kb)
                    tma_load_4d(ktb + kb * BLK, &tm_k, cx.bar + B_K_FULL + sq, kb * 64, h,
                                sp.off + t0, 0);
                // a later chunk's tiles start streaming from DRAM into L2 now
                const int cq = c + 2;
                if (cq < NT) {
                    const int tq = (sp.chunk0 + cq) * H + h;
#pragma unroll
                    for (int kb = 0; kb < KB; ++kb) {
                        tma_prefetch_l2_4d(&tm_q, kb * 64, h, sp.off + cq * C, 0);
                        tma_prefetch_l2_4d(&tm_k, kb * 64, h, sp.off + cq * C, 0);
                        tma_prefetch_l2_3d(&tm_w, kb * 64, 0, tq);
                    }
                    if (!p.v_zero) tma_prefetch_l2_4d(&tm_v, v0, h, sp.off + cq * C, 0);
                    tma_prefetch_l2_3d(&tm_pt, 0, 0, tq);
                }
            }
            TW(c, 2);
            n_k = c + 1;
        }
        // never leave with copies in flight: wait (bounded) for the last phases
        if (lane == 0) {
            const auto drain = [&](uint64_t *bar, uint32_t parity) {
                const uint64_t t0 = tc::now_ns();
                while (!mbar_try_wait(bar, parity) && tc::now_ns() - t0 < tc::kTimeoutNs) {
                }
            };
            for (int c = n_qw - NQ < 0 ? 0 : n_qw - NQ; c < n_qw; ++c)
                drain(cx.bar + B_QW_FULL + c % NQ, (c / NQ) & 1);
            for (int c = n_k - NQ < 0 ? 0 : n_k - NQ; c < n_k; ++c)
                drain(cx.bar + B_K_FULL + c % NQ, (c / NQ) & 1);
            for (int c = n_vp - 2 < 0 ? 0 : n_vp - 2; c < n_vp; ++c)
                drain(cx.bar + B_VP_FULL + (c & 1), (c >> 1) & 1);
        }
    } else if (warp == W_UMMA) {
        // ---------------------------------------------- MMA: U = [P; T''] V
        const uint32_t idesc_u = idesc_bf16(128, DVT, false, true);
        for (int c = 0; c < NT; ++c) {
            const int s = c & 1;
            const uint32_t vp = smem_u32(base + SM_VP + s * VP_STAGE);
            if (!tc::warp_wait(cx, B_VP_FULL + s, (c >> 1) & 1)) break;
            if (c >= 1 && !tc::warp_wait(cx, B_U_EMPTY, (c - 1) & 1)) break;
            tc_fence_after();
            if (lane == 0) {
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    mma_bf16(tmem + TM_U, desc_sw128(vp + BLK + kk * 32, 16, 1024),
                             desc_sw128(vp + kk * 2048, 16, 1024), idesc_u, kk > 0);
                mma_commit(cx.bar + B_U_FULL);
            }
            __syncwarp();
            TW(c, 3);
        }
    } else if (warp == W_CHAIN) {
        // ---------------------------------------------- MMA: sequential chain
        const uint32_t idesc_x = idesc_bf16(128, DVT, false, true);
        const uint32_t idesc_s = idesc_bf16(128, DVT, true, true);
        const uint32_t sb = smem_u32(base + SM_SB), un = smem_u32(base + SM_UN),
                       up = smem_u32(base + SM_UP);
        for (int c = 0; c < NT; ++c) {
            const int s = c & 1, sq = c % NQ, pq = (c / NQ) & 1;
            const uint32_t vp = smem_u32(base + SM_VP + s * VP_STAGE);
            const uint32_t qw = smem_u32(base + SM_QW + sq * L::QW_BYTES);
            const uint32_t kt = smem_u32(base + SM_KT + sq * L::K_BYTES);
            if (!tc::warp_wait(cx, B_QW_FULL + sq, pq)) break;
            if (!tc::warp_wait(cx, B_S_READY, c & 1)) break;
            TW(c, 4);
            tc_fence_after();
            // X = [Q; W] S^T: A K-major (per key block, Q rows then W rows), B = S^T MN-major
            if (lane == 0) {
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk)
                    mma_bf16(tmem + TM_X, desc_sw128(qw + (kk >> 2) * 2 * BLK + (kk & 3) * 32, 16, 1024),
                             desc_sw128(sb + kk * 2048, 16, 1024), idesc_x, kk > 0);
                mma_commit(cx.bar + B_X_FULL);
                mma_commit(cx.bar + B_QW_EMPTY + sq);
            }
            __syncwarp();
            TW(c, 5);
            if (!tc::warp_wait(cx, B_U_READY, c & 1)) break;
            if (!tc::warp_wait(cx, B_K_FULL + sq, pq)) break;
            if (!tc::warp_wait(cx, B_VP_FULL + s, (c >> 1) & 1)) break;
            TW(c, 6);
            tc_fence_after();
            if (lane == 0) {
                // S^T_h += K_h^T (decayed U') for the key halves: A = K^T (MN-major,
                // two 64-key blocks 8 KiB apart), B = decayed U' (MN-major)
#pragma unroll
                for (int hk = 0; hk < NH; ++hk)
#pragma unroll
                    for (int kk = 0; kk < C / 16; ++kk)
                        mma_bf16(tmem + TM_ST + 64 * hk,
                                 desc_sw128(kt + hk * 2 * BLK + kk * 2048, BLK, 1024),
                                 desc_sw128(up + kk * 2048, 16, 1024), idesc_s, 1u);
                mma_commit(cx.bar + B_ST_FULL);
                mma_commit(cx.bar + B_K_EMPTY + sq);
                // Y += [P; T''] U'  (Y holds gamma Q S^T; rows 64-127 unused); a call
                // without an output (the states alone) skips it
                if (p.o) {
#pragma unroll
                    for (int kk = 0; kk < C / 16; ++kk)
                        mma_bf16(tmem + TM_Y, desc_sw128(vp + BLK + kk * 32, 16, 1024),
                                 desc_sw128(un + kk * 2048, 16, 1024), idesc_x, 1u);
                    mma_commit(cx.bar + B_Y_FULL);
                }
                mma_commit(cx.bar + B_VP_EMPTY + s);
            }
            __syncwarp();
            TW(c, 7);
        }
    } else if (warp >= W_STATE0) {
        // ------------------------------------------------------------ STATE
        // warp w reads TMEM lanes 32 (w % 4) .. + 31; hf selects the 32-column
        // half of X / U / Y (epilogues) and, in the hand-off, the key half of S^T
        // (Dk = 256: 64 value columns of keys 128 hf + lane) or the 32 value
        // columns (Dk = 128)
        constexpr int NPC = 2 * NH;  // 16-column pieces of S^T per thread
        const int q = warp & 3, hf = (warp - W_STATE0) >> 2;
        const int lrow = 32 * q + lane;
        const int key = (NH == 2 ? 128 * hf : 0) + lrow;  // this thread's row of S^T
        const int col0 = NH == 2 ? 0 : 32 * hf;           // its first value column
        const uint32_t lane_addr = tmem + ((uint32_t)(q * 32) << 16);
        const uint32_t st_col = TM_ST + (NH == 2 ? 64 * hf : 0) + col0;
        uint8_t *sbuf = base + SM_SB;
        // initial state: S^T row `key` = S0[v0 .. v0 + 63][key]; TMEM copy pre-scaled by gamma_last
        const bool cw = p.glk != nullptr;
        {
            const bool have = tc::warp_wait(cx, B_VP_FULL + 0, 0);
            const float gl = cw ? gv_all[GV_GLK + key] : gv_all[GV_GL];
#pragma unroll
            for (int pc = 0; pc < NPC; ++pc) {
                float sv[16];
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    sv[j] = p.S0 ? p.S0[(head * p.Dv + v0 + col0 + 16 * pc + j) * DK + key] : 0.f;
                tc::store16_bf16(sbuf, key, col0 / 16 + pc, sv);
                if (p.S_hist)
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        p.S_hist[((size_t)head * NT * p.Dv + v0 + col0 + 16 * pc + j) * DK + key] =
                            __float2bfloat16_rn(sv[j]);
#pragma unroll
                for (int j = 0; j < 16; ++j) sv[j] *= gl;
                if (have) tmem_st16(lane_addr + st_col + 16 * pc, sv);
            }
            fence_async_smem();
            tmem_wait_st();
            tc_fence_before();
            tc::warp_arrive(cx, B_S_READY);
        }
        for (int c = 0; c < NT; ++c) {
            if (__any_sync(0xffffffffu, *cx.abort != 0u)) break;
            const int s = c & 1, t0 = c * C;
            const float *gv = gv_all + s * GV_STRIDE;
            if (!tc::warp_wait(cx, B_X_FULL, c & 1)) break;
            if (warp == W_STATE0 + 2) TW(c, 8);
            tc_fence_after();
            if (q >= 2) {
                // U' = U - W S^T for chunk row r -> U' and its decayed copy (bf16)
                const int r = lrow - 64;
                if (!tc::warp_wait(cx, B_U_FULL, c & 1)) break;
                tc_fence_after();
                const float dc = gv[GV_DCY + r];
                float x0[16], x1[16], u0[16], u1[16];
                tmem_ld16(lane_addr + TM_X + 32 * hf, x0);
                tmem_ld16(lane_addr + TM_X + 32 * hf + 16, x1);
                tmem_ld16(lane_addr + TM_U + 32 * hf, u0);
                tmem_ld16(lane_addr + TM_U + 32 * hf + 16, u1);
                tmem_wait_ld();
                tc_fence_before();
                tc::warp_arrive(cx, B_U_EMPTY);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    u0[j] -= x0[j];
                    u1[j] -= x1[j];
                }
                tc::store16_bf16(base + SM_UN, r, 2 * hf, u0);
                tc::store16_bf16(base + SM_UN, r, 2 * hf + 1, u1);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    u0[j] *= dc;
                    u1[j] *= dc;
                }
                tc::store16_bf16(base + SM_UP, r, 2 * hf, u0);
                tc::store16_bf16(base + SM_UP, r, 2 * hf + 1, u1);
                fence_async_smem();
                tc_fence_before();
                tc::warp_arrive(cx, B_U_READY);
                if (warp == W_STATE0 + 2) TW(c, 9);
            } else {
                // inter-chunk part of the output, gamma_r (Q S^T)_r, into Y (when there
                // is an output)
                if (p.o) {
                    const float gr = gv[GV_GAM + lrow];
                    float x0[16], x1[16];
                    tmem_ld16(lane_addr + TM_X + 32 * hf, x0);
                    tmem_ld16(lane_addr + TM_X + 32 * hf + 16, x1);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        x0[j] *= gr;
                        x1[j] *= gr;
                    }
                    tmem_st16(lane_addr + TM_Y + 32 * hf, x0);
                    tmem_st16(lane_addr + TM_Y + 32 * hf + 16, x1);
                    tmem_wait_st();
                }
                tc_fence_before();
                tc::warp_arrive(cx, B_U_READY);
                if (warp == W_STATE0) TW(c, 13);
            }
            // state hand-off: S^T (updated) -> bf16 copy; TMEM pre-scaled by the
            // next chunk's gamma_last
            if (!tc::warp_wait(cx, B_ST_FULL, c & 1)) break;
            if (warp == W_STATE0) TW(c, 10);
            tc_fence_after();
            {
                const bool last = c + 1 >= NT;
                bool have = false;
                float gl = 1.f;
                if (!last) {
                    have = tc::warp_wait(cx, B_VP_FULL + (s ^ 1), ((c + 1) >> 1) & 1);
                    gl = gv_all[(s ^ 1) * GV_STRIDE + (cw ? GV_GLK + key : GV_GL)];
                }
                float sv[NPC][16];
#pragma unroll
                for (int pc = 0; pc < NPC; ++pc) tmem_ld16(lane_addr + st_col + 16 * pc, sv[pc]);
                tmem_wait_ld();
                if (!last) {
#pragma unroll
                    for (int pc = 0; pc < NPC; ++pc) tc::store16_bf16(sbuf, key, col0 / 16 + pc, sv[pc]);
#pragma unroll
                    for (int pc = 0; pc < NPC; ++pc)
#pragma unroll
                        for (int j = 0; j < 16; ++j) sv[pc][j] *= gl;
                    if (have)
#pragma unroll
                        for (int pc = 0; pc < NPC; ++pc) tmem_st16(lane_addr + st_col + 16 * pc, sv[pc]);
                    fence_async_smem();
                    tmem_wait_st();
                } else if (p.S_T) {
#pragma unroll
                    for (int pc = 0; pc < NPC; ++pc)
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            p.S_T[(head * p.Dv + v0 + col0 + 16 * pc + j) * DK + key] = sv[pc][j];
                }
                tc_fence_before();
                tc::warp_arrive(cx, B_S_READY);
                if (warp == W_STATE0) TW(c, 11);
                if (!last && p.S_hist) {
                    // the state entering chunk c + 1, from this thread's own bf16 row
                    // of the copy (after the hand-off, beside the next X product)
                    auto *dst = reinterpret_cast<unsigned short *>(p.S_hist) +
                                (((size_t)head * NT + c + 1) * p.Dv + v0 + col0) * DK + key;
#pragma unroll
                    for (int pc = 0; pc < NPC; ++pc)
#pragma unroll
                        for (int k8 = 0; k8 < 2; ++k8) {
                            const uint4 u = *reinterpret_cast<const uint4 *>(
                                sbuf + sw128_offset(key, (2 * (col0 / 16 + pc) + k8) * 16));
                            const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                dst[(size_t)(16 * pc + 8 * k8 + e) * DK] =
                                    (unsigned short)(e & 1 ? wd[e >> 1] >> 16 : wd[e >> 1] & 0xffffu);
                        }
                }
                if (!last && !have) break;
            }
            // chunk output rows (TMEM lanes 0-63)
            if (q < 2 && p.o) {
                if (!tc::warp_wait(cx, B_Y_FULL, c & 1)) break;
                tc_fence_after();
                float y0[16], y1[16];
                tmem_ld16(lane_addr + TM_Y + 32 * hf, y0);
                tmem_ld16(lane_addr + TM_Y + 32 * hf + 16, y1);
                tmem_wait_ld();
                if (t0 + lrow < T) {
                    uint4 *dst = reinterpret_cast<uint4 *>(
                        p.o + ((size_t)(sp.off + t0 + lrow) * H + h) * p.Dv + v0 + 32 * hf);
#pragma unroll
                    for (int kq = 0; kq < 2; ++kq) {
                        dst[kq] = make_uint4(tc::pack_bf16(y0[8 * kq + 0], y0[8 * kq + 1]),
                                             tc::pack_bf16(y0[8 * kq + 2], y0[8 * kq + 3]),
                                             tc::pack_bf16(y0[8 * kq + 4], y0[8 * kq + 5]),
                                             tc::pack_bf16(y0[8 * kq + 6], y0[8 * kq + 7]));
                        dst[2 + kq] = make_uint4(tc::pack_bf16(y1[8 * kq + 0], y1[8 * kq + 1]),
                                                 tc::pack_bf16(y1[8 * kq + 2], y1[8 * kq + 3]),
                                                 tc::pack_bf16(y1[8 * kq + 4], y1[8 * kq + 5]),
                                                 tc::pack_bf16(y1[8 * kq + 6], y1[8 * kq + 7]));
                    }
                }
                tc_fence_before();
                if (warp == W_STATE0) TW(c, 12);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == W_CHAIN) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

// W tiles, [n_tiles, 64, DK] bf16: box of 64 keys x 64 rows of one tile, 128B swizzle.
bool make_map_w(CUtensorMap *m, const void *ptr, long long n_tiles, int DK) {
    auto enc = tc::encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)DK, (cuuint64_t)C, (cuuint64_t)n_tiles};
    cuuint64_t strides[2] = {(cuuint64_t)DK * 2, (cuuint64_t)C * DK * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)C, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box,
               es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tcw

// Workspace: [chunk offsets and launch order, variable lengths only][[P; T'']
// tiles][W tiles][1/|q|, 1/|k| per chunk row, normalising only].
size_t tcw_workspace_bytes_seqs(int n_seq, long long total_chunks, int H, bool varlen,
                                unsigned flags, int Dk) {
    const size_t tiles = (size_t)total_chunks * H;
    const size_t norm = (flags & kFlagL2Norm) ? tiles * 2 * tc::C * sizeof(float) : 0;
    return tc_offsets_bytes(n_seq, varlen) +
           tiles * (tcw::PT_ELEMS + (size_t)tc::C * Dk) * sizeof(__nv_bfloat16) + norm;
}

namespace tcw {

template <int DK, bool kNorm>
cudaError_t launch(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                   const CUtensorMap &mw, const CUtensorMap &mp, const Params &p,
                   const float *log_alpha, const float *beta, __nv_bfloat16 *pt,
                   __nv_bfloat16 *wt, float *rqk, long long total_chunks, int n_seq,
                   cudaStream_t st) {
    auto *ut = gdn_utw_kernel<DK, kNorm>;
    auto *seq = gdn_chunk_tcw_kernel<DK, kNorm>;
    constexpr int ut_smem = UtDims<DK>::UT_SMEM, seq_smem = SeqDims<DK>::SMEM_BYTES;
    cudaError_t e = cudaFuncSetAttribute(ut, cudaFuncAttributeMaxDynamicSharedMemorySize, ut_smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(seq, cudaFuncAttributeMaxDynamicSharedMemorySize, seq_smem);
    if (e != cudaSuccess) return e;
    if (total_chunks > 0)
        ut<<<dim3((unsigned)total_chunks, p.H, 1), UT_THREADS, ut_smem, st>>>(
            mq, mk, log_alpha, beta, pt, wt, nullptr, rqk, p.sq, p.H, p.flags);
    e = cudaPeekAtLastError();
    if (e != cudaSuccess) return e;
    // programmatic dependent launch: the CTAs may set up while the UT kernel
    // drains; the TMA warp waits for its completion before the first load
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.Dv / DVT, p.H, n_seq);
    cfg.blockDim = dim3(NTHREADS);
    cfg.dynamicSmemBytes = seq_smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, seq, mq, mk, mv, mw, mp, p);
    if (e != cudaSuccess) return e;
    return cudaPeekAtLastError();
}

}  // namespace tcw

// ------------------------------------------------------------ split sequences
// Where the sequential grid covers less than a quarter of the GPU, each sequence of
// a fixed-length batch (Dk = 128, T a multiple of the segment length) is cut into
// G segments of whole chunks and the chain runs on all segments at once.  The
// chunk recurrence is affine in the state, so a segment maps its start state to
// its end state as S_end = S_start M + N (M = the product over its chunks of
// gamma_last I - W^T diag(exp(g_last - g)) K, Dk x Dk; N its end state from a zero
// start): pass 1 forms N (the chain from S = 0) and M (the chain with V = 0 from
// S = I, Dk rows of "values") for every segment but the last of each sequence, a
// scan (chunk_split.cu) chains the segments' start states, and pass 2 runs the
// chain on every segment from its true start state for the outputs and the final
// state.  About three chain passes over the sequence instead of one, on G times as
// many CTAs.
int tcw_split_segments(int B, int T, int H, int Dk, int Dv) {
    static const int sms = [] {
        int dev = 0, n = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
            n = 148;
        return n;
    }();
    if (Dk != 128 || B < 1 || T < 1 || T % tc::C != 0 || Dv % tcw::DVT != 0) return 1;
    const long long ctas = (long long)(Dv / tcw::DVT) * H * B;
    if (ctas * 4 > sms) return 1;
    const int NT = T / tc::C;
    for (int G = 8; G >= 2; --G)
        if (NT % G == 0 && NT / G >= 16 && ctas * G <= sms) return G;
    return 1;
}

namespace tcw {

// Regions of a split call's workspace after the tiles ([P; T''], W, 1/|q| and 1/|k|):
// N and S_T of every segment ([B G][H][Dv][128] float32), M ([B G][H][128][128]),
// the segments' start states ([B G][H][Dv][128]), 64 zero token rows ([64][H][128]
// bf16) and pass 1's launch order (the segments but the last of each sequence).
struct SplitWs {
    __nv_bfloat16 *pt, *wt, *zrow;
    float *rqk, *N, *M, *Ss, *STs;
    int *order;
    size_t bytes;
};

inline size_t up256(size_t n) { return (n + 255) & ~size_t(255); }

SplitWs split_carve(void *base, int B, int T, int H, int Dv, unsigned flags) {
    constexpr int DK = 128;
    const int G = tcw_split_segments(B, T, H, DK, Dv);
    const long long NT = T / tc::C, total_chunks = (long long)B * NT;
    const size_t tiles = (size_t)total_chunks * H;
    const size_t nseg = (size_t)B * G * H;
    const size_t sz[9] = {tiles * PT_ELEMS * 2, tiles * tc::C * DK * 2,
                          (flags & kFlagL2Norm) ? tiles * 2 * tc::C * 4 : 0,
                          nseg * Dv * DK * 4, nseg * DK * DK * 4, nseg * Dv * DK * 4,
                          nseg * Dv * DK * 4, (size_t)tc::C * H * DK * 2,
                          (size_t)B * G * sizeof(int)};
    uint8_t *p = static_cast<uint8_t *>(base);
    size_t off[9], o = 0;
    for (int i = 0; i < 9; ++i) {
        off[i] = o;
        o += up256(sz[i]);
    }
    SplitWs w;
    w.pt = reinterpret_cast<__nv_bfloat16 *>(p + off[0]);
    w.wt = reinterpret_cast<__nv_bfloat16 *>(p + off[1]);
    w.rqk = sz[2] ? reinterpret_cast<float *>(p + off[2]) : nullptr;
    w.N = reinterpret_cast<float *>(p + off[3]);
    w.M = reinterpret_cast<float *>(p + off[4]);
    w.Ss = reinterpret_cast<float *>(p + off[5]);
    w.STs = reinterpret_cast<float *>(p + off[6]);
    w.zrow = reinterpret_cast<__nv_bfloat16 *>(p + off[7]);
    w.order = reinterpret_cast<int *>(p + off[8]);
    w.bytes = o;
    return w;
}

template <bool kNorm>
cudaError_t launch_split_t(const void *q, const void *k, const void *v, const float *log_alpha,
                           const float *beta, const float *S0, void *o, float *S_T, int B, int T,
                           int H, int Dv, unsigned flags, void *workspace, cudaStream_t st) {
    constexpr int DK = 128;
    const int G = tcw_split_segments(B, T, H, DK, Dv);
    const int NT = T / tc::C, nseg = B * G;
    const long long total_chunks = (long long)B * NT, n_tiles = total_chunks * H;
    SplitWs w = split_carve(workspace, B, T, H, Dv, flags);
    CUtensorMap mq, mk, mv, mz, mw, mp;
    if (!tc::make_map(&mq, q, 1, B * T, H, DK) || !tc::make_map(&mk, k, 1, B * T, H, DK) ||
        !tc::make_map(&mv, v, 1, B * T, H, Dv) || !tc::make_map(&mz, w.zrow, 1, tc::C, H, DK) ||
        !make_map_w(&mw, w.wt, n_tiles, DK) || !tc::make_map_tt(&mp, w.pt, n_tiles))
        return cudaErrorInvalidValue;
    // M = I for every segment, the zero token rows, pass 1's order
    cudaError_t e = launch_split_init(w.M, (long long)nseg * H, w.zrow, tc::C * H, w.order, B, G, st);
    if (e != cudaSuccess) return e;
    // the tiles of every chunk, once (the sequences as given)
    auto *ut = gdn_utw_kernel<DK, kNorm>;
    auto *seq = gdn_chunk_tcw_kernel<DK, kNorm>;
    constexpr int ut_smem = UtDims<DK>::UT_SMEM, seq_smem = SeqDims<DK>::SMEM_BYTES;
    e = cudaFuncSetAttribute(ut, cudaFuncAttributeMaxDynamicSharedMemorySize, ut_smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(seq, cudaFuncAttributeMaxDynamicSharedMemorySize, seq_smem);
    if (e != cudaSuccess) return e;
    ut<<<dim3((unsigned)total_chunks, H, 1), UT_THREADS, ut_smem, st>>>(
        mq, mk, log_alpha, beta, w.pt, w.wt, nullptr, w.rqk, tc::Seqs{nullptr, nullptr, nullptr, T, B},
        H, flags);
    e = cudaPeekAtLastError();
    if (e != cudaSuccess) return e;
    // the segments as sequences of T / G tokens: global chunk b NT + c keeps its tile
    Params p;
    p.log_alpha = log_alpha;
    p.rqk = w.rqk;
    p.glk = nullptr;
    p.S_hist = nullptr;
    p.sq = tc::Seqs{nullptr, nullptr, nullptr, T / G, nseg};
    p.H = H;
    p.flags = flags;
    // pdl: programmatic dependent launch after the previous kernel (the state warps
    // read S0 before the TMA warp's wait, so only where S0 was written earlier)
    const auto run = [&](const CUtensorMap &vmap, int dv, bool pdl, int n_ctas_z) -> cudaError_t {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(dv / DVT, H, n_ctas_z);
        cfg.blockDim = dim3(NTHREADS);
        cfg.dynamicSmemBytes = seq_smem;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = pdl ? 1 : 0;
        p.Dv = dv;
        const cudaError_t e1 = cudaLaunchKernelEx(&cfg, seq, mq, mk, vmap, mw, mp, p);
        return e1 != cudaSuccess ? e1 : cudaPeekAtLastError();
    };
    // pass 1, every segment but the last of each sequence (blockIdx.z through the
    // order array): N from a zero start; M with V = 0 from S = I (in place)
    p.sq.order = w.order;
    p.S0 = nullptr;
    p.S_T = w.N;
    p.o = nullptr;
    p.v_zero = false;
    if ((e = run(mv, Dv, true, B * (G - 1))) != cudaSuccess) return e;
    p.S0 = w.M;
    p.S_T = w.M;
    p.v_zero = true;
    if ((e = run(mz, DK, true, B * (G - 1))) != cudaSuccess) return e;
    p.sq.order = nullptr;
    // the segments' start states
    if ((e = launch_split_scan(S0, w.N, w.M, w.Ss, B, G, H, Dv, st)) != cudaSuccess) return e;
    // pass 2: every segment from its start state
    p.S0 = w.Ss;
    p.S_T = w.STs;
    p.o = static_cast<__nv_bfloat16 *>(o);
    p.v_zero = false;
    if ((e = run(mv, Dv, false, nseg)) != cudaSuccess) return e;
    if (S_T) {
        const size_t per = (size_t)H * Dv * DK;
        for (int b = 0; b < B; ++b) {
            e = cudaMemcpyAsync(S_T + b * per, w.STs + ((size_t)b * G + G - 1) * per,
                                per * sizeof(float), cudaMemcpyDeviceToDevice, st);
            if (e != cudaSuccess) return e;
        }
    }
    return cudaSuccess;
}

}  // namespace tcw

size_t tcw_split_workspace_bytes(int B, int T, int H, int Dv, unsigned flags) {
    return tcw::split_carve(nullptr, B, T, H, Dv, flags).bytes;
}

cudaError_t launch_chunk_tcw_split(const void *q, const void *k, const void *v,
                                   const float *log_alpha, const float *beta, const float *S0,
                                   void *o, float *S_T, int B, int T, int H, int Dv,
                                   unsigned flags, void *workspace, cudaStream_t st) {
    return (flags & kFlagL2Norm)
               ? tcw::launch_split_t<true>(q, k, v, log_alpha, beta, S0, o, S_T, B, T, H, Dv,
                                           flags, workspace, st)
               : tcw::launch_split_t<false>(q, k, v, log_alpha, beta, S0, o, S_T, B, T, H, Dv,
                                            flags, workspace, st);
}

cudaError_t launch_chunk_tcw_seqs(const void *q, const void *k, const void *v,
                                  const float *log_alpha, const float *beta, const float *S0,
                                  void *o, float *S_T, int n_seq, int T_fixed, long long total_T,
                                  const int *cu_seqlens, long long total_chunks, int H, int Dk,
                                  int Dv, unsigned flags, void *workspace, cudaStream_t st) {
    if (Dk != 128 && Dk != 256) return cudaErrorInvalidValue;
    const bool varlen = cu_seqlens != nullptr;
    if (!varlen && n_seq > 0 && tcw_split_segments(n_seq, T_fixed, H, Dk, Dv) > 1)
        return launch_chunk_tcw_split(q, k, v, log_alpha, beta, S0, o, S_T, n_seq, T_fixed, H, Dv,
                                      flags, workspace, st);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int *cu_chunks = varlen ? reinterpret_cast<int *>(ws) : nullptr;
    const size_t tiles = (size_t)total_chunks * H;
    auto *pt = reinterpret_cast<__nv_bfloat16 *>(ws + tc_offsets_bytes(n_seq, varlen));
    __nv_bfloat16 *wt = pt + tiles * tcw::PT_ELEMS;
    float *rqk = (flags & kFlagL2Norm) ? reinterpret_cast<float *>(wt + tiles * tc::C * Dk)
                                       : nullptr;
    const long long n_maps = total_chunks > 0 ? (long long)tiles : 1;
    CUtensorMap mq, mk, mv, mw, mp;
    if (!tc::make_map(&mq, q, 1, (int)total_T, H, Dk) ||
        !tc::make_map(&mk, k, 1, (int)total_T, H, Dk) ||
        !tc::make_map(&mv, v, 1, (int)total_T, H, Dv) || !tcw::make_map_w(&mw, wt, n_maps, Dk) ||
        !tc::make_map_tt(&mp, pt, n_maps))
        return cudaErrorInvalidValue;
    if (varlen) {
        const cudaError_t e0 = launch_seq_schedule(cu_seqlens, n_seq, cu_chunks,
                                                   cu_chunks + n_seq + 1, st);
        if (e0 != cudaSuccess) return e0;
    }
    tcw::Params p;
    p.log_alpha = log_alpha;
    p.S0 = S0;
    p.o = static_cast<__nv_bfloat16 *>(o);
    p.S_T = S_T;
    p.rqk = rqk;
    p.glk = nullptr;
    p.S_hist = nullptr;
    p.v_zero = false;
    p.sq = tc::Seqs{cu_seqlens, cu_chunks, varlen ? cu_chunks + n_seq + 1 : nullptr, T_fixed,
                    n_seq};
    p.H = H;
    p.Dv = Dv;
    p.flags = flags;
    const bool norm = (flags & kFlagL2Norm) != 0;
    if (Dk == 256)
        return norm ? tcw::launch<256, true>(mq, mk, mv, mw, mp, p, log_alpha, beta, pt, wt, rqk,
                                             total_chunks, n_seq, st)
                    : tcw::launch<256, false>(mq, mk, mv, mw, mp, p, log_alpha, beta, pt, wt, rqk,
                                              total_chunks, n_seq, st);
    return norm ? tcw::launch<128, true>(mq, mk, mv, mw, mp, p, log_alpha, beta, pt, wt, rqk,
                                         total_chunks, n_seq, st)
                : tcw::launch<128, false>(mq, mk, mv, mw, mp, p, log_alpha, beta, pt, wt, rqk,
                                          total_chunks, n_seq, st);
}

cudaError_t launch_chunk_tcw_seq_cw(const void *qe, const void *kd, const void *vw,
                                    const void *pt, const void *wt, const float *glk,
                                    const float *S0, void *o, float *S_T, int B, int T, int H,
                                    int Dv, cudaStream_t st) {
    constexpr int DK = 128;
    const long long NT = ((long long)T + tc::C - 1) / tc::C;
    const long long n_tiles = (long long)B * NT * H;
    CUtensorMap mq, mk, mv, mw, mp;
    if (!tc::make_map(&mq, qe, 1, B * T, H, DK) || !tc::make_map(&mk, kd, 1, B * T, H, DK) ||
        !tc::make_map(&mv, vw, 1, B * T, H, Dv) || !tcw::make_map_w(&mw, wt, n_tiles, DK) ||
        !tc::make_map_tt(&mp, pt, n_tiles))
        return cudaErrorInvalidValue;
    tcw::Params p;
    p.log_alpha = nullptr;
    p.S0 = S0;
    p.o = static_cast<__nv_bfloat16 *>(o);
    p.S_T = S_T;
    p.rqk = nullptr;
    p.glk = glk;
    p.S_hist = nullptr;
    p.v_zero = false;
    p.sq = tc::Seqs{nullptr, nullptr, nullptr, T, B};
    p.H = H;
    p.Dv = Dv;
    p.flags = 0u;
    auto *seq = tcw::gdn_chunk_tcw_kernel<DK, false>;
    constexpr int seq_smem = tcw::SeqDims<DK>::SMEM_BYTES;
    cudaError_t e = cudaFuncSetAttribute(seq, cudaFuncAttributeMaxDynamicSharedMemorySize, seq_smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(Dv / tcw::DVT, H, B);
    cfg.blockDim = dim3(tcw::NTHREADS);
    cfg.dynamicSmemBytes = seq_smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, seq, mq, mk, mv, mw, mp, p);
    if (e != cudaSuccess) return e;
    return cudaPeekAtLastError();
}

// The backward's recompute (Dk = 128, gates as given, B sequences of T tokens):
// the parallel kernel writes per chunk and head the [P; T''] tile, the W tile and
// T itself (tile index (b NT + c) H + h); the sequential kernel, fed those tiles,
// records the state entering every chunk in bf16 ([B*H][NT][Dv][128]) and forms
// no output.
cudaError_t launch_recompute_bwd(const void *q, const void *k, const void *v,
                                 const float *log_alpha, const float *beta, const float *S0,
                                 int B, int T, int H, int Dv, void *pt, void *wt, void *tr,
                                 void *S_hist, cudaStream_t st) {
    constexpr int DK = 128;
    const long long NT = ((long long)T + tc::C - 1) / tc::C;
    if (B < 1 || NT < 1) return cudaSuccess;
    CUtensorMap mq, mk;
    if (!tc::make_map(&mq, q, 1, B * T, H, DK) || !tc::make_map(&mk, k, 1, B * T, H, DK))
        return cudaErrorInvalidValue;
    auto *ut = tcw::gdn_utw_kernel<DK, false>;
    constexpr int ut_smem = tcw::UtDims<DK>::UT_SMEM;
    cudaError_t e = cudaFuncSetAttribute(ut, cudaFuncAttributeMaxDynamicSharedMemorySize, ut_smem);
    if (e != cudaSuccess) return e;
    const tc::Seqs sq{nullptr, nullptr, nullptr, T, B};
    ut<<<dim3((unsigned)(B * NT), H, 1), tcw::UT_THREADS, ut_smem, st>>>(
        mq, mk, log_alpha, beta, static_cast<__nv_bfloat16 *>(pt),
        static_cast<__nv_bfloat16 *>(wt), static_cast<__nv_bfloat16 *>(tr), nullptr, sq, H, 0u);
    e = cudaPeekAtLastError();
    if (e != cudaSuccess) return e;
    const long long n_tiles = (long long)B * NT * H;
    CUtensorMap mv, mw, mp;
    if (!tc::make_map(&mv, v, 1, B * T, H, Dv) || !tcw::make_map_w(&mw, wt, n_tiles, DK) ||
        !tc::make_map_tt(&mp, pt, n_tiles))
        return cudaErrorInvalidValue;
    tcw::Params p;
    p.log_alpha = log_alpha;
    p.S0 = S0;
    p.o = nullptr;
    p.S_T = nullptr;
    p.rqk = nullptr;
    p.glk = nullptr;
    p.S_hist = static_cast<__nv_bfloat16 *>(S_hist);
    p.v_zero = false;
    p.sq = sq;
    p.H = H;
    p.Dv = Dv;
    p.flags = 0u;
    auto *seq = tcw::gdn_chunk_tcw_kernel<DK, false>;
    constexpr int seq_smem = tcw::SeqDims<DK>::SMEM_BYTES;
    e = cudaFuncSetAttribute(seq, cudaFuncAttributeMaxDynamicSharedMemorySize, seq_smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(Dv / tcw::DVT, H, B);
    cfg.blockDim = dim3(tcw::NTHREADS);
    cfg.dynamicSmemBytes = seq_smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, seq, mq, mk, mv, mw, mp, p);
    if (e != cudaSuccess) return e;
    return cudaPeekAtLastError();
}

#ifdef GDN_TRACE
extern "C" int gdn_tracew_wide_read(unsigned long long *dst) {
    return (int)cudaMemcpyFromSymbol(dst, g_trace_wide, sizeof(g_trace_wide));
}
#endif

cudaError_t read_and_clear_device_error_wide(unsigned int *flag) {
    cudaError_t e = cudaMemcpyFromSymbol(flag, g_tcw_error, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_tcw_error, &zero, sizeof(unsigned int));
}

}  // namespace gdn
