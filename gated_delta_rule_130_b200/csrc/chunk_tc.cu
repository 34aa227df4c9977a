// Chunkwise forward of the gated delta rule on sm_100a tensor cores (tcgen05 +
// TMEM + TMA), bf16 q/k/v/o, float32 gates, state and accumulation.
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
//
// Two kernels on one stream:
//  1. gdn_ut_kernel, one CTA per (batch, head, chunk), all chunks in parallel:
//     the Gram matrix (one tcgen05 product of the TMA-loaded K chunk, float32
//     in tensor memory), its gating, the UT solve in float32 and the bf16 tile
//     [T'; T''] = [T diag(beta gamma);
//     T diag(beta)] (128 x 64) into a workspace.  None of it depends on S, and
//     the solve is a chain of small dependent steps: run wide, it is hidden by
//     parallelism instead of sitting in front of the sequential pass.
//  2. gdn_chunk_tc_kernel, one CTA per (batch, head, 64-wide slice of value
//     channels), walking the chunks of that head in order with its slice of
//     S^T (Dk x 64, float32) resident in tensor memory.  Warp roles:
//       warp 0       TMA     K, Q, V and [T'; T''] into a two-stage ring, gate vectors
//       warp 1       MMA     the sequential products; owns the TMEM allocation
//       warps 2,3,6,7  P     the gated, masked Q K^T of each chunk (bf16)
//                            (warps 2-5 when q and k are normalised in the kernel)
//       warp 4 (6)   MMA     G of each chunk
//       warp 5 (7)   MMA     WU = [T';T''] [K | V] of each chunk
//       warps 8-15   STATE   W to shared memory, U' = U - W S^T, the chunk
//                            output, the state hand-off
//     Every product is a tcgen05.mma (bf16 operands in 128-byte swizzled shared
//     memory, float32 accumulators in TMEM), M = 128 but for G when normalising:
//       G  = [K;Q] K^T            rows 64-127 Q K^T (rows 0-63 unused); normalising,
//                                 G = Q [K;Q]^T with M = 64 (chunk row r in TMEM lane
//                                 32 (r / 16) + r % 16, one P warp per lane quarter)
//       WU = [T';T''] [K | V]     W = rows 0-63 x K columns, U = rows 64-127 x V columns
//       X  = [Q;W] S^T            rows 0-63 Q S^T, rows 64-127 W S^T
//       Y  = [P;*] U'             rows 0-63 intra-chunk output
//       S^T += K^T diag(exp(g_last - g)) U'   (S^T kept pre-scaled by gamma_last)
//     Shared-memory stage layout per 64-wide key block: K | Q | W (8 KiB each),
//     so that [K;Q] and [Q;W] are contiguous 128-row operands, and the K blocks
//     and the V tile sit 24 KiB apart so [K | V] is one MN-major operand of
//     width Dk + 64.
//
// Rows past the end of the sequence are loaded as zeros and get beta = 0,
// log alpha = 0, which leaves the real rows' results unchanged.  Every mbarrier
// wait is bounded (about two seconds); on a timeout the CTA records an error
// flag, stops all roles, waits for its outstanding copies and releases its
// tensor memory.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tc_common.cuh"

namespace gdn {

// Set by a fused-kernel CTA that gave up waiting (read with gdn_check_device_status).
__device__ unsigned int g_tc_error = 0;

// Test hook of the bounded waits (gdn_debug_withhold_first_arrival): when set,
// the TMA warp of every sequential-kernel CTA withholds its arrival on the first
// stage, so every role's first wait runs out and the CTA takes its abort path
// (flag set, roles stopped, copies drained, tensor memory released).
__device__ unsigned int g_tc_withhold_first = 0;

// Optional per-role timeline of CTA (0,0,0) for performance work: build with
// -DGDN_TRACE; that build alone exports gdn_trace_read() and gdn_tracew_read()
// (end of this file) to copy the timelines out.  Compiled out otherwise.
#ifdef GDN_TRACE
__device__ unsigned long long g_trace[64 * 32];
__device__ unsigned long long g_tracew[16 * 32 * 20];
#define GDN_TRACE_AT(c, ev)                                                            \
    do {                                                                               \
        if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && (c) < 64)        \
            g_trace[(c) * 32 + (ev)] = clock64();                                      \
    } while (0)
// warp-collective variants (every lane calls them; lane 0 records, then the
// warp reconverges so that no later barrier sees a diverged warp)
#define GDN_TRACE_W(c, ev)                                                             \
    do {                                                                               \
        if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && (c) < 16 &&      \
            (threadIdx.x & 31) == 0)                                                   \
            g_tracew[((c) * 32 + (ev)) * 20 + (threadIdx.x >> 5)] = clock64();         \
        __syncwarp();                                                                  \
    } while (0)
#define GDN_TRACE_WARP(c, ev, w)                                                       \
    do {                                                                               \
        if ((threadIdx.x >> 5) == (w) && (threadIdx.x & 31) == 0) GDN_TRACE_AT(c, ev); \
        __syncwarp();                                                                  \
    } while (0)
#else
#define GDN_TRACE_W(c, ev) \
    do {                   \
    } while (0)
#define GDN_TRACE_WARP(c, ev, w) \
    do {                         \
    } while (0)
#define GDN_TRACE_AT(c, ev) \
    do {                    \
    } while (0)
#endif

namespace tc {

using namespace sm100;

constexpr int DVT = 64;        // value channels per CTA
constexpr int DK = 128;        // key channels
constexpr int KB = DK / 64;    // 64-wide key blocks
constexpr int NSTAGE = 2;
constexpr int L2_AHEAD = 2;    // chunks between a tile's L2 prefetch and its shared-memory load
constexpr int BLK = 8192;      // one 64 x 64 bf16 tile (64 rows of 128 bytes)
constexpr int GRP = 3 * BLK;   // K | Q | W of one key block
constexpr int STAGE = KB * GRP + 3 * BLK;  // + V tile + [T'; T''] (16 KiB)
constexpr int OFF_K = 0, OFF_Q = BLK, OFF_W = 2 * BLK, OFF_V = KB * GRP, OFF_TT = KB * GRP + BLK;

// Per-stage gate vectors (float offsets), written by the TMA warp:
constexpr int GV_G2 = 0;       // g_r log2(e), g_r = sum of log alpha over rows <= r
constexpr int GV_BETA = 64;    // beta_r
constexpr int GV_GAM = 128;    // gamma_r = exp(g_r)
constexpr int GV_DCY = 192;    // exp(g_last - g_r)
constexpr int GV_U = 256;      // exp(g_r - g_{16 R(r)})            (R(r) = r / 16)
constexpr int GV_W = 320;      // [R][i]: exp(g_{16R} - g_i) for i < 16R, else 0
constexpr int GV_GL = 576;     // gamma_last = exp(g_last)
constexpr int GV_RK = 640;     // 1/|k_r| (1 unless q and k are L2-normalised in the kernel)
constexpr int GV_RQ = 704;     // 1/|q_r| (written by the P warps)
constexpr int GV_STRIDE = 768;

// shared-memory map (bytes from the 1024-aligned base)
constexpr int SM_STAGE = 0;
constexpr int SM_SB = NSTAGE * STAGE;          // S^T bf16, DK rows x 128 B (MN-major B)
// P tiles for even / odd chunks.  The Y product reads its A operand as 128 rows
// [P; *]: the 8 KiB after each P tile must be shared memory of this CTA (rows
// 64-127 only feed accumulator lanes that are never read), hence U' follows.
constexpr int SM_PT = SM_SB + DK * 128;
constexpr int SM_UN = SM_PT + 2 * BLK;         // U' bf16, 64 rows (MN-major B)
constexpr int SM_UP = SM_UN + BLK;             // diag(exp(g_last - g)) U' bf16
constexpr int SM_GV = SM_UP + BLK;             // gate vectors, NSTAGE x GV_STRIDE floats
constexpr int SM_BAR = SM_GV + NSTAGE * GV_STRIDE * 4;
constexpr int NBAR = 20;
constexpr int SM_MISC = SM_BAR + NBAR * 8;     // tmem base, abort flag
constexpr int SM_TOTAL = SM_MISC + 16;
constexpr int SMEM_BYTES = SM_TOTAL + 1024;    // + alignment slack
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
static_assert(OFF_TT % 1024 == 0 && STAGE % 1024 == 0, "1024-byte aligned swizzled tiles");
static_assert(SM_PT + (NSTAGE + 1) * BLK <= SM_GV, "[P; *] operand rows stay inside the P/U' tiles");
static_assert(SM_BAR % 8 == 0, "mbarrier alignment");

// TMEM columns
// G is 128 columns wide when q and k are normalised in the kernel (Q [K;Q]^T:
// the diagonal of Q Q^T gives |q|^2), 64 otherwise ([K;Q] K^T).
constexpr uint32_t TM_ST = 0, TM_X = 64, TM_G = 128, TM_WU = 256, TM_Y = 448;
constexpr uint32_t TM_U = TM_WU + DK;
static_assert(TM_G + 128 <= TM_WU && TM_U + DVT <= TM_Y && TM_Y + DVT == 512, "TMEM columns");
constexpr uint32_t TM_COLS = 512;

// barrier indices (arrivals)
enum {
    B_IN_FULL = 0,      // [2] TMA warp: gate vectors + tx bytes (1)
    B_IN_EMPTY = 2,     // [2] chain MMA commit after the last use of the stage (1)
    B_G_FULL = 4,       // Gram MMA commit (1)
    B_G_EMPTY = 5,      // P warps (4)
    B_WU_FULL = 7,      // WY MMA commit (1)
    B_WU_EMPTY = 8,     // state warps: W copied (lanes 0-63), U read (lanes 64-127) (8)
    B_PREP_FULL = 9,    // [2] P warps (4) + state warps that copied W (4)
    B_PT_EMPTY = 11,    // [2] chain MMA commit (1)
    B_X_FULL = 13,      // chain MMA commit (1)
    B_U_READY = 14,     // state warps (8)
    B_Y_FULL = 15,      // chain MMA commit (1)
    B_ST_FULL = 16,     // chain MMA commit (1)
    B_S_READY = 17,     // state warps (8)
};

// warp roles of the fused kernel (a warp reaches TMEM lanes 32 (warp % 4) .. + 31)
constexpr int W_TMA = 0;                  // TMA loads and gate vectors
constexpr int W_CHAIN = 1;                // sequential MMAs, TMEM owner
// The Gram product is M = 128, [K;Q] K^T, with the P warps 2, 3, 6, 7 on TMEM
// lanes 64-127; with normalisation it is M = 64, Q [K;Q]^T (half the A operand
// of the widened product), with the P warps 2-5, one per lane quarter, and the
// Gram and WY issuers on warps 6 and 7.  (M = 64 without normalisation measured
// 0.4 % slower on the headline call; with it, 3.9 % faster.)
template <bool kNorm> struct Roles {
    static constexpr int W_GMMA = kNorm ? 6 : 4;  // Gram product of each chunk
    static constexpr int W_PMMA = kNorm ? 7 : 5;  // WY product of each chunk
};
constexpr int NPW = 4;                    // P warps
constexpr int W_STATE0 = 8;               // warps 8-15: sequential state / output
constexpr int NSTATEW = 8;
constexpr int NTHREADS = 32 * (W_STATE0 + NSTATEW);

// Gated, masked Q K^T row, one 16-column piece (columns i = 16 B + j) of row r:
// out[i] = Gamma(r, i) gram[i] for i <= r, zero above, Gamma(r, i) = exp(g_r - g_i).
// Off the row's diagonal 16-block R the decay factors as u_r * w_R[i] (u_r =
// exp(g_r - g_{16R}), w_R[i] = exp(g_{16R} - g_i) for i < 16 R and 0 from 16 R on,
// both <= 1, so nothing overflows); inside it, exp2 of the log2-domain
// difference.  kDiag: some lane of the warp has B == R (the exp2 path is then
// evaluated for every lane and selected, so the warp never diverges).
template <bool kDiag>
__device__ __forceinline__ void gated_piece(float (&v)[16], int B, int r, float su,
                                            const float *g2s, const float *w_all) {
    const int R = r >> 4;
    const float *w = w_all + R * 64 + 16 * B;
    const float gr = g2s[r];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const int i = 16 * B + j;
        float f = su * w[j];
        if (kDiag) {
            const float e = ex2(gr - g2s[i]);
            f = (B == R) ? ((i <= r) ? e : 0.f) : f;
        }
        v[j] *= f;
    }
}

// Bucket of a sequence by its chunk count on a quarter-octave scale (exact below
// 4 chunks, then 4 buckets per power of two): non-decreasing in the count.
constexpr int kLenBuckets = 128;
__device__ __forceinline__ int len_bucket(int chunks) {
    if (chunks < 4) return chunks;
    const int msb = 31 - __clz(chunks);
    return min(kLenBuckets - 1, 4 * msb - 4 + ((chunks >> (msb - 2)) & 3));
}

// Sequence schedule, one block: cu_chunks[b] = sum over earlier sequences of
// ceil(len / C) (cu_chunks[n] = all chunks), and order[] = the sequences longest
// first (by bucket; ties in any order).  The sequential kernel takes sequence
// order[blockIdx.z], so the CTAs of the longest sequences, which set the
// critical path, are dispatched in the first wave.
constexpr int kScheduleThreads = 1024;
__global__ void __launch_bounds__(kScheduleThreads)
seq_schedule(const int *__restrict__ cu, int n, int *__restrict__ cu_chunks,
             int *__restrict__ order) {
    __shared__ int hist[kLenBuckets];
    __shared__ int warp_sum[kScheduleThreads / 32];
    __shared__ int carry;
    const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
    constexpr int NW = kScheduleThreads / 32;
    for (int i = tid; i < kLenBuckets; i += kScheduleThreads) hist[i] = 0;
    if (tid == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < n; base += kScheduleThreads) {
        const int b = base + tid;
        const int nc = b < n ? (cu[b + 1] - cu[b] + C - 1) / C : 0;
        if (b < n) atomicAdd(&hist[len_bucket(nc)], 1);
        int x = nc;  // inclusive scan within the warp
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_sum[warp] = x;
        __syncthreads();
        if (warp == 0) {  // exclusive scan of the warp totals
            const int t = warp_sum[lane];
            int y = t;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int z = __shfl_up_sync(0xffffffffu, y, o);
                if (lane >= o) y += z;
            }
            warp_sum[lane] = y - t;
        }
        __syncthreads();
        const int excl = carry + warp_sum[warp] + x - nc;
        if (b < n) cu_chunks[b] = excl;
        __syncthreads();  // every thread has read carry
        if (tid == kScheduleThreads - 1) carry = excl + nc;
        __syncthreads();
    }
    static_assert(NW == 32, "one warp scans the warp totals");
    if (tid == 0) {
        cu_chunks[n] = carry;
        int acc = 0;  // bucket starts, longest bucket first
        for (int k = kLenBuckets - 1; k >= 0; --k) {
            const int c = hist[k];
            hist[k] = acc;
            acc += c;
        }
    }
    __syncthreads();
    for (int b = tid; b < n; b += kScheduleThreads) {
        const int nc = (cu[b + 1] - cu[b] + C - 1) / C;
        order[atomicAdd(&hist[len_bucket(nc)], 1)] = b;
    }
}

// ------------------------------------------------------------- UT kernel --
// One CTA of 4 warps per (global chunk g, head h): [T'; T''] of that chunk,
// bf16, 128 rows x 64 columns, row-major, at tt + (g H + h) 128 x 64.
// The chunk's K rows arrive by TMA (128-byte swizzle) and the Gram matrix K K^T
// is one tcgen05 product (M = N = 64, K = 128) into tensor memory, from where
// each warp reads 16 rows (an M = 64 product puts row m in TMEM lane
// 32 (m / 16) + m % 16).  Six CTAs fit on an SM (37 KiB of shared memory, 64
// TMEM columns, 80 registers a thread), so six chunks are in flight per SM and
// the solve's dependent steps overlap across chunks.
constexpr int UT_THREADS = 128;
constexpr int UT_SM_KT = 0;                        // K chunk (KB blocks of 64 x 128 B), then T
constexpr int UT_SM_AF = C * LDA * 4;              // A (64 x LDA f32); N_IJ overwrite A_IJ
constexpr int UT_SM_GT = UT_SM_AF + C * LDA * 4;   // g log2(e), beta, beta gamma |k|^-1, |k|^-1
constexpr int UT_SM_BAR = UT_SM_GT + 4 * C * 4;    // 2 mbarriers, TMEM base, abort flag
constexpr int UT_SMEM = UT_SM_BAR + 32 + 1024;     // + alignment slack (1024-byte tiles)
constexpr uint32_t UT_TM_COLS = 64;
constexpr int TT_ELEMS = 2 * C * C;                // one [T'; T''] tile
static_assert(KB * 8192 <= UT_SM_AF, "K chunk fits in the T buffer");
static_assert(UT_SM_GT % 16 == 0 && UT_SM_BAR % 8 == 0, "aligned UT buffers");
static_assert(6 * (UT_SMEM + 1024) <= 228 * 1024, "six CTAs per SM");

// kNorm: q and k are L2-normalised inside the kernels (1/|k| folded into the
// Gram rows and T', and written to rk_out); without it the kernel is unchanged.
template <bool kNorm>
__global__ void __launch_bounds__(UT_THREADS, 6)
gdn_ut_kernel(const __grid_constant__ CUtensorMap tm_k, const float *__restrict__ log_alpha,
              const float *__restrict__ beta, __nv_bfloat16 *__restrict__ tt,
              float *__restrict__ rk_out, const Seqs sq, int H, unsigned flags) {
    extern __shared__ __align__(1024) uint8_t ut_raw[];
    uint8_t *ut_smem = ut_raw + ((1024u - (smem_u32(ut_raw) & 1023u)) & 1023u);
    // the sequential kernel that follows on the stream may be scheduled now (it
    // waits for this grid's completion before it reads the tiles)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // global chunk g of head h: chunk c of sequence b, whose tokens start at sp.off
    const int gch = blockIdx.x, h = blockIdx.y;
    const int b = seq_of_chunk(sq, gch);
    const Span sp = seq_span(sq, b);
    const int c = gch - sp.chunk0, T = sp.len;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t0 = c * C;
    float *TF = reinterpret_cast<float *>(ut_smem + UT_SM_KT);
    float *AF = reinterpret_cast<float *>(ut_smem + UT_SM_AF);
    float *g2s = reinterpret_cast<float *>(ut_smem + UT_SM_GT);
    float *bes = g2s + C, *bgs = g2s + 2 * C, *rks = g2s + 3 * C;
    Ctx cx;
    cx.base = ut_smem;
    cx.bar = reinterpret_cast<uint64_t *>(ut_smem + UT_SM_BAR);  // [0] K landed, [1] Gram done
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(ut_smem + UT_SM_BAR + 16);
    cx.abort = reinterpret_cast<volatile uint32_t *>(ut_smem + UT_SM_BAR + 20);
    cx.err = &g_tc_error;

    if (tid == 0) {
        mbar_init(cx.bar + 0, 1);
        mbar_init(cx.bar + 1, 1);
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
    // K rows of the chunk.  Rows past the end of the sequence (the next
    // sequence's, or TMA's zero fill past the last token) get beta = 0 and
    // log alpha = 0 below, which zeroes their rows of A and their columns of
    // T' and T'' (T restricted to them is the identity).
    if (tid == 0) {
        mbar_arrive_expect_tx(cx.bar + 0, KB * 8192);
#pragma unroll
        for (int kb = 0; kb < KB; ++kb)
            tma_load_4d(ut_smem + UT_SM_KT + kb * 8192, &tm_k, cx.bar + 0, kb * 64, h, sp.off + t0, 0);
    }
    if (warp == 0) {
        // running sum of log alpha over rows lane and lane + 32, in log2 units
        constexpr float LOG2E = 1.4426950408889634f;
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
            bgs[lane + 32 * hh] = be[hh] * ex2(g2);
        }
    } else if (warp == 1) {
        // Gram G = K K^T: A = K (K-major, per key block), B = K (K-major: N rows = tokens)
        const bool landed = warp_wait(cx, 0, 0);
        tc_fence_after();
        if (landed && lane == 0) {
            const uint32_t kt = smem_u32(ut_smem + UT_SM_KT);
            const uint32_t idesc = idesc_bf16(64, 64, false, false);
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk) {
                const uint32_t koff = (kk >> 2) * 8192 + (kk & 3) * 32;
                mma_bf16(tmem, desc_sw128(kt + koff, 16, 1024), desc_sw128(kt + koff, 16, 1024),
                         idesc, kk > 0);
            }
            mma_commit(cx.bar + 1);
        }
        __syncwarp();
    }
    __syncthreads();  // the gate vectors are written
    // row r = 16 w + l % 16 of G (TMEM lane 32 w + l % 16 of warp w), columns
    // 32 hc .. + 31 with hc = l / 16: the 16-lane loads give lanes 16-31 the second
    // half of the row
    const int r = 16 * warp + (lane & 15), hc = lane >> 4;
    const bool row_lane = lane < 16;
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    const bool done = warp_wait(cx, 1, 0);
    tc_fence_after();
    const auto load_half = [&](float (&v)[32]) {
        if (done) {
            float a[16], b2[16];
            tmem_ld16x2<32>(lane_addr, a);
            tmem_ld16x2<32>(lane_addr + 16, b2);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                v[j] = a[j];
                v[16 + j] = b2[j];
            }
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = 0.f;
        }
    };
    if constexpr (kNorm) {
        // |k_r|^2 is the diagonal of K K^T; 1/|k| folds into the Gram rows and T',
        // and is kept in the workspace for the sequential kernel
        // row r = 16 w + l has its diagonal in columns 16 w .. + 15 (warp-uniform)
        float v[16];
        tmem_ld16(lane_addr + 16 * warp, v);
        tmem_wait_ld();
        if (row_lane) {
            float d = 0.f;
#pragma unroll
            for (int j = 0; j < 16; ++j) d = (j == lane) ? v[j] : d;
            if (!done) d = 0.f;
            const float rkv = rsqrtf(fmaxf(d, 0.f) + kNormEps);
            rks[r] = rkv;
            bgs[r] *= rkv;
            rk_out[((size_t)gch * H + h) * C + r] = rkv;
        }
        __syncthreads();
    }
    // A_ri = beta_r exp(g_r - g_i) (k_r . k_i) for i < r, else 0 (row r, columns 32 hc .. + 31)
    {
        float v[32];
        load_half(v);
        {
            const float grl = g2s[r], br = kNorm ? bes[r] * rks[r] : bes[r];
#pragma unroll
            for (int i4 = 0; i4 < 8; ++i4) {
                float a[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i = 32 * hc + 4 * i4 + e;
                    const float sc = kNorm ? br * rks[i] : br;
                    a[e] = (i < r) ? sc * ex2(grl - g2s[i]) * v[4 * i4 + e] : 0.f;
                }
                *reinterpret_cast<float4 *>(AF + r * LDA + 32 * hc + 4 * i4) =
                    make_float4(a[0], a[1], a[2], a[3]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();  // A complete; TMEM and K no longer read (K's buffer becomes T)
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, UT_TM_COLS);
    }
    if (tid < C) ut_diag(AF, TF, tid);
    __syncthreads();
    ut_offdiag4(AF, TF, tid);  // ends with a CTA-wide barrier

    // [T'; T''] rows: T'(r, i) = T(r, i) beta_i gamma_i / |k_i|, T''(r, i) = T(r, i) beta_i
    // for i <= r; thread -> (row, 4-column piece): 16 threads read one T row with
    // no bank conflict and write its 128 bytes
    __nv_bfloat16 *dst = tt + ((size_t)gch * H + h) * TT_ELEMS;
#pragma unroll 4
    for (int m = 0; m < TT_ELEMS / 4 / UT_THREADS; ++m) {
        const int idx = tid + UT_THREADS * m;
        const int rt = idx >> 4, i0 = 4 * (idx & 15), r = rt & (C - 1);
        const float *sc = rt < C ? bgs : bes;
        const float4 tv = *reinterpret_cast<const float4 *>(TF + r * LDA + i0);
        const float4 sv = *reinterpret_cast<const float4 *>(sc + i0);
        const float x0 = i0 + 0 <= r ? tv.x * sv.x : 0.f, x1 = i0 + 1 <= r ? tv.y * sv.y : 0.f;
        const float x2 = i0 + 2 <= r ? tv.z * sv.z : 0.f, x3 = i0 + 3 <= r ? tv.w * sv.w : 0.f;
        *reinterpret_cast<uint2 *>(dst + rt * C + i0) = make_uint2(pack_bf16(x0, x1), pack_bf16(x2, x3));
    }
}

struct Params {
    const float *log_alpha;
    const float *beta;
    const float *S0;
    __nv_bfloat16 *o;
    float *S_T;
    const float *rk;       // 1/|k| per token from the UT kernel (L2-normalising only)
    Seqs sq;               // the sequences (one per blockIdx.z)
    float *S_hist;         // optional (fixed-length batches): the state entering every
                           // chunk, [B*H][NT][Dv][Dk] float32, for the backward
    int H, Dv;
    unsigned flags;        // input prologue (kFlagL2Norm, kFlagGateLogits)
};

// kNorm: as for gdn_ut_kernel (G widens to [K;Q][K;Q]^T, whose Q Q^T diagonal
// gives |q|^2, and 1/|k|, 1/|q| scale P and the U' epilogue).
template <bool kNorm>
__global__ void __launch_bounds__(NTHREADS, 1)
gdn_chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_tt,
                    const Params p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base, derived by pointer arithmetic so that the compiler
    // keeps every access below in the shared address space
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    Ctx cx;
    cx.base = base;
    cx.bar = reinterpret_cast<uint64_t *>(base + SM_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + SM_MISC);
    cx.abort = reinterpret_cast<volatile uint32_t *>(base + SM_MISC + 4);
    cx.err = &g_tc_error;
    float *gv_all = reinterpret_cast<float *>(base + SM_GV);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int vt = blockIdx.x, h = blockIdx.y;
    const int b = p.sq.order ? p.sq.order[blockIdx.z] : (int)blockIdx.z;
    const int v0 = vt * DVT;
    const int H = p.H;
    // sequence b: tokens sp.off .. sp.off + T of the packed rows, chunks sp.chunk0 ..
    const Span sp = seq_span(p.sq, b);
    const int T = sp.len, NT = (T + C - 1) / C;
    if (NT == 0) {
        // an empty sequence: the final state is the initial one (this CTA's slice)
        if (p.S_T)
            for (int e = threadIdx.x; e < DVT * DK; e += NTHREADS) {
                const size_t idx = ((size_t)b * H + h) * p.Dv * DK + (size_t)v0 * DK + e;
                p.S_T[idx] = p.S0 ? p.S0[idx] : 0.f;
            }
        return;
    }

    if (tid == 0) {
        int counts[NBAR];
        for (int i = 0; i < NBAR; ++i) counts[i] = 1;
        // one arrival per arriving warp
        counts[B_G_EMPTY] = NPW;
        counts[B_WU_EMPTY] = NSTATEW;
        counts[B_PREP_FULL] = counts[B_PREP_FULL + 1] = NPW + NSTATEW / 2;
        counts[B_U_READY] = counts[B_S_READY] = NSTATEW;
        for (int i = 0; i < NBAR; ++i) mbar_init(cx.bar + i, counts[i]);
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
        prefetch_tensormap(&tm_tt);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == W_TMA) {
        // ------------------------------------- TMA loads + per-chunk gate vectors
        // The gate values of chunk c + 1 are fetched while chunk c is handled, and
        // each stage's copies are started before its gate vectors are computed
        // (the stage's barrier gets the byte count first and the warp's arrival
        // after the vectors are written).
        constexpr float LOG2E = 1.4426950408889634f;
        int armed = 0;
        float nla[2], nbe[2], nrk[2];  // gate values of the next chunk (rows lane, lane + 32)
        constexpr bool l2n = kNorm;
        const auto fetch_gates = [&](int cc) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int r = lane + 32 * hh;
                const bool in = cc * C + r < T;
                const size_t gi = (size_t)(sp.off + cc * C + r) * H + h;
                nla[hh] = in ? p.log_alpha[gi] : 0.f;
                nbe[hh] = in ? p.beta[gi] : 0.f;
                nrk[hh] = l2n ? p.rk[((size_t)(sp.chunk0 + cc) * H + h) * C + r] : 1.f;
            }
        };
        // the [T'; T''] tiles (and 1/|k|) come from the UT kernel launched just
        // before this one (programmatic dependent launch): wait for its completion
        asm volatile("griddepcontrol.wait;" ::: "memory");
        const bool withhold = *reinterpret_cast<volatile unsigned int *>(&g_tc_withhold_first) != 0u;
        fetch_gates(0);
        for (int c = 0; c < NT; ++c) {
            const int s = c & 1;
            const int t0 = c * C;
            float la[2], be[2];
            const float rk2[2] = {nrk[0], nrk[1]};
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                // rows past the end keep log alpha = beta = 0
                const bool in = t0 + lane + 32 * hh < T;
                const float2 gp = in ? gate_pair(nla[hh], nbe[hh], p.flags) : make_float2(0.f, 0.f);
                la[hh] = gp.x;
                be[hh] = gp.y;
            }
            if (c + 1 < NT) fetch_gates(c + 1);
            if (c >= 2 && !warp_wait(cx, B_IN_EMPTY + s, ((c - 2) >> 1) & 1)) break;
            GDN_TRACE_WARP(c, 31, W_TMA);
            if (lane == 0) {
                uint8_t *st = base + SM_STAGE + s * STAGE;
                mbar_expect_tx(cx.bar + B_IN_FULL + s, (2 * KB + 3) * BLK);
#pragma unroll
                for (int kb = 0; kb < KB; ++kb) {
                    tma_load_4d(st + kb * GRP + OFF_K, &tm_k, cx.bar + B_IN_FULL + s, kb * 64, h,
                                sp.off + t0, 0);
                    tma_load_4d(st + kb * GRP + OFF_Q, &tm_q, cx.bar + B_IN_FULL + s, kb * 64, h,
                                sp.off + t0, 0);
                }
                tma_load_4d(st + OFF_V, &tm_v, cx.bar + B_IN_FULL + s, v0, h, sp.off + t0, 0);
                tma_load_3d(st + OFF_TT, &tm_tt, cx.bar + B_IN_FULL + s, 0, 0,
                            (sp.chunk0 + c) * H + h);
                GDN_TRACE_AT(c, 24);
                // the tiles of a later chunk start streaming from DRAM into L2 now,
                // so that its shared-memory load, once a stage is free, hits L2
                for (int cq = (c == 0 ? 1 : c + L2_AHEAD); cq <= c + L2_AHEAD && cq < NT; ++cq) {
#pragma unroll
                    for (int kb = 0; kb < KB; ++kb) {
                        tma_prefetch_l2_4d(&tm_k, kb * 64, h, sp.off + cq * C, 0);
                        tma_prefetch_l2_4d(&tm_q, kb * 64, h, sp.off + cq * C, 0);
                    }
                    tma_prefetch_l2_4d(&tm_v, v0, h, sp.off + cq * C, 0);
                    tma_prefetch_l2_3d(&tm_tt, 0, 0, (sp.chunk0 + cq) * H + h);
                }
            }
            armed = c + 1;
            // running sums over rows lane (lo) and lane + 32 (hi); rows past the
            // end of the sequence carry zeros
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
            const float g0 = la[0] * LOG2E, g1 = la[1] * LOG2E;  // rows lane, lane + 32
            const float glast = __shfl_sync(0xffffffffu, g1, 31);
            const float gb0 = __shfl_sync(0xffffffffu, g0, lane & 16);   // g at the row's 16-block start
            const float gb1 = __shfl_sync(0xffffffffu, g1, lane & 16);
            const float g16 = __shfl_sync(0xffffffffu, g0, 16);
            const float g32 = __shfl_sync(0xffffffffu, g1, 0);
            const float g48 = __shfl_sync(0xffffffffu, g1, 16);
            float *gv = gv_all + s * GV_STRIDE;
            gv[GV_G2 + lane] = g0;
            gv[GV_G2 + 32 + lane] = g1;
            gv[GV_BETA + lane] = be[0];
            gv[GV_BETA + 32 + lane] = be[1];
            if constexpr (kNorm) {
                gv[GV_RK + lane] = rk2[0];
                gv[GV_RK + 32 + lane] = rk2[1];
            }
            gv[GV_GAM + lane] = ex2(g0);
            gv[GV_GAM + 32 + lane] = ex2(g1);
            gv[GV_DCY + lane] = ex2(glast - g0);
            gv[GV_DCY + 32 + lane] = ex2(glast - g1);
            gv[GV_U + lane] = ex2(g0 - gb0);
            gv[GV_U + 32 + lane] = ex2(g1 - gb1);
            gv[GV_W + 0 * 64 + lane] = 0.f;
            gv[GV_W + 0 * 64 + 32 + lane] = 0.f;
            gv[GV_W + 1 * 64 + lane] = lane < 16 ? ex2(g16 - g0) : 0.f;
            gv[GV_W + 1 * 64 + 32 + lane] = 0.f;
            gv[GV_W + 2 * 64 + lane] = ex2(g32 - g0);
            gv[GV_W + 2 * 64 + 32 + lane] = 0.f;
            gv[GV_W + 3 * 64 + lane] = ex2(g48 - g0);
            gv[GV_W + 3 * 64 + 32 + lane] = lane < 16 ? ex2(g48 - g1) : 0.f;
            if (lane == 0) gv[GV_GL] = ex2(glast);
            __syncwarp();
            if (lane == 0 && !(withhold && c == 0)) mbar_arrive(cx.bar + B_IN_FULL + s);
        }
        // never leave with copies in flight: wait for the last two stages
        if (lane == 0) {
            for (int c = armed - 2 < 0 ? 0 : armed - 2; c < armed; ++c) {
                uint64_t *fb = cx.bar + B_IN_FULL + (c & 1);
                const uint64_t t0 = now_ns();
                while (!mbar_try_wait(fb, (c >> 1) & 1) && now_ns() - t0 < kTimeoutNs) {
                }
            }
        }
    } else if (warp == Roles<kNorm>::W_GMMA) {
        // ------------------------------------------------- MMA: Gram products
        // the whole warp waits (fast path: a test and a vote); lane 0 issues
        // A = [K; Q] (M = 128) and B = K, or, normalising, A = Q (M = 64) and
        // B = [K; Q] (contiguous per key block: the diagonal of Q Q^T gives |q|)
        const uint32_t idesc_g = idesc_bf16(kNorm ? 64 : 128, kNorm ? 128 : 64, false, false);
        for (int c = 0; c < NT; ++c) {
            const int s = c & 1;
            const uint32_t st = smem_u32(base + SM_STAGE + s * STAGE);
            if (!warp_wait(cx, B_IN_FULL + s, (c >> 1) & 1)) break;
            if (c >= 1 && !warp_wait(cx, B_G_EMPTY, (c - 1) & 1)) break;
            tc_fence_after();
            if (lane == 0) {
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk) {
                    const uint32_t koff = (kk >> 2) * GRP + (kk & 3) * 32;
                    mma_bf16(tmem + TM_G, desc_sw128(st + (kNorm ? OFF_Q : OFF_K) + koff, 16, 1024),
                             desc_sw128(st + OFF_K + koff, 16, 1024), idesc_g, kk > 0);
                }
                mma_commit(cx.bar + B_G_FULL);
                GDN_TRACE_AT(c, 8);
            }
            __syncwarp();
        }
    } else if (warp == Roles<kNorm>::W_PMMA) {
        // --------------------------------------------------- MMA: WY products
        const uint32_t idesc_wu = idesc_bf16(128, DK + DVT, false, true);
        for (int c = 0; c < NT; ++c) {
            const uint32_t st = smem_u32(base + SM_STAGE + (c & 1) * STAGE);
            const uint32_t tt = st + OFF_TT;
            if (!warp_wait(cx, B_IN_FULL + (c & 1), (c >> 1) & 1)) break;
            if (c >= 1 && !warp_wait(cx, B_WU_EMPTY, (c - 1) & 1)) break;
            tc_fence_after();
            if (lane == 0) {
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    mma_bf16(tmem + TM_WU, desc_sw128(tt + kk * 32, 16, 1024),
                             desc_sw128(st + OFF_K + kk * 2048, GRP, 1024), idesc_wu, kk > 0);
                mma_commit(cx.bar + B_WU_FULL);
                GDN_TRACE_AT(c, 9);
            }
            __syncwarp();
        }
    } else if (warp == W_CHAIN) {
        // ---------------------------------------------- MMA: sequential chain
        const uint32_t idesc_x = idesc_bf16(128, DVT, false, true);
        const uint32_t idesc_y = idesc_bf16(128, DVT, false, true);
        const uint32_t idesc_s = idesc_bf16(128, DVT, true, true);
        const uint32_t sb = smem_u32(base + SM_SB), un = smem_u32(base + SM_UN),
                       up = smem_u32(base + SM_UP);
        for (int c = 0; c < NT; ++c) {
            const int s = c & 1;
            const uint32_t st = smem_u32(base + SM_STAGE + s * STAGE);
            if (!warp_wait(cx, B_IN_FULL + s, (c >> 1) & 1)) break;
            GDN_TRACE_WARP(c, 5, W_CHAIN);
            if (!warp_wait(cx, B_PREP_FULL + s, (c >> 1) & 1)) break;
            GDN_TRACE_WARP(c, 6, W_CHAIN);
            if (!warp_wait(cx, B_S_READY, c & 1)) break;
            GDN_TRACE_WARP(c, 7, W_CHAIN);
            tc_fence_after();
            // X = [Q; W] S^T : A K-major (rows 0-63 Q, 64-127 W), B = S^T MN-major
            if (lane == 0) {
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk) {
                    const uint32_t koff = (kk >> 2) * GRP + (kk & 3) * 32;
                    mma_bf16(tmem + TM_X, desc_sw128(st + OFF_Q + koff, 16, 1024),
                             desc_sw128(sb + kk * 2048, 16, 1024), idesc_x, kk > 0);
                }
                mma_commit(cx.bar + B_X_FULL);
                GDN_TRACE_AT(c, 12);
            }
            __syncwarp();
            if (!warp_wait(cx, B_U_READY, c & 1)) break;
            GDN_TRACE_WARP(c, 13, W_CHAIN);
            tc_fence_after();
            if (lane == 0) {
                // S^T += K^T (decay U') : A = K^T (MN-major, key blocks GRP apart).
                // Issued first: the next chunk waits on it.
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    mma_bf16(tmem + TM_ST, desc_sw128(st + OFF_K + kk * 2048, GRP, 1024),
                             desc_sw128(up + kk * 2048, 16, 1024), idesc_s, 1u);
                mma_commit(cx.bar + B_ST_FULL);
                // the stage (K, Q, W) is not read after MMA3 and MMA1
                mma_commit(cx.bar + B_IN_EMPTY + s);
                // Y += [P; *] U'  (Y holds diag(gamma) Q S^T; rows 64-127 of A unused)
                const uint32_t pt = smem_u32(base + SM_PT + s * BLK);
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    mma_bf16(tmem + TM_Y, desc_sw128(pt + kk * 32, 16, 1024),
                             desc_sw128(un + kk * 2048, 16, 1024), idesc_y, 1u);
                mma_commit(cx.bar + B_Y_FULL);
                mma_commit(cx.bar + B_PT_EMPTY + s);
            }
            __syncwarp();
        }
    } else if (warp < W_STATE0) {
        if constexpr (kNorm) {
            // ---------------------------------------------------------------- P
            // (normalising) warps 2-5: the M = 64 product G = Q [K;Q]^T puts chunk row r in TMEM lane
            // 32 (r / 16) + r % 16, so warp w (lane quarter q = w % 4) holds rows
            // 16 q .. + 15 in its lanes 0-15.  The 16-lane loads give lanes 0-15 the
            // 16-column pieces 0 and 1 of the row and lanes 16-31 the pieces 2 and 3;
            // the row's diagonal 16-block is piece q, in the first load for even q and
            // the second for odd q.  P (bf16) goes to the chunk's P tile.
            const int q = warp & 3, sub = lane >> 4;
            const int r = 16 * q + (lane & 15);
            const int B0 = 2 * sub, B1 = 2 * sub + 1;
            const uint32_t lane_addr = tmem + ((uint32_t)(q * 32) << 16);
            for (int c = 0; c < NT; ++c) {
                const int s = c & 1;
                const float *gv = gv_all + s * GV_STRIDE;
                if (!warp_wait(cx, B_IN_FULL + s, (c >> 1) & 1)) break;
                if (!warp_wait(cx, B_G_FULL, c & 1)) break;
                GDN_TRACE_WARP(c, 22, 2);
                if (c >= 2 && !warp_wait(cx, B_PT_EMPTY + s, ((c - 2) >> 1) & 1)) break;
                GDN_TRACE_WARP(c, 3, 2);
                tc_fence_after();
                const float su = gv[GV_U + r];
                float v0[16], v1[16];
                tmem_ld16x2<32>(lane_addr + TM_G, v0);
                tmem_ld16x2<32>(lane_addr + TM_G + 16, v1);
                // with normalisation: the row's 16 x 16 diagonal block of Q Q^T (columns
                // 64 + 16 q ..; lane l < 16 needs column l; lanes 16-31 read unused TMEM
                // lanes and take lane l - 16's value below), read before G is released
                float d0[16];
                if constexpr (kNorm) tmem_ld16(lane_addr + TM_G + 64 + 16 * q, d0);
                tmem_wait_ld();
                GDN_TRACE_WARP(c, 27, 2);
                tc_fence_before();
                warp_arrive(cx, B_G_EMPTY);
                if ((q & 1) == 0) {
                    gated_piece<true>(v0, B0, r, su, gv + GV_G2, gv + GV_W);
                    gated_piece<false>(v1, B1, r, su, gv + GV_G2, gv + GV_W);
                } else {
                    gated_piece<false>(v0, B0, r, su, gv + GV_G2, gv + GV_W);
                    gated_piece<true>(v1, B1, r, su, gv + GV_G2, gv + GV_W);
                }
                if constexpr (kNorm) {
                    // P_ri = Gamma_ri (q_r . k_i) / (|q_r| |k_i|): |q_r|^2 is the diagonal of
                    // Q Q^T (G columns 64 + r), 1/|k_i| comes with the gate vectors
                    float qq = 0.f;
#pragma unroll
                    for (int j = 0; j < 16; ++j) qq = ((lane & 15) == j) ? d0[j] : qq;
                    qq = __shfl_sync(0xffffffffu, qq, lane & 15);
                    const float rq = rsqrtf(fmaxf(qq, 0.f) + kNormEps);
                    if (sub == 0) gv_all[s * GV_STRIDE + GV_RQ + r] = rq;
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        v0[j] *= rq * gv[GV_RK + 16 * B0 + j];
                        v1[j] *= rq * gv[GV_RK + 16 * B1 + j];
                    }
                }
                GDN_TRACE_WARP(c, 28, 2);
                store16_bf16(base + SM_PT + s * BLK, r, B0, v0);
                store16_bf16(base + SM_PT + s * BLK, r, B1, v1);
                fence_async_smem();
                GDN_TRACE_WARP(c, 29, 2);
                warp_arrive(cx, B_PREP_FULL + s);
                GDN_TRACE_WARP(c, 23, 2);
                GDN_TRACE_WARP(c, 30, 7);
            }
        } else {
            // ---------------------------------------------------------------- P
            // (M = 128 Gram) warps 2, 3, 6, 7: TMEM lanes 64-127 of G hold Q K^T.  Warp w reads
            // lanes 32 (w % 4) .. + 31 (chunk rows r = that lane - 64, 16-blocks
            // 2 qr and 2 qr + 1) and the 16-column pieces hf and hf + 2 (hf = w / 4):
            // every warp meets the diagonal in exactly one of its pieces (piece hf
            // for qr = 0, piece hf + 2 for qr = 1).  P (bf16) goes to the chunk's P tile.
            const int q = warp & 3, hf = warp >> 2, qr = q - 2;
            const int r = 32 * q + lane - 64;
            const uint32_t lane_addr = tmem + ((uint32_t)(q * 32) << 16);
            for (int c = 0; c < NT; ++c) {
                const int s = c & 1;
                const float *gv = gv_all + s * GV_STRIDE;
                if (!warp_wait(cx, B_IN_FULL + s, (c >> 1) & 1)) break;
                if (!warp_wait(cx, B_G_FULL, c & 1)) break;
                GDN_TRACE_WARP(c, 22, 2);
                if (c >= 2 && !warp_wait(cx, B_PT_EMPTY + s, ((c - 2) >> 1) & 1)) break;
                GDN_TRACE_WARP(c, 3, 2);
                tc_fence_after();
                const float su = gv[GV_U + r];
                float v0[16], v1[16];
                tmem_ld16(lane_addr + TM_G + 16 * hf, v0);
                tmem_ld16(lane_addr + TM_G + 16 * hf + 32, v1);
                tmem_wait_ld();
                GDN_TRACE_WARP(c, 27, 2);
                tc_fence_before();
                warp_arrive(cx, B_G_EMPTY);
                if (qr == 0) {
                    gated_piece<true>(v0, hf, r, su, gv + GV_G2, gv + GV_W);
                    gated_piece<false>(v1, hf + 2, r, su, gv + GV_G2, gv + GV_W);
                } else {
                    gated_piece<false>(v0, hf, r, su, gv + GV_G2, gv + GV_W);
                    gated_piece<true>(v1, hf + 2, r, su, gv + GV_G2, gv + GV_W);
                }
                GDN_TRACE_WARP(c, 28, 2);
                store16_bf16(base + SM_PT + s * BLK, r, hf, v0);
                store16_bf16(base + SM_PT + s * BLK, r, hf + 2, v1);
                fence_async_smem();
                GDN_TRACE_WARP(c, 29, 2);
                warp_arrive(cx, B_PREP_FULL + s);
                GDN_TRACE_WARP(c, 23, 2);
                GDN_TRACE_WARP(c, 30, 7);
            }
        }
    } else {
        // ------------------------------------------------------------ STATE
        // 8 warps; warp w reads TMEM lanes 32 (w % 4) .. + 31 (a key channel of
        // S^T, or a chunk row of X / Y) and handles half of that lane's 64
        // columns (hf), its twin the other half.
        const int q = warp & 3, hf = (warp - W_STATE0) >> 2;
        const int lrow = 32 * q + lane;
        const uint32_t lane_addr = tmem + ((uint32_t)(q * 32) << 16);
        uint8_t *sbuf = base + SM_SB;
        const size_t head = (size_t)b * H + h;
        const auto copy_w = [&](int cc) -> bool {
            if (q >= 2) return true;
            const bool fine = warp_wait(cx, B_WU_FULL, cc & 1);
            GDN_TRACE_WARP(cc, 25, W_STATE0);
            tc_fence_after();
            const int kb = hf;
            float w0[16], w1[16], w2[16], w3[16];
            tmem_ld16(lane_addr + TM_WU + 64 * kb, w0);
            tmem_ld16(lane_addr + TM_WU + 64 * kb + 16, w1);
            tmem_ld16(lane_addr + TM_WU + 64 * kb + 32, w2);
            tmem_ld16(lane_addr + TM_WU + 64 * kb + 48, w3);
            tmem_wait_ld();
            uint8_t *wt = base + SM_STAGE + (cc & 1) * STAGE + kb * GRP + OFF_W;
            store16_bf16(wt, lrow, 0, w0);
            store16_bf16(wt, lrow, 1, w1);
            store16_bf16(wt, lrow, 2, w2);
            store16_bf16(wt, lrow, 3, w3);
            fence_async_smem();
            tc_fence_before();
            warp_arrive(cx, B_WU_EMPTY);
            warp_arrive(cx, B_PREP_FULL + (cc & 1));
            GDN_TRACE_WARP(cc, 26, W_STATE0);
            return fine;
        };
        // initial state: S^T row lrow = S0[v0 .. v0+63][lrow]; TMEM copy pre-scaled by gamma_last
        {
            const bool have = warp_wait(cx, B_IN_FULL + 0, 0);
            const float gl = gv_all[GV_GL];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int B = 2 * hf + k;
                float sv[16];
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    sv[j] = p.S0 ? p.S0[(head * p.Dv + v0 + 16 * B + j) * DK + lrow] : 0.f;
                if (p.S_hist)
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        p.S_hist[((size_t)head * NT * p.Dv + v0 + 16 * B + j) * DK + lrow] = sv[j];
                store16_bf16(sbuf, lrow, B, sv);
#pragma unroll
                for (int j = 0; j < 16; ++j) sv[j] *= gl;
                if (have) tmem_st16(lane_addr + TM_ST + 16 * B, sv);
            }
            fence_async_smem();
            tmem_wait_st();
            tc_fence_before();
            warp_arrive(cx, B_S_READY);
        }
        if (NT > 0) copy_w(0);
        for (int c = 0; c < NT; ++c) {
            if (__any_sync(0xffffffffu, *cx.abort != 0u)) break;
            const int s = c & 1;
            const int t0 = c * C;
            const float *gv = gv_all + s * GV_STRIDE;
            if (!warp_wait(cx, B_X_FULL, c & 1)) break;
            GDN_TRACE_WARP(c, 16, W_STATE0);
            tc_fence_after();
            if (q >= 2) {
                // U' = U - W S^T for chunk row r -> U' and diag(exp(g_last - g)) U' (bf16)
                const int r = lrow - 64;
                // K enters the state update normalised: scale U' rows by 1/|k_r| too
                const float dc = kNorm ? gv[GV_DCY + r] * gv[GV_RK + r] : gv[GV_DCY + r];
                float x0[16], x1[16], u0[16], u1[16];
                tmem_ld16(lane_addr + TM_X + 32 * hf, x0);
                tmem_ld16(lane_addr + TM_X + 32 * hf + 16, x1);
                tmem_ld16(lane_addr + TM_U + 32 * hf, u0);
                tmem_ld16(lane_addr + TM_U + 32 * hf + 16, u1);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    u0[j] -= x0[j];
                    u1[j] -= x1[j];
                }
                store16_bf16(base + SM_UN, r, 2 * hf, u0);
                store16_bf16(base + SM_UN, r, 2 * hf + 1, u1);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    u0[j] *= dc;
                    u1[j] *= dc;
                }
                store16_bf16(base + SM_UP, r, 2 * hf, u0);
                store16_bf16(base + SM_UP, r, 2 * hf + 1, u1);
                fence_async_smem();
                tc_fence_before();
                warp_arrive(cx, B_U_READY);
                warp_arrive(cx, B_WU_EMPTY);
                GDN_TRACE_WARP(c, 18, W_STATE0 + 2);
            } else {
                // inter-chunk part of the output, gamma_r (Q S^T)_r, into Y; the
                // intra-chunk MMA accumulates onto it
                // 1/|q_r| comes from the P warps (published with this chunk's P tile)
                if (kNorm && !warp_wait(cx, B_PREP_FULL + s, (c >> 1) & 1)) break;
                const float gr = kNorm ? gv[GV_GAM + lrow] * gv[GV_RQ + lrow] : gv[GV_GAM + lrow];
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
                tc_fence_before();
                warp_arrive(cx, B_U_READY);
            }
            // state hand-off: S^T (gamma-scaled + update) -> bf16 copy; TMEM pre-scaled
            if (!warp_wait(cx, B_ST_FULL, c & 1)) break;
            GDN_TRACE_WARP(c, 20, W_STATE0);
            tc_fence_after();
            {
                const bool last = c + 1 >= NT;
                bool have = false;
                float gl = 1.f;
                if (!last) {
                    have = warp_wait(cx, B_IN_FULL + (s ^ 1), ((c + 1) >> 1) & 1);
                    gl = gv_all[(s ^ 1) * GV_STRIDE + GV_GL];
                }
                float s0[16], s1[16];
                tmem_ld16(lane_addr + TM_ST + 32 * hf, s0);
                tmem_ld16(lane_addr + TM_ST + 32 * hf + 16, s1);
                tmem_wait_ld();
                if (!last) {
                    store16_bf16(sbuf, lrow, 2 * hf, s0);
                    store16_bf16(sbuf, lrow, 2 * hf + 1, s1);
                    if (p.S_hist) {  // the state entering chunk c + 1
                        float *dst = p.S_hist + (((size_t)head * NT + c + 1) * p.Dv + v0 + 32 * hf) * DK + lrow;
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            dst[j * DK] = s0[j];
                            dst[(16 + j) * DK] = s1[j];
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        s0[j] *= gl;
                        s1[j] *= gl;
                    }
                    if (have) {
                        tmem_st16(lane_addr + TM_ST + 32 * hf, s0);
                        tmem_st16(lane_addr + TM_ST + 32 * hf + 16, s1);
                    }
                    fence_async_smem();
                    tmem_wait_st();
                } else if (p.S_T) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        p.S_T[(head * p.Dv + v0 + 32 * hf + j) * DK + lrow] = s0[j];
                        p.S_T[(head * p.Dv + v0 + 32 * hf + 16 + j) * DK + lrow] = s1[j];
                    }
                }
                tc_fence_before();
                warp_arrive(cx, B_S_READY);
                GDN_TRACE_WARP(c, 21, W_STATE0);
                GDN_TRACE_WARP(c, 4, W_STATE0 + 7);
                if (!last && !have) break;
            }
            if (c + 1 < NT) copy_w(c + 1);
            // chunk output rows (lanes 0-63)
            if (q < 2) {
                if (!warp_wait(cx, B_Y_FULL, c & 1)) break;
                GDN_TRACE_WARP(c, 19, W_STATE0);
                tc_fence_after();
                float y0[16], y1[16];
                tmem_ld16(lane_addr + TM_Y + 32 * hf, y0);
                tmem_ld16(lane_addr + TM_Y + 32 * hf + 16, y1);
                tmem_wait_ld();
                if (t0 + lrow < T) {
                    uint4 *dst = reinterpret_cast<uint4 *>(
                        p.o + ((size_t)(sp.off + t0 + lrow) * H + h) * p.Dv + v0 + 32 * hf);
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        dst[k] = make_uint4(pack_bf16(y0[8 * k + 0], y0[8 * k + 1]),
                                            pack_bf16(y0[8 * k + 2], y0[8 * k + 3]),
                                            pack_bf16(y0[8 * k + 4], y0[8 * k + 5]),
                                            pack_bf16(y0[8 * k + 6], y0[8 * k + 7]));
                        dst[2 + k] = make_uint4(pack_bf16(y1[8 * k + 0], y1[8 * k + 1]),
                                                pack_bf16(y1[8 * k + 2], y1[8 * k + 3]),
                                                pack_bf16(y1[8 * k + 4], y1[8 * k + 5]),
                                                pack_bf16(y1[8 * k + 6], y1[8 * k + 7]));
                    }
                }
                tc_fence_before();
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

// Workspace of [T'; T''] tiles, [n_tiles, 128, 64] bf16: box of one whole tile, 128B swizzle.
bool make_map_tt(CUtensorMap *m, const void *ptr, long long n_tiles) {
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)C, (cuuint64_t)(2 * C), (cuuint64_t)n_tiles};
    cuuint64_t strides[2] = {(cuuint64_t)C * 2, (cuuint64_t)TT_ELEMS * 2};
    cuuint32_t box[3] = {(cuuint32_t)C, (cuuint32_t)(2 * C), 1};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box,
               es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tc

// Workspace: [chunk offsets of the sequences, variable lengths only, padded to
// 256 B][one [T'; T''] tile per chunk and head][1/|k| per token, normalising only].
// chunk offsets (n + 1) and launch order (n) of the sequences
size_t tc_offsets_bytes(int n_seq, bool varlen) {
    return varlen ? ((2 * (size_t)n_seq + 1) * sizeof(int) + 255) & ~size_t(255) : 0;
}

// The fused variant's sequential grid has Dv / 64 x H x (sequences) CTAs of one
// SM each; below this many the GPU is mostly idle, HBM bandwidth is to spare,
// and the precomputed variant's shorter per-chunk chain wins.
constexpr int kFewSeqCtas = 74;

bool tc_precomputed(int n_seq, int H, int Dk, int Dv) {
    return Dk == 256 || (long long)(Dv / tc::DVT) * H * n_seq < kFewSeqCtas;
}

static size_t fused_workspace_bytes(int n_seq, long long total_chunks, int H, bool varlen,
                                    unsigned flags) {
    const size_t tiles = (size_t)total_chunks * H * tc::TT_ELEMS * sizeof(__nv_bfloat16);
    const size_t rk = (flags & kFlagL2Norm) ? (size_t)total_chunks * H * tc::C * sizeof(float) : 0;
    return tc_offsets_bytes(n_seq, varlen) + tiles + rk;
}

size_t tc_workspace_bytes_seqs(int n_seq, long long total_chunks, int H, bool varlen,
                               unsigned flags, int Dk, int Dv) {
    if (tc_precomputed(n_seq, H, Dk, Dv))
        return tcw_workspace_bytes_seqs(n_seq, total_chunks, H, varlen, flags, Dk);
    return fused_workspace_bytes(n_seq, total_chunks, H, varlen, flags);
}

size_t tc_workspace_bytes(int B, int T, int H, unsigned flags, int Dk, int Dv) {
    if (tc_precomputed(B, H, Dk, Dv) && tcw_split_segments(B, T, H, Dk, Dv) > 1)
        return tcw_split_workspace_bytes(B, T, H, Dv, flags);
    const long long NT = ((long long)T + tc::C - 1) / tc::C;
    return tc_workspace_bytes_seqs(B, (long long)B * NT, H, false, flags, Dk, Dv);
}

size_t tc_workspace_bytes_fused(int B, int T, int H, unsigned flags) {
    const long long NT = ((long long)T + tc::C - 1) / tc::C;
    return fused_workspace_bytes(B, (long long)B * NT, H, false, flags);
}

bool tc_supported(int B, int T, int H, int Dk, int Dv, int chunk, bool bf16) {
    return bf16 && chunk == tc::C && (Dk == tc::DK || Dk == 256) && Dv % tc::DVT == 0 &&
           B >= 1 && T >= 1 && H >= 1 && tc::encode_fn() != nullptr;
}

cudaError_t launch_seq_schedule(const int *cu_seqlens, int n_seq, int *cu_chunks, int *order,
                                cudaStream_t st) {
    tc::seq_schedule<<<1, tc::kScheduleThreads, 0, st>>>(cu_seqlens, n_seq, cu_chunks, order);
    return cudaPeekAtLastError();
}

cudaError_t launch_chunk_tc_seqs(const void *q, const void *k, const void *v,
                                 const float *log_alpha, const float *beta, const float *S0,
                                 void *o, float *S_T, int n_seq, int T_fixed, long long total_T,
                                 const int *cu_seqlens, long long total_chunks, int H, int Dk,
                                 int Dv, unsigned flags, void *workspace, cudaStream_t st,
                                 float *S_hist) {
    // the state history (for the backward) is a feature of the fused variant
    if (S_hist && Dk != tc::DK) return cudaErrorInvalidValue;
    if (!S_hist && tc_precomputed(n_seq, H, Dk, Dv))
        return launch_chunk_tcw_seqs(q, k, v, log_alpha, beta, S0, o, S_T, n_seq, T_fixed, total_T,
                                     cu_seqlens, total_chunks, H, Dk, Dv, flags, workspace, st);
    const bool varlen = cu_seqlens != nullptr;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int *cu_chunks = varlen ? reinterpret_cast<int *>(ws) : nullptr;
    auto *tt = reinterpret_cast<__nv_bfloat16 *>(ws + tc_offsets_bytes(n_seq, varlen));
    float *rk = (flags & kFlagL2Norm)
                    ? reinterpret_cast<float *>(tt + (size_t)total_chunks * H * tc::TT_ELEMS)
                    : nullptr;
    CUtensorMap mq, mk, mv, mt;
    if (!tc::make_map(&mq, q, 1, (int)total_T, H, Dk) ||
        !tc::make_map(&mk, k, 1, (int)total_T, H, Dk) ||
        !tc::make_map(&mv, v, 1, (int)total_T, H, Dv) ||
        !tc::make_map_tt(&mt, tt, total_chunks > 0 ? total_chunks * H : 1))
        return cudaErrorInvalidValue;
    if (varlen) {
        const cudaError_t e0 = launch_seq_schedule(cu_seqlens, n_seq, cu_chunks,
                                                   cu_chunks + n_seq + 1, st);
        if (e0 != cudaSuccess) return e0;
    }
    tc::Params p;
    p.log_alpha = log_alpha;
    p.beta = beta;
    p.S0 = S0;
    p.o = static_cast<__nv_bfloat16 *>(o);
    p.S_T = S_T;
    p.sq = tc::Seqs{cu_seqlens, cu_chunks, varlen ? cu_chunks + n_seq + 1 : nullptr, T_fixed,
                    n_seq};
    p.H = H;
    p.Dv = Dv;
    p.rk = rk;
    p.flags = flags;
    p.S_hist = varlen ? nullptr : S_hist;
    const bool norm = (flags & kFlagL2Norm) != 0;
    auto *ut = norm ? tc::gdn_ut_kernel<true> : tc::gdn_ut_kernel<false>;
    auto *seq = norm ? tc::gdn_chunk_tc_kernel<true> : tc::gdn_chunk_tc_kernel<false>;
    const int ut_smem = tc::UT_SMEM;
    cudaError_t e = cudaFuncSetAttribute(ut, cudaFuncAttributeMaxDynamicSharedMemorySize, ut_smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(seq, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (total_chunks > 0)
        ut<<<dim3((unsigned)total_chunks, H, 1), tc::UT_THREADS, ut_smem, st>>>(
            mk, log_alpha, beta, tt, rk, p.sq, H, flags);
    e = cudaPeekAtLastError();
    if (e != cudaSuccess) return e;
    // programmatic dependent launch: the CTAs may start (TMEM, barriers, the initial
    // state) while the UT kernel drains; the TMA warp waits for it before loading
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(Dv / tc::DVT, H, n_seq);
    cfg.blockDim = dim3(tc::NTHREADS);
    cfg.dynamicSmemBytes = tc::SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, seq, mq, mk, mv, mt, p);
    if (e != cudaSuccess) return e;
    return cudaPeekAtLastError();
}

cudaError_t launch_chunk_tc(const void *q, const void *k, const void *v, const float *log_alpha,
                            const float *beta, const float *S0, void *o, float *S_T, int B, int T,
                            int H, int Dk, int Dv, unsigned flags, void *workspace,
                            cudaStream_t st, float *S_hist) {
    // a fixed-length batch is B packed sequences of length T
    const long long NT = ((long long)T + tc::C - 1) / tc::C;
    return launch_chunk_tc_seqs(q, k, v, log_alpha, beta, S0, o, S_T, B, T, (long long)B * T,
                                nullptr, (long long)B * NT, H, Dk, Dv, flags, workspace, st,
                                S_hist);
}

#ifdef GDN_TRACE
extern "C" int gdn_trace_read(unsigned long long *dst) {
    return (int)cudaMemcpyFromSymbol(dst, g_trace, sizeof(g_trace));
}
extern "C" int gdn_tracew_read(unsigned long long *dst) {
    return (int)cudaMemcpyFromSymbol(dst, g_tracew, sizeof(g_tracew));
}
#endif

cudaError_t set_withhold_first_arrival(bool on) {
    const unsigned int v = on ? 1u : 0u;
    return cudaMemcpyToSymbol(g_tc_withhold_first, &v, sizeof(v));
}

cudaError_t read_and_clear_device_error(unsigned int *flag) {
    cudaError_t e = cudaMemcpyFromSymbol(flag, g_tc_error, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_tc_error, &zero, sizeof(unsigned int));
}

}  // namespace gdn
