// Pieces shared by the tcgen05 chunkwise-forward kernels (chunk_tc.cu for
// Dk = 128, chunk_tc_wide.cu for Dk = 256): bounded mbarrier waits with a CTA
// abort flag, bf16 packing into 128-byte-swizzled tiles, the blocked UT
// transform T = (I + A)^-1 of a 64 x 64 chunk, and the description of packed
// sequences.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "sm100.cuh"

namespace gdn {
namespace tc {

using namespace sm100;

constexpr int C = 64;          // chunk length (tokens)
constexpr int LDA = 68;        // padded float32 row stride of A and T (16-B rows)

constexpr uint64_t kTimeoutNs = 2000000000ull;

__device__ __forceinline__ uint64_t now_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// 2^x (hardware approximation, relative error about 2^-22)
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

struct Ctx {
    uint8_t *base;
    uint64_t *bar;
    volatile uint32_t *abort;
    unsigned int *err;     // the kernel's device-wide error flag (set on a timeout)
};

// Bounded wait; false (and the CTA-wide abort flag set) on timeout or abort.
static __device__ __noinline__ bool wait_bar(const Ctx &cx, int idx, uint32_t parity) {
    uint64_t *b = cx.bar + idx;
#ifdef GDN_WAIT_TEST_SLEEP_NS
    {
        if (mbar_test_wait(b, parity)) return true;
        const uint64_t t0 = now_ns();
        for (uint32_t it = 1;; ++it) {
            __nanosleep(GDN_WAIT_TEST_SLEEP_NS);
            if (mbar_test_wait(b, parity)) return true;
            if ((it & 63u) == 0) {
                if (*cx.abort) return false;
                if (now_ns() - t0 > kTimeoutNs) {
                    *cx.abort = 1u;
                    atomicOr(cx.err, 1u);
                    return false;
                }
            }
        }
    }
#endif
    if (mbar_try_wait(b, parity)) return true;
    const uint64_t t0 = now_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(b, parity)) return true;
#ifdef GDN_WAIT_BACKOFF_NS
        if (it > 32) __nanosleep(GDN_WAIT_BACKOFF_NS);
#endif
        if ((it & 255u) == 0) {
            if (*cx.abort) return false;
            if (now_ns() - t0 > kTimeoutNs) {
                *cx.abort = 1u;
                atomicOr(cx.err, 1u);
                return false;
            }
        }
    }
}

// Slow path of warp_wait: lane 0 polls (so waiting warps do not compete with
// working warps for the shared-memory pipe) and the result is broadcast.
static __device__ __noinline__ bool warp_wait_slow(const Ctx &cx, int idx, uint32_t parity) {
    bool ok = true;
    if ((threadIdx.x & 31) == 0) ok = wait_bar(cx, idx, parity);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    __syncwarp();  // orders the other lanes' later accesses after lane 0's acquire
    return ok;
}

// A wait on behalf of a whole warp.  The common case (the phase has already
// completed) is one test and a vote, with no divergent branch; the result is
// warp-uniform, so a timeout never splits a warp in front of a warp-collective
// tcgen05 access.
__device__ __forceinline__ bool warp_wait(const Ctx &cx, int idx, uint32_t parity) {
    if (__all_sync(0xffffffffu, mbar_try_wait(cx.bar + idx, parity))) return true;
    return warp_wait_slow(cx, idx, parity);
}

// One arrival on behalf of a whole warp, after every lane's prior writes
// (lane 0 arrives, predicated rather than branched).
__device__ __forceinline__ void warp_arrive(const Ctx &cx, int idx) {
    __syncwarp();
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.eq.u32 p, %1, 0;\n\t"
        "@p mbarrier.arrive.shared::cta.b64 _, [%0];\n\t}" ::"r"(smem_u32(cx.bar + idx)),
        "r"(threadIdx.x & 31u)
        : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// Columns [16 piece, 16 piece + 16) of bf16 row `row` of a 128B-swizzled tile.
__device__ __forceinline__ void store16_bf16(uint8_t *tile, int row, int piece, const float (&v)[16]) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        uint4 q;
        q.x = pack_bf16(v[8 * k + 0], v[8 * k + 1]);
        q.y = pack_bf16(v[8 * k + 2], v[8 * k + 3]);
        q.z = pack_bf16(v[8 * k + 4], v[8 * k + 5]);
        q.w = pack_bf16(v[8 * k + 6], v[8 * k + 7]);
        *reinterpret_cast<uint4 *>(tile + sw128_offset(row, (2 * piece + k) * 16)) = q;
    }
}

__device__ __forceinline__ void tmem_ld16w(uint32_t taddr, float (&v)[16]) {
    tmem_ld16(taddr, v);
    tmem_wait_ld();
}

// The UT transform T = (I + A)^-1 of the 64 x 64 strictly lower A (AF, float32,
// stride LDA), blocked by 16 with D_I = I + A_II:
//   T_II = D_I^-1                                   (ut_diag, forward substitution)
//   N_IJ = T_II A_IJ,  I > J                        (ut_offdiag4 phase 1, all six blocks)
//   T_IJ = -sum_{J <= K < I} N_IK T_KJ              (phase 2, one warp per block column)
// TF receives the lower triangle and the diagonal; its strict upper part is not
// written (and never read).

// Column j of T_II for block I = p / 16 (p < 64).
__device__ __forceinline__ void ut_diag(const float *__restrict__ AF, float *__restrict__ TF, int p) {
    const int I = p >> 4, j = p & 15, o = 16 * I;
    float x[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        float a[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 v = *reinterpret_cast<const float4 *>(AF + (o + r) * LDA + o + 4 * q);
            a[4 * q] = v.x; a[4 * q + 1] = v.y; a[4 * q + 2] = v.z; a[4 * q + 3] = v.w;
        }
        float acc0 = 0.f, acc1 = 0.f;  // two partial sums: shorter dependency chains
#pragma unroll
        for (int i = 0; i < r; ++i) {
            if (i & 1) acc1 = fmaf(a[i], x[i], acc1);
            else acc0 = fmaf(a[i], x[i], acc0);
        }
        x[r] = (r == j) ? 1.f : ((r < j) ? 0.f : -(acc0 + acc1));
    }
#pragma unroll
    for (int r = 0; r < 16; ++r) TF[(o + r) * LDA + o + j] = x[r];
}

// acc (16 x 16 as two 16 x 8 mma tiles) += Ablk (16 x 16, stride lda) * Bblk
// (16 x 16, stride ldb), TF32 tensor-core products with float32 accumulation;
// one warp.
__device__ __forceinline__ void mma16(float (&acc)[2][4], const float *__restrict__ A, int lda,
                                      const float *__restrict__ B, int ldb, int g, int t) {
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        const int k0 = 8 * ks;
        const uint32_t a[4] = {to_tf32(A[g * lda + k0 + t]), to_tf32(A[(g + 8) * lda + k0 + t]),
                               to_tf32(A[g * lda + k0 + t + 4]), to_tf32(A[(g + 8) * lda + k0 + t + 4])};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const uint32_t bb[2] = {to_tf32(B[(k0 + t) * ldb + 8 * nt + g]),
                                    to_tf32(B[(k0 + t + 4) * ldb + 8 * nt + g])};
            mma_tf32_16x8x8(acc[nt], a, bb);
        }
    }
}

__device__ __forceinline__ void store16x16(const float (&acc)[2][4], float *__restrict__ D, int ld,
                                           float sign, int g, int t) {
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        *reinterpret_cast<float2 *>(D + g * ld + 8 * nt + 2 * t) = make_float2(sign * acc[nt][0], sign * acc[nt][1]);
        *reinterpret_cast<float2 *>(D + (g + 8) * ld + 8 * nt + 2 * t) = make_float2(sign * acc[nt][2], sign * acc[nt][3]);
    }
}

// Off-diagonal blocks of T with 4 warps, N_IJ = T_II A_IJ stored over A_IJ:
//   phase 1  N for the six blocks (1,0) (2,0) (2,1) (3,0) (3,1) (3,2), two rounds
//   phase 2  T_{J+1,J} = -N_{J+1,J} T_JJ                              (3 warps)
//   phase 3  T_{J+2,J} = -(N_{J+2,J} T_JJ + N_{J+2,J+1} T_{J+1,J})    (2 warps)
//   phase 4  T_30 = -(N_30 T_00 + N_31 T_10 + N_32 T_20)              (1 warp)
// kBar = 0: the CTA has exactly these 4 warps and synchronises with
// __syncthreads; kBar > 0: only warps 0-3 of a larger CTA call it and they
// synchronise on named barrier kBar (128 threads).
template <int kBar = 0>
__device__ __forceinline__ void ut_offdiag4(float *__restrict__ AF, float *__restrict__ TF,
                                            int p) {
    const int w = p >> 5, lane = p & 31, g = lane >> 2, t = lane & 3;
    const auto blk = [&](float *M, int I, int J) { return M + 16 * I * LDA + 16 * J; };
#pragma unroll
    for (int round = 0; round < 2; ++round) {
        const int k = w + 4 * round;  // block (I, J) in the order listed above
        if (k < 6) {
            const int I = k == 0 ? 1 : (k < 3 ? 2 : 3), J = k == 0 ? 0 : (k < 3 ? k - 1 : k - 3);
            float acc[2][4] = {};
            mma16(acc, blk(TF, I, I), LDA, blk(AF, I, J), LDA, g, t);
            __syncwarp();
            store16x16(acc, blk(AF, I, J), LDA, 1.f, g, t);
        }
    }
    if constexpr (kBar > 0)
        named_barrier(kBar, 128);
    else
        __syncthreads();
    // block column J of T needs only its own earlier blocks and the N blocks:
    // warp J walks down it, T_IJ = -sum_{K=J}^{I-1} N_IK T_KJ, with no CTA barrier
    if (w < 3) {
        const int J = w;
        for (int I = J + 1; I < 4; ++I) {
            float acc[2][4] = {};
            for (int K = J; K < I; ++K)
                mma16(acc, blk(AF, I, K), LDA, blk(TF, K, J), LDA, g, t);
            store16x16(acc, blk(TF, I, J), LDA, -1.f, g, t);
            __syncwarp();
        }
    }
    if constexpr (kBar > 0)
        named_barrier(kBar, 128);
    else
        __syncthreads();
}

// ------------------------------------------------------------- sequences --
// Where each sequence lives in the packed token dimension ([tokens, H, D] rows):
// a fixed-length batch (cu == nullptr: sequence b is tokens [b T, b T + T)) or
// variable lengths (tokens cu[b] .. cu[b + 1]).  Chunks are numbered globally,
// sequence by sequence: sequence b owns chunks chunk0 .. chunk0 + ceil(len / C).
struct Seqs {
    const int *cu;         // n + 1 token offsets (device), or null
    const int *cu_chunks;  // n + 1 chunk offsets (device), or null
    const int *order;      // launch order of the sequences (device), or null
    int T;                 // the common length when cu is null
    int n;                 // number of sequences
};

struct Span {
    int off, len, chunk0;
};

__device__ __forceinline__ Span seq_span(const Seqs &q, int b) {
    if (q.cu) return Span{q.cu[b], q.cu[b + 1] - q.cu[b], q.cu_chunks[b]};
    return Span{b * q.T, q.T, b * ((q.T + C - 1) / C)};
}

// The sequence a global chunk index belongs to: the last b with cu_chunks[b] <= g
// (empty sequences share their start with the next one and are skipped).
__device__ __forceinline__ int seq_of_chunk(const Seqs &q, int g) {
    if (!q.cu) return g / ((q.T + C - 1) / C);
    int lo = 0, hi = q.n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (q.cu_chunks[mid] <= g) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Host side, defined in chunk_tc.cu: the driver's tensor-map encoder, and the
// maps of a [B, T, H, D] bf16 tensor (box 64 channels x 1 head x 64 tokens x 1,
// 128-byte swizzle) and of a [n_tiles, 128, 64] bf16 tile array (box one tile).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn();
bool make_map(CUtensorMap *m, const void *ptr, int B, int T, int H, int D);
bool make_map_tt(CUtensorMap *m, const void *ptr, long long n_tiles);

}  // namespace tc
}  // namespace gdn
