// C-ABI entry points of libgdn.so (declared in include/gdn.h): argument checks
// on the host, then dispatch to the kernels.  Nothing is launched when a check
// fails, and the library allocates nothing.
#include <stdint.h>

#include "../../include/gdn.h"
#include "kernels.h"

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Byte ranges [a, a+na) and [b, b+nb) intersect.
bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

constexpr int kMaxDk = 256, kMaxDv = 512, kMaxGrid = 65535;
constexpr unsigned long long kMaxTokenHeads = 1ull << 40;

// 0 = fine, otherwise the status to return.
gdn_status_t check_sizes(int B, int T, int H, int Dk, int Dv, int chunk, gdn_dtype_t dtype) {
    if (B < 0 || T < 0 || H < 0 || Dk <= 0 || Dv <= 0) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (Dk > kMaxDk || Dv > kMaxDv) return GDN_ERR_UNSUPPORTED;
    if (chunk != 16 && chunk != 32 && chunk != 64) return GDN_ERR_UNSUPPORTED;
    if (B > kMaxGrid || H > kMaxGrid) return GDN_ERR_UNSUPPORTED;
    // bound the token-head count so that every byte count derived from the sizes
    // (tensors, states, workspaces) stays far inside size_t
    if ((unsigned long long)B * (unsigned long long)H * ((unsigned long long)T + 64) > kMaxTokenHeads)
        return GDN_ERR_UNSUPPORTED;
    return GDN_OK;
}

bool empty_problem(int B, int T, int H) { return B == 0 || H == 0 || T == 0; }

constexpr unsigned kKnownFlags = GDN_FLAG_L2NORM_QK | GDN_FLAG_GATE_LOGITS;
size_t align256(size_t n) { return (n + 255) & ~size_t(255); }

// Packed-sequence offsets: N + 1 ints from 0, non-decreasing, total below 2^31.
struct Offsets {
    long long total = 0, chunks64 = 0;  // tokens; chunks of 64 tokens over all sequences
    int max_len = 0;
};
bool read_offsets(const int *cu, int N, Offsets *out) {
    if (!cu || N < 0 || cu[0] != 0) return false;
    for (int n = 0; n < N; ++n) {
        const long long len = (long long)cu[n + 1] - cu[n];
        if (len < 0) return false;
        out->chunks64 += (len + 63) / 64;
        if (len > out->max_len) out->max_len = (int)len;
    }
    out->total = cu[N];
    return true;
}

}  // namespace

extern "C" {

const char *gdn_status_string(gdn_status_t status) {
    switch (status) {
        case GDN_OK: return "ok";
        case GDN_ERR_INVALID_ARG: return "invalid argument";
        case GDN_ERR_UNSUPPORTED: return "unsupported size or type";
        case GDN_ERR_CUDA: return "CUDA launch failed";
    }
    return "unknown status";
}

int gdn_chunk_fwd_path(int B, int T, int H, int Dk, int Dv, int chunk, gdn_dtype_t dtype) {
    if (check_sizes(B, T, H, Dk, Dv, chunk, dtype) != GDN_OK) return -1;
    if (empty_problem(B, T, H)) return GDN_PATH_NONE;
    if (gdn::tc_supported(B, T, H, Dk, Dv, chunk, dtype == GDN_BF16)) return GDN_PATH_TCGEN05;
    return GDN_PATH_SIMT;
}

int gdn_chunk_fwd_variant(int B, int T, int H, int Dk, int Dv, int chunk, gdn_dtype_t dtype) {
    if (gdn_chunk_fwd_path(B, T, H, Dk, Dv, chunk, dtype) != GDN_PATH_TCGEN05) return 0;
    if (!gdn::tc_precomputed(B, H, Dk, Dv)) return 1;
    return gdn::tcw_split_segments(B, T, H, Dk, Dv) > 1 ? 3 : 2;
}

size_t gdn_chunk_fwd_workspace_size_ex(int B, int T, int H, int Dk, int Dv, int chunk,
                                       gdn_dtype_t dtype, unsigned flags) {
    const int path = gdn_chunk_fwd_path(B, T, H, Dk, Dv, chunk, dtype);
    if (flags & ~kKnownFlags) return 0;
    if (path == GDN_PATH_TCGEN05) return gdn::tc_workspace_bytes(B, T, H, flags, Dk, Dv);
    if (path == GDN_PATH_SIMT) {
        const size_t base = gdn::simt_workspace_bytes(B, T, H, chunk);
        return flags ? align256(base) + gdn::prologue_bytes(B, T, H, Dk, dtype == GDN_BF16, flags)
                     : base;
    }
    return 0;
}

size_t gdn_chunk_fwd_workspace_size(int B, int T, int H, int Dk, int Dv, int chunk,
                                    gdn_dtype_t dtype) {
    return gdn_chunk_fwd_workspace_size_ex(B, T, H, Dk, Dv, chunk, dtype, 0u);
}

gdn_status_t gdn_chunk_fwd(const void *q, const void *k, const void *v, const float *log_alpha,
                           const float *beta, const float *S0, void *o, float *S_T, int B, int T,
                           int H, int Dk, int Dv, int chunk, gdn_dtype_t dtype, void *workspace,
                           size_t workspace_bytes, void *stream) {
    return gdn_chunk_fwd_ex(q, k, v, log_alpha, beta, S0, o, S_T, B, T, H, Dk, Dv, chunk, dtype,
                            0u, workspace, workspace_bytes, stream);
}

gdn_status_t gdn_chunk_fwd_ex(const void *q, const void *k, const void *v,
                              const float *log_alpha, const float *beta, const float *S0, void *o,
                              float *S_T, int B, int T, int H, int Dk, int Dv, int chunk,
                              gdn_dtype_t dtype, unsigned flags, void *workspace,
                              size_t workspace_bytes, void *stream) {
    const gdn_status_t sz = check_sizes(B, T, H, Dk, Dv, chunk, dtype);
    if (sz != GDN_OK) return sz;
    if (flags & ~kKnownFlags) return GDN_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t esz = dtype == GDN_BF16 ? 2 : 4;
    const size_t n_tok = (size_t)B * T * H;
    const size_t state_bytes = (size_t)B * H * Dv * Dk * sizeof(float);
    if (B == 0 || H == 0) return GDN_OK;
    if (T == 0) {  // no tokens: the final state is the initial one
        if (!S_T) return GDN_OK;
        if (!aligned16(S_T) || (S0 && !aligned16(S0))) return GDN_ERR_INVALID_ARG;
        cudaError_t e = S0 ? (S0 == S_T ? cudaSuccess
                                        : cudaMemcpyAsync(S_T, S0, state_bytes,
                                                          cudaMemcpyDeviceToDevice, st))
                           : cudaMemsetAsync(S_T, 0, state_bytes, st);
        return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
    }
    if (!q || !k || !v || !log_alpha || !beta || !o) return GDN_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, log_alpha, beta, S0, o, S_T, workspace};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
    const size_t o_bytes = n_tok * Dv * esz;
    if (overlaps(o, o_bytes, q, n_tok * Dk * esz) || overlaps(o, o_bytes, k, n_tok * Dk * esz) ||
        overlaps(o, o_bytes, v, n_tok * Dv * esz))
        return GDN_ERR_INVALID_ARG;
    if (S_T && S0 && S_T != S0 && overlaps(S_T, state_bytes, S0, state_bytes))
        return GDN_ERR_INVALID_ARG;

    const bool bf16 = dtype == GDN_BF16;
    const bool tc = gdn::tc_supported(B, T, H, Dk, Dv, chunk, bf16);
    const size_t need = gdn_chunk_fwd_workspace_size_ex(B, T, H, Dk, Dv, chunk, dtype, flags);
    if (!workspace || workspace_bytes < need) return GDN_ERR_INVALID_ARG;
    // the workspace is scratch written by the kernels: it must not alias anything else
    if (overlaps(workspace, need, q, n_tok * Dk * esz) ||
        overlaps(workspace, need, k, n_tok * Dk * esz) ||
        overlaps(workspace, need, v, n_tok * Dv * esz) ||
        overlaps(workspace, need, log_alpha, n_tok * sizeof(float)) ||
        overlaps(workspace, need, beta, n_tok * sizeof(float)) ||
        overlaps(workspace, need, o, o_bytes) ||
        (S0 && overlaps(workspace, need, S0, state_bytes)) ||
        (S_T && overlaps(workspace, need, S_T, state_bytes)))
        return GDN_ERR_INVALID_ARG;
    cudaError_t e;
    if (tc) {
        e = gdn::launch_chunk_tc(q, k, v, log_alpha, beta, S0, o, S_T, B, T, H, Dk, Dv, flags,
                                 workspace, st);
    } else {
        // the prologue's output sits after the CUDA-core path's own scratch
        gdn::Prepared in{q, k, log_alpha, beta};
        e = cudaSuccess;
        if (flags)
            e = gdn::launch_prologue(
                q, k, log_alpha, beta, B, T, H, Dk, bf16, flags,
                static_cast<uint8_t *>(workspace) + align256(gdn::simt_workspace_bytes(B, T, H, chunk)),
                &in, st);
        if (e == cudaSuccess)
            e = gdn::launch_chunk_simt(in.q, in.k, v, in.log_alpha, in.beta, S0, o, S_T, B, T, H,
                                       Dk, Dv, chunk, bf16, workspace, st);
    }
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

size_t gdn_chunk_fwd_varlen_workspace_size(const int *cu_seqlens_host, int N, int H, int Dk,
                                           int Dv, int chunk, gdn_dtype_t dtype, unsigned flags) {
    Offsets off;
    if ((flags & ~kKnownFlags) || !read_offsets(cu_seqlens_host, N, &off)) return 0;
    if (check_sizes(N, off.max_len, H, Dk, Dv, chunk, dtype) != GDN_OK) return 0;
    if (N == 0 || H == 0 || off.total == 0) return 0;
    const bool bf16 = dtype == GDN_BF16;
    if (gdn::tc_supported(N, off.max_len, H, Dk, Dv, chunk, bf16))
        return gdn::tc_workspace_bytes_seqs(N, off.chunks64, H, true, flags, Dk, Dv);
    // CUDA-core path: one sequence at a time (scratch for the longest), prologue once
    const size_t base = gdn::simt_workspace_bytes(1, off.max_len, H, chunk);
    return flags ? align256(base) +
                       gdn::prologue_bytes(1, (int)off.total, H, Dk, bf16, flags)
                 : base;
}

gdn_status_t gdn_chunk_fwd_varlen(const void *q, const void *k, const void *v,
                                  const float *log_alpha, const float *beta, const float *S0,
                                  void *o, float *S_T, const int *cu_seqlens,
                                  const int *cu_seqlens_host, int N, int H, int Dk, int Dv,
                                  int chunk, gdn_dtype_t dtype, unsigned flags, void *workspace,
                                  size_t workspace_bytes, void *stream) {
    if (flags & ~kKnownFlags) return GDN_ERR_INVALID_ARG;
    Offsets off;
    if (!read_offsets(cu_seqlens_host, N, &off)) return GDN_ERR_INVALID_ARG;
    const gdn_status_t sz = check_sizes(N, off.max_len, H, Dk, Dv, chunk, dtype);
    if (sz != GDN_OK) return sz;
    if (off.total > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t esz = dtype == GDN_BF16 ? 2 : 4;
    const size_t n_tok = (size_t)off.total * H;
    const size_t head_state = (size_t)H * Dv * Dk;  // floats of one sequence's state
    const size_t state_bytes = (size_t)N * head_state * sizeof(float);
    if (N == 0 || H == 0) return GDN_OK;
    if (S_T && (!aligned16(S_T) || (S0 && !aligned16(S0)))) return GDN_ERR_INVALID_ARG;
    if (S_T && S0 && S_T != S0 && overlaps(S_T, state_bytes, S0, state_bytes))
        return GDN_ERR_INVALID_ARG;
    const auto copy_state = [&](int n) -> cudaError_t {  // empty sequence n: S_T = S0
        if (!S_T) return cudaSuccess;
        float *dst = S_T + (size_t)n * head_state;
        if (!S0) return cudaMemsetAsync(dst, 0, head_state * sizeof(float), st);
        const float *src = S0 + (size_t)n * head_state;
        return src == dst ? cudaSuccess
                          : cudaMemcpyAsync(dst, src, head_state * sizeof(float),
                                            cudaMemcpyDeviceToDevice, st);
    };
    if (off.total == 0) {
        for (int n = 0; n < N; ++n)
            if (copy_state(n) != cudaSuccess) return GDN_ERR_CUDA;
        return GDN_OK;
    }
    if (!q || !k || !v || !log_alpha || !beta || !o || !cu_seqlens) return GDN_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, log_alpha, beta, o, workspace};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
    const size_t o_bytes = n_tok * Dv * esz;
    if (overlaps(o, o_bytes, q, n_tok * Dk * esz) || overlaps(o, o_bytes, k, n_tok * Dk * esz) ||
        overlaps(o, o_bytes, v, n_tok * Dv * esz))
        return GDN_ERR_INVALID_ARG;
    const size_t need =
        gdn_chunk_fwd_varlen_workspace_size(cu_seqlens_host, N, H, Dk, Dv, chunk, dtype, flags);
    if (!workspace || workspace_bytes < need) return GDN_ERR_INVALID_ARG;
    if (overlaps(workspace, need, q, n_tok * Dk * esz) ||
        overlaps(workspace, need, k, n_tok * Dk * esz) ||
        overlaps(workspace, need, v, n_tok * Dv * esz) ||
        overlaps(workspace, need, log_alpha, n_tok * sizeof(float)) ||
        overlaps(workspace, need, beta, n_tok * sizeof(float)) ||
        overlaps(workspace, need, o, o_bytes) ||
        (S0 && overlaps(workspace, need, S0, state_bytes)) ||
        (S_T && overlaps(workspace, need, S_T, state_bytes)) ||
        overlaps(workspace, need, cu_seqlens, ((size_t)N + 1) * sizeof(int)))
        return GDN_ERR_INVALID_ARG;
    const bool bf16 = dtype == GDN_BF16;
    cudaError_t e = cudaSuccess;
    if (gdn::tc_supported(N, off.max_len, H, Dk, Dv, chunk, bf16)) {
        e = gdn::launch_chunk_tc_seqs(q, k, v, log_alpha, beta, S0, o, S_T, N, 0, off.total,
                                      cu_seqlens, off.chunks64, H, Dk, Dv, flags, workspace, st);
    } else {
        // the CUDA-core path, one sequence at a time on the caller's stream (they reuse
        // the scratch in turn); the prologue runs once over all tokens
        gdn::Prepared in{q, k, log_alpha, beta};
        const size_t base = align256(gdn::simt_workspace_bytes(1, off.max_len, H, chunk));
        if (flags)
            e = gdn::launch_prologue(q, k, log_alpha, beta, 1, (int)off.total, H, Dk, bf16, flags,
                                     static_cast<uint8_t *>(workspace) + base, &in, st);
        for (int n = 0; n < N && e == cudaSuccess; ++n) {
            const int t0 = cu_seqlens_host[n], len = cu_seqlens_host[n + 1] - t0;
            if (len == 0) {
                e = copy_state(n);
                continue;
            }
            const size_t tk = (size_t)t0 * H;
            e = gdn::launch_chunk_simt(
                static_cast<const uint8_t *>(in.q) + tk * Dk * esz,
                static_cast<const uint8_t *>(in.k) + tk * Dk * esz,
                static_cast<const uint8_t *>(v) + tk * Dv * esz, in.log_alpha + tk, in.beta + tk,
                S0 ? S0 + (size_t)n * head_state : nullptr, static_cast<uint8_t *>(o) + tk * Dv * esz,
                S_T ? S_T + (size_t)n * head_state : nullptr, 1, len, H, Dk, Dv, chunk, bf16,
                workspace, st);
        }
    }
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

size_t gdn_chunk_bwd_workspace_size(int B, int T, int H, int Dk, int Dv, int chunk,
                                    gdn_dtype_t dtype) {
    if (check_sizes(B, T, H, Dk, Dv, chunk, dtype) != GDN_OK || !gdn::bwd_supported(Dk, chunk))
        return 0;
    if (empty_problem(B, T, H)) return 0;
    return gdn::bwd_workspace_bytes(B, T, H, Dk, Dv, chunk, dtype == GDN_BF16);
}

gdn_status_t gdn_chunk_bwd(const void *q, const void *k, const void *v, const float *log_alpha,
                           const float *beta, const float *S0, const void *d_o,
                           const float *dS_T, void *dq, void *dk, void *dv, float *dlog_alpha,
                           float *dbeta, float *dS0, int B, int T, int H, int Dk, int Dv,
                           int chunk, gdn_dtype_t dtype, void *workspace, size_t workspace_bytes,
                           void *stream) {
    const gdn_status_t sz = check_sizes(B, T, H, Dk, Dv, chunk, dtype);
    if (sz != GDN_OK) return sz;
    if (!gdn::bwd_supported(Dk, chunk)) return GDN_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t esz = dtype == GDN_BF16 ? 2 : 4;
    const size_t n_tok = (size_t)B * T * H;
    const size_t state_bytes = (size_t)B * H * Dv * Dk * sizeof(float);
    if (B == 0 || H == 0) return GDN_OK;
    if (T == 0) {  // no tokens: dS0 = dS_T
        if (!dS0) return GDN_OK;
        if (!aligned16(dS0) || (dS_T && !aligned16(dS_T))) return GDN_ERR_INVALID_ARG;
        if (dS_T && dS_T != dS0 && overlaps(dS0, state_bytes, dS_T, state_bytes))
            return GDN_ERR_INVALID_ARG;
        cudaError_t e = dS_T ? (dS_T == dS0 ? cudaSuccess
                                            : cudaMemcpyAsync(dS0, dS_T, state_bytes,
                                                              cudaMemcpyDeviceToDevice, st))
                             : cudaMemsetAsync(dS0, 0, state_bytes, st);
        return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
    }
    if (!q || !k || !v || !log_alpha || !beta || !d_o || !dq || !dk || !dv || !dlog_alpha ||
        !dbeta)
        return GDN_ERR_INVALID_ARG;
    const struct { const void *p; size_t n; } in[] = {
        {q, n_tok * Dk * esz}, {k, n_tok * Dk * esz}, {v, n_tok * Dv * esz},
        {log_alpha, n_tok * sizeof(float)}, {beta, n_tok * sizeof(float)}, {S0, state_bytes},
        {d_o, n_tok * Dv * esz}, {dS_T, state_bytes}};
    const struct { const void *p; size_t n; } out[] = {
        {dq, n_tok * Dk * esz}, {dk, n_tok * Dk * esz}, {dv, n_tok * Dv * esz},
        {dlog_alpha, n_tok * sizeof(float)}, {dbeta, n_tok * sizeof(float)}, {dS0, state_bytes}};
    for (const auto &a : in)
        if (a.p && !aligned16(a.p)) return GDN_ERR_INVALID_ARG;
    for (const auto &a : out)
        if (a.p && !aligned16(a.p)) return GDN_ERR_INVALID_ARG;
    if (workspace && !aligned16(workspace)) return GDN_ERR_INVALID_ARG;
    // outputs alias neither an input nor one another
    for (size_t i = 0; i < sizeof(out) / sizeof(out[0]); ++i) {
        for (const auto &a : in)
            if (overlaps(out[i].p, out[i].n, a.p, a.n)) return GDN_ERR_INVALID_ARG;
        for (size_t j = i + 1; j < sizeof(out) / sizeof(out[0]); ++j)
            if (overlaps(out[i].p, out[i].n, out[j].p, out[j].n)) return GDN_ERR_INVALID_ARG;
    }
    const size_t need = gdn::bwd_workspace_bytes(B, T, H, Dk, Dv, chunk, dtype == GDN_BF16);
    if (!workspace || workspace_bytes < need) return GDN_ERR_INVALID_ARG;
    for (const auto &a : in)
        if (overlaps(workspace, need, a.p, a.n)) return GDN_ERR_INVALID_ARG;
    for (const auto &a : out)
        if (overlaps(workspace, need, a.p, a.n)) return GDN_ERR_INVALID_ARG;
    const cudaError_t e = gdn::launch_chunk_bwd(q, k, v, log_alpha, beta, S0, d_o, dS_T, dq, dk, dv,
                                                dlog_alpha, dbeta, dS0, B, T, H, Dk, Dv, chunk,
                                                dtype == GDN_BF16, workspace, st);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

int gdn_chunk_bwd_path(int B, int T, int H, int Dk, int Dv, int chunk, gdn_dtype_t dtype) {
    if (check_sizes(B, T, H, Dk, Dv, chunk, dtype) != GDN_OK || !gdn::bwd_supported(Dk, chunk))
        return -1;
    if (empty_problem(B, T, H)) return GDN_PATH_NONE;
    if (gdn::bwd_tc_supported(B, T, H, Dk, Dv, chunk, dtype == GDN_BF16)) return GDN_PATH_TCGEN05;
    return GDN_PATH_SIMT;
}

int gdn_chunk_fwd_cw_path(int B, int T, int H, int Dk, int Dv, int chunk, gdn_dtype_t dtype) {
    if (check_sizes(B, T, H, Dk, Dv, chunk, dtype) != GDN_OK || !gdn::cw_supported(Dk, chunk))
        return -1;
    if (empty_problem(B, T, H)) return GDN_PATH_NONE;
    if (gdn::cw_tc_supported(B, T, H, Dk, Dv, chunk, dtype == GDN_BF16)) return GDN_PATH_TCGEN05;
    return GDN_PATH_SIMT;
}

size_t gdn_chunk_fwd_cw_workspace_size(int B, int T, int H, int Dk, int Dv, int chunk,
                                       gdn_dtype_t dtype) {
    const int path = gdn_chunk_fwd_cw_path(B, T, H, Dk, Dv, chunk, dtype);
    if (path == GDN_PATH_TCGEN05) return gdn::cw_tc_workspace_bytes(B, T, H, Dv);
    if (path == GDN_PATH_SIMT) return gdn::cw_workspace_bytes(B, T, H, Dk, chunk);
    return 0;
}

gdn_status_t gdn_chunk_fwd_cw(const void *q, const void *k, const void *v,
                              const float *log_alpha, const float *b, const float *w,
                              const float *S0, void *o, float *S_T, int B, int T, int H, int Dk,
                              int Dv, int chunk, gdn_dtype_t dtype, void *workspace,
                              size_t workspace_bytes, void *stream) {
    const gdn_status_t sz = check_sizes(B, T, H, Dk, Dv, chunk, dtype);
    if (sz != GDN_OK) return sz;
    if (!gdn::cw_supported(Dk, chunk)) return GDN_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t esz = dtype == GDN_BF16 ? 2 : 4;
    const size_t n_tok = (size_t)B * T * H;
    const size_t state_bytes = (size_t)B * H * Dv * Dk * sizeof(float);
    if (B == 0 || H == 0) return GDN_OK;
    if (T == 0) {  // no tokens: the final state is the initial one
        if (!S_T) return GDN_OK;
        if (!aligned16(S_T) || (S0 && !aligned16(S0))) return GDN_ERR_INVALID_ARG;
        if (S0 && S0 != S_T && overlaps(S_T, state_bytes, S0, state_bytes))
            return GDN_ERR_INVALID_ARG;
        cudaError_t e = S0 ? (S0 == S_T ? cudaSuccess
                                        : cudaMemcpyAsync(S_T, S0, state_bytes,
                                                          cudaMemcpyDeviceToDevice, st))
                           : cudaMemsetAsync(S_T, 0, state_bytes, st);
        return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
    }
    if (!q || !k || !v || !log_alpha || !b || !w || !o) return GDN_ERR_INVALID_ARG;
    const struct { const void *p; size_t n; } in[] = {
        {q, n_tok * Dk * esz}, {k, n_tok * Dk * esz}, {v, n_tok * Dv * esz},
        {log_alpha, n_tok * Dk * sizeof(float)}, {b, n_tok * Dk * sizeof(float)},
        {w, n_tok * Dv * sizeof(float)}, {S0, state_bytes}};
    for (const auto &a : in)
        if (a.p && !aligned16(a.p)) return GDN_ERR_INVALID_ARG;
    if (!aligned16(o) || (S_T && !aligned16(S_T)) || (workspace && !aligned16(workspace)))
        return GDN_ERR_INVALID_ARG;
    const size_t o_bytes = n_tok * Dv * esz;
    for (const auto &a : in) {
        if (overlaps(o, o_bytes, a.p, a.n)) return GDN_ERR_INVALID_ARG;
        // S_T may be S0 itself (in-place continuation), nothing else
        if (S_T && a.p != S0 && overlaps(S_T, state_bytes, a.p, a.n)) return GDN_ERR_INVALID_ARG;
    }
    if (S_T && S0 && S_T != S0 && overlaps(S_T, state_bytes, S0, state_bytes))
        return GDN_ERR_INVALID_ARG;
    if (S_T && overlaps(S_T, state_bytes, o, o_bytes)) return GDN_ERR_INVALID_ARG;
    const size_t need = gdn_chunk_fwd_cw_workspace_size(B, T, H, Dk, Dv, chunk, dtype);
    if (!workspace || workspace_bytes < need) return GDN_ERR_INVALID_ARG;
    for (const auto &a : in)
        if (overlaps(workspace, need, a.p, a.n)) return GDN_ERR_INVALID_ARG;
    if (overlaps(workspace, need, o, o_bytes) ||
        (S_T && overlaps(workspace, need, S_T, state_bytes)))
        return GDN_ERR_INVALID_ARG;
    const bool tc = gdn::cw_tc_supported(B, T, H, Dk, Dv, chunk, dtype == GDN_BF16);
    const cudaError_t e =
        tc ? gdn::launch_chunk_cw_tc(q, k, v, log_alpha, b, w, S0, o, S_T, B, T, H, Dv, workspace,
                                     st)
           : gdn::launch_chunk_cw(q, k, v, log_alpha, b, w, S0, o, S_T, B, T, H, Dk, Dv, chunk,
                                  dtype == GDN_BF16, workspace, st);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status_t gdn_decode_step_cw(const void *q, const void *k, const void *v,
                                const float *log_alpha, const float *b, const float *w, float *S,
                                void *o, int B, int H, int Dk, int Dv, gdn_dtype_t dtype,
                                void *stream) {
    const gdn_status_t sz = check_sizes(B, 1, H, Dk, Dv, 16, dtype);
    if (sz != GDN_OK) return sz;
    if (B == 0 || H == 0) return GDN_OK;
    if (!q || !k || !v || !log_alpha || !b || !w || !S || !o) return GDN_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, log_alpha, b, w, S, o};
    for (const void *p : ptrs)
        if (!aligned16(p)) return GDN_ERR_INVALID_ARG;
    const size_t esz = dtype == GDN_BF16 ? 2 : 4, heads = (size_t)B * H;
    const size_t s_bytes = heads * Dv * Dk * sizeof(float), o_bytes = heads * Dv * esz;
    const struct { const void *p; size_t n; } in[] = {
        {q, heads * Dk * esz}, {k, heads * Dk * esz}, {v, heads * Dv * esz},
        {log_alpha, heads * Dk * sizeof(float)}, {b, heads * Dk * sizeof(float)},
        {w, heads * Dv * sizeof(float)}};
    for (const auto &a : in)
        if (overlaps(o, o_bytes, a.p, a.n) || overlaps(S, s_bytes, a.p, a.n))
            return GDN_ERR_INVALID_ARG;
    if (overlaps(o, o_bytes, S, s_bytes)) return GDN_ERR_INVALID_ARG;
    const cudaError_t e = gdn::launch_decode_cw(q, k, v, log_alpha, b, w, S, o, B, H, Dk, Dv,
                                                dtype == GDN_BF16,
                                                static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status_t gdn_debug_withhold_first_arrival(int enable) {
    return gdn::set_withhold_first_arrival(enable != 0) == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status_t gdn_check_device_status(void) {
    if (cudaDeviceSynchronize() != cudaSuccess) return GDN_ERR_CUDA;
    unsigned int flag = 0, flag_wide = 0, flag_bwd = 0;
    if (gdn::read_and_clear_device_error(&flag) != cudaSuccess ||
        gdn::read_and_clear_device_error_wide(&flag_wide) != cudaSuccess ||
        gdn::read_and_clear_device_error_bwd(&flag_bwd) != cudaSuccess)
        return GDN_ERR_CUDA;
    return (flag | flag_wide | flag_bwd) ? GDN_ERR_CUDA : GDN_OK;
}

gdn_status_t gdn_decode_step(const void *q, const void *k, const void *v, const float *log_alpha,
                             const float *beta, float *S, void *o, int B, int H, int Dk, int Dv,
                             gdn_dtype_t dtype, void *stream) {
    return gdn_decode_step_ex(q, k, v, log_alpha, beta, S, o, B, H, Dk, Dv, dtype, 0u, stream);
}

gdn_status_t gdn_decode_step_ex(const void *q, const void *k, const void *v,
                                const float *log_alpha, const float *beta, float *S, void *o,
                                int B, int H, int Dk, int Dv, gdn_dtype_t dtype, unsigned flags,
                                void *stream) {
    if (B < 0 || H < 0 || Dk <= 0 || Dv <= 0) return GDN_ERR_INVALID_ARG;
    if (flags & ~kKnownFlags) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (Dk > kMaxDk || Dv > kMaxDv) return GDN_ERR_UNSUPPORTED;
    if (B == 0 || H == 0) return GDN_OK;
    if (!q || !k || !v || !log_alpha || !beta || !S || !o) return GDN_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, log_alpha, beta, S, o};
    for (const void *p : ptrs)
        if (!aligned16(p)) return GDN_ERR_INVALID_ARG;
    const size_t esz = dtype == GDN_BF16 ? 2 : 4;
    const size_t heads = (size_t)B * H;
    if (overlaps(o, heads * Dv * esz, S, heads * Dv * Dk * sizeof(float)))
        return GDN_ERR_INVALID_ARG;
    const cudaError_t e = gdn::launch_decode(q, k, v, log_alpha, beta, S, o, B, H, Dk, Dv,
                                             dtype == GDN_BF16, flags,
                                             static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // extern "C"
