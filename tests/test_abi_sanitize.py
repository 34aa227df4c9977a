"""The C-ABI layer's host code (argument checks, offsets, overlap and size
arithmetic in csrc/gdn_api.cu) under AddressSanitizer and
UndefinedBehaviorSanitizer.  The file is compiled as host C++ with g++ against
stand-ins for the kernel launchers and for the few CUDA runtime calls it makes
(which record the call and succeed), and a harness drives every entry point
with adversarial arguments: negative, zero and extreme sizes, null, misaligned
and overlapping pointers, bad and extreme packed-sequence offsets.  CPU only;
skipped where the compiler has no sanitizer runtime or the CUDA headers are
missing.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "gated_delta_rule_130_b200", "csrc")
CUDA_INC = "/usr/local/cuda/include"

STUBS = r"""
#include <cuda_runtime.h>
#include <stddef.h>
#include "kernels.h"

int g_runtime_calls = 0;
extern "C" {
cudaError_t cudaMemcpyAsync(void *, const void *, size_t, cudaMemcpyKind, cudaStream_t) {
    ++g_runtime_calls; return cudaSuccess; }
cudaError_t cudaMemsetAsync(void *, int, size_t, cudaStream_t) { ++g_runtime_calls; return cudaSuccess; }
cudaError_t cudaDeviceSynchronize(void) { ++g_runtime_calls; return cudaSuccess; }
}
namespace gdn {
static cudaError_t ok() { return cudaSuccess; }
cudaError_t launch_decode(const void *, const void *, const void *, const float *, const float *,
                          float *, void *, int, int, int, int, bool, unsigned, cudaStream_t) { return ok(); }
size_t prologue_bytes(int B, int T, int H, int Dk, bool bf16, unsigned flags) {
    return flags ? (size_t)B * T * H * (2 * Dk * (bf16 ? 2 : 4) + 8) : 0; }
cudaError_t launch_prologue(const void *q, const void *k, const float *la, const float *be, int,
                            int, int, int, bool, unsigned, void *, Prepared *out, cudaStream_t) {
    out->q = q; out->k = k; out->log_alpha = la; out->beta = be; return ok(); }
size_t simt_workspace_bytes(int B, int T, int H, int C) {
    return (size_t)B * H * (((size_t)T + C - 1) / C) * (2 * (size_t)C * C + C) * 4; }
cudaError_t launch_chunk_simt(const void *, const void *, const void *, const float *, const float *,
                              const float *, void *, float *, int, int, int, int, int, int, bool,
                              void *, cudaStream_t) { return ok(); }
bool tc_supported(int, int, int, int, int, int, bool) { return false; }
bool tc_precomputed(int, int, int Dk, int) { return Dk == 256; }
size_t tc_workspace_bytes(int B, int T, int H, unsigned, int Dk, int) {
    return (size_t)B * H * (((size_t)T + 63) / 64) * (Dk == 256 ? 49152 : 16384); }
size_t tc_workspace_bytes_fused(int B, int T, int H, unsigned) {
    return (size_t)B * H * (((size_t)T + 63) / 64) * 16384; }
cudaError_t launch_chunk_tc(const void *, const void *, const void *, const float *, const float *,
                            const float *, void *, float *, int, int, int, int, int, unsigned,
                            void *, cudaStream_t, float *) { return ok(); }
size_t tc_workspace_bytes_seqs(int n, long long chunks, int H, bool, unsigned, int Dk, int) {
    return ((size_t)n + 1) * 8 + (size_t)chunks * H * (Dk == 256 ? 49152 : 16384); }
cudaError_t launch_chunk_tc_seqs(const void *, const void *, const void *, const float *,
                                 const float *, const float *, void *, float *, int, int, long long,
                                 const int *, long long, int, int, int, unsigned, void *,
                                 cudaStream_t, float *) { return ok(); }
cudaError_t launch_bwd_recompute(const void *, const void *, const void *, const float *,
                                 const float *, const float *, int, int, int, int, int, int, bool,
                                 float *, float *, cudaStream_t) { return ok(); }
bool bwd_supported(int Dk, int chunk) { return Dk <= 128 && (chunk == 16 || chunk == 32 || chunk == 64); }
size_t bwd_workspace_bytes(int B, int T, int H, int Dk, int Dv, int C, bool) {
    return (size_t)B * H * (((size_t)T + C - 1) / C) * (2 * (size_t)C * C + C + 2 * (size_t)Dv * Dk) * 4; }
cudaError_t launch_chunk_bwd(const void *, const void *, const void *, const float *, const float *,
                             const float *, const void *, const float *, void *, void *, void *,
                             float *, float *, float *, int, int, int, int, int, int, bool, void *,
                             cudaStream_t) { return ok(); }
bool cw_tc_supported(int, int, int, int, int, int, bool) { return false; }
size_t cw_tc_workspace_bytes(int, int, int, int) { return 0; }
cudaError_t launch_chunk_cw_tc(const void *, const void *, const void *, const float *,
                               const float *, const float *, const float *, void *, float *, int,
                               int, int, int, void *, cudaStream_t) { return ok(); }
bool cw_supported(int Dk, int chunk) { return Dk <= 128 && (chunk == 16 || chunk == 32 || chunk == 64); }
size_t cw_workspace_bytes(int B, int T, int H, int Dk, int C) {
    return (size_t)B * H * (((size_t)T + C - 1) / C) * (2 * (size_t)C * C + (size_t)C * Dk) * 4; }
cudaError_t launch_chunk_cw(const void *, const void *, const void *, const float *, const float *,
                            const float *, const float *, void *, float *, int, int, int, int, int,
                            int, bool, void *, cudaStream_t) { return ok(); }
cudaError_t launch_decode_cw(const void *, const void *, const void *, const float *, const float *,
                             const float *, float *, void *, int, int, int, int, bool,
                             cudaStream_t) { return ok(); }
cudaError_t read_and_clear_device_error(unsigned int *flag) { *flag = 0; return ok(); }
cudaError_t read_and_clear_device_error_wide(unsigned int *flag) { *flag = 0; return ok(); }
cudaError_t read_and_clear_device_error_bwd(unsigned int *flag) { *flag = 0; return ok(); }
bool bwd_tc_supported(int, int, int, int, int, int, bool) { return false; }
int tcw_split_segments(int, int, int, int, int) { return 1; }
cudaError_t set_withhold_first_arrival(bool) { return ok(); }
}  // namespace gdn
"""

HARNESS = r"""
#include <climits>
#include <cstdint>
#include <cstdio>
#include <vector>
#include "gdn.h"

extern int g_runtime_calls;
#define P(x) reinterpret_cast<void *>(uintptr_t(x))
#define F(x) reinterpret_cast<float *>(uintptr_t(x))
static int fails = 0;
static void expect(int got, int want, const char *what) {
    if (got != want) { std::printf("FAIL %s: got %d want %d\n", what, got, want); ++fails; }
}

int main() {
    const uintptr_t A = 1ull << 32, Bb = 1ull << 36, Cc = 1ull << 40, WS = 1ull << 44;
    const int sizes[][5] = {{1, 8, 1, 16, 16}, {0, 8, 1, 16, 16}, {1, 0, 1, 16, 16},
                            {-1, 8, 1, 16, 16}, {1, -8, 1, 16, 16}, {1, 8, -1, 16, 16},
                            {1, 8, 1, 0, 16}, {1, 8, 1, 300, 16}, {1, 8, 1, 16, 600},
                            {65535, INT_MAX, 65535, 256, 512}, {1, INT_MAX, 1, 128, 128},
                            {65536, 8, 1, 16, 16}, {1, 8, 65536, 16, 16}};
    for (auto &z : sizes) {
        for (int chunk : {16, 48, 64}) {
            for (int dt : {0, 1, 7}) {
                gdn_chunk_fwd_workspace_size_ex(z[0], z[1], z[2], z[3], z[4], chunk, (gdn_dtype_t)dt, 3u);
                gdn_chunk_fwd_path(z[0], z[1], z[2], z[3], z[4], chunk, (gdn_dtype_t)dt);
                gdn_chunk_fwd_ex(P(A), P(A + 1024), P(A + 4096), F(Bb), F(Bb + 256), nullptr, P(Cc),
                                 nullptr, z[0], z[1], z[2], z[3], z[4], chunk, (gdn_dtype_t)dt, 3u,
                                 P(WS), 1ull << 30, nullptr);
                gdn_chunk_bwd(P(A), P(A + 1024), P(A + 4096), F(Bb), F(Bb + 256), nullptr, P(Bb + 4096),
                              nullptr, P(Cc), P(Cc + (1ull << 34)), P(Cc + (2ull << 34)),
                              F(Cc + (3ull << 34)), F(Cc + (4ull << 34)), nullptr, z[0], z[1], z[2],
                              z[3], z[4], chunk, (gdn_dtype_t)dt, P(WS), 1ull << 30, nullptr);
                gdn_chunk_fwd_cw(P(A), P(A + 1024), P(A + 4096), F(Bb), F(Bb + 256), F(Bb + 512),
                                 nullptr, P(Cc), nullptr, z[0], z[1], z[2], z[3], z[4], chunk,
                                 (gdn_dtype_t)dt, P(WS), 1ull << 30, nullptr);
                gdn_decode_step_ex(P(A), P(A + 1024), P(A + 4096), F(Bb), F(Bb + 256), F(Cc),
                                   P(WS), z[0], z[2], z[3], z[4], (gdn_dtype_t)dt, 3u, nullptr);
            }
        }
    }
    // packed-sequence offsets: bad, empty, extreme
    std::vector<std::vector<int>> offs = {{0}, {0, 0, 0}, {1, 2}, {0, 5, 3}, {0, -1},
                                          {0, INT_MAX}, {0, INT_MAX - 1, INT_MAX},
                                          {0, 3, 3, 70, 71}};
    for (auto &cu : offs) {
        const int N = (int)cu.size() - 1;
        for (int H : {1, 65535, 65536}) {
            gdn_chunk_fwd_varlen_workspace_size(cu.data(), N, H, 16, 16, 16, GDN_F32, 0u);
            gdn_chunk_fwd_varlen(P(A), P(A + 1024), P(A + 4096), F(Bb), F(Bb + 256), nullptr, P(Cc),
                                 nullptr, reinterpret_cast<const int *>(P(Bb + 8192)), cu.data(), N,
                                 H, 16, 16, 16, GDN_F32, 0u, P(WS), 1ull << 30, nullptr);
        }
    }
    expect(gdn_chunk_fwd_varlen_workspace_size(nullptr, 2, 1, 16, 16, 16, GDN_F32, 0u), 0, "null offsets");
    const int bad[] = {0, 5, 3};
    expect(gdn_chunk_fwd_varlen(P(A), P(A), P(A), F(A), F(A), nullptr, P(Cc), nullptr, bad + 0, bad, 2,
                                1, 16, 16, 16, GDN_F32, 0u, P(WS), 1 << 30, nullptr), 1, "decreasing offsets");
    // empty problems reach the state copy (the runtime stand-ins), nothing else
    const int before = g_runtime_calls;
    expect(gdn_chunk_fwd(nullptr, nullptr, nullptr, nullptr, nullptr, F(A), nullptr, F(Bb), 2, 0, 3,
                         16, 16, 16, GDN_F32, nullptr, 0, nullptr), 0, "T = 0 copies S0");
    expect(gdn_chunk_bwd(nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                         nullptr, nullptr, nullptr, nullptr, nullptr, F(Bb), 2, 0, 3, 16, 16, 16,
                         GDN_F32, nullptr, 0, nullptr), 0, "T = 0 zeroes dS0");
    expect(g_runtime_calls - before, 2, "runtime calls for empty problems");
    expect(gdn_check_device_status(), 0, "device status");
    for (int s = -1; s < 6; ++s) gdn_status_string((gdn_status_t)s);
    if (fails) return 1;
    std::printf("sanitized ABI ok\n");
    return 0;
}
"""


def test_abi_layer_under_address_and_undefined_behaviour_sanitizers(tmp_path):
    cxx = shutil.which("g++")
    if cxx is None or not os.path.isdir(CUDA_INC):
        pytest.skip("no g++ or no CUDA headers")
    (tmp_path / "stubs.cpp").write_text(STUBS)
    (tmp_path / "harness.cpp").write_text(HARNESS)
    exe = tmp_path / "abi_harness"
    cmd = [cxx, "-std=c++17", "-O1", "-g", "-fno-omit-frame-pointer",
           "-fsanitize=address,undefined", "-fno-sanitize-recover=undefined",
           "-I", CUDA_INC, "-I", CSRC, "-I", os.path.join(ROOT, "include"),
           "-x", "c++", os.path.join(CSRC, "gdn_api.cu"),
           "-x", "c++", str(tmp_path / "stubs.cpp"), str(tmp_path / "harness.cpp"),
           "-o", str(exe)]
    build = subprocess.run(cmd, capture_output=True, text=True)
    if build.returncode != 0 and "sanitize" in build.stderr:
        pytest.skip("compiler without sanitizer runtime")
    assert build.returncode == 0, build.stderr[-3000:]
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120,
                         env=dict(os.environ, ASAN_OPTIONS="detect_leaks=1"))
    assert run.returncode == 0, (run.stdout + run.stderr)[-3000:]
    assert "sanitized ABI ok" in run.stdout
