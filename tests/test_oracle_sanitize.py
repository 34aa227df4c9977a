"""The oracle's C source under AddressSanitizer and UndefinedBehaviorSanitizer:
a small harness compiled with it calls every entry point on exactly-sized heap
buffers (so any read or write past an array is reported), over sequences that
cross the backward's checkpoint blocks, with and without initial states and
unit lists, and with rejected arguments.  CPU only; skipped where the compiler
has no sanitizer runtime.
"""
import os
import shutil
import subprocess

import pytest

from oracle import oracle as O

HARNESS = r"""
#include <stdio.h>
#include <stdlib.h>

int gdn_oracle_forward(const double *, const double *, const double *, const double *,
                       const double *, const double *, double *, double *, long, long, long,
                       long, long, const int *, int, int);
int gdn_oracle_decode(const double *, const double *, const double *, const double *,
                      const double *, double *, double *, long, long, long, long, long,
                      const int *, int, int);
int gdn_oracle_backward(const double *, const double *, const double *, const double *,
                        const double *, const double *, const double *, const double *,
                        double *, double *, double *, double *, double *, double *,
                        long, long, long, long, long, const int *, int, int);
int gdn_oracle_forward_cw(const double *, const double *, const double *, const double *,
                          const double *, const double *, const double *, double *, double *,
                          long, long, long, long, long, const int *, int, int);

static double *arr(long n, unsigned *seed, double lo, double hi) {
    double *p = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    for (long i = 0; i < n; ++i) {
        *seed = *seed * 1664525u + 1013904223u;
        p[i] = lo + (hi - lo) * (double)(*seed >> 8) / 16777216.0;
    }
    return p;
}

int main(void) {
    unsigned s = 12345u;
    const long B = 2, T = 70, H = 3, Dk = 5, Dv = 4;
    const long nqk = B * T * H * Dk, nv = B * T * H * Dv, ng = B * T * H, ns = B * H * Dv * Dk;
    double *q = arr(nqk, &s, -1, 1), *k = arr(nqk, &s, -0.5, 0.5), *v = arr(nv, &s, -1, 1);
    double *la = arr(ng, &s, -1, 0), *be = arr(ng, &s, 0, 1), *S0 = arr(ns, &s, -0.1, 0.1);
    double *o = arr(nv, &s, 0, 0), *ST = arr(ns, &s, 0, 0), *d_o = arr(nv, &s, -1, 1);
    double *dST = arr(ns, &s, -1, 1);
    double *dq = arr(nqk, &s, 0, 0), *dk = arr(nqk, &s, 0, 0), *dv = arr(nv, &s, 0, 0);
    double *dla = arr(ng, &s, 0, 0), *dbe = arr(ng, &s, 0, 0), *dS0 = arr(ns, &s, 0, 0);
    double *lac = arr(nqk, &s, -1, 0), *bc = arr(nqk, &s, 0, 1), *wc = arr(nv, &s, 0, 1);
    int units[2] = {1, 5};
    int bad[1] = {6};
    int rc = 0;
    rc |= gdn_oracle_forward(q, k, v, la, be, S0, o, ST, B, T, H, Dk, Dv, NULL, 0, 3);
    rc |= gdn_oracle_forward(q, k, v, la, be, NULL, o, ST, B, T, H, Dk, Dv, units, 2, 2);
    rc |= gdn_oracle_forward(q, k, v, la, be, S0, o, ST, B, 0, H, Dk, Dv, NULL, 0, 1);
    rc |= gdn_oracle_backward(q, k, v, la, be, S0, d_o, dST, dq, dk, dv, dla, dbe, dS0,
                              B, T, H, Dk, Dv, NULL, 0, 4);
    rc |= gdn_oracle_backward(q, k, v, la, be, NULL, d_o, NULL, dq, dk, dv, dla, dbe, dS0,
                              B, T, H, Dk, Dv, units, 2, 1);
    rc |= gdn_oracle_forward_cw(q, k, v, lac, bc, wc, S0, o, ST, B, T, H, Dk, Dv, NULL, 0, 3);
    rc |= gdn_oracle_forward_cw(q, k, v, lac, bc, wc, NULL, o, ST, B, T, H, Dk, Dv, units, 2, 1);
    /* decode: T steps of [B,H,*] tokens read from the same buffers */
    rc |= gdn_oracle_decode(q, k, v, la, be, ST, o, T, B, H, Dk, Dv, NULL, 0, 2);
    if (rc != 0) { fprintf(stderr, "a valid call failed\n"); return 2; }
    if (gdn_oracle_forward(q, k, v, la, be, S0, o, ST, B, T, H, Dk, Dv, bad, 1, 1) != -1 ||
        gdn_oracle_backward(q, k, v, la, be, S0, NULL, dST, dq, dk, dv, dla, dbe, dS0,
                            B, T, H, Dk, Dv, NULL, 0, 1) != -1 ||
        gdn_oracle_forward_cw(q, k, v, lac, NULL, wc, S0, o, ST, B, T, H, Dk, Dv, NULL, 0, 1) != -1) {
        fprintf(stderr, "a bad argument was accepted\n");
        return 3;
    }
    free(q); free(k); free(v); free(la); free(be); free(S0); free(o); free(ST); free(d_o);
    free(dST); free(dq); free(dk); free(dv); free(dla); free(dbe); free(dS0); free(lac);
    free(bc); free(wc);
    printf("sanitized oracle ok\n");
    return 0;
}
"""


def test_oracle_under_address_and_undefined_behaviour_sanitizers(tmp_path):
    cc = shutil.which("gcc")
    if cc is None:
        pytest.skip("no gcc")
    src = tmp_path / "harness.c"
    src.write_text(HARNESS)
    exe = tmp_path / "harness"
    cmd = [cc, "-O1", "-g", "-fno-omit-frame-pointer", "-fsanitize=address,undefined",
           "-fno-sanitize-recover=undefined", "-pthread", str(src), O.SOURCE, "-o", str(exe), "-lm"]
    build = subprocess.run(cmd, capture_output=True, text=True)
    if build.returncode != 0 and "sanitize" in build.stderr:
        pytest.skip("compiler without sanitizer runtime: " + build.stderr.splitlines()[0])
    assert build.returncode == 0, build.stderr
    env = dict(os.environ, ASAN_OPTIONS="detect_leaks=1:abort_on_error=0",
               UBSAN_OPTIONS="print_stacktrace=1")
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120, env=env)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "sanitized oracle ok" in run.stdout
