"""The C oracle under AddressSanitizer and UndefinedBehaviorSanitizer (CPU).

Every parity test trusts the oracle's buffers, so it is built here with both
sanitizers and driven through all six entry points (double and long double;
causal, bidirectional and gate-logit modes) on ragged shapes, T = 0, a NULL
and an in-place state, on one and on three threads.  Any out-of-bounds
access, use after free or undefined arithmetic aborts the run.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

DRIVER = r"""
#include <stdio.h>
#include <stdlib.h>
int gdn_oracle_fwd(const float*, const float*, const float*, const float*, const float*, const double*, double*, double*, int, int, int, int, int, int);
int gdn_oracle_bidir(const float*, const float*, const float*, const float*, const float*, const double*, double*, double*, int, int, int, int, int, int);
int gdn_oracle_fwd_logits(const float*, const float*, const float*, const float*, const float*, const double*, double*, double*, int, int, int, int, int, int);
int gdn_oracle_bidir_logits(const float*, const float*, const float*, const float*, const float*, const double*, double*, double*, int, int, int, int, int, int);
int gdn_oracle_fwd_ld(const float*, const float*, const float*, const float*, const float*, const long double*, long double*, long double*, int, int, int, int, int, int);
int gdn_oracle_bidir_ld(const float*, const float*, const float*, const float*, const float*, const long double*, long double*, long double*, int, int, int, int, int, int);
static float* rnd(size_t n, float lo, float hi) {
  float* p = malloc(n * sizeof(float));
  for (size_t i = 0; i < n; ++i) p[i] = lo + (hi - lo) * (float)rand() / (float)RAND_MAX;
  return p;
}
int main(void) {
  const int shapes[][5] = {{1, 1, 1, 1, 1}, {2, 7, 3, 5, 4}, {1, 33, 2, 16, 8}, {3, 0, 2, 4, 4}, {2, 19, 1, 3, 7}};
  for (size_t s = 0; s < sizeof(shapes) / sizeof(shapes[0]); ++s) {
    const int B = shapes[s][0], T = shapes[s][1], H = shapes[s][2], Dk = shapes[s][3], Dv = shapes[s][4];
    const size_t rows = (size_t)B * T * H, sn = (size_t)B * H * Dk * Dv;
    float *q = rnd(rows * Dk + (rows == 0), -1, 1), *k = rnd(rows * Dk + (rows == 0), -1, 1);
    float *v = rnd(rows * Dv + (rows == 0), -1, 1), *g = rnd(rows + (rows == 0), -3, 0), *b = rnd(rows + (rows == 0), 0, 1);
    double *si = malloc(sn * sizeof(double)), *so = malloc(sn * sizeof(double)), *o = malloc((rows * Dv + 1) * sizeof(double));
    long double *sil = malloc(sn * sizeof(long double)), *sol = malloc(sn * sizeof(long double)), *ol = malloc((rows * Dv + 1) * sizeof(long double));
    for (size_t i = 0; i < sn; ++i) { si[i] = 0.01 * (double)i; sil[i] = si[i]; }
    for (int nt = 1; nt <= 3; nt += 2) {
      if (gdn_oracle_fwd(q, k, v, g, b, si, so, o, B, T, H, Dk, Dv, nt)) return 1;
      if (gdn_oracle_bidir(q, k, v, g, b, NULL, so, o, B, T, H, Dk, Dv, nt)) return 2;
      if (gdn_oracle_fwd_logits(q, k, v, g, b, si, NULL, o, B, T, H, Dk, Dv, nt)) return 3;
      if (gdn_oracle_bidir_logits(q, k, v, g, b, si, si, o, B, T, H, Dk, Dv, nt)) return 4;  /* in place */
      if (gdn_oracle_fwd_ld(q, k, v, g, b, sil, sol, ol, B, T, H, Dk, Dv, nt)) return 5;
      if (gdn_oracle_bidir_ld(q, k, v, g, b, NULL, NULL, ol, B, T, H, Dk, Dv, nt)) return 6;
    }
    free(q); free(k); free(v); free(g); free(b); free(si); free(so); free(o); free(sil); free(sol); free(ol);
  }
  puts("ok");
  return 0;
}
"""


def test_oracle_is_clean_under_asan_and_ubsan(tmp_path):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no gcc")
    (tmp_path / "driver.c").write_text(DRIVER)
    exe = tmp_path / "driver"
    cc = subprocess.run([gcc, "-std=c11", "-D_GNU_SOURCE", "-O1", "-g", "-fsanitize=address,undefined",
                         "-fno-omit-frame-pointer", "-fno-sanitize-recover=all",
                         str(tmp_path / "driver.c"), os.path.join(ROOT, "oracle", "gdn_oracle.c"),
                         os.path.join(ROOT, "oracle", "gdn_oracle_ld.c"), "-lm", "-lpthread",
                         "-o", str(exe)], capture_output=True, text=True)
    if cc.returncode != 0 and "asan" in (cc.stderr + cc.stdout).lower():
        pytest.skip("no sanitizer runtime: " + cc.stderr[-200:])
    assert cc.returncode == 0, cc.stderr
    env = dict(os.environ, ASAN_OPTIONS="detect_leaks=1:abort_on_error=0")
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300, env=env)
    assert run.returncode == 0 and run.stdout.strip() == "ok", run.stdout + run.stderr[-3000:]
