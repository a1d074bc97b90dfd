"""Host logic of the stream-K partition used by the tensor-core contractions
(csrc/umma_layout.cuh): compiled host-only with nvcc and checked on the CPU
for many shapes and CTA counts."""
import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "expanded_rank_matrix_b200", "csrc")

PROGRAM = r'''
#include <cstdio>
#include <vector>
#include "umma_layout.cuh"
using namespace externd::umma;
// For T tiles, C chunks and G CTAs: every unit owned by exactly one CTA, CTA
// ranges contiguous and ordered, a tile's segments owned by consecutive CTAs
// starting at sk_first with sk_nseg of them, slots in [0, nseg).
static int check(int T, int C, int G) {
  const long long U = (long long)T * C;
  if (G < 1 || G > U) return 0;
  long long prev_end = 0;
  for (int b = 0; b < G; ++b) {
    const long long u0 = sk_u0(b, U, G), u1 = sk_u0(b + 1, U, G);
    if (u0 != prev_end || u1 <= u0) { printf("range %d %d %d b=%d\n", T, C, G, b); return 1; }
    prev_end = u1;
    for (long long u = u0; u < u1; ++u)
      if (sk_owner(u, U, G) != b) { printf("owner %d %d %d u=%lld\n", T, C, G, u); return 1; }
  }
  if (prev_end != U) { printf("cover %d %d %d\n", T, C, G); return 1; }
  for (int t = 0; t < T; ++t) {
    const int f = sk_first(t, C, U, G), ns = sk_nseg(t, C, U, G);
    if (f != sk_owner((long long)t * C, U, G) || ns < 1) { printf("first %d %d %d t=%d\n", T, C, G, t); return 1; }
    for (int b = f; b < f + ns; ++b) {  // each segment CTA holds part of tile t
      const long long u0 = sk_u0(b, U, G), u1 = sk_u0(b + 1, U, G);
      if (u1 <= (long long)t * C || u0 >= (long long)(t + 1) * C) { printf("seg %d %d %d t=%d\n", T, C, G, t); return 1; }
    }
    if (f + ns < G) {  // the next CTA starts in a later tile
      if (sk_u0(f + ns, U, G) < (long long)(t + 1) * C) { printf("next %d %d %d t=%d\n", T, C, G, t); return 1; }
    }
  }
  return 0;
}
int main() {
  int bad = 0, cases = 0;
  const int Ts[] = {1, 2, 7, 8, 20, 76, 77, 300};
  const int Cs[] = {1, 2, 5, 25, 32, 80, 81, 304};
  const int Gs[] = {1, 2, 3, 15, 105, 120, 147, 148, 1000};
  for (int T : Ts) for (int C : Cs) for (int G : Gs) { bad |= check(T, C, G); ++cases; }
  // the plan's CTA count keeps every tile within 16 segment slots and one SM free
  for (int T : Ts) for (int C : Cs) {
    const int G = sk_ctas(T, C, 148, 16);
    int S = 0;
    for (int t = 0; t < T; ++t) { const int ns = sk_nseg(t, C, (long long)T * C, G); S = ns > S ? ns : S; }
    if (S > 16 || G > 147 || G < 1 || G > T * C) { printf("plan %d %d G=%d S=%d\n", T, C, G, S); bad = 1; }
    bad |= check(T, C, G);
    ++cases;
  }
  printf("cases %d bad %d\n", cases, bad);
  return bad;
}
'''


@pytest.mark.skipif(shutil.which("nvcc") is None, reason="needs nvcc (host-only compile)")
def test_stream_k_partition_invariants():
    with tempfile.TemporaryDirectory() as tmp:
        src = os.path.join(tmp, "plan.cu")
        exe = os.path.join(tmp, "plan")
        open(src, "w").write(PROGRAM)
        subprocess.run(["nvcc", "-std=c++17", "-O1", "-I", CSRC, src, "-o", exe], check=True,
                       capture_output=True)
        r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
        assert r.returncode == 0, r.stdout + r.stderr
        assert "bad 0" in r.stdout
