"""The workspace layout (host code, CPU only): the shared expert's calls reuse the layer's
workspace with the layout of their own shape (one group of all T tokens, E = 1, k = 1), so
every region that layout places must end before the layer layout's group-offsets slot, and
the layout must grow with T.  Compiled from the library's own layout code with nvcc."""
import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r'''
#include <cstdio>
#include "common.cuh"
using namespace moe;
int main() {
  int bad = 0, n = 0;
  const long long Ts[] = {1, 7, 128, 1000, 8192, 16384, 65536};
  const int ds[] = {128, 2048, 4096}, Es[] = {1, 2, 8, 64, 128, 256}, ks[] = {1, 2, 4, 8}, fs[] = {128, 1024};
  for (long long T : Ts) for (int d : ds) for (int E : Es) for (int k : ks) for (int f : fs)
    for (int prec = 0; prec < 2; ++prec) for (int dt = 0; dt < 2; ++dt) {
      if (k > E || (prec == MOE_PREC_MXFP8 && dt == MOE_F32)) continue;
      Shape s; s.T = T; s.d = d; s.E = E; s.k = k; s.f = f; s.dtype = dt == 0 ? MOE_BF16 : MOE_F32; s.prec = prec;
      Shape t = s; t.E = 1; t.k = 1;
      const WsLayout L = ws_layout(s), M = ws_layout(t);
      ++n;
      // the shared expert's calls touch its layout's regions, all below its own slot
      if (M.group_offsets > L.group_offsets) { ++bad; printf("overlap T=%lld d=%d E=%d k=%d f=%d prec=%d\n", T, d, E, k, f, prec); }
      if (L.group_offsets + 8 > L.total) { ++bad; printf("slot T=%lld\n", T); }
      Shape u = s; u.T = T + 1;
      if (ws_layout(u).total < L.total) { ++bad; printf("shrinks T=%lld\n", T); }
    }
  printf("%d shapes, %d bad\n", n, bad);
  return bad != 0;
}
'''


@pytest.mark.skipif(shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"),
                    reason="needs nvcc")
def test_shared_expert_layout_stays_below_the_group_offsets():
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    csrc = os.path.join(ROOT, "routing_grouped_expert_softmax_b200", "csrc")
    with tempfile.TemporaryDirectory() as tmp:
        src = os.path.join(tmp, "layout.cu")
        exe = os.path.join(tmp, "layout")
        with open(src, "w") as fh:
            fh.write(PROGRAM)
        r = subprocess.run([nvcc, "-std=c++17", "-I", csrc, "-I", os.path.join(ROOT, "include"), src, "-o", exe],
                           capture_output=True, text=True)
        assert r.returncode == 0, r.stderr
        r = subprocess.run([exe], capture_output=True, text=True)
        assert r.returncode == 0, r.stdout
        assert " 0 bad" in r.stdout
