"""Host-side index logic of the CUDA path, compiled with g++ and run on the CPU:
the context-split ranges partition [0, L) at multiples of the 32-token unit,
the prefetch ranges cover them for every length up to the capacity, the
CTA coordinates of a split grid (with head sub-groups) cover every query head
of every batch exactly once per split, and the tensor-core QKV projection's
split of the hidden dimension stays within its cluster, its shared memory and
its staged x region."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "long_context_decoding_saga_b200", "csrc")

PROGRAM = r"""
#define __host__
#define __device__
#include <cstdio>
#include <vector>
struct Dim3 { unsigned x, y, z; };
static Dim3 blockIdx;  // stand-in for the CUDA built-in: the test sets it per CTA
static unsigned atomicOr(unsigned* a, unsigned v) { unsigned o = *a; *a |= v; return o; }
#include "saga_internal.h"
using namespace saga;

static int fails = 0;
#define CHECK(c, ...) do { if (!(c)) { ++fails; if (fails < 20) { std::printf(__VA_ARGS__); std::printf("\n"); } } } while (0)

int main() {
  const int Ps[] = {1, 31, 32, 33, 1000, 4097, 32769, 131073, 131104};
  const int Ss[] = {1, 2, 7, 37, 136, 148, 296};
  for (int P : Ps) for (int S : Ss) {
    const int l_cap = P + 200;
    const int Ls[] = {P, P + 1, P + 5, P + 100, P + 200, P > 10 ? P - 10 : 1};
    for (int L : Ls) {
      int prev_end = 0;
      for (int s = 0; s < S; ++s) {
        int st, en, cst, cen;
        split_range(P, S, s, L, &st, &en);
        split_cap_range(P, S, s, l_cap, &cst, &cen);
        CHECK(st == prev_end, "P=%d S=%d L=%d s=%d: start %d != previous end %d", P, S, L, s, st, prev_end);
        CHECK(st <= en, "P=%d S=%d L=%d s=%d: start %d > end %d", P, S, L, s, st, en);
        CHECK(st == L || st % kUnit == 0, "P=%d S=%d L=%d s=%d: start %d not on the unit", P, S, L, s, st);
        CHECK(st == en || (st >= cst && en <= cen), "P=%d S=%d L=%d s=%d: [%d,%d) outside the prefetch range [%d,%d)",
              P, S, L, s, st, en, cst, cen);
        prev_end = en;
      }
      CHECK(prev_end == L, "P=%d S=%d L=%d: splits end at %d", P, S, L, prev_end);
    }
  }
  // CTA coordinates: grid (S * hsplit, h_k, B), G query heads per CTA
  const int hsplits[] = {1, 2, 4};
  for (int hsplit : hsplits) {
    const int S = 3, h_k = 2, B = 2, G = 8, h_q = h_k * hsplit * G;
    SplitParams p{};
    p.hsplit = hsplit;
    p.G = G;
    std::vector<int> seen((size_t)S * B * h_q, 0);
    for (unsigned z = 0; z < (unsigned)B; ++z)
      for (unsigned y = 0; y < (unsigned)h_k; ++y)
        for (unsigned x = 0; x < (unsigned)(S * hsplit); ++x) {
          blockIdx = {x, y, z};
          const CtaCoord c = cta_coord(p);
          CHECK(c.s >= 0 && c.s < S && c.h == (int)y && c.b == (int)z, "coord out of range");
          for (int j = c.j0; j < c.j0 + G; ++j) {
            CHECK(j >= 0 && j < h_q, "head %d out of range", j);
            CHECK(j * h_k / h_q == c.h, "head %d is not in key head %d's group", j, c.h);
            if (j >= 0 && j < h_q) seen[((size_t)c.s * B + c.b) * h_q + j] += 1;
          }
        }
    for (size_t i = 0; i < seen.size(); ++i) CHECK(seen[i] == 1, "hsplit %d: (split, batch, head) %zu seen %d times", hsplit, i, seen[i]);
  }
  // tensor-core QKV projection plan: splits in [1, 8] and <= the k-blocks, every
  // split non-empty and within the staged x region, shared memory within a CTA's
  const int ncols[] = {1, 64, 127, 128, 129, 448, 1088, 2176, 2688, 18944, 40000};
  const int hiddens[] = {8, 64, 72, 1000, 1536, 2048, 2056, 4096, 4104, 8192, 16384};
  const int smss[] = {1, 132, 148};
  for (int nc : ncols) for (int hd : hiddens) for (int sms : smss) {
    int mt, sp, kbt, st, kbm;
    qkv_mma_plan(nc, hd, sms, &mt, &sp, &kbt, &st, &kbm);
    CHECK(mt * kQkvTileM >= nc && (mt - 1) * kQkvTileM < nc, "qkv n=%d: %d tiles", nc, mt);
    CHECK(sp >= 1 && sp <= kQkvMaxSplits && sp <= kbt, "qkv n=%d D=%d: %d splits of %d k-blocks", nc, hd, sp, kbt);
    CHECK(kbm <= kQkvMaxKb && st >= 1 && st <= kQkvMaxStages && st <= kbm, "qkv D=%d: kbs_max %d stages %d", hd, kbm, st);
    CHECK(qkv_mma_smem_bytes(st, kbm) <= 232448, "qkv D=%d: %d bytes of shared memory", hd, qkv_mma_smem_bytes(st, kbm));
    for (int s = 0; s < sp; ++s) {
      const int kb0 = (int)((long long)s * kbt / sp), nkb = (int)((long long)(s + 1) * kbt / sp) - kb0;
      CHECK(nkb >= 1 && nkb <= kbm, "qkv D=%d split %d: %d k-blocks (max %d)", hd, s, nkb, kbm);
    }
  }
  std::printf(fails ? "FAIL %d\n" : "ok\n", fails);
  return fails ? 1 : 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_split_ranges_and_cta_coords(tmp_path):
    src = tmp_path / "host_ranges.cpp"
    src.write_text(PROGRAM)
    exe = tmp_path / "host_ranges"
    build = subprocess.run(["g++", "-std=c++17", "-O1", "-I", os.path.join(ROOT, "include"), "-I", CSRC,
                            str(src), "-o", str(exe)], capture_output=True, text=True)
    assert build.returncode == 0, build.stderr[-2000:]
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0 and run.stdout.strip().endswith("ok"), run.stdout[-2000:]
