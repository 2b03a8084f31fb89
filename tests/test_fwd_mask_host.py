"""The forward's key-tile range and masks on the host, against the definition.

The forward tile kernel (csrc/fwd_tc.cuh) visits key tiles [0, nkv) for its
query tile and masks scores to -inf inside them. This test cuts the nkv
expression and the masking block out of the source as they are, wraps them in
host functions for both key-tile sizes (128 rows at d = 64, 64 at d = 128),
and checks every (query tile, key tile, row, column) of many segment lengths,
with and without a sequence-parallel tile offset: a valid query row keeps
exactly the keys at or before it (causal) or every key of the segment
(non-causal), and nkv is exactly the number of key tiles those keys touch. No
GPU is touched."""
import os
import subprocess

import pytest

from tests.test_schedule_host import CSRC, _nvcc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _program() -> str:
    fwd = open(os.path.join(CSRC, "fwd_tc.cuh"), encoding="utf-8").read()
    i = fwd.index("  const int nkv = ")
    nkv = fwd[i:fwd.index(";", i) + 1]
    j = fwd.index("      if (p.causal) {\n        // key it * BN + c against query")
    mask = fwd[j:fwd.index("      // row max: four independent chains", j)]
    return r"""
#include <algorithm>
#include <cstdint>
#include <cstdio>
using std::min;
constexpr int BM = 128;
struct P { int causal; };
struct S { int n; };
struct W { int t; };

// key tiles of query tile wu.t (the kernel's expression)
template <int BN>
static int host_nkv(const P& p, const S& si, const W& wu, int kv_n, int tq, int qbase) {
""" + nkv + r"""
  return nkv;
}

// scores of key tile it for query row `row` after the kernel's masking
template <int BN>
static void host_mask(const P& p, int it, int tq, int qbase, int row, int nkv, int kv_n,
                      uint32_t* raw) {
""" + mask + r"""
}

static long long bad = 0, checks = 0;

template <int BN>
static void check(int causal, int si_n, int toff, int kv_n) {
  const P p{causal};
  const S si{si_n};
  for (int t = 0; t * BM < si_n; ++t) {
    const W wu{t};
    const int tq = t + toff, qbase = tq * BM;
    const int nkv = host_nkv<BN>(p, si, wu, kv_n, tq, qbase);
    const int rows = min(BM, si_n - t * BM);          // valid query rows of the tile
    const int last_q = qbase + rows - 1;               // key index of the last one
    const int want = causal ? last_q / BN + 1 : (kv_n + BN - 1) / BN;
    ++checks;
    if (nkv != want) {
      if (bad < 5) printf("BN=%d causal=%d n=%d toff=%d t=%d: nkv %d want %d\n", BN, causal,
                          si_n, toff, t, nkv, want);
      ++bad;
      continue;
    }
    for (int it = 0; it < nkv; ++it)
      for (int row = 0; row < rows; ++row) {
        uint32_t raw[BN];
        for (int c = 0; c < BN; ++c) raw[c] = 0x3f800000u;  // 1.0f
        host_mask<BN>(p, it, tq, qbase, row, nkv, kv_n, raw);
        for (int c = 0; c < BN; ++c) {
          ++checks;
          const int key = it * BN + c, query = qbase + row;
          const bool keep = causal ? key <= query : key < kv_n;
          if ((raw[c] == 0xff800000u) == keep || (keep && raw[c] != 0x3f800000u)) {
            if (bad < 5) printf("BN=%d causal=%d n=%d t=%d it=%d row=%d c=%d\n", BN, causal,
                                si_n, t, it, row, c);
            ++bad;
          }
        }
      }
  }
}

int main() {
  uint64_t s = 0x9E3779B97F4A7C15ull;
  auto next = [&]() { s ^= s << 13; s ^= s >> 7; s ^= s << 17; return s; };
  for (int causal = 0; causal < 2; ++causal) {
    for (int n = 1; n <= 700; n += (n < 300 ? 1 : 37)) {
      check<128>(causal, n, 0, n);
      check<64>(causal, n, 0, n);
    }
    // a sequence-parallel rank: its rows sit at tile toff of the gathered sequence
    for (int c = 0; c < 60; ++c) {
      const int ranks = 2 + (int)(next() % 3), rank_rows = 128 * (1 + (int)(next() % 3));
      const int g = (int)(next() % ranks);
      const int toff = g * (rank_rows / BM), kv_n = ranks * rank_rows;
      check<128>(causal, rank_rows, toff, kv_n);
      check<64>(causal, rank_rows, toff, kv_n);
    }
  }
  printf("checks %lld bad %lld\n", checks, bad);
  return bad != 0;
}
"""


@pytest.mark.skipif(_nvcc() is None, reason="nvcc not found")
def test_key_tiles_and_masks(tmp_path):
    src = tmp_path / "mask.cu"
    src.write_text(_program())
    exe = tmp_path / "mask"
    build = subprocess.run([_nvcc(), "-O2", "-std=c++17", "-o", str(exe), str(src)],
                           capture_output=True, text=True, timeout=600)
    assert build.returncode == 0, build.stdout + build.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "bad 0" in run.stdout, run.stdout
