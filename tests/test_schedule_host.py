"""The forward's unit schedule on the host, exhaustively.

The tile kernel launches one CTA per unit index and maps the index to a
(pattern, segment, batch, head, query tile) with decode_unit (csrc/common.cuh);
the host builds the schedule it decodes with make_geoms, pick_merger and
make_schedule (csrc/dilattn.cu). This test cuts those four functions out of
the sources as they are (decode_unit renamed, its device qualifiers dropped),
compiles them with nvcc into a host program and decodes every unit of many
geometries: fixed ones (the LongNet-base layer, the geometric family at 1M,
two r = 1 patterns, no r = 1 pattern, ragged and r > w shapes) and random ones.
Every (pattern, segment, batch, head, tile) must come out exactly once, the
tile level must never rise within a schedule, the partial-storing patterns'
units must all precede the merging pattern's, and the unit counts must be the
sums of nseg * B * H * ntiles. The backward's schedule gets the same check
from the decode part of bwd_unit (csrc/bwd_tc.cuh) and the group-order block of
launch_bwd: every (pattern, segment, batch, head, key tile) once, patterns in
groups by descending tile count, a unit with rows exactly when its key tile
holds a kept row, and its query tiles from its own (causal) or the first
through the segment's last. A third program checks, for every position of
every (pattern, head), partial_row (csrc/fwd_tc.cuh: where the merging tiles
look up another pattern's partial result) against the row the storing tile
wrote, -1 for rows the pattern does not keep, and view_coords
(csrc/common.cuh) against the position and the bounds of the view the kernel
picks, whose rows are exactly the positions below N of that phase, and
row_pos (csrc/simt.cuh, the fp32 path's inverse of the position map) against
seg_info. No GPU is touched."""
import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "sparse_long_sequence_dilated_b200", "csrc")


def _cut(text: str, head: str) -> str:
    """The definition that starts at `head`, through its matching closing brace."""
    i = text.index(head)
    j = text.index("{", i)
    depth = 0
    for k in range(j, len(text)):
        if text[k] == "{":
            depth += 1
        elif text[k] == "}":
            depth -= 1
            if depth == 0:
                return text[i:k + 1]
    raise ValueError(head)


def _program() -> str:
    common = open(os.path.join(CSRC, "common.cuh"), encoding="utf-8").read()
    host = open(os.path.join(CSRC, "dilattn.cu"), encoding="utf-8").read()
    decode = _cut(common, "__device__ __forceinline__ TileUnit decode_unit(")
    decode = re.sub(r"^__device__ __forceinline__ TileUnit decode_unit\(",
                    "static inline TileUnit host_decode_unit(", decode)
    funcs = "\n\n".join(_cut(host, h) for h in ("long long make_geoms(", "int pick_merger(",
                                               "long long make_schedule("))
    return r"""
#include <algorithm>
#include <climits>
#include <cstdio>
#include <cstring>
#include <vector>
#include "common.cuh"
namespace dil {
""" + decode + "\n\n" + funcs + r"""
}  // namespace dil
using namespace dil;

static uint64_t state = 0x9E3779B97F4A7C15ull;
static uint64_t next() { state ^= state << 13; state ^= state >> 7; state ^= state << 17; return state; }
static long long checks = 0;

// Returns the number of violations for one geometry.
static long long check(int B, int N, int H, int npat, const int* w, const int* r) {
  PatternGeom geo[kMaxPat];
  const int merger = pick_merger(w, r, npat);
  make_geoms(B, N, H, w, r, npat, geo, merger);
  const unsigned all = (1u << npat) - 1u, mbit = merger >= 0 ? (1u << merger) : 0u;
  Sched sp, sm;
  const long long up = make_schedule(geo, npat, B, H, sp, all & ~mbit);
  const long long um = mbit ? make_schedule(geo, npat, B, H, sm, mbit) : 0;
  long long base[kMaxPat + 1];
  base[0] = 0;
  for (int i = 0; i < npat; ++i)
    base[i + 1] = base[i] + (long long)geo[i].nseg * B * H * geo[i].ntiles;
  long long want_p = 0;
  for (int i = 0; i < npat; ++i)
    if (i != merger) want_p += base[i + 1] - base[i];
  std::vector<char> seen((size_t)base[npat], 0);
  long long bad = 0;
  if (up != want_p || up + um != base[npat]) ++bad;
  auto visit = [&](const Sched& sc, long long units, unsigned mask) {
    int prev_t = INT_MAX;
    for (long long u = 0; u < units; ++u) {
      ++checks;
      const TileUnit t = host_decode_unit(sc, geo, B, H, u);
      if (t.pat < 0 || t.pat >= npat || !((mask >> t.pat) & 1u) || t.seg < 0 ||
          t.seg >= geo[t.pat].nseg || t.b < 0 || t.b >= B || t.h < 0 || t.h >= H || t.t < 0 ||
          t.t >= geo[t.pat].ntiles) {
        if (bad < 3) printf("N=%d u=%lld out of range: pat %d seg %d b %d h %d t %d\n", N, u,
                            t.pat, t.seg, t.b, t.h, t.t);
        ++bad;
        continue;
      }
      if (t.t > prev_t) ++bad;  // longest first: the level never rises
      prev_t = t.t;
      const long long idx =
          base[t.pat] + (((long long)t.seg * B + t.b) * H + t.h) * geo[t.pat].ntiles + t.t;
      if (seen[(size_t)idx]) ++bad;
      seen[(size_t)idx] = 1;
    }
  };
  visit(sp, up, all & ~mbit);
  visit(sm, um, mbit);
  for (char c : seen)
    if (!c) ++bad;
  return bad;
}

int main() {
  long long bad = 0;
  {  // the LongNet-base layer, and at B = 4
    const int w[] = {2048, 4096, 8192, 16384, 32768}, r[] = {1, 2, 4, 6, 12};
    bad += check(1, 32768, 12, 5, w, r);
    bad += check(4, 32768, 12, 5, w, r);
  }
  {  // the geometric family at 1M, two batches
    int w[10], r[10];
    for (int i = 0; i < 10; ++i) { w[i] = 2048 << i; r[i] = 1 << i; }
    bad += check(2, 1 << 20, 12, 10, w, r);
  }
  {  // two r = 1 patterns; no r = 1 pattern; ragged; r > w; one row
    const int w1[] = {256, 1024, 512}, r1[] = {1, 1, 2};
    bad += check(2, 1100, 3, 3, w1, r1);
    const int w2[] = {500, 1536}, r2[] = {2, 3};
    bad += check(2, 1536, 4, 2, w2, r2);
    const int w3[] = {384, 700, 1000, 1100}, r3[] = {1, 3, 6, 12};
    bad += check(2, 1100, 3, 4, w3, r3);
    const int w4[] = {64, 96, 1100}, r4[] = {5, 200, 7};
    bad += check(2, 1100, 3, 3, w4, r4);
    const int w5[] = {1}, r5[] = {1};
    bad += check(1, 1, 2, 1, w5, r5);
  }
  {  // sixteen patterns
    int w[16], r[16];
    for (int i = 0; i < 16; ++i) { w[i] = 64 * (i + 1); r[i] = 1 + i % 5; }
    bad += check(1, 3000, 2, 16, w, r);
  }
  for (int c = 0; c < 3000; ++c) {  // random geometries
    const int N = 1 + (int)(next() % 5000);
    const int B = 1 + (int)(next() % 3), H = 1 + (int)(next() % 5);
    const int npat = 1 + (int)(next() % 6);
    int w[kMaxPat], r[kMaxPat];
    for (int i = 0; i < npat; ++i) {
      w[i] = 1 + (int)(next() % (uint64_t)(N + N / 2 + 1));
      r[i] = 1 + (int)(next() % 300);
      if (next() % 4 == 0) r[i] = 1;
    }
    bad += check(B, N, H, npat, w, r);
  }
  printf("checks %lld bad %lld\n", checks, bad);
  return bad != 0;
}
"""


def _nvcc():
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return None


@pytest.mark.skipif(_nvcc() is None, reason="nvcc not found")
def test_every_unit_decodes_once(tmp_path):
    src = tmp_path / "sched.cu"
    src.write_text(_program())
    exe = tmp_path / "sched"
    build = subprocess.run([_nvcc(), "-O2", "-std=c++17", "-I", CSRC, "-o", str(exe), str(src)],
                           capture_output=True, text=True, timeout=600)
    assert build.returncode == 0, build.stdout + build.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "bad 0" in run.stdout, run.stdout


def _bwd_program() -> str:
    """The backward's unit order (built inline in launch_bwd) and the decode part
    of bwd_unit, cut from the sources, over a stand-in for the parameter block
    holding the fields they read."""
    bwd = open(os.path.join(CSRC, "bwd_tc.cuh"), encoding="utf-8").read()
    host = open(os.path.join(CSRC, "dilattn.cu"), encoding="utf-8").read()
    i = bwd.index("__device__ __forceinline__ bool bwd_unit(")
    j = bwd.index("  // all tiles of a (pattern, segment, head) share one phase", i)
    decode = bwd[i:j].replace("__device__ __forceinline__ bool bwd_unit(",
                              "static inline bool host_bwd_unit(") + "  return true;\n}\n"
    order = _cut(host, "  // group-major unit order:")  # the comment and its block
    funcs = _cut(host, "long long make_geoms(")
    return r"""
#include <algorithm>
#include <climits>
#include <cstdio>
#include <cstring>
#include <vector>
#include "common.cuh"
namespace dil {
struct BwdParams {
  PatternGeom pat[kMaxPat];
  int npat, B, N, H, causal;
  int gorder[kMaxPat];
  long long gstart[kMaxPat + 1];
};
struct BwdUnit {
  TileUnit wu;
  PatternGeom g;
  SegInfo si;
  int u, t0, np;
};
""" + decode + "\n" + funcs + r"""
static long long build_order(BwdParams& p, int npat, int B, int H) {
""" + order + r"""
  return p.gstart[npat];
}
}  // namespace dil
using namespace dil;

static uint64_t state = 0xD1B54A32D192ED03ull;
static uint64_t next() { state ^= state << 13; state ^= state >> 7; state ^= state << 17; return state; }
static long long checks = 0;

static long long check(int B, int N, int H, int npat, const int* w, const int* r, int causal) {
  BwdParams p;
  memset(&p, 0, sizeof(p));
  p.npat = npat; p.B = B; p.N = N; p.H = H; p.causal = causal;
  make_geoms(B, N, H, w, r, npat, p.pat);
  const long long units = build_order(p, npat, B, H);
  long long base[kMaxPat + 1];
  base[0] = 0;
  for (int i = 0; i < npat; ++i)
    base[i + 1] = base[i] + (long long)p.pat[i].nseg * B * H * p.pat[i].ntiles;
  long long bad = units != base[npat] ? 1 : 0;
  std::vector<char> seen((size_t)base[npat], 0);
  int prev_pat = -1, prev_ntiles = INT_MAX;
  for (long long uu = 0; uu < units; ++uu) {
    ++checks;
    BwdUnit U;
    const bool has = host_bwd_unit(p, uu, U);
    const TileUnit& t = U.wu;
    if (t.pat < 0 || t.pat >= npat || t.seg < 0 || t.seg >= p.pat[t.pat].nseg || t.b < 0 ||
        t.b >= B || t.h < 0 || t.h >= H || U.u < 0 || U.u >= p.pat[t.pat].ntiles) {
      if (bad < 3) printf("N=%d uu=%lld out of range\n", N, uu);
      ++bad;
      continue;
    }
    // patterns in groups, by tile count, descending
    if (t.pat != prev_pat) {
      if (p.pat[t.pat].ntiles > prev_ntiles) ++bad;
      prev_ntiles = p.pat[t.pat].ntiles;
      prev_pat = t.pat;
    }
    const long long idx =
        base[t.pat] + (((long long)t.seg * B + t.b) * H + t.h) * p.pat[t.pat].ntiles + U.u;
    if (seen[(size_t)idx]) ++bad;
    seen[(size_t)idx] = 1;
    // a unit has rows iff its key tile holds a kept row; then it runs the query
    // tiles from its own (causal) or the first, through the segment's last
    const SegInfo si = seg_info(p.pat[t.pat], N, t.h, t.seg);
    const int nq = (si.n + BM - 1) / BM;
    if (has != (U.u < nq)) ++bad;
    if (has && (U.t0 != (causal ? U.u : 0) || U.np != nq - U.t0 || U.np < 1)) ++bad;
  }
  for (char c : seen)
    if (!c) ++bad;
  return bad;
}

int main() {
  long long bad = 0;
  for (int causal = 0; causal < 2; ++causal) {
    const int w[] = {2048, 4096, 8192, 16384, 32768}, r[] = {1, 2, 4, 6, 12};
    bad += check(1, 32768, 12, 5, w, r, causal);
    bad += check(4, 32768, 12, 5, w, r, causal);
    const int w4[] = {64, 96, 1100}, r4[] = {5, 200, 7};
    bad += check(2, 1100, 3, 3, w4, r4, causal);
    const int w5[] = {1}, r5[] = {1};
    bad += check(1, 1, 2, 1, w5, r5, causal);
  }
  {
    int w[10], r[10];
    for (int i = 0; i < 10; ++i) { w[i] = 2048 << i; r[i] = 1 << i; }
    bad += check(1, 1 << 20, 12, 10, w, r, 1);
  }
  for (int c = 0; c < 3000; ++c) {
    const int N = 1 + (int)(next() % 5000);
    const int B = 1 + (int)(next() % 3), H = 1 + (int)(next() % 5);
    const int npat = 1 + (int)(next() % 6);
    int w[kMaxPat], r[kMaxPat];
    for (int i = 0; i < npat; ++i) {
      w[i] = 1 + (int)(next() % (uint64_t)(N + N / 2 + 1));
      r[i] = 1 + (int)(next() % 300);
      if (next() % 4 == 0) r[i] = 1;
    }
    bad += check(B, N, H, npat, w, r, (int)(next() & 1));
  }
  printf("checks %lld bad %lld\n", checks, bad);
  return bad != 0;
}
"""


@pytest.mark.skipif(_nvcc() is None, reason="nvcc not found")
def test_every_backward_unit_decodes_once(tmp_path):
    src = tmp_path / "bsched.cu"
    src.write_text(_bwd_program())
    exe = tmp_path / "bsched"
    build = subprocess.run([_nvcc(), "-O2", "-std=c++17", "-I", CSRC, "-o", str(exe), str(src)],
                           capture_output=True, text=True, timeout=600)
    assert build.returncode == 0, build.stdout + build.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "bad 0" in run.stdout, run.stdout


def _rows_program() -> str:
    """partial_row (csrc/fwd_tc.cuh) and view_coords (csrc/common.cuh), cut from
    the sources, with make_geoms from csrc/dilattn.cu."""
    common = open(os.path.join(CSRC, "common.cuh"), encoding="utf-8").read()
    fwd = open(os.path.join(CSRC, "fwd_tc.cuh"), encoding="utf-8").read()
    host = open(os.path.join(CSRC, "dilattn.cu"), encoding="utf-8").read()
    prow = _cut(fwd, "__device__ __forceinline__ int partial_row(").replace(
        "__device__ __forceinline__ int partial_row(", "static inline int host_partial_row(")
    view = _cut(common, "__device__ __forceinline__ void view_coords(").replace(
        "__device__ __forceinline__ void view_coords(", "static inline void host_view_coords(")
    simt = open(os.path.join(CSRC, "simt.cuh"), encoding="utf-8").read()
    rowpos = _cut(simt, "struct RowPos {") + ";\n\n" + _cut(
        simt, "__device__ __forceinline__ RowPos row_pos(").replace(
        "__device__ __forceinline__ RowPos row_pos(", "static inline RowPos host_row_pos(")
    funcs = _cut(host, "long long make_geoms(")
    return r"""
#include <algorithm>
#include <cstdio>
#include <cstring>
#include "common.cuh"
namespace dil {
""" + prow + "\n\n" + view + "\n\n" + rowpos + "\n\n" + funcs + r"""
}  // namespace dil
using namespace dil;

static uint64_t state = 0x2545F4914F6CDD1Dull;
static uint64_t next() { state ^= state << 13; state ^= state >> 7; state ^= state << 17; return state; }
static long long checks = 0;

// Every position of every (pattern, head): the kept rows' view coordinates and
// partial rows, and -1 for the rows a pattern does not keep.
static long long check(int B, int N, int H, int npat, const int* w, const int* r) {
  PatternGeom geo[kMaxPat];
  make_geoms(B, N, H, w, r, npat, geo);
  long long bad = 0;
  for (int i = 0; i < npat; ++i) {
    const PatternGeom& g = geo[i];
    const int nfloor = N / g.r, nmod = N % g.r;
    // the view a phase selects holds exactly the positions below N of that phase
    for (int ph = 0; ph < g.r; ++ph) {
      ++checks;
      const int rows = ph < nmod ? nfloor + 1 : nfloor;
      const int want = ph < N ? (N - ph + g.r - 1) / g.r : 0;
      if (rows != want) ++bad;
    }
    for (int b = 0; b < B; b += (B > 1 ? B - 1 : 1)) {   // first and last batch
      for (int h = 0; h < H; ++h) {
        const int bh = b * H + h;
        for (int n = 0; n < N; ++n) {
          ++checks;
          const int seg = n / g.w;
          const SegInfo si = seg_info(g, N, h, seg);
          const long long rel = n - si.start - si.off;
          const bool kept = rel >= 0 && rel % g.r == 0;
          const int got = host_partial_row(g, n, si.off, bh);
          // the fp32 path's inverse of the position map
          const RowPos rp = host_row_pos(g, N, h, n);
          if (rp.kept != kept || rp.seg != seg || rp.start != si.start || rp.off != si.off ||
              rp.end != std::min<long long>(si.start + g.w, N) ||
              rp.v != (kept ? (int)(rel / g.r) : -1))
            ++bad;
          if (!kept) {
            if (got != -1) ++bad;
            continue;
          }
          const int v = (int)(rel / g.r);
          if (v >= si.n) ++bad;
          const long long want =
              g.part_base + ((long long)bh * g.nseg + seg) * g.pstride + v;
          if (got != want) {
            if (bad < 3) printf("N=%d w=%d r=%d h=%d n=%d partial %d want %lld\n", N, g.w, g.r,
                                h, n, got, want);
            ++bad;
          }
          int ph, m;
          host_view_coords(g, si, v, ph, m);
          const int rows = ph < nmod ? nfloor + 1 : nfloor;   // the view the kernel picks
          if (ph < 0 || ph >= g.r || (long long)ph + (long long)m * g.r != n || m < 0 ||
              m >= rows)
            ++bad;
        }
      }
    }
  }
  return bad;
}

int main() {
  long long bad = 0;
  {
    const int w[] = {2048, 4096, 8192, 16384, 32768}, r[] = {1, 2, 4, 6, 12};
    bad += check(2, 32768, 12, 5, w, r);
  }
  {
    int w[8], r[8];
    for (int i = 0; i < 8; ++i) { w[i] = 2048 << i; r[i] = 1 << i; }
    bad += check(1, 262144, 4, 8, w, r);
  }
  {
    const int w[] = {64, 96, 1100, 384, 700}, r[] = {5, 200, 7, 1, 3};
    bad += check(3, 1100, 3, 5, w, r);
  }
  for (int c = 0; c < 600; ++c) {
    const int N = 1 + (int)(next() % 3000);
    const int B = 1 + (int)(next() % 3), H = 1 + (int)(next() % 4);
    const int npat = 1 + (int)(next() % 6);
    int w[kMaxPat], r[kMaxPat];
    for (int i = 0; i < npat; ++i) {
      w[i] = 1 + (int)(next() % (uint64_t)(N + N / 2 + 1));
      r[i] = 1 + (int)(next() % 300);
    }
    bad += check(B, N, H, npat, w, r);
  }
  printf("checks %lld bad %lld\n", checks, bad);
  return bad != 0;
}
"""


@pytest.mark.skipif(_nvcc() is None, reason="nvcc not found")
def test_partial_rows_and_view_coordinates(tmp_path):
    src = tmp_path / "rows.cu"
    src.write_text(_rows_program())
    exe = tmp_path / "rows"
    build = subprocess.run([_nvcc(), "-O2", "-std=c++17", "-I", CSRC, "-o", str(exe), str(src)],
                           capture_output=True, text=True, timeout=600)
    assert build.returncode == 0, build.stdout + build.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "bad 0" in run.stdout, run.stdout
