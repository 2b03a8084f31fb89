"""The library's TMA descriptors on the host, against a recording encoder.

strided_map and gathered_map (csrc/dilattn.cu) are cut out of the source as
they are and compiled into a host program in which cuTensorMapEncodeTiled is a
stand-in that records its arguments. For many geometries, every element type
the library uses (bf16, fp32, fp16, e4m3) and both box heights, the test
checks what the encoder's documentation requires (rank 5, a 16-byte aligned
base, every dimension at least 1 and at most 2^32, strides multiples of 16
below 2^40, boxes of 1..256 elements whose inner extent is the 128 bytes of the
128-byte swizzle) and what the kernels rely on: every in-bounds coordinate of
a view addresses the row the kernels mean (row ph + m r of batch b for a
strided view, dilated row j of rank g's block for a gathered one), inside the
caller's tensor, and no two coordinates share a row. A strided view reaching
past its tensor is the fault class an earlier single-view design hit. No GPU
is touched."""
import os
import subprocess

import pytest

from tests.test_schedule_host import CSRC, _cut, _nvcc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _program() -> str:
    host = open(os.path.join(CSRC, "dilattn.cu"), encoding="utf-8").read()
    i = host.index("using MapKey =")
    decls = host[i:host.index("int strided_map(", i)]
    funcs = _cut(host, "int strided_map(") + "\n\n" + _cut(host, "int gathered_map(")
    return r"""
#include <cuda.h>
#include <cudaTypedefs.h>
#include <algorithm>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>
#include "dilattn.h"
#include "common.cuh"
namespace dil {
thread_local char g_last_error[512] = "";
static long long bad = 0, checks = 0;
struct Call {
  int rank, dtype;
  const void* addr;
  cuuint64_t dims[5], strides[4];
  cuuint32_t box[5], estr[5];
  int swizzle;
};
static Call last;
static int esize(CUtensorMapDataType t) {
  return t == CU_TENSOR_MAP_DATA_TYPE_FLOAT32 ? 4 : t == CU_TENSOR_MAP_DATA_TYPE_UINT8 ? 1 : 2;
}
static CUresult fake_encode(CUtensorMap* m, CUtensorMapDataType dt, cuuint32_t rank, void* addr,
                            const cuuint64_t* dims, const cuuint64_t* strides,
                            const cuuint32_t* box, const cuuint32_t* estr,
                            CUtensorMapInterleave il, CUtensorMapSwizzle sw,
                            CUtensorMapL2promotion, CUtensorMapFloatOOBfill) {
  memset(m, 0, sizeof(*m));
  last.rank = (int)rank;
  last.dtype = (int)dt;
  last.addr = addr;
  last.swizzle = (int)sw;
  const int e = esize(dt);
  if (rank != 5 || il != CU_TENSOR_MAP_INTERLEAVE_NONE || sw != CU_TENSOR_MAP_SWIZZLE_128B) ++bad;
  if ((reinterpret_cast<uintptr_t>(addr) & 15) != 0) ++bad;
  for (int k = 0; k < 5; ++k) {
    last.dims[k] = dims[k];
    last.box[k] = box[k];
    last.estr[k] = estr[k];
    if (dims[k] < 1 || dims[k] > (1ull << 32)) ++bad;
    if (box[k] < 1 || box[k] > 256 || estr[k] < 1 || estr[k] > 8) ++bad;
  }
  for (int k = 0; k < 4; ++k) {
    last.strides[k] = strides[k];
    if (strides[k] % 16 != 0 || strides[k] >= (1ull << 40)) ++bad;
  }
  if ((unsigned long long)box[0] * e != 128) ++bad;  // the 128-byte swizzle's inner extent
  return CUDA_SUCCESS;
}
PFN_cuTensorMapEncodeTiled_v12000 g_encode = fake_encode;
static int get_encoder() { return DILATTN_OK; }
""" + decls + funcs + r"""
}  // namespace dil
using namespace dil;

static uint64_t state = 0x853C49E6748FEA9Bull;
static uint64_t next() { state ^= state << 13; state ^= state >> 7; state ^= state << 17; return state; }

// A strided view of [B][N][H][d]: in-bounds coordinates (ph, m, b) address row
// ph + m r < N of batch b, each row once; heads and columns stay inside the row.
static void check_strided(int B, int N, int H, int d, int r, int tail, int f32, int box_rows) {
  const void* base = reinterpret_cast<const void*>((uintptr_t)(1ull << 30) + 4096 * (next() % 64));
  CUtensorMap m;
  memset(&last, 0, sizeof(last));
  const int rc = strided_map(base, B, N, H, d, r, tail, &m, f32, box_rows);
  ++checks;
  if (rc != DILATTN_OK) { ++bad; return; }
  const int nmod = N % r;
  const long long nfloor = N / r;
  if ((tail && nmod == 0) || (!tail && nfloor == 0)) {  // an empty view: no encoder call
    if (last.rank != 0) ++bad;
    return;
  }
  if (last.addr != base) ++bad;
  const int e = f32 == 1 ? 4 : f32 == 3 ? 1 : 2;
  const unsigned long long rowb = (unsigned long long)H * d * e;
  const unsigned long long total = (unsigned long long)B * N * rowb;
  if (last.dims[0] != (cuuint64_t)d || last.dims[1] != (cuuint64_t)H || last.box[3] != (cuuint32_t)box_rows)
    ++bad;
  // inner extent: columns and heads stay inside one row
  if ((last.dims[0] - 1) * e + (last.dims[1] - 1) * last.strides[0] + e > rowb ||
      last.strides[0] != (cuuint64_t)d * e)
    ++bad;
  std::vector<char> seen((size_t)B * N, 0);
  for (cuuint64_t b = 0; b < last.dims[4]; ++b)
    for (cuuint64_t mm = 0; mm < last.dims[3]; ++mm)
      for (cuuint64_t ph = 0; ph < last.dims[2]; ++ph) {
        ++checks;
        const unsigned long long off = ph * last.strides[1] + mm * last.strides[2] + b * last.strides[3];
        const long long pos = (long long)(ph + mm * (unsigned long long)r);
        if (off % rowb != 0 || off + rowb > total || pos >= N ||
            off / rowb != (unsigned long long)(b * N + pos) || ph >= (cuuint64_t)r) {
          if (bad < 5) printf("strided B=%d N=%d r=%d tail=%d: (%llu,%llu,%llu) off %llu\n", B, N,
                              r, tail, (unsigned long long)ph, (unsigned long long)mm,
                              (unsigned long long)b, off);
          ++bad;
          continue;
        }
        char& s = seen[(size_t)(off / rowb)];
        if (s) ++bad;
        s = 1;
      }
}

// A gathered buffer [ranks][B][rank_rows][H][d] bf16: coordinate (j, g, b) is
// dilated row j of rank g's block of batch b, each once.
static void check_gathered(int B, int H, int d, int rank_rows, int ranks, int box_rows) {
  const void* base = reinterpret_cast<const void*>((uintptr_t)(1ull << 31) + 256 * (next() % 64));
  CUtensorMap m;
  memset(&last, 0, sizeof(last));
  const int rc = gathered_map(base, B, H, d, rank_rows, ranks, &m, box_rows);
  ++checks;
  if (rc != DILATTN_OK || last.addr != base) { ++bad; return; }
  const unsigned long long rowb = (unsigned long long)H * d * 2;
  const unsigned long long total = (unsigned long long)ranks * B * rank_rows * rowb;
  if (last.dims[0] != (cuuint64_t)d || last.dims[1] != (cuuint64_t)H ||
      last.dims[2] != (cuuint64_t)rank_rows || last.dims[3] != (cuuint64_t)ranks ||
      last.dims[4] != (cuuint64_t)B || last.box[2] != (cuuint32_t)box_rows)
    ++bad;
  std::vector<char> seen((size_t)ranks * B * rank_rows, 0);
  for (int b = 0; b < B; ++b)
    for (int g = 0; g < ranks; ++g)
      for (int j = 0; j < rank_rows; ++j) {
        ++checks;
        const unsigned long long off = j * last.strides[1] + g * last.strides[2] + b * last.strides[3];
        const unsigned long long want = (((unsigned long long)g * B + b) * rank_rows + j) * rowb;
        if (off != want || off + rowb > total) { ++bad; continue; }
        char& s = seen[(size_t)(off / rowb)];
        if (s) ++bad;
        s = 1;
      }
  // a box of box_rows rows never crosses a rank's block
  if (rank_rows % box_rows != 0) ++bad;
}

int main() {
  const int types[4] = {0, 1, 2, 3};
  for (int t = 0; t < 4; ++t)
    for (int tail = 0; tail < 2; ++tail) {
      // the workloads' shapes
      check_strided(1, 32768, 12, 64, 6, tail, types[t], 128);
      check_strided(1, 32768, 12, 64, 12, tail, types[t], 32);
      check_strided(2, 131072, 32, 128, 64, tail, types[t], 64);
      check_strided(1, 1 << 20, 12, 64, 512, tail, types[t], 128);
    }
  for (int c = 0; c < 4000; ++c) {
    const int B = 1 + (int)(next() % 3), H = 1 + (int)(next() % 4);
    const int N = 1 + (int)(next() % 3000), r = 1 + (int)(next() % 400);
    const int f32 = (int)(next() % 4);
    const int d = (f32 == 3 || next() % 2) ? 128 : 64;
    const int box_rows = f32 == 1 ? 32 : (next() % 2 ? 128 : 64);
    check_strided(B, N, H, d, r, (int)(next() % 2), f32, box_rows);
  }
  for (int c = 0; c < 500; ++c) {
    const int B = 1 + (int)(next() % 3), H = 1 + (int)(next() % 4);
    const int ranks = 1 + (int)(next() % 8), rank_rows = 128 * (1 + (int)(next() % 8));
    check_gathered(B, H, next() % 2 ? 128 : 64, rank_rows, ranks, next() % 2 ? 128 : 64);
  }
  printf("checks %lld bad %lld\n", checks, bad);
  return bad != 0;
}
"""


@pytest.mark.skipif(_nvcc() is None, reason="nvcc not found")
def test_tensor_maps(tmp_path):
    src = tmp_path / "maps.cu"
    src.write_text(_program())
    exe = tmp_path / "maps"
    build = subprocess.run([_nvcc(), "-O2", "-std=c++17", "-I", CSRC, "-I",
                            os.path.join(ROOT, "include"), "-o", str(exe), str(src)],
                           capture_output=True, text=True, timeout=600)
    assert build.returncode == 0, build.stdout + build.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "bad 0" in run.stdout, run.stdout
