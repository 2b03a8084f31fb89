// libdilattn: C-ABI entry points (validation, TMA descriptor set-up, launches).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "dilattn.h"
#include "common.cuh"
#include "fwd_tc.cuh"
#include "bwd_tc.cuh"
#include "simt.cuh"

namespace dil {

__device__ int g_dev_error;  // device-side error word (bounded waits that ran out)

// Self-test of the failure path: warp 0 waits on an mbarrier that nothing
// arrives on, with a limit of limit_ns; warp 1 waits on another one with the
// kernels' ordinary 4 s limit and must give up as soon as warp 0 has raised
// the CTA's abort flag. result[0], result[1]: 1 if the warp's wait completed
// (it must not), 0 if it gave up; result[2], result[3]: nanoseconds each
// warp waited.
__global__ void selftest_wait_kernel(ErrCtx err, unsigned long long limit_ns, int* result) {
  __shared__ __align__(8) uint64_t bars[2];
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars[0]), 1);
    mbar_init(smem_u32(&bars[1]), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    const unsigned long long t0 = globaltimer_ns();
    const bool ok = warp == 0
        ? mbar_wait(smem_u32(&bars[0]), 0, &abort_flag, err, limit_ns)
        : mbar_wait(smem_u32(&bars[1]), 0, &abort_flag, err);
    result[warp] = ok ? 1 : 0;
    result[2 + warp] = (int)min(globaltimer_ns() - t0, 2000000000ull);
  }
}

namespace {

thread_local char g_last_error[512] = "";

// Launch tags for the device error word (see ErrCtx): 1 .. 2^23 - 1, cycling.
std::atomic<unsigned> g_launch_tag{0};
int next_tag() { return (int)(g_launch_tag.fetch_add(1u) % 0x7FFFFFu) + 1; }


int cuda_fail(cudaError_t e, const char* what) {
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%d)", what, cudaGetErrorString(e),
           (int)e);
  return DILATTN_ERR_CUDA;
}

thread_local cudaEvent_t g_trace_begin = nullptr;
thread_local cudaEvent_t g_trace_end = nullptr;

int trace_mark(cudaEvent_t ev, cudaStream_t stream) {
  if (ev == nullptr) return DILATTN_OK;
  cudaError_t e = cudaEventRecord(ev, stream);
  return e == cudaSuccess ? DILATTN_OK : cuda_fail(e, "cudaEventRecord");
}

// ------------------------------------------------------------------ device state
struct DeviceState {
  bool init = false;
  bool arch_ok = false;
  int* err_word = nullptr;
  int num_sms = 0;
};

std::mutex g_mu;
std::map<int, DeviceState> g_devices;

int device_state(DeviceState** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState& st = g_devices[dev];
  if (!st.init) {
    int major = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    st.arch_ok = (major == 10);
    if (st.arch_ok) {
      e = cudaDeviceGetAttribute(&st.num_sms, cudaDevAttrMultiProcessorCount, dev);
      if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
      e = cudaGetSymbolAddress(reinterpret_cast<void**>(&st.err_word), g_dev_error);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
      e = cudaFuncSetAttribute(fwd_tile_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               FwdCfg<64>::SMEM_BYTES);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
      e = cudaFuncSetAttribute(fwd_tile_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               FwdCfg<128>::SMEM_BYTES);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
      e = cudaFuncSetAttribute(bwd_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               BwdCfg::SMEM_BYTES);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    }
    st.init = true;
  }
  if (!st.arch_ok) return DILATTN_ERR_UNSUPPORTED;
  *out = &st;
  return DILATTN_OK;
}

// ------------------------------------------------------------------ TMA descriptors
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

int get_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_encode) {
    snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled unavailable");
    return DILATTN_ERR_CUDA;
  }
  return DILATTN_OK;
}

// Strided view of a [B][N][H][d] tensor (bf16, or fp32 when f32 is set) that
// gathers every r-th row, with the tensor's own base address: dims
// {d, H, P, M, B}, byte strides {e d, e H d, e H d r, e H d N} for element
// size e, so element (c, h, ph, m, b) is row ph + m*r of batch b. The main
// view has P = r phases and M = floor(N/r) rows; the tail view has
// P = N mod r and M = floor(N/r) + 1. Either way every in-bounds coordinate is
// a row below N; loads read zeros and stores/reduces skip rows past it. Box:
// 128 bytes of columns (128-byte swizzle) x box_rows rows (128, or 32 for the
// backward's per-warp reduce-adds).
using MapKey = std::tuple<const void*, int, int, int, int, int, int, int, int>;
std::mutex g_map_mu;
std::map<MapKey, CUtensorMap> g_maps;

int strided_map(const void* ptr, int B, int N, int H, int d, int r, int tail, CUtensorMap* out,
                int f32 = 0, int box_rows = BM) {
  const long long nfloor = N / r;
  const int nmod = N % r;
  if ((tail && nmod == 0) || (!tail && nfloor == 0)) {
    memset(out, 0, sizeof(*out));  // a view no tile of this problem can address
    return DILATTN_OK;
  }
  MapKey key{ptr, B, N, H, d, r, tail, f32, box_rows};
  {
    std::lock_guard<std::mutex> lk(g_map_mu);
    auto it = g_maps.find(key);
    if (it != g_maps.end()) {
      *out = it->second;
      return DILATTN_OK;
    }
  }
  int rc = get_encoder();
  if (rc != DILATTN_OK) return rc;
  const int esz = f32 ? 4 : 2;
  const long long rowb = (long long)H * d * esz;
  cuuint64_t dims[5] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)(tail ? nmod : r),
                        (cuuint64_t)(tail ? nfloor + 1 : nfloor), (cuuint64_t)B};
  cuuint64_t strides[4] = {(cuuint64_t)d * esz, (cuuint64_t)rowb, (cuuint64_t)(rowb * r),
                           (cuuint64_t)(rowb * N)};
  cuuint32_t box[5] = {(cuuint32_t)(128 / esz), 1, 1, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUtensorMap m;
  CUresult cr = g_encode(&m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                         5, const_cast<void*>(ptr), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) {
    snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled failed (%d)", (int)cr);
    return DILATTN_ERR_CUDA;
  }
  {
    std::lock_guard<std::mutex> lk(g_map_mu);
    if (g_maps.size() > 4096) g_maps.clear();
    g_maps[key] = m;
  }
  *out = m;
  return DILATTN_OK;
}

// 2-D view of the forward's fp32 partial outputs [rows][d] for TMA stores:
// box 32 columns (128 bytes, 128-byte swizzle) x 128 rows.
int partial_map(const float* ptr, long long rows, int d, CUtensorMap* out) {
  MapKey key{ptr, (int)(rows >> 31), (int)(rows & 0x7fffffff), d, -1, -1, -1, 2, BM};
  {
    std::lock_guard<std::mutex> lk(g_map_mu);
    auto it = g_maps.find(key);
    if (it != g_maps.end()) {
      *out = it->second;
      return DILATTN_OK;
    }
  }
  int rc = get_encoder();
  if (rc != DILATTN_OK) return rc;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 4};
  cuuint32_t box[2] = {32, (cuuint32_t)BM};
  cuuint32_t estr[2] = {1, 1};
  CUtensorMap m;
  CUresult cr = g_encode(&m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(ptr), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) {
    snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled failed (%d)", (int)cr);
    return DILATTN_ERR_CUDA;
  }
  {
    std::lock_guard<std::mutex> lk(g_map_mu);
    if (g_maps.size() > 4096) g_maps.clear();
    g_maps[key] = m;
  }
  *out = m;
  return DILATTN_OK;
}

// ------------------------------------------------------------------ validation
int check_shape(int B, int N, int H, int d, const int* w, const int* r, int npat, int causal) {
  if (B < 1 || N < 1 || H < 1 || d < 1) return DILATTN_ERR_INVALID_ARG;
  if (npat < 1 || npat > DILATTN_MAX_PATTERNS || w == nullptr || r == nullptr)
    return DILATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return DILATTN_ERR_INVALID_ARG;
  const double elems = (double)B * N * H * d;
  if (elems >= 1099511627776.0) return DILATTN_ERR_INVALID_ARG;
  for (int i = 0; i < npat; ++i) {
    if (w[i] < 1 || r[i] < 1) return DILATTN_ERR_INVALID_ARG;
    if ((double)r[i] * H * d * 4 >= 1099511627776.0) return DILATTN_ERR_INVALID_ARG;
  }
  return DILATTN_OK;
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

bool overlaps(const void* a, size_t an, const void* b, size_t bn) {
  const char* x = (const char*)a;
  const char* y = (const char*)b;
  return x < y + bn && y < x + an;
}

long long make_geoms(int B, int N, int H, const int* w, const int* r, int npat,
                     PatternGeom* geo) {
  long long rows = 0;
  for (int i = 0; i < npat; ++i) {
    PatternGeom& g = geo[i];
    g.w = w[i];
    g.r = r[i];
    g.nseg = (int)(((long long)N + w[i] - 1) / w[i]);
    const long long span = std::min<long long>(w[i], N);
    g.nmax = (int)((span + r[i] - 1) / r[i]);
    g.ntiles = (g.nmax + BM - 1) / BM;
    g.pstride = g.ntiles * BM;
    g.nmod = N % r[i];
    g.part_base = rows;
    rows += (long long)B * H * g.nseg * g.pstride;
  }
  return rows;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Longest-first unit order for the tile kernels (see Sched).
long long make_schedule(const PatternGeom* pat, int npat, int B, int H, Sched& sc) {
  std::vector<int> order(npat);
  for (int i = 0; i < npat; ++i) order[i] = i;
  std::stable_sort(order.begin(), order.end(),
                   [&](int a, int b) { return pat[a].ntiles > pat[b].ntiles; });
  std::vector<int> vals;
  for (int i : order)
    if (vals.empty() || vals.back() != pat[i].ntiles) vals.push_back(pat[i].ntiles);
  for (int i = 0; i < npat; ++i) sc.order[i] = order[i];
  sc.nband = (int)vals.size();
  sc.start[0] = 0;
  for (int j = 0; j < sc.nband; ++j) {
    const int lo = j + 1 < sc.nband ? vals[j + 1] : 0;
    sc.nt[j] = vals[j];
    int act = 0;
    long long per = 0;
    for (int a = 0; a < npat; ++a) {
      if (pat[order[a]].ntiles >= vals[j]) {
        ++act;
        per += (long long)pat[order[a]].nseg * B * H;
      }
    }
    sc.npat_active[j] = act;
    sc.per_level[j] = per;
    sc.start[j + 1] = sc.start[j] + (long long)(vals[j] - lo) * per;
  }
  sc.nt[sc.nband] = 0;
  return sc.start[sc.nband];
}

// The fp32 copy of out inside a forward workspace of `rows` partial rows.
float* fwd_out_f32(void* ws, long long rows, int d) {
  return reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + align256((size_t)rows * d * 4) +
                                  align256((size_t)rows * 4));
}

template <int D>
int launch_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int N,
               int H, const int* w, const int* r, int npat, int causal, void* ws,
               DeviceState* st, cudaStream_t stream) {
  static_assert(sizeof(FwdParams) < 32000, "kernel parameter block too large");
  FwdParams p;
  memset(&p, 0, sizeof(p));
  p.npat = npat;
  p.B = B;
  p.N = N;
  p.H = H;
  p.causal = causal;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  const long long rows = make_geoms(B, N, H, w, r, npat, p.pat);
  p.part_o = reinterpret_cast<float*>(ws);
  p.part_lse = reinterpret_cast<float*>((char*)ws + align256((size_t)rows * D * 4));
  p.err = ErrCtx{st->err_word, next_tag()};
  {
    int rc = partial_map(p.part_o, rows, D, &p.tm_po);
    if (rc != DILATTN_OK) return rc;
  }
  for (int i = 0; i < npat; ++i) {
    const void* src[3] = {q, k, v};
    CUtensorMap* dst[3] = {&p.tmq[i], &p.tmk[i], &p.tmv[i]};
    CUtensorMap* dst_t[3] = {&p.tmq_t[i], &p.tmk_t[i], &p.tmv_t[i]};
    for (int j = 0; j < 3; ++j) {
      int rc = strided_map(src[j], B, N, H, D, r[i], 0, dst[j]);
      if (rc == DILATTN_OK) rc = strided_map(src[j], B, N, H, D, r[i], 1, dst_t[j]);
      if (rc != DILATTN_OK) return rc;
    }
  }
  const long long units = make_schedule(p.pat, npat, B, H, p.sched);
  if (units > 0x7fffffffLL) return DILATTN_ERR_UNSUPPORTED;
  int rc = trace_mark(g_trace_begin, stream);
  if (rc != DILATTN_OK) return rc;
  fwd_tile_kernel<D><<<(unsigned)units, FwdCfg<D>::THREADS, FwdCfg<D>::SMEM_BYTES, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fwd_tile_kernel launch");
  rc = trace_mark(g_trace_end, stream);
  if (rc != DILATTN_OK) return rc;

  MergeParams mp;
  memset(&mp, 0, sizeof(mp));
  memcpy(mp.pat, p.pat, sizeof(mp.pat));
  mp.npat = npat;
  mp.B = B;
  mp.N = N;
  mp.H = H;
  mp.part_o = p.part_o;
  mp.part_lse = p.part_lse;
  mp.out = reinterpret_cast<__nv_bfloat16*>(out);
  mp.out_f32 = fwd_out_f32(ws, rows, D);
  mp.lse = lse;
  const long long total_rows = (long long)B * N * H;
  constexpr int rows_per_block = 256 / DILATTN_MERGE_TPR;
  const long long blocks = (total_rows + rows_per_block - 1) / rows_per_block;
  merge_kernel<D><<<(unsigned)blocks, 256, 0, stream>>>(mp);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "merge_kernel launch");
  return DILATTN_OK;
}

int launch_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse,
               const void* dout, void* dq, void* dk, void* dv, int B, int N, int H,
               const int* w, const int* r, int npat, int causal, const float* out_f32, void* ws,
               DeviceState* st, cudaStream_t stream) {
  constexpr int D = 64;
  static_assert(sizeof(BwdParams) < 32000, "kernel parameter block too large");
  BwdParams p;
  memset(&p, 0, sizeof(p));
  p.npat = npat;
  p.B = B;
  p.N = N;
  p.H = H;
  p.causal = causal;
  p.tau = (float)(1.0 / std::sqrt((double)D));
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  make_geoms(B, N, H, w, r, npat, p.pat);
  // [3B][N][H][64] fp32: dq for batches 0..B-1, then dk, then dv (B*N*H*64*4
  // is a multiple of 256, so the three align256 blocks are adjacent)
  const size_t tbytes = align256((size_t)B * N * H * D * 4);
  char* wsb = reinterpret_cast<char*>(ws);
  float* dq_acc = reinterpret_cast<float*>(wsb);
  float* dk_acc = reinterpret_cast<float*>(wsb + tbytes);
  float* dv_acc = reinterpret_cast<float*>(wsb + 2 * tbytes);
  float* drow = reinterpret_cast<float*>(wsb + 3 * tbytes);
  p.drow = drow;
  p.lse = lse;
  p.err = ErrCtx{st->err_word, next_tag()};
  for (int i = 0; i < npat; ++i) {
    const void* src[4] = {q, k, v, dout};
    CUtensorMap* dst[4] = {&p.tmq[i], &p.tmk[i], &p.tmv[i], &p.tmdo[i]};
    CUtensorMap* dst_t[4] = {&p.tmq_t[i], &p.tmk_t[i], &p.tmv_t[i], &p.tmdo_t[i]};
    for (int j = 0; j < 4; ++j) {
      int rc = strided_map(src[j], B, N, H, D, r[i], 0, dst[j]);
      if (rc == DILATTN_OK) rc = strided_map(src[j], B, N, H, D, r[i], 1, dst_t[j]);
      if (rc != DILATTN_OK) return rc;
    }
    // reduce-add targets: one row warp adds a 32-row x 32-column block
    int rc = strided_map(dq_acc, 3 * B, N, H, D, r[i], 0, &p.tmacc[i], 1, 32);
    if (rc == DILATTN_OK) rc = strided_map(dq_acc, 3 * B, N, H, D, r[i], 1, &p.tmacc_t[i], 1, 32);
    if (rc != DILATTN_OK) return rc;
  }
  // group-major unit order: patterns by tile count (descending, stable), then
  // (segment, batch, head) groups, then key tiles
  {
    std::vector<int> order(npat);
    for (int i = 0; i < npat; ++i) order[i] = i;
    std::stable_sort(order.begin(), order.end(),
                     [&](int a, int b) { return p.pat[a].ntiles > p.pat[b].ntiles; });
    p.gstart[0] = 0;
    for (int a = 0; a < npat; ++a) {
      const PatternGeom& g = p.pat[order[a]];
      p.gorder[a] = order[a];
      p.gstart[a + 1] = p.gstart[a] + (long long)g.nseg * B * H * g.ntiles;
    }
  }
  const long long units = p.gstart[npat];
  if (units > 0x7fffffffLL) return DILATTN_ERR_UNSUPPORTED;
  const long long rows = (long long)B * N * H;
  p.counter = reinterpret_cast<int*>(wsb + 3 * tbytes + align256((size_t)B * H * N * 4));

  PrepParams pp;
  pp.B = B;
  pp.N = N;
  pp.H = H;
  pp.out = reinterpret_cast<const __nv_bfloat16*>(out);
  pp.out_f32 = out_f32;
  pp.dout = reinterpret_cast<const __nv_bfloat16*>(dout);
  pp.drow = drow;
  pp.dq_acc = dq_acc;
  pp.dk_acc = dk_acc;
  pp.dv_acc = dv_acc;
  pp.counter = p.counter;
  bwd_prep_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(pp);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "bwd_prep_kernel launch");
  int rc = trace_mark(g_trace_begin, stream);
  if (rc != DILATTN_OK) return rc;
  // persistent: one CTA per SM, each taking units of the longest-first list from the counter
  p.units = units;
  const long long grid = std::min<long long>(units, (long long)st->num_sms);
  if (grid > 0)
    bwd_tile_kernel<<<(unsigned)grid, BwdCfg::THREADS, BwdCfg::SMEM_BYTES, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "bwd_tile_kernel launch");
  rc = trace_mark(g_trace_end, stream);
  if (rc != DILATTN_OK) return rc;
  const long long n4 = rows * D / 4;
  const long long cblocks = std::min<long long>((n4 + 255) / 256, (long long)st->num_sms * 16);
  bwd_convert_kernel<<<(unsigned)cblocks, 256, 0, stream>>>(
      n4, reinterpret_cast<const float4*>(dq_acc), reinterpret_cast<const float4*>(dk_acc),
      reinterpret_cast<const float4*>(dv_acc), reinterpret_cast<uint2*>(dq),
      reinterpret_cast<uint2*>(dk), reinterpret_cast<uint2*>(dv));
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "bwd_convert_kernel launch");
  return DILATTN_OK;
}

RowParams make_row_params(int B, int N, int H, int d, const int* w, const int* r, int npat,
                          int causal) {
  RowParams p;
  memset(&p, 0, sizeof(p));
  make_geoms(B, N, H, w, r, npat, p.pat);
  p.npat = npat;
  p.B = B;
  p.N = N;
  p.H = H;
  p.causal = causal;
  p.tau = (float)(1.0 / std::sqrt((double)d));
  return p;
}

}  // namespace
}  // namespace dil

using namespace dil;

extern "C" {

const char* dilattn_status_string(int status) {
  switch (status) {
    case DILATTN_OK: return "DILATTN_OK";
    case DILATTN_ERR_INVALID_ARG: return "DILATTN_ERR_INVALID_ARG";
    case DILATTN_ERR_UNSUPPORTED: return "DILATTN_ERR_UNSUPPORTED";
    case DILATTN_ERR_CUDA: return "DILATTN_ERR_CUDA";
    case DILATTN_ERR_WORKSPACE: return "DILATTN_ERR_WORKSPACE";
    case DILATTN_ERR_INTERNAL: return "DILATTN_ERR_INTERNAL";
    default: return "DILATTN_UNKNOWN_STATUS";
  }
}

const char* dilattn_last_error(void) { return g_last_error; }

size_t dilattn_fwd_workspace_size(int B, int N, int H, int d, const int* w, const int* r,
                                  int npat) {
  if (check_shape(B, N, H, d, w, r, npat, 1) != DILATTN_OK) return 0;
  PatternGeom geo[kMaxPat];
  const long long rows = make_geoms(B, N, H, w, r, npat, geo);
  return align256((size_t)rows * d * 4) + align256((size_t)rows * 4) +
         align256((size_t)B * N * H * d * 4);
}

int dilattn_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int N,
                int H, int d, const int* w, const int* r, int npat, int causal, void* workspace,
                size_t workspace_bytes, cudaStream_t stream) {
  int rc = check_shape(B, N, H, d, w, r, npat, causal);
  if (rc != DILATTN_OK) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return DILATTN_ERR_INVALID_ARG;
  if (lse != nullptr && !aligned16(lse)) return DILATTN_ERR_INVALID_ARG;
  const size_t tb = (size_t)B * N * H * d * 2;
  if (overlaps(out, tb, q, tb) || overlaps(out, tb, k, tb) || overlaps(out, tb, v, tb))
    return DILATTN_ERR_INVALID_ARG;
  if (lse != nullptr) {
    const size_t lb = (size_t)B * H * N * 4;
    if (overlaps(lse, lb, q, tb) || overlaps(lse, lb, k, tb) || overlaps(lse, lb, v, tb) ||
        overlaps(lse, lb, out, tb))
      return DILATTN_ERR_INVALID_ARG;
  }
  if (d != 64 && d != 128) return DILATTN_ERR_UNSUPPORTED;
  const size_t need = dilattn_fwd_workspace_size(B, N, H, d, w, r, npat);
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255) != 0 ||
      workspace_bytes < need)
    return DILATTN_ERR_WORKSPACE;
  DeviceState* st = nullptr;
  rc = device_state(&st);
  if (rc != DILATTN_OK) return rc;
  if (d == 64)
    return launch_fwd<64>(q, k, v, out, lse, B, N, H, w, r, npat, causal, workspace, st, stream);
  return launch_fwd<128>(q, k, v, out, lse, B, N, H, w, r, npat, causal, workspace, st, stream);
}

size_t dilattn_bwd_workspace_size(int B, int N, int H, int d, const int* w, const int* r,
                                  int npat) {
  if (check_shape(B, N, H, d, w, r, npat, 1) != DILATTN_OK) return 0;
  const size_t t = (size_t)B * N * H * d * 4;
  return 3 * align256(t) + align256((size_t)B * H * N * 4) + 256;  // + the unit counter
}

int dilattn_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse,
                const void* dout, void* dq, void* dk, void* dv, int B, int N, int H, int d,
                const int* w, const int* r, int npat, int causal, const void* fwd_workspace,
                size_t fwd_workspace_bytes, void* workspace, size_t workspace_bytes,
                cudaStream_t stream) {
  int rc = check_shape(B, N, H, d, w, r, npat, causal);
  if (rc != DILATTN_OK) return rc;
  const void* ins[6] = {q, k, v, out, lse, dout};
  for (const void* x : ins)
    if (!aligned16(x)) return DILATTN_ERR_INVALID_ARG;
  if (!aligned16(dq) || !aligned16(dk) || !aligned16(dv)) return DILATTN_ERR_INVALID_ARG;
  const size_t tb = (size_t)B * N * H * d * 2;
  const size_t lb = (size_t)B * H * N * 4;
  void* outs[3] = {dq, dk, dv};
  for (void* o : outs)
    for (int j = 0; j < 6; ++j)
      if (overlaps(o, tb, ins[j], j == 4 ? lb : tb)) return DILATTN_ERR_INVALID_ARG;
  if (overlaps(dq, tb, dk, tb) || overlaps(dq, tb, dv, tb) || overlaps(dk, tb, dv, tb))
    return DILATTN_ERR_INVALID_ARG;
  if (d != 64) {
    snprintf(g_last_error, sizeof(g_last_error), "bf16 backward is built for d = 64");
    return DILATTN_ERR_UNSUPPORTED;
  }
  const size_t need = dilattn_bwd_workspace_size(B, N, H, d, w, r, npat);
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255) != 0 ||
      workspace_bytes < need)
    return DILATTN_ERR_WORKSPACE;
  DeviceState* st = nullptr;
  rc = device_state(&st);
  if (rc != DILATTN_OK) return rc;
  const float* out_f32 = nullptr;
  if (fwd_workspace != nullptr) {
    if ((reinterpret_cast<uintptr_t>(fwd_workspace) & 255) != 0 ||
        fwd_workspace_bytes < dilattn_fwd_workspace_size(B, N, H, d, w, r, npat))
      return DILATTN_ERR_WORKSPACE;
    PatternGeom geo[kMaxPat];
    const long long rows = make_geoms(B, N, H, w, r, npat, geo);
    out_f32 = fwd_out_f32(const_cast<void*>(fwd_workspace), rows, d);
    if (overlaps(fwd_workspace, fwd_workspace_bytes, workspace, workspace_bytes))
      return DILATTN_ERR_INVALID_ARG;
  }
  return launch_bwd(q, k, v, out, lse, dout, dq, dk, dv, B, N, H, w, r, npat, causal, out_f32,
                    workspace, st, stream);
}

int dilattn_fwd_f32(const float* q, const float* k, const float* v, float* out, float* lse, int B,
                    int N, int H, int d, const int* w, const int* r, int npat, int causal,
                    cudaStream_t stream) {
  int rc = check_shape(B, N, H, d, w, r, npat, causal);
  if (rc != DILATTN_OK) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return DILATTN_ERR_INVALID_ARG;
  if (lse != nullptr && !aligned16(lse)) return DILATTN_ERR_INVALID_ARG;
  const size_t tb = (size_t)B * N * H * d * 4;
  if (overlaps(out, tb, q, tb) || overlaps(out, tb, k, tb) || overlaps(out, tb, v, tb))
    return DILATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return DILATTN_ERR_UNSUPPORTED;
  DeviceState* st = nullptr;
  rc = device_state(&st);
  if (rc != DILATTN_OK) return rc;
  RowParams p = make_row_params(B, N, H, d, w, r, npat, causal);
  const long long rows = (long long)B * N * H;
  const unsigned blocks = (unsigned)((rows + 127) / 128);
  if (d == 64)
    fwd_f32_kernel<64><<<blocks, 128, 0, stream>>>(p, q, k, v, out, lse);
  else
    fwd_f32_kernel<128><<<blocks, 128, 0, stream>>>(p, q, k, v, out, lse);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fwd_f32_kernel launch");
  return DILATTN_OK;
}

int dilattn_bwd_f32(const float* q, const float* k, const float* v, const float* out,
                    const float* lse, const float* dout, float* dq, float* dk, float* dv, int B,
                    int N, int H, int d, const int* w, const int* r, int npat, int causal,
                    cudaStream_t stream) {
  int rc = check_shape(B, N, H, d, w, r, npat, causal);
  if (rc != DILATTN_OK) return rc;
  const void* ins[6] = {q, k, v, out, lse, dout};
  for (const void* x : ins)
    if (!aligned16(x)) return DILATTN_ERR_INVALID_ARG;
  if (!aligned16(dq) || !aligned16(dk) || !aligned16(dv)) return DILATTN_ERR_INVALID_ARG;
  const size_t tb = (size_t)B * N * H * d * 4;
  const size_t lb = (size_t)B * H * N * 4;
  void* outs[3] = {dq, dk, dv};
  for (void* o : outs) {
    for (int j = 0; j < 6; ++j)
      if (overlaps(o, tb, ins[j], j == 4 ? lb : tb)) return DILATTN_ERR_INVALID_ARG;
  }
  if (overlaps(dq, tb, dk, tb) || overlaps(dq, tb, dv, tb) || overlaps(dk, tb, dv, tb))
    return DILATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return DILATTN_ERR_UNSUPPORTED;
  DeviceState* st = nullptr;
  rc = device_state(&st);
  if (rc != DILATTN_OK) return rc;
  RowParams p = make_row_params(B, N, H, d, w, r, npat, causal);
  const long long rows = (long long)B * N * H;
  const unsigned blocks = (unsigned)((rows + 127) / 128);
  if (d == 64) {
    bwd_dq_f32_kernel<64><<<blocks, 128, 0, stream>>>(p, q, k, v, out, lse, dout, dq);
    bwd_dkdv_f32_kernel<64><<<blocks, 128, 0, stream>>>(p, q, k, v, out, lse, dout, dk, dv);
  } else {
    bwd_dq_f32_kernel<128><<<blocks, 128, 0, stream>>>(p, q, k, v, out, lse, dout, dq);
    bwd_dkdv_f32_kernel<128><<<blocks, 128, 0, stream>>>(p, q, k, v, out, lse, dout, dk, dv);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "bwd_f32 launch");
  return DILATTN_OK;
}

int dilattn_selection(uint32_t* sig, int N, int H, const int* w, const int* r, int npat,
                      cudaStream_t stream) {
  int rc = check_shape(1, N, H, 1, w, r, npat, 1);
  if (rc != DILATTN_OK) return rc;
  if (!aligned16(sig)) return DILATTN_ERR_INVALID_ARG;
  DeviceState* st = nullptr;
  rc = device_state(&st);
  if (rc != DILATTN_OK) return rc;
  PatternGeom geo[kMaxPat];
  make_geoms(1, N, H, w, r, npat, geo);
  cudaError_t e = cudaMemsetAsync(sig, 0, (size_t)H * N * 4, stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  for (int i = 0; i < npat; ++i) {
    const long long gx = (long long)geo[i].nseg * H;
    if (gx > 0x7fffffffLL) return DILATTN_ERR_UNSUPPORTED;
    const int gy = std::min(64, (geo[i].nmax + 255) / 256);
    selection_kernel<<<dim3((unsigned)gx, gy), 256, 0, stream>>>(geo[i], i, N, H, sig);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "selection_kernel launch");
  return DILATTN_OK;
}

int dilattn_set_trace_events(cudaEvent_t tile_begin, cudaEvent_t tile_end) {
  if ((tile_begin == nullptr) != (tile_end == nullptr)) return DILATTN_ERR_INVALID_ARG;
  g_trace_begin = tile_begin;
  g_trace_end = tile_end;
  return DILATTN_OK;
}

int dilattn_device_error(cudaStream_t stream, int* code) {
  if (code == nullptr) return DILATTN_ERR_INVALID_ARG;
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc != DILATTN_OK) return rc;
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int v = 0;
  e = cudaMemcpy(&v, st->err_word, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy");
  const int zero = 0;
  e = cudaMemcpy(st->err_word, &zero, sizeof(int), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy");
  *code = v & 0xff;  // the word holds (launch tag << 8) | code
  return DILATTN_OK;
}

int dilattn_selftest_wait_timeout(unsigned long long limit_ns, int* result, cudaStream_t stream) {
  if (result == nullptr || !aligned16(result) || limit_ns == 0 || limit_ns > 1000000000ull)
    return DILATTN_ERR_INVALID_ARG;
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc != DILATTN_OK) return rc;
  selftest_wait_kernel<<<1, 64, 0, stream>>>(ErrCtx{st->err_word, next_tag()}, limit_ns, result);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "selftest_wait_kernel launch");
  return DILATTN_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Forward with a scratch array compiled into the library (no allocation)
// ---------------------------------------------------------------------------
namespace dil {

// Scratch of dilattn_fwd_noalloc. In host code this name is only a stand-in
// for the device array: kernels get the address cudaGetSymbolAddress returns.
static __device__ __align__(256) unsigned char g_noalloc_scratch[DILATTN_NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_noalloc_mu;
std::map<int, void*> g_noalloc_addr;  // device ordinal -> device address of the scratch

// Device address of the scratch on the current device, looked up once per device.
int noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  auto it = g_noalloc_addr.find(dev);
  if (it == g_noalloc_addr.end()) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(g_noalloc_scratch)");
    it = g_noalloc_addr.emplace(dev, ptr).first;
  }
  *out = it->second;
  return DILATTN_OK;
}
}  // namespace
}  // namespace dil

extern "C" int dilattn_fwd_noalloc(const void* q, const void* k, const void* v, void* out,
                                   float* lse, int B, int N, int H, int d, const int* w,
                                   const int* r, int npat, int causal, cudaStream_t stream) {
  int rc = check_shape(B, N, H, d, w, r, npat, causal);
  if (rc != DILATTN_OK) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return DILATTN_ERR_INVALID_ARG;
  if (lse != nullptr && !aligned16(lse)) return DILATTN_ERR_INVALID_ARG;
  const size_t tb = (size_t)B * N * H * d * 2;
  if (overlaps(out, tb, q, tb) || overlaps(out, tb, k, tb) || overlaps(out, tb, v, tb))
    return DILATTN_ERR_INVALID_ARG;
  if (lse != nullptr) {
    const size_t lb = (size_t)B * H * N * 4;
    if (overlaps(lse, lb, q, tb) || overlaps(lse, lb, k, tb) || overlaps(lse, lb, v, tb) ||
        overlaps(lse, lb, out, tb))
      return DILATTN_ERR_INVALID_ARG;
  }
  if (d != 64 && d != 128) return DILATTN_ERR_UNSUPPORTED;
  const size_t need = dilattn_fwd_workspace_size(B, N, H, d, w, r, npat);
  if (need > (size_t)DILATTN_NOALLOC_SCRATCH_BYTES) {
    snprintf(g_last_error, sizeof(g_last_error),
             "dilattn_fwd_noalloc: this problem needs %zu bytes of scratch; the built-in "
             "scratch holds %zu bytes (use dilattn_fwd with a workspace)",
             need, (size_t)DILATTN_NOALLOC_SCRATCH_BYTES);
    return DILATTN_ERR_WORKSPACE;
  }
  DeviceState* st = nullptr;
  rc = device_state(&st);
  if (rc != DILATTN_OK) return rc;
  void* scratch = nullptr;
  rc = noalloc_scratch(&scratch);
  if (rc != DILATTN_OK) return rc;
  if (d == 64)
    return launch_fwd<64>(q, k, v, out, lse, B, N, H, w, r, npat, causal, scratch, st, stream);
  return launch_fwd<128>(q, k, v, out, lse, B, N, H, w, r, npat, causal, scratch, st, stream);
}
