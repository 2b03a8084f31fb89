// libdilattn: C-ABI entry points (validation, TMA descriptor set-up, launches).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

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
  int dev = 0;
  cudaMemPool_t pool = nullptr;  // the forward's scratch pool, created on first use
};

std::mutex g_mu;
std::map<int, DeviceState> g_devices;

int device_state(DeviceState** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState& st = g_devices[dev];
  st.dev = dev;
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
      e = cudaFuncSetAttribute(fwd_tile_kernel<128, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               FwdCfg<128, true>::SMEM_BYTES);
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

// Stream-ordered memory pool of the device for the forward's scratch. Freed
// blocks stay in the pool (release threshold: never), so after the first call
// of a given size the forward maps no new memory.
int scratch_pool(DeviceState* st, cudaMemPool_t* out) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (st->pool == nullptr) {
    cudaMemPoolProps props;
    memset(&props, 0, sizeof(props));
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = st->dev;
    cudaMemPool_t pool = nullptr;
    cudaError_t e = cudaMemPoolCreate(&pool, &props);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemPoolCreate");
    uint64_t keep = ~0ull;
    e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemPoolSetAttribute");
    st->pool = pool;
  }
  *out = st->pool;
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
  const int esz = f32 == 1 ? 4 : f32 == 3 ? 1 : 2;  // f32: 0 bf16, 1 fp32, 2 fp16, 3 e4m3
  const long long rowb = (long long)H * d * esz;
  cuuint64_t dims[5] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)(tail ? nmod : r),
                        (cuuint64_t)(tail ? nfloor + 1 : nfloor), (cuuint64_t)B};
  cuuint64_t strides[4] = {(cuuint64_t)d * esz, (cuuint64_t)rowb, (cuuint64_t)(rowb * r),
                           (cuuint64_t)(rowb * N)};
  cuuint32_t box[5] = {(cuuint32_t)(128 / esz), 1, 1, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUtensorMap m;
  const CUtensorMapDataType dt = f32 == 1 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                 : f32 == 2 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                 : f32 == 3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                            : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUresult cr = g_encode(&m, dt, 5, const_cast<void*>(ptr), dims,
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

// View of a gathered dilated buffer [ranks][B][rank_rows][H][d] bf16 whose
// row j of head h is dilated row j of that head's segment: dims
// {d, H, rank_rows, ranks, B}; a box of box_rows (64 or 128) rows never
// crosses a rank's block (rank_rows is a multiple of 128).
int gathered_map(const void* ptr, int B, int H, int d, int rank_rows, int ranks, CUtensorMap* out,
                 int box_rows = BM) {
  MapKey key{ptr, B, rank_rows, H, d, -ranks, 2, 0, box_rows};
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
  const cuuint64_t rowb = (cuuint64_t)H * d * 2;
  cuuint64_t dims[5] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)rank_rows, (cuuint64_t)ranks,
                        (cuuint64_t)B};
  cuuint64_t strides[4] = {(cuuint64_t)d * 2, rowb, rowb * rank_rows * B, rowb * rank_rows};
  cuuint32_t box[5] = {64, 1, (cuuint32_t)box_rows, 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUtensorMap m;
  CUresult cr = g_encode(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(ptr), dims,
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

// One sequence-parallel rank's per-pattern inputs (see FwdParams): patterns
// with kv_rows > 0 take K and V from the gathered buffers kg, vg.
struct SeqParPlan {
  int kv_rows[kMaxPat];
  int kv_rank_rows[kMaxPat];
  int ranks[kMaxPat];
  int toff[kMaxPat];
  const void* kg[kMaxPat];
  const void* vg[kMaxPat];
};

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

// Pattern geometry and partial-buffer layout. Pattern `skip` (the merging
// pattern, or -1) stores no partials and gets no rows. Returns the partial rows.
// Argument checks shared by the forward entry points.
int check_fwd_args(const void* q, const void* k, const void* v, const void* out, const float* lse,
                   int B, int N, int H, int d, const int* w, const int* r, int npat, int causal) {
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
  return DILATTN_OK;
}

long long make_geoms(int B, int N, int H, const int* w, const int* r, int npat,
                     PatternGeom* geo, int skip = -1) {
  long long rows = 0;
  for (int i = 0; i < npat; ++i) {
    PatternGeom& g = geo[i];
    g.w = w[i];
    g.r = r[i];
    divisor_magic((uint32_t)w[i], g.w_mul, g.w_sh);
    divisor_magic((uint32_t)r[i], g.r_mul, g.r_sh);
    g.nseg = (int)(((long long)N + w[i] - 1) / w[i]);
    const long long span = std::min<long long>(w[i], N);
    g.nmax = (int)((span + r[i] - 1) / r[i]);
    g.ntiles = (g.nmax + BM - 1) / BM;
    g.pstride = g.ntiles * BM;
    g.nmod = N % r[i];
    g.part_base = rows;
    if (i != skip) rows += (long long)B * H * g.nseg * g.pstride;
  }
  return rows;
}

// The merging pattern: one with r = 1 keeps every row of every head, so its
// tiles can finish the merge of all patterns. The shortest such pattern is
// taken (its tiles are the shortest, which keeps the end of the launch short).
int pick_merger(const int* w, const int* r, int npat) {
  int m = -1;
  for (int i = 0; i < npat; ++i)
    if (r[i] == 1 && (m < 0 || w[i] < w[m])) m = i;
  return m;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Longest-first unit order for the tile kernels (see Sched).
long long make_schedule(const PatternGeom* pat, int npat, int B, int H, Sched& sc,
                        unsigned include = 0xffffffffu) {
  std::vector<int> order;
  for (int i = 0; i < npat; ++i)
    if (include >> i & 1u) order.push_back(i);
  const int nsel = (int)order.size();
  memset(&sc, 0, sizeof(sc));
  if (nsel == 0) return 0;
  std::stable_sort(order.begin(), order.end(),
                   [&](int a, int b) { return pat[a].ntiles > pat[b].ntiles; });
  std::vector<int> vals;
  for (int i : order)
    if (vals.empty() || vals.back() != pat[i].ntiles) vals.push_back(pat[i].ntiles);
  for (int i = 0; i < nsel; ++i) sc.order[i] = order[i];
  sc.nband = (int)vals.size();
  sc.start[0] = 0;
  for (int j = 0; j < sc.nband; ++j) {
    const int lo = j + 1 < sc.nband ? vals[j + 1] : 0;
    sc.nt[j] = vals[j];
    int act = 0;
    long long per = 0;
    for (int a = 0; a < nsel; ++a) {
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

// Forward scratch: [rows][d] fp32 partial outputs, [rows] fp32 partial lse,
// one flag per 128-row block of partials, and the ticket counter.
struct FwdScratch {
  size_t o_bytes, lse_bytes, flag_bytes;
  size_t total() const { return o_bytes + lse_bytes + flag_bytes; }
};
FwdScratch fwd_scratch_layout(long long rows, int d) {
  FwdScratch f;
  f.o_bytes = align256((size_t)rows * d * 4);
  f.lse_bytes = align256((size_t)rows * 4);
  f.flag_bytes = align256((size_t)(rows / BM + 1) * 4 + 8);  // flags, the ticket and done counters
  return f;
}

size_t fwd_scratch_bytes(int B, int N, int H, int d, const int* w, const int* r, int npat) {
  PatternGeom geo[kMaxPat];
  const long long rows = make_geoms(B, N, H, w, r, npat, geo, pick_merger(w, r, npat));
  return fwd_scratch_layout(rows, d).total();
}

// A named host-side range for profilers (NVTX; a no-op unless a tool is
// attached), around each launch sequence.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

template <int D, bool QK8 = false>
int launch_fwd(const void* q, const void* k, const void* v, void* out, void* out_res, float* lse,
               int B, int N, int H, const int* w, const int* r, int npat, int causal, void* ws,
               DeviceState* st, cudaStream_t stream, const SeqParPlan* sp = nullptr,
               float qk_scale = 1.f) {
  static_assert(sizeof(FwdParams) < 32000, "kernel parameter block too large");
  NvtxRange range(QK8 ? "dilattn forward (e4m3 q, k)" : sp != nullptr ? "dilattn forward (sequence-parallel rank)"
                                                                        : "dilattn forward");
  FwdParams p;
  memset(&p, 0, sizeof(p));
  p.npat = npat;
  p.B = B;
  p.N = N;
  p.H = H;
  p.causal = causal;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D) * (double)qk_scale);
  p.merger = pick_merger(w, r, npat);
  const long long rows = make_geoms(B, N, H, w, r, npat, p.pat, p.merger);
  const FwdScratch lay = fwd_scratch_layout(rows, D);
  char* wsb = reinterpret_cast<char*>(ws);
  p.part_o = reinterpret_cast<float*>(wsb);
  p.part_lse = reinterpret_cast<float*>(wsb + lay.o_bytes);
  p.flags = reinterpret_cast<int*>(wsb + lay.o_bytes + lay.lse_bytes);
  p.counter = p.flags + rows / BM + 1;
  p.done = p.counter + 1;
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.out_res = reinterpret_cast<__nv_bfloat16*>(out_res);
  p.lse = lse;
  p.err = ErrCtx{st->err_word, next_tag()};
  for (int i = 0; i < npat; ++i) {
    const void* src[3] = {q, k, v};
    const int dtype[3] = {QK8 ? 3 : 0, QK8 ? 3 : 0, 0};
    CUtensorMap* dst[3] = {&p.tmq[i], &p.tmk[i], &p.tmv[i]};
    CUtensorMap* dst_t[3] = {&p.tmq_t[i], &p.tmk_t[i], &p.tmv_t[i]};
    // Q tiles are BM rows; K and V tiles the kernel's key-tile rows
    constexpr int kbn = FwdCfg<D, QK8>::BN;
    for (int j = 0; j < 3; ++j) {
      const int rows = j == 0 ? BM : kbn;
      int rc = strided_map(src[j], B, N, H, D, r[i], 0, dst[j], dtype[j], rows);
      if (rc == DILATTN_OK) rc = strided_map(src[j], B, N, H, D, r[i], 1, dst_t[j], dtype[j], rows);
      if (rc != DILATTN_OK) return rc;
    }
    if (sp != nullptr && sp->kv_rows[i] > 0) {
      p.kv_rows[i] = sp->kv_rows[i];
      p.kv_rank_rows[i] = sp->kv_rank_rows[i];
      p.toff[i] = sp->toff[i];
      int rc = gathered_map(sp->kg[i], B, H, D, sp->kv_rank_rows[i], sp->ranks[i], &p.tmk[i], kbn);
      if (rc == DILATTN_OK)
        rc = gathered_map(sp->vg[i], B, H, D, sp->kv_rank_rows[i], sp->ranks[i], &p.tmv[i], kbn);
      if (rc != DILATTN_OK) return rc;
    }
  }
  const unsigned all = (1u << npat) - 1u;
  const unsigned mbit = p.merger >= 0 ? (1u << p.merger) : 0u;
  p.units_p = make_schedule(p.pat, npat, B, H, p.sched, all & ~mbit);
  const long long units_m = mbit ? make_schedule(p.pat, npat, B, H, p.sched_m, mbit) : 0;
  const long long units = p.units_p + units_m;
  if (units > 0x7fffffffLL) return DILATTN_ERR_UNSUPPORTED;
  cudaError_t e = cudaMemsetAsync(p.flags, 0, lay.flag_bytes, stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  int rc = trace_mark(g_trace_begin, stream);
  if (rc != DILATTN_OK) return rc;
  if (units > 0)
    fwd_tile_kernel<D, QK8>
        <<<(unsigned)units, FwdCfg<D, QK8>::THREADS, FwdCfg<D, QK8>::SMEM_BYTES, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fwd_tile_kernel launch");
  rc = trace_mark(g_trace_end, stream);
  if (rc != DILATTN_OK) return rc;
  if (p.merger >= 0) return DILATTN_OK;

  // No pattern keeps every row: a separate pass merges the partials.
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
  mp.out_res = reinterpret_cast<__nv_bfloat16*>(out_res);
  mp.lse = lse;
  const long long total_rows = (long long)B * N * H;
  constexpr int rows_per_block = 256 / kMergeTpr;
  const long long blocks = (total_rows + rows_per_block - 1) / rows_per_block;
  merge_kernel<D><<<(unsigned)blocks, 256, 0, stream>>>(mp);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "merge_kernel launch");
  return DILATTN_OK;
}

int launch_bwd(const void* q, const void* k, const void* v, const void* out, const void* out_res,
               const float* lse, const void* dout, float* dq, float* dk, float* dv, int B, int N,
               int H,
               const int* w, const int* r, int npat, int causal, void* ws,
               DeviceState* st, cudaStream_t stream) {
  NvtxRange range("dilattn backward");
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
  // workspace: D [B][H][N] fp32, 256 bytes for the key-tile kernel's unit
  // counter, then fp16 copies of q and k
  char* wsb = reinterpret_cast<char*>(ws);
  float* drow = reinterpret_cast<float*>(wsb);
  p.drow = drow;
  p.lse = lse;
  const size_t dbytes = align256((size_t)B * H * N * 4);
  p.counter = reinterpret_cast<int*>(wsb + dbytes);
  __half* q16 = reinterpret_cast<__half*>(wsb + dbytes + 256);
  __half* k16 = reinterpret_cast<__half*>(wsb + dbytes + 256 + align256((size_t)B * N * H * D * 2));
  p.err = ErrCtx{st->err_word, next_tag()};
  for (int i = 0; i < npat; ++i) {
    const void* src[4] = {q16, k16, v, dout};
    const int dtype[4] = {2, 2, 0, 0};
    CUtensorMap* dst[4] = {&p.tmq[i], &p.tmk[i], &p.tmv[i], &p.tmdo[i]};
    CUtensorMap* dst_t[4] = {&p.tmq_t[i], &p.tmk_t[i], &p.tmv_t[i], &p.tmdo_t[i]};
    for (int j = 0; j < 4; ++j) {
      int rc = strided_map(src[j], B, N, H, D, r[i], 0, dst[j], dtype[j]);
      if (rc == DILATTN_OK) rc = strided_map(src[j], B, N, H, D, r[i], 1, dst_t[j], dtype[j]);
      if (rc != DILATTN_OK) return rc;
    }
    // reduce-add targets: one row warp adds a 32-row x 32-column block
    const float* grad[3] = {dq, dk, dv};
    CUtensorMap* gm[3] = {&p.tmdq[i], &p.tmdk[i], &p.tmdv[i]};
    CUtensorMap* gm_t[3] = {&p.tmdq_t[i], &p.tmdk_t[i], &p.tmdv_t[i]};
    for (int j = 0; j < 3; ++j) {
      int rc = strided_map(grad[j], B, N, H, D, r[i], 0, gm[j], 1, 32);
      if (rc == DILATTN_OK) rc = strided_map(grad[j], B, N, H, D, r[i], 1, gm_t[j], 1, 32);
      if (rc != DILATTN_OK) return rc;
    }
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

  PrepParams pp;
  pp.B = B;
  pp.N = N;
  pp.H = H;
  pp.q = reinterpret_cast<const __nv_bfloat16*>(q);
  pp.k = reinterpret_cast<const __nv_bfloat16*>(k);
  pp.q16 = q16;
  pp.k16 = k16;
  pp.err = p.err;
  pp.out = reinterpret_cast<const __nv_bfloat16*>(out);
  pp.out_res = reinterpret_cast<const __nv_bfloat16*>(out_res);
  pp.dout = reinterpret_cast<const __nv_bfloat16*>(dout);
  pp.drow = drow;
  pp.dq = dq;
  pp.dk = dk;
  pp.dv = dv;
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
  return trace_mark(g_trace_end, stream);
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

size_t dilattn_fwd_scratch_size(int B, int N, int H, int d, const int* w, const int* r,
                                int npat) {
  if (check_shape(B, N, H, d, w, r, npat, 1) != DILATTN_OK) return 0;
  return fwd_scratch_bytes(B, N, H, d, w, r, npat);
}

}  // extern "C"

namespace dil {
namespace {
// dilattn_fwd and dilattn_fwd_train: scratch from the library's pool.
int fwd_pooled(const void* q, const void* k, const void* v, void* out, void* out_res, float* lse,
               int B, int N, int H, int d, const int* w, const int* r, int npat, int causal,
               cudaStream_t stream) {
  int rc = check_fwd_args(q, k, v, out, lse, B, N, H, d, w, r, npat, causal);
  if (rc != DILATTN_OK) return rc;
  if (out_res != nullptr) {
    const size_t tb = (size_t)B * N * H * d * 2;
    if (!aligned16(out_res) || overlaps(out_res, tb, q, tb) || overlaps(out_res, tb, k, tb) ||
        overlaps(out_res, tb, v, tb) || overlaps(out_res, tb, out, tb) ||
        (lse != nullptr && overlaps(out_res, tb, lse, (size_t)B * H * N * 4)))
      return DILATTN_ERR_INVALID_ARG;
  }
  DeviceState* st = nullptr;
  rc = device_state(&st);
  if (rc != DILATTN_OK) return rc;
  cudaMemPool_t pool = nullptr;
  rc = scratch_pool(st, &pool);
  if (rc != DILATTN_OK) return rc;
  const size_t need = fwd_scratch_bytes(B, N, H, d, w, r, npat);
  void* scratch = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(&scratch, need, pool, stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMallocFromPoolAsync (forward scratch)");
  rc = d == 64 ? launch_fwd<64>(q, k, v, out, out_res, lse, B, N, H, w, r, npat, causal, scratch,
                                st, stream)
               : launch_fwd<128>(q, k, v, out, out_res, lse, B, N, H, w, r, npat, causal, scratch,
                                 st, stream);
  e = cudaFreeAsync(scratch, stream);  // stream-ordered: after the kernels that use it
  if (rc == DILATTN_OK && e != cudaSuccess) return cuda_fail(e, "cudaFreeAsync (forward scratch)");
  return rc;
}
}  // namespace
}  // namespace dil

extern "C" {

int dilattn_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int N,
                int H, int d, const int* w, const int* r, int npat, int causal,
                cudaStream_t stream) {
  return fwd_pooled(q, k, v, out, nullptr, lse, B, N, H, d, w, r, npat, causal, stream);
}

int dilattn_fwd_fp8(const void* q8, const void* k8, const void* v, void* out, float* lse, int B,
                    int N, int H, int d, const int* w, const int* r, int npat, int causal,
                    float q_scale, float k_scale, cudaStream_t stream) {
  int rc = check_shape(B, N, H, d, w, r, npat, causal);
  if (rc != DILATTN_OK) return rc;
  if (d != 128) {
    snprintf(g_last_error, sizeof(g_last_error), "the fp8 forward is built for d = 128");
    return DILATTN_ERR_UNSUPPORTED;
  }
  if (!(q_scale > 0.f) || !(k_scale > 0.f) || !std::isfinite(q_scale) || !std::isfinite(k_scale))
    return DILATTN_ERR_INVALID_ARG;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v) || !aligned16(out) ||
      (lse != nullptr && !aligned16(lse)))
    return DILATTN_ERR_INVALID_ARG;
  const size_t t8 = (size_t)B * N * H * d, tb = 2 * t8, lb = (size_t)B * H * N * 4;
  if (overlaps(out, tb, q8, t8) || overlaps(out, tb, k8, t8) || overlaps(out, tb, v, tb) ||
      (lse != nullptr && (overlaps(lse, lb, q8, t8) || overlaps(lse, lb, k8, t8) ||
                          overlaps(lse, lb, v, tb) || overlaps(lse, lb, out, tb))))
    return DILATTN_ERR_INVALID_ARG;
  DeviceState* st = nullptr;
  rc = device_state(&st);
  if (rc != DILATTN_OK) return rc;
  cudaMemPool_t pool = nullptr;
  rc = scratch_pool(st, &pool);
  if (rc != DILATTN_OK) return rc;
  const size_t need = fwd_scratch_bytes(B, N, H, d, w, r, npat);
  void* scratch = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(&scratch, need, pool, stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMallocFromPoolAsync (forward scratch)");
  rc = launch_fwd<128, true>(q8, k8, v, out, nullptr, lse, B, N, H, w, r, npat, causal, scratch,
                             st, stream, nullptr, q_scale * k_scale);
  e = cudaFreeAsync(scratch, stream);
  if (rc == DILATTN_OK && e != cudaSuccess) return cuda_fail(e, "cudaFreeAsync (forward scratch)");
  return rc;
}

int dilattn_fwd_train(const void* q, const void* k, const void* v, void* out, void* out_res,
                      float* lse, int B, int N, int H, int d, const int* w, const int* r, int npat,
                      int causal, cudaStream_t stream) {
  if (out_res == nullptr) return DILATTN_ERR_INVALID_ARG;
  return fwd_pooled(q, k, v, out, out_res, lse, B, N, H, d, w, r, npat, causal, stream);
}

size_t dilattn_bwd_workspace_size(int B, int N, int H, int d) {
  if (B < 1 || N < 1 || H < 1 || d < 1 || (double)B * N * H * d >= 1099511627776.0) return 0;
  // D, the unit counter, then fp16 copies of q and k
  return align256((size_t)B * H * N * 4) + 256 + 2 * align256((size_t)B * N * H * d * 2);
}

int dilattn_bwd(const void* q, const void* k, const void* v, const void* out,
                const void* out_res, const float* lse, const void* dout, float* dq, float* dk,
                float* dv, int B, int N, int H, int d, const int* w, const int* r, int npat,
                int causal, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  int rc = check_shape(B, N, H, d, w, r, npat, causal);
  if (rc != DILATTN_OK) return rc;
  const void* ins[7] = {q, k, v, out, lse, dout, out_res};
  for (const void* x : ins)
    if (!aligned16(x)) return DILATTN_ERR_INVALID_ARG;
  if (!aligned16(dq) || !aligned16(dk) || !aligned16(dv)) return DILATTN_ERR_INVALID_ARG;
  const size_t tb = (size_t)B * N * H * d * 2;  // a bf16 input
  const size_t gb = 2 * tb;                     // an fp32 gradient
  const size_t lb = (size_t)B * H * N * 4;
  void* outs[3] = {dq, dk, dv};
  for (void* o : outs)
    for (int j = 0; j < 7; ++j)
      if (overlaps(o, gb, ins[j], j == 4 ? lb : tb)) return DILATTN_ERR_INVALID_ARG;
  if (overlaps(dq, gb, dk, gb) || overlaps(dq, gb, dv, gb) || overlaps(dk, gb, dv, gb))
    return DILATTN_ERR_INVALID_ARG;
  if (d != 64) {
    snprintf(g_last_error, sizeof(g_last_error), "bf16 backward is built for d = 64");
    return DILATTN_ERR_UNSUPPORTED;
  }
  const size_t need = dilattn_bwd_workspace_size(B, N, H, d);
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255) != 0 ||
      workspace_bytes < need)
    return DILATTN_ERR_WORKSPACE;
  for (int j = 0; j < 7; ++j)
    if (overlaps(workspace, need, ins[j], j == 4 ? lb : tb)) return DILATTN_ERR_INVALID_ARG;
  for (void* o : outs)
    if (overlaps(workspace, need, o, gb)) return DILATTN_ERR_INVALID_ARG;
  DeviceState* st = nullptr;
  rc = device_state(&st);
  if (rc != DILATTN_OK) return rc;
  return launch_bwd(q, k, v, out, out_res, lse, dout, dq, dk, dv, B, N, H, w, r, npat, causal,
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
  if (lse != nullptr) {
    const size_t lb = (size_t)B * H * N * 4;
    if (overlaps(lse, lb, q, tb) || overlaps(lse, lb, k, tb) || overlaps(lse, lb, v, tb) ||
        overlaps(lse, lb, out, tb))
      return DILATTN_ERR_INVALID_ARG;
  }
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

int dilattn_pack_dilated(const void* x, void* buf, int B, int L, int H, int d, int r,
                         cudaStream_t stream) {
  if (B < 1 || L < 1 || H < 1 || r < 1 || L % r != 0 || (d != 64 && d != 128))
    return DILATTN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(buf)) return DILATTN_ERR_INVALID_ARG;
  const size_t bytes = (size_t)B * L * H * d * 2;
  if (overlaps(x, bytes, buf, bytes / r)) return DILATTN_ERR_INVALID_ARG;
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc != DILATTN_OK) return rc;
  const long long n16 = (long long)B * (L / r) * H * (d / 8);  // 16-byte pieces
  const long long blocks = std::min<long long>((n16 + 255) / 256, (long long)st->num_sms * 32);
  pack_dilated_kernel<<<(unsigned)blocks, 256, 0, stream>>>(
      reinterpret_cast<const uint4*>(x), reinterpret_cast<uint4*>(buf), B, L, H, d / 8, r);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "pack_dilated_kernel launch");
  return DILATTN_OK;
}

int dilattn_fwd_seqpar(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                       int L, int H, int d, const int* w, const int* r, int npat, int causal,
                       int rank, int world, const void* const* kg, const void* const* vg,
                       cudaStream_t stream) {
  int rc = check_fwd_args(q, k, v, out, lse, B, L, H, d, w, r, npat, causal);
  if (rc != DILATTN_OK) return rc;
  if (world < 1 || rank < 0 || rank >= world || (long long)L * world > 0x7fffffffLL)
    return DILATTN_ERR_INVALID_ARG;
  const long long N = (long long)L * world;
  SeqParPlan sp;
  memset(&sp, 0, sizeof(sp));
  int wl[kMaxPat];
  for (int i = 0; i < npat; ++i) {
    if (w[i] <= L) {  // every segment lies in one rank's block
      if (L % w[i] != 0) return DILATTN_ERR_INVALID_ARG;
      wl[i] = w[i];
      continue;
    }
    const long long span = std::min<long long>(w[i], N);  // a segment spans span / L ranks
    if (span % L != 0 || (w[i] < N && N % w[i] != 0) || L % r[i] != 0 || (L / r[i]) % BM != 0)
      return DILATTN_ERR_INVALID_ARG;
    if (kg == nullptr || vg == nullptr || !aligned16(kg[i]) || !aligned16(vg[i]))
      return DILATTN_ERR_INVALID_ARG;
    wl[i] = L;  // this rank's kept rows: offset h mod r, stride r, over its whole block
    sp.ranks[i] = (int)(span / L);
    sp.kv_rank_rows[i] = L / r[i];
    sp.kv_rows[i] = sp.ranks[i] * sp.kv_rank_rows[i];
    sp.toff[i] = (rank % sp.ranks[i]) * (sp.kv_rank_rows[i] / BM);
    sp.kg[i] = kg[i];
    sp.vg[i] = vg[i];
    // the gathered rows are read while out and lse are written
    const size_t gb = (size_t)sp.kv_rows[i] * B * H * d * 2;
    const size_t tb = (size_t)B * L * H * d * 2, lb = (size_t)B * H * L * 4;
    if (overlaps(out, tb, kg[i], gb) || overlaps(out, tb, vg[i], gb) ||
        (lse != nullptr && (overlaps(lse, lb, kg[i], gb) || overlaps(lse, lb, vg[i], gb))))
      return DILATTN_ERR_INVALID_ARG;
  }
  DeviceState* st = nullptr;
  rc = device_state(&st);
  if (rc != DILATTN_OK) return rc;
  cudaMemPool_t pool = nullptr;
  rc = scratch_pool(st, &pool);
  if (rc != DILATTN_OK) return rc;
  const size_t need = fwd_scratch_bytes(B, L, H, d, wl, r, npat);
  void* scratch = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(&scratch, need, pool, stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMallocFromPoolAsync (forward scratch)");
  rc = d == 64
      ? launch_fwd<64>(q, k, v, out, nullptr, lse, B, L, H, wl, r, npat, causal, scratch, st,
                       stream, &sp)
      : launch_fwd<128>(q, k, v, out, nullptr, lse, B, L, H, wl, r, npat, causal, scratch, st,
                        stream, &sp);
  e = cudaFreeAsync(scratch, stream);
  if (rc == DILATTN_OK && e != cudaSuccess) return cuda_fail(e, "cudaFreeAsync (forward scratch)");
  return rc;
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
  int rc = check_fwd_args(q, k, v, out, lse, B, N, H, d, w, r, npat, causal);
  if (rc != DILATTN_OK) return rc;
  const size_t need = fwd_scratch_bytes(B, N, H, d, w, r, npat);
  if (need > (size_t)DILATTN_NOALLOC_SCRATCH_BYTES) {
    snprintf(g_last_error, sizeof(g_last_error),
             "dilattn_fwd_noalloc: this problem needs %zu bytes of scratch; the built-in "
             "scratch holds %zu bytes (use dilattn_fwd)",
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
    return launch_fwd<64>(q, k, v, out, nullptr, lse, B, N, H, w, r, npat, causal, scratch, st,
                          stream);
  return launch_fwd<128>(q, k, v, out, nullptr, lse, B, N, H, w, r, npat, causal, scratch, st,
                         stream);
}
