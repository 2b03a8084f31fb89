// Forward tile kernel: tcgen05 tensor cores, TMA-gathered dilated rows,
// fp32 online softmax; one CTA per (pattern, segment, batch, head, query tile).
//
// Each CTA runs causal softmax attention between 128 kept query rows of one
// pattern segment and the segment's kept key rows (the dilated, per-head
// offset rows of the LongNet method description: gptget.net summary of arXiv
// 2307.02486, "方法详解"). Kept rows are addressed by a 5-D TMA view of the
// [B][N][H][d] tensor, {d, H, r (phase), N/r, B}, so the stride-r gather
// happens inside the copy engine with no materialised copy. Each stride r
// has two views with the tensor's own base address: phases [0, r) over
// floor(N/r) rows, and phases [0, N mod r) over floor(N/r) + 1 rows; a tile
// at phase ph uses the second when ph < N mod r, so the view's bounds are
// exactly the rows below N and rows past N read as zeros. A CTA of the
// merging pattern (r = 1: it keeps every row) combines every pattern's result
// for its rows and writes out; the other patterns' CTAs write their
// normalised output O_i and log-sum-exp to an fp32 partial buffer for it
// (families with no r = 1 pattern combine them in a separate merge kernel).
//
// Warp roles (192 threads, two CTAs per SM at d = 64 and at d = 128):
//   warp 0      TMA producer: lane 0 loads the Q tile once, then the K ring;
//               lane 1 the V ring.
//   warp 1      TMEM allocator and MMA issuer (the whole warp runs the
//               loop, one elected lane issues each group):
//               S = Q K^T (SMEM x SMEM -> TMEM), O += P V (TMEM x SMEM -> TMEM).
//   warps 2..5  softmax: warp w takes TMEM lanes 32 (w % 4) .. + 31, one query
//               row per thread: fp32 row max (3-input max), P = exp2(S*scale - m)
//               with packed fp32x2 arithmetic and the exp2 on the MUFU unit, P
//               stored to TMEM as bf16, O rescaled in TMEM when the reference
//               max moves, epilogue.
// Rows are one per thread: at d = 64 the softmax, not the MMA, bounds a tile,
// so its issue slots are the budget every choice above is made against.
// Key tiles are 128 rows at d = 64 and 64 rows at d = 128, so that at both
// sizes two CTAs share an SM (99.6 KB of shared memory and 256 TMEM columns
// each). TMEM columns: S [0, BN), P [BN, 3 BN / 2) (bf16 pairs), O
// [3 BN / 2, 3 BN / 2 + D).
#pragma once

#include "common.cuh"

namespace dil {

struct FwdParams {
  CUtensorMap tmq[kMaxPat];   // phases [0, r), floor(N/r) rows
  CUtensorMap tmk[kMaxPat];
  CUtensorMap tmv[kMaxPat];
  CUtensorMap tmq_t[kMaxPat]; // phases [0, N mod r), floor(N/r) + 1 rows
  CUtensorMap tmk_t[kMaxPat];
  CUtensorMap tmv_t[kMaxPat];
  PatternGeom pat[kMaxPat];
  int npat, B, N, H, causal;
  float scale_log2;  // log2(e) / sqrt(d)
  Sched sched;       // tiles of every pattern that stores partials, longest first
  Sched sched_m;     // tiles of the merging pattern (r = 1), longest first, after those
  long long units_p; // units of `sched`
  int merger;        // index of the merging pattern, or -1 (a separate merge kernel combines)
  int* counter;      // ticket counter: the order in which CTAs take units (zero at launch)
  int* done;         // partial-storing units finished (zero at launch)
  int* flags;        // one per 128-row block of partial rows: nonzero once the block is stored
  float* part_o;     // [rows][D] normalised per-pattern outputs
  float* part_lse;   // [rows] natural-log lse of each pattern's partial
  __nv_bfloat16* out;      // [B][N][H][D]
  __nv_bfloat16* out_res;  // [B][N][H][D] bf16(O - out), the rounding residual; may be null
  float* lse;              // [B][H][N], may be null
  // Sequence-parallel rank (LongNet's distributed algorithm): for a pattern
  // whose segments span several ranks, K and V come from a gathered buffer
  // [ranks][B][kv_rank_rows][H][D] of every rank's dilated rows of the
  // segment (kv_rows = ranks * kv_rank_rows rows per head, a multiple of 128),
  // and this rank's query tiles start at key tile toff of that sequence.
  int kv_rows[kMaxPat];       // 0: K and V from the strided views of k, v
  int kv_rank_rows[kMaxPat];
  int toff[kMaxPat];
  ErrCtx err;  // device error word and this launch's tag
};

// Acquire load of a flag word (gpu scope).
__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_gpu(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Bounded wait for a partial block's flag, same limits as mbar_wait.
__device__ __forceinline__ bool wait_flag(const int* f, volatile int* abort, const ErrCtx& err) {
  if (ld_acquire_gpu(f) != 0) return true;
  const unsigned long long t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    __nanosleep(128);
    if (ld_acquire_gpu(f) != 0) return true;
    if ((it & 63u) == 0) {
      if (*abort) return false;
      if (err.raised()) {
        *abort = 1;
        return false;
      }
      if (globaltimer_ns() - t0 > 4000000000ull) {
        err.raise(kErrWaitTimeout);
        *abort = 1;
        return false;
      }
    }
  }
}

// Partial row of position n in pattern g for head h of slice bh (= b * H + h),
// or -1 when g does not keep n: segment n / w, kept iff rel = n - start -
// (h mod r) is a non-negative multiple of r, row rel / r of the segment's
// block. off = h mod r. The quotients use the patterns' reciprocal
// multipliers (udiv), so the lookup costs a few instructions per pattern.
__device__ __forceinline__ int partial_row(const PatternGeom& g, int n, int off, int bh) {
  const uint32_t seg = udiv((uint32_t)n, g.w_mul, g.w_sh);
  const int rel = n - (int)(seg * (uint32_t)g.w) - off;
  if (rel < 0) return -1;
  const uint32_t v = udiv((uint32_t)rel, g.r_mul, g.r_sh);
  if ((int)(v * (uint32_t)g.r) != rel) return -1;
  return (int)(g.part_base + ((long long)bh * g.nseg + seg) * g.pstride + v);
}

// QK8: q and k are e4m3 (one byte per element; the fp8 variant, d = 128):
// each of their rows is a single 128-byte chunk and S = Q K^T runs as
// kind::f8f6f4; V, P and O stay as in the bf16 kernel.
template <int D, bool QK8 = false>
struct FwdCfg {
  static constexpr int BN = (D == 128) ? 64 : 128;  // key rows per tile (MMA N of S = Q K^T)
  static constexpr int KCH = D / 64;                 // 128-byte chunks of a bf16 row (V)
  static constexpr int KCH_QK = QK8 ? D / 128 : D / 64;  // 128-byte chunks of a Q or K row
  static constexpr int KST = (D == 128) ? 2 : 3;     // K ring depth (a stage frees after its S MMA)
  static constexpr int VST = 2;                      // V ring depth (a stage frees after its PV MMA)
  static constexpr int Q_CHUNK = BM * 128;           // one 128-byte column chunk of the Q tile
  static constexpr int KV_CHUNK = BN * 128;          // ... of a K or V tile
  static constexpr int Q_BYTES = KCH_QK * Q_CHUNK;
  static constexpr int K_BYTES = KCH_QK * KV_CHUNK;
  static constexpr int V_BYTES = KCH * KV_CHUNK;
  static constexpr int QK_COLS = QK8 ? 128 : 64;     // elements of a 128-byte chunk of Q or K
  static constexpr int S_KSTEPS = QK8 ? D / 32 : D / 16;  // MMA K steps of S (32 bytes each)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + KST * K_BYTES;
  static constexpr int OFF_BAR = OFF_V + VST * V_BYTES;
  static constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;  // + alignment slack
  static constexpr int TM_S = 0, TM_P = BN, TM_O = BN + BN / 2;
  static constexpr int TMEM_COLS = (TM_O + D <= 256) ? 256 : 512;
  static constexpr int MIN_BLOCKS = (TMEM_COLS == 256) ? 2 : 1;
  static constexpr int SM_WARPS = 4;             // softmax warps: one query row per thread
  static constexpr int THREADS = 64 + 32 * SM_WARPS;
};

// Epilogue of a tile of the merging pattern (r = 1, so it keeps every row):
// the tile's own online softmax (O in TMEM relative to m_run, sum l_run, in
// log2 units) is combined with the stored partials (O_i normalised, lse_i)
// of every other pattern that keeps the row, weighting each by its share of
// the shared denominator: O = sum_i Z_i O_i / sum_i Z_i, lse = log sum_i Z_i.
// One thread per row; out is written once, in bf16 (and, for training, the
// bf16 rounding residual of out, so that the backward's D = dO . O keeps
// fp32-grade accuracy).

struct MergeWeights {
  float M;                // the largest of the row's log2 denominators
  float Z;                // sum of the weights, own included
  float w_own;            // weight of the tile's own O accumulator (already / l)
  float w[kMaxPat];       // weight of pattern i's partial, 0 if it does not keep the row
  int pr[kMaxPat];        // pattern i's partial row of this row, -1 if none
  bool ok;
};

// Part 1 runs once the tile's last P is stored, while its last PV product is
// still in flight: which partial rows the row has (checking that they are
// stored), their lse_i turned into weights, and an L2 prefetch of their O_i
// rows so that part 2 finds them on chip.
template <int D>
__device__ __forceinline__ MergeWeights merge_weights(const FwdParams& p, const TileUnit& wu,
                                                      const SegInfo& si, int vq, float m_run,
                                                      float l_run, bool all_done,
                                                      volatile int* abort_flag) {
  constexpr float kLog2e = 1.4426950408889634f;
  MergeWeights mw;
  mw.ok = true;
  const int n = (int)si.start + vq;  // r = 1, offset 0
  const int bh = wu.b * p.H + wu.h;
  const bool valid = vq < si.n;
  const float own = m_run + __log2f(l_run);
#pragma unroll
  for (int i = 0; i < kMaxPat; ++i) {
    mw.pr[i] = -1;
    if (i >= p.npat || i == p.merger || !valid) continue;
    const PatternGeom& gi = p.pat[i];
    const int off = wu.h - (int)(udiv((uint32_t)wu.h, gi.r_mul, gi.r_sh) * (uint32_t)gi.r);
    mw.pr[i] = partial_row(gi, n, off, bh);
  }
  // every row's flag first (skipped once every partial-storing unit is done),
  // then the lse loads, independent of one another
  if (!all_done) {
#pragma unroll
    for (int i = 0; i < kMaxPat; ++i)
      if (mw.pr[i] >= 0 && !wait_flag(p.flags + (mw.pr[i] >> 7), abort_flag, p.err)) mw.ok = false;
  }
  float L[kMaxPat];
  mw.M = own;
#pragma unroll
  for (int i = 0; i < kMaxPat; ++i) {
    L[i] = -INFINITY;
    if (mw.pr[i] < 0) continue;
    L[i] = __ldcg(p.part_lse + mw.pr[i]) * kLog2e;
    const char* row = reinterpret_cast<const char*>(p.part_o + (long long)mw.pr[i] * D);
#pragma unroll
    for (int c = 0; c < D * 4; c += 128) prefetch_l2(row + c);
    mw.M = fmaxf(mw.M, L[i]);
  }
  mw.Z = ex2(own - mw.M);
  mw.w_own = mw.Z / l_run;
#pragma unroll
  for (int i = 0; i < kMaxPat; ++i) {
    mw.w[i] = L[i] == -INFINITY ? 0.f : ex2(L[i] - mw.M);
    mw.Z += mw.w[i];
  }
  return mw;
}

// Part 2, once the last PV is complete: O from TMEM, the partials' rows, the
// normalised result to out (and out_res), lse.
// All D columns at once (d = 64).
template <int D>
__device__ __forceinline__ void merge_epilogue_whole(const FwdParams& p, const TileUnit& wu,
                                               const SegInfo& si, int vq, uint32_t tl_o,
                                               const MergeWeights& mw) {
  float acc[D];
#pragma unroll
  for (int c4 = 0; c4 < D / 32; ++c4) {
    uint32_t r[32];
    tmem_ld32_sync(tl_o + c4 * 32, r);  // warp-collective: every lane loads
#pragma unroll
    for (int c = 0; c < 32; ++c) acc[c4 * 32 + c] = __uint_as_float(r[c]) * mw.w_own;
  }
  if (vq >= si.n || !mw.ok) return;
  const int n = (int)si.start + vq;
  const int bh = wu.b * p.H + wu.h;
#pragma unroll
  for (int i = 0; i < kMaxPat; ++i) {
    if (mw.pr[i] < 0 || mw.w[i] == 0.f) continue;
    const float wi = mw.w[i];
    const float4* src = reinterpret_cast<const float4*>(p.part_o + (long long)mw.pr[i] * D);
#pragma unroll
    for (int e = 0; e < D / 4; ++e) {
      const float4 x = __ldcg(src + e);
      acc[4 * e] = fmaf(wi, x.x, acc[4 * e]);
      acc[4 * e + 1] = fmaf(wi, x.y, acc[4 * e + 1]);
      acc[4 * e + 2] = fmaf(wi, x.z, acc[4 * e + 2]);
      acc[4 * e + 3] = fmaf(wi, x.w, acc[4 * e + 3]);
    }
  }
  const float inv = 1.f / mw.Z;
  const long long o0 = (((long long)wu.b * p.N + n) * p.H + wu.h) * D;
  uint4* dst = reinterpret_cast<uint4*>(p.out + o0);
  uint4* rdst = p.out_res != nullptr ? reinterpret_cast<uint4*>(p.out_res + o0) : nullptr;
#pragma unroll
  for (int e = 0; e < D / 8; ++e) {
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float a = acc[8 * e + 2 * j] * inv, b = acc[8 * e + 2 * j + 1] * inv;
      hi[j] = pack_bf16_rn(a, b);
      lo[j] = pack_bf16_rn(a - __uint_as_float(hi[j] << 16), b - __uint_as_float(hi[j] & 0xffff0000u));
    }
    dst[e] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    if (rdst != nullptr) rdst[e] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
  if (p.lse != nullptr)
    p.lse[(long long)bh * p.N + n] = (mw.M + __log2f(mw.Z)) * 0.69314718055994531f;
}

// In column halves of 64, which bounds the registers the accumulator takes
// (d = 128).
template <int D>
__device__ __forceinline__ void merge_epilogue_halves(const FwdParams& p, const TileUnit& wu,
                                               const SegInfo& si, int vq, uint32_t tl_o,
                                               const MergeWeights& mw) {
  constexpr int CW = 64;
#pragma unroll
  for (int h = 0; h < D / CW; ++h) {
    float acc[CW];
#pragma unroll
    for (int c4 = 0; c4 < CW / 32; ++c4) {
      uint32_t r[32];
      tmem_ld32_sync(tl_o + h * CW + c4 * 32, r);  // warp-collective: every lane loads
#pragma unroll
      for (int c = 0; c < 32; ++c) acc[c4 * 32 + c] = __uint_as_float(r[c]) * mw.w_own;
    }
    // rows with no result skip the rest, but still take part in the next
    // half's (warp-collective) TMEM load
    if (vq >= si.n || !mw.ok) continue;
    const int n = (int)si.start + vq;
#pragma unroll
    for (int i = 0; i < kMaxPat; ++i) {
      if (mw.pr[i] < 0 || mw.w[i] == 0.f) continue;
      const float wi = mw.w[i];
      const float4* src =
          reinterpret_cast<const float4*>(p.part_o + (long long)mw.pr[i] * D + h * CW);
#pragma unroll
      for (int e = 0; e < CW / 4; ++e) {
        const float4 x = __ldcg(src + e);
        acc[4 * e] = fmaf(wi, x.x, acc[4 * e]);
        acc[4 * e + 1] = fmaf(wi, x.y, acc[4 * e + 1]);
        acc[4 * e + 2] = fmaf(wi, x.z, acc[4 * e + 2]);
        acc[4 * e + 3] = fmaf(wi, x.w, acc[4 * e + 3]);
      }
    }
    const float inv = 1.f / mw.Z;
    const long long o0 = (((long long)wu.b * p.N + n) * p.H + wu.h) * D + h * CW;
    uint4* dst = reinterpret_cast<uint4*>(p.out + o0);
    uint4* rdst = p.out_res != nullptr ? reinterpret_cast<uint4*>(p.out_res + o0) : nullptr;
#pragma unroll
    for (int e = 0; e < CW / 8; ++e) {
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float a = acc[8 * e + 2 * j] * inv, b = acc[8 * e + 2 * j + 1] * inv;
        hi[j] = pack_bf16_rn(a, b);
        lo[j] = pack_bf16_rn(a - __uint_as_float(hi[j] << 16), b - __uint_as_float(hi[j] & 0xffff0000u));
      }
      dst[e] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      if (rdst != nullptr) rdst[e] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
    if (h == D / CW - 1 && p.lse != nullptr)
      p.lse[(long long)(wu.b * p.H + wu.h) * p.N + n] = (mw.M + __log2f(mw.Z)) * 0.69314718055994531f;
  }
}

template <int D>
__device__ __forceinline__ void merge_epilogue(const FwdParams& p, const TileUnit& wu,
                                               const SegInfo& si, int vq, uint32_t tl_o,
                                               const MergeWeights& mw) {
  if constexpr (D <= 64)
    merge_epilogue_whole<D>(p, wu, si, vq, tl_o, mw);
  else
    merge_epilogue_halves<D>(p, wu, si, vq, tl_o, mw);
}

template <int D, bool QK8 = false>
__global__ void __launch_bounds__(FwdCfg<D, QK8>::THREADS, FwdCfg<D, QK8>::MIN_BLOCKS)
    fwd_tile_kernel(const __grid_constant__ FwdParams p) {
  using C = FwdCfg<D, QK8>;
  constexpr int BN = C::BN;  // this kernel's key-tile rows (the library-wide BN is 128)
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t base = (raw_s + 1023u) & ~1023u;
  uint8_t* base_g = smem_raw + (base - raw_s);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const uint32_t sQ = base + C::OFF_Q;
  const uint32_t sK = base + C::OFF_K;
  const uint32_t sV = base + C::OFF_V;
  const uint32_t bars = base + C::OFF_BAR;
  const uint32_t b_qfull = bars;
  auto b_kfull = [&](int s) { return bars + 8u + 8u * s; };
  auto b_kempty = [&](int s) { return bars + 8u + 8u * C::KST + 8u * s; };
  auto b_vfull = [&](int s) { return bars + 8u + 16u * C::KST + 8u * s; };
  auto b_vempty = [&](int s) { return bars + 8u + 16u * C::KST + 8u * C::VST + 8u * s; };
  const uint32_t b_sfull = bars + 8u + 16u * C::KST + 16u * C::VST;
  const uint32_t b_sfree = b_sfull + 8u;
  const uint32_t b_pfull = b_sfull + 16u;
  const uint32_t b_odone = b_sfull + 24u;
  const uint32_t b_epi = b_sfull + 32u;  // the four softmax warps have stored their partial rows
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_g + C::OFF_BAR + 224);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base_g + C::OFF_BAR + 228);

  // Units are taken in ticket order, not blockIdx order: every tile that
  // stores partials has a smaller ticket than every merging tile, so a merging
  // tile only ever waits for tiles that running CTAs already hold. The
  // barriers and the TMEM allocation do not depend on the unit, so they are
  // set up while the ticket's atomic is in flight.
  __shared__ int s_ticket;
  if (threadIdx.x == 0) s_ticket = atomicAdd(p.counter, 1);
  if (threadIdx.x == 64) {
    mbar_init(b_qfull, 1);
    for (int s = 0; s < C::KST; ++s) {
      mbar_init(b_kfull(s), 1);
      mbar_init(b_kempty(s), 1);
    }
    for (int s = 0; s < C::VST; ++s) {
      mbar_init(b_vfull(s), 1);
      mbar_init(b_vempty(s), 1);
    }
    mbar_init(b_sfull, 1);
    mbar_init(b_sfree, C::SM_WARPS);
    mbar_init(b_pfull, C::SM_WARPS);
    mbar_init(b_odone, 1);
    mbar_init(b_epi, 4);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
  const long long ticket = s_ticket;
  const TileUnit wu = ticket < p.units_p
      ? decode_unit(p.sched, p.pat, p.B, p.H, ticket)
      : decode_unit(p.sched_m, p.pat, p.B, p.H, ticket - p.units_p);
  const PatternGeom g = p.pat[wu.pat];
  const SegInfo si = seg_info(g, p.N, wu.h, wu.seg);
  if (wu.t * BM >= si.n) {  // tile past the segment's kept rows (uniform exit)
    if (threadIdx.x == 0 && ticket < p.units_p) atomicAdd(p.done, 1);
    if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
    return;
  }
  const bool merging = wu.pat == p.merger;
  const bool gathered = p.kv_rows[wu.pat] > 0;
  const int kv_n = gathered ? p.kv_rows[wu.pat] : si.n;  // key rows of the segment
  const int tq = wu.t + p.toff[wu.pat];                   // the query tile among the key tiles
  const int qbase = tq * BM;  // key index of the tile's first query row
  // causal: key tiles up to the one holding the tile's last query row (with
  // BN = BM, the query tile's own)
  const int nkv = !p.causal ? (kv_n + BN - 1) / BN
                 : BN == BM ? tq + 1
                            : (qbase + min(BM, si.n - wu.t * BM) - 1) / BN + 1;

  // All tiles of a (pattern, segment, head) share one phase, hence one view.
  int phase0, m0;
  view_coords(g, si, 0, phase0, m0);
  const bool tail_view = phase0 < g.nmod;
  const CUtensorMap* mq = tail_view ? &p.tmq_t[wu.pat] : &p.tmq[wu.pat];
  const CUtensorMap* mk = tail_view && !gathered ? &p.tmk_t[wu.pat] : &p.tmk[wu.pat];
  const CUtensorMap* mv = tail_view && !gathered ? &p.tmv_t[wu.pat] : &p.tmv[wu.pat];
  // coordinates of key tile `it`: the strided view's (phase, row), or the
  // gathered buffer's (row within a rank's block, rank)
  auto kv_coords = [&](int it, int& c2, int& c3) {
    if (gathered) {
      const uint32_t j = (uint32_t)(it * BN), rr = (uint32_t)p.kv_rank_rows[wu.pat];
      c3 = (int)(j / rr);
      c2 = (int)(j - (uint32_t)c3 * rr);
    } else {
      view_coords(g, si, it * BN, c2, c3);
    }
  };
  if (warp == 0 && lane == 0) {
    prefetch_tmap(mq);
    prefetch_tmap(mk);
    prefetch_tmap(mv);
  }

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // lane 0 streams Q then the K ring, lane 1 the V ring, independently
    if (lane == 0) {
      int ph, m;
      view_coords(g, si, wu.t * BM, ph, m);
      mbar_arrive_expect_tx(b_qfull, C::Q_BYTES);
      for (int c = 0; c < C::KCH_QK; ++c)
        tma_load_5d(sQ + c * C::Q_CHUNK, mq, b_qfull, c * C::QK_COLS, wu.h, ph, m, wu.b);
      int issued = 0;
      for (int it = 0; it < nkv; ++it) {
        const int s = it % C::KST;
        if (!mbar_wait(b_kempty(s), ((it / C::KST) & 1) ^ 1, abort_flag, p.err)) break;
        kv_coords(it, ph, m);
        mbar_arrive_expect_tx(b_kfull(s), C::K_BYTES);
        for (int c = 0; c < C::KCH_QK; ++c)
          tma_load_5d(sK + s * C::K_BYTES + c * C::KV_CHUNK, mk, b_kfull(s), c * C::QK_COLS,
                      wu.h, ph, m, wu.b);
        ++issued;
      }
      if (*abort_flag) {
        // Drain copies still in flight before the CTA's shared memory goes away.
        volatile int no_abort = 0;
        mbar_wait(b_qfull, 0, &no_abort, ErrCtx{}, 200000000ull);
        for (int it = issued - C::KST; it < issued; ++it)
          if (it >= 0)
            mbar_wait(b_kfull(it % C::KST), (it / C::KST) & 1, &no_abort, ErrCtx{}, 200000000ull);
      }
    } else if (lane == 1) {
      int ph, m, issued = 0;
      for (int it = 0; it < nkv; ++it) {
        const int s = it % C::VST;
        if (!mbar_wait(b_vempty(s), ((it / C::VST) & 1) ^ 1, abort_flag, p.err)) break;
        kv_coords(it, ph, m);
        mbar_arrive_expect_tx(b_vfull(s), C::V_BYTES);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_5d(sV + s * C::V_BYTES + c * C::KV_CHUNK, mv, b_vfull(s), c * 64, wu.h, ph,
                      m, wu.b);
        ++issued;
      }
      if (*abort_flag) {
        volatile int no_abort = 0;
        for (int it = issued - C::VST; it < issued; ++it)
          if (it >= 0)
            mbar_wait(b_vfull(it % C::VST), (it / C::VST) & 1, &no_abort, ErrCtx{}, 200000000ull);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // S(j) = Q K_j^T once K_j is resident and the softmax has read S(j-1);
    // PV(j) once P(j) and V_j are ready. The whole warp runs the loop; one
    // elected lane issues each MMA group (descriptors are built once and
    // advanced by adds).
    {
      // Q (K-major) x K (K-major): bf16, or e4m3 (format code 0 of kind::f8f6f4)
      constexpr uint32_t kIdS = QK8 ? idesc_f16(BM, BN, 0, 0) : idesc_bf16(BM, BN, 0, 0);
      constexpr uint32_t kIdO = idesc_bf16(BM, D, 0, 1);   // P (TMEM) x V (MN-major)
      const SDesc dQ = sdesc_sw128(sQ, 16, 1024), dK = sdesc_sw128(sK, 16, 1024);
      const SDesc dV = sdesc_sw128(sV, C::KV_CHUNK, 1024);
      // S(j + 1) needs only that the softmax has read S(j), which it does
      // before it stores P(j), so the products go S(0), S(1), PV(0), S(2),
      // PV(1), ...; each wait suspends the warp in hardware.
      auto issue_s = [&](int j) {
        const uint32_t ko = (j % C::KST) * C::K_BYTES;
        if (elect_one_sync()) {
#pragma unroll
          for (int kk = 0; kk < C::S_KSTEPS; ++kk) {
            const uint32_t oq = (kk >> 2) * C::Q_CHUNK + (kk & 3) * 32;
            const uint32_t okk = C::Q_CHUNK == C::KV_CHUNK ? oq : (kk >> 2) * C::KV_CHUNK + (kk & 3) * 32;
            if (QK8)
              mma_ss_f8(tmem + C::TM_S, dQ.at(oq), dK.at(ko + okk), kIdS, kk > 0 ? 1u : 0u);
            else
              mma_ss(tmem + C::TM_S, dQ.at(oq), dK.at(ko + okk), kIdS, kk > 0 ? 1u : 0u);
          }
          mma_commit(b_sfull);
          mma_commit(b_kempty(j % C::KST));
        }
        __syncwarp();
      };
      auto issue_pv = [&](int j) {
        const uint32_t vo = (j % C::VST) * C::V_BYTES;
        if (elect_one_sync()) {
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)
            mma_ts(tmem + C::TM_O, tmem + C::TM_P + kk * 8, dV.at(vo + kk * 2048), kIdO,
                   (j > 0 || kk > 0) ? 1u : 0u);
          mma_commit(b_vempty(j % C::VST));
          mma_commit(b_odone);
        }
        __syncwarp();
      };
      bool ok = warp_wait(b_qfull, 0, abort_flag, p.err);
      for (int j = 0; ok && j <= nkv; ++j) {
        if (j < nkv) {
          ok = warp_wait(b_kfull(j % C::KST), (j / C::KST) & 1, abort_flag, p.err) &&
               (j == 0 || warp_wait(b_sfree, (j - 1) & 1, abort_flag, p.err));
          if (!ok) break;
          tc_fence_after();
          issue_s(j);
        }
        if (j > 0) {
          ok = warp_wait(b_pfull, (j - 1) & 1, abort_flag, p.err) &&
               warp_wait(b_vfull((j - 1) % C::VST), ((j - 1) / C::VST) & 1, abort_flag, p.err);
          if (!ok) break;
          tc_fence_after();
          issue_pv(j - 1);
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const int vq = wu.t * BM + row;
    const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
    const float sc = p.scale_log2;
    const uint64_t sc2 = f2_pack(sc, sc);
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int it = 0; it < nkv; ++it) {
      if (!warp_wait(b_sfull, it & 1, abort_flag, p.err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t raw[BN];
      if constexpr (BN == 128)
        tmem_ld128_sync(tl + C::TM_S, raw);
      else
        tmem_ld32x2_sync(tl + C::TM_S, tl + C::TM_S + 32, *reinterpret_cast<uint32_t(*)[32]>(&raw[0]),
                         *reinterpret_cast<uint32_t(*)[32]>(&raw[32]));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(b_sfree);

      if (p.causal) {
        // key it * BN + c against query qbase + row; only tiles that reach
        // the diagonal hold masked columns (with BN = BM, the last one)
        if constexpr (BN == BM) {
          if (it == tq) {
#pragma unroll
            for (int c = 0; c < BN; ++c)
              if (c > row) raw[c] = 0xff800000u;  // -inf
          }
        } else {
          const int off = it * BN - qbase;
          if (off > -BN) {
#pragma unroll
            for (int c = 0; c < BN; ++c)
              if (c + off > row) raw[c] = 0xff800000u;
          }
        }
      } else if (it == nkv - 1) {
        const int lim = kv_n - it * BN;
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (c >= lim) raw[c] = 0xff800000u;
      }
      // row max: four independent chains of 3-input max over columns
      // [4, BN - 4), then the last four columns
      static_assert(BN % 8 == 0, "the row max takes columns in groups of 8");
      float a0 = __uint_as_float(raw[0]), a1 = __uint_as_float(raw[1]);
      float a2 = __uint_as_float(raw[2]), a3 = __uint_as_float(raw[3]);
#pragma unroll
      for (int c = 4; c + 8 <= BN; c += 8) {
        a0 = max3(a0, __uint_as_float(raw[c]), __uint_as_float(raw[c + 1]));
        a1 = max3(a1, __uint_as_float(raw[c + 2]), __uint_as_float(raw[c + 3]));
        a2 = max3(a2, __uint_as_float(raw[c + 4]), __uint_as_float(raw[c + 5]));
        a3 = max3(a3, __uint_as_float(raw[c + 6]), __uint_as_float(raw[c + 7]));
      }
      a0 = max3(a0, __uint_as_float(raw[BN - 4]), __uint_as_float(raw[BN - 3]));
      a1 = max3(a1, __uint_as_float(raw[BN - 2]), __uint_as_float(raw[BN - 1]));
      const float mx = max3(a0, a1, fmaxf(a2, a3));
      // The exponent reference m_run moves only when the tile's max exceeds it
      // by more than 8 (log2 units); otherwise P <= 2^8 and O is not rescaled.
      // out = O / l and lse = m_run + log2(l) use the same reference, so the
      // result is unchanged.
      const float m_tile = mx * sc;
      const bool move = m_tile > m_run + 8.f;
      const float m_new = move ? m_tile : m_run;
      const float alpha = move ? ex2(m_run - m_new) : 1.f;
      const uint64_t negm2 = f2_pack(-m_new, -m_new);
      uint64_t sum2a = 0, sum2b = 0;  // +0.0f pairs
      uint32_t pk[BN / 2];
#pragma unroll
      for (int c = 0; c < BN / 2; ++c) {
        const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(raw[2 * c]),
                                           __uint_as_float(raw[2 * c + 1])), sc2, negm2);
        const uint64_t p2 = f2_pack(ex2(f2_lo(x2)), ex2(f2_hi(x2)));
        if (c & 1)
          sum2a = f2_add(sum2a, p2);
        else
          sum2b = f2_add(sum2b, p2);
        pk[c] = pack_bf16_rn(f2_lo(p2), f2_hi(p2));
      }
      const uint64_t sum2 = f2_add(sum2a, sum2b);
      l_run = l_run * alpha + (f2_lo(sum2) + f2_hi(sum2));
      m_run = m_new;

      if (it > 0) {
        // PV of the previous tile must be complete before O is rescaled and P overwritten.
        if (!warp_wait(b_odone, (it - 1) & 1, abort_flag, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, move)) {
#pragma unroll
          for (int c4 = 0; c4 < D / 32; ++c4) {
            uint32_t r[32];
            tmem_ld32_sync(tl + C::TM_O + c4 * 32, r);
#pragma unroll
            for (int c = 0; c < 32; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) * alpha);
            tmem_st32_sync(tl + C::TM_O + c4 * 32, r);
          }
        }
      }
#pragma unroll
      for (int c4 = 0; c4 < BN / 32; ++c4)
        tmem_st16(tl + C::TM_P + c4 * 16, *reinterpret_cast<const uint32_t(*)[16]>(&pk[c4 * 16]));
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(b_pfull);
    }
    MergeWeights mw;
    if (ok && merging) {
      // while the last PV runs: the other patterns' lse values and the
      // weights, after checking that the partials are stored (once every
      // partial-storing unit is done, no per-block flag needs reading)
      int all_done = 0;
      if (lane == 0) all_done = ld_acquire_gpu(p.done) >= (int)p.units_p;
      all_done = __shfl_sync(0xffffffffu, all_done, 0);
      mw = merge_weights<D>(p, wu, si, vq, m_run, l_run, all_done != 0, abort_flag);
    }
    if (ok && warp_wait(b_odone, (nkv - 1) & 1, abort_flag, p.err)) {
      tc_fence_after();
      if (merging) {
        merge_epilogue<D>(p, wu, si, vq, tl + C::TM_O, mw);
      } else {
        // The tile's 128 partial rows are one contiguous block of the partial
        // buffer (segments own whole tiles there); each thread stores its row
        // of O / l and its lse, then the block's flag is released.
        const long long prow0 =
            g.part_base + ((long long)(wu.b * p.H + wu.h) * g.nseg + wu.seg) * g.pstride +
            (long long)wu.t * BM;
        const float inv = 1.f / l_run;
        float4* dst = reinterpret_cast<float4*>(p.part_o + (prow0 + row) * D);
#pragma unroll
        for (int c4 = 0; c4 < D / 32; ++c4) {
          uint32_t r[32];
          tmem_ld32_sync(tl + C::TM_O + c4 * 32, r);
          if (vq < si.n) {
#pragma unroll
            for (int k = 0; k < 8; ++k)
              dst[c4 * 8 + k] = make_float4(__uint_as_float(r[4 * k]) * inv,
                                            __uint_as_float(r[4 * k + 1]) * inv,
                                            __uint_as_float(r[4 * k + 2]) * inv,
                                            __uint_as_float(r[4 * k + 3]) * inv);
          }
        }
        if (vq < si.n) p.part_lse[prow0 + row] = (m_run + __log2f(l_run)) * 0.69314718055994531f;
        // The block's flag is released once all four softmax warps have
        // stored their rows (mbarrier, release/acquire within the CTA; a
        // bounded wait: an aborted warp never arrives, and then no flag is
        // released), by one thread whose gpu-scope fence and release store
        // cover the stores the mbarrier ordered before it.
        __syncwarp();
        if (lane == 0) mbar_arrive(b_epi);
        if (warp == 2 && lane == 0 && mbar_wait(b_epi, 0, abort_flag, p.err)) {
          __threadfence();
          st_release_gpu(p.flags + (prow0 >> 7), 1);
          atomicAdd(p.done, 1);
        }
      }
    }
    tc_fence_before();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace dil
