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
// exactly the rows below N and rows past N read as zeros. The CTA writes
// the pattern's normalised output O_i and its log-sum-exp for those rows to
// an fp32 partial buffer; the merge kernel combines patterns.
//
// Warp roles (192 threads, two CTAs per SM at d = 64):
//   warp 0      TMA producer: lane 0 loads the Q tile once, then the K ring;
//               lane 1 the V ring.
//   warp 1      TMEM allocator and MMA issuer (the whole warp runs the event
//               loop, one elected lane issues each group):
//               S = Q K^T (SMEM x SMEM -> TMEM), O += P V (TMEM x SMEM -> TMEM).
//   warps 2..5  softmax: warp w takes TMEM lanes 32 (w % 4) .. + 31, one query
//               row per thread: fp32 row max (3-input max), P = exp2(S*scale - m)
//               with packed fp32x2 arithmetic and the exp2 on the MUFU unit
//               (DILATTN_FWD_POLY moves a share to an FMA-pipe polynomial), P
//               stored to TMEM as bf16, O rescaled in TMEM when the reference
//               max moves, epilogue.
// Rows are one per thread: at d = 64 the softmax, not the MMA, bounds a tile,
// so its issue slots are the budget every choice above is made against.
// TMEM columns: S [0,128), P [128,192) (bf16 pairs), O [192, 192+D).
#pragma once

#include "common.cuh"

// Column pairs, of every 8, whose exp2 runs as a polynomial on the FMA pipe
// instead of the MUFU unit.
#ifndef DILATTN_FWD_POLY
#define DILATTN_FWD_POLY 0
#endif

namespace dil {

struct FwdParams {
  CUtensorMap tmq[kMaxPat];   // phases [0, r), floor(N/r) rows
  CUtensorMap tmk[kMaxPat];
  CUtensorMap tmv[kMaxPat];
  CUtensorMap tmq_t[kMaxPat]; // phases [0, N mod r), floor(N/r) + 1 rows
  CUtensorMap tmk_t[kMaxPat];
  CUtensorMap tmv_t[kMaxPat];
  CUtensorMap tm_po;          // partial outputs [rows][D] fp32, box 32 x 128 (128-byte swizzle)
  PatternGeom pat[kMaxPat];
  int npat, B, N, H, causal;
  float scale_log2;  // log2(e) / sqrt(d)
  Sched sched;
  float* part_o;    // [rows][D]
  float* part_lse;  // [rows] natural-log lse of each pattern's partial
  ErrCtx err;  // device error word and this launch's tag
};

template <int D>
struct FwdCfg {
  static constexpr int KCH = D / 64;                 // 128-byte column chunks per row
  static constexpr int KST = 3;                      // K ring depth (a stage frees after its S MMA)
  static constexpr int VST = 2;                      // V ring depth (a stage frees after its PV MMA)
  static constexpr int CHUNK_BYTES = BM * 128;       // 128 rows x 64 bf16
  static constexpr int Q_BYTES = KCH * CHUNK_BYTES;
  static constexpr int KV_BYTES = KCH * CHUNK_BYTES;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + KST * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + VST * KV_BYTES;
  static constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;  // + alignment slack
  static constexpr int TM_S = 0, TM_P = 128, TM_O = 192;
  static constexpr int TMEM_COLS = (TM_O + D <= 256) ? 256 : 512;
  static constexpr int MIN_BLOCKS = (D == 64) ? 2 : 1;
  static constexpr int SM_WARPS = 4;             // softmax warps: one query row per thread
  static constexpr int THREADS = 64 + 32 * SM_WARPS;
};

template <int D>
__global__ void __launch_bounds__(FwdCfg<D>::THREADS, FwdCfg<D>::MIN_BLOCKS)
    fwd_tile_kernel(const __grid_constant__ FwdParams p) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t base = (raw_s + 1023u) & ~1023u;
  uint8_t* base_g = smem_raw + (base - raw_s);

  const TileUnit wu = decode_unit(p.sched, p.pat, p.B, p.H, blockIdx.x);
  const PatternGeom g = p.pat[wu.pat];
  const SegInfo si = seg_info(g, p.N, wu.h, wu.seg);
  if (wu.t * BM >= si.n) return;  // tile past the segment's kept rows (uniform exit)
  const int nkv = p.causal ? (wu.t + 1) : (si.n + BN - 1) / BN;

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
  const uint32_t b_epi = b_sfull + 32u;  // the four softmax warps have staged their output rows
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_g + C::OFF_BAR + 224);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base_g + C::OFF_BAR + 228);

  if (threadIdx.x == 0) {
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
  // All tiles of a (pattern, segment, head) share one phase, hence one view.
  int phase0, m0;
  view_coords(g, si, 0, phase0, m0);
  const bool tail_view = phase0 < g.nmod;
  const CUtensorMap* mq = tail_view ? &p.tmq_t[wu.pat] : &p.tmq[wu.pat];
  const CUtensorMap* mk = tail_view ? &p.tmk_t[wu.pat] : &p.tmk[wu.pat];
  const CUtensorMap* mv = tail_view ? &p.tmv_t[wu.pat] : &p.tmv[wu.pat];
  if (warp == 0 && lane == 0) {
    prefetch_tmap(mq);
    prefetch_tmap(mk);
    prefetch_tmap(mv);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // lane 0 streams Q then the K ring, lane 1 the V ring, independently
    if (lane == 0) {
      int ph, m;
      view_coords(g, si, wu.t * BM, ph, m);
      mbar_arrive_expect_tx(b_qfull, C::Q_BYTES);
      for (int c = 0; c < C::KCH; ++c)
        tma_load_5d(sQ + c * C::CHUNK_BYTES, mq, b_qfull, c * 64, wu.h, ph, m, wu.b);
      int issued = 0;
      for (int it = 0; it < nkv; ++it) {
        const int s = it % C::KST;
        if (!mbar_wait(b_kempty(s), ((it / C::KST) & 1) ^ 1, abort_flag, p.err)) break;
        view_coords(g, si, it * BN, ph, m);
        mbar_arrive_expect_tx(b_kfull(s), C::KV_BYTES);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_5d(sK + s * C::KV_BYTES + c * C::CHUNK_BYTES, mk, b_kfull(s), c * 64, wu.h, ph,
                      m, wu.b);
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
        view_coords(g, si, it * BN, ph, m);
        mbar_arrive_expect_tx(b_vfull(s), C::KV_BYTES);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_5d(sV + s * C::KV_BYTES + c * C::CHUNK_BYTES, mv, b_vfull(s), c * 64, wu.h, ph,
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
    // Event loop: S(j) = Q K_j^T as soon as K_j is resident and the softmax has
    // read S(j-1); PV(j) as soon as P(j) and V_j are ready. Neither waits for
    // the other's operands. The whole warp runs the loop; one elected lane
    // issues each MMA group (descriptors are built once and advanced by adds).
    {
      constexpr uint32_t kIdS = idesc_bf16(BM, BN, 0, 0);  // Q (K-major) x K (K-major)
      constexpr uint32_t kIdO = idesc_bf16(BM, D, 0, 1);   // P (TMEM) x V (MN-major)
      const SDesc dQ = sdesc_sw128(sQ, 16, 1024), dK = sdesc_sw128(sK, 16, 1024);
      const SDesc dV = sdesc_sw128(sV, C::CHUNK_BYTES, 1024);
      auto test = [&](uint32_t bar, uint32_t par) -> bool {
        return __shfl_sync(0xffffffffu, mbar_test(bar, par) ? 1 : 0, 0) != 0;
      };
      bool ok = warp_wait(b_qfull, 0, abort_flag, p.err);
      int ns = 0, npv = 0;
      PollGuard pg;
      while (ok && npv < nkv) {
        bool progressed = false;
        if (ns < nkv && test(b_kfull(ns % C::KST), (ns / C::KST) & 1) &&
            (ns == 0 || test(b_sfree, (ns - 1) & 1))) {
          tc_fence_after();
          const uint32_t ko = (ns % C::KST) * C::KV_BYTES;
          if (elect_one_sync()) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * C::CHUNK_BYTES + (kk & 3) * 32;
              mma_ss(tmem + C::TM_S, dQ.at(off), dK.at(ko + off), kIdS, kk > 0 ? 1u : 0u);
            }
            mma_commit(b_sfull);
            mma_commit(b_kempty(ns % C::KST));
          }
          __syncwarp();
          ++ns;
          progressed = true;
        }
        if (npv < ns && test(b_pfull, npv & 1) &&
            test(b_vfull(npv % C::VST), (npv / C::VST) & 1)) {
          tc_fence_after();
          const uint32_t vo = (npv % C::VST) * C::KV_BYTES;
          if (elect_one_sync()) {
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk)
              mma_ts(tmem + C::TM_O, tmem + C::TM_P + kk * 8, dV.at(vo + kk * 2048), kIdO,
                     (npv > 0 || kk > 0) ? 1u : 0u);
            mma_commit(b_vempty(npv % C::VST));
            mma_commit(b_odone);
          }
          __syncwarp();
          ++npv;
          progressed = true;
        }
        if (!__all_sync(0xffffffffu, pg.step(progressed, abort_flag, p.err))) ok = false;
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
      tmem_ld128_sync(tl + C::TM_S, raw);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(b_sfree);

      if (p.causal) {
        if (it == wu.t) {
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (c > row) raw[c] = 0xff800000u;  // -inf
        }
      } else if (it == nkv - 1) {
        const int lim = si.n - it * BN;
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (c >= lim) raw[c] = 0xff800000u;
      }
      // row max: four independent chains of 3-input max
      float a0 = __uint_as_float(raw[0]), a1 = __uint_as_float(raw[1]);
      float a2 = __uint_as_float(raw[2]), a3 = __uint_as_float(raw[3]);
#pragma unroll
      for (int c = 4; c < BN; c += 8) {
        a0 = max3(a0, __uint_as_float(raw[c]), __uint_as_float(raw[c + 1]));
        a1 = max3(a1, __uint_as_float(raw[c + 2]), __uint_as_float(raw[c + 3]));
        a2 = max3(a2, __uint_as_float(raw[c + 4]), __uint_as_float(raw[c + 5]));
        a3 = max3(a3, __uint_as_float(raw[c + 6]), __uint_as_float(raw[c + 7]));
      }
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
        uint64_t p2;
        if ((c & 7) >= 8 - DILATTN_FWD_POLY) {
          p2 = ex2_poly2(x2);  // DILATTN_FWD_POLY pairs in 8 on the FMA pipe
        } else {
          p2 = f2_pack(ex2(f2_lo(x2)), ex2(f2_hi(x2)));
        }
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
    if (ok && warp_wait(b_odone, (nkv - 1) & 1, abort_flag, p.err)) {
      tc_fence_after();
      // The tile's 128 partial rows are one contiguous block of the partial
      // buffer (segments own whole tiles there; rows past the segment land in
      // padding no one reads). O / l goes through the now idle K ring, staged
      // as D/32 chunks of [128 rows][32 fp32] with 128-byte swizzle, and leaves
      // by TMA stores.
      const long long prow0 =
          g.part_base + ((long long)(wu.b * p.H + wu.h) * g.nseg + wu.seg) * g.pstride +
          (long long)wu.t * BM;
      const float inv = 1.f / l_run;
      uint8_t* stg = base_g + C::OFF_K;
#pragma unroll
      for (int c4 = 0; c4 < D / 32; ++c4) {
        uint32_t r[32];
        tmem_ld32_sync(tl + C::TM_O + c4 * 32, r);
        uint8_t* rowp = stg + c4 * (BM * 128) + row * 128;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float4 v = make_float4(__uint_as_float(r[4 * k]) * inv,
                                       __uint_as_float(r[4 * k + 1]) * inv,
                                       __uint_as_float(r[4 * k + 2]) * inv,
                                       __uint_as_float(r[4 * k + 3]) * inv);
          *reinterpret_cast<float4*>(rowp + ((k ^ (row & 7)) * 16)) = v;
        }
      }
      if (vq < si.n) p.part_lse[prow0 + row] = (m_run + __log2f(l_run)) * 0.69314718055994531f;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(b_epi);
      if (warp_wait(b_epi, 0, abort_flag, p.err) && warp == 2 && lane == 0) {
#pragma unroll
        for (int c4 = 0; c4 < D / 32; ++c4)
          tma_store_2d(&p.tm_po, sK + c4 * (BM * 128), c4 * 32, (int)prow0);
        bulk_commit();
        bulk_wait_read<0>();  // the staging buffer stays until the stores have read it
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
