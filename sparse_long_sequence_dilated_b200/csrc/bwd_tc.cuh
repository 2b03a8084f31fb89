// Backward kernels: preprocess (D = rowsum(dO * O) from the forward's fp32
// copy of O when given, else from the bf16 O; zero the fp32 accumulators),
// the tcgen05 key-tile kernel, and the fp32 -> bf16 convert.
//
// The merged forward is one softmax over the multiset union of the keys the
// patterns give a row (LongNet pages: segments, dilation and per-head
// offsets from the gptget.net summary of arXiv 2307.02486, "方法详解"; the
// shared-denominator merge from the DarcStar commentary). So with the merged
// lse L and D = rowsum(dO * O) every (pattern, segment) contributes the
// ordinary attention-backward terms with P = exp(tau S - L), and the
// contributions of different patterns simply add up.
//
// Key-tile kernel: one CTA per (pattern, segment, batch, head, key tile u),
// looping over the segment's query tiles t (t >= u when causal). Per pair:
//   S^T  = K Q^T,  dP^T = V dO^T                     (SMEM x SMEM -> TMEM)
//   P^T  = exp2(S^T tau log2e - L log2e), dS^T = P^T (dP^T - D)   (threads)
//   dV  += P^T dO,  dK += dS^T Q                     (TMEM x SMEM -> TMEM)
//   dQ   = dS K                                      (SMEM x SMEM -> TMEM)
// P and dS enter their products as two bf16 halves each, hi + lo, so the
// products are fp32-grade: the gradients' own bf16 rounding (half an ulp is
// 0.0078 at |g| in [2, 4)) leaves no room for a 2^-9 rounding of P or dS under
// a 2e-2 bound.
// dQ is staged in shared memory after every pair and added to an fp32
// accumulator by a TMA reduce-add; dK, dV are added the same way once at the
// end (other patterns and tiles reach the same rows). The three accumulators
// form one [3B][N][H][64] fp32 tensor read through the same strided views.
//
// Warp roles (64 + 128 NCG threads): warp 0 TMA producer (+ per-tile L and D
// rows), warp 1 TMEM allocator and MMA issuer, warps 2.. the row work: warp w
// serves TMEM lanes 32 (w % 4) .. + 31 and column group (w - 2) / 4, i.e. the
// CPT = 4 / NCG consecutive 32-column chunks of that group.
// TMEM columns: S^T / P^T [0,128), dP^T / dS^T [128,256), dV [256,320),
// dK [320,384), dQ [384,448). P^T and dS^T (hi, lo) overwrite S^T and dP^T in
// place, each 32-column quarter by the warps that read it: query columns
// [32q, 32q + 32) keep P^T hi at TM_S + 32q + [0, 16), lo at TM_S + 32q + [16, 32),
// and dS^T hi / lo at TM_DP + 32q + [0, 16) / [16, 32).
#pragma once

#include "common.cuh"

namespace dil {

struct BwdParams {
  CUtensorMap tmq[kMaxPat], tmk[kMaxPat], tmv[kMaxPat], tmdo[kMaxPat];
  CUtensorMap tmq_t[kMaxPat], tmk_t[kMaxPat], tmv_t[kMaxPat], tmdo_t[kMaxPat];
  PatternGeom pat[kMaxPat];
  int npat, B, N, H, causal;
  float scale_log2;  // log2(e) / sqrt(d)
  float tau;         // 1 / sqrt(d)
  Sched sched;
  CUtensorMap tmacc[kMaxPat], tmacc_t[kMaxPat];  // fp32 [3B][N][H][64]: dq, dk, dv
  const float* lse;   // [B][H][N] natural log
  const float* drow;  // [B][H][N]
  int* err;
};

#ifndef DILATTN_BWD_SPLIT_DS
#define DILATTN_BWD_SPLIT_DS 1
#endif

struct BwdCfg {
  static constexpr int D = 64;
  static constexpr bool SPLIT_DS = DILATTN_BWD_SPLIT_DS != 0;  // dS as bf16 hi + lo
  static constexpr int NCG = 2;                    // column groups of the row warps
  static constexpr int CPT = 4 / NCG;              // 32-column chunks per row thread
  static constexpr int ROW_WARPS = 4 * NCG;
  static constexpr int THREADS = 64 + 32 * ROW_WARPS;
  static constexpr int STAGES = 2;
  static constexpr int TILE = BM * 128;  // 128 rows x 64 bf16
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_Q = OFF_V + TILE;                 // STAGES tiles
  static constexpr int OFF_DO = OFF_Q + STAGES * TILE;       // STAGES tiles
  static constexpr int OFF_DS = OFF_DO + STAGES * TILE;      // dS hi: 2 chunks of [128 kv][64 q]
  static constexpr int OFF_DSL = OFF_DS + 2 * TILE;          // dS lo, same layout
  static constexpr int OFF_STG = OFF_DSL + 2 * TILE;         // fp32 [2][128][32] staging
  static constexpr int STG_BYTES = 2 * BM * 128;             // one 128 x 64 fp32 tile
  static constexpr int OFF_L = OFF_STG + STG_BYTES;          // STAGES x 128 floats
  static constexpr int OFF_D = OFF_L + STAGES * BM * 4;      // STAGES x 128 floats
  static constexpr int OFF_BAR = OFF_D + STAGES * BM * 4;
  static constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;
  static constexpr int TM_S = 0, TM_DP = 128, TM_DV = 256, TM_DK = 320, TM_DQ = 384;
  static constexpr int TMEM_COLS = 512;
};

// Thread `row` writes 16 fp32 = 16-byte pieces [piece0, piece0 + 4) of one
// 128-byte row of a [128][32] fp32 chunk with 128-byte swizzle (piece k lands
// at k ^ (row % 8)), scaled by `scale`.
__device__ __forceinline__ void stage_row16(uint8_t* chunk, int row, int piece0,
                                            const uint32_t (&r)[16], float scale) {
  uint8_t* rowp = chunk + row * 128;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float4 v = make_float4(__uint_as_float(r[4 * k]) * scale,
                                 __uint_as_float(r[4 * k + 1]) * scale,
                                 __uint_as_float(r[4 * k + 2]) * scale,
                                 __uint_as_float(r[4 * k + 3]) * scale);
    *reinterpret_cast<float4*>(rowp + (((piece0 + k) ^ (row & 7)) * 16)) = v;
  }
}

__global__ void __launch_bounds__(BwdCfg::THREADS, 1) bwd_tile_kernel(const __grid_constant__ BwdParams p) {
  using C = BwdCfg;
  constexpr int D = C::D;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t base = (raw_s + 1023u) & ~1023u;
  uint8_t* base_g = smem_raw + (base - raw_s);

  const TileUnit wu = decode_unit(p.sched, p.pat, p.B, p.H, blockIdx.x);
  const PatternGeom g = p.pat[wu.pat];
  const SegInfo si = seg_info(g, p.N, wu.h, wu.seg);
  const int nq = (si.n + BM - 1) / BM;
  const int u = g.ntiles - 1 - wu.t;  // key tile; long (small u) tiles come first
  if (u >= nq) return;                // uniform exit: no key rows here
  const int t0 = p.causal ? u : 0;
  const int npairs = nq - t0;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t sK = base + C::OFF_K, sV = base + C::OFF_V;
  const uint32_t sQ = base + C::OFF_Q, sDO = base + C::OFF_DO, sDS = base + C::OFF_DS;
  const uint32_t sDSL = base + C::OFF_DSL;
  float* sL = reinterpret_cast<float*>(base_g + C::OFF_L);
  float* sD = reinterpret_cast<float*>(base_g + C::OFF_D);
  const uint32_t bars = base + C::OFF_BAR;
  const uint32_t b_kvfull = bars;
  auto b_qfull = [&](int s) { return bars + 8u + 8u * s; };
  auto b_qempty = [&](int s) { return bars + 8u + 8u * C::STAGES + 8u * s; };
  const uint32_t b_sdp = bars + 8u + 16u * C::STAGES;
  const uint32_t b_ds = b_sdp + 8u;
  const uint32_t b_dq = b_sdp + 16u;
  const uint32_t b_kv2 = b_sdp + 24u;
  const uint32_t b_grp = b_sdp + 32u;  // sync point of the row warps (bounded, unlike bar.sync)
  const uint32_t sSTG = base + C::OFF_STG;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_g + C::OFF_BAR + 224);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base_g + C::OFF_BAR + 228);

  int phase0, m0;
  view_coords(g, si, 0, phase0, m0);
  const bool tail_view = phase0 < g.nmod;
  const CUtensorMap* mq = tail_view ? &p.tmq_t[wu.pat] : &p.tmq[wu.pat];
  const CUtensorMap* mk = tail_view ? &p.tmk_t[wu.pat] : &p.tmk[wu.pat];
  const CUtensorMap* mv = tail_view ? &p.tmv_t[wu.pat] : &p.tmv[wu.pat];
  const CUtensorMap* mdo = tail_view ? &p.tmdo_t[wu.pat] : &p.tmdo[wu.pat];
  const CUtensorMap* macc = tail_view ? &p.tmacc_t[wu.pat] : &p.tmacc[wu.pat];

  if (threadIdx.x == 0) {
    mbar_init(b_kvfull, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(b_qfull(s), 1);
      mbar_init(b_qempty(s), 1);
    }
    mbar_init(b_sdp, 1);
    mbar_init(b_ds, C::ROW_WARPS);
    mbar_init(b_dq, 1);
    mbar_init(b_kv2, 1);
    mbar_init(b_grp, C::ROW_WARPS);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(mq);
    prefetch_tmap(mk);
    prefetch_tmap(mv);
    prefetch_tmap(mdo);
    prefetch_tmap(macc);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
  const long long lrow0 = ((long long)wu.b * p.H + wu.h) * p.N;  // lse / D row base
  const float log2e = 1.4426950408889634f;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int ph, m;
    if (lane == 0) {
      view_coords(g, si, u * BN, ph, m);
      mbar_arrive_expect_tx(b_kvfull, 2 * C::TILE);
      tma_load_5d(sK, mk, b_kvfull, 0, wu.h, ph, m, wu.b);
      tma_load_5d(sV, mv, b_kvfull, 0, wu.h, ph, m, wu.b);
    }
    int issued = 0;
    for (int it = 0; it < npairs; ++it) {
      const int s = it % C::STAGES;
      const int t = t0 + it;
      if (!warp_wait(b_qempty(s), ((it / C::STAGES) & 1) ^ 1, abort_flag, p.err)) break;
      // merged lse (log2 units) and D for the tile's query rows; rows past the
      // segment get L = +inf, so their probabilities are exactly zero
#pragma unroll
      for (int jj = 0; jj < BM / 32; ++jj) {
        const int j = lane + 32 * jj;
        const int vq = t * BM + j;
        float L = INFINITY, Dv = 0.f;
        if (vq < si.n) {
          const long long pos = si.start + si.off + (long long)vq * g.r;
          L = p.lse[lrow0 + pos] * log2e;
          Dv = p.drow[lrow0 + pos];
        }
        sL[s * BM + j] = L;
        sD[s * BM + j] = Dv;
      }
      __syncwarp();
      if (lane == 0) {
        view_coords(g, si, t * BM, ph, m);
        mbar_arrive_expect_tx(b_qfull(s), 2 * C::TILE);
        tma_load_5d(sQ + s * C::TILE, mq, b_qfull(s), 0, wu.h, ph, m, wu.b);
        tma_load_5d(sDO + s * C::TILE, mdo, b_qfull(s), 0, wu.h, ph, m, wu.b);
      }
      ++issued;
    }
    if (lane == 0 && *abort_flag) {
      volatile int no_abort = 0;
      mbar_wait(b_kvfull, 0, &no_abort, nullptr, 200000000ull);
      for (int it = issued - C::STAGES; it < issued; ++it) {
        if (it < 0) continue;
        mbar_wait(b_qfull(it % C::STAGES), (it / C::STAGES) & 1, &no_abort, nullptr, 200000000ull);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16(BM, BM, 0, 0);   // K x Q^T, V x dO^T
      constexpr uint32_t kIdKV = idesc_bf16(BM, D, 0, 1);   // P^T (TMEM) x dO, dS^T (TMEM) x Q
      constexpr uint32_t kIdQ = idesc_bf16(BM, D, 1, 1);    // dS (MN-major SMEM) x K
      bool ok = mbar_wait(b_kvfull, 0, abort_flag, p.err);
      for (int it = 0; ok && it < npairs; ++it) {
        const int s = it % C::STAGES;
        if (!mbar_wait(b_qfull(s), (it / C::STAGES) & 1, abort_flag, p.err)) break;
        // the dV / dK MMAs of the previous pair (readers of TMEM P^T / dS^T) are
        // complete; its dQ MMA (SMEM dS, TMEM dQ) may still run
        if (it > 0 && !mbar_wait(b_kv2, (it - 1) & 1, abort_flag, p.err)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t a = sw128_desc(sK + kk * 32, 16, 1024);
          const uint64_t b = sw128_desc(sQ + s * C::TILE + kk * 32, 16, 1024);
          mma_ss(tmem + C::TM_S, a, b, kIdS, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t a = sw128_desc(sV + kk * 32, 16, 1024);
          const uint64_t b = sw128_desc(sDO + s * C::TILE + kk * 32, 16, 1024);
          mma_ss(tmem + C::TM_DP, a, b, kIdS, kk > 0 ? 1u : 0u);
        }
        mma_commit(b_sdp);
        if (!mbar_wait(b_ds, it & 1, abort_flag, p.err)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk) {
          const uint64_t bdo = sw128_desc(sDO + s * C::TILE + kk * 2048, C::TILE, 1024);
          const uint32_t a_hi = tmem + C::TM_S + (kk >> 1) * 32 + (kk & 1) * 8;
          mma_ts(tmem + C::TM_DV, a_hi, bdo, kIdKV, (it > 0 || kk > 0) ? 1u : 0u);
          mma_ts(tmem + C::TM_DV, a_hi + 16, bdo, kIdKV, 1u);
        }
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk) {
          const uint64_t bq = sw128_desc(sQ + s * C::TILE + kk * 2048, C::TILE, 1024);
          const uint32_t a_ds = tmem + C::TM_DP + (kk >> 1) * 32 + (kk & 1) * 8;
          mma_ts(tmem + C::TM_DK, a_ds, bq, kIdKV, (it > 0 || kk > 0) ? 1u : 0u);
          if (C::SPLIT_DS) mma_ts(tmem + C::TM_DK, a_ds + 16, bq, kIdKV, 1u);
        }
        mma_commit(b_kv2);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t a = sw128_desc(sDS + kk * 2048, C::TILE, 1024);
          const uint64_t al = sw128_desc(sDSL + kk * 2048, C::TILE, 1024);
          const uint64_t b = sw128_desc(sK + kk * 2048, C::TILE, 1024);
          mma_ss(tmem + C::TM_DQ, a, b, kIdQ, kk > 0 ? 1u : 0u);
          if (C::SPLIT_DS) mma_ss(tmem + C::TM_DQ, al, b, kIdQ, 1u);
        }
        mma_commit(b_qempty(s));
        mma_commit(b_dq);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ lanes = rows
    const int q4 = warp & 3;
    const int cg = (warp - 2) >> 2;          // column group: chunks [CPT cg, CPT cg + CPT)
    const int c = q4 * 32 + lane;            // key row of S^T / dP^T / dV / dK, query row of dQ
    const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
    const bool key_valid = u * BN + c < si.n;
    const float sc = p.scale_log2;
    bool ok = true;
    uint32_t gphase = 0;
    // all row warps meet here; every wait is bounded
    auto group_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(b_grp);
      const bool r = warp_wait(b_grp, gphase & 1, abort_flag, p.err);
      ++gphase;
      return r;
    };
    for (int it = 0; it < npairs; ++it) {
      const int s = it % C::STAGES;
      const int t = t0 + it;
      if (!warp_wait(b_qfull(s), (it / C::STAGES) & 1, abort_flag, p.err) ||
          !warp_wait(b_sdp, it & 1, abort_flag, p.err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const bool diag = p.causal && t == u;
#pragma unroll 1
      for (int q = cg * C::CPT; q < cg * C::CPT + C::CPT; ++q) {
        const float4* L4 = reinterpret_cast<const float4*>(sL + s * BM + q * 32);
        const float4* D4 = reinterpret_cast<const float4*>(sD + s * BM + q * 32);
        uint32_t pk[16], plo[16], dk[16], dkl[16];
        {
          uint32_t sv[32], dv[32];
          tmem_ld32x2_sync(tl + C::TM_S + q * 32, tl + C::TM_DP + q * 32, sv, dv);
          // key rows past the segment, and (on the diagonal) queries before the
          // key, get P = 0; elsewhere no mask is needed
          const int jmin = !key_valid ? 1 << 30 : (diag ? c - q * 32 : 0);
          const bool masked = jmin > 0;
          const uint64_t sc2 = f2_pack(sc, sc);
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const float4 Lq = L4[e4], Dq = D4[e4];
            const uint64_t nl2[2] = {f2_pack(-Lq.x, -Lq.y), f2_pack(-Lq.z, -Lq.w)};
            const uint64_t dd2[2] = {f2_pack(Dq.x, Dq.y), f2_pack(Dq.z, Dq.w)};
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int e = 4 * e4 + 2 * h2;
              const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])),
                                         sc2, nl2[h2]);
              float p0 = ex2(f2_lo(x2)), p1 = ex2(f2_hi(x2));
              if (masked) {
                p0 = e >= jmin ? p0 : 0.f;
                p1 = e + 1 >= jmin ? p1 : 0.f;
              }
              const uint64_t p2 = f2_pack(p0, p1);
              // dS = P (dP - D)
              const uint64_t ds2 = f2_mul(
                  p2, f2_sub(f2_pack(__uint_as_float(dv[e]), __uint_as_float(dv[e + 1])), dd2[h2]));
              // P = hi + lo, both bf16: dV takes both halves, so P's own rounding
              // (2^-9 relative) does not reach dV on top of dV's final bf16 rounding
              const uint32_t hi = pack_bf16_rn(p0, p1);
              const uint64_t hi2 = f2_pack(__uint_as_float(hi << 16), __uint_as_float(hi & 0xffff0000u));
              const uint64_t lo2 = f2_sub(p2, hi2);
              pk[e / 2] = hi;
              plo[e / 2] = pack_bf16_rn(f2_lo(lo2), f2_hi(lo2));
              const uint32_t dhi = pack_bf16_rn(f2_lo(ds2), f2_hi(ds2));
              const uint64_t dhi2 =
                  f2_pack(__uint_as_float(dhi << 16), __uint_as_float(dhi & 0xffff0000u));
              const uint64_t dlo2 = f2_sub(ds2, dhi2);
              dk[e / 2] = dhi;
              dkl[e / 2] = pack_bf16_rn(f2_lo(dlo2), f2_hi(dlo2));
            }
          }
        }
        // in place over this chunk's own (already read) columns
        tmem_st16(tl + C::TM_S + q * 32, pk);
        tmem_st16(tl + C::TM_S + q * 32 + 16, plo);
        tmem_st16(tl + C::TM_DP + q * 32, dk);
        tmem_st16(tl + C::TM_DP + q * 32 + 16, dkl);
        // dS (query-major) into SMEM for dQ = dS K: row c of chunk (j / 64)
        // holds dS[j][c] for 64 consecutive j, 16-byte pieces XOR-swizzled by c % 8
        {
          const int chunk = q >> 1;
          const int piece0 = (q & 1) * 4;
          uint8_t* rowp = base_g + C::OFF_DS + chunk * C::TILE + c * 128;
          uint8_t* rowl = base_g + C::OFF_DSL + chunk * C::TILE + c * 128;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int piece = (piece0 + k) ^ (c & 7);
            *reinterpret_cast<uint4*>(rowp + piece * 16) =
                make_uint4(dk[4 * k], dk[4 * k + 1], dk[4 * k + 2], dk[4 * k + 3]);
            *reinterpret_cast<uint4*>(rowl + piece * 16) =
                make_uint4(dkl[4 * k], dkl[4 * k + 1], dkl[4 * k + 2], dkl[4 * k + 3]);
          }
        }
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(b_ds);

      // dQ of this query tile (TMEM lane c = query row t*128 + c) -> staging
      // buffer (it & 1) -> TMA reduce-add into the fp32 dq accumulator. Rows
      // past the segment hold exact zeros (their P is 0); rows past N are
      // clipped by the view.
      if (!warp_wait(b_dq, it & 1, abort_flag, p.err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (threadIdx.x == 64) bulk_wait_read<0>();  // the previous reduce has read the staging buffer
      if (!group_sync()) {
        ok = false;
        break;
      }
      uint8_t* stg = base_g + C::OFF_STG;
#pragma unroll
      for (int k = 0; k < C::CPT; ++k) {
        const int col = (cg * C::CPT + k) * 16;  // dQ columns [col, col + 16)
        uint32_t r[16];
        tmem_ld16_sync(tl + C::TM_DQ + col, r);
        stage_row16(stg + (col >> 5) * (C::STG_BYTES / 2), c, ((col >> 4) & 1) * 4, r, p.tau);
      }
      fence_proxy_async_smem();
      if (!group_sync()) {
        ok = false;
        break;
      }
      if (threadIdx.x == 64) {
        int ph, m;
        view_coords(g, si, t * BM, ph, m);
        const uint32_t src = sSTG;
        tma_reduce_add_5d(macc, src, 0, wu.h, ph, m, wu.b);
        tma_reduce_add_5d(macc, src + C::STG_BYTES / 2, 32, wu.h, ph, m, wu.b);
        bulk_commit();
      }
      tc_fence_before();
    }
    // dK, dV of the key tile (all pairs are complete after the last dQ wait):
    // dV -> the staging buffer, tau * dK -> the dS area (idle now), TMA
    // reduce-add into the dv and dk accumulators (batch slots 2B + b and
    // B + b). Rows past the segment are exact zeros (their P was forced to 0).
    if (ok) {
      if (threadIdx.x == 64) bulk_wait_read<0>();
      ok = group_sync();
    }
    if (ok) {
      uint8_t* stg = base_g + C::OFF_STG;
#pragma unroll
      for (int k = 0; k < C::CPT; ++k) {
        const int col = (cg * C::CPT + k) * 16;  // dV, dK columns [col, col + 16)
        uint32_t r[16];
        tmem_ld16_sync(tl + C::TM_DV + col, r);
        stage_row16(stg + (col >> 5) * (C::STG_BYTES / 2), c, ((col >> 4) & 1) * 4, r, 1.f);
        tmem_ld16_sync(tl + C::TM_DK + col, r);
        stage_row16(base_g + C::OFF_DS + (col >> 5) * (C::STG_BYTES / 2), c, ((col >> 4) & 1) * 4,
                    r, p.tau);
      }
      fence_proxy_async_smem();
      ok = group_sync();
    }
    if (ok) {
      if (threadIdx.x == 64) {
        int ph, m;
        view_coords(g, si, u * BN, ph, m);
        tma_reduce_add_5d(macc, sSTG, 0, wu.h, ph, m, 2 * p.B + wu.b);
        tma_reduce_add_5d(macc, sSTG + C::STG_BYTES / 2, 32, wu.h, ph, m, 2 * p.B + wu.b);
        tma_reduce_add_5d(macc, sDS, 0, wu.h, ph, m, p.B + wu.b);
        tma_reduce_add_5d(macc, sDS + C::STG_BYTES / 2, 32, wu.h, ph, m, p.B + wu.b);
        bulk_commit();
      }
    }
    if (threadIdx.x == 64) bulk_wait_all();  // shared memory stays until the reduces finish
    tc_fence_before();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// D = rowsum(dO * O) per (b, h, n) and zeroed fp32 accumulators; one warp per row.
struct PrepParams {
  int B, N, H;
  const __nv_bfloat16* out;
  const float* out_f32;  // the forward's fp32 copy of out, or null
  const __nv_bfloat16* dout;
  float* drow;
  float* dq_acc;
  float* dk_acc;
  float* dv_acc;
};

__global__ void __launch_bounds__(256) bwd_prep_kernel(PrepParams p) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= (long long)p.B * p.N * p.H) return;
  const __nv_bfloat162 d = reinterpret_cast<const __nv_bfloat162*>(p.dout + row * 64)[lane];
  float2 o;
  if (p.out_f32 != nullptr) {
    o = reinterpret_cast<const float2*>(p.out_f32 + row * 64)[lane];
  } else {
    const __nv_bfloat162 ob = reinterpret_cast<const __nv_bfloat162*>(p.out + row * 64)[lane];
    o = make_float2(__low2float(ob), __high2float(ob));
  }
  float acc = o.x * __low2float(d) + o.y * __high2float(d);
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
  const float2 z = make_float2(0.f, 0.f);
  reinterpret_cast<float2*>(p.dq_acc + row * 64)[lane] = z;
  reinterpret_cast<float2*>(p.dk_acc + row * 64)[lane] = z;
  reinterpret_cast<float2*>(p.dv_acc + row * 64)[lane] = z;
  if (lane == 0) {
    const int h = (int)(row % p.H);
    const long long bn = row / p.H;
    const int n = (int)(bn % p.N);
    const int b = (int)(bn / p.N);
    p.drow[((long long)b * p.H + h) * p.N + n] = acc;
  }
}

// fp32 accumulators -> bf16 gradients (round to nearest even).
__global__ void __launch_bounds__(256) bwd_convert_kernel(long long n4, const float4* dq,
                                                          const float4* dk, const float4* dv,
                                                          uint2* gq, uint2* gk, uint2* gv) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (long long)gridDim.x * blockDim.x) {
    const float4 a = dq[i], b = dk[i], c = dv[i];
    gq[i] = make_uint2(pack_bf16(a.x, a.y), pack_bf16(a.z, a.w));
    gk[i] = make_uint2(pack_bf16(b.x, b.y), pack_bf16(b.z, b.w));
    gv[i] = make_uint2(pack_bf16(c.x, c.y), pack_bf16(c.z, c.w));
  }
}

}  // namespace dil
