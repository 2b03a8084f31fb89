// Backward kernels: the preprocess (D = rowsum(dO * O) from out + out_res, fp16
// copies of q and k, the caller's fp32 gradients zeroed) and the tcgen05
// key-tile kernel, which adds into those gradients.
//
// The merged forward is one softmax over the multiset union of the keys the
// patterns give a row (LongNet pages: segments, dilation and per-head
// offsets from the gptget.net summary of arXiv 2307.02486, "方法详解"; the
// shared-denominator merge from the DarcStar commentary). So with the merged
// lse L and D = rowsum(dO * O) every (pattern, segment) contributes the
// ordinary attention-backward terms with P = exp(tau S - L), and the
// contributions of different patterns simply add up.
//
// Key-tile kernel. A unit is (pattern, segment, batch, head, key tile u); it
// loops over the segment's query tiles t (t >= u when causal). The grid is
// persistent, one CTA per SM; CTAs take units from a global counter in
// group-major order: patterns with the most tiles first, then (segment,
// batch, head) groups, then u ascending, so the key tiles of one group run at
// the same time on different SMs and share its Q, dO tiles and dq rows in L2.
// Each query tile is handled as two halves h of 64
// queries so that the tensor pipe and the row threads overlap:
//   S^T_h  = K Q_h^T,  dP^T_h = V dO_h^T                   (TMEM x SMEM -> TMEM)
//   P^T_h  = exp2(S^T_h tau log2e - L log2e), dS^T_h = P^T_h (dP^T_h - D)  (threads)
//   dV += P^T_h dO_h,  dK += dS^T_h Q_h                    (TMEM x SMEM -> TMEM)
//   dQ  = dS K  (both halves; dS from SMEM)                (SMEM x SMEM -> TMEM)
// MMA issue order per pair i: dVdK_0(i), SdP_0(i+1), dQ(i), dVdK_1(i),
// SdP_1(i+1); the row threads work on half 1 of pair i while dVdK_0(i) and
// SdP_0(i+1) run, and on half 0 of pair i+1 while dVdK_1(i), dQ(i) and
// SdP_1(i+1) run. An S / dP half is overwritten only by MMAs issued after
// the MMAs that read its P / dS, and tcgen05 MMAs of one thread execute in
// issue order.
// P enters dV as bf16 and dS enters dK and dQ as fp16 (dS reaches tens, where
// bf16's 8 significant bits cost up to 2e-2 in dq and dk; q and k are
// converted exactly to fp16 for those products, and for S). On the first
// query tile of a segment (rows with few keys, where single probabilities
// approach 1) P enters dV and dS enters dK as two halves, hi + lo, so those
// products are fp32-grade. Elsewhere a row spreads its weight over at least
// 129 keys, and the rounding of P averages out far inside the bound.
// dQ goes through a double-buffered TMEM accumulator; after each pair every
// row warp stages its 32 x 32 block in a private shared-memory slab and adds
// it to the fp32 accumulator with a TMA reduce-add. dK, dV are added the same
// way once per unit (other patterns and tiles reach the same rows). The
// gradients are fp32 [B][N][H][64] tensors, reached through the same strided
// views as the inputs; they are the accumulators themselves.
//
// Warp roles (320 threads): warp 0 TMA producer (+ per-tile L and D rows and
// an L2 prefetch of the next unit's key tile), warp 1 TMEM allocator and MMA
// issuer, warps 2..9 the row work: warp w serves TMEM lanes 32 (w % 4) .. + 31
// (key rows) and column group cg = (w - 2) / 4, i.e. 32-column chunk 2h + cg
// of half h.
// Key tiles rotate through three shared-memory slots: unit k's K sits in slot
// k % 3 (the B operand of its dQ products) and its V in slot (k + 1) % 3 (read
// only by the copy into TMEM). Both of unit k + 1's slots are free once unit
// k's copy into TMEM has completed (that commit also covers every earlier MMA,
// unit k - 1's last dQ included), so the producer loads the next key tile
// while the current unit runs and the MMA thread moves from one unit to the
// next without waiting for a load. The row warps read dV and dK after the
// commit that follows the unit's last dV / dK products.
// TMEM columns: S^T [0,128) (half h at 64h), dP^T [128,256), dV [256,320),
// dK [320,384), dQ [384,448), the unit's K [448,480) and V [480,512) (fp16 and
// bf16 pairs). P^T and dS^T (hi, lo) overwrite S^T and dP^T in place: chunk
// q = [32q, 32q + 32) keeps hi at +[0,16) and lo at +[16,32).
// K and V are the A operands of every S^T and dP^T product of their unit, so
// at the start of a unit the MMA thread copies them from shared memory into
// TMEM (tcgen05.cp) and those products read only Q and dO from shared memory:
// half the operand bytes of a shared x shared product. One dQ accumulator
// suffices: the row warps read pair g's dQ out while they work on half 0 of
// pair g + 1, before dQ of pair g + 1 is issued.
#pragma once

#include "common.cuh"

namespace dil {

struct BwdParams {
  CUtensorMap tmq[kMaxPat], tmk[kMaxPat], tmv[kMaxPat], tmdo[kMaxPat];
  CUtensorMap tmq_t[kMaxPat], tmk_t[kMaxPat], tmv_t[kMaxPat], tmdo_t[kMaxPat];
  // reduce-add targets, the fp32 gradients [B][N][H][64] (32 x 32 boxes)
  CUtensorMap tmdq[kMaxPat], tmdk[kMaxPat], tmdv[kMaxPat];
  CUtensorMap tmdq_t[kMaxPat], tmdk_t[kMaxPat], tmdv_t[kMaxPat];
  PatternGeom pat[kMaxPat];
  int npat, B, N, H, causal;
  float scale_log2;  // log2(e) / sqrt(d)
  float tau;         // 1 / sqrt(d)
  int gorder[kMaxPat];           // patterns by tile count, descending
  long long gstart[kMaxPat + 1];  // first unit of each pattern in that order
  long long units;
  int* counter;                   // next unit to hand out (zeroed by the preprocess)
  const float* lse;   // [B][H][N] natural log
  const float* drow;  // [B][H][N]
  ErrCtx err;  // device error word and this launch's tag
};

struct BwdCfg {
  static constexpr int D = 64;
  // P and dS enter dV and dK as hi + lo on the first query tile of a segment
  __host__ __device__ static constexpr bool split(int t) { return t == 0; }
  static constexpr int ROW_WARPS = 8;
  static constexpr int THREADS = 64 + 32 * ROW_WARPS;
  static constexpr int TILE = BM * 128;   // 128 rows x 64 bf16
  static constexpr int HALF = TILE / 2;   // 64 rows
  static constexpr int SLAB = 32 * 128;   // one row warp's 32 x 32 fp32 staging block
  // K / V slots: unit k keeps K in slot k % 3 and V in slot (k + 1) % 3, so
  // the next unit's key tile loads while this unit runs
  static constexpr int KVS = 3;
  static constexpr int OFF_KV = 0;
  static constexpr int QST = 3;                               // Q / dO / L / D stages
  static constexpr int OFF_Q = OFF_KV + KVS * TILE;
  static constexpr int OFF_DO = OFF_Q + QST * TILE;
  static constexpr int OFF_DS = OFF_DO + QST * TILE;          // 2 halves x [128 keys][64 q]
  static constexpr int OFF_STG = OFF_DS + 2 * TILE;           // ROW_WARPS slabs
  static constexpr int OFF_L = OFF_STG + ROW_WARPS * SLAB;    // QST x 128 floats
  static constexpr int OFF_D = OFF_L + QST * BM * 4;          // QST x 128 floats
  static constexpr int OFF_BAR = OFF_D + QST * BM * 4;
  static constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;
  static constexpr int TM_S = 0, TM_DP = 128, TM_DV = 256, TM_DK = 320, TM_DQ = 384;
  static constexpr int TM_K = 448, TM_V = 480;
  static constexpr int TMEM_COLS = 512;
};
static_assert(BwdCfg::SMEM_BYTES <= 232448, "backward tile kernel exceeds shared memory");

// Row `row` of a [32][32] fp32 slab with 128-byte swizzle (16-byte piece k of
// the row lands at k ^ (row % 8)), scaled by `scale`.
__device__ __forceinline__ void stage_row32(uint8_t* slab, int row, const uint32_t (&r)[32],
                                            float scale) {
  uint8_t* rowp = slab + row * 128;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float4 v = make_float4(__uint_as_float(r[4 * k]) * scale,
                                 __uint_as_float(r[4 * k + 1]) * scale,
                                 __uint_as_float(r[4 * k + 2]) * scale,
                                 __uint_as_float(r[4 * k + 3]) * scale);
    *reinterpret_cast<float4*>(rowp + ((k ^ (row & 7)) * 16)) = v;
  }
}

// P^T and dS^T of queries [E0, E0 + NE) of a 32-query chunk of key row c:
// P = exp2(S tau log2e - L) (zero for e < jmin), dS = P (dP - D), packed to
// bf16 pairs at index (e - E0) / 2; with SPLIT also the bf16 remainders
// lo = x - hi.
template <bool SPLIT, int E0, int NE>
__device__ __forceinline__ void bwd_chunk(const uint32_t (&sv)[32], const uint32_t (&dv)[32],
                                          const float* sLq, const float* sDq, float sc, int jmin,
                                          uint32_t* pk, uint32_t* plo, uint32_t* dk, uint32_t* dkl) {
  const float4* L4 = reinterpret_cast<const float4*>(sLq);
  const float4* D4 = reinterpret_cast<const float4*>(sDq);
  const bool masked = jmin > 0;
  const uint64_t sc2 = f2_pack(sc, sc);
#pragma unroll
  for (int e4 = E0 / 4; e4 < (E0 + NE) / 4; ++e4) {
    const float4 Lq = L4[e4], Dq = D4[e4];
    const uint64_t nl2[2] = {f2_pack(-Lq.x, -Lq.y), f2_pack(-Lq.z, -Lq.w)};
    const uint64_t dd2[2] = {f2_pack(Dq.x, Dq.y), f2_pack(Dq.z, Dq.w)};
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const int e = 4 * e4 + 2 * h2;
      const int o = (e - E0) / 2;
      const uint64_t x2 =
          f2_fma(f2_pack(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), sc2, nl2[h2]);
      float p0 = ex2(f2_lo(x2)), p1 = ex2(f2_hi(x2));
      if (masked) {
        p0 = e >= jmin ? p0 : 0.f;
        p1 = e + 1 >= jmin ? p1 : 0.f;
      }
      const uint64_t p2 = f2_pack(p0, p1);
      const uint64_t ds2 = f2_mul(
          p2, f2_sub(f2_pack(__uint_as_float(dv[e]), __uint_as_float(dv[e + 1])), dd2[h2]));
      const uint32_t hi = pack_bf16_rn(p0, p1);
      const uint32_t dhi = pack_f16_rn(f2_lo(ds2), f2_hi(ds2));
      pk[o] = hi;
      dk[o] = dhi;
      if (SPLIT) {
        const uint64_t lo2 =
            f2_sub(p2, f2_pack(__uint_as_float(hi << 16), __uint_as_float(hi & 0xffff0000u)));
        plo[o] = pack_bf16_rn(f2_lo(lo2), f2_hi(lo2));
        const uint64_t dlo2 = f2_sub(ds2, f2_pack(f16_lo(dhi), f16_hi(dhi)));
        dkl[o] = pack_f16_rn(f2_lo(dlo2), f2_hi(dlo2));
      }
    }
  }
}

// One backward unit: (pattern, segment, batch, head, key tile u) and the
// views its tiles are read through. False when the key tile holds no row.
struct BwdUnit {
  TileUnit wu;
  PatternGeom g;
  SegInfo si;
  int u, t0, np;
  const CUtensorMap *mq, *mk, *mv, *mdo, *mdq, *mdk, *mdv;
};

__device__ __forceinline__ bool bwd_unit(const BwdParams& p, long long uu, BwdUnit& U) {
  int a = 0;
  while (a + 1 < p.npat && uu >= p.gstart[a + 1]) ++a;
  const int i = p.gorder[a];
  // the host rejects 2^31 units or more: 32-bit unsigned arithmetic (fast divisions)
  uint32_t rem = (uint32_t)(uu - p.gstart[a]);
  U.g = p.pat[i];
  const uint32_t q1 = rem / (uint32_t)U.g.ntiles;
  U.u = (int)(rem - q1 * (uint32_t)U.g.ntiles);  // key tile; long (small u) tiles come first
  U.wu.pat = i;
  U.wu.t = U.u;
  const uint32_t q2 = q1 / (uint32_t)p.H;
  U.wu.h = (int)(q1 - q2 * (uint32_t)p.H);
  const uint32_t q3 = q2 / (uint32_t)p.B;
  U.wu.b = (int)(q2 - q3 * (uint32_t)p.B);
  U.wu.seg = (int)q3;
  U.si = seg_info(U.g, p.N, U.wu.h, U.wu.seg);
  const int nq = (U.si.n + BM - 1) / BM;
  if (U.u >= nq) return false;
  U.t0 = p.causal ? U.u : 0;
  U.np = nq - U.t0;
  // all tiles of a (pattern, segment, head) share one phase, hence one view
  int ph0, m0;
  view_coords(U.g, U.si, 0, ph0, m0);
  const bool tv = ph0 < U.g.nmod;
  U.mq = tv ? &p.tmq_t[i] : &p.tmq[i];
  U.mk = tv ? &p.tmk_t[i] : &p.tmk[i];
  U.mv = tv ? &p.tmv_t[i] : &p.tmv[i];
  U.mdo = tv ? &p.tmdo_t[i] : &p.tmdo[i];
  U.mdq = tv ? &p.tmdq_t[i] : &p.tmdq[i];
  U.mdk = tv ? &p.tmdk_t[i] : &p.tmdk[i];
  U.mdv = tv ? &p.tmdv_t[i] : &p.tmdv[i];
  return true;
}

__global__ void __launch_bounds__(BwdCfg::THREADS, 1) bwd_tile_kernel(const __grid_constant__ BwdParams p) {
  using C = BwdCfg;
  constexpr int D = C::D;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t base = (raw_s + 1023u) & ~1023u;
  uint8_t* base_g = smem_raw + (base - raw_s);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t sKV = base + C::OFF_KV;
  const uint32_t sQ = base + C::OFF_Q, sDO = base + C::OFF_DO, sDS = base + C::OFF_DS;
  float* sL = reinterpret_cast<float*>(base_g + C::OFF_L);
  float* sD = reinterpret_cast<float*>(base_g + C::OFF_D);
  const uint32_t bars = base + C::OFF_BAR;
  const uint32_t b_kvfull = bars;         // K, V of the unit landed
  // K, V of the unit copied into TMEM, and every MMA issued before that
  // complete: the previous unit's V slot and the unit before's K slot are free
  const uint32_t b_cpdone = bars + 8u;
  const uint32_t b_accdone = bars + 16u;  // every MMA of the unit is complete (dV, dK final)
  auto b_qfull = [&](int s) { return bars + 144u + 8u * s; };   // Q, dO, L, D of stage s
  auto b_qempty = [&](int s) { return bars + 168u + 8u * s; };
  auto b_sdp = [&](int h) { return bars + 48u + 8u * h; };      // S^T_h, dP^T_h in TMEM
  auto b_rows = [&](int h) { return bars + 64u + 8u * h; };     // P^T_h, dS^T_h written
  auto b_dq = [&](int j) { return bars + 80u + 8u * j; };       // dQ of pairs g = j mod 2 complete
  auto b_dqfree = [&](int j) { return bars + 96u + 8u * j; };   // dQ of pairs g = j mod 2 read out
  const uint32_t b_accfree = bars + 112u;  // dV, dK of the unit read out
  const uint32_t b_fin = bars + 120u;      // MMA pipe drained at exit
  auto b_unit = [&](int j) { return bars + 192u + 8u * j; };    // unit index published in slot j
  volatile int* uslot = reinterpret_cast<volatile int*>(base_g + C::OFF_BAR + 232);  // 4 slots
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_g + C::OFF_BAR + 224);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base_g + C::OFF_BAR + 228);

  if (threadIdx.x == 0) {
    mbar_init(b_kvfull, 1);
    mbar_init(b_cpdone, 1);
    mbar_init(b_accdone, 1);
    for (int s = 0; s < C::QST; ++s) {
      mbar_init(b_qfull(s), 1);
      mbar_init(b_qempty(s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(b_sdp(s), 1);
      mbar_init(b_rows(s), C::ROW_WARPS);
      mbar_init(b_dq(s), 1);
      mbar_init(b_dqfree(s), C::ROW_WARPS);
    }
    mbar_init(b_accfree, C::ROW_WARPS);
    mbar_init(b_fin, 1);
    for (int j = 0; j < 4; ++j) mbar_init(b_unit(j), 1);
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
  const float log2e = 1.4426950408889634f;
  // The producer takes units from the global counter one ahead of use and
  // publishes each in slot k & 3 (phase k >> 2); p.units marks the end. It
  // publishes unit k + 2 only after unit k's K and V were copied into TMEM,
  // when the row warps are at unit k - 1 or later; they read slot k & 3 at
  // the start of unit k, before it is rewritten with unit k + 4.

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    uint32_t gp = 0, k = 0;  // pairs and units issued so far
    bool ok = true;
    // next unit with key rows, or p.units when none is left (lane 0)
    auto fetch = [&]() -> long long {
      for (;;) {
        const long long x = atomicAdd(p.counter, 1);
        BwdUnit t;
        if (x >= p.units) return p.units;
        if (bwd_unit(p, x, t)) return x;
      }
    };
    long long cur = 0;
    if (lane == 0) {
      cur = fetch();
      uslot[0] = (int)cur;
      mbar_arrive(b_unit(0));
    }
    cur = __shfl_sync(0xffffffffu, cur, 0);
    while (cur < p.units) {
      BwdUnit U;
      bwd_unit(p, cur, U);
      // unit k's slots held V of unit k - 1 and K of unit k - 2
      if (k > 0 && !warp_wait(b_cpdone, (k - 1) & 1, abort_flag, p.err)) {
        ok = false;
        break;
      }
      long long nxt = 0;
      if (lane == 0) {
        nxt = fetch();
        uslot[(k + 1) & 3] = (int)nxt;
        mbar_arrive(b_unit((k + 1) & 3));
        int ph, m;
        view_coords(U.g, U.si, U.u * BN, ph, m);
        mbar_arrive_expect_tx(b_kvfull, 2 * C::TILE);
        tma_load_5d(sKV + (k % C::KVS) * C::TILE, U.mk, b_kvfull, 0, U.wu.h, ph, m, U.wu.b);
        tma_load_5d(sKV + ((k + 1) % C::KVS) * C::TILE, U.mv, b_kvfull, 0, U.wu.h, ph, m, U.wu.b);
        BwdUnit nx;
        if (nxt < p.units && bwd_unit(p, nxt, nx)) {  // warm the L2 for the next unit
          view_coords(nx.g, nx.si, nx.u * BN, ph, m);
          tma_prefetch_l2_5d(nx.mk, 0, nx.wu.h, ph, m, nx.wu.b);
          tma_prefetch_l2_5d(nx.mv, 0, nx.wu.h, ph, m, nx.wu.b);
          view_coords(nx.g, nx.si, nx.t0 * BM, ph, m);
          tma_prefetch_l2_5d(nx.mq, 0, nx.wu.h, ph, m, nx.wu.b);
          tma_prefetch_l2_5d(nx.mdo, 0, nx.wu.h, ph, m, nx.wu.b);
        }
      }
      nxt = __shfl_sync(0xffffffffu, nxt, 0);
      ++k;
      const long long lrow0 = ((long long)U.wu.b * p.H + U.wu.h) * p.N;  // lse / D row base
      // merged lse (log2 units) and D of query tile t, lane j holding rows
      // j + 32 jj; rows past the segment get L = +inf, so their probabilities
      // are exactly zero. Loaded one pair ahead, so the gather overlaps the wait.
      float Lr[BM / 32], Dr[BM / 32];
      auto load_ld = [&](int t) {
#pragma unroll
        for (int jj = 0; jj < BM / 32; ++jj) {
          const int vq = t * BM + lane + 32 * jj;
          Lr[jj] = INFINITY;
          Dr[jj] = 0.f;
          if (vq < U.si.n) {
            const long long pos = U.si.start + U.si.off + (long long)vq * U.g.r;
            Lr[jj] = p.lse[lrow0 + pos] * log2e;
            Dr[jj] = p.drow[lrow0 + pos];
          }
        }
      };
      load_ld(U.t0);
      for (int it = 0; it < U.np; ++it, ++gp) {
        const int s = gp % C::QST;
        const int t = U.t0 + it;
        if (!warp_wait(b_qempty(s), ((gp / C::QST) & 1) ^ 1, abort_flag, p.err)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          int ph, m;
          view_coords(U.g, U.si, t * BM, ph, m);
          mbar_expect_tx(b_qfull(s), 2 * C::TILE);
          tma_load_5d(sQ + s * C::TILE, U.mq, b_qfull(s), 0, U.wu.h, ph, m, U.wu.b);
          tma_load_5d(sDO + s * C::TILE, U.mdo, b_qfull(s), 0, U.wu.h, ph, m, U.wu.b);
          if (it + 2 < U.np) {  // warm the L2 two pairs ahead
            view_coords(U.g, U.si, (t + 2) * BM, ph, m);
            tma_prefetch_l2_5d(U.mq, 0, U.wu.h, ph, m, U.wu.b);
            tma_prefetch_l2_5d(U.mdo, 0, U.wu.h, ph, m, U.wu.b);
          }
        }
#pragma unroll
        for (int jj = 0; jj < BM / 32; ++jj) {
          sL[s * BM + lane + 32 * jj] = Lr[jj];
          sD[s * BM + lane + 32 * jj] = Dr[jj];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(b_qfull(s));  // the phase ends once the copies land too
        if (it + 1 < U.np) load_ld(t + 1);
      }
      if (!ok) break;
      cur = nxt;
    }
    if (!ok && lane == 0) {
      // Drain copies still in flight before the CTA's shared memory goes away.
      volatile int no_abort = 0;
      if (k > 0) mbar_wait(b_kvfull, (k - 1) & 1, &no_abort, ErrCtx{}, 200000000ull);
      for (uint32_t g = (gp >= C::QST ? gp - C::QST : 0); g < gp; ++g)
        mbar_wait(b_qfull(g % C::QST), (g / C::QST) & 1, &no_abort, ErrCtx{}, 200000000ull);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop; one elected lane issues each MMA group.
    {
      // Q, K (and dS) are fp16, V, dO (and P) bf16: every product has one type
      constexpr uint32_t kIdS = idesc_f16(BM, 64, 0, 0);    // K (TMEM) x Q_h^T
      constexpr uint32_t kIdDP = idesc_bf16(BM, 64, 0, 0);  // V (TMEM) x dO_h^T
      constexpr uint32_t kIdV = idesc_bf16(BM, D, 0, 1);    // P^T (TMEM) x dO
      constexpr uint32_t kIdK = idesc_f16(BM, D, 0, 1);     // dS^T (TMEM) x Q
      constexpr uint32_t kIdQ = idesc_f16(BM, D, 1, 1);     // dS (MN-major SMEM) x K
      // Descriptors are built once (the K / V slot ones once per unit); each
      // MMA only adds a byte offset to the low word, which keeps the issuing
      // thread's work per MMA small (it shares its scheduler with two row warps).
      const SDesc dQk = sdesc_sw128(sQ, 16, 1024), dDOk = sdesc_sw128(sDO, 16, 1024);
      const SDesc dQm = sdesc_sw128(sQ, C::TILE, 1024), dDOm = sdesc_sw128(sDO, C::TILE, 1024);
      const SDesc dDSm = sdesc_sw128(sDS, C::TILE, 1024);
      SDesc dKm = sdesc_sw128(sKV, C::TILE, 1024);
      // unit k's K and V (slots k % 3, (k + 1) % 3) into TMEM, 16 columns of
      // a row per copy; K stays in its slot as the B operand of dQ
      auto copy_kv = [&](uint32_t k) {
        const uint32_t sK = sKV + (k % C::KVS) * C::TILE, sV = sKV + ((k + 1) % C::KVS) * C::TILE;
        const SDesc dKk = sdesc_sw128(sK, 16, 1024), dVk = sdesc_sw128(sV, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          tmem_cp_128x256b(tmem + C::TM_K + kk * 8, dKk.at(kk * 32));
          tmem_cp_128x256b(tmem + C::TM_V + kk * 8, dVk.at(kk * 32));
        }
      };
      // S^T_h = K Q_h^T and dP^T_h = V dO_h^T for the 64 queries of half h
      auto issue_sdp = [&](uint32_t g, int h) {
        const uint32_t qo = (g % C::QST) * C::TILE + h * C::HALF;
        const uint32_t ts = tmem + C::TM_S + h * 64, tp = tmem + C::TM_DP + h * 64;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ts(ts, tmem + C::TM_K + kk * 8, dQk.at(qo + kk * 32), kIdS, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ts(tp, tmem + C::TM_V + kk * 8, dDOk.at(qo + kk * 32), kIdDP, kk > 0 ? 1u : 0u);
        mma_commit(b_sdp(h));
      };
      // dV += P^T_h dO_h, dK += dS^T_h Q_h (each hi + lo when `split`); `first`
      // starts the accumulators
      auto issue_dvdk = [&](uint32_t g, int h, bool first, bool split) {
        const uint32_t qo = (g % C::QST) * C::TILE;
#pragma unroll
        for (int kq = 0; kq < 4; ++kq) {
          const int kk = 4 * h + kq;  // 16 queries
          const uint64_t bdo = dDOm.at(qo + kk * 2048);
          const uint32_t a = tmem + C::TM_S + (kk >> 1) * 32 + (kk & 1) * 8;
          mma_ts(tmem + C::TM_DV, a, bdo, kIdV, (first && kq == 0) ? 0u : 1u);
          if (split) mma_ts(tmem + C::TM_DV, a + 16, bdo, kIdV, 1u);
        }
#pragma unroll
        for (int kq = 0; kq < 4; ++kq) {
          const int kk = 4 * h + kq;
          const uint64_t bq = dQm.at(qo + kk * 2048);
          const uint32_t a = tmem + C::TM_DP + (kk >> 1) * 32 + (kk & 1) * 8;
          mma_ts(tmem + C::TM_DK, a, bq, kIdK, (first && kq == 0) ? 0u : 1u);
          if (split) mma_ts(tmem + C::TM_DK, a + 16, bq, kIdK, 1u);
        }
      };
      // dQ = dS K into the TMEM accumulator (dS from shared memory)
      auto issue_dq = [&](uint32_t g) {
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          mma_ss(tmem + C::TM_DQ, dDSm.at(kk * 2048), dKm.at(kk * 2048), kIdQ, kk > 0 ? 1u : 0u);
        mma_commit(b_dq(g & 1));
      };
      uint32_t gp = 0, k = 0;
      bool ok = true;
      for (;; ++k) {
        if (!warp_wait(b_unit(k & 3), (k >> 2) & 1, abort_flag, p.err)) break;
        const long long uu = uslot[k & 3];
        if (uu >= p.units) break;
        BwdUnit U;
        bwd_unit(p, uu, U);
        dKm = sdesc_sw128(sKV + (k % C::KVS) * C::TILE, C::TILE, 1024);
        if (!warp_wait(b_kvfull, k & 1, abort_flag, p.err) ||
            !warp_wait(b_qfull(gp % C::QST), (gp / C::QST) & 1, abort_flag, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // The previous unit's S^T / dP^T products, the only readers of the
        // TMEM copies of K and V, are complete: the row warps have read them.
        if (elect_one_sync()) {
          copy_kv(k);
          mma_commit(b_cpdone);
          issue_sdp(gp, 0);
          issue_sdp(gp, 1);
        }
        __syncwarp();
        for (int it = 0; it < U.np; ++it, ++gp) {
          const bool more = it + 1 < U.np;
          if (!warp_wait(b_rows(0), gp & 1, abort_flag, p.err) ||
              (it == 0 && k > 0 && !warp_wait(b_accfree, (k - 1) & 1, abort_flag, p.err))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const bool split = C::split(U.t0 + it);
          if (elect_one_sync()) issue_dvdk(gp, 0, it == 0, split);
          __syncwarp();
          // Then S / dP half 0 of the next pair (its Q, dO have landed: the
          // producer runs up to three pairs ahead), and dV / dK half 1 plus dQ
          // of this pair once half 1 is written and the dQ accumulator read
          // out. Both waits suspend the warp in hardware, leaving its
          // scheduler's issue slots to the row warps that share it. S / dP
          // half 1 of the next pair goes last: it overwrites what dV / dK
          // half 1 reads.
          if (more) {
            if (!warp_wait(b_qfull((gp + 1) % C::QST), ((gp + 1) / C::QST) & 1, abort_flag, p.err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            if (elect_one_sync()) issue_sdp(gp + 1, 0);
            __syncwarp();
          }
          if (!warp_wait(b_rows(1), gp & 1, abort_flag, p.err) ||
              (gp >= 1 && !warp_wait(b_dqfree((gp - 1) & 1), ((gp - 1) >> 1) & 1, abort_flag, p.err))) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (elect_one_sync()) {
            issue_dq(gp);  // first: the row warps wait for it before their next dS store
            issue_dvdk(gp, 1, false, split);
            mma_commit(b_qempty(gp % C::QST));
          }
          __syncwarp();
          if (!ok) break;
          if (elect_one_sync()) {
            if (more) issue_sdp(gp + 1, 1);
            else mma_commit(b_accdone);
          }
          __syncwarp();
        }
        if (!ok) break;
      }
      // every MMA issued so far completes before TMEM is released
      if (elect_one_sync()) mma_commit(b_fin);
      __syncwarp();
      volatile int no_abort = 0;
      mbar_wait(b_fin, 0, &no_abort, ErrCtx{}, 200000000ull);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ row warps
    const int rw = warp - 2;
    const int q4 = warp & 3;   // TMEM lane quarter
    const int cg = rw >> 2;    // column group
    const int c = q4 * 32 + lane;  // key row of S^T / dP^T / dV / dK, query row of dQ
    const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
    uint8_t* slab_g = base_g + C::OFF_STG + rw * C::SLAB;
    const uint32_t slab = base + C::OFF_STG + rw * C::SLAB;
    const float sc = p.scale_log2;
    uint32_t gp = 0;
    bool ok = true;
    // dQ of pair g (query tile t): this warp's 32 x 32 block -> slab -> TMA
    // reduce-add into the fp32 dq accumulator. Rows past the segment hold
    // exact zeros (their P is 0); rows past N are clipped by the view.
    auto dq_out = [&](const BwdUnit& U, uint32_t g, int t) -> bool {
      const int j = g & 1;
      if (!warp_wait(b_dq(j), (g >> 1) & 1, abort_flag, p.err)) return false;
      tc_fence_after();
      uint32_t r[32];
      tmem_ld32_sync(tl + C::TM_DQ + cg * 32, r);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(b_dqfree(j));
        bulk_wait_read<0>();  // this warp's previous reduce has read the slab
      }
      __syncwarp();
      stage_row32(slab_g, lane, r, p.tau);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        int ph, m;
        view_coords(U.g, U.si, t * BM + q4 * 32, ph, m);
        tma_reduce_add_5d(U.mdq, slab, cg * 32, U.wu.h, ph, m, U.wu.b);
        bulk_commit();
      }
      return true;
    };
    for (uint32_t k = 0; ok; ++k) {
      if (!warp_wait(b_unit(k & 3), (k >> 2) & 1, abort_flag, p.err)) break;
      const long long uu = uslot[k & 3];
      if (uu >= p.units) break;
      BwdUnit U;
      bwd_unit(p, uu, U);
      const bool key_valid = U.u * BN + c < U.si.n;
      int tprev = 0;
      for (int it = 0; it < U.np; ++it, ++gp) {
        const int s = gp % C::QST;
        const int t = U.t0 + it;
        const bool diag = p.causal && t == U.u;
        if (!warp_wait(b_qfull(s), (gp / C::QST) & 1, abort_flag, p.err)) {
          ok = false;
          break;
        }
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          if (!warp_wait(b_sdp(h), gp & 1, abort_flag, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int q = 2 * h + cg;  // this thread's 32 query columns: [32q, 32q + 32)
          const bool split = C::split(t);
          // key rows past the segment, and (on the diagonal) queries before the
          // key, get P = 0; elsewhere no mask is needed
          const int jmin = !key_valid ? 1 << 30 : (diag ? c - q * 32 : 0);
          const float* sLq = sL + s * BM + q * 32;
          const float* sDq = sD + s * BM + q * 32;
          // dS (query-major) into shared memory for dQ = dS K: row c of half h
          // holds dS[64h + j][c] for its 64 queries j, 16-byte pieces
          // XOR-swizzled by c % 8
          uint8_t* dsrow = base_g + C::OFF_DS + h * C::TILE + c * 128;
          uint32_t dk[16];
          {
            uint32_t sv[32], dv[32];
            tmem_ld32x2_sync(tl + C::TM_S + q * 32, tl + C::TM_DP + q * 32, sv, dv);
            // P^T, dS^T go in place over this chunk's own (already read) columns
            if (!split) {
              uint32_t pk[16];
              bwd_chunk<false, 0, 32>(sv, dv, sLq, sDq, sc, jmin, pk, nullptr, dk, nullptr);
              tmem_st16(tl + C::TM_S + q * 32, pk);
              tmem_st16(tl + C::TM_DP + q * 32, dk);
            } else {
              // two 16-query halves; hi at +[0,16), lo at +[16,32): every column
              // is already in registers before any store
              {
                uint32_t pk[8], plo[8], dkl[8];
                bwd_chunk<true, 0, 16>(sv, dv, sLq, sDq, sc, jmin, pk, plo, dk, dkl);
                tmem_st8(tl + C::TM_S + q * 32, pk);
                tmem_st8(tl + C::TM_S + q * 32 + 16, plo);
                tmem_st8(tl + C::TM_DP + q * 32, dk);
                tmem_st8(tl + C::TM_DP + q * 32 + 16, dkl);
              }
              {
                uint32_t pk[8], plo[8], dkl[8];
                bwd_chunk<true, 16, 16>(sv, dv, sLq, sDq, sc, jmin, pk, plo, dk + 8, dkl);
                tmem_st8(tl + C::TM_S + q * 32 + 8, pk);
                tmem_st8(tl + C::TM_S + q * 32 + 24, plo);
                tmem_st8(tl + C::TM_DP + q * 32 + 8, dk + 8);
                tmem_st8(tl + C::TM_DP + q * 32 + 24, dkl);
              }
            }
          }
          auto store_ds = [&]() {
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4)
              *reinterpret_cast<uint4*>(dsrow + (((cg * 4 + k4) ^ (c & 7)) * 16)) =
                  make_uint4(dk[4 * k4], dk[4 * k4 + 1], dk[4 * k4 + 2], dk[4 * k4 + 3]);
          };
          // The single dS buffer is free once the previous pair's dQ MMA has
          // completed: half 0 waits for that in dq_out below (except on a
          // unit's first pair, where the previous unit's last dq_out did).
          if (h == 1 || it == 0) store_ds();
          tmem_wait_st();
          fence_proxy_async_smem();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(b_rows(h));
          // the previous pair's dQ leaves while the tensor pipe works on this one
          if (h == 0 && it > 0) {
            if (!dq_out(U, gp - 1, tprev)) {
              ok = false;
              break;
            }
            store_ds();
          }
        }
        if (!ok) break;
        tprev = t;
      }
      if (!ok || !dq_out(U, gp - 1, tprev)) {
        ok = false;
        break;
      }
      // dV, dK of the key tile, once the unit's last dV / dK products are
      // complete (they are issued after the last dQ, so its commit does not
      // cover them). Rows past the segment are exact zeros (their P was forced
      // to 0).
      if (!warp_wait(b_accdone, k & 1, abort_flag, p.err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      {
        uint32_t rv[32], rk[32];
        tmem_ld32_sync(tl + C::TM_DV + cg * 32, rv);
        tmem_ld32_sync(tl + C::TM_DK + cg * 32, rk);
        tc_fence_before();
        __syncwarp();
        int ph, m;
        view_coords(U.g, U.si, U.u * BN + q4 * 32, ph, m);
        if (lane == 0) {
          mbar_arrive(b_accfree);
          bulk_wait_read<0>();
        }
        __syncwarp();
        stage_row32(slab_g, lane, rv, 1.f);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_5d(U.mdv, slab, cg * 32, U.wu.h, ph, m, U.wu.b);
          bulk_commit();
          bulk_wait_read<0>();
        }
        __syncwarp();
        stage_row32(slab_g, lane, rk, p.tau);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_5d(U.mdk, slab, cg * 32, U.wu.h, ph, m, U.wu.b);
          bulk_commit();
        }
      }
    }
    if (lane == 0) bulk_wait_all();  // shared memory stays until the reduces finish
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// D = rowsum(dO * O) per (b, h, n) from out + out_res (O to about 16
// significant bits), and zeroed fp32 gradients; one warp per row.
struct PrepParams {
  int B, N, H;
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  __half* q16;  // fp16 copies of q and k for the products with dS
  __half* k16;
  ErrCtx err;   // a value outside the fp16 range records kErrF16Range
  const __nv_bfloat16* out;
  const __nv_bfloat16* out_res;  // bf16(O - out) from the training forward
  const __nv_bfloat16* dout;
  float* drow;
  float* dq;
  float* dk;
  float* dv;
  int* counter;  // the key-tile kernel's unit counter
};

__global__ void __launch_bounds__(256) bwd_prep_kernel(PrepParams p) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row == 0 && threadIdx.x == 0) *p.counter = 0;
  if (row >= (long long)p.B * p.N * p.H) return;
  const __nv_bfloat162 d = reinterpret_cast<const __nv_bfloat162*>(p.dout + row * 64)[lane];
  const __nv_bfloat162 ob = reinterpret_cast<const __nv_bfloat162*>(p.out + row * 64)[lane];
  const __nv_bfloat162 rb = reinterpret_cast<const __nv_bfloat162*>(p.out_res + row * 64)[lane];
  const float o0 = __low2float(ob) + __low2float(rb), o1 = __high2float(ob) + __high2float(rb);
  float acc = o0 * __low2float(d) + o1 * __high2float(d);
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
  {
    const __nv_bfloat162 a = reinterpret_cast<const __nv_bfloat162*>(p.q + row * 64)[lane];
    const __nv_bfloat162 b = reinterpret_cast<const __nv_bfloat162*>(p.k + row * 64)[lane];
    const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    if (fmaxf(fmaxf(fabsf(fa.x), fabsf(fa.y)), fmaxf(fabsf(fb.x), fabsf(fb.y))) > 65504.f)
      p.err.raise(kErrF16Range);
    reinterpret_cast<__half2*>(p.q16 + row * 64)[lane] = __float22half2_rn(fa);
    reinterpret_cast<__half2*>(p.k16 + row * 64)[lane] = __float22half2_rn(fb);
  }
  const float2 z = make_float2(0.f, 0.f);
  reinterpret_cast<float2*>(p.dq + row * 64)[lane] = z;
  reinterpret_cast<float2*>(p.dk + row * 64)[lane] = z;
  reinterpret_cast<float2*>(p.dv + row * 64)[lane] = z;
  if (lane == 0) {
    const int h = (int)(row % p.H);
    const long long bn = row / p.H;
    const int n = (int)(bn % p.N);
    const int b = (int)(bn / p.N);
    p.drow[((long long)b * p.H + h) * p.N + n] = acc;
  }
}

}  // namespace dil
