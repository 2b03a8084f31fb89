// CUDA-core kernels: the cross-pattern merge, the row-selection map, and the
// fp32 forward / backward (one thread per output row).
#pragma once

#include "common.cuh"

namespace dil {

struct RowParams {
  PatternGeom pat[kMaxPat];
  int npat, B, N, H, causal;
  float tau;  // 1 / sqrt(d)
};

// Where row n of head h sits in pattern g: segment, kept index, and whether
// the pattern keeps it. Inverse of seg_info's position map.
struct RowPos {
  bool kept;
  int seg;
  int v;
  long long start;
  long long end;
  int off;
};

__device__ __forceinline__ RowPos row_pos(const PatternGeom& g, int N, int h, int n) {
  RowPos rp;
  rp.seg = n / g.w;
  rp.start = (long long)rp.seg * g.w;
  rp.end = rp.start + g.w;
  if (rp.end > N) rp.end = N;
  rp.off = h % g.r;
  const long long rel = n - rp.start - rp.off;
  rp.kept = rel >= 0 && (rel % g.r) == 0;
  rp.v = rp.kept ? (int)(rel / g.r) : -1;
  return rp;
}

// ---------------------------------------------------------------------------
// Merge of per-pattern partials: L = log sum_i exp(lse_i),
// O = sum_i exp(lse_i - L) O_i.
// ---------------------------------------------------------------------------
struct MergeParams {
  PatternGeom pat[kMaxPat];
  int npat, B, N, H;
  const float* part_o;
  const float* part_lse;
  __nv_bfloat16* out;
  __nv_bfloat16* out_res;  // bf16(O - out), may be null
  float* lse;              // may be null
};

// kMergeTpr threads per output row (8 and 16 were measured slower at d = 64),
// each owning D / kMergeTpr consecutive columns; 256 / kMergeTpr rows per
// 256-thread block. Single pass with a running max, so every partial load is
// independent of the previous pattern's result.
constexpr int kMergeTpr = 4;
template <int D>
__global__ void __launch_bounds__(256) merge_kernel(const __grid_constant__ MergeParams p) {
  constexpr int TPR = kMergeTpr;  // threads per output row
  constexpr int PER = D / TPR;            // floats per thread
  static_assert(PER % 4 == 0, "each thread owns whole float4 groups");
  const long long row = (long long)blockIdx.x * (256 / TPR) + (threadIdx.x / TPR);
  const int sub = threadIdx.x % TPR;
  const long long total = (long long)p.B * p.N * p.H;
  if (row >= total) return;
  const int h = (int)(row % p.H);
  const long long bn = row / p.H;
  const int n = (int)(bn % p.N);
  const int b = (int)(bn / p.N);
  const int bh = b * p.H + h;

  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  float m = -INFINITY, l = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxPat; ++i) {
    if (i >= p.npat) break;
    const PatternGeom& g = p.pat[i];
    const int seg = n / g.w;
    const int rel = n - seg * g.w - h % g.r;
    if (rel < 0 || rel % g.r != 0) continue;
    const long long pr = g.part_base + ((long long)bh * g.nseg + seg) * g.pstride + rel / g.r;
    const float li = __ldg(p.part_lse + pr);
    const float4* src = reinterpret_cast<const float4*>(p.part_o + pr * D + sub * PER);
    float4 x[PER / 4];
#pragma unroll
    for (int e = 0; e < PER / 4; ++e) x[e] = __ldg(src + e);
    // running merge of normalised partials: weights exp(li - m) relative to the running max
    const float m_new = fmaxf(m, li);
    const float c_old = expf(m - m_new);  // 0 on the first kept pattern
    const float c_new = expf(li - m_new);
    l = l * c_old + c_new;
#pragma unroll
    for (int e = 0; e < PER / 4; ++e) {
      acc[4 * e] = acc[4 * e] * c_old + c_new * x[e].x;
      acc[4 * e + 1] = acc[4 * e + 1] * c_old + c_new * x[e].y;
      acc[4 * e + 2] = acc[4 * e + 2] * c_old + c_new * x[e].z;
      acc[4 * e + 3] = acc[4 * e + 3] * c_old + c_new * x[e].w;
    }
    m = m_new;
  }
  float L = -INFINITY;
  if (l > 0.f) {
    const float inv = 1.f / l;
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] *= inv;
    L = m + logf(l);
  }
  uint32_t pk[PER / 2], rk[PER / 2];
#pragma unroll
  for (int e = 0; e < PER / 2; ++e) {
    pk[e] = pack_bf16(acc[2 * e], acc[2 * e + 1]);
    rk[e] = pack_bf16(acc[2 * e] - __uint_as_float(pk[e] << 16),
                      acc[2 * e + 1] - __uint_as_float(pk[e] & 0xffff0000u));
  }
  if (PER % 8 == 0) {
    uint4* dst = reinterpret_cast<uint4*>(p.out + row * D + sub * PER);
    uint4* rdst = p.out_res != nullptr ? reinterpret_cast<uint4*>(p.out_res + row * D + sub * PER)
                                       : nullptr;
#pragma unroll
    for (int e = 0; e < PER / 8; ++e) {
      dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
      if (rdst != nullptr) rdst[e] = make_uint4(rk[4 * e], rk[4 * e + 1], rk[4 * e + 2], rk[4 * e + 3]);
    }
  } else {
    uint2* dst = reinterpret_cast<uint2*>(p.out + row * D + sub * PER);
    uint2* rdst = p.out_res != nullptr ? reinterpret_cast<uint2*>(p.out_res + row * D + sub * PER)
                                       : nullptr;
#pragma unroll
    for (int e = 0; e < PER / 4; ++e) {
      dst[e] = make_uint2(pk[2 * e], pk[2 * e + 1]);
      if (rdst != nullptr) rdst[e] = make_uint2(rk[2 * e], rk[2 * e + 1]);
    }
  }
  if (p.lse != nullptr && sub == 0) p.lse[(long long)bh * p.N + n] = L;
}

// ---------------------------------------------------------------------------
// Dilated rows of one rank's block for a sequence-parallel pattern:
// buf[b][m][h] = x[b][(h mod r) + m r][h] for m < L / r (rows of 16-byte
// pieces; pieces = d / 8 per row).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) pack_dilated_kernel(const uint4* __restrict__ x,
                                                           uint4* __restrict__ buf, int B, int L,
                                                           int H, int pieces, int r) {
  const long long Lr = L / r;
  const long long total = (long long)B * Lr * H * pieces;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(i % pieces);
    long long t = i / pieces;
    const int h = (int)(t % H);
    t /= H;
    const long long m = t % Lr;
    const long long b = t / Lr;
    const long long src_row = b * L + (h % r) + m * r;
    buf[i] = x[(src_row * H + h) * pieces + c];
  }
}

// ---------------------------------------------------------------------------
// Selection map: enumerate the kept rows of (pattern, head, segment) with the
// same seg_info used by the tile kernels and set bit i at [h][pos].
// ---------------------------------------------------------------------------
__global__ void selection_kernel(PatternGeom g, int i, int N, int H, uint32_t* sig) {
  const int h = blockIdx.x % H;
  const int s = blockIdx.x / H;
  const SegInfo si = seg_info(g, N, h, s);
  for (int v = blockIdx.y * blockDim.x + threadIdx.x; v < si.n; v += gridDim.y * blockDim.x) {
    const long long pos = si.start + si.off + (long long)v * g.r;
    atomicOr(sig + (long long)h * N + pos, 1u << i);
  }
}

// ---------------------------------------------------------------------------
// fp32 path: one thread per (b, n, h) row, exact fp32 FMA, accurate expf.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128) fwd_f32_kernel(const __grid_constant__ RowParams p,
                                                      const float* __restrict__ q,
                                                      const float* __restrict__ k,
                                                      const float* __restrict__ v,
                                                      float* __restrict__ out,
                                                      float* __restrict__ lse) {
  const long long row = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long total = (long long)p.B * p.N * p.H;
  if (row >= total) return;
  const int h = (int)(row % p.H);
  const int n = (int)((row / p.H) % p.N);
  const int b = (int)(row / ((long long)p.H * p.N));
  const long long hstride = (long long)p.H * D;
  const long long bbase = (long long)b * p.N * hstride + (long long)h * D;
  float qr[D], o[D];
#pragma unroll
  for (int c = 0; c < D; ++c) {
    qr[c] = q[row * D + c];
    o[c] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int i = 0; i < p.npat; ++i) {
    const PatternGeom& g = p.pat[i];
    const RowPos rp = row_pos(g, p.N, h, n);
    if (!rp.kept) continue;
    const long long kend = p.causal ? (long long)n : rp.end - 1;
    for (long long kp = rp.start + rp.off; kp <= kend; kp += g.r) {
      const float* kr = k + bbase + kp * hstride;
      float dot = 0.f;
#pragma unroll
      for (int c = 0; c < D; ++c) dot = fmaf(qr[c], kr[c], dot);
      const float s = dot * p.tau;
      if (s > m) {
        const float corr = expf(m - s);
        l *= corr;
#pragma unroll
        for (int c = 0; c < D; ++c) o[c] *= corr;
        m = s;
      }
      const float e = expf(s - m);
      l += e;
      const float* vr = v + bbase + kp * hstride;
#pragma unroll
      for (int c = 0; c < D; ++c) o[c] = fmaf(e, vr[c], o[c]);
    }
  }
  if (l > 0.f) {
    const float inv = 1.f / l;
#pragma unroll
    for (int c = 0; c < D; ++c) out[row * D + c] = o[c] * inv;
    if (lse) lse[((long long)b * p.H + h) * p.N + n] = m + logf(l);
  } else {
#pragma unroll
    for (int c = 0; c < D; ++c) out[row * D + c] = 0.f;
    if (lse) lse[((long long)b * p.H + h) * p.N + n] = -INFINITY;
  }
}

// dq for one query row: dq = tau * sum_c P_nc (dO_n . v_c - D_n) k_c over the
// multiset of keys every pattern keeping n gives it, P from the merged lse.
template <int D>
__global__ void __launch_bounds__(128) bwd_dq_f32_kernel(
    const __grid_constant__ RowParams p, const float* __restrict__ q,
    const float* __restrict__ k, const float* __restrict__ v, const float* __restrict__ out,
    const float* __restrict__ lse, const float* __restrict__ dout, float* __restrict__ dq) {
  const long long row = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long total = (long long)p.B * p.N * p.H;
  if (row >= total) return;
  const int h = (int)(row % p.H);
  const int n = (int)((row / p.H) % p.N);
  const int b = (int)(row / ((long long)p.H * p.N));
  const long long hstride = (long long)p.H * D;
  const long long bbase = (long long)b * p.N * hstride + (long long)h * D;
  const float L = lse[((long long)b * p.H + h) * p.N + n];
  float qr[D], dor[D], acc[D];
  float Dn = 0.f;
#pragma unroll
  for (int c = 0; c < D; ++c) {
    qr[c] = q[row * D + c];
    dor[c] = dout[row * D + c];
    Dn = fmaf(dor[c], out[row * D + c], Dn);
    acc[c] = 0.f;
  }
  if (L != -INFINITY) {
    for (int i = 0; i < p.npat; ++i) {
      const PatternGeom& g = p.pat[i];
      const RowPos rp = row_pos(g, p.N, h, n);
      if (!rp.kept) continue;
      const long long kend = p.causal ? (long long)n : rp.end - 1;
      for (long long kp = rp.start + rp.off; kp <= kend; kp += g.r) {
        const float* kr = k + bbase + kp * hstride;
        const float* vr = v + bbase + kp * hstride;
        float dot = 0.f, dp = 0.f;
#pragma unroll
        for (int c = 0; c < D; ++c) {
          dot = fmaf(qr[c], kr[c], dot);
          dp = fmaf(dor[c], vr[c], dp);
        }
        const float pr = expf(dot * p.tau - L);
        const float ds = pr * (dp - Dn) * p.tau;
#pragma unroll
        for (int c = 0; c < D; ++c) acc[c] = fmaf(ds, kr[c], acc[c]);
      }
    }
  }
#pragma unroll
  for (int c = 0; c < D; ++c) dq[row * D + c] = acc[c];
}

// dk, dv for one key row c: sums over every pattern that keeps c and every
// query n of c's segment in that pattern (n >= c when causal).
template <int D>
__global__ void __launch_bounds__(128) bwd_dkdv_f32_kernel(
    const __grid_constant__ RowParams p, const float* __restrict__ q,
    const float* __restrict__ k, const float* __restrict__ v, const float* __restrict__ out,
    const float* __restrict__ lse, const float* __restrict__ dout, float* __restrict__ dk,
    float* __restrict__ dv) {
  const long long row = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long total = (long long)p.B * p.N * p.H;
  if (row >= total) return;
  const int h = (int)(row % p.H);
  const int c0 = (int)((row / p.H) % p.N);
  const int b = (int)(row / ((long long)p.H * p.N));
  const long long hstride = (long long)p.H * D;
  const long long bbase = (long long)b * p.N * hstride + (long long)h * D;
  float kr[D], vr[D], ak[D], av[D];
#pragma unroll
  for (int c = 0; c < D; ++c) {
    kr[c] = k[row * D + c];
    vr[c] = v[row * D + c];
    ak[c] = 0.f;
    av[c] = 0.f;
  }
  for (int i = 0; i < p.npat; ++i) {
    const PatternGeom& g = p.pat[i];
    const RowPos rp = row_pos(g, p.N, h, c0);
    if (!rp.kept) continue;
    const long long first = p.causal ? (long long)c0 : rp.start + rp.off;
    for (long long n = first; n < rp.end; n += g.r) {
      const float* qn = q + bbase + n * hstride;
      const float* dn = dout + bbase + n * hstride;
      const float* on = out + bbase + n * hstride;
      const float L = lse[((long long)b * p.H + h) * p.N + n];
      float dot = 0.f, dp = 0.f, Dn = 0.f;
#pragma unroll
      for (int c = 0; c < D; ++c) {
        dot = fmaf(qn[c], kr[c], dot);
        dp = fmaf(dn[c], vr[c], dp);
        Dn = fmaf(dn[c], on[c], Dn);
      }
      const float pr = expf(dot * p.tau - L);
      const float ds = pr * (dp - Dn) * p.tau;
#pragma unroll
      for (int c = 0; c < D; ++c) {
        av[c] = fmaf(pr, dn[c], av[c]);
        ak[c] = fmaf(ds, qn[c], ak[c]);
      }
    }
  }
#pragma unroll
  for (int c = 0; c < D; ++c) {
    dk[row * D + c] = ak[c];
    dv[row * D + c] = av[c];
  }
}

}  // namespace dil
