// variants.cuh -- routing variants of the MoBA gate.
//
// The pages present MoBA's gate as a family: sliding-window attention is a
// gate that always picks the most recent blocks, sink attention one that
// always picks the initial and the most recent blocks (wispaper.ai blog,
// "Why the Change Is Plausible"), and Quest is MoBA with smaller blocks and
// min/max pooling (elamur summary card, "Key points").
//
//   minmax_pool_kernel  elementwise max and min of each block's keys, stored as
//                       bf16 (the extremes of bf16 values are bf16 values)
//   gate_minmax_kernel  per row: s_j = sum_c max(q_c max_jc, q_c min_jc) for
//                       every past block (Quest's bound on q . k over the
//                       block), top-(k-1) by (score desc, index asc), own
//                       block appended; per-block counts as the mean gate
//   static_select_kernel window / sink selections, no scores
// The selections they write have the mean gate's format, so the rest of the
// forward (bucketing, attention, merge) runs unchanged on them.
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"
#include "layout.cuh"

namespace moba {

enum RouteMode { kRouteWindow = 0, kRouteSink = 1 };

// mm[g][J][0][:] = max, mm[g][J][1][:] = min over the tokens of global block J.
// Grid (NBmax, Hkv), 256 threads; 16-byte loads.
template <int D>
__global__ void __launch_bounds__(256) minmax_pool_kernel(const __nv_bfloat16* __restrict__ k,
                                                          int Hkv, Plan P, int NBmax,
                                                          __nv_bfloat16* __restrict__ mm) {
  constexpr int CH = D / 8;      // 16-byte chunks per row
  constexpr int RPI = 256 / CH;  // rows per iteration
  __shared__ float rmax[RPI][D + 4], rmin[RPI][D + 4];
  const int J = blockIdx.x, g = blockIdx.y;
  if (J >= P.totals[0]) return;
  const int64_t t0 = P.blk_tok[J];
  const int len = P.blk_len[J];
  const int c = threadIdx.x % CH, rs = threadIdx.x / CH;
  float mx[8], mn[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    mx[e] = __int_as_float(0xff800000);
    mn[e] = __int_as_float(0x7f800000);
  }
  const uint4* base = reinterpret_cast<const uint4*>(k + ((size_t)t0 * Hkv + g) * D) + c;
  const size_t rstride = (size_t)Hkv * D / 8;
  for (int r = rs; r < len; r += RPI) {
    const uint4 v = __ldg(base + (size_t)r * rstride);
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h2[e]);
      mx[2 * e] = fmaxf(mx[2 * e], f.x);
      mx[2 * e + 1] = fmaxf(mx[2 * e + 1], f.y);
      mn[2 * e] = fminf(mn[2 * e], f.x);
      mn[2 * e + 1] = fminf(mn[2 * e + 1], f.y);
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    rmax[rs][c * 8 + e] = mx[e];
    rmin[rs][c * 8 + e] = mn[e];
  }
  __syncthreads();
  if (threadIdx.x < D) {
    float a = __int_as_float(0xff800000), b = __int_as_float(0x7f800000);
    for (int q = 0; q < RPI; ++q) {
      a = fmaxf(a, rmax[q][threadIdx.x]);
      b = fminf(b, rmin[q][threadIdx.x]);
    }
    __nv_bfloat16* out = mm + ((size_t)g * NBmax + J) * 2 * D;
    out[threadIdx.x] = __float2bfloat16_rn(a);  // exact: a is one of the bf16 keys
    out[D + threadIdx.x] = __float2bfloat16_rn(b);
  }
}

constexpr int kMinmaxChunk = 32;  // blocks staged in shared memory at once

// One CTA per (query tile, query head), one thread per row.  The score term
// max(q_c M_c, q_c m_c) equals q_c * (q_c >= 0 ? M_c : m_c) because M_c >= m_c,
// so each element costs one select and one fused multiply-add; the product of
// two bf16 values is exact in fp32.
template <int D, int KM>
__global__ void __launch_bounds__(128) gate_minmax_kernel(
    const __nv_bfloat16* __restrict__ q, int Hq, int G, int B, int topk, SeqLayout L, Plan P,
    int NBmax, const __nv_bfloat16* __restrict__ mm, int32_t* __restrict__ sel, RowLayout R,
    uint32_t* __restrict__ count_out, uint32_t* __restrict__ status) {
  extern __shared__ __align__(16) unsigned char gm_smem[];
  float* kb = reinterpret_cast<float*>(gm_smem);                               // [chunk][2][D]
  uint32_t* cnt = reinterpret_cast<uint32_t*>(kb + kMinmaxChunk * 2 * D);      // [blocks]
  const int qt = blockIdx.x, h = blockIdx.y;
  if (qt >= P.totals[1]) return;
  const int s = upper_index(P.qt_off, L.nseq + 1, qt);
  const int64_t st = seq_start(L, s), len = seq_len(L, s);
  const int64_t p0 = (int64_t)(qt - P.qt_off[s]) * kTileM;
  const int i = (int)(p0 / B);
  const int r = threadIdx.x;
  const int64_t pos = p0 + r;
  const bool valid = pos < len;
  const int64_t tok = st + pos;
  const int g = h / G;
  const int npast = topk - 1;

  int32_t chosen[KM];
  int nchosen = 0;
  const bool all_past = (i <= npast) || (npast == 0);
  if (all_past) {
#pragma unroll
    for (int u = 0; u < KM; ++u) chosen[u] = -1;
    nchosen = min(i, npast);
  } else {
    float qv[D];
    uint32_t neg[D / 32];  // bit c: q_c < 0 (take the block minimum)
#pragma unroll
    for (int w = 0; w < D / 32; ++w) neg[w] = 0u;
    if (valid) {
      const uint4* qr = reinterpret_cast<const uint4*>(q + ((size_t)tok * Hq + h) * D);
#pragma unroll
      for (int c = 0; c < D / 8; ++c) {
        uint4 v = __ldg(qr + c);
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float2 f = __bfloat1622float2(h2[e]);
          qv[8 * c + 2 * e] = f.x;
          qv[8 * c + 2 * e + 1] = f.y;
        }
      }
    } else {
#pragma unroll
      for (int c = 0; c < D; ++c) qv[c] = 0.f;
    }
#pragma unroll
    for (int c = 0; c < D; ++c)
      if (qv[c] < 0.f) neg[c / 32] |= 1u << (c % 32);
    float bs[KM];
    int32_t bj[KM];
#pragma unroll
    for (int u = 0; u < KM; ++u) {
      bs[u] = (u < KM - npast) ? __int_as_float(0x7f800000) : __int_as_float(0xff800000);
      bj[u] = -1;
    }
    const __nv_bfloat16* mm_g = mm + ((size_t)g * NBmax + P.blk_off[s]) * 2 * D;
    for (int j0 = 0; j0 < i; j0 += kMinmaxChunk) {
      const int nj = min(kMinmaxChunk, i - j0);
      __syncthreads();
      for (int e = threadIdx.x; e < nj * 2 * D / 8; e += blockDim.x) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(mm_g + (size_t)j0 * 2 * D) + e);
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const float2 f = __bfloat1622float2(h2[x]);
          kb[8 * e + 2 * x] = f.x;
          kb[8 * e + 2 * x + 1] = f.y;
        }
      }
      __syncthreads();
      for (int jj = 0; jj < nj; ++jj) {
        const float* kmax = kb + jj * 2 * D;
        const float* kmin = kmax + D;
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
        for (int c = 0; c < D; c += 4) {
          const uint32_t nb = neg[c / 32] >> (c % 32);
          a0 = fmaf(qv[c + 0], (nb & 1u) ? kmin[c + 0] : kmax[c + 0], a0);
          a1 = fmaf(qv[c + 1], (nb & 2u) ? kmin[c + 1] : kmax[c + 1], a1);
          a2 = fmaf(qv[c + 2], (nb & 4u) ? kmin[c + 2] : kmax[c + 2], a2);
          a3 = fmaf(qv[c + 3], (nb & 8u) ? kmin[c + 3] : kmax[c + 3], a3);
        }
        const float sc = (a0 + a1) + (a2 + a3);
        if (sc > bs[KM - 1]) {  // strict: an equal earlier block keeps its place
          bs[KM - 1] = sc;
          bj[KM - 1] = j0 + jj;
#pragma unroll
          for (int u = KM - 1; u > 0; --u) {
            const bool up = bs[u] > bs[u - 1];
            const float ts = up ? bs[u - 1] : bs[u];
            const int32_t tj = up ? bj[u - 1] : bj[u];
            bs[u - 1] = up ? bs[u] : bs[u - 1];
            bj[u - 1] = up ? bj[u] : bj[u - 1];
            bs[u] = ts;
            bj[u] = tj;
          }
        }
      }
    }
#pragma unroll
    for (int u = 0; u < KM; ++u) chosen[u] = (u >= KM - npast) ? bj[u] : 0x7fffffff;
#pragma unroll
    for (int rd = 0; rd < KM; ++rd) {
#pragma unroll
      for (int u = (rd & 1); u + 1 < KM; u += 2) {
        const int32_t x0 = chosen[u], x1 = chosen[u + 1];
        chosen[u] = min(x0, x1);
        chosen[u + 1] = max(x0, x1);
      }
    }
#pragma unroll
    for (int u = 0; u < KM; ++u) chosen[u] = (u < npast) ? chosen[u] : -1;
    nchosen = npast;
  }

  if (valid) {
    int32_t* out = sel + row_index(R, s, h, pos, tok) * topk;
    for (int u = 0; u < topk; ++u) {
      int32_t v;
      if (u == nchosen) {
        v = i;
      } else if (u > nchosen) {
        v = -1;
      } else if (all_past) {
        v = u;
      } else {
        v = -1;
#pragma unroll
        for (int w = 0; w < KM; ++w)
          if (w == u) v = chosen[w];
      }
      out[u] = v;
    }
  }
  if (count_out) {
    if (i > kMaxBlocksPerSeq) {  // uniform over the CTA
      if (threadIdx.x == 0) atomicOr(status, MOBA_DEV_CAPACITY);
      return;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < i; j += blockDim.x) cnt[j] = 0;
    __syncthreads();
    if (valid) {
      if (all_past) {
        for (int j = 0; j < nchosen; ++j) atomicAdd(&cnt[j], 1u);
      } else {
#pragma unroll
        for (int w = 0; w < KM; ++w)
          if (w < nchosen) atomicAdd(&cnt[chosen[w]], 1u);
      }
    }
    __syncthreads();
    uint32_t* dst = count_out + (size_t)g * NBmax + P.blk_off[s];
    for (int j = threadIdx.x; j < i; j += blockDim.x)
      if (cnt[j]) atomicAdd(&dst[j], cnt[j]);
  }
}

// Window / sink selections: the own block i and min(k-1, i) past blocks,
// the most recent ones (window) or block 0 plus the most recent ones (sink).
// Batch layout sel [b][Hq][N][k] (row x = (b, h, pos)); packed sequences
// (L.cu set) sel [Hq][T][k] (row x = (h, token)), positions counted from
// each sequence's start.
__global__ void static_select_kernel(int32_t* __restrict__ sel, int64_t rows, SeqLayout L,
                                     int Hq, int B, int topk, int mode) {
  const int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (x >= rows) return;
  int64_t pos;
  if (L.cu) {
    const int64_t t = x % L.T;
    pos = t - seq_start(L, seq_of_token(L, t));
  } else {
    pos = x % L.N;
  }
  const int i = (int)(pos / B);
  const int npast = min(topk - 1, i);
  int32_t* out = sel + x * topk;
  int u = 0;
  if (mode == kRouteSink && npast > 0 && npast < i) {
    out[u++] = 0;
    for (int j = i - npast + 1; j < i; ++j) out[u++] = j;
  } else {
    for (int j = i - npast; j < i; ++j) out[u++] = j;
  }
  out[u++] = i;
  for (; u < topk; ++u) out[u] = -1;
}

}  // namespace moba
