// decode.cuh -- one MoBA decode step: a single new query per sequence
// against that sequence's KV cache and its cache of block means.
//
// The new token of sequence b sits at position t = len_b - 1 of the cache,
// in block i = t / B.  Its selection follows the same routing and causality
// rules as the prefill (MoBA: Mixture of Block Attention, wispaper.ai blog,
// "The Change": affinity with the block mean, top-k over past blocks, own
// block always kept, ties to the lower block; sherconan.github.io steps 2-4),
// and its output is exact softmax attention over the chosen blocks, causal
// in the own block (which ends at t), combined by online softmax
// ("Efficiency and Implementation").
//
// Kernels:
//   kbar_cache_kernel   block means of complete cache blocks (all of them, or
//                       the one the newest token completed)
//   decode_gate_kernel  per (sequence, q head): scores against every past
//                       block mean, top-(k-1) by repeated block-wide argmax
//                       (ties to the lower index), own block appended
//   decode_attn_kernel  per (sequence, q head, chosen block, chunk of keys):
//                       partial max / sum / output over the chunk (split-KV)
//   decode_merge_kernel per (sequence, q head): combines the partials in a
//                       fixed order into O (bf16) and lse (natural log)
// Everything here is bandwidth-bound: the chosen blocks' K and V are read
// once per q head (the heads of a kv group that choose the same block share
// it through L2).
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"

namespace moba {

constexpr int kDecodeChunk = 512;         // keys per split-KV work item
constexpr int kDecodeMaxBlocks = 8192;    // blocks per sequence the gate handles

struct DecodeArgs {
  const __nv_bfloat16* q;       // [b][Hq][D]
  const __nv_bfloat16* kc;      // [b][cap][Hkv][D]
  const __nv_bfloat16* vc;      // [b][cap][Hkv][D]
  const int32_t* lens;          // [b] tokens in the cache, the new one included
  float* kbar;                  // [b][Hkv][nbcap][D] (written only by kbar_cache_kernel)
  int32_t* sel;                 // [b][Hq][k]
  float* part;                  // [b][Hq][k][nchunk][D + 2]: O (unnormalised), m, l (log2)
  __nv_bfloat16* o;             // [b][Hq][D]
  float* lse;                   // [b][Hq]
  int batch, cap, Hq, Hkv, G, B, topk, nbcap, nchunk;
  float scale_log2;
  uint32_t* status;
};

// Mean of cache block j of (sequence b, kv head g) over its B tokens, in a
// fixed order (rows split over 4 row groups, then added in group order).
// Grid (blocks, Hkv, batch) for a full rebuild, or (1, Hkv, batch) for the
// block completed by the newest token (nothing when len % B != 0).
template <int D>
__global__ void __launch_bounds__(128) kbar_cache_kernel(const DecodeArgs a, int only_last) {
  constexpr int C4 = D / 4;           // float4 columns per row
  constexpr int RG = 128 / C4;        // row groups
  __shared__ float red[RG][D];
  const int g = blockIdx.y, b = blockIdx.z;
  const int len = a.lens[b];
  if (len < 1 || len > a.cap) {
    if (threadIdx.x == 0) atomicOr(a.status, MOBA_DEV_BAD_SEQLENS);
    return;
  }
  int j;
  if (only_last) {
    if (len % a.B != 0) return;
    j = len / a.B - 1;
  } else {
    j = blockIdx.x;
    if (j >= len / a.B) return;  // only complete blocks
  }
  if (j >= a.nbcap) return;
  const int c4 = threadIdx.x % C4, rg = threadIdx.x / C4;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  const size_t rstride = (size_t)a.Hkv * D;
  const __nv_bfloat16* base = a.kc + (((size_t)b * a.cap + (size_t)j * a.B) * a.Hkv + g) * D + 4 * c4;
  for (int r = rg; r < a.B; r += RG) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(base + (size_t)r * rstride));
    const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.x));
    const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.y));
    acc[0] += f0.x;
    acc[1] += f0.y;
    acc[2] += f1.x;
    acc[3] += f1.y;
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) red[rg][4 * c4 + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < D) {
    float s = 0.f;
#pragma unroll
    for (int q = 0; q < RG; ++q) s += red[q][threadIdx.x];
    a.kbar[(((size_t)b * a.Hkv + g) * a.nbcap + j) * D + threadIdx.x] = s / (float)a.B;
  }
}

// Gate for the new token of (sequence b, q head h).  256 threads: scores of
// the past blocks into shared memory, then k-1 rounds of block-wide argmax
// by (score desc, index asc).
template <int D>
__global__ void __launch_bounds__(256) decode_gate_kernel(const DecodeArgs a) {
  extern __shared__ float dg_smem[];  // scores [nbcap]
  __shared__ float qs[D];
  __shared__ float red_v[8];
  __shared__ int red_j[8];
  __shared__ int chosen[64];
  const int h = blockIdx.x, b = blockIdx.y;
  const int g = h / a.G;
  const int len = a.lens[b];
  int32_t* out = a.sel + ((size_t)b * a.Hq + h) * a.topk;
  if (len < 1 || len > a.cap) {
    if (threadIdx.x == 0) atomicOr(a.status, MOBA_DEV_BAD_SEQLENS);
    for (int u = threadIdx.x; u < a.topk; u += blockDim.x) out[u] = -1;
    return;
  }
  const int i = (len - 1) / a.B;
  const int npast = a.topk - 1;
  if (i <= npast) {  // every past block is kept (or k = 1 keeps none)
    const int nch = min(i, npast);
    for (int u = threadIdx.x; u < a.topk; u += blockDim.x)
      out[u] = u < nch ? u : (u == nch ? i : -1);
    return;
  }
  if (i > kDecodeMaxBlocks || i > a.nbcap) {
    if (threadIdx.x == 0) atomicOr(a.status, MOBA_DEV_CAPACITY);
    for (int u = threadIdx.x; u < a.topk; u += blockDim.x) out[u] = -1;
    return;
  }
  if (threadIdx.x < D)
    qs[threadIdx.x] = __bfloat162float(a.q[((size_t)b * a.Hq + h) * D + threadIdx.x]);
  __syncthreads();
  const float* kb = a.kbar + ((size_t)b * a.Hkv + g) * a.nbcap * D;
  for (int j = threadIdx.x; j < i; j += blockDim.x) {
    const float4* kr = reinterpret_cast<const float4*>(kb + (size_t)j * D);
    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll 8
    for (int c = 0; c < D / 4; ++c) {
      const float4 w = __ldg(kr + c);
      s0 = fmaf(qs[4 * c + 0], w.x, s0);
      s1 = fmaf(qs[4 * c + 1], w.y, s1);
      s2 = fmaf(qs[4 * c + 2], w.z, s2);
      s3 = fmaf(qs[4 * c + 3], w.w, s3);
    }
    dg_smem[j] = (s0 + s1) + (s2 + s3);
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int round = 0; round < npast; ++round) {
    float bv = __int_as_float(0xff800000);
    int bj = 0x7fffffff;
    for (int j = threadIdx.x; j < i; j += blockDim.x) {
      const float v = dg_smem[j];
      if (v > bv || (v == bv && j < bj)) {  // removed entries hold NaN: never taken
        bv = v;
        bj = j;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
      if (ov > bv || (ov == bv && oj < bj)) {
        bv = ov;
        bj = oj;
      }
    }
    if (lane == 0) {
      red_v[warp] = bv;
      red_j[warp] = bj;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      float v = red_v[0];
      int jj = red_j[0];
      for (int w = 1; w < 8; ++w)
        if (red_v[w] > v || (red_v[w] == v && red_j[w] < jj)) {
          v = red_v[w];
          jj = red_j[w];
        }
      // a row of non-finite scores can leave nothing selectable
      chosen[round] = (jj >= 0 && jj < i) ? jj : -1;
      if (jj >= 0 && jj < i) dg_smem[jj] = __int_as_float(0x7fc00000);
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    // ascending block order; an unfilled round (-1) sorts last
    for (int u = 1; u < npast; ++u) {
      const unsigned x = (unsigned)chosen[u];
      int p = u - 1;
      while (p >= 0 && (unsigned)chosen[p] > x) {
        chosen[p + 1] = chosen[p];
        --p;
      }
      chosen[p + 1] = (int)x;
    }
    for (int u = 0; u < npast; ++u) out[u] = chosen[u];
    out[npast] = i;
  }
}

// Split-KV partial over keys [kb0, kb1) of one chosen block: 4 warps, each a
// contiguous quarter of the chunk; lane l holds D/32 query and output
// elements.  Writes O (unnormalised, fp32), m (log2 domain) and l.
template <int D>
__global__ void __launch_bounds__(128) decode_attn_kernel(const DecodeArgs a) {
  constexpr int EPL = D / 32;  // elements per lane
  __shared__ float wm[4], wl[4];
  __shared__ float wo[4][D];
  const int bh = blockIdx.x, u = blockIdx.y, c = blockIdx.z;
  const int b = bh / a.Hq, h = bh % a.Hq, g = h / a.G;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float* dst = a.part + (((size_t)bh * a.topk + u) * a.nchunk + c) * (D + 2);
  const int len = a.lens[b];
  const int32_t blk = a.sel[(size_t)bh * a.topk + u];
  int kb0 = 0, kb1 = 0;
  if (len >= 1 && len <= a.cap && blk >= 0) {
    const int i = (len - 1) / a.B;
    if (blk <= i) {
      const int bend = (blk == i) ? len : (blk + 1) * a.B;  // own block ends at the new token
      kb0 = blk * a.B + c * kDecodeChunk;
      kb1 = min(bend, kb0 + kDecodeChunk);
    } else if (threadIdx.x == 0) {
      atomicOr(a.status, MOBA_DEV_BAD_INDEX);
    }
  }
  if (kb0 >= kb1) {  // empty: a neutral partial
    if (threadIdx.x < D) dst[threadIdx.x] = 0.f;
    if (threadIdx.x == 0) {
      dst[D] = __int_as_float(0xff800000);
      dst[D + 1] = 0.f;
    }
    return;
  }
  float qv[EPL];
  {
    const __nv_bfloat16* qp = a.q + (size_t)bh * D + lane * EPL;
#pragma unroll
    for (int e = 0; e < EPL; ++e) qv[e] = __bfloat162float(qp[e]) * a.scale_log2;
  }
  const int per = (kb1 - kb0 + 3) / 4;
  const int w0 = kb0 + warp * per, w1 = min(kb1, w0 + per);
  float m = __int_as_float(0xff800000), l = 0.f;
  float ov[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) ov[e] = 0.f;
  const size_t rstride = (size_t)a.Hkv * D;
  const __nv_bfloat16* kbase = a.kc + ((size_t)b * a.cap * a.Hkv + g) * D + lane * EPL;
  const __nv_bfloat16* vbase = a.vc + ((size_t)b * a.cap * a.Hkv + g) * D + lane * EPL;
  constexpr int U = 4;  // keys in flight per warp step
  for (int t0 = w0; t0 < w1; t0 += U) {
    float kf[U][EPL], vf[U][EPL];
#pragma unroll
    for (int x = 0; x < U; ++x) {
      const int t = min(t0 + x, w1 - 1);
      const __nv_bfloat16* kp = kbase + (size_t)t * rstride;
      const __nv_bfloat16* vp = vbase + (size_t)t * rstride;
      if constexpr (EPL == 4) {
        const uint2 kk = __ldg(reinterpret_cast<const uint2*>(kp));
        const uint2 vv = __ldg(reinterpret_cast<const uint2*>(vp));
        const float2 k0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kk.x));
        const float2 k1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kk.y));
        const float2 v0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vv.x));
        const float2 v1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vv.y));
        kf[x][0] = k0.x;
        kf[x][1] = k0.y;
        kf[x][2] = k1.x;
        kf[x][3] = k1.y;
        vf[x][0] = v0.x;
        vf[x][1] = v0.y;
        vf[x][2] = v1.x;
        vf[x][3] = v1.y;
      } else {
        const uint32_t kk = __ldg(reinterpret_cast<const uint32_t*>(kp));
        const uint32_t vv = __ldg(reinterpret_cast<const uint32_t*>(vp));
        const float2 k0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kk));
        const float2 v0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vv));
        kf[x][0] = k0.x;
        kf[x][1] = k0.y;
        vf[x][0] = v0.x;
        vf[x][1] = v0.y;
      }
    }
    float s[U];
#pragma unroll
    for (int x = 0; x < U; ++x) {
      float d = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) d = fmaf(qv[e], kf[x][e], d);
      s[x] = d;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int x = 0; x < U; ++x) s[x] += __shfl_xor_sync(0xffffffffu, s[x], o);
    float mx = m;
#pragma unroll
    for (int x = 0; x < U; ++x)
      if (t0 + x < w1) mx = fmaxf(mx, s[x]);
    const float alpha = ex2_approx(m - mx);  // m = -inf on the first step: 0
    l *= alpha;
#pragma unroll
    for (int e = 0; e < EPL; ++e) ov[e] *= alpha;
#pragma unroll
    for (int x = 0; x < U; ++x) {
      const float p = (t0 + x < w1) ? ex2_approx(s[x] - mx) : 0.f;
      l += p;
#pragma unroll
      for (int e = 0; e < EPL; ++e) ov[e] = fmaf(p, vf[x][e], ov[e]);
    }
    m = mx;
  }
  // combine the 4 warps (fixed order)
  if (lane == 0) {
    wm[warp] = m;
    wl[warp] = l;
  }
#pragma unroll
  for (int e = 0; e < EPL; ++e) wo[warp][lane * EPL + e] = ov[e];
  __syncthreads();
  if (threadIdx.x < D) {
    float M = wm[0];
#pragma unroll
    for (int w = 1; w < 4; ++w) M = fmaxf(M, wm[w]);
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float f = (wm[w] == __int_as_float(0xff800000)) ? 0.f : ex2_approx(wm[w] - M);
      L += f * wl[w];
      O += f * wo[w][threadIdx.x];
    }
    dst[threadIdx.x] = O;
    if (threadIdx.x == 0) {
      dst[D] = M;
      dst[D + 1] = L;
    }
  }
}

// O = sum_p 2^(m_p - M) O_p / sum_p 2^(m_p - M) l_p over the (slot, chunk)
// partials in ascending order; lse = (M + log2 L) ln 2.
template <int D>
__global__ void __launch_bounds__(D) decode_merge_kernel(const DecodeArgs a) {
  const int bh = blockIdx.x;
  const float* src = a.part + (size_t)bh * a.topk * a.nchunk * (D + 2);
  const int np = a.topk * a.nchunk;
  float M = __int_as_float(0xff800000);
  for (int p = 0; p < np; ++p) M = fmaxf(M, src[(size_t)p * (D + 2) + D]);
  float L = 0.f, O = 0.f;
  if (M != __int_as_float(0xff800000)) {
    for (int p = 0; p < np; ++p) {
      const float* pp = src + (size_t)p * (D + 2);
      const float mp = pp[D];
      if (mp == __int_as_float(0xff800000)) continue;
      const float f = ex2_approx(mp - M);
      L += f * pp[D + 1];
      O += f * pp[threadIdx.x];
    }
  }
  const bool ok = L > 0.f;
  a.o[(size_t)bh * D + threadIdx.x] = __float2bfloat16_rn(ok ? O / L : 0.f);
  if (threadIdx.x == 0)
    a.lse[bh] = ok ? (M + lg2_approx(L)) * 0.6931471805599453f : __int_as_float(0xff800000);
}

}  // namespace moba
