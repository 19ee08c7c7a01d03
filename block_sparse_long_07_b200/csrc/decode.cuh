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
//   kbar_part_kernel,   block means of complete cache blocks (all of them, or
//   kbar_reduce_kernel  the one the newest token completed), split over CTAs
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
  float* kbar;                  // [b][Hkv][nbcap][D] (written only by kbar_reduce_kernel)
  int32_t* sel;                 // [b][Hq][k]
  float* part;                  // [b][Hq][k][nchunk][D + 2]: O (unnormalised), m, l (log2)
  __nv_bfloat16* o;             // [b][Hq][D]
  float* lse;                   // [b][Hq]
  int batch, cap, Hq, Hkv, G, B, topk, nbcap, nchunk;
  float scale_log2;
  uint32_t* status;
};

// Block means of the cache, in two deterministic steps.  kbar_part_kernel:
// CTA (x = j_local * S + split, kv head, sequence) sums rows
// [split * kKbarRows, (split + 1) * kKbarRows) of block j (4 row groups, 8
// loads in flight per thread, groups added in order) into part[...][split].
// kbar_reduce_kernel adds the S partials in split order and divides by B.
// only_last = 0: every complete block (j < len / B); otherwise only the block
// the newest token completed (j = len / B - 1 when len % B == 0).
constexpr int kKbarRows = 128;  // rows per partial (block sizes are multiples of 128)

__device__ __forceinline__ int kbar_block(const DecodeArgs& a, int b, int jl, int only_last,
                                          bool report) {
  const int len = a.lens[b];
  if (len < 1 || len > a.cap) {
    if (report) atomicOr(a.status, MOBA_DEV_BAD_SEQLENS);
    return -1;
  }
  int j;
  if (only_last) {
    if (len % a.B != 0) return -1;
    j = len / a.B - 1;
  } else {
    j = jl;
    if (j >= len / a.B) return -1;  // only complete blocks
  }
  return j < a.nbcap ? j : -1;
}

template <int D>
__global__ void __launch_bounds__(128) kbar_part_kernel(const DecodeArgs a, int only_last,
                                                        float* __restrict__ part) {
  constexpr int C4 = D / 4;     // 8-byte (4 x bf16) columns per row
  constexpr int RG = 128 / C4;  // row groups
  constexpr int U = 8;          // loads in flight
  __shared__ float red[RG][D];
  const int S = a.B / kKbarRows;
  const int jl = blockIdx.x / S, sp = blockIdx.x % S;
  const int g = blockIdx.y, b = blockIdx.z;
  const int j = kbar_block(a, b, jl, only_last, blockIdx.x == 0 && g == 0 && threadIdx.x == 0);
  if (j < 0) return;
  const int c4 = threadIdx.x % C4, rg = threadIdx.x / C4;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  const size_t rstride = (size_t)a.Hkv * D;
  const __nv_bfloat16* base =
      a.kc + (((size_t)b * a.cap + (size_t)j * a.B + (size_t)sp * kKbarRows) * a.Hkv + g) * D +
      4 * c4;
  for (int r0 = rg; r0 < kKbarRows; r0 += RG * U) {
    uint2 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int r = r0 + u * RG;
      v[u] = r < kKbarRows ? __ldg(reinterpret_cast<const uint2*>(base + (size_t)r * rstride))
                           : make_uint2(0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v[u].x));
      const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v[u].y));
      acc[0] += f0.x;
      acc[1] += f0.y;
      acc[2] += f1.x;
      acc[3] += f1.y;
    }
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) red[rg][4 * c4 + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < D) {
    float s = 0.f;
#pragma unroll
    for (int q = 0; q < RG; ++q) s += red[q][threadIdx.x];
    const int nsel = only_last ? 1 : a.nbcap;
    part[((((size_t)b * a.Hkv + g) * nsel + (only_last ? 0 : j)) * S + sp) * D + threadIdx.x] = s;
  }
}

template <int D>
__global__ void __launch_bounds__(D) kbar_reduce_kernel(const DecodeArgs a, int only_last,
                                                        const float* __restrict__ part) {
  const int jl = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int j = kbar_block(a, b, jl, only_last, false);
  if (j < 0) return;
  const int S = a.B / kKbarRows;
  const int nsel = only_last ? 1 : a.nbcap;
  const float* src = part + (((size_t)b * a.Hkv + g) * nsel + (only_last ? 0 : j)) * S * D;
  float s = 0.f;
  for (int sp = 0; sp < S; ++sp) s += src[(size_t)sp * D + threadIdx.x];
  a.kbar[(((size_t)b * a.Hkv + g) * a.nbcap + j) * D + threadIdx.x] = s / (float)a.B;
}

// Gate for the new token of (sequence b, q head h).  256 threads score the
// past blocks into shared memory; warp 0 then takes k-1 rounds of argmax by
// (score desc, index asc).
template <int D>
__global__ void __launch_bounds__(256) decode_gate_kernel(const DecodeArgs a) {
  extern __shared__ float dg_smem[];  // scores [nbcap]
  __shared__ float qs[D];
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
  if (threadIdx.x >= 32) return;
  // warp 0: k-1 rounds of argmax by (score desc, index asc); a taken score
  // becomes NaN, which no comparison selects again
  const int lane = threadIdx.x;
  for (int round = 0; round < npast; ++round) {
    float bv = __int_as_float(0xff800000);
    int bj = 0x7fffffff;
    for (int j = lane; j < i; j += 32) {
      const float v = dg_smem[j];
      if (v > bv || (v == bv && j < bj)) {
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
    // a row of non-finite scores can leave nothing selectable
    const bool hit = bj >= 0 && bj < i;
    if (lane == 0) chosen[round] = hit ? bj : -1;
    if (hit && lane == (bj & 31)) dg_smem[bj] = __int_as_float(0x7fc00000);
    __syncwarp();
  }
  if (lane == 0) {
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
// partials in ascending order; lse = (M + log2 L) ln 2.  The partials' m and
// l are staged in shared memory; each thread then walks its output column
// with 8 independent loads in flight.
constexpr int kDecodeMaxParts = 65 * 64;  // top_k <= 65, chunks per block <= 64 staged

template <int D>
__global__ void __launch_bounds__(D) decode_merge_kernel(const DecodeArgs a) {
  __shared__ float sw[kDecodeMaxParts];  // weight 2^(m_p - M), 0 for empty partials
  __shared__ float red[D / 32];
  __shared__ float sM;
  const int bh = blockIdx.x;
  const float* src = a.part + (size_t)bh * a.topk * a.nchunk * (D + 2);
  const int np = a.topk * a.nchunk;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float M = __int_as_float(0xff800000);
  for (int p = threadIdx.x; p < np; p += D) {
    const float mp = src[(size_t)p * (D + 2) + D];
    sw[p] = mp;
    M = fmaxf(M, mp);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if (lane == 0) red[warp] = M;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = red[0];
    for (int w = 1; w < D / 32; ++w) m = fmaxf(m, red[w]);
    sM = m;
  }
  __syncthreads();
  M = sM;
  const bool any = M != __int_as_float(0xff800000);
  for (int p = threadIdx.x; p < np; p += D) {
    const float mp = sw[p];
    sw[p] = (any && mp != __int_as_float(0xff800000)) ? ex2_approx(mp - M) : 0.f;
  }
  __syncthreads();
  float L = 0.f, O = 0.f;
  for (int p0 = 0; p0 < np; p0 += 8) {
    float ov[8], lv[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int p = min(p0 + u, np - 1);
      ov[u] = src[(size_t)p * (D + 2) + threadIdx.x];
      lv[u] = src[(size_t)p * (D + 2) + D + 1];
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float wgt = (p0 + u < np) ? sw[p0 + u] : 0.f;
      L = fmaf(wgt, lv[u], L);
      O = fmaf(wgt, ov[u], O);
    }
  }
  const bool ok = L > 0.f;
  a.o[(size_t)bh * D + threadIdx.x] = __float2bfloat16_rn(ok ? O / L : 0.f);
  if (threadIdx.x == 0)
    a.lse[bh] = ok ? (M + lg2_approx(L)) * 0.6931471805599453f : __int_as_float(0xff800000);
}

}  // namespace moba
