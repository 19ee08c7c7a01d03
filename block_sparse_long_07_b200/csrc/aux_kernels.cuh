// aux_kernels.cuh -- the bandwidth- and integer-bound steps of the MoBA
// prefill forward: sequence plan, block mean-pool, gate (scores + top-k),
// query<->block bucketing (scan + scatter) and the online-softmax merge.
//
// Method: MoBA: Mixture of Block Attention for Long-Context LLMs.
//   pool   -- wispaper.ai blog, "The Change", affinity equation (mean-pooled
//             block key); sherconan.github.io step 2.
//   gate   -- same passages (s_i = <q, mean_pool(K[I_i])>), the routing rule
//             (top-k indicator) and the causality rule (no future block, own
//             block forced); sherconan.github.io steps 3-4.
//   bucket -- "arranges queries according to their selected KV blocks"
//             (wispaper.ai blog, "Efficiency and Implementation";
//             sherconan.github.io step 5, query-to-block assignment).
//   merge  -- "combines outputs with online softmax" (same passages).
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"
#include "layout.cuh"

namespace moba {

// ------------------------------------------------------------------- plan
// One CTA.  Validates cu_seqlens and writes block / query-tile numbering.
__global__ void plan_kernel(SeqLayout L, int B, Plan P, int NBmax, int NQTmax,
                            uint32_t* status) {
  __shared__ int32_t carry_b, carry_q, carry_p;
  __shared__ int bad;
  __shared__ int32_t sb[1024], sq[1024], sp[1024];
  const int tid = threadIdx.x, nt = blockDim.x;
  if (tid == 0) {
    status[1] = 0u;  // the largest |v| seen by vbound_kernel (see there)
    carry_b = 0;
    carry_q = 0;
    carry_p = 0;
    bad = 0;
    if (L.cu && (L.cu[0] != 0 || (int64_t)L.cu[L.nseq] != L.T)) bad = 1;
  }
  __syncthreads();
  for (int base = 0; base < L.nseq; base += nt) {
    int s = base + tid;
    int32_t nb = 0, nq = 0, np = 0;
    if (s < L.nseq) {
      int64_t len = seq_len(L, s);
      if (len < 0) {
        bad = 1;
        len = 0;
      }
      nb = (int32_t)((len + B - 1) / B);
      nq = (int32_t)((len + kTileM - 1) / kTileM);
      np = (int32_t)((len + 2 * kTileM - 1) / (2 * kTileM));
    }
    sb[tid] = nb;
    sq[tid] = nq;
    sp[tid] = np;
    __syncthreads();
    for (int off = 1; off < nt; off <<= 1) {  // inclusive Hillis-Steele scan
      int32_t vb = tid >= off ? sb[tid - off] : 0;
      int32_t vq = tid >= off ? sq[tid - off] : 0;
      int32_t vp = tid >= off ? sp[tid - off] : 0;
      __syncthreads();
      sb[tid] += vb;
      sq[tid] += vq;
      sp[tid] += vp;
      __syncthreads();
    }
    if (s < L.nseq) {
      P.blk_off[s] = carry_b + sb[tid] - nb;
      P.qt_off[s] = carry_q + sq[tid] - nq;
      P.pair_off[s] = carry_p + sp[tid] - np;
    }
    __syncthreads();
    if (tid == nt - 1) {
      carry_b += sb[tid];
      carry_q += sq[tid];
      carry_p += sp[tid];
    }
    __syncthreads();
  }
  if (tid == 0) {
    int nbt = carry_b, nqt = carry_q, npt = carry_p;
    if (nbt > NBmax || nqt > NQTmax) bad = 1;
    if (bad) {
      atomicOr(status, MOBA_DEV_BAD_SEQLENS);
      nbt = 0;
      nqt = 0;
      npt = 0;
    }
    P.blk_off[L.nseq] = nbt;
    P.qt_off[L.nseq] = nqt;
    P.pair_off[L.nseq] = npt;
    P.totals[0] = nbt;
    P.totals[1] = nqt;
    P.totals[2] = npt;
  }
  __syncthreads();
  if (bad) return;
  // per-block first token and length
  for (int s = 0; s < L.nseq; ++s) {
    int64_t st = seq_start(L, s), len = seq_len(L, s);
    int32_t b0 = P.blk_off[s], nb = P.blk_off[s + 1] - b0;
    for (int j = tid; j < nb; j += nt) {
      int64_t a = (int64_t)j * B;
      P.blk_tok[b0 + j] = (int32_t)(st + a);
      P.blk_len[b0 + j] = (int32_t)((len - a) < B ? (len - a) : B);
    }
  }
}

// ------------------------------------------------------------------- pool
// Kbar[g][J][:] = mean over the tokens of global block J of K[t][g][:].
// Grid (NBmax, Hkv), 256 threads; 16-byte loads, fixed summation order.
template <int D>
__global__ void __launch_bounds__(256) pool_kernel(const __nv_bfloat16* __restrict__ k, int Hkv,
                                                   Plan P, int NBmax, float* __restrict__ kbar,
                                                   int g0 = 0) {
  constexpr int CH = D / 8;          // 16-byte chunks per row
  constexpr int RPI = 256 / CH;      // rows per iteration
  __shared__ float red[RPI][D + 4];
  const int J = blockIdx.x, g = g0 + blockIdx.y;  // kv heads g0 .. g0 + gridDim.y - 1
  if (J >= P.totals[0]) return;
  const int64_t t0 = P.blk_tok[J];
  const int len = P.blk_len[J];
  const int c = threadIdx.x % CH, rs = threadIdx.x / CH;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  const uint4* base = reinterpret_cast<const uint4*>(k + ((size_t)t0 * Hkv + g) * D) + c;
  const size_t rstride = (size_t)Hkv * D / 8;  // in uint4
  int r = rs;
  for (; r + 3 * RPI < len; r += 4 * RPI) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = __ldg(base + (size_t)(r + u * RPI) * rstride);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v[u]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float2 f = __bfloat1622float2(h2[e]);
        acc[2 * e] += f.x;
        acc[2 * e + 1] += f.y;
      }
    }
  }
  for (; r < len; r += RPI) {
    uint4 v = __ldg(base + (size_t)r * rstride);
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float2 f = __bfloat1622float2(h2[e]);
      acc[2 * e] += f.x;
      acc[2 * e + 1] += f.y;
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[rs][c * 8 + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < D) {
    float s = 0.f;
#pragma unroll 4
    for (int q = 0; q < RPI; ++q) s += red[q][threadIdx.x];
    kbar[((size_t)g * NBmax + J) * D + threadIdx.x] = s / (float)len;
  }
}

// ------------------------------------------------------------------- |v| bound
// The routed partial outputs are stored in fp16 (see the attention
// epilogue).  A partial is a convex combination of its block's v rows, so
// its magnitude is below the largest |v|.  This kernel takes the largest
// |v| magnitude, as its bf16 bit pattern without the sign (integer order of
// those patterns is the order of the magnitudes; NaN sorts above inf), over
// every block of kv heads g0 .. g0 + gridDim.y - 1 into *vmag (atomic max;
// the plan kernel zeroes it).  From it the attention and the merge derive
// one power-of-two scale for the partials (partial_scale_log2), so that no
// valid bf16 input overflows fp16.  Grid (NBmax, heads), 256 threads,
// 16-byte loads.
template <int D>
__global__ void __launch_bounds__(256) vbound_kernel(const __nv_bfloat16* __restrict__ v,
                                                     int Hkv, Plan P, uint32_t* __restrict__ vmag,
                                                     int g0 = 0) {
  constexpr int CH = D / 8;
  constexpr int RPI = 256 / CH;
  const int J = blockIdx.x, g = g0 + blockIdx.y;
  if (J >= P.totals[0]) return;
  const int64_t t0 = P.blk_tok[J];
  const int len = P.blk_len[J];
  const int c = threadIdx.x % CH, rs = threadIdx.x / CH;
  const uint4* base = reinterpret_cast<const uint4*>(v + ((size_t)t0 * Hkv + g) * D) + c;
  const size_t rstride = (size_t)Hkv * D / 8;
  uint32_t mx = 0u;  // two 16-bit magnitudes, packed
  int r = rs;
  for (; r + 3 * RPI < len; r += 4 * RPI) {
    uint4 x[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) x[u] = __ldg(base + (size_t)(r + u * RPI) * rstride);
#pragma unroll
    for (int u = 0; u < 4; ++u)
      mx = __vmaxu2(__vmaxu2(mx, x[u].x & 0x7fff7fffu),
                    __vmaxu2(__vmaxu2(x[u].y & 0x7fff7fffu, x[u].z & 0x7fff7fffu),
                             x[u].w & 0x7fff7fffu));
  }
  for (; r < len; r += RPI) {
    const uint4 x = __ldg(base + (size_t)r * rstride);
    mx = __vmaxu2(__vmaxu2(mx, x.x & 0x7fff7fffu),
                  __vmaxu2(__vmaxu2(x.y & 0x7fff7fffu, x.z & 0x7fff7fffu), x.w & 0x7fff7fffu));
  }
  uint32_t m = max(mx & 0xffffu, mx >> 16);
  m = __reduce_max_sync(0xffffffffu, m);
  __shared__ uint32_t wm[8];
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t b = wm[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) b = max(b, wm[w]);
    if (b) atomicMax(vmag, b);
  }
}

// log2 of the factor the routed partials are multiplied by before their fp16
// store (and divided by again in the merge): 0 while every |v| < 2^15, else
// just enough that a partial, at most max|v| (1 + 2^-8) with the bf16
// rounding of the weights, stays below 2^15 * 1.004 < 65504.  The magnitude
// is a bf16 pattern: exponent field e means |v| < 2^(e - 126).  Inf or NaN
// inputs give 0 (their rows come out non-finite and the merge reports them).
__device__ __forceinline__ int partial_scale_log2(uint32_t vmag) {
  if (vmag >= 0x7f80u) return 0;
  const int e = (int)(vmag >> 7);
  return e > 141 ? e - 141 : 0;
}

// ------------------------------------------------------------------- gate
// One CTA per (query tile, query head), one thread per query row.
// Scores s_j = <q, Kbar_j> for the past blocks j < i (fp32), top-(k-1) by
// (score desc, index asc) kept in a register list of KM entries, the own
// block i added, the list written ascending and -1 padded.  With
// count_out != nullptr the CTA also adds, per past block, how many of its
// rows chose it (bucket sizes for the routed attention).
constexpr int kGateChunk = 32;          // Kbar rows staged in shared memory at once
constexpr int kMaxBlocksPerSeq = 8192;  // limit of the per-CTA block counters

template <int D, int KM>
__global__ void __launch_bounds__(128) gate_kernel(
    const __nv_bfloat16* __restrict__ q, int Hq, int G, int B, int topk, SeqLayout L, Plan P,
    int NBmax, const float* __restrict__ kbar, int32_t* __restrict__ sel, RowLayout R,
    uint32_t* __restrict__ count_out, uint32_t* __restrict__ status, int h0 = 0,
    int min_past = -1) {
  extern __shared__ __align__(16) unsigned char gate_smem[];
  float* kb = reinterpret_cast<float*>(gate_smem);                             // [chunk][D]
  uint32_t* cnt = reinterpret_cast<uint32_t*>(kb + kGateChunk * D);           // [blocks]
  const int qt = blockIdx.x, h = h0 + blockIdx.y;  // q heads h0 .. h0 + gridDim.y - 1
  if (qt >= P.totals[1]) return;
  const int s = upper_index(P.qt_off, L.nseq + 1, qt);
  const int64_t st = seq_start(L, s), len = seq_len(L, s);
  const int64_t p0 = (int64_t)(qt - P.qt_off[s]) * kTileM;
  const int i = (int)(p0 / B);  // own block of every row in the tile
  // as the tensor-core gate's companion (min_past >= 0): only tiles with
  // more than min_past past blocks are this kernel's (uniform over the CTA)
  if (i <= min_past) return;
  const int r = threadIdx.x;
  const int64_t pos = p0 + r;
  const bool valid = pos < len;
  const int64_t tok = st + pos;
  const int g = h / G;
  const int npast = topk - 1;

  int32_t chosen[KM];  // ascending block ids, -1 padded
  int nchosen = 0;
  const bool all_past = (i <= npast) || (npast == 0);
  if (all_past) {
    // no ranking needed: either every past block fits (i <= k-1) or none is
    // wanted (k = 1); rows take blocks 0 .. nchosen-1 and their own block
#pragma unroll
    for (int u = 0; u < KM; ++u) chosen[u] = -1;
    nchosen = min(i, npast);
  } else {
    float qv[D];
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
    // list sorted by (score desc, index asc); the first KM-npast entries are
    // +inf sentinels that never move, the last npast entries are the kept set
    float bs[KM];
    int32_t bj[KM];
#pragma unroll
    for (int u = 0; u < KM; ++u) {
      bs[u] = (u < KM - npast) ? __int_as_float(0x7f800000) : __int_as_float(0xff800000);
      bj[u] = -1;
    }
    const float* kb_g = kbar + ((size_t)g * NBmax + P.blk_off[s]) * D;
    for (int j0 = 0; j0 < i; j0 += kGateChunk) {
      const int nj = min(kGateChunk, i - j0);
      __syncthreads();
      for (int e = threadIdx.x; e < nj * D / 4; e += blockDim.x)
        reinterpret_cast<float4*>(kb)[e] =
            __ldg(reinterpret_cast<const float4*>(kb_g + (size_t)j0 * D) + e);
      __syncthreads();
      for (int jj = 0; jj < nj; ++jj) {
        const float4* kr = reinterpret_cast<const float4*>(kb + jj * D);
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
        for (int c = 0; c < D / 4; ++c) {
          float4 w = kr[c];
          a0 = fmaf(qv[4 * c + 0], w.x, a0);
          a1 = fmaf(qv[4 * c + 1], w.y, a1);
          a2 = fmaf(qv[4 * c + 2], w.z, a2);
          a3 = fmaf(qv[4 * c + 3], w.w, a3);
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
    // sort the kept ids ascending (odd-even transposition network)
#pragma unroll
    for (int u = 0; u < KM; ++u) chosen[u] = (u >= KM - npast) ? bj[u] : 0x7fffffff;
#pragma unroll
    for (int rd = 0; rd < KM; ++rd) {
#pragma unroll
      for (int u = (rd & 1); u + 1 < KM; u += 2) {
        const int32_t a = chosen[u], b = chosen[u + 1];
        chosen[u] = min(a, b);
        chosen[u + 1] = max(a, b);
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

// ------------------------------------------------------------------- scan
// One CTA.  For the units (kv heads) of one pass, flattened as f = u*NB + J:
// entry_off = exclusive scan of the bucket sizes, tile_off = exclusive scan
// of ceil(size/item_rows) (attention work items); both get a final total.  Also clears the scatter cursors.
__global__ void bucket_scan_kernel(const uint32_t* __restrict__ counts, int u0, int nu,
                                   int item_rows, const Plan P, int NBmax,
                                   int32_t* __restrict__ entry_off,
                                   int32_t* __restrict__ tile_off,
                                   uint32_t* __restrict__ cursor) {
  __shared__ int64_t se[1024], stl[1024];
  __shared__ int64_t carry_e, carry_t;
  const int tid = threadIdx.x, nt = blockDim.x;
  const int NB = P.totals[0];
  const int M = nu * NB;
  if (tid == 0) {
    carry_e = 0;
    carry_t = 0;
  }
  __syncthreads();
  for (int base = 0; base < M; base += nt) {
    const int f = base + tid;
    int64_t c = 0, tl = 0;
    if (f < M) {
      const int u = f / NB, J = f % NB;
      c = counts[(size_t)(u0 + u) * NBmax + J];
      tl = (c + item_rows - 1) / item_rows;
      cursor[f] = 0;
    }
    se[tid] = c;
    stl[tid] = tl;
    __syncthreads();
    for (int off = 1; off < nt; off <<= 1) {
      int64_t ve = tid >= off ? se[tid - off] : 0;
      int64_t vt = tid >= off ? stl[tid - off] : 0;
      __syncthreads();
      se[tid] += ve;
      stl[tid] += vt;
      __syncthreads();
    }
    if (f < M) {
      entry_off[f] = (int32_t)(carry_e + se[tid] - c);
      tile_off[f] = (int32_t)(carry_t + stl[tid] - tl);
    }
    __syncthreads();
    if (tid == nt - 1) {
      carry_e += se[tid];
      carry_t += stl[tid];
    }
    __syncthreads();
  }
  if (tid == 0) {
    entry_off[M] = (int32_t)carry_e;
    tile_off[M] = (int32_t)carry_t;
  }
}

// ---------------------------------------------------------------- scatter
// One CTA per (query tile, query head of the pass).  Every routed
// (row, head, slot) -- a past block in the row's selection -- is written to
// its bucket as {token, hh | slot << 16}.  Ranks inside the CTA come from
// shared-memory counters, one global atomic per (CTA, block) gives the base.
template <int KMAXS>
__global__ void __launch_bounds__(128) bucket_scatter_kernel(
    const int32_t* __restrict__ sel, RowLayout R, int topk, int B, int G, int u0, int nu,
    SeqLayout L, Plan P, const int32_t* __restrict__ entry_off, uint32_t* __restrict__ cursor,
    uint2* __restrict__ entries, uint32_t* __restrict__ status) {
  extern __shared__ uint32_t lcnt[];  // [blocks of the sequence]
  const int qt = blockIdx.x, hl = blockIdx.y;
  if (qt >= P.totals[1]) return;
  const int NB = P.totals[0];
  const int h = u0 * G + hl, u = hl / G, hh = hl % G;
  const int s = upper_index(P.qt_off, L.nseq + 1, qt);
  const int64_t st = seq_start(L, s), len = seq_len(L, s);
  const int64_t p0 = (int64_t)(qt - P.qt_off[s]) * kTileM;
  const int i = (int)(p0 / B);
  if (i == 0 || topk == 1) return;  // no past blocks in this tile
  if (i > kMaxBlocksPerSeq) {       // uniform over the CTA: counters would not fit
    if (threadIdx.x == 0) atomicOr(status, MOBA_DEV_CAPACITY);
    return;
  }
  const int r = threadIdx.x;
  const int64_t pos = p0 + r;
  const bool valid = pos < len;
  const int64_t tok = st + pos;
  const int npast = min(topk - 1, i);
  for (int j = r; j < i; j += blockDim.x) lcnt[j] = 0;
  __syncthreads();
  int32_t blk[KMAXS];
  uint32_t rank[KMAXS];
  const int32_t* row = sel + row_index(R, s, h, pos, tok) * topk;
#pragma unroll
  for (int w = 0; w < KMAXS; ++w) {
    blk[w] = -1;
    if (valid && w < npast) {
      int32_t j = row[w];
      if (j < 0 || j >= i) {
        atomicOr(status, MOBA_DEV_BAD_INDEX);
        j = -1;
      }
      blk[w] = j;
      if (j >= 0) rank[w] = atomicAdd(&lcnt[j], 1u);
    }
  }
  __syncthreads();
  const int J0 = P.blk_off[s];
  for (int j = r; j < i; j += blockDim.x) {
    const uint32_t c = lcnt[j];
    if (c) lcnt[j] = atomicAdd(&cursor[(size_t)u * NB + J0 + j], c);
  }
  __syncthreads();
#pragma unroll
  for (int w = 0; w < KMAXS; ++w) {
    if (blk[w] >= 0) {
      const int f = u * NB + J0 + blk[w];
      const int64_t e = (int64_t)entry_off[f] + lcnt[blk[w]] + rank[w];
      if (e < entry_off[f + 1])
        entries[e] = make_uint2((uint32_t)tok, (uint32_t)hh | ((uint32_t)w << 16));
      else
        atomicOr(status, MOBA_DEV_BAD_INDEX);  // bucket larger than the gate counted
    }
  }
}

// ------------------------------------------------------------------ merge
// The row's partials -- one per routed past block (fp16 O, log2-domain lse)
// and the own-block partial (fp32 O, log2 lse) -- are combined by the
// online-softmax rule
//   m = max lse_s, w_s = 2^(lse_s - m), O = sum w_s O_s / sum w_s,
//   lse = m + log2(sum w_s)   (output converted to natural log),
// with m the running maximum (sums rescaled when it grows).
// A group of D/8 lanes owns one (token, head) row; each lane owns 8 of its
// columns, so every partial row is read with one 16-byte load per lane and
// eight slots (O rows and lse) are loaded before any is used.  Rows whose
// selection is the own block alone were finished by the own-block kernel and
// are skipped.  The own-block partial is combined first, then the routed
// slots in ascending order.  The routed partials were stored multiplied by
// 2^-S (S from partial_scale_log2, 0 unless some |v| reaches 2^15); their
// weights carry the 2^S back.  A merged row that is not finite (non-finite
// inputs) is reported in the status word as MOBA_DEV_CAPACITY.
template <int D>
__global__ void __launch_bounds__(256) merge_kernel(
    const __half* __restrict__ part_O, const float* __restrict__ part_lse,
    const float* __restrict__ own_O, const float* __restrict__ own_lse, int topk, int B, int G,
    int Hq, int u0, int nu, SeqLayout L, __nv_bfloat16* __restrict__ o, float* __restrict__ lse,
    RowLayout R, uint32_t* __restrict__ status) {
  const float unscale = exp2f((float)partial_scale_log2(status[1]));
  constexpr int LPR = D / 8;       // lanes per row
  constexpr int RPW = 32 / LPR;    // rows per warp
  const int lane = threadIdx.x & 31;
  const int sub = lane % LPR;
  const int64_t row =
      ((int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5)) * RPW + lane / LPR;
  const int HP = nu * G;
  if (row >= L.T * HP) return;
  const int64_t t = row / HP;
  const int hl = (int)(row % HP);
  const int u = hl / G, hh = hl % G, h = u0 * G + hl;
  const int s = seq_of_token(L, t);
  const int64_t pos = t - seq_start(L, s);
  const int i = (int)(pos / B);
  const int cnt = min(topk, i + 1);
  if (cnt == 1) return;
  const int npast = cnt - 1;
  const int64_t prow = ((int64_t)u * L.T + t) * G + hh;  // partial row
  const int64_t pbase = prow * (topk - 1);
  const float* lrow = part_lse + pbase;
  // One pass with a running maximum: each batch's lse and O rows are loaded
  // together, 8 slots in flight, instead of every lse before any O row.
  float m = own_lse[prow];
  float den = 1.f;  // the own partial's weight, relative to m
  float acc[8];
  {
    const float4* src = reinterpret_cast<const float4*>(own_O + prow * D + sub * 8);
    const float4 a = src[0], b = src[1];
    acc[0] = a.x;
    acc[1] = a.y;
    acc[2] = a.z;
    acc[3] = a.w;
    acc[4] = b.x;
    acc[5] = b.y;
    acc[6] = b.z;
    acc[7] = b.w;
  }
  const uint4* orow = reinterpret_cast<const uint4*>(part_O + pbase * D) + sub;
  constexpr int kStride = D / 8;  // uint4 per partial row
  constexpr int kBatch = 8;
  for (int sl = 0; sl < npast; sl += kBatch) {
    uint4 v[kBatch];
    float l[kBatch];
#pragma unroll
    for (int q = 0; q < kBatch; ++q) {
      const bool in = sl + q < npast;
      v[q] = in ? orow[(sl + q) * kStride] : make_uint4(0u, 0u, 0u, 0u);
      l[q] = in ? lrow[sl + q] : -INFINITY;
    }
    float mb = l[0];
#pragma unroll
    for (int q = 1; q < kBatch; ++q) mb = fmaxf(mb, l[q]);
    if (mb > m) {  // rescale what is summed so far to the new maximum
      const float sc = ex2_approx(m - mb);
      den *= sc;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] *= sc;
      m = mb;
    }
#pragma unroll
    for (int q = 0; q < kBatch; ++q) {
      const float w = ex2_approx(l[q] - m);  // 0 past the row's slots
      den += w;
      const float wo = w * unscale;
      const __half2* h2 = reinterpret_cast<const __half2*>(&v[q]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(h2[e]);
        acc[2 * e] = fmaf(wo, f.x, acc[2 * e]);
        acc[2 * e + 1] = fmaf(wo, f.y, acc[2 * e + 1]);
      }
    }
  }
  bool finite = true;
#pragma unroll
  for (int e = 0; e < 8; ++e) finite = finite && fabsf(acc[e]) <= 3.4028234663852886e38f;
  if (!finite) atomicOr(status, MOBA_DEV_CAPACITY);
  const float inv = 1.f / den;
  uint4 out;
  out.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  out.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
  out.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
  out.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
  *(reinterpret_cast<uint4*>(o + ((size_t)t * Hq + h) * D) + sub) = out;
  if (sub == 0) lse[row_index(R, s, h, pos, t)] = (m + lg2_approx(den)) * 0.6931471805599453f;
}

}  // namespace moba
