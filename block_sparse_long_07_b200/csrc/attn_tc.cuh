// attn_tc.cuh -- exact softmax attention on the sm_100a tensor cores
// (tcgen05.mma with TMEM accumulators, TMA-fed K/V ring), in three modes:
//
//   kRouted : a tile of up to 128 gathered (token, q-head) rows that all
//             chose the same past block J, against the B keys of J, no mask.
//             Writes one normalised partial O (bf16) and its log2-domain lse
//             per row into the row's slot.  This is the "MoBA attention"
//             over historical blocks (MoBA: Mixture of Block Attention,
//             wispaper.ai blog, "Efficiency and Implementation").
//   kOwn    : 128 consecutive query rows of one head against the keys of
//             their own block up to the diagonal, causal mask on the
//             diagonal tile ("current-block attention" with the causal mask
//             inside the block; wispaper.ai blog, "The Change", causality
//             rule).  Rows whose selection is the own block alone write the
//             final O / lse; the others write an fp32 partial for the merge.
//   kDense  : 128 query rows against every earlier key of their sequence:
//             full causal attention, the k = n limit (wispaper.ai blog,
//             "The Change": k = n recovers full attention).
//
// CTA = 7 warps, one CTA per SM, persistent over work tiles:
//   warps 0-3  softmax + epilogue; thread r owns query row r = TMEM lane r
//   warp  4    TMA producer: Q tiles (own/dense) and the K/V ring
//   warp  5    Q gather for routed tiles (cp.async rows into swizzled smem)
//   warp  6    TMEM allocation and the single-thread MMA issuer
// Per KV tile j: S_j = Q K_j^T  (M=128, N=128, K=d) into one of two TMEM S
// buffers; the softmax warps turn S_j into P_j (bf16, shared memory) with an
// online max / sum; O += P_j V_j (M=128, N=d, K=128) accumulates in TMEM.
// S_{j+1} is issued before PV_j so the tensor core works while the softmax
// runs.  The running max is rescaled lazily: O is only rescaled when the max
// grows by more than 2^8.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"
#include "layout.cuh"

namespace moba {

enum AttnMode : int { kRouted = 0, kOwn = 1, kDense = 2 };

struct AttnArgs {
  const __nv_bfloat16* q;  // [T][Hq][D] (routed gather)
  int Hq, Hkv, G, B, topk;
  float scale_log2;        // softmax scale * log2(e)
  SeqLayout L;
  Plan P;
  RowLayout R;             // lse row layout of the final outputs
  // pass: kv heads u0 .. u0+nu-1
  int u0, nu;
  // routed work list
  const int32_t* tile_off;   // [nu*NB + 1]
  const int32_t* entry_off;  // [nu*NB + 1]
  const uint2* entries;
  __nv_bfloat16* part_O;     // [nu][T][G][topk-1][D]
  float* part_lse;           // [nu][T][G][topk-1]
  // own-block partials
  float* own_O;              // [nu][T][G][D]
  float* own_lse;            // [nu][T][G]
  // final outputs
  __nv_bfloat16* o;          // [T][Hq][D]
  float* lse;
  uint32_t* status;
};

template <int D>
struct AttnCfg {
  static constexpr int kStages = (D == 128) ? 3 : 4;        // K/V ring slots
  static constexpr int kHalfBytes = kTileM * 128;            // one 64-column half tile
  static constexpr int kQBytes = kTileM * D * 2;
  static constexpr int kKVBytes = kTileN * D * 2;
  static constexpr int kPBytes = kTileM * kTileN * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = kOffQ + 2 * kQBytes;
  static constexpr int kOffP = kOffKV + kStages * kKVBytes;
  static constexpr int kOffBar = kOffP + kPBytes;
  static constexpr int kNumBars = 2 + 2 + 2 * kStages + 2 + 2 + 1 + 1 + 1;
  static constexpr int kSmemBytes = kOffBar + kNumBars * 8 + 16 + 1024;  // + align slack
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS = 0;     // two S buffers: 0 and 128
  static constexpr uint32_t kColO = 256;   // O accumulator, D columns
  static constexpr uint32_t kIdescS = idesc_bf16_f32(kTileM, kTileN, false, false);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(kTileM, D, false, true);
  static constexpr int kThreads = 224;
};

struct TileInfo {
  int g, h, u, hh;
  int64_t kstart;   // first key token of KV tile 0
  int nkv;          // KV tiles
  int64_t qstart;   // own/dense: first query token
  int qrows;        // valid rows
  int seq;
  int64_t seq_start;
  int own_block;    // own/dense: block of the tile within its sequence
  int64_t e0;       // routed: first entry
};

template <int MODE>
__device__ __forceinline__ int64_t num_items(const AttnArgs& a) {
  if (MODE == kRouted) return a.tile_off[a.nu * a.P.totals[0]];
  if (MODE == kOwn) return (int64_t)a.P.totals[1] * a.nu * a.G;
  return (int64_t)a.P.totals[1] * a.Hq;
}

template <int MODE>
__device__ __forceinline__ TileInfo tile_info(const AttnArgs& a, int64_t w) {
  TileInfo ti;
  if (MODE == kRouted) {
    const int NB = a.P.totals[0];
    const int M = a.nu * NB;
    const int f = upper_index(a.tile_off, M + 1, w);  // bucket of tile w
    const int u = f / NB, J = f % NB;
    const int64_t row0 = (w - a.tile_off[f]) * (int64_t)kTileM;
    const int64_t cnt = (int64_t)a.entry_off[f + 1] - a.entry_off[f];
    ti.u = u;
    ti.g = a.u0 + u;
    ti.h = -1;
    ti.hh = -1;
    ti.kstart = a.P.blk_tok[J];
    ti.nkv = a.B / kTileN;
    ti.qstart = 0;
    ti.qrows = (int)min((int64_t)kTileM, cnt - row0);
    ti.seq = 0;
    ti.seq_start = 0;
    ti.own_block = 0;
    ti.e0 = a.entry_off[f] + row0;
  } else {
    const int HP = (MODE == kOwn) ? a.nu * a.G : a.Hq;
    const int NQT = a.P.totals[1];
    int64_t qt = w / HP;
    const int hl = (int)(w % HP);
    if (MODE == kDense) qt = NQT - 1 - qt;  // longest rows first
    const int s = upper_index(a.P.qt_off, a.L.nseq + 1, qt);
    const int64_t st = seq_start(a.L, s), len = seq_len(a.L, s);
    const int64_t p0 = (qt - a.P.qt_off[s]) * (int64_t)kTileM;
    ti.h = (MODE == kOwn) ? a.u0 * a.G + hl : hl;
    ti.g = ti.h / a.G;
    ti.u = (MODE == kOwn) ? hl / a.G : 0;
    ti.hh = ti.h % a.G;
    ti.seq = s;
    ti.seq_start = st;
    ti.qstart = st + p0;
    ti.qrows = (int)min((int64_t)kTileM, len - p0);
    ti.own_block = (int)(p0 / a.B);
    const int64_t k0 = (MODE == kOwn) ? (int64_t)ti.own_block * a.B : 0;
    ti.kstart = st + k0;
    ti.nkv = (int)((p0 - k0) / kTileN) + 1;
    ti.e0 = 0;
  }
  return ti;
}

template <int D, int MODE>
__global__ void __launch_bounds__(224, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const AttnArgs a) {
  using C = AttnCfg<D>;
  constexpr int ST = C::kStages;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sQ = smem + C::kOffQ;
  unsigned char* sKV = smem + C::kOffKV;
  unsigned char* sP = smem + C::kOffP;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 2;
  uint64_t* kv_full = bars + 4;
  uint64_t* kv_empty = bars + 4 + ST;
  uint64_t* s_full = bars + 4 + 2 * ST;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* pv_done = p_full + 1;
  uint64_t* td_bar = pv_done + 1;
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(td_bar + 1);
  volatile uint32_t* abort_flag = tmem_base_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&q_full[0], 1);
    mbar_init(&q_full[1], 1);
    mbar_init(&q_empty[0], 1);
    mbar_init(&q_empty[1], 1);
    for (int sl = 0; sl < ST; ++sl) {
      mbar_init(&kv_full[sl], 1);
      mbar_init(&kv_empty[sl], 1);
    }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(&s_free[0], kTileM);
    mbar_init(&s_free[1], kTileM);
    mbar_init(p_full, kTileM);
    mbar_init(pv_done, 1);
    mbar_init(td_bar, 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 6) {
    tmem_alloc(tmem_base_slot, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    if (MODE != kRouted) tma_prefetch_desc(&tm_q);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_slot;
  const int64_t items = num_items<MODE>(a);
  const int64_t first = blockIdx.x, step = gridDim.x;
  uint32_t* st = a.status;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t kv_it = 0, lt = 0;
      bool ok = true;
      for (int64_t w = first; w < items && ok; w += step, ++lt) {
        const TileInfo ti = tile_info<MODE>(a, w);
        if (MODE != kRouted) {
          const int qb = lt & 1;
          ok = mbar_wait(&q_empty[qb], ((lt >> 1) & 1) ^ 1, abort_flag, st);
          if (!ok) break;
          mbar_arrive_expect_tx(&q_full[qb], C::kQBytes);
#pragma unroll
          for (int hx = 0; hx < D / 64; ++hx)
            tma_load_3d(sQ + qb * C::kQBytes + hx * C::kHalfBytes, &tm_q, &q_full[qb], hx * 64,
                        ti.h, (int)ti.qstart);
        }
        for (int j = 0; j < ti.nkv && ok; ++j) {
          const int krow = (int)(ti.kstart + (int64_t)j * kTileN);
#pragma unroll
          for (int which = 0; which < 2; ++which) {
            const int sl = kv_it % ST;
            ok = mbar_wait(&kv_empty[sl], ((kv_it / ST) & 1) ^ 1, abort_flag, st);
            if (!ok) break;
            mbar_arrive_expect_tx(&kv_full[sl], C::kKVBytes);
#pragma unroll
            for (int hx = 0; hx < D / 64; ++hx)
              tma_load_3d(sKV + sl * C::kKVBytes + hx * C::kHalfBytes, which ? &tm_v : &tm_k,
                          &kv_full[sl], hx * 64, ti.g, krow);
            ++kv_it;
          }
        }
      }
      if (!ok) {
        // let every TMA load this thread issued land before the CTA exits
        const uint32_t n = kv_it < (uint32_t)ST ? kv_it : (uint32_t)ST;
        for (uint32_t b = 0; b < n; ++b) {
          const uint32_t it = kv_it - 1 - b;
          mbar_wait_teardown(&kv_full[it % ST], (it / ST) & 1, 200000000ull);
        }
        if (MODE != kRouted && lt > 0) {
          for (uint32_t b = 0; b < (lt < 2 ? lt : 2u); ++b) {
            const uint32_t l = lt - 1 - b;
            mbar_wait_teardown(&q_full[l & 1], (l >> 1) & 1, 200000000ull);
          }
        }
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ Q gather
    if (MODE == kRouted) {
      uint32_t lt = 0;
      bool ok = true;
      constexpr int CPR = D / 8;        // 16-B chunks per row
      constexpr int RPI = 32 / CPR;     // rows per warp instruction
      for (int64_t w = first; w < items && ok; w += step, ++lt) {
        const TileInfo ti = tile_info<MODE>(a, w);
        const int qb = lt & 1;
        ok = mbar_wait(&q_empty[qb], ((lt >> 1) & 1) ^ 1, abort_flag, st);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        // lane l holds the entries of rows l, l+32, l+64, l+96
        uint2 ent[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          int r = lane + 32 * m;
          if (r >= ti.qrows) r = 0;
          ent[m] = a.entries[ti.e0 + r];
        }
        const int c = lane % CPR;
        unsigned char* qdst = sQ + qb * C::kQBytes + (c >> 3) * C::kHalfBytes;
#pragma unroll
        for (int it = 0; it < kTileM / RPI; ++it) {
          const int r = it * RPI + lane / CPR;
          const int m = (it * RPI) / 32;  // uniform across the warp
          const uint2 e = make_uint2(__shfl_sync(0xffffffffu, ent[m].x, r & 31),
                                     __shfl_sync(0xffffffffu, ent[m].y, r & 31));
          const bool good = e.x < (uint32_t)a.L.T && (e.y & 0xFFFFu) < (uint32_t)a.G;
          const int hq = ti.g * a.G + (good ? (int)(e.y & 0xFFFFu) : 0);
          const __nv_bfloat16* src = a.q + ((size_t)(good ? e.x : 0u) * a.Hq + hq) * D + c * 8;
          cp_async_16(qdst + sw128_offset(r, c & 7), src);
        }
        cp_async_wait_all();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&q_full[qb]);
      }
      cp_async_wait_all();
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t kv_it = 0, n = 0, lt = 0;
      bool ok = true;
      bool pend = false;
      uint32_t pend_slot = 0, pend_par = 0, pend_n = 0, pend_acc = 0;
      const uint32_t sQa = smem_u32(sQ), sKVa = smem_u32(sKV), sPa = smem_u32(sP);
      auto issue_pv = [&]() -> bool {
        if (!mbar_wait(p_full, pend_n & 1, abort_flag, st)) return false;
        if (!mbar_wait(&kv_full[pend_slot], pend_par, abort_flag, st)) return false;
        tc_fence_after();
        const uint32_t vbase = sKVa + pend_slot * C::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < kTileN / 16; ++kk) {
          const uint64_t ad = sdesc_kmajor_sw128(sPa + (kk >> 2) * C::kHalfBytes + (kk & 3) * 32);
          const uint64_t bd = sdesc_mnmajor_sw128(vbase + kk * 2048, C::kHalfBytes, 1024);
          tc_mma_ss(tmem + C::kColO, ad, bd, C::kIdescPV, (pend_acc || kk > 0) ? 1u : 0u);
        }
        tc_commit(pv_done);
        tc_commit(&kv_empty[pend_slot]);
        return true;
      };
      for (int64_t w = first; w < items && ok; w += step, ++lt) {
        const TileInfo ti = tile_info<MODE>(a, w);
        const int qb = lt & 1;
        ok = mbar_wait(&q_full[qb], (lt >> 1) & 1, abort_flag, st);
        if (!ok) break;
        const uint32_t qbase = sQa + qb * C::kQBytes;
        for (int j = 0; j < ti.nkv; ++j) {
          const uint32_t ks = kv_it % ST;
          ok = mbar_wait(&kv_full[ks], (kv_it / ST) & 1, abort_flag, st);
          if (!ok) break;
          ++kv_it;
          const uint32_t sb = n & 1;
          ok = mbar_wait(&s_free[sb], ((n >> 1) & 1) ^ 1, abort_flag, st);
          if (!ok) break;
          tc_fence_after();
          const uint32_t kbase = sKVa + ks * C::kKVBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::kHalfBytes + (kk & 3) * 32;
            tc_mma_ss(tmem + C::kColS + sb * kTileN, sdesc_kmajor_sw128(qbase + off),
                      sdesc_kmajor_sw128(kbase + off), C::kIdescS, kk > 0 ? 1u : 0u);
          }
          tc_commit(&s_full[sb]);
          tc_commit(&kv_empty[ks]);
          if (j == ti.nkv - 1) tc_commit(&q_empty[qb]);
          if (pend) {
            ok = issue_pv();
            if (!ok) break;
          }
          pend = true;
          pend_slot = kv_it % ST;
          pend_par = (kv_it / ST) & 1;
          pend_n = n;
          pend_acc = j > 0 ? 1u : 0u;
          ++kv_it;
          ++n;
        }
      }
      if (ok && pend) ok = issue_pv();
      // every MMA issued by this thread must finish before TMEM is freed
      tc_commit(td_bar);
      mbar_wait_teardown(td_bar, 0, 500000000ull);
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 0-3)
    const int r = threadIdx.x;  // query row = TMEM lane
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const uint32_t sPa = smem_u32(sP);
    uint32_t n = 0;
    bool ok = true;
    for (int64_t w = first; w < items && ok; w += step) {
      const TileInfo ti = tile_info<MODE>(a, w);
      float m_run = -INFINITY, l_run = 0.f;
      for (int j = 0; j < ti.nkv; ++j) {
        const uint32_t sb = n & 1;
        ok = mbar_wait(&s_full[sb], (n >> 1) & 1, abort_flag, st);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        float s[kTileN];
#pragma unroll
        for (int c4 = 0; c4 < kTileN / 32; ++c4)
          tmem_ld32(tmem + lane_off + C::kColS + sb * kTileN + c4 * 32,
                    *reinterpret_cast<uint32_t(*)[32]>(&s[c4 * 32]));
        tc_wait_ld();
        tc_fence_before();
        mbar_arrive(&s_free[sb]);
        if (MODE != kRouted && j == ti.nkv - 1) {
          // diagonal tile: key kstart + j*128 + c is visible to query qstart + r
          // only when it is not later
          const int64_t lim = ti.qstart + r - (ti.kstart + (int64_t)j * kTileN);
#pragma unroll
          for (int c = 0; c < kTileN; ++c)
            if (c > lim) s[c] = -INFINITY;
        }
        // row max: 8 independent chains of 3-input max, then a short tree
        float mp[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mp[e] = fmaxf(s[e], s[e + 8]);
#pragma unroll
        for (int c = 16; c < kTileN; c += 16) {
#pragma unroll
          for (int e = 0; e < 8; ++e) mp[e] = fmax3f(mp[e], s[c + e], s[c + 8 + e]);
        }
        const float mx = fmaxf(fmax3f(mp[0], mp[1], mp[2]),
                               fmax3f(fmax3f(mp[3], mp[4], mp[5]), mp[6], mp[7]));
        const float m_new = fmaxf(m_run, mx * a.scale_log2);
        const bool need = (j == 0) || (m_new > m_run + 8.0f);
        const float m_use = need ? m_new : m_run;
        const float alpha = (j == 0) ? 0.f : (need ? ex2_approx(m_run - m_use) : 1.f);
        uint32_t pk[kTileN / 2];
        float sp[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) sp[e] = 0.f;
#pragma unroll
        for (int c = 0; c < kTileN; c += 2) {
          const float p0 = ex2_approx(fmaf(s[c], a.scale_log2, -m_use));
          const float p1 = ex2_approx(fmaf(s[c + 1], a.scale_log2, -m_use));
          sp[(c / 2) & 7] += p0 + p1;
          pk[c / 2] = pack_bf16x2(p0, p1);
        }
        const float sum = ((sp[0] + sp[1]) + (sp[2] + sp[3])) + ((sp[4] + sp[5]) + (sp[6] + sp[7]));
        // previous PV done: P buffer free, O stable
        if (n > 0) {
          ok = mbar_wait(pv_done, (n - 1) & 1, abort_flag, st);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
        }
        if (__any_sync(0xffffffffu, j > 0 && need)) {
          tc_fence_after();
          const float f = (j > 0 && need) ? alpha : 1.f;
#pragma unroll
          for (int c4 = 0; c4 < D / 32; ++c4) {
            uint32_t ov[32];
            tmem_ld32(tmem + lane_off + C::kColO + c4 * 32, ov);
            tc_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f);
            tmem_st32(tmem + lane_off + C::kColO + c4 * 32, ov);
          }
          tc_wait_st();
        }
        l_run = l_run * alpha + sum;
        m_run = m_use;
        // P row r -> two 128-B-swizzled halves (keys 0-63, 64-127)
#pragma unroll
        for (int cc = 0; cc < kTileN / 8; ++cc) {
          const uint32_t addr = sPa + (cc >> 3) * C::kHalfBytes + sw128_offset(r, cc & 7);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[cc * 4]),
                       "r"(pk[cc * 4 + 1]), "r"(pk[cc * 4 + 2]), "r"(pk[cc * 4 + 3])
                       : "memory");
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(p_full);
        ++n;
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      ok = mbar_wait(pv_done, (n - 1) & 1, abort_flag, st);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      float o[D];
#pragma unroll
      for (int c4 = 0; c4 < D / 32; ++c4)
        tmem_ld32(tmem + lane_off + C::kColO + c4 * 32,
                  *reinterpret_cast<uint32_t(*)[32]>(&o[c4 * 32]));
      tc_wait_ld();
      tc_fence_before();
      if (r < ti.qrows) {
        const float inv = 1.f / l_run;
        const float lse2 = m_run + lg2_approx(l_run);
        if (MODE == kRouted) {
          const uint2 e = a.entries[ti.e0 + r];
          const int hh = (int)(e.y & 0xFFFFu), sl = (int)(e.y >> 16);
          if (e.x >= (uint32_t)a.L.T || hh >= a.G || sl >= a.topk - 1) {
            atomicOr(a.status, MOBA_DEV_BAD_INDEX);
            continue;
          }
          const int64_t prow = (((int64_t)ti.u * a.L.T + e.x) * a.G + hh) * (a.topk - 1) + sl;
          uint4* dst = reinterpret_cast<uint4*>(a.part_O + prow * D);
#pragma unroll
          for (int c8 = 0; c8 < D / 8; ++c8)
            dst[c8] = make_uint4(pack_bf16x2(o[8 * c8 + 0] * inv, o[8 * c8 + 1] * inv),
                                 pack_bf16x2(o[8 * c8 + 2] * inv, o[8 * c8 + 3] * inv),
                                 pack_bf16x2(o[8 * c8 + 4] * inv, o[8 * c8 + 5] * inv),
                                 pack_bf16x2(o[8 * c8 + 6] * inv, o[8 * c8 + 7] * inv));
          a.part_lse[prow] = lse2;
        } else {
          const int64_t t = ti.qstart + r;
          const bool final_row = (MODE == kDense) || a.topk == 1 || ti.own_block == 0;
          if (final_row) {
            uint4* dst = reinterpret_cast<uint4*>(a.o + ((size_t)t * a.Hq + ti.h) * D);
#pragma unroll
            for (int c8 = 0; c8 < D / 8; ++c8)
              dst[c8] = make_uint4(pack_bf16x2(o[8 * c8 + 0] * inv, o[8 * c8 + 1] * inv),
                                   pack_bf16x2(o[8 * c8 + 2] * inv, o[8 * c8 + 3] * inv),
                                   pack_bf16x2(o[8 * c8 + 4] * inv, o[8 * c8 + 5] * inv),
                                   pack_bf16x2(o[8 * c8 + 6] * inv, o[8 * c8 + 7] * inv));
            a.lse[row_index(a.R, ti.seq, ti.h, t - ti.seq_start, t)] =
                lse2 * 0.6931471805599453f;
          } else {
            const int64_t prow = ((int64_t)ti.u * a.L.T + t) * a.G + ti.hh;
            float4* dst = reinterpret_cast<float4*>(a.own_O + prow * D);
#pragma unroll
            for (int c4 = 0; c4 < D / 4; ++c4)
              dst[c4] = make_float4(o[4 * c4] * inv, o[4 * c4 + 1] * inv, o[4 * c4 + 2] * inv,
                                    o[4 * c4 + 3] * inv);
            a.own_lse[prow] = lse2;
          }
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 6) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace moba
