// gate_tc.cuh -- the MoBA gate with its scores on the sm_100a tensor cores.
//
// For every query row t of head h (kv head g = h / G) whose own block is i,
// the gate needs the affinity s_j = <q_t, Kbar_j> with the mean key of every
// past block j < i, keeps the k-1 largest (ties to the lower block index) and
// appends the own block (MoBA: Mixture of Block Attention, wispaper.ai blog,
// "The Change": affinity score, top-k routing, causality; sherconan.github.io
// steps 2-4).  The output row is the k-1 kept past blocks in ascending order
// followed by i.
//
// Scores.  S = Q_tile (128 rows x d, bf16) x Kbar^T is a dense contraction
// and runs as tcgen05 MMAs into TMEM (M = 128, N = the past blocks rounded up
// to 16, at most 256).  Kbar is fp32; it enters the MMA as two bf16 parts,
// hi = bf16(Kbar) and lo = bf16(Kbar - hi), accumulated into the same fp32
// tile, so the score carries about 16 significant bits of Kbar.
//
// Selection, per row (one thread per row, the row is its TMEM lane):
//   1. a lower bound T0 on the row's (k-1)-th largest score: the (k-1)-th
//      largest of the maxima of groups of GS consecutive scores (there are at
//      least 2(k-1) groups, and each group maximum is a score, so at least
//      k-1 scores are >= T0);
//   2. the candidates (scores >= T0) are compacted, in ascending block order,
//      into a per-row list in shared memory (a few dozen at most);
//   3. T1 = the (k-1)-th largest candidate; the kept set is every candidate
//      above T1 plus, in ascending block order, as many candidates equal to T1
//      as are still needed.
// The work per score is branch-free; the only divergent step is a rare
// fallback (a row with more candidates than the list holds, e.g. many equal
// scores) that ranks the whole row with an insertion list.
//
// Persistent CTA, one per SM, 11 warps:
//   warps 0-3  select for the score buffer 0 (even scored items)
//   warps 4-7  select for the score buffer 1 (odd scored items)
//   warp  8    TMA producer of the Q tiles (double-buffered)
//   warp  9    TMEM allocation and the MMA issue (one elected lane)
//   warp 10    Kbar loader: fp32 block means -> bf16 hi / lo, swizzled in
//              shared memory
// Work items are (kv head, query tile, head of the group), CTA c taking items
// c, c + gridDim.x, ...  Successive items of a CTA therefore keep the same kv
// head and move forward through the sequence, so the block means it holds
// stay valid and only the newly needed rows are appended.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"
#include "layout.cuh"

namespace moba {

constexpr int kGateTcMaxPast = 256;  // past blocks one score tile holds (TMEM columns)
constexpr int kGateTcMaxKeep = 32;   // largest k-1 this kernel ranks
// k-1 <= 16: score tiles of up to 256 past blocks, 24 candidate slots per row;
// 16 < k-1 <= 32: up to 128 past blocks (the block means of 256 would not fit
// shared memory beside the longer candidate lists), 48 slots.
constexpr int gate_tc_max_past(int KM) { return KM <= 16 ? 256 : 128; }

struct GateTcArgs {
  const float* kbar;  // [Hkv][NBmax][D] fp32 block means
  int Hq, G, B, topk, NBmax;
  SeqLayout L;
  Plan P;
  RowLayout R;
  int32_t* sel;
  uint32_t* status;
  int g0, ng;     // kv heads g0 .. g0 + ng - 1 (their items are contiguous)
  int companion;  // 1: query tiles with more past blocks than a score tile holds
                  // are left to the SIMT gate, launched after this kernel
};

template <int D, int KM>
struct GateTcCfg {
  static constexpr int kMaxPast = gate_tc_max_past(KM);
  static constexpr int kCap = KM <= 16 ? 24 : 48;           // candidate slots per row
  static constexpr int kQHalf = kTileM * 128;               // 128 rows x 64 columns bf16
  static constexpr int kQBytes = kTileM * D * 2;
  static constexpr int kKbHalf = kMaxPast * 128;            // kMaxPast rows x 64 columns bf16
  static constexpr int kKbBytes = kMaxPast * D * 2;         // one part (hi or lo)
  static constexpr int kOffQ = 0;
  static constexpr int kOffKb = kOffQ + 2 * kQBytes;
  static constexpr int kOffCv = kOffKb + 2 * kKbBytes;                  // float [2][cap][128]
  static constexpr int kOffCi = kOffCv + 2 * kCap * kTileM * 4;         // uint8 [2][cap][128]
  static constexpr int kOffBar = kOffCi + 2 * kCap * kTileM;
  static constexpr int kNumBars = 2 * 6 + 1;
  static constexpr int kSmemBytes = kOffBar + kNumBars * 8 + 16 + 1024;
  static constexpr int kThreads = 352;
  static constexpr uint32_t kTmemCols = 512;  // two 256-column score buffers
  static_assert(kSmemBytes <= 232448, "gate shared memory beyond the per-CTA limit");
};

struct GateTcItem {
  int g, h, s, i, rows;
  int64_t st, p0;
  bool direct;  // no scoring: k = 1, or every past block is kept
  bool bad;     // more past blocks than a score tile holds (the SIMT gate's)
};

__device__ __forceinline__ GateTcItem gate_tc_item(const GateTcArgs& a, int64_t w,
                                                   int max_past) {
  GateTcItem it;
  const int NQT = a.P.totals[1];
  const int64_t per_g = (int64_t)NQT * a.G;
  it.g = (int)(w / per_g);
  const int64_t rem = w - (int64_t)it.g * per_g;
  const int qt = (int)(rem / a.G);
  it.h = it.g * a.G + (int)(rem - (int64_t)qt * a.G);
  it.s = upper_index(a.P.qt_off, a.L.nseq + 1, qt);
  it.st = seq_start(a.L, it.s);
  it.p0 = (int64_t)(qt - a.P.qt_off[it.s]) * kTileM;
  it.i = (int)(it.p0 / a.B);
  it.rows = (int)min((int64_t)kTileM, seq_len(a.L, it.s) - it.p0);
  const int npast = a.topk - 1;
  it.direct = (npast == 0) || (it.i <= npast);
  it.bad = !it.direct && it.i > max_past;
  return it;
}

// Insert v into the descending list t[0..KM) (values only, branch-free).
template <int KM>
__device__ __forceinline__ void chain_insert(float (&t)[KM], float v) {
#pragma unroll
  for (int u = 0; u < KM; ++u) {
    const float hi = fmaxf(t[u], v);
    v = fminf(t[u], v);
    t[u] = hi;
  }
}

// Insert v into the ascending list t[0..L) of the L smallest values.
template <int L>
__device__ __forceinline__ void chain_insert_min(float (&t)[L], float v) {
#pragma unroll
  for (int u = 0; u < L; ++u) {
    const float lo = fminf(t[u], v);
    v = fmaxf(t[u], v);
    t[u] = lo;
  }
}

template <int KM>
__device__ __forceinline__ float list_at(const float (&t)[KM], int idx) {
  float r = t[0];
#pragma unroll
  for (int u = 1; u < KM; ++u)
    if (u == idx) r = t[u];
  return r;
}

// Pass 1 over one 32-score chunk: maxima of GS-score groups into the list.
template <int GS, int KM>
__device__ __forceinline__ void chunk_group_max(const float (&v)[32], float (&t)[KM]) {
#pragma unroll
  for (int g0 = 0; g0 < 32; g0 += GS) {
    float m = v[g0];
#pragma unroll
    for (int e = 1; e < GS; ++e) m = fmaxf(m, v[g0 + e]);
    chain_insert<KM>(t, m);
  }
}

// Candidate store: score v at shared address av and its column id at ai,
// when take != 0 (predicated stores, so the caller's loop has no branch).
__device__ __forceinline__ void st_shared_pred(uint32_t av, uint32_t ai, float v, int id,
                                               uint32_t take) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.u32 p, %4, 0;\n\t"
      "@p st.shared.f32 [%0], %2;\n\t"
      "@p st.shared.u8 [%1], %3;\n\t}" ::"r"(av),
      "r"(ai), "f"(v), "r"(id), "r"(take)
      : "memory");
}

// Scores of columns [c, c + 32) of this lane's TMEM row; columns >= ncol -> -inf.
__device__ __forceinline__ void load_scores(uint32_t taddr, int c, int ncol, float (&v)[32]) {
  uint32_t u[32];
  tmem_ld32(taddr + c, u);
  tc_wait_ld();
#pragma unroll
  for (int e = 0; e < 32; ++e)
    v[e] = (c + e < ncol) ? __uint_as_float(u[e]) : __int_as_float(0xff800000);
}

template <int D, int KM>
__global__ void __launch_bounds__(352, 1)
    gate_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const GateTcArgs a) {
  using C = GateTcCfg<D, KM>;
  constexpr int kCap = C::kCap;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sQ = smem + C::kOffQ;
  unsigned char* sKb = smem + C::kOffKb;
  float* cv_all = reinterpret_cast<float*>(smem + C::kOffCv);
  uint8_t* ci_all = smem + C::kOffCi;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 2;
  uint64_t* kb_full = bars + 4;
  uint64_t* kb_empty = bars + 6;
  uint64_t* s_full = bars + 8;
  uint64_t* s_free = bars + 10;
  uint64_t* td_bar = bars + 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&q_full[b], 1);
      mbar_init(&q_empty[b], 1);
      mbar_init(&kb_full[b], 1);
      mbar_init(&kb_empty[b], 1);
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], 4);  // one elected arrival per select warp
    }
    mbar_init(td_bar, 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int64_t per_g = (int64_t)a.P.totals[1] * a.G;
  const int64_t items = (int64_t)(a.g0 + a.ng) * per_g;
  const int64_t first = (int64_t)a.g0 * per_g + blockIdx.x, step = gridDim.x;
  uint32_t* st = a.status;
  const int npast = a.topk - 1;

  if (warp == 8) {
    // ------------------------------------------------------------ Q producer
    if (lane == 0) {
      uint32_t n = 0;
      bool ok = true;
      for (int64_t w = first; w < items && ok; w += step) {
        const GateTcItem it = gate_tc_item(a, w, C::kMaxPast);
        if (it.direct || it.bad) continue;
        const int b = n & 1;
        ok = mbar_wait(&q_empty[b], ((n >> 1) & 1) ^ 1, abort_flag, st);
        if (!ok) break;
        mbar_arrive_expect_tx(&q_full[b], C::kQBytes);
#pragma unroll
        for (int hx = 0; hx < D / 64; ++hx)
          tma_load_3d(sQ + b * C::kQBytes + hx * C::kQHalf, &tm_q, &q_full[b], hx * 64, it.h,
                      (int)(it.st + it.p0));
        ++n;
      }
      if (!ok) {
        for (uint32_t k = 0; k < (n < 2u ? n : 2u); ++k) {
          const uint32_t l = n - 1 - k;
          mbar_wait_teardown(&q_full[l & 1], (l >> 1) & 1, 200000000ull);
        }
      }
    }
  } else if (warp == 10) {
    // ------------------------------------------------------------ Kbar loader
    constexpr int C4 = D / 4;        // float4 per Kbar row
    constexpr int RPI = 32 / C4;     // rows per warp step
    const int sub = lane % C4, rsub = lane / C4;
    const int c = 4 * sub, hx = c / 64, cc = c % 64;
    const uint32_t col_off = (uint32_t)hx * C::kKbHalf + (uint32_t)(cc % 8) * 2;
    uint32_t n = 0;
    int cur_s = -1, cur_g = -1, loaded = 0;
    bool ok = true;
    for (int64_t w = first; w < items && ok; w += step) {
      const GateTcItem it = gate_tc_item(a, w, C::kMaxPast);
      if (it.direct || it.bad) continue;
      const int b = n & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&kb_empty[b], ((n >> 1) & 1) ^ 1, abort_flag, st));
      if (!ok) break;
      int from = loaded;
      if (it.s != cur_s || it.g != cur_g || it.i < loaded) {
        // rows below `loaded` change: wait until the MMAs of the previous
        // item (and so of every earlier one) have read them
        if (n > 0) {
          const uint32_t pn = n - 1;
          ok = __all_sync(0xffffffffu,
                          mbar_wait(&kb_empty[pn & 1], (pn >> 1) & 1, abort_flag, st));
          if (!ok) break;
        }
        from = 0;
        loaded = 0;
        cur_s = it.s;
        cur_g = it.g;
      }
      const float* src = a.kbar + ((size_t)it.g * a.NBmax + a.P.blk_off[it.s]) * D;
      for (int j0 = from; j0 < it.i; j0 += RPI) {
        const int j = j0 + rsub;
        if (j < it.i) {
          const float4 x = __ldg(reinterpret_cast<const float4*>(src + (size_t)j * D) + sub);
          const __nv_bfloat162 h01 = __floats2bfloat162_rn(x.x, x.y);
          const __nv_bfloat162 h23 = __floats2bfloat162_rn(x.z, x.w);
          const float2 f01 = __bfloat1622float2(h01), f23 = __bfloat1622float2(h23);
          const __nv_bfloat162 l01 = __floats2bfloat162_rn(x.x - f01.x, x.y - f01.y);
          const __nv_bfloat162 l23 = __floats2bfloat162_rn(x.z - f23.x, x.w - f23.y);
          const uint32_t off = col_off + sw128_offset((uint32_t)j, (uint32_t)(cc / 8));
          *reinterpret_cast<uint2*>(sKb + off) =
              make_uint2(*reinterpret_cast<const uint32_t*>(&h01),
                         *reinterpret_cast<const uint32_t*>(&h23));
          *reinterpret_cast<uint2*>(sKb + C::kKbBytes + off) =
              make_uint2(*reinterpret_cast<const uint32_t*>(&l01),
                         *reinterpret_cast<const uint32_t*>(&l23));
        }
      }
      if (it.i > loaded) loaded = it.i;
      fence_proxy_async_smem();  // generic stores -> visible to the tensor core
      __syncwarp();
      if (lane == 0) mbar_arrive(&kb_full[b]);
      ++n;
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    uint32_t n = 0;
    bool ok = true;
    const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sKb);
    auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, st));
    };
    for (int64_t w = first; w < items && ok; w += step) {
      const GateTcItem it = gate_tc_item(a, w, C::kMaxPast);
      if (it.direct || it.bad) continue;
      const int b = n & 1;
      const uint32_t ph = (n >> 1) & 1;
      if (!(ok = wait(&q_full[b], ph))) break;
      if (!(ok = wait(&kb_full[b], ph))) break;
      if (!(ok = wait(&s_free[b], ph ^ 1))) break;
      tc_fence_after();
      const int ncol = it.i < 16 ? 16 : ((it.i + 15) & ~15);
      const uint32_t idesc = idesc_bf16_f32(kTileM, ncol, false, false);
      const uint32_t qbase = sQa + b * C::kQBytes;
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        const uint32_t kbase = sKa + part * C::kKbBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t qoff = (kk >> 2) * C::kQHalf + (kk & 3) * 32;
          const uint32_t koff = (kk >> 2) * C::kKbHalf + (kk & 3) * 32;
          tc_mma_ss_warp(tmem + b * 256, sdesc_kmajor_sw128(qbase + qoff),
                         sdesc_kmajor_sw128(kbase + koff), idesc,
                         (part > 0 || kk > 0) ? 1u : 0u);
        }
      }
      tc_commit_warp(&s_full[b]);
      tc_commit_warp(&q_empty[b]);
      tc_commit_warp(&kb_empty[b]);
      ++n;
    }
    tc_commit_warp(td_bar);
    mbar_wait_teardown(td_bar, 0, 500000000ull);
  } else {
    // ------------------------------------------------------------ select (warps 0-7)
    const int grp = warp >> 2, quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t tS = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)grp * 256;
    float* cv = cv_all + grp * kCap * kTileM + r;    // slot q at cv[q * kTileM]
    uint8_t* ci = ci_all + grp * kCap * kTileM + r;
    const uint32_t cv_s = smem_u32(cv), ci_s = smem_u32(ci);
    uint32_t n = 0, li = 0;
    bool ok = true;
    for (int64_t w = first; w < items && ok; w += step, ++li) {
      const GateTcItem it = gate_tc_item(a, w, C::kMaxPast);
      const bool valid = r < it.rows;
      const int64_t pos = it.p0 + r;
      int32_t* out = a.sel + row_index(a.R, it.s, it.h, pos, it.st + pos) * a.topk;
      if (it.direct || it.bad) {
        if ((int)(li & 1) != grp) continue;
        if (it.bad) {
          if (r == 0 && !a.companion) atomicOr(st, MOBA_DEV_CAPACITY);
          continue;
        }
        if (valid) {
          const int nch = min(it.i, npast);
          for (int u = 0; u < a.topk; ++u) out[u] = u < nch ? u : (u == nch ? it.i : -1);
        }
        continue;
      }
      const uint32_t my = n++;
      if ((int)(my & 1) != grp) continue;
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[grp], (my >> 1) & 1, abort_flag, st));
      if (!ok) break;
      tc_fence_after();
      const int ncol = it.i;
      // ---- pass 1: T0 from group maxima.  At least 2(k-1) groups: with
      // i.i.d. scores that leaves about k + 2 candidates and almost never
      // more than the list holds (with exactly k-1 groups, a quarter of the
      // rows overflowed at 200 blocks).
      int gs = 16;
      while (gs > 1 && (ncol + gs - 1) / gs < 2 * npast) gs >>= 1;
      float t[KM];
#pragma unroll
      for (int u = 0; u < KM; ++u) t[u] = __int_as_float(0xff800000);
      for (int c = 0; c < ncol; c += 32) {
        float v[32];
        load_scores(tS, c, ncol, v);
        switch (gs) {
          case 16: chunk_group_max<16, KM>(v, t); break;
          case 8: chunk_group_max<8, KM>(v, t); break;
          case 4: chunk_group_max<4, KM>(v, t); break;
          case 2: chunk_group_max<2, KM>(v, t); break;
          default: chunk_group_max<1, KM>(v, t); break;
        }
      }
      const float T0 = list_at<KM>(t, npast - 1);
      // ---- pass 2: candidates (>= T0) in ascending block order
      int nc = 0;
      for (int c = 0; c < ncol; c += 32) {
        float v[32];
        load_scores(tS, c, ncol, v);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const uint32_t take = v[e] >= T0 ? 1u : 0u;
          const uint32_t slot = (uint32_t)min(nc, kCap - 1);
          // predicated stores, no branch: a row takes a candidate here or not
          st_shared_pred(cv_s + slot * (kTileM * 4), ci_s + slot * kTileM, v[e], c + e, take);
          nc += (int)take;
        }
      }
      if (!valid) nc = 0;
      const bool overflow = nc > kCap;
      // ---- rare fallback: rank the whole row with an insertion list
      int32_t fb[KM];
      if (__any_sync(0xffffffffu, overflow)) {
        float bs[KM];
#pragma unroll
        for (int u = 0; u < KM; ++u) {
          bs[u] = (u < KM - npast) ? __int_as_float(0x7f800000) : __int_as_float(0xff800000);
          fb[u] = -1;
        }
        for (int c = 0; c < ncol; c += 32) {
          float v[32];
          load_scores(tS, c, ncol, v);
          if (overflow) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float sc = v[e];
              if (c + e < ncol && sc > bs[KM - 1]) {  // strict: an equal earlier block stays
                bs[KM - 1] = sc;
                fb[KM - 1] = c + e;
#pragma unroll
                for (int u = KM - 1; u > 0; --u) {
                  const bool up = bs[u] > bs[u - 1];
                  const float ts = up ? bs[u - 1] : bs[u];
                  const int32_t tj = up ? fb[u - 1] : fb[u];
                  bs[u - 1] = up ? bs[u] : bs[u - 1];
                  fb[u - 1] = up ? fb[u] : fb[u - 1];
                  bs[u] = ts;
                  fb[u] = tj;
                }
              }
            }
          }
        }
        // kept ids ascending (odd-even transposition network)
#pragma unroll
        for (int u = 0; u < KM; ++u) fb[u] = (u >= KM - npast) ? fb[u] : 0x7fffffff;
#pragma unroll
        for (int rd = 0; rd < KM; ++rd) {
#pragma unroll
          for (int u = (rd & 1); u + 1 < KM; u += 2) {
            const int32_t x0 = fb[u], x1 = fb[u + 1];
            fb[u] = min(x0, x1);
            fb[u + 1] = max(x0, x1);
          }
        }
      }
      // the score buffer is no longer read
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[grp]);
      if (!valid) continue;
      if (overflow) {
        for (int u = 0; u < npast; ++u) {
          int32_t v = -1;
#pragma unroll
          for (int q = 0; q < KM; ++q)
            if (q == u) v = fb[q];
          out[u] = v;
        }
        out[npast] = it.i;
        continue;
      }
      // ---- pass 3: T1 = (k-1)-th largest candidate, then the kept set
#pragma unroll
      for (int u = 0; u < KM; ++u) t[u] = __int_as_float(0xff800000);
      int kept = 0;
      if (kCap <= 24) {
        // short lists: every slot into registers (independent loads), slots
        // past nc as -inf, then fixed-length loops with no divergence
        float cvr[kCap];
#pragma unroll
        for (int q = 0; q < kCap; ++q) {
          const float x = cv[q * kTileM];
          cvr[q] = q < nc ? x : __int_as_float(0xff800000);
        }
        // T1 = the (k-1)-th largest candidate = the (nc - (k-1) + 1)-th
        // smallest.  A row has a few candidates more than k-1 (about two
        // for i.i.d. scores), so a list of the 4 smallest usually settles it.
        const int drop = max(nc - npast, 0);
        float T1;
        // the lanes here are this warp's valid rows without an overflow
        if (__all_sync(__activemask(), drop < 4)) {
          float sm[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) sm[u] = __int_as_float(0x7f800000);
#pragma unroll
          for (int q = 0; q < kCap; ++q)
            chain_insert_min<4>(sm, q < nc ? cvr[q] : __int_as_float(0x7f800000));
          T1 = list_at<4>(sm, drop);
        } else {
#pragma unroll
          for (int q = 0; q < kCap; ++q) chain_insert<KM>(t, cvr[q]);
          T1 = list_at<KM>(t, npast - 1);
        }
        int gt = 0;
#pragma unroll
        for (int q = 0; q < kCap; ++q) gt += cvr[q] > T1 ? 1 : 0;
        int eq_left = npast - gt;  // candidates equal to T1 still to keep, lowest blocks first
#pragma unroll
        for (int q = 0; q < kCap; ++q) {
          const bool eq = q < nc && cvr[q] == T1;
          const bool take = cvr[q] > T1 || (eq && eq_left > 0);
          eq_left -= (eq && take) ? 1 : 0;
          const int32_t id = (int32_t)ci[q * kTileM];
          if (take && kept < npast) out[kept] = id;
          kept += take ? 1 : 0;
        }
      } else if (nc <= npast) {
        // no more candidates than kept blocks (pass 1's bound was exact, as
        // it is whenever every score is its own group): keep them all
        for (int q = 0; q < nc; ++q) out[q] = (int32_t)ci[q * kTileM];
        kept = nc;
      } else {
        for (int q = 0; q < nc; ++q) chain_insert<KM>(t, cv[q * kTileM]);
        const float T1 = list_at<KM>(t, npast - 1);
        int gt = 0;
        for (int q = 0; q < nc; ++q) gt += cv[q * kTileM] > T1 ? 1 : 0;
        int eq_left = npast - gt;  // candidates equal to T1 still to keep, lowest blocks first
        for (int q = 0; q < nc; ++q) {
          const float v = cv[q * kTileM];
          bool take = v > T1;
          if (v == T1 && eq_left > 0) {
            take = true;
            --eq_left;
          }
          if (take && kept < npast) out[kept] = (int32_t)ci[q * kTileM];
          kept += take ? 1 : 0;
        }
      }
      for (int u = kept; u < npast; ++u) out[u] = -1;  // only with non-finite scores
      out[npast] = it.i;
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// Bucket sizes for the routed attention from the selections: counts[g][J]
// += the (row, head, slot) selections of global past block J by the heads of
// kv head g.  One CTA per (query tile, kv head), counters in shared memory.
__global__ void __launch_bounds__(128) gate_count_kernel(
    const int32_t* __restrict__ sel, RowLayout R, int topk, int B, int G, SeqLayout L, Plan P,
    int NBmax, uint32_t* __restrict__ counts, uint32_t* __restrict__ status, int g0 = 0) {
  extern __shared__ uint32_t ccnt[];  // [blocks of the sequence]
  const int qt = blockIdx.x, g = g0 + blockIdx.y;  // kv heads g0 .. g0 + gridDim.y - 1
  if (qt >= P.totals[1]) return;
  const int s = upper_index(P.qt_off, L.nseq + 1, qt);
  const int64_t st = seq_start(L, s), len = seq_len(L, s);
  const int64_t p0 = (int64_t)(qt - P.qt_off[s]) * kTileM;
  const int i = (int)(p0 / B);
  if (i == 0 || topk == 1) return;
  if (i > kMaxBlocksPerSeq) {  // uniform over the CTA
    if (threadIdx.x == 0) atomicOr(status, MOBA_DEV_CAPACITY);
    return;
  }
  for (int j = threadIdx.x; j < i; j += blockDim.x) ccnt[j] = 0;
  __syncthreads();
  const int npast = min(topk - 1, i);
  const int64_t pos = p0 + threadIdx.x;
  if (pos < len) {
    for (int hh = 0; hh < G; ++hh) {
      const int32_t* row = sel + row_index(R, s, g * G + hh, pos, st + pos) * topk;
      for (int u = 0; u < npast; ++u) {
        const int32_t j = row[u];
        if (j >= 0 && j < i) atomicAdd(&ccnt[j], 1u);
      }
    }
  }
  __syncthreads();
  uint32_t* dst = counts + (size_t)g * NBmax + P.blk_off[s];
  for (int j = threadIdx.x; j < i; j += blockDim.x)
    if (ccnt[j]) atomicAdd(&dst[j], ccnt[j]);
}

}  // namespace moba
