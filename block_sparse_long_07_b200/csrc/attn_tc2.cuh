// attn_tc2.cuh -- exact softmax attention on the sm_100a tensor cores for the
// MoBA prefill forward, two query sub-tiles per CTA.
//
// Modes (MoBA: Mixture of Block Attention, wispaper.ai blog, "Efficiency and
// Implementation": current-block attention plus attention over the routed
// historical blocks, combined by online softmax):
//   kRouted : up to 256 gathered (token, q-head) rows that chose the same past
//             block J, against the B keys of J, no mask.  Each row writes a
//             normalised partial O (fp16) and its log2-domain lse to its slot.
//   kOwn    : two consecutive 128-row query tiles of one head against their
//             own block up to the diagonal, causal mask on the diagonal tile
//             (wispaper.ai blog, "The Change": the current block is always
//             attended, causally).  Rows whose selection is the own block
//             alone write the final O / lse; the others an fp32 partial.
//   kDense  : two consecutive 128-row tiles against every earlier key of the
//             sequence: full causal attention, the k = n limit.
//
// Work item = two 128-row sub-tiles (X = 0, 1) sharing one stream of 128-key
// K/V tiles; sub-tile X uses the first nkv[X] of them.  CTA = 11 warps:
//   warps 0-3   softmax + epilogue of sub-tile 0 (thread r = row r = TMEM lane r)
//   warps 4-7   softmax + epilogue of sub-tile 1
//   warp  8     TMA producer: Q tiles (own/dense) and the K/V ring
//   warp  9     TMEM allocation and MMA issue (one elected lane per MMA)
//   warp 10     Q row gather for routed items (TMA four-row gathers)
// Each Q buffer carries its item's descriptor in shared memory, written by
// whoever fills the buffer and released by the softmax warps once read.  The
// buffer itself is released when the item's last S MMAs complete, one KV step
// before its last PV MMAs.
// TMEM (512 columns): S_X at 128*X (fp32 scores; after the softmax the first
// 64 columns hold P_X as packed bf16, and on the first tile of an own/dense
// block columns 64..95 hold the residual weights of rows 0..63), O_X at
// 256 + D*X.
// Per KV tile j and sub-tile X: S_X = Q_X K_j^T (both operands in shared
// memory); the softmax reads S_X, keeps a running max / sum, writes P_X back
// into TMEM; O_X += P_X V_j takes P_X straight from TMEM, so P never touches
// shared memory.  The MMA thread alternates the sub-tiles, so one softmax
// warpgroup works while the tensor core runs the other sub-tile's MMAs.  The
// softmax signals once the first 64 keys of P_X are in TMEM (p_half) and
// again when all are (p_full): the first half of the PV MMAs runs while the
// second half of the exponentials is computed.
// Tensor-core operations issued by one thread complete in issue order: when
// S_X(j) is complete, PV_X(j-1) (issued before it) is too, which is what lets
// the softmax rescale O_X right after seeing S_X(j).  The max is rescaled
// lazily (only when it grows by more than 2^8).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "aux_kernels.cuh"
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
  int u0, nu;              // pass: kv heads u0 .. u0+nu-1
  const int32_t* tile_off;   // routed: [nu*NB + 1] work items per bucket, prefix
  const int32_t* entry_off;  // routed: [nu*NB + 1] bucket entries, prefix
  const uint2* entries;
  __half* part_O;            // [nu][T][G][topk-1][D], fp16 (see the epilogue)
  float* part_lse;           // [nu][T][G][topk-1]
  float* own_O;              // [nu][T][G][D]
  float* own_lse;            // [nu][T][G]
  __nv_bfloat16* o;          // [T][Hq][D]
  float* lse;
  uint32_t* status;  // status[1]: largest |v| magnitude (vbound_kernel)
};

// QB = Q buffers.  Long items (a block of 8 or more KV tiles, and the dense
// kernel) take one Q buffer and a deep K/V ring: the ring runs a full KV step
// ahead so that each TMA load has an MMA iteration to land in, and refilling
// Q once per item costs little.  Short items (blocks of up to 1024 keys) take
// two Q buffers, so the next item's rows are gathered (or loaded) while this
// item computes; for d = 128 that leaves room for three ring slots.
template <int D, int QB>
struct Attn2Cfg {
  static constexpr int kQBufs = QB;
  static constexpr int kStages = (D == 64) ? 8 : (QB == 2 ? 3 : 5);
  static constexpr int kHalfBytes = kTileM * 128;          // 128 rows x 64 columns bf16
  static constexpr int kSubQBytes = kTileM * D * 2;        // one 128-row Q sub-tile
  static constexpr int kQBytes = 2 * kSubQBytes;           // one work item's Q
  static constexpr int kKVBytes = kTileN * D * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = kOffQ + kQBufs * kQBytes;
  static constexpr int kOffBar = kOffKV + kStages * kKVBytes;
  static constexpr int kNumBars = 3 * kQBufs + 2 * kStages + 2 + 2 + 2 + 2 + 1 + 2;
  static constexpr int kOffItem = kOffBar + kNumBars * 8 + 16;  // [QB] item descriptors
  static constexpr int kItemBytes = 96;
  static constexpr int kSmemBytes = kOffItem + kQBufs * kItemBytes + 1024;
  static_assert(kSmemBytes <= 232448, "attention shared memory beyond the per-CTA limit");
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kIdescS = idesc_bf16_f32(kTileM, kTileN, false, false);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(kTileM, D, false, true);
  static constexpr int kThreads = 352;
  static __host__ __device__ constexpr uint32_t col_s(int x) { return 128u * x; }
  static __host__ __device__ constexpr uint32_t col_o(int x) { return 256u + D * x; }
};

struct Item {
  int g;              // kv head
  int h;              // q head (own/dense)
  int u;              // unit (kv head) within the pass
  int64_t kstart;     // first key of KV tile 0
  int nkv;            // KV tiles streamed (max over sub-tiles)
  int nkv_x[2];       // KV tiles each sub-tile uses (0 = sub-tile idle)
  int rows_x[2];      // valid rows of each sub-tile
  int64_t qstart;     // own/dense: first query token of sub-tile 0
  int seq;
  int64_t seq_start;
  int own_block;      // own/dense: block index of the tiles within the sequence
  int64_t e0;         // routed: first entry of sub-tile 0
};

template <int MODE>
__device__ __forceinline__ int64_t num_items2(const AttnArgs& a, int pair_own) {
  if (MODE == kRouted) return a.tile_off[a.nu * a.P.totals[0]];
  const int64_t HP = (MODE == kOwn) ? (int64_t)a.nu * a.G : a.Hq;
  // items per head: query-tile pairs (or single tiles when own tiles cannot pair)
  const int64_t tiles = a.P.totals[1];
  const int64_t per_head = (MODE == kOwn && !pair_own) ? tiles : a.P.totals[2];
  return per_head * HP;
}

// Routed item w of bucket f, from the bucket's first item tile_lo, its
// entry range [e_lo, e_hi) and its block's first token.
__device__ __forceinline__ Item routed_fill(const AttnArgs& a, int64_t w, int f, int tile_lo,
                                            int e_lo, int e_hi, int blk_tok) {
  Item it;
  const int NB = a.P.totals[0];
  const int64_t row0 = (w - tile_lo) * (int64_t)(2 * kTileM);
  const int64_t left = (int64_t)(e_hi - e_lo) - row0;
  it.u = f / NB;
  it.g = a.u0 + it.u;
  it.h = -1;
  it.kstart = blk_tok;
  it.nkv = a.B / kTileN;
  it.rows_x[0] = (int)min((int64_t)kTileM, left);
  it.rows_x[1] = (int)max((int64_t)0, min((int64_t)kTileM, left - kTileM));
  it.nkv_x[0] = it.nkv;
  it.nkv_x[1] = it.rows_x[1] > 0 ? it.nkv : 0;
  it.qstart = 0;
  it.seq = 0;
  it.seq_start = 0;
  it.own_block = 0;
  it.e0 = e_lo + row0;
  return it;
}

// Routed item w of bucket f (tile_off[f] <= w < tile_off[f + 1]).
__device__ __forceinline__ Item routed_item(const AttnArgs& a, int64_t w, int f) {
  return routed_fill(a, w, f, a.tile_off[f], a.entry_off[f], a.entry_off[f + 1],
                     a.P.blk_tok[f % a.P.totals[0]]);
}

// Routed item w for a whole warp, searched forward from the bucket f of an
// earlier item (a CTA visits its items in increasing order): lane l reads
// bucket f + l's bounds, entry range and block start in one round of loads,
// and the first bucket whose end lies past w is the item's.  Falls back to
// a binary search after two rounds.  Returns the bucket.
__device__ __forceinline__ int routed_next(const AttnArgs& a, int64_t w, int f, int lane,
                                           Item& it) {
  const int NB = a.P.totals[0];
  const int M = a.nu * NB;
#pragma unroll 1
  for (int round = 0; round < 2; ++round, f += 32) {
    const int i = f + lane;
    const bool in = i < M;
    const int64_t end = in ? (int64_t)a.tile_off[i + 1] : INT64_MAX;
    const int lo = in ? a.tile_off[i] : 0;
    const int e_lo = in ? a.entry_off[i] : 0;
    const int e_hi = in ? a.entry_off[i + 1] : 0;
    const int bt = in ? a.P.blk_tok[i % NB] : 0;
    const unsigned b = __ballot_sync(0xffffffffu, end > w);
    if (b) {
      const int L = __ffs(b) - 1;
      it = routed_fill(a, w, f + L, __shfl_sync(0xffffffffu, lo, L),
                       __shfl_sync(0xffffffffu, e_lo, L), __shfl_sync(0xffffffffu, e_hi, L),
                       __shfl_sync(0xffffffffu, bt, L));
      return f + L;
    }
  }
  f += upper_index(a.tile_off + f, M + 1 - f, w);
  it = routed_item(a, w, f);
  return f;
}

// Work item w of the launch.  For own/dense modes the items of one head are
// query-tile pairs numbered through P.totals[2] / P.pair_off (see plan).
template <int MODE>
__device__ __forceinline__ Item item_info(const AttnArgs& a, int64_t w, int pair_own) {
  Item it;
  if (MODE == kRouted) {
    const int M = a.nu * a.P.totals[0];
    it = routed_item(a, w, upper_index(a.tile_off, M + 1, w));
  } else {
    const int HP = (MODE == kOwn) ? a.nu * a.G : a.Hq;
    const bool paired = (MODE == kDense) || pair_own;
    const int64_t per_head = paired ? a.P.totals[2] : a.P.totals[1];
    int64_t idx = w / HP;
    const int hl = (int)(w % HP);
    if (MODE == kDense) idx = per_head - 1 - idx;  // longest rows first
    int s;
    int64_t p0;
    if (paired) {
      s = upper_index(a.P.pair_off, a.L.nseq + 1, idx);
      p0 = (idx - a.P.pair_off[s]) * (int64_t)(2 * kTileM);
    } else {
      s = upper_index(a.P.qt_off, a.L.nseq + 1, idx);
      p0 = (idx - a.P.qt_off[s]) * (int64_t)kTileM;
    }
    const int64_t st = seq_start(a.L, s), len = seq_len(a.L, s);
    it.h = (MODE == kOwn) ? a.u0 * a.G + hl : hl;
    it.g = it.h / a.G;
    it.u = (MODE == kOwn) ? hl / a.G : 0;
    it.seq = s;
    it.seq_start = st;
    it.qstart = st + p0;
    it.own_block = (int)(p0 / a.B);
    const int64_t k0 = (MODE == kOwn) ? (int64_t)it.own_block * a.B : 0;
    it.kstart = st + k0;
    it.rows_x[0] = (int)min((int64_t)kTileM, len - p0);
    it.rows_x[1] = paired ? (int)max((int64_t)0, min((int64_t)kTileM, len - p0 - kTileM)) : 0;
    it.nkv_x[0] = (int)((p0 - k0) / kTileN) + 1;
    it.nkv_x[1] = it.rows_x[1] > 0 ? it.nkv_x[0] + 1 : 0;
    it.nkv = max(it.nkv_x[0], it.nkv_x[1]);
    it.e0 = 0;
  }
  return it;
}

// Row max of one 128-key score tile held in TMEM (this thread's lane),
// read 64 columns at a time.  MASK hides keys c > r (diagonal tile).
template <bool MASK>
__device__ __forceinline__ float tile_row_max(uint32_t tS, int r) {
  float mp[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) mp[e] = -INFINITY;
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2) {
    float sv[64];
    tmem_ld32(tS + h2 * 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
    tmem_ld32(tS + h2 * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
    tc_wait_ld();
    if (MASK) {
#pragma unroll
      for (int c = 0; c < 64; ++c)
        if (h2 * 64 + c > r) sv[c] = -INFINITY;
    }
#pragma unroll
    for (int c = 0; c < 64; c += 16) {
#pragma unroll
      for (int e = 0; e < 8; ++e) mp[e] = fmax3f(mp[e], sv[c + e], sv[c + 8 + e]);
    }
  }
  return fmaxf(fmax3f(mp[0], mp[1], mp[2]), fmax3f(fmax3f(mp[3], mp[4], mp[5]), mp[6], mp[7]));
}

// 2^x of score pair e of a 16-pair group: one pair in eight on the FMA
// pipe, the rest on the special-function unit, whose throughput otherwise
// bounds the softmax.  Deterministic, so a second evaluation of the same
// pair reproduces the first bit for bit.
__device__ __forceinline__ void pair_exp2(float& p0, float& p1, float s0, float s1,
                                          float scale_log2, float m_use, int e) {
  float x0, x1;
  ffma2(x0, x1, s0, s1, scale_log2, scale_log2, -m_use, -m_use);
  if ((e & 7) == 7) {
    exp2_poly2(p0, p1, x0, x1);
  } else {
    p0 = ex2_approx(x0);
    p1 = ex2_approx(x1);
  }
}

// P = 2^(s * scale_log2 - m) for one score tile, written back as packed bf16
// pairs into the tile's first 64 TMEM columns (chunk h2 of 64 scores becomes
// 32 packed columns, which never overlap scores still to be read).  Returns
// the row sum of the fp32 probabilities.  Scale-and-shift and the sums run
// as packed pairs.
//
// lo_mode (warp-uniform, diagonal tiles only) serves the first tile of a
// block, whose first rows have a handful of keys: there the 2^-9 relative
// rounding of each bf16 weight does not average out.  Rows 0..63 (lo_mode 1)
// also write the residual P - bf16(P), as bf16, into columns 64..95; their
// keys 64..127 are all masked, so the scores held there are never needed.
// Rows 64..127 (lo_mode 2) write zeros there once they have read those
// scores.  A second set of PV MMAs over columns 64..95 then gives rows 0..63
// about 16 bits of each weight.
template <bool MASK>
__device__ __forceinline__ float tile_exp_to_p(uint32_t tS, int r, float scale_log2,
                                               float m_use, uint64_t* half_bar, int lane,
                                               int lo_mode) {
  float sp[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) sp[e] = 0.f;
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2) {
    float sv[64];
    tmem_ld32(tS + h2 * 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
    tmem_ld32(tS + h2 * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
    tc_wait_ld();
    if (MASK) {
#pragma unroll
      for (int c = 0; c < 64; ++c)
        if (h2 * 64 + c > r) sv[c] = -INFINITY;
      if (h2 == 1 && lo_mode == 2) {
        uint32_t z[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) z[e] = 0u;
        tmem_st16(tS + 64, z);
        tmem_st16(tS + 80, z);
      }
    }
#pragma unroll
    for (int q2 = 0; q2 < 2; ++q2) {
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        float p0, p1;
        pair_exp2(p0, p1, sv[q2 * 32 + 2 * e], sv[q2 * 32 + 2 * e + 1], scale_log2, m_use, e);
        fadd2(sp[2 * (e & 3)], sp[2 * (e & 3) + 1], p0, p1);
        pk[e] = pack_bf16x2(p0, p1);
      }
      tmem_st16(tS + h2 * 32 + q2 * 16, pk);
      if (MASK && h2 == 0 && lo_mode == 1) {
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float p0, p1;
          pair_exp2(p0, p1, sv[q2 * 32 + 2 * e], sv[q2 * 32 + 2 * e + 1], scale_log2, m_use, e);
          const __nv_bfloat162 hi = __floats2bfloat162_rn(p0, p1);
          pk[e] = pack_bf16x2(p0 - __low2float(hi), p1 - __high2float(hi));
        }
        tmem_st16(tS + 64 + q2 * 16, pk);
      }
    }
    if (h2 == 0) {  // P of keys 0..63 is in TMEM: the first half of PV may start
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(half_bar);
    }
  }
  return ((sp[0] + sp[1]) + (sp[2] + sp[3])) + ((sp[4] + sp[5]) + (sp[6] + sp[7]));
}

// 32-byte global store (one instruction for eight 32-bit words; the address
// must be 32-byte aligned).  Used for the partials, whose workspace rows are
// 32-byte aligned: each lane writes its own row, so the store width halves
// the requests of a scattered epilogue (measured 10 % faster at 256-key
// blocks).  The caller's o is only required to be 16-byte aligned and keeps
// 16-byte stores.
__device__ __forceinline__ void st_global_v8(void* p, uint32_t a0, uint32_t a1, uint32_t a2,
                                             uint32_t a3, uint32_t a4, uint32_t a5,
                                             uint32_t a6, uint32_t a7) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a0),
               "r"(a1), "r"(a2), "r"(a3), "r"(a4), "r"(a5), "r"(a6), "r"(a7)
               : "memory");
}

template <int D, int MODE, int QBUFS>
__global__ void __launch_bounds__(352, 1)
    attn2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const AttnArgs a, int pair_own) {
  using C = Attn2Cfg<D, QBUFS>;
  static_assert(sizeof(Item) <= C::kItemBytes, "item descriptor slot too small");
  constexpr int ST = C::kStages;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sQ = smem + C::kOffQ;
  unsigned char* sKV = smem + C::kOffKV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  constexpr int QB = C::kQBufs;
  uint64_t* q_full = bars + 0;          // [QB] Q buffer loaded
  uint64_t* q_empty = bars + QB;        // [QB] Q buffer free (last S MMAs done)
  uint64_t* kv_full = bars + 2 * QB;    // [ST]
  uint64_t* kv_empty = kv_full + ST;    // [ST]
  uint64_t* s_full = kv_empty + ST;     // [2] S_X written
  uint64_t* p_full = s_full + 2;        // [2] P_X in TMEM (and O_X rescaled)
  uint64_t* o_full = p_full + 2;        // [2] last PV_X of an item done
  uint64_t* o_free = o_full + 2;        // [2] epilogue has read O_X
  uint64_t* td_bar = o_free + 2;
  uint64_t* p_half = td_bar + 1;        // [2] first 64 keys of P_X in TMEM
  uint64_t* desc_free = p_half + 2;     // [QB] every softmax warp has read the item descriptor
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(desc_free + QB);
  Item* sItem = reinterpret_cast<Item*>(smem + C::kOffItem);  // [QB], with the Q buffers
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int b = 0; b < QB; ++b) {
      mbar_init(&q_full[b], 1);
      mbar_init(&q_empty[b], 1);
      mbar_init(&desc_free[b], 8);  // one elected arrival per softmax warp
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], kTileM / 32);  // one elected arrival per softmax warp
      mbar_init(&p_half[b], kTileM / 32);
      mbar_init(&o_full[b], 1);
      mbar_init(&o_free[b], kTileM / 32);
    }
    for (int sl = 0; sl < ST; ++sl) {
      mbar_init(&kv_full[sl], 1);
      mbar_init(&kv_empty[sl], 1);
    }
    mbar_init(td_bar, 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_q);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int64_t items = num_items2<MODE>(a, pair_own);
  const int64_t first = blockIdx.x, step = gridDim.x;
  uint32_t* st = a.status;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t kv_it = 0, lt = 0;
      bool ok = true;
      for (int64_t w = first; w < items && ok; w += step, ++lt) {
        const Item it = item_info<MODE>(a, w, pair_own);
        if (MODE != kRouted) {
          const int qb = lt % QB;
          ok = mbar_wait(&q_empty[qb], ((lt / QB) & 1) ^ 1, abort_flag, st);
          if (ok) ok = mbar_wait(&desc_free[qb], ((lt / QB) & 1) ^ 1, abort_flag, st);
          if (!ok) break;
          sItem[qb] = it;  // published by the arrive below, with the Q tile
          mbar_arrive_expect_tx(&q_full[qb], C::kQBytes);
#pragma unroll
          for (int x = 0; x < 2; ++x)
#pragma unroll
            for (int hx = 0; hx < D / 64; ++hx)
              tma_load_3d(sQ + qb * C::kQBytes + x * C::kSubQBytes + hx * C::kHalfBytes, &tm_q,
                          &q_full[qb], hx * 64, it.h, (int)(it.qstart + x * kTileM));
        }
        for (int j = 0; j < it.nkv && ok; ++j) {
          const int krow = (int)(it.kstart + (int64_t)j * kTileN);
#pragma unroll
          for (int which = 0; which < 2; ++which) {
            const int sl = kv_it % ST;
            ok = mbar_wait(&kv_empty[sl], ((kv_it / ST) & 1) ^ 1, abort_flag, st);
            if (!ok) break;
            mbar_arrive_expect_tx(&kv_full[sl], C::kKVBytes);
#pragma unroll
            for (int hx = 0; hx < D / 64; ++hx)
              tma_load_3d(sKV + sl * C::kKVBytes + hx * C::kHalfBytes, which ? &tm_v : &tm_k,
                          &kv_full[sl], hx * 64, it.g, krow);
            ++kv_it;
          }
        }
      }
      if (!ok) {
        const uint32_t n = kv_it < (uint32_t)ST ? kv_it : (uint32_t)ST;
        for (uint32_t b = 0; b < n; ++b) {
          const uint32_t i2 = kv_it - 1 - b;
          mbar_wait_teardown(&kv_full[i2 % ST], (i2 / ST) & 1, 200000000ull);
        }
        if (MODE != kRouted && lt > 0) {
          for (uint32_t b = 0; b < (lt < (uint32_t)QB ? lt : (uint32_t)QB); ++b) {
            const uint32_t l = lt - 1 - b;
            mbar_wait_teardown(&q_full[l % QB], (l / QB) & 1, 200000000ull);
          }
        }
      }
    }
  } else if (warp == 10) {
    // ------------------------------------------------------------ Q gather
    // Routed items: the rows the bucket entries name, four rows per TMA
    // gather from q viewed as [T*Hq][D] (one-row boxes of 64 columns,
    // 128-B swizzle), so that the TMA engine, not this warp, carries the
    // latency of 256 scattered rows.  Lane l brings rows 4l..4l+3 of each
    // sub-tile; rows past the item's end repeat its first row (their
    // results are never stored).
    if (MODE == kRouted) {
      uint32_t lt = 0;
      bool ok = true;
      // The next item and its entries are looked up before this item's
      // gathers are issued, so that the entry loads land while the TMA
      // requests queue (a clock trace put the lookup and the entry loads at
      // 3 k cycles, the gather issue at 8-9 k, for a 256-row item).
      int f = -1;  // bucket of the item looked up last
      Item nxt;
      uint2 nent[2][4];
      auto lookup = [&](int64_t w2) {
        if (f < 0) {
          f = upper_index(a.tile_off, a.nu * a.P.totals[0] + 1, w2);
          nxt = routed_item(a, w2, f);
        } else {
          f = routed_next(a, w2, f, lane, nxt);
        }
        const int nrows = nxt.rows_x[0] + nxt.rows_x[1];
#pragma unroll
        for (int x = 0; x < 2; ++x)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            int r = x * kTileM + 4 * lane + i;
            if (r >= nrows) r = 0;
            nent[x][i] = a.entries[nxt.e0 + r];
          }
      };
      if (first < items) lookup(first);
      for (int64_t w = first; w < items && ok; w += step, ++lt) {
        const Item it = nxt;
        int ys[2][4];
#pragma unroll
        for (int x = 0; x < 2; ++x)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint2 e = nent[x][i];
            const bool good = e.x < (uint32_t)a.L.T && (e.y & 0xFFFFu) < (uint32_t)a.G;
            const int hq = it.g * a.G + (good ? (int)(e.y & 0xFFFFu) : 0);
            ys[x][i] = (int)((int64_t)(good ? e.x : 0u) * a.Hq + hq);
          }
        if (w + step < items) lookup(w + step);
        const int qb = lt % QB;
        ok = mbar_wait(&q_empty[qb], ((lt / QB) & 1) ^ 1, abort_flag, st);
        if (ok) ok = mbar_wait(&desc_free[qb], ((lt / QB) & 1) ^ 1, abort_flag, st);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        if (lane == 0) {
          sItem[qb] = it;  // published by q_full, with the rows
          mbar_arrive_expect_tx(&q_full[qb], C::kQBytes);
        }
        __syncwarp();
#pragma unroll
        for (int x = 0; x < 2; ++x)
#pragma unroll
          for (int hx = 0; hx < D / 64; ++hx)
            tma_gather4(sQ + qb * C::kQBytes + x * C::kSubQBytes + hx * C::kHalfBytes +
                            lane * 4 * 128,
                        &tm_q, &q_full[qb], hx * 64, ys[x][0], ys[x][1], ys[x][2], ys[x][3]);
        if (QB == 1 && w + step < items) {
          // one Q buffer (long items): the next item's rows can only be
          // gathered once this item's MMAs are done, so bring them into L2 now
#pragma unroll
          for (int x = 0; x < 2; ++x)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint2 e = nent[x][i];
              const bool good = e.x < (uint32_t)a.L.T && (e.y & 0xFFFFu) < (uint32_t)a.G;
              const int hq = nxt.g * a.G + (good ? (int)(e.y & 0xFFFFu) : 0);
              ys[x][i] = (int)((int64_t)(good ? e.x : 0u) * a.Hq + hq);
            }
#pragma unroll
          for (int x = 0; x < 2; ++x)
#pragma unroll
            for (int hx = 0; hx < D / 64; ++hx)
              tma_prefetch_gather4(&tm_q, hx * 64, ys[x][0], ys[x][1], ys[x][2], ys[x][3]);
        }
      }
      if (!ok && lane == 0) {  // let the gathers in flight land before the CTA exits
        for (uint32_t b = 0; b < (lt < (uint32_t)QB ? lt : (uint32_t)QB); ++b) {
          const uint32_t l = lt - 1 - b;
          mbar_wait_teardown(&q_full[l % QB], (l / QB) & 1, 200000000ull);
        }
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop in lock-step (all values warp-uniform);
    // each tcgen05 instruction is issued by one elected lane.
    uint32_t kv_it = 0, lt = 0;
    uint32_t ns0 = 0, ns1 = 0;  // S MMAs issued per sub-tile (p_full phases follow)
    uint32_t no0 = 0, no1 = 0;  // items per sub-tile (o_full / o_free phases)
    bool ok = true;
    const uint32_t sQa = smem_u32(sQ), sKVa = smem_u32(sKV);
    auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      const bool r = mbar_wait(bar, parity, abort_flag, st);
      return __all_sync(0xffffffffu, r);
    };
    auto issue_s = [&](int x, uint32_t qbase, uint32_t ks) {
      const uint32_t kbase = sKVa + ks * C::kKVBytes;
      const uint32_t qx = qbase + x * C::kSubQBytes;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * C::kHalfBytes + (kk & 3) * 32;
        tc_mma_ss_warp(tmem + C::col_s(x), sdesc_kmajor_sw128(qx + off),
                       sdesc_kmajor_sw128(kbase + off), C::kIdescS, kk > 0 ? 1u : 0u);
      }
      tc_commit_warp(&s_full[x]);
      if (x == 0) ++ns0; else ++ns1;
    };
    auto issue_pv = [&](int x, uint32_t vs, bool acc, int kk0, int kk1) {
      const uint32_t vbase = sKVa + vs * C::kKVBytes;
#pragma unroll
      for (int kk = kk0; kk < kk1; ++kk)
        tc_mma_ts_warp(tmem + C::col_o(x), tmem + C::col_s(x) + kk * 8,
                       sdesc_mnmajor_sw128(vbase + kk * 2048, C::kHalfBytes, 1024), C::kIdescPV,
                       (acc || kk > 0) ? 1u : 0u);
    };
    // K_{j+1}: its slot and ring position are assigned in order when step j
    // starts.  With two Q buffers (a three-slot ring) the wait happens only
    // before the first S MMA that reads it, so PV_0(j) never waits on the
    // next K tile's load (that load starts only when PV(j-1) frees a slot).
    // With the deep ring the wait comes first, where it overlaps the wait
    // for the softmax (measured: 4 % faster at 4096-key blocks).
    constexpr bool kLateK = (QBUFS == 2);
    uint32_t k_pos = 0;
    bool k_pending = false;
    auto ensure_k = [&]() -> bool {
      if (!k_pending) return true;
      k_pending = false;
      return wait(&kv_full[k_pos % ST], (k_pos / ST) & 1);
    };
    // one sub-tile's share of KV step j: PV_X(j), then S_X(j+1)
    auto kv_step = [&](int x, const Item& it, int j, uint32_t vs, uint32_t ks2, uint32_t qbase) {
      if (j >= it.nkv_x[x]) return true;
      const uint32_t nsx = x == 0 ? ns0 : ns1;
      const uint32_t nox = x == 0 ? no0 : no1;
      if (!wait(&p_half[x], (nsx - 1) & 1)) return false;  // keys 0..63 of P_X(j)
      if (j == 0 && nox > 0 && !wait(&o_free[x], (nox - 1) & 1)) return false;
      tc_fence_after();
      issue_pv(x, vs, j > 0, 0, kTileN / 32);
      if (!wait(&p_full[x], (nsx - 1) & 1)) return false;  // all of P_X(j)
      tc_fence_after();
      issue_pv(x, vs, true, kTileN / 32, kTileN / 16);
      if (MODE != kRouted && it.nkv_x[x] == 1) {
        // residual weights of keys 0..63 in columns 64..95 (first tile of a block)
        const uint32_t vbase = sKVa + vs * C::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < kTileN / 32; ++kk)
          tc_mma_ts_warp(tmem + C::col_o(x), tmem + C::col_s(x) + 64 + kk * 8,
                         sdesc_mnmajor_sw128(vbase + kk * 2048, C::kHalfBytes, 1024), C::kIdescPV,
                         1u);
      }
      if (j == it.nkv_x[x] - 1) {
        tc_commit_warp(&o_full[x]);
        if (x == 0) ++no0; else ++no1;
      }
      if (j + 1 < it.nkv_x[x]) {
        if (!ensure_k()) return false;
        tc_fence_after();
        issue_s(x, qbase, ks2);
      }
      return true;
    };
    for (int64_t w = first; w < items && ok; w += step, ++lt) {
      const int qb = lt % QB;
      const uint32_t qbase = sQa + qb * C::kQBytes;
      if (!(ok = wait(&q_full[qb], (lt / QB) & 1))) break;
      const Item it = sItem[qb];  // written by the Q buffer's filler
      const uint32_t ks = kv_it % ST;
      if (!(ok = wait(&kv_full[ks], (kv_it / ST) & 1))) break;
      ++kv_it;
      tc_fence_after();
      if (it.nkv_x[0] > 0) issue_s(0, qbase, ks);
      if (it.nkv_x[1] > 0) issue_s(1, qbase, ks);
      tc_commit_warp(&kv_empty[ks]);
      // The Q buffer is free once the item's last S MMAs complete, before
      // its last PV MMAs: the next item's rows start loading that much
      // earlier (the commit covers every MMA issued so far).
      if (it.nkv == 1) tc_commit_warp(&q_empty[qb]);
      for (int j = 0; j < it.nkv && ok; ++j) {
        const uint32_t vs = kv_it % ST;
        if (!(ok = wait(&kv_full[vs], (kv_it / ST) & 1))) break;
        ++kv_it;
        const bool more = (j + 1 < it.nkv);
        uint32_t ks2 = 0;
        if (more) {
          ks2 = kv_it % ST;
          k_pos = kv_it;
          k_pending = true;
          ++kv_it;
          if (!kLateK && !(ok = ensure_k())) break;
        }
        if (!(ok = kv_step(0, it, j, vs, ks2, qbase))) break;
        if (!(ok = kv_step(1, it, j, vs, ks2, qbase))) break;
        if (j == it.nkv - 2) tc_commit_warp(&q_empty[qb]);  // every S of the item issued
        // a slot is released only after its load has been waited for
        if (!(ok = ensure_k())) break;
        tc_commit_warp(&kv_empty[vs]);
        if (more) tc_commit_warp(&kv_empty[ks2]);
      }
    }
    tc_commit_warp(td_bar);
    mbar_wait_teardown(td_bar, 0, 500000000ull);
  } else {
    // ------------------------------------------------------------ softmax (warps 0-7)
    const int x = warp >> 2;               // sub-tile
    const int r = threadIdx.x & 127;       // row = TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::col_s(x);
    const uint32_t tO = tmem + lane_off + C::col_o(x);
    // routed partials are stored times 2^-S (see partial_scale_log2)
    const float pscale = (MODE == kRouted) ? exp2f(-(float)partial_scale_log2(a.status[1])) : 1.f;
    uint32_t ns = 0, no = 0;
    bool ok = true;
    // The item comes from its descriptor in shared memory, published with
    // the Q buffer (a clock trace put the global-memory decode at 3-5 k
    // cycles per item here, twice per item); the fields the epilogue needs
    // are kept in registers, since the descriptor's slot is refilled once
    // every softmax warp has read it.
    uint32_t lt = 0;
    for (int64_t w = first; w < items && ok; w += step, ++lt) {
      const int qb = lt % QB;
      ok = mbar_wait(&q_full[qb], (lt / QB) & 1, abort_flag, st);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      const int nkv = sItem[qb].nkv_x[x];
      const int rows_x = sItem[qb].rows_x[x];
      const int it_u = sItem[qb].u, it_h = sItem[qb].h, it_seq = sItem[qb].seq;
      const int it_own = sItem[qb].own_block;
      const int64_t it_e0 = sItem[qb].e0, it_q0 = sItem[qb].qstart;
      const int64_t it_s0 = sItem[qb].seq_start;
      __syncwarp();
      if (lane == 0) mbar_arrive(&desc_free[qb]);
      if (nkv == 0) continue;
      // routed: this row's bucket entry, loaded now so that its latency
      // hides behind the softmax instead of opening the epilogue
      uint2 ent = make_uint2(0xFFFFFFFFu, 0u);
      if (MODE == kRouted && r < rows_x) ent = a.entries[it_e0 + x * kTileM + r];
      float m_run = -INFINITY, l_run = 0.f;
      for (int j = 0; j < nkv; ++j) {
        ok = mbar_wait(&s_full[x], ns & 1, abort_flag, st);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        // diagonal tile (own/dense): key c of the tile is visible to row r
        // only when c <= r, since the tile starts at the sub-tile's first row
        const bool diag_tile = (MODE != kRouted) && (j == nkv - 1);
        const float mx = diag_tile ? tile_row_max<true>(tS, r) : tile_row_max<false>(tS, r);
        const float m_new = fmaxf(m_run, mx * a.scale_log2);
        const bool need = (j == 0) || (m_new > m_run + 8.0f);
        const float m_use = need ? m_new : m_run;
        const float alpha = (j == 0) ? 0.f : (need ? ex2_approx(m_run - m_use) : 1.f);
        // O_X rescale: PV_X(j-1) finished before S_X(j), which we have seen
        if (__any_sync(0xffffffffu, j > 0 && need)) {
          const float f = (j > 0 && need) ? alpha : 1.f;
#pragma unroll
          for (int c4 = 0; c4 < D / 32; ++c4) {
            uint32_t ov[32];
            tmem_ld32(tO + c4 * 32, ov);
            tc_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f);
            tmem_st32(tO + c4 * 32, ov);
          }
        }
        // first tile of a block: residual weights for rows 0..63 (see tile_exp_to_p)
        const int lo_mode = (diag_tile && nkv == 1) ? ((warp & 3) < 2 ? 1 : 2) : 0;
        const float sum =
            diag_tile ? tile_exp_to_p<true>(tS, r, a.scale_log2, m_use, &p_half[x], lane, lo_mode)
                      : tile_exp_to_p<false>(tS, r, a.scale_log2, m_use, &p_half[x], lane, 0);
        l_run = l_run * alpha + sum;
        m_run = m_use;
        tc_wait_st();
        tc_fence_before();
        __syncwarp();  // the warp's TMEM stores are ordered before lane 0's arrival
        if (lane == 0) mbar_arrive(&p_full[x]);
        ++ns;
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      ok = mbar_wait(&o_full[x], no & 1, abort_flag, st);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const bool valid = r < rows_x;
      const float inv = 1.f / l_run;
      const float lse2 = m_run + lg2_approx(l_run);
      // destination of this row
      int kind = 0;  // 0 skip, 1 fp16 partial, 2 fp32 partial, 3 final (bf16)
      __nv_bfloat16* dst16 = nullptr;
      __half* dsth = nullptr;
      float* dst32 = nullptr;
      float* lse_dst = nullptr;
      float lse_val = lse2;
      if (valid) {
        if (MODE == kRouted) {
          const uint2 e = ent;
          const int hh = (int)(e.y & 0xFFFFu), sl = (int)(e.y >> 16);
          if (e.x < (uint32_t)a.L.T && hh < a.G && sl < a.topk - 1) {
            const int64_t prow =
                (((int64_t)it_u * a.L.T + e.x) * a.G + hh) * (a.topk - 1) + sl;
            kind = 1;
            dsth = a.part_O + prow * D;
            lse_dst = a.part_lse + prow;
          } else {
            atomicOr(a.status, MOBA_DEV_BAD_INDEX);
          }
        } else {
          const int64_t t = it_q0 + (int64_t)x * kTileM + r;
          const bool final_row = (MODE == kDense) || a.topk == 1 || it_own == 0;
          if (final_row) {
            kind = 3;
            dst16 = a.o + ((size_t)t * a.Hq + it_h) * D;
            lse_dst = a.lse + row_index(a.R, it_seq, it_h, t - it_s0, t);
            lse_val = lse2 * 0.6931471805599453f;
          } else {
            const int64_t prow = ((int64_t)it_u * a.L.T + t) * a.G + (it_h % a.G);
            kind = 2;
            dst32 = a.own_O + prow * D;
            lse_dst = a.own_lse + prow;
          }
        }
      }
#pragma unroll
      for (int c4 = 0; c4 < D / 32; ++c4) {
        uint32_t ov[32];
        tmem_ld32(tO + c4 * 32, ov);
        tc_wait_ld();
        if (kind == 3) {
          uint4* d4 = reinterpret_cast<uint4*>(dst16 + c4 * 32);
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            const float* f = reinterpret_cast<const float*>(&ov[q8 * 8]);
            d4[q8] = make_uint4(pack_bf16x2(f[0] * inv, f[1] * inv),
                                pack_bf16x2(f[2] * inv, f[3] * inv),
                                pack_bf16x2(f[4] * inv, f[5] * inv),
                                pack_bf16x2(f[6] * inv, f[7] * inv));
          }
        } else if (kind == 1) {
          // Routed partial O in fp16: a convex combination of V rows, so
          // |O| <= max |v|; 8x finer than bf16, for the second rounding
          // the merge adds before the final bf16 output.  Scaled by 2^-S,
          // which keeps it below the fp16 maximum whatever the bf16 input.
          const float ps = inv * pscale;
#pragma unroll
          for (int q16 = 0; q16 < 2; ++q16) {
            const float* f = reinterpret_cast<const float*>(&ov[q16 * 16]);
            st_global_v8(dsth + c4 * 32 + q16 * 16, pack_half2(f[0] * ps, f[1] * ps),
                         pack_half2(f[2] * ps, f[3] * ps), pack_half2(f[4] * ps, f[5] * ps),
                         pack_half2(f[6] * ps, f[7] * ps), pack_half2(f[8] * ps, f[9] * ps),
                         pack_half2(f[10] * ps, f[11] * ps), pack_half2(f[12] * ps, f[13] * ps),
                         pack_half2(f[14] * ps, f[15] * ps));
          }
        } else if (kind == 2) {
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            const uint32_t* u = &ov[8 * q8];
            st_global_v8(dst32 + c4 * 32 + q8 * 8,
                         __float_as_uint(__uint_as_float(u[0]) * inv),
                         __float_as_uint(__uint_as_float(u[1]) * inv),
                         __float_as_uint(__uint_as_float(u[2]) * inv),
                         __float_as_uint(__uint_as_float(u[3]) * inv),
                         __float_as_uint(__uint_as_float(u[4]) * inv),
                         __float_as_uint(__uint_as_float(u[5]) * inv),
                         __float_as_uint(__uint_as_float(u[6]) * inv),
                         __float_as_uint(__uint_as_float(u[7]) * inv));
          }
        }
      }
      if (kind != 0) *lse_dst = lse_val;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_free[x]);
      ++no;
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

}  // namespace moba
