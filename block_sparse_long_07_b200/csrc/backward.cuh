// backward.cuh -- gradients of the MoBA attention over a fixed selection.
//
// No gradient passes through the hard top-k gate (wispaper.ai blog, "The
// Change": the gradient does not flow through the discrete selection), so
// the backward is that of exact softmax attention over each row's key set
// I: with P_u = exp(scale q.k_u - lse) (the forward's lse), D = dO . O,
//   dS_u = P_u (dO . v_u - D)
//   dQ    = scale sum_u dS_u k_u,  dK_u += scale dS_u q,  dV_u += P_u dO.
//
// Work is organised like the forward.  For the routed part, the rows that
// chose past block J (the forward's bucket of (kv head, J), gathered rows)
// meet J's keys; for the own part, each block's rows meet the same block's
// keys, causally.  Two kernels per part, each recomputing S and P:
//   bw_kv2_kernel one CTA per (bucket or own block, 128-key tile), warp
//                 roles: it loops over the rows in tiles of 64; S^T = K Q^T and
//                 dP^T = V dO^T (keys on the TMEM lanes, two tiles' worth of
//                 TMEM), P^T and dS^T packed as bf16 over them, which are the
//                 TMEM A operands of dV += P^T dO and dK += dS^T Q, accumulated
//                 in TMEM; the elementwise pass of a tile overlaps the MMAs
//                 of its neighbours
//   bw_q2_kernel  one CTA per tile of 128 rows (gathered or own), warp
//                 roles: walks the block's key tiles in halves of 64 keys; dS
//                 packed as bf16 into TMEM is the A operand of dQ += dS K
// The Q / dO tiles ([rows][d], 128-byte swizzled) serve both as K-major
// operands (S, dP and their transposes) and as MN-major B operands (dK, dV);
// K / V tiles likewise.
// Gradients are summed in fp32 buffers with atomic adds (each key gets one
// routed and one own contribution per kv head; each row one per chosen
// block) and converted to bf16 at the end.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"
#include "layout.cuh"

namespace moba {

enum { kBwRouted = 0, kBwOwn = 1 };

struct BwArgs {
  const __nv_bfloat16* q;   // [T][Hq][D]
  const __nv_bfloat16* dO;  // [T][Hq][D]
  const float2* dl;         // [T][Hq]: (D = dO . O, lse in log2 units)
  float* dq32;              // [T][Hq][D]
  float* dk32;              // [T][Hkv][D]
  float* dv32;              // [T][Hkv][D]
  const int32_t* entry_off; // routed: per (unit, block) bucket, as the forward
  const int32_t* tile_off;  //         128-row items
  const uint2* entries;
  int Hq, Hkv, G, B, u0, nu, NBmax;
  float scale_log2, scale;
  SeqLayout L;
  Plan P;
  uint32_t* status;
};

template <int D>
struct BwCfg {
  static constexpr int kHalf = kTileM * 128;    // 128 rows x 64 columns bf16
  static constexpr int kTile = kTileM * D * 2;  // one [128][D] bf16 tile
};

// (D = dO . O, lse * log2 e) per (token, q head), one warp per row.
template <int D>
__global__ void __launch_bounds__(256) bw_prep_kernel(const __nv_bfloat16* __restrict__ o,
                                                      const __nv_bfloat16* __restrict__ dO,
                                                      const float* __restrict__ lse, int Hq,
                                                      SeqLayout L, RowLayout R,
                                                      float2* __restrict__ dl) {
  constexpr int EPL = D / 32;
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);  // t * Hq + h
  const int lane = threadIdx.x & 31;
  if (row >= L.T * Hq) return;
  const int64_t t = row / Hq;
  const int h = (int)(row % Hq);
  float acc = 0.f;
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    const size_t idx = (size_t)row * D + lane * EPL + e;
    acc = fmaf(__bfloat162float(o[idx]), __bfloat162float(dO[idx]), acc);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) {
    const int s = seq_of_token(L, t);
    const float l = lse[row_index(R, s, h, t - seq_start(L, s), t)];
    dl[row] = make_float2(acc, l * 1.4426950408889634f);
  }
}

// One thread per row of a 128-row tile: the row's (token, q head) or -1.
struct BwRow {
  int64_t t;
  int h;
};

// Rows of tile `tile` of a CTA's work: routed -> entries[e0 + ...]; own ->
// contiguous tokens of a block for one head.
__device__ __forceinline__ BwRow bw_row_routed(const BwArgs& a, int g, int64_t e0, int64_t e1,
                                               int r) {
  BwRow x{-1, 0};
  if (e0 + r < e1) {
    const uint2 e = a.entries[e0 + r];
    const int hh = (int)(e.y & 0xFFFFu);
    if (e.x < (uint32_t)a.L.T && hh < a.G) {
      x.t = e.x;
      x.h = g * a.G + hh;
    } else {
      atomicOr(a.status, MOBA_DEV_BAD_INDEX);
    }
  }
  return x;
}

// Copy half hg (columns hg * D / 2 .. + D / 2) of row r's q and dO into the
// tiles (128-byte swizzled halves of 64 columns); two threads share a row.
// A row with t < 0 copies token 0's data (finite; its P and dS are forced to
// zero).
template <int D>
__device__ __forceinline__ void bw_load_row(const BwArgs& a, BwRow x, int r, int hg,
                                            unsigned char* sQ, unsigned char* sDO) {
  using C = BwCfg<D>;
  const int64_t t = x.t < 0 ? 0 : x.t;
  const __nv_bfloat16* qs = a.q + ((size_t)t * a.Hq + x.h) * D;
  const __nv_bfloat16* gs = a.dO + ((size_t)t * a.Hq + x.h) * D;
#pragma unroll
  for (int c = hg * (D / 16); c < (hg + 1) * (D / 16); ++c) {
    const uint32_t off = (uint32_t)(c >> 3) * C::kHalf + sw128_offset(r, c & 7);
    cp_async_16(sQ + off, qs + c * 8);
    cp_async_16(sDO + off, gs + c * 8);
  }
}

// ---------------------------------------------------------------- dK / dV, warp-specialised
// One CTA per (bucket or own block, 128-key tile), with the
// rows in 64-row tiles so that TMEM holds two tiles' S^T / dP^T next to the
// dV / dK accumulators: the elementwise pass of tile n runs while the tensor
// core computes dV / dK of tile n - 1 and S^T / dP^T of tile n + 1.
//   warps 0-7  elementwise: warp w takes keys 32 (w % 4) .. + 31 (its TMEM lane
//              quarter) and rows 32 (w / 4) .. + 31 of the tile; forms P^T and
//              dS^T = P^T (dP^T - D) and packs them as bf16 over the columns it
//              read (rows 2j, 2j + 1 -> column j of its half)
//   warp  8    TMEM allocation, the K / V load and the MMA issue
//   warps 9-10 row gather (q, dO and (D, lse2) of 32 rows each) into a
//              three-stage ring, two tiles in flight
// MMA order: S^T(n), dP^T(n) [buffer n % 2], then dV / dK(n - 1) once its P^T /
// dS^T are packed.  S^T(n + 2) reuses buffer n % 2; it is issued after dV /
// dK(n), the last reader of the packed values there, and tensor-core
// operations from one thread complete in issue order.
template <int D>
struct BwKv2Cfg {
  static constexpr int kRows = 64;                   // rows per tile
  static constexpr int kStages = 3;                  // row-tile ring
  static constexpr int kKVTile = kTileN * D * 2;     // one 128-key K or V tile
  static constexpr int kKVHalf = kTileN * 128;       // 128 rows x 64 columns bf16
  static constexpr int kRowTile = kRows * D * 2;     // one 64-row q or dO tile
  static constexpr int kRowHalf = kRows * 128;       // 64 rows x 64 columns bf16
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kKVTile;
  static constexpr int kOffQ = kOffV + kKVTile;               // [stage]
  static constexpr int kOffDO = kOffQ + kStages * kRowTile;   // [stage]
  static constexpr int kOffDL = kOffDO + kStages * kRowTile;  // [stage][64] (D, lse2)
  static constexpr int kOffBar = kOffDL + kStages * kRows * 8;
  static constexpr int kNumBars = 1 + 2 * kStages + 2 + 2 + 1;
  static constexpr int kSmemBytes = kOffBar + kNumBars * 8 + 16 + 1024;
  static constexpr int kThreads = 352;
  static constexpr uint32_t kColS = 0;         // [2] x 64 columns: S^T, then packed P^T
  static constexpr uint32_t kColDP = 128;      // [2] x 64 columns: dP^T, then packed dS^T
  static constexpr uint32_t kColV = 256;       // dV accumulator
  static constexpr uint32_t kColK = 256 + D;   // dK accumulator
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kSmemBytes <= 232448, "bw_kv2 shared memory beyond the per-CTA limit");
};

// Packed column of the A operand for rows 16 kk .. 16 kk + 15 of a tile:
// rows 0..31 pack into columns 0..15, rows 32..63 into 32..47.
__host__ __device__ constexpr uint32_t bw2_packed_col(int kk) {
  return kk < 2 ? 8u * kk : 16u + 8u * kk;
}

template <int D, int MODE>
__global__ void __launch_bounds__(352, 1)
    bw_kv2_kernel(const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const BwArgs a) {
  using C = BwKv2Cfg<D>;
  constexpr int ST = C::kStages;
  constexpr int RT = C::kRows;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* kv_bar = bars;               // K / V landed
  uint64_t* rows_full = bars + 1;        // [ST] a row tile gathered
  uint64_t* rows_empty = rows_full + ST; // [ST] its dV / dK MMAs done
  uint64_t* s_full = rows_empty + ST;    // [2] S^T / dP^T of a tile in TMEM
  uint64_t* p_full = s_full + 2;         // [2] P^T / dS^T packed
  uint64_t* done_bar = p_full + 2;       // every MMA done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int NB = a.P.totals[0];
  const int KT = a.B / kTileN;
  const int64_t f = blockIdx.x / KT;
  const int kt = (int)(blockIdx.x % KT);
  if (f >= (int64_t)a.nu * NB) return;
  const int u = (int)(f / NB), J = (int)(f % NB);
  const int g = a.u0 + u;
  const int blen = a.P.blk_len[J];
  const int nkeys = min(kTileN, blen - kt * kTileN);
  if (nkeys <= 0) return;
  const int64_t kstart = (int64_t)a.P.blk_tok[J] + (int64_t)kt * kTileN;
  const int64_t bend = (int64_t)a.P.blk_tok[J] + blen;
  int64_t e0 = 0, e1 = 0;
  int ntiles, own_tiles = 0;
  if (MODE == kBwRouted) {
    e0 = a.entry_off[f];
    e1 = a.entry_off[f + 1];
    ntiles = (int)((e1 - e0 + RT - 1) / RT);
  } else {
    own_tiles = (int)((bend - kstart + RT - 1) / RT);  // row tiles from the key tile on
    ntiles = own_tiles * a.G;
  }
  if (ntiles == 0) return;

  if (threadIdx.x == 0) {
    mbar_init(kv_bar, 1);
    for (int q = 0; q < ST; ++q) {
      mbar_init(&rows_full[q], 2);
      mbar_init(&rows_empty[q], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 8);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 8) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  uint32_t* st = a.status;
  unsigned char* sK = smem + C::kOffK;
  unsigned char* sV = smem + C::kOffV;
  float2* sdl = reinterpret_cast<float2*>(smem + C::kOffDL);

  if (warp >= 9) {
    // ------------------------------------------------------------ row gather
    // Warp gw gathers rows 32 gw .. 32 gw + 31 of each tile.  Lane l reads the
    // entry of row 32 gw + l (one tile ahead); the copies then take RPI rows
    // per instruction, CPR consecutive 16-byte chunks of a row per group of
    // lanes, so one instruction reads a few contiguous rows instead of 32
    // scattered pieces.
    constexpr int CPR = D / 8;     // 16-byte chunks per row
    constexpr int RPI = 32 / CPR;  // rows per instruction
    const int rbase = (warp - 9) * 32;
    auto row_of = [&](int n) -> BwRow {
      BwRow x{-1, 0};
      if (n >= ntiles) return x;
      const int r = rbase + lane;
      if (MODE == kBwRouted) {
        x = bw_row_routed(a, g, e0 + (int64_t)n * RT, e1, r);
      } else {
        const int hh = n / own_tiles;
        const int64_t t = kstart + (int64_t)(n % own_tiles) * RT + r;
        if (t < bend) {
          x.t = t;
          x.h = g * a.G + hh;
        }
      }
      return x;
    };
    bool ok = true;
    int n = 0;
    BwRow xn = row_of(0);
    for (; n < ntiles && ok; ++n) {
      const int sg = n % ST;
      ok = __all_sync(0xffffffffu,
                      mbar_wait(&rows_empty[sg], ((n / ST) & 1) ^ 1, abort_flag, st));
      if (!ok) break;
      const BwRow x = xn;
      xn = row_of(n + 1);  // next tile's entry, in flight while this one copies
      // a missing row reads token 0, head 0 (finite); its P is forced to 0
      const int64_t my_t = x.t < 0 ? 0 : x.t;
      const int my_h = x.t < 0 ? 0 : x.h;
      unsigned char* dq_ = smem + C::kOffQ + sg * C::kRowTile;
      unsigned char* ddo = smem + C::kOffDO + sg * C::kRowTile;
      const int c = lane % CPR;
#pragma unroll
      for (int i = 0; i < 32 / RPI; ++i) {
        const int rl = i * RPI + lane / CPR;  // row within this warp's 32
        const int64_t t = __shfl_sync(0xffffffffu, my_t, rl);
        const int h = __shfl_sync(0xffffffffu, my_h, rl);
        const size_t src = ((size_t)t * a.Hq + h) * D + c * 8;
        const uint32_t off = (uint32_t)(c >> 3) * C::kRowHalf + sw128_offset(rbase + rl, c & 7);
        cp_async_16(dq_ + off, a.q + src);
        cp_async_16(ddo + off, a.dO + src);
      }
      float2* d = sdl + sg * RT + rbase + lane;
      if (x.t >= 0)
        cp_async_8(d, a.dl + (size_t)x.t * a.Hq + x.h);
      else
        *d = make_float2(0.f, __int_as_float(0x7f800000));
      cp_async_commit();
      if (n > 0) {  // tile n - 1 landed: publish it (two tiles in flight)
        cp_async_wait_group<1>();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&rows_full[(n - 1) % ST]);
      }
    }
    cp_async_wait_all();
    if (ok && n > 0) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&rows_full[(n - 1) % ST]);
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ K / V load, MMA issue
    if (lane == 0) {
      mbar_arrive_expect_tx(kv_bar, 2 * C::kKVTile);
#pragma unroll
      for (int hx = 0; hx < D / 64; ++hx) {
        tma_load_3d(sK + hx * C::kKVHalf, &tm_k, kv_bar, hx * 64, g, (int)kstart);
        tma_load_3d(sV + hx * C::kKVHalf, &tm_v, kv_bar, hx * 64, g, (int)kstart);
      }
    }
    __syncwarp();
    auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, st));
    };
    constexpr uint32_t idS = idesc_bf16_f32(kTileN, RT, false, false);  // M = keys, N = rows
    constexpr uint32_t idG = idesc_bf16_f32(kTileN, D, false, true);    // A in TMEM, B MN-major
    const uint32_t sKa = smem_u32(sK), sVa = smem_u32(sV);
    const uint32_t sQa = smem_u32(smem + C::kOffQ), sDOa = smem_u32(smem + C::kOffDO);
    bool ok = wait(kv_bar, 0);
    // dV / dK of tile m (its P^T / dS^T packed in buffer m % 2)
    auto grad_mmas = [&](int m) -> bool {
      const int b = m & 1, sg = m % ST;
      if (!wait(&p_full[b], (m >> 1) & 1)) return false;
      tc_fence_after();
      const uint32_t qb = sQa + sg * C::kRowTile, ob = sDOa + sg * C::kRowTile;
#pragma unroll
      for (int kk = 0; kk < RT / 16; ++kk) {  // K = rows, 16 per step
        const uint32_t acc = (m > 0 || kk > 0) ? 1u : 0u;
        tc_mma_ts_warp(tmem + C::kColV, tmem + C::kColS + 64u * b + bw2_packed_col(kk),
                       sdesc_mnmajor_sw128(ob + kk * 2048, C::kRowHalf, 1024), idG, acc);
        tc_mma_ts_warp(tmem + C::kColK, tmem + C::kColDP + 64u * b + bw2_packed_col(kk),
                       sdesc_mnmajor_sw128(qb + kk * 2048, C::kRowHalf, 1024), idG, acc);
      }
      tc_commit_warp(&rows_empty[sg]);
      return true;
    };
    int n = 0;
    for (; n < ntiles && ok; ++n) {
      const int b = n & 1, sg = n % ST;
      if (!(ok = wait(&rows_full[sg], (n / ST) & 1))) break;
      tc_fence_after();
      const uint32_t qb = sQa + sg * C::kRowTile, ob = sDOa + sg * C::kRowTile;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t koff = (kk >> 2) * C::kKVHalf + (kk & 3) * 32;
        const uint32_t roff = (kk >> 2) * C::kRowHalf + (kk & 3) * 32;
        tc_mma_ss_warp(tmem + C::kColS + 64u * b, sdesc_kmajor_sw128(sKa + koff),
                       sdesc_kmajor_sw128(qb + roff), idS, kk > 0 ? 1u : 0u);
        tc_mma_ss_warp(tmem + C::kColDP + 64u * b, sdesc_kmajor_sw128(sVa + koff),
                       sdesc_kmajor_sw128(ob + roff), idS, kk > 0 ? 1u : 0u);
      }
      tc_commit_warp(&s_full[b]);
      if (n > 0 && !(ok = grad_mmas(n - 1))) break;
    }
    if (ok && n > 0) ok = grad_mmas(n - 1);
    tc_commit_warp(done_bar);  // every MMA of this CTA (also after an abort)
  } else {
    // ------------------------------------------------------------ elementwise (warps 0-7)
    const int quad = warp & 3, hc = warp >> 2;
    const int key = quad * 32 + lane;  // TMEM lane
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const bool key_ok = key < nkeys;
    const int64_t key_tok = kstart + key;
    bool ok = true;
    for (int n = 0; n < ntiles && ok; ++n) {
      const int b = n & 1, sg = n % ST;
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[b], (n >> 1) & 1, abort_flag, st));
      if (!ok) break;
      // the tile's (D, lse2) were published with its rows
      ok = __all_sync(0xffffffffu, mbar_wait(&rows_full[sg], (n / ST) & 1, abort_flag, st));
      if (!ok) break;
      tc_fence_after();
      const int c0 = 32 * hc;
      const uint32_t tS = tmem + lane_off + C::kColS + 64u * b;
      const uint32_t tDP = tmem + lane_off + C::kColDP + 64u * b;
      uint32_t sv[32], dv[32];
      tmem_ld32(tS + c0, sv);
      tmem_ld32(tDP + c0, dv);
      tc_wait_ld();
      int64_t row_tok0 = 0;
      if (MODE == kBwOwn) row_tok0 = kstart + (int64_t)(n % own_tiles) * RT + c0;
      const float2* dl = sdl + sg * RT + c0;
      uint32_t pp[16], dd[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float4 l = *reinterpret_cast<const float4*>(dl + 2 * e);  // (D, lse2) of 2 rows
        float p2[2], d2[2];
#pragma unroll
        for (int xx = 0; xx < 2; ++xx) {
          bool keep = key_ok;
          if (MODE == kBwOwn) keep = keep && (key_tok <= row_tok0 + 2 * e + xx);
          const float Dc = xx ? l.z : l.x, lc = xx ? l.w : l.y;
          const float p =
              keep ? ex2_approx(fmaf(__uint_as_float(sv[2 * e + xx]), a.scale_log2, -lc)) : 0.f;
          p2[xx] = p;
          d2[xx] = p * (__uint_as_float(dv[2 * e + xx]) - Dc);
        }
        pp[e] = pack_bf16x2(p2[0], p2[1]);
        dd[e] = pack_bf16x2(d2[0], d2[1]);
      }
      // rows c0 .. c0 + 31 pack into columns c0 / 2 * ... see bw2_packed_col
      const uint32_t pc = hc ? 32u : 0u;
      tmem_st16(tS + pc, pp);
      tmem_st16(tDP + pc, dd);
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[b]);
    }
    // every MMA done: add the accumulators (row = key, columns of half hc)
    const bool done = __all_sync(0xffffffffu, mbar_wait(done_bar, 0, abort_flag, st));
    if (ok && done) {
      tc_fence_after();
      float* dvp = a.dv32 + ((size_t)key_tok * a.Hkv + g) * D;
      float* dkp = a.dk32 + ((size_t)key_tok * a.Hkv + g) * D;
#pragma unroll 1
      for (int cc = hc * (D / 2); cc < (hc + 1) * (D / 2); cc += 32) {
        uint32_t va[32], vb[32];
        tmem_ld32(tmem + lane_off + C::kColV + cc, va);
        tmem_ld32(tmem + lane_off + C::kColK + cc, vb);
        tc_wait_ld();
        if (key_ok) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            atomicAdd(dvp + cc + e, __uint_as_float(va[e]));
            atomicAdd(dkp + cc + e, __uint_as_float(vb[e]) * a.scale);
          }
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  // after an abort: every MMA was committed to done_bar by the MMA warp, and
  // the K / V load may still be in flight; wait for both (bounded)
  if (threadIdx.x == 0) {
    mbar_wait_teardown(done_bar, 0, 500000000ull);
    mbar_wait_teardown(kv_bar, 0, 200000000ull);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ---------------------------------------------------------------- dQ, warp-specialised
// One CTA per 128-row tile, with each 128-key K / V tile taken
// in two halves of 64 keys so that TMEM holds two halves' S / dP next to the
// dQ accumulator: the elementwise pass of half m runs while the tensor core
// computes dQ of half m - 1 and S / dP of half m + 1.
//   warps 0-7  gather the tile's q / dO rows (two threads a row), then the
//              elementwise pass: warp w takes rows 32 (w % 4) .. + 31 (its TMEM
//              lane quarter) and keys 32 (w / 4) .. + 31 of the half; dS is
//              packed as bf16 over the S columns it read (see bw2_packed_col)
//   warp  8    TMEM allocation and the MMA issue
//   warp  9    K / V tiles by TMA into a two-stage ring
template <int D>
struct BwQ2Cfg {
  static constexpr int kStages = 2;
  static constexpr int kTile = kTileM * D * 2;          // one [128][D] bf16 tile
  static constexpr int kHalf = kTileM * 128;            // 128 rows x 64 columns bf16
  static constexpr int kOffQ = 0;
  static constexpr int kOffDO = kOffQ + kTile;
  static constexpr int kOffK = kOffDO + kTile;          // [stage]
  static constexpr int kOffV = kOffK + kStages * kTile; // [stage]
  static constexpr int kOffBar = kOffV + kStages * kTile;
  static constexpr int kNumBars = 2 * kStages + 2 + 2 + 1;
  static constexpr int kSmemBytes = kOffBar + kNumBars * 8 + 16 + 1024;
  static constexpr int kThreads = 320;
  static constexpr uint32_t kColS = 0;       // [2] x 64 columns: S, then packed dS
  static constexpr uint32_t kColDP = 128;    // [2] x 64 columns: dP
  static constexpr uint32_t kColQ = 256;     // dQ accumulator
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kSmemBytes <= 232448, "bw_q2 shared memory beyond the per-CTA limit");
};

template <int D, int MODE>
__global__ void __launch_bounds__(320, 1)
    bw_q2_kernel(const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const BwArgs a) {
  using C = BwQ2Cfg<D>;
  constexpr int ST = C::kStages;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* kv_full = bars;            // [ST] K / V tile landed
  uint64_t* kv_empty = kv_full + ST;   // [ST] its last dQ MMA done
  uint64_t* s_full = kv_empty + ST;    // [2] S / dP of a half in TMEM
  uint64_t* p_full = s_full + 2;       // [2] dS of a half packed
  uint64_t* done_bar = p_full + 2;     // every MMA done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = threadIdx.x & 127;  // row of this thread (warps 0-7)
  const int hc = (warp >> 2) & 1;   // key half within a 64-key half (elementwise) / row half (gather)
  const int NB = a.P.totals[0];

  int g, J, nkt, blen;
  int64_t kblock;
  BwRow x{-1, 0};
  if (MODE == kBwRouted) {
    const int64_t nitems = a.tile_off[a.nu * NB];
    if (blockIdx.x >= nitems) return;
    const int f = upper_index(a.tile_off, a.nu * NB + 1, blockIdx.x);
    const int u = f / NB;
    J = f % NB;
    g = a.u0 + u;
    const int64_t e0 = a.entry_off[f] + (int64_t)(blockIdx.x - a.tile_off[f]) * kTileM;
    if (warp < 8) x = bw_row_routed(a, g, e0, a.entry_off[f + 1], r);
    blen = a.P.blk_len[J];
    kblock = a.P.blk_tok[J];
    nkt = (blen + kTileN - 1) / kTileN;
  } else {
    const int NQT = a.P.totals[1];
    const int64_t idx = blockIdx.x;
    const int hl = (int)(idx / NQT);
    const int qt = (int)(idx % NQT);
    if (hl >= a.nu * a.G) return;
    const int s = upper_index(a.P.qt_off, a.L.nseq + 1, qt);
    const int64_t st0 = seq_start(a.L, s), len = seq_len(a.L, s);
    const int64_t p0 = (int64_t)(qt - a.P.qt_off[s]) * kTileM;
    const int i = (int)(p0 / a.B);
    J = a.P.blk_off[s] + i;
    g = a.u0 + hl / a.G;
    blen = a.P.blk_len[J];
    kblock = a.P.blk_tok[J];
    nkt = (int)((p0 - (int64_t)i * a.B) / kTileN) + 1;  // up to the diagonal tile
    if (warp < 8 && p0 + r < len) {
      x.t = st0 + p0 + r;
      x.h = g * a.G + hl % a.G;
    }
  }
  const int nh = 2 * nkt;  // 64-key halves

  if (threadIdx.x == 0) {
    for (int q = 0; q < ST; ++q) {
      mbar_init(&kv_full[q], 1);
      mbar_init(&kv_empty[q], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 8);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 8) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  unsigned char* sQ = smem + C::kOffQ;
  unsigned char* sDO = smem + C::kOffDO;
  float lse2 = __int_as_float(0x7f800000), Dr = 0.f;
  if (warp < 8) {
    if (x.t >= 0) {
      const float2 v = a.dl[(size_t)x.t * a.Hq + x.h];
      Dr = v.x;
      lse2 = v.y;
    }
    bw_load_row<D>(a, x, r, hc, sQ, sDO);
    cp_async_wait_all();
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  uint32_t* st = a.status;

  if (warp == 9) {
    // ------------------------------------------------------------ K / V producer
    if (lane == 0) {
      int t = 0;
      bool ok = true;
      for (; t < nkt && ok; ++t) {
        const int sg = t % ST;
        ok = mbar_wait(&kv_empty[sg], ((t / ST) & 1) ^ 1, abort_flag, st);
        if (!ok) break;
        mbar_arrive_expect_tx(&kv_full[sg], 2 * C::kTile);
        const int64_t kb = kblock + (int64_t)t * kTileN;
#pragma unroll
        for (int hx = 0; hx < D / 64; ++hx) {
          tma_load_3d(smem + C::kOffK + sg * C::kTile + hx * C::kHalf, &tm_k, &kv_full[sg],
                      hx * 64, g, (int)kb);
          tma_load_3d(smem + C::kOffV + sg * C::kTile + hx * C::kHalf, &tm_v, &kv_full[sg],
                      hx * 64, g, (int)kb);
        }
      }
      if (!ok) {  // loads still in flight: the last ST issued
        for (int b = 0; b < ST && b < t; ++b) {
          const int l = t - 1 - b;
          mbar_wait_teardown(&kv_full[l % ST], (l / ST) & 1, 200000000ull);
        }
      }
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ MMA issue
    auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, st));
    };
    constexpr uint32_t idS = idesc_bf16_f32(kTileM, 64, false, false);  // M = rows, N = keys
    constexpr uint32_t idQ = idesc_bf16_f32(kTileM, D, false, true);    // A in TMEM, B MN-major
    const uint32_t sQa = smem_u32(sQ), sDOa = smem_u32(sDO);
    const uint32_t sKa = smem_u32(smem + C::kOffK), sVa = smem_u32(smem + C::kOffV);
    // dQ += dS(m) K(m): A = dS packed in buffer m % 2, B = the half's 64 keys x D
    auto dq_mmas = [&](int m) -> bool {
      const int b = m & 1, t = m >> 1, hf = m & 1, sg = t % ST;
      if (!wait(&p_full[b], (m >> 1) & 1)) return false;
      tc_fence_after();
      const uint32_t kb = sKa + sg * C::kTile + hf * 8192;  // keys 64 hf .. : 64 rows of 128 B
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)  // K = keys, 16 per step
        tc_mma_ts_warp(tmem + C::kColQ, tmem + C::kColS + 64u * b + bw2_packed_col(kk),
                       sdesc_mnmajor_sw128(kb + kk * 2048, C::kHalf, 1024), idQ,
                       (m > 0 || kk > 0) ? 1u : 0u);
      if (hf == 1) tc_commit_warp(&kv_empty[sg]);  // the tile's last reader
      return true;
    };
    bool ok = true;
    int m = 0;
    for (; m < nh && ok; ++m) {
      const int b = m & 1, t = m >> 1, hf = m & 1, sg = t % ST;
      if (hf == 0 && !(ok = wait(&kv_full[sg], (t / ST) & 1))) break;
      tc_fence_after();
      const uint32_t kb = sKa + sg * C::kTile + hf * 8192;
      const uint32_t vb = sVa + sg * C::kTile + hf * 8192;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * C::kHalf + (kk & 3) * 32;
        tc_mma_ss_warp(tmem + C::kColS + 64u * b, sdesc_kmajor_sw128(sQa + off),
                       sdesc_kmajor_sw128(kb + off), idS, kk > 0 ? 1u : 0u);
        tc_mma_ss_warp(tmem + C::kColDP + 64u * b, sdesc_kmajor_sw128(sDOa + off),
                       sdesc_kmajor_sw128(vb + off), idS, kk > 0 ? 1u : 0u);
      }
      tc_commit_warp(&s_full[b]);
      if (m > 0 && !(ok = dq_mmas(m - 1))) break;
    }
    if (ok && m > 0) ok = dq_mmas(m - 1);
    tc_commit_warp(done_bar);  // every MMA of this CTA (also after an abort)
  } else {
    // ------------------------------------------------------------ elementwise (warps 0-7)
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    bool ok = true;
    for (int m = 0; m < nh && ok; ++m) {
      const int b = m & 1, t = m >> 1, hf = m & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[b], (m >> 1) & 1, abort_flag, st));
      if (!ok) break;
      tc_fence_after();
      const int c0 = 32 * hc;  // this warp's keys within the half
      const uint32_t tS = tmem + lane_off + C::kColS + 64u * b;
      const uint32_t tDP = tmem + lane_off + C::kColDP + 64u * b;
      uint32_t sv[32], dv[32];
      tmem_ld32(tS + c0, sv);
      tmem_ld32(tDP + c0, dv);
      tc_wait_ld();
      const int key0 = t * kTileN + hf * 64 + c0;  // key of column 0 within the block
      const int64_t ktok0 = kblock + key0;
      uint32_t dd[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        float d2[2];
#pragma unroll
        for (int xx = 0; xx < 2; ++xx) {
          const int j = 2 * e + xx;
          bool keep = key0 + j < blen;
          if (MODE == kBwOwn) keep = keep && (ktok0 + j <= x.t);
          const float p =
              keep ? ex2_approx(fmaf(__uint_as_float(sv[j]), a.scale_log2, -lse2)) : 0.f;
          d2[xx] = p * (__uint_as_float(dv[j]) - Dr);
        }
        dd[e] = pack_bf16x2(d2[0], d2[1]);
      }
      tmem_st16(tS + (hc ? 32u : 0u), dd);
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[b]);
    }
    const bool done = __all_sync(0xffffffffu, mbar_wait(done_bar, 0, abort_flag, st));
    if (ok && done) {
      tc_fence_after();
#pragma unroll 1
      for (int cc = hc * (D / 2); cc < (hc + 1) * (D / 2); cc += 32) {
        uint32_t va[32];
        tmem_ld32(tmem + lane_off + C::kColQ + cc, va);
        tc_wait_ld();
        if (x.t >= 0) {
          float* dq = a.dq32 + ((size_t)x.t * a.Hq + x.h) * D + cc;
#pragma unroll
          for (int e = 0; e < 32; ++e) atomicAdd(dq + e, __uint_as_float(va[e]) * a.scale);
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  if (threadIdx.x == 0) mbar_wait_teardown(done_bar, 0, 500000000ull);
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// fp32 accumulators -> bf16 gradients.
__global__ void bw_finish_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                                 int64_t n) {
  const int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (i + 3 < n) {
    const float4 v = *reinterpret_cast<const float4*>(src + i);
    *reinterpret_cast<uint2*>(dst + i) = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
  } else {
    for (int64_t j = i; j < n; ++j) dst[j] = __float2bfloat16_rn(src[j]);
  }
}

}  // namespace moba
