// layout.cuh -- how tokens, blocks and query tiles are numbered on the device.
//
// Every call is handled as a set of packed sequences: q/k/v/o are [T][H][d]
// with sequence s covering tokens [start(s), start(s) + len(s)).  A batch of
// b sequences of length N is the case start(s) = s*N (no cu_seqlens array).
//
// Blocks (MoBA: Mixture of Block Attention, wispaper.ai blog, "The Change":
// block partition) are contiguous runs of B tokens from each sequence's
// start; the last block of a sequence may be short.  Blocks are numbered
// globally, sequence by sequence.  Query tiles are runs of 128 tokens from
// each sequence's start; because B is a multiple of 128 a tile never spans
// two blocks.
#pragma once
#include <stdint.h>

namespace moba {

constexpr int kTileM = 128;  // query rows per tile
constexpr int kTileN = 128;  // keys per KV tile

struct SeqLayout {
  const int32_t* cu;  // device cu_seqlens [nseq+1], or nullptr for a fixed-length batch
  int nseq;
  int N;              // sequence length when cu == nullptr
  int64_t T;          // total tokens
};

// Device plan written by plan_kernel (workspace).
struct Plan {
  int32_t* totals;    // [0] blocks NB, [1] query tiles NQT, [2] query-tile pairs
  int32_t* blk_off;   // [nseq+1] first global block of each sequence
  int32_t* qt_off;    // [nseq+1] first query tile of each sequence
  int32_t* pair_off;  // [nseq+1] first query-tile pair (256 rows) of each sequence
  int32_t* blk_tok;   // [NBmax] first token of each global block
  int32_t* blk_len;   // [NBmax] tokens in each global block
};

// Row index of (sequence, head, position, token) in lse [.][H][.] and sel.
struct RowLayout {
  int64_t seq_stride;
  int64_t head_stride;
  int use_token;  // 1: index by global token (varlen), 0: by position (batch)
};

__device__ __forceinline__ int64_t seq_start(const SeqLayout& L, int s) {
  return L.cu ? (int64_t)L.cu[s] : (int64_t)s * L.N;
}
__device__ __forceinline__ int64_t seq_len(const SeqLayout& L, int s) {
  return L.cu ? (int64_t)(L.cu[s + 1] - L.cu[s]) : (int64_t)L.N;
}
__device__ __forceinline__ int64_t row_index(const RowLayout& R, int s, int h, int64_t pos,
                                             int64_t tok) {
  return (int64_t)s * R.seq_stride + (int64_t)h * R.head_stride + (R.use_token ? tok : pos);
}

// Largest i in [0, n) with a[i] <= x (a non-decreasing, a[0] <= x).
__device__ __forceinline__ int upper_index(const int32_t* a, int n, int64_t x) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if ((int64_t)a[mid] <= x)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}
__device__ __forceinline__ int seq_of_token(const SeqLayout& L, int64_t t) {
  if (!L.cu) return (int)(t / L.N);
  return upper_index(L.cu, L.nseq + 1, t);
}

}  // namespace moba
