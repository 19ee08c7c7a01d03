// moba_api.cu -- the C ABI of libmoba (declared in include/moba.h): argument
// checks, workspace carving, TMA descriptor encoding and the launch sequence
// of the MoBA causal prefill forward on one sm_100a GPU.
//
// Launch sequence of moba_forward (one stream, no host synchronisation):
//   plan -> pool -> gate -> for each pass of kv heads:
//     bucket scan -> bucket scatter -> routed attention -> own-block
//     attention -> merge
// The routed/own split and the online-softmax merge follow the method's
// implementation outline (MoBA: Mixture of Block Attention, wispaper.ai
// blog, "Efficiency and Implementation"; sherconan.github.io step 5):
// queries are arranged by their selected past blocks (bucketing), attention
// runs per block, and the per-block results are recombined by online
// softmax.  Each step is a kernel of this library.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <mutex>
#include <vector>

#include "moba.h"
#include "aux_kernels.cuh"
#include "attn_tc2.cuh"
#include "gate_tc.cuh"
#include "decode.cuh"
#include "variants.cuh"
#include "backward.cuh"
#include "common.cuh"
#include "layout.cuh"

using namespace moba;

namespace {

// ------------------------------------------------------------ kernel timer
enum KernelClass {
  kKPlan, kKPool, kKGate, kKGateCount, kKScan, kKScatter, kKRouted, kKOwn, kKMerge, kKDense,
  kKKbarCache, kKDecGate, kKDecAttn, kKDecMerge, kKMinmaxPool, kKGateMinmax, kKStaticSel,
  kKBwPrep, kKBwKv, kKBwQ, kKBwFinish, kKVbound, kKNum
};
const char* const kKernelNames[kKNum] = {
    "plan",        "pool",        "gate",         "gate_count",  "bucket_scan",
    "bucket_scatter", "attn_routed", "attn_own",  "merge",       "attn_dense",
    "kbar_cache",  "decode_gate", "decode_attn",  "decode_merge", "minmax_pool",
    "gate_minmax", "static_select", "bw_prep", "bw_kv", "bw_q", "bw_finish", "vbound"};
struct TimedLaunch {
  int cls;
  cudaEvent_t a, b;
};
struct KernelTimer {
  bool on = false;
  std::vector<TimedLaunch> pending;
  int launches[kKNum] = {};
  double ms[kKNum] = {};
};
KernelTimer& timer() {
  static KernelTimer t;
  return t;
}
// RAII bracket around one launch: events on the launch stream when enabled.
struct Timed {
  int cls;
  cudaStream_t st;
  cudaEvent_t a = nullptr, b = nullptr;
  Timed(int c, cudaStream_t s) : cls(c), st(s) {
    if (!timer().on) return;
    if (cudaEventCreate(&a) != cudaSuccess || cudaEventCreate(&b) != cudaSuccess) {
      a = b = nullptr;
      return;
    }
    cudaEventRecord(a, st);
  }
  ~Timed() {
    if (!a) return;
    cudaEventRecord(b, st);
    timer().pending.push_back(TimedLaunch{cls, a, b});
  }
};

// Last CUDA runtime error seen by this thread inside the library.
thread_local const char* g_last_cuda_error = "no error";

// Device address of the allocation-free gate's scratch (defined with it).
moba_status gate_scratch_address(void** out);

moba_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return MOBA_OK;
  g_last_cuda_error = cudaGetErrorString(e);
  return MOBA_ERR_CUDA;
}

#define MOBA_TRY(x)                      \
  do {                                   \
    moba_status _s = (x);                \
    if (_s != MOBA_OK) return _s;        \
  } while (0)
#define MOBA_CUDA(x)                                   \
  do {                                                 \
    moba_status _c = cuda_status(x);                   \
    if (_c != MOBA_OK) return _c;                      \
  } while (0)

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct Problem {
  bool varlen;
  int nseq;
  int N;          // batch: seqlen
  int64_t T;
  const int32_t* cu;
  int Hq, Hkv, G, D, B, topk;
  float scale;
  int64_t NBmax, NQTmax;
  int64_t max_blocks_per_seq;  // upper bound
  RowLayout R;
};

struct Ws {
  uint32_t* status;
  Plan P;
  float* kbar;
  uint32_t* counts;
  int32_t* entry_off;
  int32_t* tile_off;
  uint32_t* cursor;
  uint2* entries;
  __half* part_O;  // routed partial O, fp16
  float* part_lse;
  float* own_O;
  float* own_lse;
  int32_t* sel;
  size_t bytes;
};

// Carve (or only measure, base == nullptr) the workspace for `nu` kv heads per pass.
Ws carve(const Problem& pr, int nu, char* base) {
  Ws w;
  memset(&w, 0, sizeof w);
  size_t off = 0;
  auto take = [&](size_t bytes) -> char* {
    char* p = base ? base + off : nullptr;
    off = align_up(off + bytes);
    return p;
  };
  const int64_t NB = pr.NBmax, NQ = pr.NQTmax;
  const int64_t np = pr.topk > 1 ? pr.topk - 1 : 0;
  (void)NQ;
  w.status = reinterpret_cast<uint32_t*>(take(kAlign));
  w.P.totals = reinterpret_cast<int32_t*>(take(4 * sizeof(int32_t)));
  w.P.blk_off = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (pr.nseq + 1)));
  w.P.qt_off = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (pr.nseq + 1)));
  w.P.pair_off = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (pr.nseq + 1)));
  w.P.blk_tok = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * NB));
  w.P.blk_len = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * NB));
  w.kbar = reinterpret_cast<float*>(take(sizeof(float) * (size_t)pr.Hkv * NB * pr.D));
  w.counts = reinterpret_cast<uint32_t*>(take(sizeof(uint32_t) * (size_t)pr.Hkv * NB));
  w.sel = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (size_t)pr.Hq * pr.T * pr.topk));
  w.entry_off = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * ((size_t)nu * NB + 1)));
  w.tile_off = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * ((size_t)nu * NB + 1)));
  w.cursor = reinterpret_cast<uint32_t*>(take(sizeof(uint32_t) * (size_t)nu * NB));
  const size_t prow = (size_t)nu * pr.T * pr.G;  // partial rows per pass
  w.entries = reinterpret_cast<uint2*>(take(sizeof(uint2) * prow * np));
  w.part_O = reinterpret_cast<__half*>(take(2 * prow * np * pr.D));
  w.part_lse = reinterpret_cast<float*>(take(sizeof(float) * prow * np));
  w.own_O = reinterpret_cast<float*>(take(sizeof(float) * prow * pr.D));
  w.own_lse = reinterpret_cast<float*>(take(sizeof(float) * prow));
  w.bytes = off;
  return w;
}

moba_status make_problem(const moba_params* p, bool varlen, const int32_t* cu, int num_seqs,
                         int64_t total_tokens, bool need_blocks, Problem* out) {
  if (!p) return MOBA_ERR_INVALID_ARG;
  Problem pr;
  memset(&pr, 0, sizeof pr);
  pr.varlen = varlen;
  if (varlen) {
    if (!cu || num_seqs <= 0 || total_tokens < 0) return MOBA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(cu) % 4) return MOBA_ERR_INVALID_ARG;
    pr.nseq = num_seqs;
    pr.N = 0;
    pr.T = total_tokens;
    pr.cu = cu;
  } else {
    if (p->batch <= 0 || p->seqlen < 0) return MOBA_ERR_INVALID_ARG;
    pr.nseq = p->batch;
    pr.N = p->seqlen;
    pr.T = (int64_t)p->batch * p->seqlen;
    pr.cu = nullptr;
  }
  if (pr.T >= (int64_t(1) << 31) - 256) return MOBA_ERR_UNSUPPORTED;
  if (p->num_q_heads <= 0 || p->num_kv_heads <= 0 || p->num_q_heads % p->num_kv_heads)
    return MOBA_ERR_INVALID_ARG;
  pr.Hq = p->num_q_heads;
  pr.Hkv = p->num_kv_heads;
  pr.G = pr.Hq / pr.Hkv;
  // q rows are addressed as one int32 index of q viewed as [T*Hq][D] (TMA
  // row gathers); that q would be 512 GB at D = 128
  if (pr.T * pr.Hq >= (int64_t)INT32_MAX) return MOBA_ERR_UNSUPPORTED;
  if (p->head_dim != 64 && p->head_dim != 128) return MOBA_ERR_UNSUPPORTED;
  pr.D = p->head_dim;
  if (need_blocks) {
    if (p->block_size <= 0 || p->top_k <= 0) return MOBA_ERR_INVALID_ARG;
    if (p->block_size % kTileM) return MOBA_ERR_UNSUPPORTED;
    pr.B = p->block_size;
    pr.topk = p->top_k;
  } else {
    pr.B = kTileM;  // block numbering unused by the dense kernel
    pr.topk = 1;
  }
  if (pr.G > 65535 || pr.topk > 65536) return MOBA_ERR_UNSUPPORTED;
  pr.scale = (p->softmax_scale > 0.f) ? p->softmax_scale : 1.0f / sqrtf((float)pr.D);
  if (!(pr.scale < INFINITY)) return MOBA_ERR_INVALID_ARG;
  if (varlen) {
    pr.NBmax = pr.T / pr.B + pr.nseq;
    pr.NQTmax = pr.T / kTileM + pr.nseq;
    pr.max_blocks_per_seq = (pr.T + pr.B - 1) / pr.B;
  } else {
    const int64_t nb = ((int64_t)pr.N + pr.B - 1) / pr.B;
    pr.NBmax = (int64_t)pr.nseq * nb;
    pr.NQTmax = (int64_t)pr.nseq * (((int64_t)pr.N + kTileM - 1) / kTileM);
    pr.max_blocks_per_seq = nb;
    if (nb > kMaxBlocksPerSeq) return MOBA_ERR_UNSUPPORTED;
  }
  if (pr.NBmax < 1) pr.NBmax = 1;
  if (pr.NQTmax < 1) pr.NQTmax = 1;
  if (pr.NBmax > INT32_MAX / 4 || pr.NQTmax > INT32_MAX / 4) return MOBA_ERR_UNSUPPORTED;
  if (varlen) {
    pr.R.seq_stride = 0;
    pr.R.head_stride = pr.T;
    pr.R.use_token = 1;
  } else {
    pr.R.seq_stride = (int64_t)pr.Hq * pr.N;
    pr.R.head_stride = pr.N;
    pr.R.use_token = 0;
  }
  *out = pr;
  return MOBA_OK;
}

int pow2_at_least(int64_t x) {
  int v = 1;
  while (v < x) v <<= 1;
  return v;
}

// ---------------------------------------------------------------- TMA maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, []() {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// [T][H][D] bf16 viewed as (x = D, y = H, z = T), box 64 x 1 x 128, 128-B swizzle.
bool make_tmap(CUtensorMap* m, const void* ptr, int H, int64_t T, int D) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)(T > 0 ? T : 1)};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)kTileM};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// [T][H][D] bf16 viewed as rows (x = D, y = T*H), box 64 x 1, 128-B swizzle:
// the routed kernel's four-row gathers of (token, head) rows.  Row indices
// are int32, so T*H must stay below 2^31 (make_problem checks).
bool make_tmap_rows(CUtensorMap* m, const void* ptr, int64_t rows, int D) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)(rows > 0 ? rows : 1)};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, 1};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

template <int D, int MODE, int QB>
moba_status launch_attn_qb(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const AttnArgs& a, int pair_own, cudaStream_t stream) {
  using C = Attn2Cfg<D, QB>;
  auto kern = attn2_kernel<D, MODE, QB>;
  MOBA_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::kSmemBytes));
  const int grid = num_sms();
  if (grid <= 0) return MOBA_ERR_CUDA;
  Timed tm(MODE == kRouted ? kKRouted : (MODE == kOwn ? kKOwn : kKDense), stream);
  kern<<<grid, C::kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, a, pair_own);
  return cuda_status(cudaGetLastError());
}

// Routed and own-block items over blocks of up to kShortBlock keys are short
// (at most 8 KV tiles): they take two Q buffers so the next item's rows load
// during this one.  Longer blocks and the dense kernel take one.
constexpr int kShortBlock = 1024;

template <int D, int MODE>
moba_status launch_attn(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                        const AttnArgs& a, int pair_own, cudaStream_t stream) {
  if (MODE != kDense && a.B <= kShortBlock)
    return launch_attn_qb<D, MODE == kDense ? kOwn : MODE, 2>(tq, tk, tv, a, pair_own, stream);
  return launch_attn_qb<D, MODE, 1>(tq, tk, tv, a, pair_own, stream);
}

template <int D, int KM>
moba_status launch_gate_km(const Problem& pr, const void* q, const Ws& w, int32_t* sel,
                           uint32_t* counts, cudaStream_t st, int g0, int ng,
                           int min_past = -1) {
  const size_t smem = sizeof(float) * kGateChunk * D + sizeof(uint32_t) * kMaxBlocksPerSeq;
  auto kern = gate_kernel<D, KM>;
  if (smem > 48 * 1024)
    MOBA_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  SeqLayout L{pr.cu, pr.nseq, pr.N, pr.T};
  dim3 grid((unsigned)pr.NQTmax, (unsigned)(ng * pr.G));
  Timed tm(kKGate, st);
  kern<<<grid, 128, smem, st>>>(reinterpret_cast<const __nv_bfloat16*>(q), pr.Hq, pr.G, pr.B,
                                pr.topk, L, w.P, (int)pr.NBmax, w.kbar, sel, pr.R, counts,
                                w.status, g0 * pr.G, min_past);
  return cuda_status(cudaGetLastError());
}

// Tensor-core gate: scores as tcgen05 MMAs, branch-free selection; then
// the bucket sizes from the written selections.
template <int D, int KM>
moba_status launch_gate_tc_km(const Problem& pr, const void* q, const Ws& w, int32_t* sel,
                              uint32_t* counts, cudaStream_t st, int g0, int ng) {
  using C = GateTcCfg<D, KM>;
  CUtensorMap tq;
  if (!make_tmap(&tq, q, pr.Hq, pr.T, D)) return MOBA_ERR_CUDA;
  auto kern = gate_tc_kernel<D, KM>;
  MOBA_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::kSmemBytes));
  const int grid = num_sms();
  if (grid <= 0) return MOBA_ERR_CUDA;
  SeqLayout L{pr.cu, pr.nseq, pr.N, pr.T};
  GateTcArgs a;
  a.kbar = w.kbar;
  a.Hq = pr.Hq;
  a.G = pr.G;
  a.B = pr.B;
  a.topk = pr.topk;
  a.NBmax = (int)pr.NBmax;
  a.L = L;
  a.P = w.P;
  a.R = pr.R;
  a.sel = sel;
  a.status = w.status;
  a.g0 = g0;
  a.ng = ng;
  // sequences longer than a score tile covers: their later query tiles go to
  // the SIMT gate (only those tiles; the others return at once)
  a.companion = pr.max_blocks_per_seq - 1 > C::kMaxPast ? 1 : 0;
  {
    Timed tm(kKGate, st);
    kern<<<grid, C::kThreads, C::kSmemBytes, st>>>(tq, a);
    MOBA_CUDA(cudaGetLastError());
  }
  if (a.companion)
    MOBA_TRY((launch_gate_km<D, (KM <= 16 ? 16 : KM)>(pr, q, w, sel, nullptr, st, g0, ng,
                                                        C::kMaxPast)));
  if (counts) {
    const size_t smem = sizeof(uint32_t) * kMaxBlocksPerSeq;
    dim3 cgrid((unsigned)pr.NQTmax, (unsigned)ng);
    Timed tm(kKGateCount, st);
    gate_count_kernel<<<cgrid, 128, smem, st>>>(sel, pr.R, pr.topk, pr.B, pr.G, L, w.P,
                                                (int)pr.NBmax, counts, w.status, g0);
    MOBA_CUDA(cudaGetLastError());
  }
  return MOBA_OK;
}

// The tensor-core gate ranks up to 32 past blocks; query tiles with more past
// blocks than its score tile holds (256, or 128 when k-1 > 16) are handed to
// the SIMT gate.
bool gate_tc_fits(const Problem& pr) {
  const int64_t npast = pr.topk - 1;
  return npast >= 1 && npast <= kGateTcMaxKeep && npast < pr.max_blocks_per_seq - 1;
}

// The gate for the q heads of kv heads g0 .. g0 + ng - 1 (default: all).
template <int D>
moba_status launch_gate(const Problem& pr, const void* q, const Ws& w, int32_t* sel,
                        uint32_t* counts, cudaStream_t st, int g0 = 0, int ng = -1) {
  if (ng < 0) ng = pr.Hkv;
  const int64_t npast = pr.topk - 1;
  if (gate_tc_fits(pr)) {
    switch (pow2_at_least(npast)) {
      case 1: return launch_gate_tc_km<D, 1>(pr, q, w, sel, counts, st, g0, ng);
      case 2: return launch_gate_tc_km<D, 2>(pr, q, w, sel, counts, st, g0, ng);
      case 4: return launch_gate_tc_km<D, 4>(pr, q, w, sel, counts, st, g0, ng);
      case 8: return launch_gate_tc_km<D, 8>(pr, q, w, sel, counts, st, g0, ng);
      case 16:
        if (npast <= 12) return launch_gate_tc_km<D, 12>(pr, q, w, sel, counts, st, g0, ng);
        return launch_gate_tc_km<D, 16>(pr, q, w, sel, counts, st, g0, ng);
      default: return launch_gate_tc_km<D, 32>(pr, q, w, sel, counts, st, g0, ng);
    }
  }
  const int64_t need = (npast >= pr.max_blocks_per_seq - 1) ? 1 : npast;
  switch (pow2_at_least(need)) {
    case 1: return launch_gate_km<D, 1>(pr, q, w, sel, counts, st, g0, ng);
    case 2: return launch_gate_km<D, 2>(pr, q, w, sel, counts, st, g0, ng);
    case 4: return launch_gate_km<D, 4>(pr, q, w, sel, counts, st, g0, ng);
    case 8: return launch_gate_km<D, 8>(pr, q, w, sel, counts, st, g0, ng);
    case 16: return launch_gate_km<D, 16>(pr, q, w, sel, counts, st, g0, ng);
    case 32: return launch_gate_km<D, 32>(pr, q, w, sel, counts, st, g0, ng);
    case 64: return launch_gate_km<D, 64>(pr, q, w, sel, counts, st, g0, ng);
    default: return MOBA_ERR_UNSUPPORTED;
  }
}

template <int KS>
moba_status launch_scatter_ks(const Problem& pr, const Ws& w, const int32_t* sel, int u0, int nu,
                              cudaStream_t st) {
  SeqLayout L{pr.cu, pr.nseq, pr.N, pr.T};
  dim3 grid((unsigned)pr.NQTmax, (unsigned)(nu * pr.G));
  Timed tm(kKScatter, st);
  bucket_scatter_kernel<KS><<<grid, 128, sizeof(uint32_t) * kMaxBlocksPerSeq, st>>>(
      sel, pr.R, pr.topk, pr.B, pr.G, u0, nu, L, w.P, w.entry_off, w.cursor, w.entries,
      w.status);
  return cuda_status(cudaGetLastError());
}

moba_status launch_scatter(const Problem& pr, const Ws& w, const int32_t* sel, int u0, int nu,
                           cudaStream_t st) {
  int64_t need = pr.topk - 1;
  if (need > pr.max_blocks_per_seq - 1) need = pr.max_blocks_per_seq - 1;
  if (need < 1) need = 1;
  switch (pow2_at_least(need)) {
    case 1: return launch_scatter_ks<1>(pr, w, sel, u0, nu, st);
    case 2: return launch_scatter_ks<2>(pr, w, sel, u0, nu, st);
    case 4: return launch_scatter_ks<4>(pr, w, sel, u0, nu, st);
    case 8: return launch_scatter_ks<8>(pr, w, sel, u0, nu, st);
    case 16: return launch_scatter_ks<16>(pr, w, sel, u0, nu, st);
    case 32: return launch_scatter_ks<32>(pr, w, sel, u0, nu, st);
    case 64: return launch_scatter_ks<64>(pr, w, sel, u0, nu, st);
    default: return MOBA_ERR_UNSUPPORTED;
  }
}

bool topk_supported(const Problem& pr) {
  const int64_t npast = pr.topk - 1;
  return npast <= 64 || npast >= pr.max_blocks_per_seq - 1;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moba_status check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) % kAlign)) return MOBA_ERR_WORKSPACE;
  if (ws_bytes < need) return MOBA_ERR_WORKSPACE;
  return MOBA_OK;
}

// Block means of kv heads g0 .. g0 + ng - 1.
moba_status run_pool(const Problem& pr, const void* k, const Ws& w, cudaStream_t st, int g0,
                     int ng) {
  dim3 grid((unsigned)pr.NBmax, (unsigned)ng);
  Timed tm(kKPool, st);
  if (pr.D == 128)
    pool_kernel<128><<<grid, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(k), pr.Hkv,
                                           w.P, (int)pr.NBmax, w.kbar, g0);
  else
    pool_kernel<64><<<grid, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(k), pr.Hkv,
                                          w.P, (int)pr.NBmax, w.kbar, g0);
  return cuda_status(cudaGetLastError());
}

// Largest |v| of kv heads g0 .. g0 + ng - 1 into status[1] (the routed
// partials' scale; see vbound_kernel).
moba_status run_vbound(const Problem& pr, const void* v, const Ws& w, cudaStream_t st, int g0,
                       int ng) {
  if (pr.topk <= 1) return MOBA_OK;  // no routed partials
  dim3 grid((unsigned)pr.NBmax, (unsigned)ng);
  Timed tm(kKVbound, st);
  if (pr.D == 128)
    vbound_kernel<128><<<grid, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(v), pr.Hkv,
                                             w.P, w.status + 1, g0);
  else
    vbound_kernel<64><<<grid, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(v), pr.Hkv,
                                            w.P, w.status + 1, g0);
  return cuda_status(cudaGetLastError());
}

moba_status run_plan_pool(const Problem& pr, const void* k, const Ws& w, cudaStream_t st) {
  SeqLayout L{pr.cu, pr.nseq, pr.N, pr.T};
  {
    Timed tm(kKPlan, st);
    plan_kernel<<<1, 1024, 0, st>>>(L, pr.B, w.P, (int)pr.NBmax, (int)pr.NQTmax, w.status);
  }
  MOBA_CUDA(cudaGetLastError());
  return run_pool(pr, k, w, st, 0, pr.Hkv);
}

// How a forward obtains its selection.
enum Routing { kRouteMeanGate = 0, kRouteMinmaxGate = 1, kRouteGiven = 2 };

moba_status run_plan(const Problem& pr, const Ws& w, cudaStream_t st) {
  SeqLayout L{pr.cu, pr.nseq, pr.N, pr.T};
  Timed tm(kKPlan, st);
  plan_kernel<<<1, 1024, 0, st>>>(L, pr.B, w.P, (int)pr.NBmax, (int)pr.NQTmax, w.status);
  return cuda_status(cudaGetLastError());
}

// Block max / min (bf16 pairs) into the block-mean buffer, which has exactly
// the room: 2 x 2 bytes per element against 4.
moba_status run_minmax_pool(const Problem& pr, const void* k, const Ws& w, cudaStream_t st) {
  dim3 grid((unsigned)pr.NBmax, (unsigned)pr.Hkv);
  __nv_bfloat16* mm = reinterpret_cast<__nv_bfloat16*>(w.kbar);
  Timed tm(kKMinmaxPool, st);
  if (pr.D == 128)
    minmax_pool_kernel<128><<<grid, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(k),
                                                  pr.Hkv, w.P, (int)pr.NBmax, mm);
  else
    minmax_pool_kernel<64><<<grid, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(k),
                                                 pr.Hkv, w.P, (int)pr.NBmax, mm);
  return cuda_status(cudaGetLastError());
}

template <int D, int KM>
moba_status launch_gate_minmax_km(const Problem& pr, const void* q, const Ws& w, int32_t* sel,
                                  uint32_t* counts, cudaStream_t st) {
  const size_t smem =
      sizeof(float) * kMinmaxChunk * 2 * D + sizeof(uint32_t) * kMaxBlocksPerSeq;
  auto kern = gate_minmax_kernel<D, KM>;
  MOBA_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  SeqLayout L{pr.cu, pr.nseq, pr.N, pr.T};
  dim3 grid((unsigned)pr.NQTmax, (unsigned)pr.Hq);
  Timed tm(kKGateMinmax, st);
  kern<<<grid, 128, smem, st>>>(reinterpret_cast<const __nv_bfloat16*>(q), pr.Hq, pr.G, pr.B,
                                pr.topk, L, w.P, (int)pr.NBmax,
                                reinterpret_cast<const __nv_bfloat16*>(w.kbar), sel, pr.R,
                                counts, w.status);
  return cuda_status(cudaGetLastError());
}

template <int D>
moba_status launch_gate_minmax(const Problem& pr, const void* q, const Ws& w, int32_t* sel,
                               uint32_t* counts, cudaStream_t st) {
  const int64_t npast = pr.topk - 1;
  const int64_t need = (npast >= pr.max_blocks_per_seq - 1) ? 1 : npast;
  switch (pow2_at_least(need)) {
    case 1: return launch_gate_minmax_km<D, 1>(pr, q, w, sel, counts, st);
    case 2: return launch_gate_minmax_km<D, 2>(pr, q, w, sel, counts, st);
    case 4: return launch_gate_minmax_km<D, 4>(pr, q, w, sel, counts, st);
    case 8: return launch_gate_minmax_km<D, 8>(pr, q, w, sel, counts, st);
    case 16: return launch_gate_minmax_km<D, 16>(pr, q, w, sel, counts, st);
    case 32: return launch_gate_minmax_km<D, 32>(pr, q, w, sel, counts, st);
    case 64: return launch_gate_minmax_km<D, 64>(pr, q, w, sel, counts, st);
    default: return MOBA_ERR_UNSUPPORTED;
  }
}

// Bucket sizes from a selection written by someone else.
moba_status launch_count(const Problem& pr, const Ws& w, const int32_t* sel, uint32_t* counts,
                         cudaStream_t st) {
  SeqLayout L{pr.cu, pr.nseq, pr.N, pr.T};
  dim3 grid((unsigned)pr.NQTmax, (unsigned)pr.Hkv);
  Timed tm(kKGateCount, st);
  gate_count_kernel<<<grid, 128, sizeof(uint32_t) * kMaxBlocksPerSeq, st>>>(
      sel, pr.R, pr.topk, pr.B, pr.G, L, w.P, (int)pr.NBmax, counts, w.status);
  return cuda_status(cudaGetLastError());
}

moba_status gate_impl(const Problem& pr, const void* q, const void* k, int32_t* sel, void* ws,
                      size_t ws_bytes, cudaStream_t st) {
  if (!q || !k || !sel || !aligned16(q) || !aligned16(k) || (reinterpret_cast<uintptr_t>(sel) & 3))
    return MOBA_ERR_INVALID_ARG;
  if (!topk_supported(pr)) return MOBA_ERR_UNSUPPORTED;
  const Ws need = carve(pr, 1, nullptr);
  MOBA_TRY(check_ws(ws, ws_bytes, need.bytes));
  if (pr.T == 0) return MOBA_OK;
  const Ws w = carve(pr, 1, static_cast<char*>(ws));
  MOBA_TRY(run_plan_pool(pr, k, w, st));
  return pr.D == 128 ? launch_gate<128>(pr, q, w, sel, nullptr, st)
                     : launch_gate<64>(pr, q, w, sel, nullptr, st);
}

// Attention arguments and tensor maps of one forward call.
struct FwdCtx {
  CUtensorMap tq, tk, tv;
  CUtensorMap tq_rows;  // q as [T*Hq][D] rows (routed gathers)
  AttnArgs a;
};

template <int D>
moba_status forward_setup(const Problem& pr, const void* q, const void* k, const void* v,
                          void* o, float* lse, const Ws& w, FwdCtx* c) {
  if (!make_tmap(&c->tq, q, pr.Hq, pr.T, D) || !make_tmap(&c->tk, k, pr.Hkv, pr.T, D) ||
      !make_tmap(&c->tv, v, pr.Hkv, pr.T, D) || !make_tmap_rows(&c->tq_rows, q, pr.T * pr.Hq, D))
    return MOBA_ERR_CUDA;
  AttnArgs& a = c->a;
  memset(&a, 0, sizeof a);
  a.q = reinterpret_cast<const __nv_bfloat16*>(q);
  a.Hq = pr.Hq;
  a.Hkv = pr.Hkv;
  a.G = pr.G;
  a.B = pr.B;
  a.topk = pr.topk;
  a.scale_log2 = pr.scale * 1.4426950408889634f;
  a.L = SeqLayout{pr.cu, pr.nseq, pr.N, pr.T};
  a.P = w.P;
  a.R = pr.R;
  a.tile_off = w.tile_off;
  a.entry_off = w.entry_off;
  a.entries = w.entries;
  a.part_O = w.part_O;
  a.part_lse = w.part_lse;
  a.own_O = w.own_O;
  a.own_lse = w.own_lse;
  a.o = reinterpret_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.status = w.status;
  return MOBA_OK;
}

// Bucketing, routed and own-block attention and merge for kv heads u0 .. u0 + nu - 1
// (their selection and bucket sizes already written).
template <int D>
moba_status forward_one_pass(const Problem& pr, FwdCtx& c, const Ws& w, const int32_t* sel,
                             void* o, float* lse, int u0, int nu, cudaStream_t st) {
  AttnArgs& a = c.a;
  a.u0 = u0;
  a.nu = nu;
  if (pr.topk > 1) {
    {
      Timed tm(kKScan, st);
      bucket_scan_kernel<<<1, 1024, 0, st>>>(w.counts, u0, nu, 2 * kTileM, w.P, (int)pr.NBmax,
                                             w.entry_off, w.tile_off, w.cursor);
    }
    MOBA_CUDA(cudaGetLastError());
    MOBA_TRY(launch_scatter(pr, w, sel, u0, nu, st));
    MOBA_TRY((launch_attn<D, kRouted>(c.tq_rows, c.tk, c.tv, a, 1, st)));
  }
  MOBA_TRY((launch_attn<D, kOwn>(c.tq, c.tk, c.tv, a, pr.B % (2 * kTileM) == 0 ? 1 : 0, st)));
  if (pr.topk > 1) {
    SeqLayout L{pr.cu, pr.nseq, pr.N, pr.T};
    const int64_t rows = pr.T * nu * pr.G;
    const int64_t rows_per_block = 8 * (32 / (D / 8));
    const unsigned blocks = (unsigned)((rows + rows_per_block - 1) / rows_per_block);
    Timed tm(kKMerge, st);
    merge_kernel<D><<<blocks, 256, 0, st>>>(w.part_O, w.part_lse, w.own_O, w.own_lse, pr.topk,
                                            pr.B, pr.G, pr.Hq, u0, nu, L,
                                            reinterpret_cast<__nv_bfloat16*>(o), lse, pr.R,
                                            w.status);
    MOBA_CUDA(cudaGetLastError());
  }
  return MOBA_OK;
}

template <int D>
moba_status forward_passes(const Problem& pr, const void* q, const void* k, const void* v,
                           void* o, float* lse, const Ws& w, int32_t* sel, int nu_max,
                           int route, cudaStream_t st) {
  FwdCtx c;
  MOBA_TRY(forward_setup<D>(pr, q, k, v, o, lse, w, &c));
  MOBA_CUDA(cudaMemsetAsync(w.counts, 0, sizeof(uint32_t) * (size_t)pr.Hkv * pr.NBmax, st));
  if (route == kRouteMeanGate)
    MOBA_TRY(launch_gate<D>(pr, q, w, sel, w.counts, st));
  else if (route == kRouteMinmaxGate)
    MOBA_TRY(launch_gate_minmax<D>(pr, q, w, sel, w.counts, st));
  else if (pr.topk > 1)
    MOBA_TRY(launch_count(pr, w, sel, w.counts, st));
  for (int u0 = 0; u0 < pr.Hkv; u0 += nu_max) {
    const int nu = (pr.Hkv - u0) < nu_max ? (pr.Hkv - u0) : nu_max;
    MOBA_TRY(forward_one_pass<D>(pr, c, w, sel, o, lse, u0, nu, st));
  }
  return MOBA_OK;
}

// ---------------------------------------------------------------- host-buffer forward
// Device buffer of a forward on host buffers: the forward's workspace first
// (its status word at offset 0, as for every workspace), then staging for
// q, k, v, o, lse and sel.
struct HostBufs {
  char *q, *k, *v, *o;
  float* lse;
  int32_t* sel;
  int32_t* cu;    // packed sequences: the device copy of cu_seqlens
  size_t staged;  // staging bytes
};

HostBufs carve_host(const Problem& pr, char* base, size_t ws_bytes) {
  HostBufs h;
  memset(&h, 0, sizeof h);
  size_t off = align_up(ws_bytes);
  auto take = [&](size_t bytes) -> char* {
    char* p = base ? base + off : nullptr;
    off = align_up(off + bytes);
    return p;
  };
  const size_t qb = (size_t)pr.T * pr.Hq * pr.D * 2, kb = (size_t)pr.T * pr.Hkv * pr.D * 2;
  h.q = take(qb);
  h.k = take(kb);
  h.v = take(kb);
  h.o = take(qb);
  h.lse = reinterpret_cast<float*>(take(sizeof(float) * (size_t)pr.T * pr.Hq));
  h.sel = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (size_t)pr.T * pr.Hq * pr.topk));
  if (pr.varlen) h.cu = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (size_t)(pr.nseq + 1)));
  h.staged = off - align_up(ws_bytes);
  return h;
}

// Two copy streams per device (host -> device, device -> host), created on
// first use.
cudaStream_t copy_stream(int which) {
  static std::mutex mu;
  static cudaStream_t streams[64][2] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!streams[dev][which] &&
      cudaStreamCreateWithFlags(&streams[dev][which], cudaStreamNonBlocking) != cudaSuccess)
    streams[dev][which] = nullptr;
  return streams[dev][which];
}

// Columns [c0, c0 + nc) of a row-major [rows][ncols] array of `esz`-byte elements.
cudaError_t copy_cols(void* dst, const void* src, int64_t rows, int64_t ncols, int64_t c0,
                      int64_t nc, size_t esz, cudaMemcpyKind kind, cudaStream_t st) {
  const size_t pitch = (size_t)ncols * esz;
  return cudaMemcpy2DAsync(static_cast<char*>(dst) + c0 * esz, pitch,
                           static_cast<const char*>(src) + c0 * esz, pitch, (size_t)nc * esz,
                           (size_t)rows, kind, st);
}

// One pass per group of kv heads: its q / k / v columns go in on one copy
// stream while the previous pass computes, its o / lse / sel come back on the
// other while the next pass computes.
template <int D>
moba_status forward_host_passes(const Problem& pr, const void* q_h, const void* k_h,
                                const void* v_h, void* o_h, float* lse_h, int32_t* sel_h,
                                const int32_t* cu_h, const HostBufs& hb, const Ws& w, int nu_max,
                                cudaStream_t st) {
  cudaStream_t h2d = copy_stream(0), d2h = copy_stream(1);
  if (!h2d || !d2h) return MOBA_ERR_CUDA;
  const int npass = (pr.Hkv + nu_max - 1) / nu_max;
  std::vector<cudaEvent_t> ev((size_t)2 * npass + 1, nullptr);
  for (auto& e : ev)
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
      for (auto& x : ev)
        if (x) cudaEventDestroy(x);
      return MOBA_ERR_CUDA;
    }
  cudaEvent_t start = ev[2 * npass];
  auto fail = [&](moba_status s) {
    for (auto& x : ev) cudaEventDestroy(x);  // released once any pending record completes
    return s;
  };
  auto in_ready = [&](int p) { return ev[p]; };
  auto done = [&](int p) { return ev[npass + p]; };
  // lse / sel rows: batch [b][Hq][N](...), packed [Hq][T](...) (one row)
  const int64_t rows_b = pr.varlen ? 1 : pr.nseq;
  const int64_t per_head_lse = pr.varlen ? pr.T : pr.N;
  const int64_t per_head_sel = per_head_lse * pr.topk;
  if (cudaEventRecord(start, st) != cudaSuccess || cudaStreamWaitEvent(h2d, start, 0) != cudaSuccess)
    return fail(MOBA_ERR_CUDA);
  if (pr.varlen && cudaMemcpyAsync(hb.cu, cu_h, sizeof(int32_t) * (size_t)(pr.nseq + 1),
                                   cudaMemcpyHostToDevice, h2d) != cudaSuccess)
    return fail(MOBA_ERR_CUDA);
  // inputs of every pass, in pass order, on the copy stream
  for (int p = 0; p < npass; ++p) {
    const int g0 = p * nu_max, ng = (pr.Hkv - g0) < nu_max ? (pr.Hkv - g0) : nu_max;
    if (copy_cols(hb.k, k_h, pr.T, (int64_t)pr.Hkv * D, (int64_t)g0 * D, (int64_t)ng * D, 2,
                  cudaMemcpyHostToDevice, h2d) != cudaSuccess ||
        copy_cols(hb.q, q_h, pr.T, (int64_t)pr.Hq * D, (int64_t)g0 * pr.G * D,
                  (int64_t)ng * pr.G * D, 2, cudaMemcpyHostToDevice, h2d) != cudaSuccess ||
        copy_cols(hb.v, v_h, pr.T, (int64_t)pr.Hkv * D, (int64_t)g0 * D, (int64_t)ng * D, 2,
                  cudaMemcpyHostToDevice, h2d) != cudaSuccess ||
        cudaEventRecord(in_ready(p), h2d) != cudaSuccess)
      return fail(MOBA_ERR_CUDA);
  }
  FwdCtx c;
  moba_status r = forward_setup<D>(pr, hb.q, hb.k, hb.v, hb.o, hb.lse, w, &c);
  if (r != MOBA_OK) return fail(r);
  if (pr.varlen && cudaStreamWaitEvent(st, in_ready(0), 0) != cudaSuccess)  // cu_seqlens in
    return fail(MOBA_ERR_CUDA);
  {
    SeqLayout L{pr.cu, pr.nseq, pr.N, pr.T};
    Timed tm(kKPlan, st);
    plan_kernel<<<1, 1024, 0, st>>>(L, pr.B, w.P, (int)pr.NBmax, (int)pr.NQTmax, w.status);
  }
  if (cudaMemsetAsync(w.counts, 0, sizeof(uint32_t) * (size_t)pr.Hkv * pr.NBmax, st) !=
      cudaSuccess)
    return fail(MOBA_ERR_CUDA);
  for (int p = 0; p < npass; ++p) {
    const int g0 = p * nu_max, ng = (pr.Hkv - g0) < nu_max ? (pr.Hkv - g0) : nu_max;
    if (cudaStreamWaitEvent(st, in_ready(p), 0) != cudaSuccess) return fail(MOBA_ERR_CUDA);
    if ((r = run_pool(pr, hb.k, w, st, g0, ng)) != MOBA_OK) return fail(r);
    if ((r = run_vbound(pr, hb.v, w, st, g0, ng)) != MOBA_OK) return fail(r);
    if ((r = launch_gate<D>(pr, hb.q, w, hb.sel, w.counts, st, g0, ng)) != MOBA_OK) return fail(r);
    if ((r = forward_one_pass<D>(pr, c, w, hb.sel, hb.o, hb.lse, g0, ng, st)) != MOBA_OK)
      return fail(r);
    if (cudaEventRecord(done(p), st) != cudaSuccess ||
        cudaStreamWaitEvent(d2h, done(p), 0) != cudaSuccess)
      return fail(MOBA_ERR_CUDA);
    const int64_t h0 = (int64_t)g0 * pr.G, nh = (int64_t)ng * pr.G;
    if (copy_cols(o_h, hb.o, pr.T, (int64_t)pr.Hq * D, h0 * D, nh * D, 2,
                  cudaMemcpyDeviceToHost, d2h) != cudaSuccess ||
        copy_cols(lse_h, hb.lse, rows_b, (int64_t)pr.Hq * per_head_lse, h0 * per_head_lse,
                  nh * per_head_lse, 4, cudaMemcpyDeviceToHost, d2h) != cudaSuccess ||
        (sel_h && copy_cols(sel_h, hb.sel, rows_b, (int64_t)pr.Hq * per_head_sel,
                            h0 * per_head_sel, nh * per_head_sel, 4, cudaMemcpyDeviceToHost,
                            d2h) != cudaSuccess))
      return fail(MOBA_ERR_CUDA);
  }
  // the caller's stream covers the output copies
  if (cudaEventRecord(start, d2h) != cudaSuccess || cudaStreamWaitEvent(st, start, 0) != cudaSuccess)
    return fail(MOBA_ERR_CUDA);
  return fail(MOBA_OK);
}

moba_status forward_impl(const Problem& pr, const void* q, const void* k, const void* v, void* o,
                         float* lse, int32_t* sel_out, void* ws, size_t ws_bytes,
                         cudaStream_t st, int route = kRouteMeanGate) {
  if (!q || !k || !v || !o || !lse) return MOBA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(lse) & 3) || (reinterpret_cast<uintptr_t>(sel_out) & 3))
    return MOBA_ERR_INVALID_ARG;
  if (!topk_supported(pr)) return MOBA_ERR_UNSUPPORTED;
  // per-pass entry indices are int32
  if ((int64_t)pr.T * pr.G * (pr.topk > 1 ? pr.topk - 1 : 1) >= INT32_MAX)
    return MOBA_ERR_UNSUPPORTED;
  const Ws need = carve(pr, 1, nullptr);
  MOBA_TRY(check_ws(ws, ws_bytes, need.bytes));
  if (pr.T == 0) return MOBA_OK;
  int nu = 1;
  while (nu < pr.Hkv && carve(pr, nu + 1, nullptr).bytes <= ws_bytes &&
         (int64_t)(nu + 1) * pr.T * pr.G * (pr.topk > 1 ? pr.topk - 1 : 1) < INT32_MAX)
    ++nu;
  const Ws w = carve(pr, nu, static_cast<char*>(ws));
  int32_t* sel = sel_out ? sel_out : w.sel;
  if (route == kRouteGiven && !sel_out) return MOBA_ERR_INVALID_ARG;
  if (route == kRouteMeanGate)
    MOBA_TRY(run_plan_pool(pr, k, w, st));
  else if (route == kRouteMinmaxGate) {
    MOBA_TRY(run_plan(pr, w, st));
    MOBA_TRY(run_minmax_pool(pr, k, w, st));
  } else {
    MOBA_TRY(run_plan(pr, w, st));
  }
  MOBA_TRY(run_vbound(pr, v, w, st, 0, pr.Hkv));
  return pr.D == 128 ? forward_passes<128>(pr, q, k, v, o, lse, w, sel, nu, route, st)
                     : forward_passes<64>(pr, q, k, v, o, lse, w, sel, nu, route, st);
}

size_t dense_ws_bytes(int64_t T, int nseq) {
  Problem pr;
  memset(&pr, 0, sizeof pr);
  pr.nseq = nseq;
  pr.T = 0;
  pr.NBmax = T / kTileM + nseq;
  pr.NQTmax = pr.NBmax;
  pr.Hkv = 1;
  pr.Hq = 1;
  pr.G = 1;
  pr.D = 64;
  pr.topk = 1;
  // status + plan arrays only: kbar/sel/partials are sized by T = 0 and Hkv = 1
  return carve(pr, 1, nullptr).bytes + align_up(sizeof(float) * 64 * (size_t)pr.NBmax);
}

moba_status dense_impl(const Problem& pr, const void* q, const void* k, const void* v, void* o,
                       float* lse, void* ws, size_t ws_bytes, cudaStream_t st) {
  if (!q || !k || !v || !o || !lse) return MOBA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(lse) & 3))
    return MOBA_ERR_INVALID_ARG;
  MOBA_TRY(check_ws(ws, ws_bytes, dense_ws_bytes(pr.T, pr.nseq)));
  if (pr.T == 0) return MOBA_OK;
  // plan only needs status + plan arrays; carve them from a T = 0 view
  Problem pv = pr;
  pv.T = 0;
  pv.Hkv = 1;
  pv.Hq = 1;
  pv.G = 1;
  pv.D = 64;
  pv.topk = 1;
  const Ws w = carve(pv, 1, static_cast<char*>(ws));
  SeqLayout L{pr.cu, pr.nseq, pr.N, pr.T};
  {
    Timed tm(kKPlan, st);
    plan_kernel<<<1, 1024, 0, st>>>(L, pr.B, w.P, (int)pr.NBmax, (int)pr.NQTmax, w.status);
  }
  MOBA_CUDA(cudaGetLastError());
  CUtensorMap tq, tk, tv;
  if (!make_tmap(&tq, q, pr.Hq, pr.T, pr.D) || !make_tmap(&tk, k, pr.Hkv, pr.T, pr.D) ||
      !make_tmap(&tv, v, pr.Hkv, pr.T, pr.D))
    return MOBA_ERR_CUDA;
  AttnArgs a;
  memset(&a, 0, sizeof a);
  a.q = reinterpret_cast<const __nv_bfloat16*>(q);
  a.Hq = pr.Hq;
  a.Hkv = pr.Hkv;
  a.G = pr.G;
  a.B = pr.B;
  a.topk = 1;
  a.scale_log2 = pr.scale * 1.4426950408889634f;
  a.L = L;
  a.P = w.P;
  a.R = pr.R;
  a.o = reinterpret_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.status = w.status;
  a.u0 = 0;
  a.nu = pr.Hkv;
  return pr.D == 128 ? launch_attn<128, kDense>(tq, tk, tv, a, 1, st)
                     : launch_attn<64, kDense>(tq, tk, tv, a, 1, st);
}

// One thread waits, with the pipelines' bounded wait and a short limit, on a
// barrier nothing ever arrives on.  The wait must give up, raise the timeout
// bit in the status word and let the kernel return.
__global__ void wait_selftest_kernel(uint32_t* status, long long limit_cycles) {
  __shared__ uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  abort_flag = 0u;
  fence_barrier_init();
  mbar_wait(&bar, 0, &abort_flag, status, limit_cycles);
}

// ---------------------------------------------------------------- backward
struct BwWs {
  Ws w;  // status, plan, counts, buckets and entries, as the forward's
  float2* dl;
  float* dq32;
  float* dk32;
  float* dv32;
  size_t bytes;
};

BwWs carve_bw(const Problem& pr, int nu, char* base) {
  BwWs b;
  memset(&b, 0, sizeof b);
  size_t off = 0;
  auto take = [&](size_t bytes) -> char* {
    char* p = base ? base + off : nullptr;
    off = align_up(off + bytes);
    return p;
  };
  const int64_t NB = pr.NBmax;
  const int64_t np = pr.topk > 1 ? pr.topk - 1 : 0;
  Ws& w = b.w;
  w.status = reinterpret_cast<uint32_t*>(take(kAlign));
  w.P.totals = reinterpret_cast<int32_t*>(take(4 * sizeof(int32_t)));
  w.P.blk_off = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (pr.nseq + 1)));
  w.P.qt_off = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (pr.nseq + 1)));
  w.P.pair_off = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (pr.nseq + 1)));
  w.P.blk_tok = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * NB));
  w.P.blk_len = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * NB));
  w.counts = reinterpret_cast<uint32_t*>(take(sizeof(uint32_t) * (size_t)pr.Hkv * NB));
  w.entry_off = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * ((size_t)nu * NB + 1)));
  w.tile_off = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * ((size_t)nu * NB + 1)));
  w.cursor = reinterpret_cast<uint32_t*>(take(sizeof(uint32_t) * (size_t)nu * NB));
  w.entries = reinterpret_cast<uint2*>(take(sizeof(uint2) * (size_t)nu * pr.T * pr.G * np));
  b.dl = reinterpret_cast<float2*>(take(sizeof(float2) * (size_t)pr.T * pr.Hq));
  b.dq32 = reinterpret_cast<float*>(take(sizeof(float) * (size_t)pr.T * pr.Hq * pr.D));
  b.dk32 = reinterpret_cast<float*>(take(sizeof(float) * (size_t)pr.T * pr.Hkv * pr.D));
  b.dv32 = reinterpret_cast<float*>(take(sizeof(float) * (size_t)pr.T * pr.Hkv * pr.D));
  b.bytes = off;
  return b;
}

template <int D>
moba_status backward_passes(const Problem& pr, const void* q, const void* k, const void* v,
                            const void* o, const float* lse, const void* dO, const int32_t* sel,
                            void* dq, void* dk, void* dv, const BwWs& b, int nu_max,
                            cudaStream_t st) {
  const Ws& w = b.w;
  SeqLayout L{pr.cu, pr.nseq, pr.N, pr.T};
  MOBA_TRY(run_plan(pr, w, st));
  if (pr.topk > 1) {
    MOBA_CUDA(cudaMemsetAsync(w.counts, 0, sizeof(uint32_t) * (size_t)pr.Hkv * pr.NBmax, st));
    MOBA_TRY(launch_count(pr, w, sel, w.counts, st));
  }
  MOBA_CUDA(cudaMemsetAsync(b.dq32, 0, sizeof(float) * (size_t)pr.T * pr.Hq * D, st));
  MOBA_CUDA(cudaMemsetAsync(b.dk32, 0, sizeof(float) * (size_t)pr.T * pr.Hkv * D, st));
  MOBA_CUDA(cudaMemsetAsync(b.dv32, 0, sizeof(float) * (size_t)pr.T * pr.Hkv * D, st));
  {
    Timed tm(kKBwPrep, st);
    const int64_t rows = pr.T * pr.Hq;
    bw_prep_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(o), reinterpret_cast<const __nv_bfloat16*>(dO),
        lse, pr.Hq, L, pr.R, b.dl);
    MOBA_CUDA(cudaGetLastError());
  }
  CUtensorMap tk, tv;
  if (!make_tmap(&tk, k, pr.Hkv, pr.T, D) || !make_tmap(&tv, v, pr.Hkv, pr.T, D))
    return MOBA_ERR_CUDA;
  using C2 = BwKv2Cfg<D>;
  MOBA_CUDA(cudaFuncSetAttribute(bw_kv2_kernel<D, kBwRouted>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, C2::kSmemBytes));
  MOBA_CUDA(cudaFuncSetAttribute(bw_kv2_kernel<D, kBwOwn>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, C2::kSmemBytes));
  using C3 = BwQ2Cfg<D>;
  MOBA_CUDA(cudaFuncSetAttribute(bw_q2_kernel<D, kBwRouted>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, C3::kSmemBytes));
  MOBA_CUDA(cudaFuncSetAttribute(bw_q2_kernel<D, kBwOwn>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, C3::kSmemBytes));
  BwArgs a;
  memset(&a, 0, sizeof a);
  a.q = reinterpret_cast<const __nv_bfloat16*>(q);
  a.dO = reinterpret_cast<const __nv_bfloat16*>(dO);
  a.dl = b.dl;
  a.dq32 = b.dq32;
  a.dk32 = b.dk32;
  a.dv32 = b.dv32;
  a.entry_off = w.entry_off;
  a.tile_off = w.tile_off;
  a.entries = w.entries;
  a.Hq = pr.Hq;
  a.Hkv = pr.Hkv;
  a.G = pr.G;
  a.B = pr.B;
  a.NBmax = (int)pr.NBmax;
  a.scale = pr.scale;
  a.scale_log2 = pr.scale * 1.4426950408889634f;
  a.L = L;
  a.P = w.P;
  a.status = w.status;
  const int64_t KT = pr.B / kTileN;
  const int64_t np = pr.topk > 1 ? pr.topk - 1 : 0;
  for (int u0 = 0; u0 < pr.Hkv; u0 += nu_max) {
    const int nu = (pr.Hkv - u0) < nu_max ? (pr.Hkv - u0) : nu_max;
    a.u0 = u0;
    a.nu = nu;
    if (pr.topk > 1) {
      {
        Timed tm(kKScan, st);
        bucket_scan_kernel<<<1, 1024, 0, st>>>(w.counts, u0, nu, kTileM, w.P, (int)pr.NBmax,
                                               w.entry_off, w.tile_off, w.cursor);
      }
      MOBA_CUDA(cudaGetLastError());
      MOBA_TRY(launch_scatter(pr, w, sel, u0, nu, st));
      {
        Timed tm(kKBwKv, st);
        bw_kv2_kernel<D, kBwRouted>
            <<<(unsigned)(nu * pr.NBmax * KT), C2::kThreads, C2::kSmemBytes, st>>>(tk, tv, a);
        MOBA_CUDA(cudaGetLastError());
      }
      {
        const int64_t items = (int64_t)nu * pr.T * pr.G * np / kTileM + (int64_t)nu * pr.NBmax;
        Timed tm(kKBwQ, st);
        bw_q2_kernel<D, kBwRouted><<<(unsigned)items, C3::kThreads, C3::kSmemBytes, st>>>(tk, tv, a);
        MOBA_CUDA(cudaGetLastError());
      }
    }
    {
      Timed tm(kKBwKv, st);
      bw_kv2_kernel<D, kBwOwn>
          <<<(unsigned)(nu * pr.NBmax * KT), C2::kThreads, C2::kSmemBytes, st>>>(tk, tv, a);
      MOBA_CUDA(cudaGetLastError());
    }
    {
      Timed tm(kKBwQ, st);
      bw_q2_kernel<D, kBwOwn>
          <<<(unsigned)(nu * pr.G * pr.NQTmax), C3::kThreads, C3::kSmemBytes, st>>>(tk, tv, a);
      MOBA_CUDA(cudaGetLastError());
    }
  }
  Timed tm(kKBwFinish, st);
  const int64_t nq = pr.T * pr.Hq * D, nk = pr.T * pr.Hkv * D;
  bw_finish_kernel<<<(unsigned)((nq / 4 + 255) / 256 + 1), 256, 0, st>>>(
      b.dq32, static_cast<__nv_bfloat16*>(dq), nq);
  bw_finish_kernel<<<(unsigned)((nk / 4 + 255) / 256 + 1), 256, 0, st>>>(
      b.dk32, static_cast<__nv_bfloat16*>(dk), nk);
  bw_finish_kernel<<<(unsigned)((nk / 4 + 255) / 256 + 1), 256, 0, st>>>(
      b.dv32, static_cast<__nv_bfloat16*>(dv), nk);
  return cuda_status(cudaGetLastError());
}

moba_status backward_impl(const Problem& pr, const void* q, const void* k, const void* v,
                          const void* o, const float* lse, const void* dO, const int32_t* sel,
                          void* dq, void* dk, void* dv, void* ws, size_t ws_bytes,
                          cudaStream_t st) {
  if (!q || !k || !v || !o || !lse || !dO || !sel || !dq || !dk || !dv)
    return MOBA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dO) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      (reinterpret_cast<uintptr_t>(lse) & 3) || (reinterpret_cast<uintptr_t>(sel) & 3))
    return MOBA_ERR_INVALID_ARG;
  if (!topk_supported(pr)) return MOBA_ERR_UNSUPPORTED;
  if ((int64_t)pr.T * pr.G * (pr.topk > 1 ? pr.topk - 1 : 1) >= INT32_MAX)
    return MOBA_ERR_UNSUPPORTED;
  MOBA_TRY(check_ws(ws, ws_bytes, carve_bw(pr, 1, nullptr).bytes));
  if (pr.T == 0) return MOBA_OK;
  int nu = 1;
  while (nu < pr.Hkv && carve_bw(pr, nu + 1, nullptr).bytes <= ws_bytes &&
         (int64_t)(nu + 1) * pr.T * pr.G * (pr.topk > 1 ? pr.topk - 1 : 1) < INT32_MAX)
    ++nu;
  const BwWs b = carve_bw(pr, nu, static_cast<char*>(ws));
  return pr.D == 128 ? backward_passes<128>(pr, q, k, v, o, lse, dO, sel, dq, dk, dv, b, nu, st)
                     : backward_passes<64>(pr, q, k, v, o, lse, dO, sel, dq, dk, dv, b, nu, st);
}

// ---------------------------------------------------------------- decode
struct DecodeShape {
  int b, cap, Hq, Hkv, G, D, B, topk, nbcap, nchunk;
  float scale;
};

moba_status make_decode_shape(const moba_decode_params* p, DecodeShape* out) {
  if (!p) return MOBA_ERR_INVALID_ARG;
  DecodeShape d;
  if (p->batch <= 0 || p->cache_len <= 0 || p->num_q_heads <= 0 || p->num_kv_heads <= 0 ||
      p->num_q_heads % p->num_kv_heads || p->block_size <= 0 || p->top_k <= 0)
    return MOBA_ERR_INVALID_ARG;
  if (p->head_dim != 64 && p->head_dim != 128) return MOBA_ERR_UNSUPPORTED;
  if (p->block_size % kTileM) return MOBA_ERR_UNSUPPORTED;
  if (p->top_k > 65) return MOBA_ERR_UNSUPPORTED;  // at most 64 ranked past blocks
  d.b = p->batch;
  d.cap = p->cache_len;
  d.Hq = p->num_q_heads;
  d.Hkv = p->num_kv_heads;
  d.G = d.Hq / d.Hkv;
  d.D = p->head_dim;
  d.B = p->block_size;
  d.topk = p->top_k;
  const int64_t nb = ((int64_t)d.cap + d.B - 1) / d.B;
  if (nb > kDecodeMaxBlocks) return MOBA_ERR_UNSUPPORTED;
  if ((int64_t)d.b * d.cap * d.Hkv * d.D >= (int64_t(1) << 40)) return MOBA_ERR_UNSUPPORTED;
  if ((int64_t)d.b * d.Hq > 65535 * 1024) return MOBA_ERR_UNSUPPORTED;
  d.nbcap = (int)nb;
  d.nchunk = (d.B + kDecodeChunk - 1) / kDecodeChunk;
  if (d.b > 65535 || d.Hkv > 65535) return MOBA_ERR_UNSUPPORTED;          // grid y / z
  if ((int64_t)d.topk * d.nchunk > kDecodeMaxParts) return MOBA_ERR_UNSUPPORTED;  // merge staging
  d.scale = (p->softmax_scale > 0.f) ? p->softmax_scale : 1.0f / sqrtf((float)d.D);
  if (!(d.scale < INFINITY)) return MOBA_ERR_INVALID_ARG;
  *out = d;
  return MOBA_OK;
}

struct DecodeWs {
  uint32_t* status;
  int32_t* sel;
  float* part;
  float* kpart;  // block-mean partial sums [b][Hkv][nbcap][B / 128][D]
  size_t bytes;
};

DecodeWs carve_decode(const DecodeShape& d, char* base) {
  DecodeWs w;
  size_t off = 0;
  auto take = [&](size_t bytes) -> char* {
    char* p = base ? base + off : nullptr;
    off = align_up(off + bytes);
    return p;
  };
  w.status = reinterpret_cast<uint32_t*>(take(kAlign));
  w.sel = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (size_t)d.b * d.Hq * d.topk));
  w.part = reinterpret_cast<float*>(
      take(sizeof(float) * (size_t)d.b * d.Hq * d.topk * d.nchunk * (d.D + 2)));
  w.kpart = reinterpret_cast<float*>(take(sizeof(float) * (size_t)d.b * d.Hkv * d.nbcap *
                                          (d.B / kKbarRows) * d.D));
  w.bytes = off;
  return w;
}

DecodeArgs decode_args(const DecodeShape& d, const DecodeWs& w, const void* q, const void* kc,
                       const void* vc, const int32_t* lens, float* kbar) {
  DecodeArgs a;
  memset(&a, 0, sizeof a);
  a.q = reinterpret_cast<const __nv_bfloat16*>(q);
  a.kc = reinterpret_cast<const __nv_bfloat16*>(kc);
  a.vc = reinterpret_cast<const __nv_bfloat16*>(vc);
  a.lens = lens;
  a.kbar = kbar;
  a.sel = w.sel;
  a.part = w.part;
  a.batch = d.b;
  a.cap = d.cap;
  a.Hq = d.Hq;
  a.Hkv = d.Hkv;
  a.G = d.G;
  a.B = d.B;
  a.topk = d.topk;
  a.nbcap = d.nbcap;
  a.nchunk = d.nchunk;
  a.scale_log2 = d.scale * 1.4426950408889634f;
  a.status = w.status;
  return a;
}

template <int D>
moba_status kbar_update_impl(const DecodeShape& d, const DecodeArgs& a, float* kpart,
                             int only_last, cudaStream_t st) {
  const unsigned nsel = only_last ? 1u : (unsigned)d.nbcap;
  const unsigned S = (unsigned)(d.B / kKbarRows);
  Timed tm(kKKbarCache, st);
  kbar_part_kernel<D><<<dim3(nsel * S, (unsigned)d.Hkv, (unsigned)d.b), 128, 0, st>>>(
      a, only_last, kpart);
  MOBA_CUDA(cudaGetLastError());
  kbar_reduce_kernel<D><<<dim3(nsel, (unsigned)d.Hkv, (unsigned)d.b), D, 0, st>>>(a, only_last,
                                                                                kpart);
  return cuda_status(cudaGetLastError());
}

template <int D>
moba_status decode_impl(const DecodeShape& d, DecodeArgs a, cudaStream_t st) {
  const size_t gsmem = sizeof(float) * (size_t)d.nbcap;
  {
    Timed tm(kKDecGate, st);
    decode_gate_kernel<D><<<dim3((unsigned)d.Hq, (unsigned)d.b), 256, gsmem, st>>>(a);
    MOBA_CUDA(cudaGetLastError());
  }
  {
    Timed tm(kKDecAttn, st);
    decode_attn_kernel<D>
        <<<dim3((unsigned)(d.b * d.Hq), (unsigned)d.topk, (unsigned)d.nchunk), 128, 0, st>>>(a);
    MOBA_CUDA(cudaGetLastError());
  }
  {
    Timed tm(kKDecMerge, st);
    decode_merge_kernel<D><<<(unsigned)(d.b * d.Hq), D, 0, st>>>(a);
    MOBA_CUDA(cudaGetLastError());
  }
  return MOBA_OK;
}

}  // namespace

extern "C" {

moba_status moba_selftest_wait_timeout(void* ws, size_t ws_bytes, long long limit_cycles,
                                       moba_stream_t stream) {
  if (limit_cycles <= 0 || limit_cycles > MOBA_WAIT_LIMIT_CYCLES) return MOBA_ERR_INVALID_ARG;
  if (!ws) {  // the allocation-free gate's status word
    MOBA_TRY(gate_scratch_address(&ws));
    ws_bytes = kAlign;
  }
  if ((reinterpret_cast<uintptr_t>(ws) % kAlign) || ws_bytes < kAlign)
    return MOBA_ERR_WORKSPACE;
  wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<uint32_t*>(ws), limit_cycles);
  return cuda_status(cudaGetLastError());
}

size_t moba_workspace_size(const moba_params* p, int heads_per_pass) {
  Problem pr;
  if (make_problem(p, false, nullptr, 0, 0, true, &pr) != MOBA_OK) return 0;
  int nu = (heads_per_pass <= 0 || heads_per_pass > pr.Hkv) ? pr.Hkv : heads_per_pass;
  return carve(pr, nu, nullptr).bytes;
}

size_t moba_workspace_size_varlen(const moba_params* p, int64_t total_tokens, int num_seqs,
                                  int heads_per_pass) {
  Problem pr;
  static const int32_t dummy = 0;
  if (make_problem(p, true, &dummy, num_seqs, total_tokens, true, &pr) != MOBA_OK) return 0;
  int nu = (heads_per_pass <= 0 || heads_per_pass > pr.Hkv) ? pr.Hkv : heads_per_pass;
  return carve(pr, nu, nullptr).bytes;
}

moba_status moba_gate(const void* q, const void* k, int32_t* sel, const moba_params* p, void* ws,
                      size_t ws_bytes, moba_stream_t stream) {
  Problem pr;
  MOBA_TRY(make_problem(p, false, nullptr, 0, 0, true, &pr));
  return gate_impl(pr, q, k, sel, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

moba_status moba_gate_varlen(const void* q, const void* k, const int32_t* cu_seqlens,
                             int num_seqs, int64_t total_tokens, int32_t* sel,
                             const moba_params* p, void* ws, size_t ws_bytes,
                             moba_stream_t stream) {
  Problem pr;
  MOBA_TRY(make_problem(p, true, cu_seqlens, num_seqs, total_tokens, true, &pr));
  return gate_impl(pr, q, k, sel, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

moba_status moba_forward(const void* q, const void* k, const void* v, void* o, float* lse,
                         int32_t* sel_out, const moba_params* p, void* ws, size_t ws_bytes,
                         moba_stream_t stream) {
  Problem pr;
  MOBA_TRY(make_problem(p, false, nullptr, 0, 0, true, &pr));
  return forward_impl(pr, q, k, v, o, lse, sel_out, ws, ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream));
}

moba_status moba_forward_varlen(const void* q, const void* k, const void* v,
                                const int32_t* cu_seqlens, int num_seqs, int64_t total_tokens,
                                void* o, float* lse, int32_t* sel_out, const moba_params* p,
                                void* ws, size_t ws_bytes, moba_stream_t stream) {
  Problem pr;
  MOBA_TRY(make_problem(p, true, cu_seqlens, num_seqs, total_tokens, true, &pr));
  return forward_impl(pr, q, k, v, o, lse, sel_out, ws, ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream));
}

size_t moba_full_causal_workspace_size(int64_t total_tokens, int num_seqs) {
  if (total_tokens < 0 || num_seqs <= 0) return 0;
  return dense_ws_bytes(total_tokens, num_seqs);
}

moba_status moba_full_causal(const void* q, const void* k, const void* v, void* o, float* lse,
                             const moba_params* p, void* ws, size_t ws_bytes,
                             moba_stream_t stream) {
  Problem pr;
  MOBA_TRY(make_problem(p, false, nullptr, 0, 0, false, &pr));
  return dense_impl(pr, q, k, v, o, lse, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

moba_status moba_full_causal_varlen(const void* q, const void* k, const void* v,
                                    const int32_t* cu_seqlens, int num_seqs,
                                    int64_t total_tokens, void* o, float* lse,
                                    const moba_params* p, void* ws, size_t ws_bytes,
                                    moba_stream_t stream) {
  Problem pr;
  MOBA_TRY(make_problem(p, true, cu_seqlens, num_seqs, total_tokens, false, &pr));
  return dense_impl(pr, q, k, v, o, lse, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

moba_status moba_last_device_status(void* ws, moba_stream_t stream) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) % kAlign)) return MOBA_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, ws, sizeof word, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return MOBA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOBA_ERR_CUDA;
  if (cudaMemsetAsync(ws, 0, sizeof word, st) != cudaSuccess) return MOBA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOBA_ERR_CUDA;
  if (word & MOBA_DEV_TIMEOUT) return MOBA_ERR_TIMEOUT;
  if (word) return MOBA_ERR_DEVICE_CHECK;
  return MOBA_OK;
}

const char* moba_status_string(moba_status s) {
  switch (s) {
    case MOBA_OK: return "MOBA_OK";
    case MOBA_ERR_INVALID_ARG: return "MOBA_ERR_INVALID_ARG";
    case MOBA_ERR_UNSUPPORTED: return "MOBA_ERR_UNSUPPORTED";
    case MOBA_ERR_WORKSPACE: return "MOBA_ERR_WORKSPACE";
    case MOBA_ERR_CUDA: return "MOBA_ERR_CUDA";
    case MOBA_ERR_TIMEOUT: return "MOBA_ERR_TIMEOUT";
    case MOBA_ERR_DEVICE_CHECK: return "MOBA_ERR_DEVICE_CHECK";
  }
  return "MOBA_ERR_UNKNOWN";
}

int moba_version(void) { return 100; }

const char* moba_last_error_string(void) { return g_last_cuda_error; }

void moba_profile_enable(int on) { timer().on = (on != 0); }

void moba_profile_reset(void) {
  KernelTimer& t = timer();
  for (auto& p : t.pending) {
    cudaEventDestroy(p.a);
    cudaEventDestroy(p.b);
  }
  t.pending.clear();
  for (int c = 0; c < kKNum; ++c) {
    t.launches[c] = 0;
    t.ms[c] = 0.0;
  }
}

int moba_profile_read(moba_kernel_time* out, int max_entries) {
  KernelTimer& t = timer();
  for (auto& p : t.pending) {
    float ms = 0.f;
    if (cudaEventSynchronize(p.b) == cudaSuccess && cudaEventElapsedTime(&ms, p.a, p.b) == cudaSuccess) {
      t.launches[p.cls] += 1;
      t.ms[p.cls] += ms;
    }
    cudaEventDestroy(p.a);
    cudaEventDestroy(p.b);
  }
  t.pending.clear();
  int n = 0;
  for (int c = 0; c < kKNum && n < max_entries; ++c) {
    if (!out) break;
    strncpy(out[n].name, kKernelNames[c], sizeof(out[n].name) - 1);
    out[n].name[sizeof(out[n].name) - 1] = 0;
    out[n].launches = t.launches[c];
    out[n].total_ms = t.ms[c];
    ++n;
  }
  return n;
}

// ---------------------------------------------------------------- routing variants
moba_status gate_minmax_impl(const Problem& pr, const void* q, const void* k, int32_t* sel,
                             void* ws, size_t ws_bytes, moba_stream_t stream);

moba_status moba_gate_minmax(const void* q, const void* k, int32_t* sel, const moba_params* p,
                             void* ws, size_t ws_bytes, moba_stream_t stream) {
  Problem pr;
  MOBA_TRY(make_problem(p, false, nullptr, 0, 0, true, &pr));
  return gate_minmax_impl(pr, q, k, sel, ws, ws_bytes, stream);
}

moba_status moba_gate_minmax_varlen(const void* q, const void* k, const int32_t* cu_seqlens,
                                    int num_seqs, int64_t total_tokens, int32_t* sel,
                                    const moba_params* p, void* ws, size_t ws_bytes,
                                    moba_stream_t stream) {
  Problem pr;
  MOBA_TRY(make_problem(p, true, cu_seqlens, num_seqs, total_tokens, true, &pr));
  return gate_minmax_impl(pr, q, k, sel, ws, ws_bytes, stream);
}

moba_status gate_minmax_impl(const Problem& pr, const void* q, const void* k, int32_t* sel,
                             void* ws, size_t ws_bytes, moba_stream_t stream) {
  if (!q || !k || !sel || !aligned16(q) || !aligned16(k) ||
      (reinterpret_cast<uintptr_t>(sel) & 3))
    return MOBA_ERR_INVALID_ARG;
  if (!topk_supported(pr)) return MOBA_ERR_UNSUPPORTED;
  MOBA_TRY(check_ws(ws, ws_bytes, carve(pr, 1, nullptr).bytes));
  if (pr.T == 0) return MOBA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const Ws w = carve(pr, 1, static_cast<char*>(ws));
  MOBA_TRY(run_plan(pr, w, st));
  MOBA_TRY(run_minmax_pool(pr, k, w, st));
  return pr.D == 128 ? launch_gate_minmax<128>(pr, q, w, sel, nullptr, st)
                     : launch_gate_minmax<64>(pr, q, w, sel, nullptr, st);
}

moba_status static_selection_impl(const Problem& pr, int32_t* sel, int mode,
                                  cudaStream_t st) {
  if (!sel || (reinterpret_cast<uintptr_t>(sel) & 3)) return MOBA_ERR_INVALID_ARG;
  if (mode != MOBA_ROUTE_WINDOW && mode != MOBA_ROUTE_SINK) return MOBA_ERR_INVALID_ARG;
  const int64_t rows = pr.T * pr.Hq;
  if (rows == 0) return MOBA_OK;
  SeqLayout L{pr.cu, pr.nseq, pr.N, pr.T};
  Timed tm(kKStaticSel, st);
  static_select_kernel<<<(unsigned)((rows + 255) / 256), 256, 0, st>>>(
      sel, rows, L, pr.Hq, pr.B, pr.topk, mode == MOBA_ROUTE_SINK ? kRouteSink : kRouteWindow);
  return cuda_status(cudaGetLastError());
}

moba_status moba_static_selection(int32_t* sel, int mode, const moba_params* p,
                                  moba_stream_t stream) {
  Problem pr;
  MOBA_TRY(make_problem(p, false, nullptr, 0, 0, true, &pr));
  return static_selection_impl(pr, sel, mode, reinterpret_cast<cudaStream_t>(stream));
}

moba_status moba_static_selection_varlen(int32_t* sel, int mode, const int32_t* cu_seqlens,
                                         int num_seqs, int64_t total_tokens,
                                         const moba_params* p, moba_stream_t stream) {
  Problem pr;
  MOBA_TRY(make_problem(p, true, cu_seqlens, num_seqs, total_tokens, true, &pr));
  return static_selection_impl(pr, sel, mode, reinterpret_cast<cudaStream_t>(stream));
}

moba_status moba_forward_selected(const void* q, const void* k, const void* v, void* o,
                                  float* lse, const int32_t* sel, const moba_params* p,
                                  void* ws, size_t ws_bytes, moba_stream_t stream) {
  Problem pr;
  MOBA_TRY(make_problem(p, false, nullptr, 0, 0, true, &pr));
  if (!sel) return MOBA_ERR_INVALID_ARG;
  return forward_impl(pr, q, k, v, o, lse, const_cast<int32_t*>(sel), ws, ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream), kRouteGiven);
}

moba_status moba_forward_minmax(const void* q, const void* k, const void* v, void* o,
                                float* lse, int32_t* sel_out, const moba_params* p, void* ws,
                                size_t ws_bytes, moba_stream_t stream) {
  Problem pr;
  MOBA_TRY(make_problem(p, false, nullptr, 0, 0, true, &pr));
  return forward_impl(pr, q, k, v, o, lse, sel_out, ws, ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream), kRouteMinmaxGate);
}

moba_status moba_forward_selected_varlen(const void* q, const void* k, const void* v,
                                         const int32_t* cu_seqlens, int num_seqs,
                                         int64_t total_tokens, void* o, float* lse,
                                         const int32_t* sel, const moba_params* p, void* ws,
                                         size_t ws_bytes, moba_stream_t stream) {
  Problem pr;
  MOBA_TRY(make_problem(p, true, cu_seqlens, num_seqs, total_tokens, true, &pr));
  if (!sel) return MOBA_ERR_INVALID_ARG;
  return forward_impl(pr, q, k, v, o, lse, const_cast<int32_t*>(sel), ws, ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream), kRouteGiven);
}

moba_status moba_forward_minmax_varlen(const void* q, const void* k, const void* v,
                                       const int32_t* cu_seqlens, int num_seqs,
                                       int64_t total_tokens, void* o, float* lse,
                                       int32_t* sel_out, const moba_params* p, void* ws,
                                       size_t ws_bytes, moba_stream_t stream) {
  Problem pr;
  MOBA_TRY(make_problem(p, true, cu_seqlens, num_seqs, total_tokens, true, &pr));
  return forward_impl(pr, q, k, v, o, lse, sel_out, ws, ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream), kRouteMinmaxGate);
}

// ---------------------------------------------------------------- host-buffer forward
size_t moba_forward_host_buffer_size(const moba_params* p, int heads_per_pass) {
  Problem pr;
  if (make_problem(p, false, nullptr, 0, 0, true, &pr) != MOBA_OK) return 0;
  int nu = (heads_per_pass <= 0 || heads_per_pass > pr.Hkv) ? pr.Hkv : heads_per_pass;
  const size_t ws = carve(pr, nu, nullptr).bytes;
  return align_up(ws) + carve_host(pr, nullptr, ws).staged;
}

moba_status forward_host_impl(Problem pr, const void* q, const void* k, const void* v, void* o,
                              float* lse, int32_t* sel_out, const int32_t* cu_h, void* dev_buf,
                              size_t dev_bytes, moba_stream_t stream);

moba_status moba_forward_host(const void* q, const void* k, const void* v, void* o, float* lse,
                              int32_t* sel_out, const moba_params* p, void* dev_buf,
                              size_t dev_bytes, moba_stream_t stream) {
  Problem pr;
  MOBA_TRY(make_problem(p, false, nullptr, 0, 0, true, &pr));
  return forward_host_impl(pr, q, k, v, o, lse, sel_out, nullptr, dev_buf, dev_bytes, stream);
}

size_t moba_forward_host_buffer_size_varlen(const moba_params* p, int64_t total_tokens,
                                            int num_seqs, int heads_per_pass) {
  Problem pr;
  static const int32_t dummy = 0;
  if (make_problem(p, true, &dummy, num_seqs, total_tokens, true, &pr) != MOBA_OK) return 0;
  int nu = (heads_per_pass <= 0 || heads_per_pass > pr.Hkv) ? pr.Hkv : heads_per_pass;
  const size_t ws = carve(pr, nu, nullptr).bytes;
  return align_up(ws) + carve_host(pr, nullptr, ws).staged;
}

moba_status moba_forward_host_varlen(const void* q, const void* k, const void* v,
                                     const int32_t* cu_seqlens, int num_seqs,
                                     int64_t total_tokens, void* o, float* lse, int32_t* sel_out,
                                     const moba_params* p, void* dev_buf, size_t dev_bytes,
                                     moba_stream_t stream) {
  Problem pr;
  static const int32_t dummy = 0;  // replaced by the device copy below
  if (!cu_seqlens) return MOBA_ERR_INVALID_ARG;
  MOBA_TRY(make_problem(p, true, &dummy, num_seqs, total_tokens, true, &pr));
  return forward_host_impl(pr, q, k, v, o, lse, sel_out, cu_seqlens, dev_buf, dev_bytes, stream);
}

moba_status forward_host_impl(Problem pr, const void* q, const void* k, const void* v, void* o,
                              float* lse, int32_t* sel_out, const int32_t* cu_h, void* dev_buf,
                              size_t dev_bytes, moba_stream_t stream) {
  if (!q || !k || !v || !o || !lse) return MOBA_ERR_INVALID_ARG;
  if (!topk_supported(pr)) return MOBA_ERR_UNSUPPORTED;
  if ((int64_t)pr.T * pr.G * (pr.topk > 1 ? pr.topk - 1 : 1) >= INT32_MAX)
    return MOBA_ERR_UNSUPPORTED;
  if (!dev_buf || (reinterpret_cast<uintptr_t>(dev_buf) % kAlign)) return MOBA_ERR_WORKSPACE;
  const size_t staged = carve_host(pr, nullptr, 0).staged;
  auto need = [&](int n) { return align_up(carve(pr, n, nullptr).bytes) + staged; };
  if (dev_bytes < need(1)) return MOBA_ERR_WORKSPACE;
  if (pr.T == 0) return MOBA_OK;
  int nu = 1;
  while (nu < pr.Hkv && need(nu + 1) <= dev_bytes &&
         (int64_t)(nu + 1) * pr.T * pr.G * (pr.topk > 1 ? pr.topk - 1 : 1) < INT32_MAX)
    ++nu;
  const Ws w = carve(pr, nu, static_cast<char*>(dev_buf));
  const HostBufs hb = carve_host(pr, static_cast<char*>(dev_buf), w.bytes);
  if (pr.varlen) pr.cu = hb.cu;  // the kernels read the staged copy
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return pr.D == 128
             ? forward_host_passes<128>(pr, q, k, v, o, lse, sel_out, cu_h, hb, w, nu, st)
             : forward_host_passes<64>(pr, q, k, v, o, lse, sel_out, cu_h, hb, w, nu, st);
}

// ---------------------------------------------------------------- backward
size_t moba_backward_workspace_size(const moba_params* p, int heads_per_pass) {
  Problem pr;
  if (make_problem(p, false, nullptr, 0, 0, true, &pr) != MOBA_OK) return 0;
  int nu = (heads_per_pass <= 0 || heads_per_pass > pr.Hkv) ? pr.Hkv : heads_per_pass;
  return carve_bw(pr, nu, nullptr).bytes;
}

moba_status moba_backward(const void* q, const void* k, const void* v, const void* o,
                          const float* lse, const void* dO, const int32_t* sel, void* dq,
                          void* dk, void* dv, const moba_params* p, void* ws, size_t ws_bytes,
                          moba_stream_t stream) {
  Problem pr;
  MOBA_TRY(make_problem(p, false, nullptr, 0, 0, true, &pr));
  return backward_impl(pr, q, k, v, o, lse, dO, sel, dq, dk, dv, ws, ws_bytes,
                       reinterpret_cast<cudaStream_t>(stream));
}

size_t moba_backward_workspace_size_varlen(const moba_params* p, int64_t total_tokens,
                                           int num_seqs, int heads_per_pass) {
  Problem pr;
  static const int32_t dummy = 0;
  if (make_problem(p, true, &dummy, num_seqs, total_tokens, true, &pr) != MOBA_OK) return 0;
  int nu = (heads_per_pass <= 0 || heads_per_pass > pr.Hkv) ? pr.Hkv : heads_per_pass;
  return carve_bw(pr, nu, nullptr).bytes;
}

moba_status moba_backward_varlen(const void* q, const void* k, const void* v, const void* o,
                                 const float* lse, const void* dO, const int32_t* sel,
                                 const int32_t* cu_seqlens, int num_seqs, int64_t total_tokens,
                                 void* dq, void* dk, void* dv, const moba_params* p, void* ws,
                                 size_t ws_bytes, moba_stream_t stream) {
  Problem pr;
  MOBA_TRY(make_problem(p, true, cu_seqlens, num_seqs, total_tokens, true, &pr));
  return backward_impl(pr, q, k, v, o, lse, dO, sel, dq, dk, dv, ws, ws_bytes,
                       reinterpret_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------- decode
size_t moba_decode_workspace_size(const moba_decode_params* p) {
  DecodeShape d;
  if (make_decode_shape(p, &d) != MOBA_OK) return 0;
  return carve_decode(d, nullptr).bytes;
}

size_t moba_kbar_cache_size(const moba_decode_params* p) {
  DecodeShape d;
  if (make_decode_shape(p, &d) != MOBA_OK) return 0;
  return sizeof(float) * (size_t)d.b * d.Hkv * d.nbcap * d.D;
}

moba_status moba_kbar_cache_update(const void* k_cache, const int32_t* seqlens,
                                   float* kbar_cache, int only_last,
                                   const moba_decode_params* p, void* ws, size_t ws_bytes,
                                   moba_stream_t stream) {
  DecodeShape d;
  MOBA_TRY(make_decode_shape(p, &d));
  if (!k_cache || !seqlens || !kbar_cache || !aligned16(k_cache) || !aligned16(kbar_cache) ||
      (reinterpret_cast<uintptr_t>(seqlens) & 3))
    return MOBA_ERR_INVALID_ARG;
  MOBA_TRY(check_ws(ws, ws_bytes, carve_decode(d, nullptr).bytes));
  const DecodeWs w = carve_decode(d, static_cast<char*>(ws));
  const DecodeArgs a = decode_args(d, w, nullptr, k_cache, nullptr, seqlens, kbar_cache);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return d.D == 128 ? kbar_update_impl<128>(d, a, w.kpart, only_last ? 1 : 0, st)
                    : kbar_update_impl<64>(d, a, w.kpart, only_last ? 1 : 0, st);
}

moba_status moba_decode(const void* q, const void* k_cache, const void* v_cache,
                        const int32_t* seqlens, const float* kbar_cache, void* o, float* lse,
                        int32_t* sel_out, const moba_decode_params* p, void* ws,
                        size_t ws_bytes, moba_stream_t stream) {
  DecodeShape d;
  MOBA_TRY(make_decode_shape(p, &d));
  if (!q || !k_cache || !v_cache || !seqlens || !kbar_cache || !o || !lse)
    return MOBA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(kbar_cache) ||
      !aligned16(o) || (reinterpret_cast<uintptr_t>(seqlens) & 3) ||
      (reinterpret_cast<uintptr_t>(lse) & 3) || (reinterpret_cast<uintptr_t>(sel_out) & 3))
    return MOBA_ERR_INVALID_ARG;
  MOBA_TRY(check_ws(ws, ws_bytes, carve_decode(d, nullptr).bytes));
  DecodeWs w = carve_decode(d, static_cast<char*>(ws));
  if (sel_out) w.sel = sel_out;
  DecodeArgs a = decode_args(d, w, q, k_cache, v_cache, seqlens, const_cast<float*>(kbar_cache));
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return d.D == 128 ? decode_impl<128>(d, a, st) : decode_impl<64>(d, a, st);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free gate.
//
// Some callers cannot hand this library a workspace: code embedded in a host
// framework that owns every device allocation and exposes no allocator to
// its plugins, or a latency-critical loop that must never call cudaMalloc
// (which can synchronise the device).  moba_gate_noalloc serves them: the
// gate's scratch (status word, block numbering, block means) lives in one
// file-scope device array of fixed size, so the call allocates nothing.
//
// Limits and sharing rules:
//   * the array holds kGateScratchBytes (16 MiB); a shape whose scratch is
//     larger is refused with MOBA_ERR_WORKSPACE before anything is launched;
//   * every GPU that loads the library holds its own copy until exit;
//   * every call on a device uses the same array and leaves its contents
//     behind, so calls that can overlap on the GPU (other streams, other
//     threads) race; the caller must order them;
//   * the first call on each device looks up the array's device address
//     (cudaGetSymbolAddress) with that device current; make that first call
//     before any stream capture.
namespace {

constexpr size_t kGateScratchBytes = size_t(16) << 20;

}  // namespace

static __device__ __align__(256) unsigned char g_gate_scratch[kGateScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_gate_scratch_mu;
void* g_gate_scratch_addr[kMaxDevices] = {};

// Device address of g_gate_scratch on the current device (looked up once).
moba_status gate_scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOBA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOBA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_gate_scratch_mu);
  if (!g_gate_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_gate_scratch) != cudaSuccess || !p) return MOBA_ERR_CUDA;
    g_gate_scratch_addr[dev] = p;
  }
  *out = g_gate_scratch_addr[dev];
  return MOBA_OK;
}

// Gate-only scratch layout (status word, plan arrays, block means).
Ws carve_gate_scratch(const Problem& pr, char* base) {
  Ws w;
  memset(&w, 0, sizeof w);
  size_t off = 0;
  auto take = [&](size_t bytes) -> char* {
    char* p = base ? base + off : nullptr;
    off = align_up(off + bytes);
    return p;
  };
  const int64_t NB = pr.NBmax;
  w.status = reinterpret_cast<uint32_t*>(take(kAlign));
  w.P.totals = reinterpret_cast<int32_t*>(take(4 * sizeof(int32_t)));
  w.P.blk_off = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (pr.nseq + 1)));
  w.P.qt_off = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (pr.nseq + 1)));
  w.P.pair_off = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (pr.nseq + 1)));
  w.P.blk_tok = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * NB));
  w.P.blk_len = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * NB));
  w.kbar = reinterpret_cast<float*>(take(sizeof(float) * (size_t)pr.Hkv * NB * pr.D));
  w.bytes = off;
  return w;
}

}  // namespace

extern "C" moba_status moba_gate_noalloc(const void* q, const void* k, int32_t* sel,
                                         const moba_params* p, moba_stream_t stream) {
  Problem pr;
  MOBA_TRY(make_problem(p, false, nullptr, 0, 0, true, &pr));
  if (!topk_supported(pr)) return MOBA_ERR_UNSUPPORTED;
  // the scratch limit first: a shape it refuses never reaches the pointers
  if (carve_gate_scratch(pr, nullptr).bytes > kGateScratchBytes) return MOBA_ERR_WORKSPACE;
  if (!q || !k || !sel || !aligned16(q) || !aligned16(k) ||
      (reinterpret_cast<uintptr_t>(sel) & 3))
    return MOBA_ERR_INVALID_ARG;
  if (pr.T == 0) return MOBA_OK;
  void* base = nullptr;
  MOBA_TRY(gate_scratch_address(&base));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const Ws w = carve_gate_scratch(pr, static_cast<char*>(base));
  // The status word is not cleared here: device checks of every call latch
  // in it until moba_gate_noalloc_status reads and clears it.  The kernels
  // only ever OR bits into it, so a latched bit changes no later result.
  MOBA_TRY(run_plan_pool(pr, k, w, st));
  return pr.D == 128 ? launch_gate<128>(pr, q, w, sel, nullptr, st)
                     : launch_gate<64>(pr, q, w, sel, nullptr, st);
}

extern "C" moba_status moba_gate_noalloc_status(moba_stream_t stream) {
  void* base = nullptr;
  MOBA_TRY(gate_scratch_address(&base));
  return moba_last_device_status(base, stream);
}
