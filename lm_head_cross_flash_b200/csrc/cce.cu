// cce.cu — host side of the C ABI declared in include/cce.h: argument
// validation, workspace layout, TMA tensor maps and kernel launches on the
// caller's stream.  Nothing here allocates device memory; the caller's
// workspace holds every intermediate.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/cce.h"
#include "aux_kernels.cuh"
#include "fused_bwd.cuh"
#include "slice_bwd.cuh"
#include "qwide_fwd.cuh"
#include "gemm_tc.cuh"

using namespace cce;

namespace {

constexpr size_t kAlign = 256;
constexpr size_t kStatusBytes = 256;
// Default G'' chunk: 1 GiB.  Fewer, longer recompute/dH launches; at the long
// pair (M=8192, V=262,144) 4 chunks instead of 16 make the step 2.7 % faster
// for 0.73 GB more workspace (measured: 21.53 -> 20.95 ms).
constexpr int64_t kDefaultChunkBytes = 1ll << 30;
constexpr uint64_t kDefaultWaitNs = 2000000000ull;

std::atomic<uint64_t> g_wait_ns{kDefaultWaitNs};
std::atomic<int> g_pairs{1};  // 2-CTA (cta_group::2) tiles for dense heads
// 4/8-bit heads: 0 = choose, 1 = dequantise inside the GEMM, 2 = staged chunks
std::atomic<int> g_qstage{0};
// Backward of dense bf16 heads: 0 = choose, 1 = the fused kernel (recompute,
// coefficient tile and dH in one kernel), 2 = the two GEMMs per vocab chunk
std::atomic<int> g_bwd_mode{0};
std::atomic<int> g_fwd_mode{0};
// Staged dequantisation pays off once enough row tiles reuse each weight;
// measured on the 4-bit long-context head (D=4096, V=128,256): the backward
// from 2 row tiles (M=192: 0.71 ms staged against 1.06 ms in-kernel), the
// forward from 3 (M=256: 0.50 against 0.42; M=384: 0.61 against 0.64), with
// chunks of at least this many rows.
constexpr int64_t kStageMinRowTilesFwd = 3;
constexpr int64_t kStageMinRowTilesBwd = 2;
constexpr int64_t kStageMinRows = 8192;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// ------------------------------------------------------------ driver API --
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t,
                                   void*, const cuuint64_t*, const cuuint64_t*,
                                   const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault,
                                &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D tensor map over a row-major [rows, cols] 16-bit matrix with row
// stride `ld` elements, box {box_c, box_r}, 128-byte swizzle, zero OOB fill.
bool make_map(CUtensorMap* m, const void* ptr, bool bf16, uint64_t cols,
              uint64_t rows, uint64_t ld, uint32_t box_c, uint32_t box_r) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {box_c, box_r};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                  2, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}


// -------------------------------------------------------------- profiler --
// Optional per-kernel timing: while enabled, every kernel launch is
// bracketed by a CUDA event pair recorded on its own stream.
enum ProfKind {
  PK_SPLIT = 0, PK_LSE, PK_MERGE, PK_ORPO, PK_SKIP, PK_GRAD, PK_DH, PK_SELFTEST, PK_DHSUM,
  PK_PREFIX, PK_DW, PK_DEQ, PK_FUSED, PK_FSUM, PK_SLICE, PK_SSUM, PK_QFWD, PK_N
};
const char* const kProfNames[PK_N] = {"operand_prep",  "fwd_lse_gemm", "lse_merge",
                                      "orpo_epilogue", "skip_plan",    "bwd_grad_gemm",
                                      "bwd_dh_gemm",   "selftest",     "dh_split_sum",
                                      "prefix_gather_scatter", "bwd_dw_gemm",
                                      "dequant_chunk", "bwd_fused",
                                      "fused_part_sum", "bwd_sliced",
                                      "sliced_part_sum", "fwd_q_small_m"};
struct ProfRec {
  int kind;
  cudaEvent_t a, b;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRec> g_prof;
std::vector<cudaEvent_t> g_ev_pool;

cudaEvent_t pool_event() {
  if (!g_ev_pool.empty()) {
    cudaEvent_t e = g_ev_pool.back();
    g_ev_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

class ProfScope {
 public:
  ProfScope(int kind, cudaStream_t st) : kind_(kind), st_(st) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    if (!g_prof_on) return;
    a_ = pool_event();
    b_ = pool_event();
    if (a_ != nullptr && b_ != nullptr) cudaEventRecord(a_, st_);
  }
  ~ProfScope() {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    if (a_ == nullptr || b_ == nullptr) return;
    cudaEventRecord(b_, st_);
    g_prof.push_back({kind_, a_, b_});
  }

 private:
  int kind_;
  cudaStream_t st_;
  cudaEvent_t a_ = nullptr, b_ = nullptr;
};

// General tiled tensor map (rank 2 or 3, row-major, strides in bytes for
// dimensions 1..rank-1), zero OOB fill.
bool make_map_ex(CUtensorMap* m, const void* ptr, CUtensorMapDataType dt, int rank,
                 const uint64_t* dims, const uint64_t* strides, const uint32_t* box,
                 CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t d[3], st[2];
  cuuint32_t b[3], e[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) st[i] = strides[i];
  return fn(m, dt, rank, const_cast<void*>(ptr), d, st, b, e, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Packed 4/8-bit head as bytes [V, D*qb/8] for the in-kernel dequantisers:
// box {box_bytes, box_rows}, no swizzle, zero fill past the last row.
bool make_packed_map(CUtensorMap* m, const cce_head* W, int qb, uint32_t box_bytes,
                     uint32_t box_rows) {
  const uint64_t row_bytes = uint64_t(W->D) * qb / 8;
  const uint64_t dims[2] = {row_bytes, uint64_t(W->V)};
  const uint64_t strides[1] = {row_bytes};
  const uint32_t box[2] = {box_bytes, box_rows};
  return make_map_ex(m, W->w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_NONE);
}

// --------------------------------------------------------- device facts --
struct DevInfo {
  int sms = 0;
  int pairs = 0;  // CTA pairs (clusters of 2) resident at once, 0 = none
  int fused_pairs = 0;  // fused backward: pairs / single CTAs resident at once
  int fused_ctas = 0;
  int slice_clusters[4] = {0, 0, 0, 0};  // sliced backward, clusters of 1, 2, 4, 8
  bool attrs = false;
};

template <Mode MODE>
int max_pairs_of() {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2);
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = smem_bytes<MODE, true>();
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, cce_tc_kernel<MODE, 0, true>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}
// Clusters of two resident at once for the fused backward's pair kernel.
int max_fused_pairs() {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2);
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = FusedCfg<true>::SMEM;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, fused_bwd_kernel<true, 128>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}
// The sliced backward's kernel for clusters of `ccl` CTAs.
using SliceKernel = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, SliceArgs);
SliceKernel slice_kernel(int ccl) {
  switch (ccl) {
    case 1: return slice_bwd_kernel<1>;
    case 2: return slice_bwd_kernel<2>;
    case 4: return slice_bwd_kernel<4>;
    default: return slice_bwd_kernel<8>;
  }
}
// Clusters of `ccl` CTAs resident at once for the sliced backward.
int max_slice_clusters(int ccl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ccl);
  cfg.blockDim = dim3(SL_THREADS);
  cfg.dynamicSmemBytes = SL_SMEM;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = ccl;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, slice_kernel(ccl), &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}
std::mutex g_dev_mu;
DevInfo g_dev[64];

cce_status device_info(int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return CCE_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DevInfo& d = g_dev[dev];
  if (!d.attrs) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return CCE_ERR_CUDA;
    const auto attr = cudaFuncAttributeMaxDynamicSharedMemorySize;
    bool ok = true;
#define CCE_SET_SMEM(MODE, QB) \
    ok = ok && cudaFuncSetAttribute(cce_tc_kernel<MODE, QB>, attr, smem_bytes<MODE, false, QB>()) == cudaSuccess;
    CCE_SET_SMEM(Mode::kLse, 0) CCE_SET_SMEM(Mode::kGrad, 0) CCE_SET_SMEM(Mode::kDh, 0)
    CCE_SET_SMEM(Mode::kLse, 4) CCE_SET_SMEM(Mode::kGrad, 4) CCE_SET_SMEM(Mode::kDh, 4)
    CCE_SET_SMEM(Mode::kLse, 8) CCE_SET_SMEM(Mode::kGrad, 8) CCE_SET_SMEM(Mode::kDh, 8)
    CCE_SET_SMEM(Mode::kDw, 0)
#undef CCE_SET_SMEM
#define CCE_SET_SMEM2(MODE) \
    ok = ok && cudaFuncSetAttribute(cce_tc_kernel<MODE, 0, true>, attr, smem_bytes<MODE, true>()) == cudaSuccess;
    CCE_SET_SMEM2(Mode::kLse) CCE_SET_SMEM2(Mode::kGrad) CCE_SET_SMEM2(Mode::kDh)
#undef CCE_SET_SMEM2
    ok = ok &&
         cudaFuncSetAttribute(fused_bwd_kernel<true, 128>, attr, FusedCfg<true>::SMEM) ==
             cudaSuccess &&
         cudaFuncSetAttribute(fused_bwd_kernel<false, 128>, attr, FusedCfg<false, 128>::SMEM) ==
             cudaSuccess &&
         cudaFuncSetAttribute(slice_bwd_kernel<1>, attr, SL_SMEM) == cudaSuccess &&
         cudaFuncSetAttribute(slice_bwd_kernel<2>, attr, SL_SMEM) == cudaSuccess &&
         cudaFuncSetAttribute(slice_bwd_kernel<4>, attr, SL_SMEM) == cudaSuccess &&
         cudaFuncSetAttribute(slice_bwd_kernel<8>, attr, SL_SMEM) == cudaSuccess &&
         cudaFuncSetAttribute(qsmall_fwd_kernel<4>, attr, QsCfg<4>::SMEM) == cudaSuccess &&
         cudaFuncSetAttribute(qsmall_fwd_kernel<8>, attr, QsCfg<8>::SMEM) == cudaSuccess &&
         cudaFuncSetAttribute(qwide_fwd_kernel<4>, attr, QwCfg<4>::SMEM) == cudaSuccess &&
         cudaFuncSetAttribute(qwide_fwd_kernel<8>, attr, QwCfg<8>::SMEM) == cudaSuccess;
    if (ok) {
      d.pairs = std::min(max_pairs_of<Mode::kLse>(),
                         std::min(max_pairs_of<Mode::kGrad>(), max_pairs_of<Mode::kDh>()));
      d.fused_pairs = max_fused_pairs();
      int per_sm = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fused_bwd_kernel<false, 128>,
                                                        NUM_THREADS, FusedCfg<false>::SMEM) !=
          cudaSuccess) {
        cudaGetLastError();
        per_sm = 0;
      }
      d.fused_ctas = per_sm * d.sms;
      for (int i = 0; i < 4; ++i) d.slice_clusters[i] = max_slice_clusters(1 << i);
    }
    if (!ok)
      return CCE_ERR_CUDA;
    d.attrs = true;
  }
  *sms = d.sms;
  return CCE_OK;
}

// CTA pairs resident at once on the current device (0: pairs unavailable).
int device_pairs() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  return g_dev[dev].pairs;
}

// ------------------------------------------------------------ validation --
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned8(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 7u) == 0; }

cce_status check_head(const cce_head* W, cce_dtype h_dtype) {
  if (W == nullptr) return CCE_ERR_INVALID_ARGUMENT;
  if (W->V <= 0 || W->D <= 0 || W->w == nullptr || !aligned16(W->w))
    return CCE_ERR_INVALID_ARGUMENT;
  if (W->V > (int64_t(1) << 30) || W->D > (int64_t(1) << 16)) return CCE_ERR_UNSUPPORTED;
  if (W->D % 64 != 0) return CCE_ERR_UNSUPPORTED;
  if (!(W->softcap >= 0.f) || W->softcap > 1e30f) return CCE_ERR_INVALID_ARGUMENT;
  if (W->format == CCE_W_DENSE) {
    if (W->dtype != CCE_F32 && W->dtype != CCE_BF16) return CCE_ERR_INVALID_ARGUMENT;
    if (W->dtype != h_dtype) return CCE_ERR_UNSUPPORTED;
    return CCE_OK;
  }
  if (W->format == CCE_W_AFFINE_Q4_G64 || W->format == CCE_W_AFFINE_Q8_G64) {
    if (W->dtype != CCE_BF16 || W->scales == nullptr || W->biases == nullptr ||
        (reinterpret_cast<uintptr_t>(W->scales) & 1u) || (reinterpret_cast<uintptr_t>(W->biases) & 1u))
      return CCE_ERR_INVALID_ARGUMENT;
    if (h_dtype != CCE_BF16) return CCE_ERR_UNSUPPORTED;
    return CCE_OK;
  }
  return CCE_ERR_INVALID_ARGUMENT;
}

// The kernels number their tiles with 32-bit ints: ceil(M/128) row tiles
// times the vocab tiles (forward, recompute) or the d-tiles of every K split
// (dH, at most 32 splits) must stay below 2^31.
bool tiles_fit(int64_t M, const cce_head* W) {
  const int64_t n_rt = (M + 127) / 128;
  const int64_t per_row = std::max<int64_t>((W->V + 255) / 256, 32 * ((W->D + 255) / 256));
  return n_rt * per_row < (int64_t(1) << 31) - 1;
}

// ------------------------------------------------------ workspace layout --
struct Layout {
  size_t status = 0;
  size_t part_s = 0, part_m = 0, tgt = 0;  // forward
  size_t hs = 0, ws = 0;                   // f32 split operands
  size_t g = 0, tile_skip = 0, row_skip = 0;
  size_t dh_part = 0;                      // K-split partial dH buffers
  size_t hg = 0;                           // coeff * H (bf16), trainable head
  size_t wq = 0;                           // staged fp16 chunk of a 4/8-bit head
  bool staged = false;
  int64_t vc = 0;                          // backward vocab chunk
  int ksplit = 1;
  size_t total = 0;
};

// SM count of the current device (148 on B200 when no device is visible).
int sm_count_guess() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) == cudaSuccess &&
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
    return n;
  cudaGetLastError();
  return 148;
}

// K split of the dH GEMM: the smallest S whose tile count fills the
// persistent grid's last wave best (each split needs its own fp32 partial
// buffer, summed once at the end).  S goes up to 4, or up to the number of
// splits that fill the grid once when there are few tiles (small M: the
// GEMM then streams W at full bandwidth; the buffers are small).  A split
// that gets no K steps of a narrow chunk only zeroes its buffer.
int choose_ksplit(int64_t tiles, int sms) {
  auto eff = [&](int S) {
    const double w = double(tiles) * S / sms;
    return w / std::ceil(w);
  };
  const int smax = int(std::max<int64_t>(4, std::min<int64_t>(32, sms / std::max<int64_t>(1, tiles))));
  int best = 1;
  double be = eff(1);
  for (int S = 2; S <= smax; ++S)
    if (eff(S) > be + 0.03) {
      best = S;
      be = eff(S);
    }
  return best;
}

// Dense heads run the S and dH GEMMs on CTA pairs unless switched off, or
// unless padding the rows to 256-row pair tiles would add more than an eighth
// to the 128-row tiles' work (M <= 128: a single row tile, HBM-bound on W).
bool pairs_wanted(int64_t M, const cce_head* W, bool staged = false) {
  if (g_pairs.load() == 0 || (W->format != CCE_W_DENSE && !staged)) return false;
  const int64_t n128 = ceil_div(M, BM);
  return n128 >= 2 && 8 * (2 * ceil_div(M, 2 * BM) - n128) <= n128;
}

int ksplit_for(int64_t M, const cce_head* W, int sms, bool staged = false) {
  if (pairs_wanted(M, W, staged)) return choose_ksplit(ceil_div(M, 2 * BM) * ceil_div(W->D, BN), sms / 2);
  return choose_ksplit(ceil_div(M, BM) * ceil_div(W->D, BN), sms);
}

Layout make_layout(int64_t M, cce_dtype h, const cce_head* W, int64_t vc, int ksplit = 1,
                   bool staged = false) {
  Layout L;
  const int64_t cols = ceil_div(W->V, BN);
  const int64_t n_rt = ceil_div(M, BM);
  size_t o = kStatusBytes;
  // forward region
  size_t f = o;
  L.part_s = f; f += align_up(size_t(cols) * M * 4);
  L.part_m = f; f += align_up(size_t(cols) * M * 4);
  L.tgt = f; f += align_up(size_t(M) * 4);
  // backward region (shares the space after the status word)
  size_t b = o;
  L.g = b; b += align_up(size_t(M) * vc * 2);
  L.tile_skip = b; b += align_up(size_t(n_rt) * cols);
  L.row_skip = b; b += align_up(size_t(n_rt));
  L.dh_part = b; b += align_up(size_t(ksplit - 1) * M * W->D * 4);
  L.ksplit = ksplit;
  if (W->format == CCE_W_DENSE) {
    L.hg = b; b += align_up(size_t(M) * W->D * 2);  // coeff * H for the dW GEMM
  }
  // split operands live after both regions
  size_t s = std::max(f, b);
  if (h == CCE_F32) {
    L.hs = s; s += align_up(size_t(M) * 3 * W->D * 2);
    L.ws = s; s += align_up(size_t(W->V) * 3 * W->D * 2);
  } else if (W->format != CCE_W_DENSE) {
    L.hs = s; s += align_up(size_t(M) * W->D * 2);  // fp16 rows (K-permuted unless staged)
    if (staged) {
      L.wq = s; s += align_up(size_t(vc) * W->D * 2);  // fp16 [vc, D] head chunk
    }
  }
  L.staged = staged && W->format != CCE_W_DENSE;
  L.vc = vc;
  L.total = s;
  return L;
}

// Row tiles per raster group of the S GEMMs: as many as keep about 48 MB of
// the hidden rows (the re-used operand) in L2.
int group_rows(int64_t n_rt, int64_t k_elems) {
  const int64_t per = int64_t(BM) * k_elems * 2;
  return int(std::max<int64_t>(1, std::min<int64_t>(n_rt, (int64_t(48) << 20) / per)));
}

// Default G'' chunk: kDefaultChunkBytes, or four times dH when that is larger
// (every chunk adds into dH once, so wider chunks save dH traffic when M*D is
// big).
int64_t default_vc(int64_t M, const cce_head* W) {
  const int64_t vmax = ceil_div(W->V, BN) * BN;
  const int64_t budget = std::max<int64_t>(kDefaultChunkBytes, 4 * M * W->D * 4);
  int64_t vc = (budget / (2 * M)) / BN * BN;
  return std::max<int64_t>(BN, std::min(vc, vmax));
}

// Widest chunk whose layout fits in ws_bytes (0 if even the narrowest
// does not fit).
int64_t fit_vc(int64_t M, cce_dtype h, const cce_head* W, size_t ws_bytes, int ksplit,
              bool staged = false) {
  const int64_t vmax = ceil_div(W->V, BN) * BN;
  if (make_layout(M, h, W, BN, ksplit, staged).total > ws_bytes) return 0;
  int64_t lo = 1, hi = vmax / BN;
  while (lo < hi) {
    const int64_t mid = (lo + hi + 1) / 2;
    if (make_layout(M, h, W, mid * BN, ksplit, staged).total <= ws_bytes) lo = mid;
    else hi = mid - 1;
  }
  return lo * BN;
}

// A 4/8-bit head is dequantised chunk by chunk into fp16 in the workspace
// (then the dense GEMMs run on it) when enough row tiles reuse each weight.
bool q_stage_wanted(int64_t M, const cce_head* W, bool forward) {
  if (W->format == CCE_W_DENSE) return false;
  const int mode = g_qstage.load();
  const int64_t min_tiles = forward ? kStageMinRowTilesFwd : kStageMinRowTilesBwd;
  return mode == 2 || (mode == 0 && ceil_div(M, BM) >= min_tiles);
}

// Smallest staged chunk worth its launches (the whole head if it is smaller).
int64_t stage_min_rows(const cce_head* W) {
  return std::min<int64_t>(kStageMinRows, ceil_div(W->V, BN) * BN);
}

// The transposed small-M forward of a 4/8-bit head, not staged, with whole
// groups of 8 scales per 16-byte load (D a multiple of 512, 16-byte aligned
// scale and bias rows): 1 = qsmall_fwd.cuh (at most 128 head rows), 2 =
// qwide_fwd.cuh (129 to 240 by default; forward mode 2 takes it for 1 to
// 256), 0 = the tiled GEMM.  The wide form's time grows with N = M rounded
// up to 16 while the GEMM's 256-row tile costs the same from 129 to 256
// rows: at D = 4,096, V = 128,256 the wide form took 0.403 ms at M = 200
// against 0.439 ms, but 0.444 against 0.438 ms at M = 256.
constexpr int64_t kQwideDefaultMaxM = 240;
int qsmall_wanted(int64_t M, const cce_head* W, bool staged) {
  const int mode = g_fwd_mode.load();
  if (mode == 1 || W->format == CCE_W_DENSE || staged || W->D % 512 != 0 ||
      !aligned16(W->scales) || !aligned16(W->biases) || M > QW_MAXM)
    return 0;
  if (mode == 2) return 2;
  return M <= QS_MAXM ? 1 : M <= kQwideDefaultMaxM ? 2 : 0;
}

// How one forward call runs for a workspace size: staged chunks of vq rows
// (4/8-bit heads at large M), else a single launch over the vocabulary.
struct FwdPlan {
  bool staged = false;
  int64_t vq = 0;
  Layout L;
};
FwdPlan plan_forward(int64_t M, cce_dtype h, const cce_head* W, size_t ws_bytes) {
  FwdPlan p;
  p.staged = q_stage_wanted(M, W, true);
  if (p.staged && (p.vq = fit_vc(M, h, W, ws_bytes, 1, true)) < stage_min_rows(W))
    p.staged = false;
  p.L = p.staged ? make_layout(M, h, W, p.vq, 1, true) : make_layout(M, h, W, BN);
  if (!p.staged) p.vq = ceil_div(W->V, BN) * BN;
  return p;
}

// How one backward call runs: the G'' chunk vc, the K split of the dH GEMM
// (fewer splits when the workspace cannot hold their buffers), staging of a
// 4/8-bit head (only with chunks of stage_min_rows or more), and whether the
// split is the one CTA pairs were sized for.  vc == 0: workspace too small.
struct BwdPlan {
  bool staged = false;
  int ksplit = 1;
  int64_t vc = 0;
  bool pairs = false;
  Layout L;
};
BwdPlan plan_backward(int64_t M, cce_dtype h, const cce_head* W, size_t ws_bytes) {
  BwdPlan p;
  p.staged = q_stage_wanted(M, W, false);
  for (int attempt = 0; attempt < 2; ++attempt) {
    p.ksplit = ksplit_for(M, W, sm_count_guess(), p.staged);
    while ((p.vc = fit_vc(M, h, W, ws_bytes, p.ksplit, p.staged)) == 0 && p.ksplit > 1)
      --p.ksplit;
    if (!p.staged || p.vc >= stage_min_rows(W)) break;
    p.staged = false;
  }
  p.pairs = pairs_wanted(M, W, p.staged) &&
            p.ksplit == ksplit_for(M, W, sm_count_guess(), p.staged);
  if (p.vc > 0) p.L = make_layout(M, h, W, p.vc, p.ksplit, p.staged);
  return p;
}

uint32_t* status_word(void* ws) { return reinterpret_cast<uint32_t*>(ws); }

cce_status launch_ok() {
  return cudaGetLastError() == cudaSuccess ? CCE_OK : CCE_ERR_CUDA;
}

int grid_for(int64_t tiles, int sms) {
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(tiles, sms)));
}

// Launch a tensor-core step on CTA pairs (clusters of two, cta_group::2).
template <Mode MODE>
cudaError_t launch_tc_pairs(int64_t pair_tiles, int max_pairs, cudaStream_t st,
                            const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mc,
                            const CUtensorMap& mc2, const TileArgs& args) {
  cudaLaunchConfig_t cfg = {};
  const int pairs = int(std::max<int64_t>(1, std::min<int64_t>(pair_tiles, max_pairs)));
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = smem_bytes<MODE, true>();
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, cce_tc_kernel<MODE, 0, true>, ma, mb, mc, mc2, args);
}

// Launch one tensor-core step; a quantised head adds the dequantisation
// warps.
template <Mode MODE>
void launch_tc(int qb, int64_t tiles, int sms, cudaStream_t st, const CUtensorMap& ma,
               const CUtensorMap& mb, const CUtensorMap& mc, const CUtensorMap& mc2,
               const TileArgs& args) {
  if (qb == 4)
    cce_tc_kernel<MODE, 4><<<grid_for(tiles, sms), NUM_THREADS_Q4, smem_bytes<MODE, false, 4>(), st>>>(
        ma, mb, mc, mc2, args);
  else if (qb == 8)
    cce_tc_kernel<MODE, 8><<<grid_for(tiles, sms), NUM_THREADS_Q4, smem_bytes<MODE, false, 8>(), st>>>(
        ma, mb, mc, mc2, args);
  else
    cce_tc_kernel<MODE, 0><<<grid_for(tiles, sms), NUM_THREADS, smem_bytes<MODE>(), st>>>(
        ma, mb, mc, mc2, args);
}

// Operands of the tensor-core GEMMs for one problem: 16-bit A (head rows)
// and B (head) with their K extents.
struct Operands {
  int qb;          // 4 / 8: quantised head, B is dequantised in-kernel, A is fp16
  int stage_qb = 0;  // 4 / 8: quantised head staged as fp16 chunks in b
  const void* a;   // [M, ka] 16-bit
  const void* b;   // [V, kb] 16-bit (dense heads)
  int64_t k;       // contraction length used by the S GEMM
  int64_t ld_a, ld_b;
  bool bf16;
  int64_t d_pass_off;  // kDh: offset (elements) of the lo half of a split head
  int npass_dh;
};

cce_status prepare_operands(const void* H, cce_dtype h, int64_t M, const cce_head* W,
                            const Layout& L, void* ws, cudaStream_t st, Operands* op) {
  const int64_t D = W->D;
  op->qb = W->format == CCE_W_AFFINE_Q4_G64 ? 4 : W->format == CCE_W_AFFINE_Q8_G64 ? 8 : 0;
  op->stage_qb = 0;
  if (op->qb) {
    // 4/8-bit heads compute in fp16: report scales or biases it cannot hold
    const int64_t n = W->V * (D / 64);
    ProfScope ps(PK_SPLIT, st);
    sb_range_kernel<<<int(std::max<int64_t>(1, std::min<int64_t>(ceil_div(n, 256), 1184))), 256, 0,
                      st>>>(static_cast<const uint16_t*>(W->scales),
                            static_cast<const uint16_t*>(W->biases), n, status_word(ws));
    if (launch_ok() != CCE_OK) return CCE_ERR_CUDA;
  }
  if (op->qb && L.staged) {
    // fp16 rows in natural order; B is the fp16 chunk staged by stage_chunk
    uint4* h16 = reinterpret_cast<uint4*>(static_cast<char*>(ws) + L.hs);
    {
      ProfScope ps(PK_SPLIT, st);
      h_to_f16_perm_kernel<0><<<1184, 256, 0, st>>>(static_cast<const uint4*>(H), M * D / 8, h16,
                                                            status_word(ws));
    }
    if (launch_ok() != CCE_OK) return CCE_ERR_CUDA;
    op->stage_qb = op->qb;
    op->qb = 0;
    op->a = h16;
    op->b = static_cast<char*>(ws) + L.wq;
    op->k = D;
    op->ld_a = D;
    op->ld_b = D;
    op->bf16 = false;
    op->d_pass_off = 0;
    op->npass_dh = 1;
    return CCE_OK;
  }
  if (op->qb) {
    uint4* h16 = reinterpret_cast<uint4*>(static_cast<char*>(ws) + L.hs);
    {
      ProfScope ps(PK_SPLIT, st);
      if (op->qb == 4)
        h_to_f16_perm_kernel<4><<<1184, 256, 0, st>>>(static_cast<const uint4*>(H), M * D / 8, h16,
                                                            status_word(ws));
      else
        h_to_f16_perm_kernel<8><<<1184, 256, 0, st>>>(static_cast<const uint4*>(H), M * D / 8, h16,
                                                            status_word(ws));
    }
    if (launch_ok() != CCE_OK) return CCE_ERR_CUDA;
    op->a = h16;
    op->b = nullptr;
    op->k = D;
    op->ld_a = D;
    op->ld_b = D;
    op->bf16 = false;
    op->d_pass_off = 0;
    op->npass_dh = 1;
    return CCE_OK;
  }
  if (h == CCE_BF16) {
    op->a = H;
    op->b = W->w;
    op->k = D;
    op->ld_a = D;
    op->ld_b = D;
    op->bf16 = true;
    op->d_pass_off = 0;
    op->npass_dh = 1;
    return CCE_OK;
  }
  // fp32: three-part bf16 split, K = 3D.
  auto* hs = reinterpret_cast<__nv_bfloat16*>(static_cast<char*>(ws) + L.hs);
  auto* wsb = reinterpret_cast<__nv_bfloat16*>(static_cast<char*>(ws) + L.ws);
  {
    ProfScope ps(PK_SPLIT, st);
    split_f32_kernel<<<1184, 256, 0, st>>>(static_cast<const float*>(H), M, int(D), 0, hs);
    split_f32_kernel<<<1184, 256, 0, st>>>(static_cast<const float*>(W->w), W->V, int(D), 1, wsb);
  }
  if (launch_ok() != CCE_OK) return CCE_ERR_CUDA;
  op->a = hs;
  op->b = wsb;
  op->k = 3 * D;
  op->ld_a = 3 * D;
  op->ld_b = 3 * D;
  op->bf16 = true;
  op->d_pass_off = D;  // columns [D, 2D) of the right split hold lo
  op->npass_dh = 2;
  return CCE_OK;
}

// Dequantise head rows [v0, v0 + rows) of a staged 4/8-bit head into the
// fp16 chunk buffer (op.b).
cce_status stage_chunk(const Operands& op, const cce_head* W, int64_t v0, int64_t rows,
                       int sms, cudaStream_t st) {
  const int64_t units = rows * (W->D / 8);
  const int grid = int(std::max<int64_t>(1, std::min<int64_t>(ceil_div(units, 256 * 4), 8 * sms)));
  const auto* qw = static_cast<const uint32_t*>(W->w);
  const auto* sc = static_cast<const uint16_t*>(W->scales);
  const auto* bi = static_cast<const uint16_t*>(W->biases);
  uint4* out = static_cast<uint4*>(const_cast<void*>(op.b));
  {
    ProfScope ps(PK_DEQ, st);
    if (op.stage_qb == 4)
      dequant_rows_f16_kernel<4><<<grid, 256, 0, st>>>(qw, sc, bi, v0, rows, int(W->D), out);
    else
      dequant_rows_f16_kernel<8><<<grid, 256, 0, st>>>(qw, sc, bi, v0, rows, int(W->D), out);
  }
  return launch_ok();
}

// ------------------------------------------------------- fused backward --
// Fused-backward units (pairs or single CTAs) resident at once: the device's
// figure, or the B200 figure where no device is visible (host-side planning).
int fused_resident(bool c2) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64 &&
      device_info(&sms) == CCE_OK) {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    return c2 ? g_dev[dev].fused_pairs : g_dev[dev].fused_ctas;
  }
  cudaGetLastError();
  return c2 ? 74 : 148;
}

// How the fused backward runs: tile shape, groups of C members, the waves
// and remainder partition of (row tile, round) units, the number of dH
// buffers, and its workspace (block-skip plan, exchange flags, the G'' ring,
// partial dH buffers).  ok = false: the problem is not one the fused kernel
// takes (4/8-bit or fp32 heads, a trainable head, the mode switch set to the
// two GEMMs, or D too wide for a group of resident units).
struct FusedPlan {
  bool ok = false;
  bool c2 = false;
  int bv = 256;  // vocab columns of an S tile
  FusedArgs a{};
  int nbuf = 1;
  int64_t ring_rows = 0;
  size_t tile_skip = 0, row_skip = 0, umask = 0, flags = 0, ring = 0, parts = 0, total = 0;
};

// Choosing between the fused backward and the two GEMMs: below this many
// rows the two GEMMs were faster on the same box (D = 2048, V = 262,144; ms):
//   M      64     128    256    512    1024   2048   4096   8192
//   fused  0.393  0.403  0.492  0.902  1.709  3.175  6.435  13.81
//   two    0.344  0.361  0.485  0.857  1.712  3.380  6.962  13.60
// (at small M the fused kernel's groups hold more W in flight than L2 keeps
// between a round's two reads, so it reads W twice as well; at 8192 the two
// are within 2 %, and the fused kernel needs 67 MB of workspace against
// 1.17 GB).  D = 1536, V = 73,440: fused 1-4 % faster from M = 512.
constexpr int64_t kFusedMinRows = 1024;

FusedPlan plan_fused(int64_t M, cce_dtype h, const cce_head* W, bool want_dw) {
  FusedPlan f;
  const int mode = g_bwd_mode.load();
  if (mode == 2 || mode == 3 || want_dw || h != CCE_BF16 || W->format != CCE_W_DENSE) return f;
  if (mode == 0 && M < kFusedMinRows) return f;
  const int64_t n128 = ceil_div(M, BM);
  f.c2 = g_pairs.load() != 0 && n128 >= 2;
  const int TH = f.c2 ? FusedCfg<true>::TH : FusedCfg<false>::TH;
  f.bv = f.c2 ? FusedCfg<true>::BV : FusedCfg<false>::BV;
  const int BV = f.bv;
  const int C = int(ceil_div(W->D, FB_DS));
  if (C > 32) return f;  // skip masks hold 32 members
  const int G = fused_resident(f.c2) / C;
  if (G < 1) return f;
  FusedArgs& a = f.a;
  a.M = int(M);
  a.V = int(W->V);
  a.D = int(W->D);
  a.n_rt = int(ceil_div(M, TH));
  a.n_rt128 = int(n128);
  a.nk = int(ceil_div(W->D, BK));
  a.C = C;
  a.G = G;
  a.n_vt = int(ceil_div(W->V, BV));
  a.n_rounds = int(ceil_div(a.n_vt, C));
  a.waves = a.n_rt / G;
  a.rem = a.n_rt % G;
  a.row_rem = int(std::min<int64_t>(M, int64_t(a.waves) * G * TH));
  // remainder: bands of rem groups sharing rounds, then the leftover
  const int64_t T = int64_t(a.rem) * a.n_rounds;
  a.nb = a.bw = a.lr = a.r0 = a.rl = a.ls = 0;
  if (a.rem > 0) {
    if (T >= G) {
      a.nb = G / a.rem;
      const int r = G % a.rem;
      if (r > 0) {
        a.bw = int(T / G);
        a.lr = r;
        a.r0 = a.nb * a.bw;
        a.rl = a.n_rounds - a.r0;
        a.ls = 1;  // r < rem: leftover groups take whole tiles first, in step
      }
    } else {
      a.lr = int(T);
      a.rl = a.n_rounds;
    }
  }
  for (int i = 0; i < a.rem; ++i) f.nbuf = std::max(f.nbuf, fb_slices(a, i));
  f.ring_rows = int64_t(G) * FB_DEPTH * C * TH;
  const int64_t cols = ceil_div(W->V, BN);
  size_t o = kStatusBytes;
  f.tile_skip = o; o += align_up(size_t(n128) * cols);
  f.row_skip = o; o += align_up(size_t(n128));
  f.umask = o; o += align_up(size_t(a.n_rt) * a.n_rounds * 4);
  f.flags = o; o += align_up((size_t(G) * FB_DEPTH * C * (2 + C) + G) * 4);
  f.ring = o; o += align_up(size_t(f.ring_rows) * BV * 2);
  f.parts = o; o += align_up(size_t(f.nbuf - 1) * (M - a.row_rem) * W->D * 4);
  // the forward's region shares the same bytes (it is dead by the backward)
  f.total = std::max(o, make_layout(M, h, W, BN).total);
  f.ok = true;
  return f;
}

cce_status fused_backward(const FusedPlan& fp, const void* H, const cce_head* W,
                          const int32_t* labels, const float* lse, const float* coeff,
                          float filter_eps, const float* blockmax, float* dH,
                          unsigned long long* skip_stats, void* ws, cudaStream_t st) {
  int sms = 0;
  cce_status s = device_info(&sms);
  if (s != CCE_OK) return s;
  char* wsc = static_cast<char*>(ws);
  const FusedArgs& p = fp.a;
  const int64_t M = p.M, V = p.V, D = p.D;
  const int64_t cols = ceil_div(V, BN);
  uint8_t* tile_skip = reinterpret_cast<uint8_t*>(wsc + fp.tile_skip);
  uint8_t* row_skip = reinterpret_cast<uint8_t*>(wsc + fp.row_skip);
  {
    const int64_t units = int64_t(p.n_rt128) * cols;
    const int wpb = 8;
    ProfScope ps(PK_SKIP, st);
    skip_plan_kernel<<<int(ceil_div(units, wpb)), wpb * 32, 0, st>>>(
        filter_eps > 0.f ? blockmax : nullptr, lse, labels, coeff, int(M), int(cols),
        p.n_rt128, filter_eps, tile_skip, row_skip, skip_stats);
    if (launch_ok() != CCE_OK) return CCE_ERR_CUDA;
  }
  const size_t flag_bytes = (size_t(p.G) * FB_DEPTH * p.C * (2 + p.C) + p.G) * 4;
  if (cudaMemsetAsync(wsc + fp.flags, 0, flag_bytes, st) != cudaSuccess) return CCE_ERR_CUDA;

  const int BV = fp.bv;
  void* ring = wsc + fp.ring;
  CUtensorMap mh, mwk, mwm, mgl, mgs, md0, md1;
  if (!make_map(&mh, H, true, D, M, D, BK, BM) ||
      !make_map(&mwk, W->w, true, D, V, D, BK, fp.c2 ? 128 : BV) ||
      !make_map(&mwm, W->w, true, D, V, D, 64, BK) ||
      !make_map(&mgl, ring, true, BV, fp.ring_rows, BV, BK, BM))
    return CCE_ERR_CUDA;
  {
    const uint64_t gd[2] = {uint64_t(BV), uint64_t(fp.ring_rows)};
    const uint64_t gs[1] = {uint64_t(BV) * 2};
    const uint32_t gb[2] = {32, 32};
    if (!make_map_ex(&mgs, ring, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, gd, gs, gb,
                     CU_TENSOR_MAP_SWIZZLE_64B))
      return CCE_ERR_CUDA;
    const uint64_t dd[3] = {uint64_t(D), uint64_t(M), 1};
    const uint64_t ds[2] = {uint64_t(D) * 4, uint64_t(M) * D * 4};
    const uint32_t db[3] = {32, 32, 1};
    if (!make_map_ex(&md0, dH, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, dd, ds, db,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return CCE_ERR_CUDA;
    md1 = md0;
    if (fp.nbuf > 1) {
      const uint64_t mr = uint64_t(M - p.row_rem);
      const uint64_t pd[3] = {uint64_t(D), mr, uint64_t(fp.nbuf - 1)};
      const uint64_t ps[2] = {uint64_t(D) * 4, mr * D * 4};
      if (!make_map_ex(&md1, wsc + fp.parts, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, pd, ps, db,
                       CU_TENSOR_MAP_SWIZZLE_128B))
        return CCE_ERR_CUDA;
    }
  }
  FusedArgs a = p;
  a.wait_ns = g_wait_ns.load();
  a.status = status_word(ws);
  a.labels = labels;
  a.lse = lse;
  a.coeff = coeff;
  a.filter_eps = filter_eps;
  // the plan marks vocab blocks only with block skip (blockmax and a filter)
  a.tile_skip = (filter_eps > 0.f && blockmax != nullptr) ? tile_skip : nullptr;
  a.skip_ld = int(cols);
  a.row_skip = row_skip;
  a.softcap = W->softcap;
  a.inv_cap = W->softcap > 0.f ? 1.f / W->softcap : 0.f;
  a.ready = reinterpret_cast<uint32_t*>(wsc + fp.flags);
  a.consumed = a.ready + size_t(p.G) * FB_DEPTH * p.C * 2;
  a.progress = a.consumed + size_t(p.G) * FB_DEPTH * p.C * p.C;
  {
    // every unit's skip mask, once, before the backward reads them
    uint32_t* um = reinterpret_cast<uint32_t*>(wsc + fp.umask);
    const int64_t units = int64_t(p.n_rt) * p.n_rounds;
    const int grid = int(std::max<int64_t>(1, std::min<int64_t>(ceil_div(units, 256), 4 * sms)));
    ProfScope ps(PK_SKIP, st);
    if (fp.c2)
      fused_mask_kernel<true, FusedCfg<true>::BV><<<grid, 256, 0, st>>>(a, um);
    else
      fused_mask_kernel<false, FusedCfg<false, 128>::BV><<<grid, 256, 0, st>>>(a, um);
    if (launch_ok() != CCE_OK) return CCE_ERR_CUDA;
    a.unit_mask = um;
  }
  {
    ProfScope ps(PK_FUSED, st);
    const int members = a.G * a.C;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    if (fp.c2) {
      cfg.gridDim = dim3(2 * members);
      cfg.dynamicSmemBytes = FusedCfg<true>::SMEM;
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = 2;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      cfg.attrs = at;
      cfg.numAttrs = 1;
      if (cudaLaunchKernelEx(&cfg, fused_bwd_kernel<true, 128>, mh, mwk, mwm, mgl, mgs, md0, md1,
                             a) != cudaSuccess)
        return CCE_ERR_CUDA;
    } else {
      cfg.gridDim = dim3(members);
      cfg.numAttrs = 0;
      cfg.dynamicSmemBytes = FusedCfg<false, 128>::SMEM;
      if (cudaLaunchKernelEx(&cfg, fused_bwd_kernel<false, 128>, mh, mwk, mwm, mgl, mgs, md0,
                             md1, a) != cudaSuccess)
        return CCE_ERR_CUDA;
    }
  }
  if (launch_ok() != CCE_OK) return CCE_ERR_CUDA;
  if (fp.nbuf > 1) {
    const int TH = fp.c2 ? FusedCfg<true>::TH : FusedCfg<false>::TH;
    const int64_t n4 = (M - a.row_rem) * (D / 4);
    ProfScope ps(PK_FSUM, st);
    fused_sum_parts_kernel<<<int(std::max<int64_t>(1, std::min<int64_t>(ceil_div(n4, 256),
                                                                          4 * sms))),
                             256, 0, st>>>(reinterpret_cast<float4*>(dH),
                                           reinterpret_cast<const float4*>(wsc + fp.parts), a,
                                           TH);
    if (launch_ok() != CCE_OK) return CCE_ERR_CUDA;
  }
  return CCE_OK;
}


// Clusters of `ccl` CTAs of the sliced backward resident at once (without a
// device: 148 SMs over clusters of ccl).
int slice_resident(int ccl) {
  int dev = 0, sms = 0;
  int i = 0;
  while ((1 << i) < ccl) ++i;
  if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64 &&
      device_info(&sms) == CCE_OK) {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    return g_dev[dev].slice_clusters[i];
  }
  cudaGetLastError();
  return 148 / ccl;
}

// How the sliced backward runs (slice_bwd.cuh): clusters of Ccl CTAs, one
// 256-column slice of D each (Ccl the power of two covering D), the vocab
// tiles dealt to the resident clusters in turn, and its workspace
// (block-skip plan, one partial dH per cluster).  ok = false: the problem is
// not one it takes (more than 64 rows, D above 2048, 4/8-bit or fp32
// heads, a trainable head), or the mode switch is not 3.  The default does
// not take it: at D = 2048, V = 262,144 it measured 0.51 ms at M = 64 (8 to
// 64 rows alike) against 0.344 ms for the two GEMMs, which read W twice but
// stream it at the HBM rate; the sliced kernel reads W once but its
// exchange between the CTAs of a cluster, double-buffered as deep as shared
// memory allows, holds each 128-row vocab tile to about 6,300 cycles.
struct SlicePlan {
  bool ok = false;
  SliceArgs a{};
  size_t tile_skip = 0, row_skip = 0, parts = 0, total = 0;
};

SlicePlan plan_slice(int64_t M, cce_dtype h, const cce_head* W, bool want_dw) {
  SlicePlan f;
  const int mode = g_bwd_mode.load();
  if (mode != 3 || want_dw || h != CCE_BF16 || W->format != CCE_W_DENSE) return f;
  if (M > SL_MP || W->D > int64_t(SL_MAXC) * SL_DS) return f;
  int ccl = 1;
  while (ccl * SL_DS < W->D) ccl <<= 1;
  const int n_vt = int(ceil_div(W->V, SL_BV));
  const int ncl = std::min(slice_resident(ccl), n_vt);
  if (ncl < 1) return f;
  SliceArgs& a = f.a;
  a.M = int(M);
  a.V = int(W->V);
  a.D = int(W->D);
  a.Ccl = ccl;
  a.n_cl = ncl;
  a.n_vt = n_vt;
  const int64_t cols = ceil_div(W->V, BN);
  size_t o = kStatusBytes;
  f.tile_skip = o; o += align_up(size_t(cols));
  f.row_skip = o; o += align_up(1);
  f.parts = o; o += align_up(size_t(ncl) * M * W->D * 4);
  f.total = std::max(o, make_layout(M, h, W, BN).total);
  f.ok = true;
  return f;
}

cce_status slice_backward(const SlicePlan& sp, const void* H, const cce_head* W,
                          const int32_t* labels, const float* lse, const float* coeff,
                          float filter_eps, const float* blockmax, float* dH,
                          unsigned long long* skip_stats, void* ws, cudaStream_t st) {
  int sms = 0;
  cce_status s = device_info(&sms);
  if (s != CCE_OK) return s;
  char* wsc = static_cast<char*>(ws);
  const int64_t M = sp.a.M, V = sp.a.V, D = sp.a.D;
  const int64_t cols = ceil_div(V, BN);
  uint8_t* tile_skip = reinterpret_cast<uint8_t*>(wsc + sp.tile_skip);
  uint8_t* row_skip = reinterpret_cast<uint8_t*>(wsc + sp.row_skip);
  {
    const int wpb = 8;
    ProfScope ps(PK_SKIP, st);
    skip_plan_kernel<<<int(ceil_div(cols, wpb)), wpb * 32, 0, st>>>(
        filter_eps > 0.f ? blockmax : nullptr, lse, labels, coeff, int(M), int(cols), 1,
        filter_eps, tile_skip, row_skip, skip_stats);
    if (launch_ok() != CCE_OK) return CCE_ERR_CUDA;
  }
  CUtensorMap mh, mws, mwd;
  if (!make_map(&mh, H, true, D, M, D, 64, SL_MP) ||
      !make_map(&mws, W->w, true, D, V, D, 64, SL_BV) ||
      !make_map(&mwd, W->w, true, D, V, D, 64, 64))
    return CCE_ERR_CUDA;
  SliceArgs a = sp.a;
  a.wait_ns = g_wait_ns.load();
  a.status = status_word(ws);
  a.labels = labels;
  a.lse = lse;
  a.coeff = coeff;
  a.filter_eps = filter_eps;
  // the plan marks vocab blocks only with block skip (blockmax and a filter)
  a.tile_skip = (filter_eps > 0.f && blockmax != nullptr) ? tile_skip : nullptr;
  a.row_skip = row_skip;
  a.softcap = W->softcap;
  a.inv_cap = W->softcap > 0.f ? 1.f / W->softcap : 0.f;
  a.parts = reinterpret_cast<float*>(wsc + sp.parts);
  {
    ProfScope ps(PK_SLICE, st);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.n_cl * a.Ccl);
    cfg.blockDim = dim3(SL_THREADS);
    cfg.dynamicSmemBytes = SL_SMEM;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = a.Ccl;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, slice_kernel(a.Ccl), mh, mws, mwd, a) != cudaSuccess)
      return CCE_ERR_CUDA;
  }
  if (launch_ok() != CCE_OK) return CCE_ERR_CUDA;
  {
    const int64_t n4 = M * D / 4;
    ProfScope ps(PK_SSUM, st);
    slice_sum_kernel<<<int(std::max<int64_t>(1, std::min<int64_t>(ceil_div(n4, 256), 4 * sms))),
                       256, 0, st>>>(reinterpret_cast<float4*>(dH),
                                     reinterpret_cast<const float4*>(a.parts), a.n_cl, n4);
    if (launch_ok() != CCE_OK) return CCE_ERR_CUDA;
  }
  return CCE_OK;
}

// Partials and target logits of the whole vocabulary from the transposed
// small-M kernel: one CTA per SM over the 256-row vocab blocks.
cce_status qsmall_forward(const Operands& op, const cce_head* W, int64_t M, bool wide, int sms,
                          cudaStream_t st, const int32_t* labels, float* part_m, float* part_s,
                          float* tgt, uint32_t* status) {
  const int Mp = int(std::max<int64_t>(16, ceil_div(M, 16) * 16));
  CUtensorMap mp, mh;
  // one K step's packed rows: one group of 64 (wide), KG groups (narrow)
  const int kg = wide ? 1 : (op.qb == 4 ? QsCfg<4>::KG : QsCfg<8>::KG);
  if (!make_packed_map(&mp, W, op.qb, uint32_t(op.qb * 8 * kg),
                       wide ? QW_UNIT : QS_BLK))
    return CCE_ERR_CUDA;
  if (!make_map(&mh, op.a, false, op.k, M, op.ld_a, 64, uint32_t(Mp))) return CCE_ERR_CUDA;
  QsArgs a;
  std::memset(&a, 0, sizeof(a));
  a.M = int(M);
  a.Mp = Mp;
  a.V = int(W->V);
  a.D = int(W->D);
  a.nk = int(W->D / 64 / kg);
  a.n_blk = int(ceil_div(W->V, QS_BLK));
  a.nacc = Mp <= 64 ? 2 : 1;
  a.wait_ns = g_wait_ns.load();
  a.status = status;
  a.labels = labels;
  a.q_scale = static_cast<const uint16_t*>(W->scales);
  a.q_bias = static_cast<const uint16_t*>(W->biases);
  a.softcap = W->softcap;
  a.inv_cap = W->softcap > 0.f ? 1.f / W->softcap : 0.f;
  a.part_m = part_m;
  a.part_s = part_s;
  a.tgt = tgt;
  const int grid = int(std::min<int64_t>(a.n_blk, sms));
  ProfScope ps(PK_QFWD, st);
  if (wide) {
    if (op.qb == 4)
      qwide_fwd_kernel<4><<<grid, QW_THREADS, QwCfg<4>::SMEM, st>>>(mp, mh, a);
    else
      qwide_fwd_kernel<8><<<grid, QW_THREADS, QwCfg<8>::SMEM, st>>>(mp, mh, a);
  } else if (op.qb == 4) {
    qsmall_fwd_kernel<4><<<grid, QS_THREADS, QsCfg<4>::SMEM, st>>>(mp, mh, a);
  } else {
    qsmall_fwd_kernel<8><<<grid, QS_THREADS, QsCfg<8>::SMEM, st>>>(mp, mh, a);
  }
  return launch_ok();
}

}  // namespace

// ========================================================================
extern "C" {

const char* cce_status_string(cce_status s) {
  switch (s) {
    case CCE_OK: return "CCE_OK";
    case CCE_ERR_INVALID_ARGUMENT: return "CCE_ERR_INVALID_ARGUMENT";
    case CCE_ERR_UNSUPPORTED: return "CCE_ERR_UNSUPPORTED";
    case CCE_ERR_CUDA: return "CCE_ERR_CUDA";
    case CCE_ERR_WORKSPACE_TOO_SMALL: return "CCE_ERR_WORKSPACE_TOO_SMALL";
    case CCE_ERR_LABEL_OUT_OF_RANGE: return "CCE_ERR_LABEL_OUT_OF_RANGE";
    case CCE_ERR_DEVICE_TIMEOUT: return "CCE_ERR_DEVICE_TIMEOUT";
    case CCE_ERR_EMPTY_SEGMENT: return "CCE_ERR_EMPTY_SEGMENT";
    case CCE_ERR_DOMAIN: return "CCE_ERR_DOMAIN";
    case CCE_ERR_FP16_RANGE: return "CCE_ERR_FP16_RANGE";
  }
  return "CCE_UNKNOWN_STATUS";
}

void cce_set_wait_limit_ns(uint64_t ns) { g_wait_ns.store(ns == 0 ? kDefaultWaitNs : ns); }

void cce_set_cta_pairs(int on) { g_pairs.store(on != 0 ? 1 : 0); }

void cce_set_quant_staging(int mode) { g_qstage.store(mode == 1 || mode == 2 ? mode : 0); }

void cce_set_backward_mode(int mode) { g_bwd_mode.store(mode >= 1 && mode <= 3 ? mode : 0); }
void cce_set_forward_mode(int mode) { g_fwd_mode.store(mode == 1 || mode == 2 ? mode : 0); }

cce_status cce_query_plan(int64_t M, cce_dtype h_dtype, const cce_head* W, size_t ws_bytes,
                          cce_plan* out) {
  if (out == nullptr || M <= 0 || M > (int64_t(1) << 30)) return CCE_ERR_INVALID_ARGUMENT;
  if (h_dtype != CCE_F32 && h_dtype != CCE_BF16) return CCE_ERR_INVALID_ARGUMENT;
  const cce_status s = check_head(W, h_dtype);
  if (s != CCE_OK) return s;
  if (!tiles_fit(M, W)) return CCE_ERR_UNSUPPORTED;
  std::memset(out, 0, sizeof(*out));
  const FwdPlan f = plan_forward(M, h_dtype, W, ws_bytes);
  const BwdPlan b = plan_backward(M, h_dtype, W, ws_bytes);
  out->fwd_ok = f.L.total <= ws_bytes;
  out->fwd_chunk = f.vq;
  out->fwd_staged = f.staged;
  out->fwd_cta_pairs = pairs_wanted(M, W, f.staged);
  out->fwd_q_small_m = qsmall_wanted(M, W, f.staged);
  if (out->fwd_q_small_m) out->fwd_cta_pairs = 0;
  out->bwd_ok = b.vc > 0;
  out->bwd_chunk = b.vc;
  out->bwd_ksplit = b.ksplit;
  out->bwd_staged = b.staged;
  out->bwd_cta_pairs = b.vc > 0 && b.pairs;
  const FusedPlan fp = plan_fused(M, h_dtype, W, false);
  if (fp.ok && fp.total <= ws_bytes) {
    out->bwd_ok = 1;
    out->bwd_fused = 1;
    out->bwd_chunk = 0;
    out->bwd_ksplit = 1;
    out->bwd_staged = 0;
    out->bwd_cta_pairs = fp.c2 ? 1 : 0;
    out->bwd_fused_groups = fp.a.G;
    out->bwd_fused_members = fp.a.C;
    out->bwd_fused_buffers = fp.nbuf;
  }
  const SlicePlan sp = plan_slice(M, h_dtype, W, false);
  if (sp.ok && sp.total <= ws_bytes) {
    out->bwd_fused = 0;
    out->bwd_fused_groups = 0;
    out->bwd_fused_members = 0;
    out->bwd_fused_buffers = 0;
    out->bwd_ok = 1;
    out->bwd_chunk = 0;
    out->bwd_ksplit = 1;
    out->bwd_staged = 0;
    out->bwd_cta_pairs = 0;
    out->bwd_sliced = 1;
    out->bwd_sliced_clusters = sp.a.n_cl;
    out->bwd_sliced_ctas = sp.a.Ccl;
  }
  return CCE_OK;
}

int64_t cce_query_fused_schedule(int64_t M, cce_dtype h_dtype, const cce_head* W,
                                 int32_t* out, int64_t cap) {
  if (M <= 0 || M > (int64_t(1) << 30) || check_head(W, h_dtype) != CCE_OK) return -1;
  const FusedPlan fp = plan_fused(M, h_dtype, W, false);
  if (!fp.ok) return -1;
  int64_t n = 0;
  for (int g = 0; g < fp.a.G; ++g) {
    const int nu = fb_units(fp.a, g);
    for (int u = 0; u < nu; ++u, ++n) {
      if (out == nullptr || n >= cap) continue;
      const FUnit x = fb_unit(fp.a, g, u);
      int32_t* o = out + 6 * n;
      o[0] = g;
      o[1] = x.r;
      o[2] = x.j;
      o[3] = x.first ? 1 : 0;
      o[4] = x.last ? 1 : 0;
      o[5] = x.buf;
    }
  }
  return n;
}

int64_t cce_blockmax_cols(int64_t V) { return V <= 0 ? 0 : ceil_div(V, BN); }

size_t cce_workspace_bytes(int64_t M, cce_dtype h_dtype, const cce_head* W) {
  if (M <= 0 || check_head(W, h_dtype) != CCE_OK) return 0;
  const SlicePlan sp = plan_slice(M, h_dtype, W, false);
  if (sp.ok) return sp.total;
  const FusedPlan fp = plan_fused(M, h_dtype, W, false);
  if (fp.ok) return fp.total;
  const bool staged = q_stage_wanted(M, W, false);  // the backward stages first
  return make_layout(M, h_dtype, W, default_vc(M, W),
                     ksplit_for(M, W, sm_count_guess(), staged), staged)
      .total;
}

size_t cce_workspace_min_bytes(int64_t M, cce_dtype h_dtype, const cce_head* W) {
  if (M <= 0 || check_head(W, h_dtype) != CCE_OK) return 0;
  return make_layout(M, h_dtype, W, BN, 1).total;  // narrowest chunk, no K split
}

cce_status cce_forward(const void* H, cce_dtype h_dtype, int64_t M, const cce_head* W,
                       const int32_t* labels, float* logp, float* lse, float* tgt_logit,
                       float* blockmax, void* ws, size_t ws_bytes, cce_stream_t stream) {
  if (H == nullptr || labels == nullptr || logp == nullptr || lse == nullptr || ws == nullptr)
    return CCE_ERR_INVALID_ARGUMENT;
  if (M <= 0 || M > (int64_t(1) << 30)) return CCE_ERR_INVALID_ARGUMENT;
  if (h_dtype != CCE_F32 && h_dtype != CCE_BF16) return CCE_ERR_INVALID_ARGUMENT;
  if (!aligned16(H) || !aligned16(ws)) return CCE_ERR_INVALID_ARGUMENT;
  cce_status s = check_head(W, h_dtype);
  if (s != CCE_OK) return s;
  if (!tiles_fit(M, W)) return CCE_ERR_UNSUPPORTED;
  // A staged 4/8-bit head takes the widest fp16 chunk the workspace holds.
  const FwdPlan plan = plan_forward(M, h_dtype, W, ws_bytes);
  const bool staged = plan.staged;
  const int64_t vq = plan.vq;
  const Layout& L = plan.L;
  if (L.total > ws_bytes) return CCE_ERR_WORKSPACE_TOO_SMALL;
  int sms = 0;
  if ((s = device_info(&sms)) != CCE_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* wsc = static_cast<char*>(ws);

  Operands op;
  if ((s = prepare_operands(H, h_dtype, M, W, L, ws, st, &op)) != CCE_OK) return s;
  const int64_t V = W->V;
  const int64_t cols = ceil_div(V, BN);
  const int64_t n_rt = ceil_div(M, BM);
  float* part_s = reinterpret_cast<float*>(wsc + L.part_s);
  float* part_m = blockmax != nullptr ? blockmax : reinterpret_cast<float*>(wsc + L.part_m);
  float* tgt = tgt_logit != nullptr ? tgt_logit : reinterpret_cast<float*>(wsc + L.tgt);

  if (op.qb && qsmall_wanted(M, W, staged)) {
    if ((s = qsmall_forward(op, W, M, qsmall_wanted(M, W, staged) == 2, sms, st, labels, part_m,
                            part_s, tgt, status_word(ws))) != CCE_OK)
      return s;
  } else {
  const int max_pairs = pairs_wanted(M, W, staged) ? device_pairs() : 0;
  const bool pairs = max_pairs > 0;  // forward tiles need no K split
  CUtensorMap ma, mb;
  if (!make_map(&ma, op.a, op.bf16, op.k, M, op.ld_a, BK, BM)) return CCE_ERR_CUDA;
  if (op.qb) {
    // kLse: one group of 64 weights of 256 rows per K step
    if (!make_packed_map(&mb, W, op.qb, 64 * op.qb / 8, BN)) return CCE_ERR_CUDA;
  } else if (staged) {
    mb = ma;  // set per staged chunk
  } else if (!make_map(&mb, op.b, op.bf16, op.k, V, op.ld_b, BK, pairs ? BN / 2 : BN))
    return CCE_ERR_CUDA;

  TileArgs a;
  std::memset(&a, 0, sizeof(a));
  a.M = int(M);
  a.n_rt = int(n_rt);
  a.n_ct = int(cols);
  a.nk = int(op.k / BK);
  a.npass = 1;
  a.b_row0 = 0;
  a.V = int(V);
  a.D = int(W->D);
  a.fmt = op.bf16 ? 1 : 0;
  a.wait_ns = g_wait_ns.load();
  a.status = status_word(ws);
  a.labels = labels;
  a.part_m = part_m;
  a.part_s = part_s;
  a.tgt = tgt;
  a.ct_off = 0;
  a.q_w = static_cast<const uint32_t*>(W->w);
  a.q_scale = static_cast<const uint16_t*>(W->scales);
  a.q_bias = static_cast<const uint16_t*>(W->biases);
  a.group_rt = group_rows(n_rt, op.k);
  a.softcap = W->softcap;
  a.inv_cap = W->softcap > 0.f ? 1.f / W->softcap : 0.f;
  a.n_rt128 = int(n_rt);
  // One launch over the whole vocabulary, or one per staged chunk.
  const int64_t step = staged ? vq : cols * BN;
  for (int64_t v0 = 0; v0 < V; v0 += step) {
    const int64_t w = std::min<int64_t>(step, V - v0);
    const int64_t ct_n = ceil_div(w, BN);
    TileArgs ac = a;
    if (staged) {
      if ((s = stage_chunk(op, W, v0, w, sms, st)) != CCE_OK) return s;
      if (!make_map(&mb, op.b, false, op.k, w, op.ld_b, BK, pairs ? BN / 2 : BN))
        return CCE_ERR_CUDA;
      ac.n_ct = int(ct_n);
      ac.b_row0 = int(v0);
      ac.b_shift = int(v0);
      ac.ct_off = int(v0 / BN);
    }
    ProfScope ps(PK_LSE, st);
    if (pairs) {
      TileArgs a2 = ac;
      a2.n_rt = int(ceil_div(M, 2 * BM));
      a2.group_rt = std::max(1, ac.group_rt / 2);
      if (launch_tc_pairs<Mode::kLse>(int64_t(a2.n_rt) * ct_n, max_pairs, st, ma, mb, ma, ma,
                                      a2) != cudaSuccess)
        return CCE_ERR_CUDA;
    } else {
      launch_tc<Mode::kLse>(op.qb, n_rt * ct_n, sms, st, ma, mb, ma, ma, ac);
    }
    if (launch_ok() != CCE_OK) return CCE_ERR_CUDA;
  }
  }

  const int rows_per_block = 8;
  {
    ProfScope ps(PK_MERGE, st);
    merge_lse_kernel<<<int(ceil_div(M, rows_per_block)), rows_per_block * 32, 0, st>>>(
        part_m, part_s, int(cols), int(M), labels, int(V), tgt, logp, lse, status_word(ws));
  }
  return launch_ok();
}

// allow_empty: a shard of a row-sharded pair may hold no chosen or rejected
// row; emptiness of the whole pair shows in the all-reduced counts instead.
static cce_status check_layout(const cce_layout* L, int64_t M, bool allow_empty = false) {
  if (L == nullptr) return CCE_ERR_INVALID_ARGUMENT;
  const int64_t r[3][2] = {{L->prompt_begin, L->prompt_end},
                           {L->chosen_begin, L->chosen_end},
                           {L->rejected_begin, L->rejected_end}};
  for (int i = 0; i < 3; ++i) {
    if (r[i][0] < 0 || r[i][1] < r[i][0] || r[i][1] > M) return CCE_ERR_INVALID_ARGUMENT;
    for (int j = 0; j < i; ++j)
      if (r[i][0] < r[j][1] && r[j][0] < r[i][1]) return CCE_ERR_INVALID_ARGUMENT;
  }
  if (!allow_empty && (r[1][1] == r[1][0] || r[2][1] == r[2][0]))
    return CCE_ERR_INVALID_ARGUMENT;
  return CCE_OK;
}

static cce_status orpo_common(const float* logp, const int32_t* labels, int64_t M,
                              const cce_layout* layout, double lambda, int scope,
                              double* out8, float* coeff, void* ws, size_t ws_bytes,
                              cce_stream_t stream, int kind = 0, double beta = 1.0,
                              double gamma = 0.0, const double* sums_in = nullptr,
                              double* sums_out = nullptr) {
  if (labels == nullptr || ws == nullptr) return CCE_ERR_INVALID_ARGUMENT;
  if (logp == nullptr && sums_in == nullptr) return CCE_ERR_INVALID_ARGUMENT;
  if (M <= 0 || M > (int64_t(1) << 31)) return CCE_ERR_INVALID_ARGUMENT;
  if (!(lambda >= 0.0) || lambda > 1e30) return CCE_ERR_INVALID_ARGUMENT;
  if (kind < 0 || kind > 2 || !(beta >= 0.0) || beta > 1e30 || !(std::fabs(gamma) <= 1e30))
    return CCE_ERR_INVALID_ARGUMENT;
  if (scope != CCE_SCOPE_FULL && scope != CCE_SCOPE_RESPONSE) return CCE_ERR_INVALID_ARGUMENT;
  if (ws_bytes < kStatusBytes || !aligned16(ws)) return CCE_ERR_WORKSPACE_TOO_SMALL;
  const bool sharded = sums_in != nullptr || sums_out != nullptr;
  if ((sums_in != nullptr && !aligned8(sums_in)) || (sums_out != nullptr && !aligned8(sums_out)))
    return CCE_ERR_INVALID_ARGUMENT;
  cce_status s = check_layout(layout, M, sharded);
  if (s != CCE_OK) return s;
  OrpoArgs o{};
  o.sums_in = sums_in;
  o.sums_out = sums_out;
  o.pb = layout->prompt_begin;
  o.pe = layout->prompt_end;
  o.cb = layout->chosen_begin;
  o.ce = layout->chosen_end;
  o.rb = layout->rejected_begin;
  o.re = layout->rejected_end;
  o.lambda = lambda;
  o.scope = scope;
  o.want_coeff = coeff != nullptr;
  o.kind = kind;
  o.beta = beta;
  o.gamma = gamma;
  {
    ProfScope ps(PK_ORPO, reinterpret_cast<cudaStream_t>(stream));
    orpo_kernel<<<1, 1024, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        logp, labels, M, o, out8, coeff, status_word(ws));
  }
  return launch_ok();
}

cce_status orpo_loss_from_logps(const float* logp, const int32_t* labels, int64_t M,
                                const cce_layout* layout, double lambda, int sft_scope,
                                double* out8, void* ws, size_t ws_bytes,
                                cce_stream_t stream) {
  if (out8 == nullptr) return CCE_ERR_INVALID_ARGUMENT;
  return orpo_common(logp, labels, M, layout, lambda, sft_scope, out8, nullptr, ws,
                     ws_bytes, stream);
}

cce_status orpo_grad_coeffs(const float* logp, const int32_t* labels, int64_t M,
                            const cce_layout* layout, double lambda, int sft_scope,
                            float* coeff, void* ws, size_t ws_bytes, cce_stream_t stream) {
  if (coeff == nullptr) return CCE_ERR_INVALID_ARGUMENT;
  return orpo_common(logp, labels, M, layout, lambda, sft_scope, nullptr, coeff, ws,
                     ws_bytes, stream);
}

cce_status orpo_partial_sums(const float* logp, const int32_t* labels, int64_t M,
                             const cce_layout* layout, double* sums6, void* ws,
                             size_t ws_bytes, cce_stream_t stream) {
  if (sums6 == nullptr || logp == nullptr) return CCE_ERR_INVALID_ARGUMENT;
  return orpo_common(logp, labels, M, layout, 0.0, CCE_SCOPE_FULL, nullptr, nullptr, ws,
                     ws_bytes, stream, 0, 1.0, 0.0, nullptr, sums6);
}

cce_status orpo_from_sums(const double* sums6, const int32_t* labels, int64_t M,
                          const cce_layout* layout, double lambda, int sft_scope,
                          double* out8, float* coeff, void* ws, size_t ws_bytes,
                          cce_stream_t stream) {
  if (sums6 == nullptr || (out8 == nullptr && coeff == nullptr)) return CCE_ERR_INVALID_ARGUMENT;
  return orpo_common(nullptr, labels, M, layout, lambda, sft_scope, out8, coeff, ws, ws_bytes,
                     stream, 0, 1.0, 0.0, sums6, nullptr);
}

static cce_status objective_args(const cce_objective* obj) {
  if (obj == nullptr) return CCE_ERR_INVALID_ARGUMENT;
  if (obj->kind != CCE_OBJ_ORPO && obj->kind != CCE_OBJ_SIMPO && obj->kind != CCE_OBJ_ORPO_MARGIN)
    return CCE_ERR_INVALID_ARGUMENT;
  return CCE_OK;
}

cce_status pref_loss_from_logps(const float* logp, const int32_t* labels, int64_t M,
                                const cce_layout* layout, const cce_objective* obj,
                                double* out8, void* ws, size_t ws_bytes, cce_stream_t stream) {
  cce_status s = objective_args(obj);
  if (s != CCE_OK) return s;
  if (out8 == nullptr) return CCE_ERR_INVALID_ARGUMENT;
  return orpo_common(logp, labels, M, layout, obj->lambda, obj->sft_scope, out8, nullptr, ws,
                     ws_bytes, stream, int(obj->kind), obj->beta, obj->gamma);
}

cce_status pref_grad_coeffs(const float* logp, const int32_t* labels, int64_t M,
                            const cce_layout* layout, const cce_objective* obj, float* coeff,
                            void* ws, size_t ws_bytes, cce_stream_t stream) {
  cce_status s = objective_args(obj);
  if (s != CCE_OK) return s;
  if (coeff == nullptr) return CCE_ERR_INVALID_ARGUMENT;
  return orpo_common(logp, labels, M, layout, obj->lambda, obj->sft_scope, nullptr, coeff, ws,
                     ws_bytes, stream, int(obj->kind), obj->beta, obj->gamma);
}

static cce_status backward_impl(const void* H, cce_dtype h_dtype, int64_t M, const cce_head* W,
                                const int32_t* labels, const float* lse, const float* coeff,
                                float filter_eps, const float* blockmax, float* dH, float* dW,
                                unsigned long long* skip_stats, void* ws, size_t ws_bytes,
                                cce_stream_t stream);

cce_status cce_backward_dh(const void* H, cce_dtype h_dtype, int64_t M, const cce_head* W,
                           const int32_t* labels, const float* lse, const float* coeff,
                           float filter_eps, const float* blockmax, float* dH,
                           unsigned long long* skip_stats, void* ws, size_t ws_bytes,
                           cce_stream_t stream) {
  return backward_impl(H, h_dtype, M, W, labels, lse, coeff, filter_eps, blockmax, dH, nullptr,
                       skip_stats, ws, ws_bytes, stream);
}

cce_status cce_backward_dh_dw(const void* H, cce_dtype h_dtype, int64_t M, const cce_head* W,
                              const int32_t* labels, const float* lse, const float* coeff,
                              float filter_eps, const float* blockmax, float* dH, float* dW,
                              unsigned long long* skip_stats, void* ws, size_t ws_bytes,
                              cce_stream_t stream) {
  if (dW == nullptr || !aligned16(dW)) return CCE_ERR_INVALID_ARGUMENT;
  if (W != nullptr && W->format != CCE_W_DENSE) return CCE_ERR_UNSUPPORTED;
  return backward_impl(H, h_dtype, M, W, labels, lse, coeff, filter_eps, blockmax, dH, dW,
                       skip_stats, ws, ws_bytes, stream);
}

static cce_status backward_impl(const void* H, cce_dtype h_dtype, int64_t M, const cce_head* W,
                                const int32_t* labels, const float* lse, const float* coeff,
                                float filter_eps, const float* blockmax, float* dH, float* dW,
                                unsigned long long* skip_stats, void* ws, size_t ws_bytes,
                                cce_stream_t stream) {
  if (H == nullptr || labels == nullptr || lse == nullptr || coeff == nullptr ||
      dH == nullptr || ws == nullptr)
    return CCE_ERR_INVALID_ARGUMENT;
  if (M <= 0 || M > (int64_t(1) << 30)) return CCE_ERR_INVALID_ARGUMENT;
  if (h_dtype != CCE_F32 && h_dtype != CCE_BF16) return CCE_ERR_INVALID_ARGUMENT;
  if (!(filter_eps >= 0.f) || filter_eps > 1.f) return CCE_ERR_INVALID_ARGUMENT;
  if (!aligned16(H) || !aligned16(ws) || !aligned16(dH)) return CCE_ERR_INVALID_ARGUMENT;
  cce_status s = check_head(W, h_dtype);
  if (s != CCE_OK) return s;
  if (!tiles_fit(M, W)) return CCE_ERR_UNSUPPORTED;
  {
    // Dense bf16 heads take a fused kernel when the workspace holds its
    // (small) layout: by default the grouped one from 1,024 rows (the
    // sliced one only when mode 3 asks for it); the two GEMMs per vocab
    // chunk cover the rest.
    const SlicePlan sp = plan_slice(M, h_dtype, W, dW != nullptr);
    if (sp.ok && sp.total <= ws_bytes)
      return slice_backward(sp, H, W, labels, lse, coeff, filter_eps, blockmax, dH, skip_stats,
                            ws, reinterpret_cast<cudaStream_t>(stream));
    if (g_bwd_mode.load() == 3)
      return sp.ok ? CCE_ERR_WORKSPACE_TOO_SMALL : CCE_ERR_UNSUPPORTED;
    const FusedPlan fp = plan_fused(M, h_dtype, W, dW != nullptr);
    if (fp.ok && fp.total <= ws_bytes)
      return fused_backward(fp, H, W, labels, lse, coeff, filter_eps, blockmax, dH, skip_stats,
                            ws, reinterpret_cast<cudaStream_t>(stream));
    if (g_bwd_mode.load() == 1 && fp.ok) return CCE_ERR_WORKSPACE_TOO_SMALL;
  }
  // K split of the dH GEMM; fall back to fewer splits if the workspace
  // cannot hold their partial buffers.
  // A staged 4/8-bit head needs chunks of stage_min_rows at least; else the
  // GEMMs dequantise in-kernel.
  const BwdPlan plan = plan_backward(M, h_dtype, W, ws_bytes);
  if (plan.vc == 0) return CCE_ERR_WORKSPACE_TOO_SMALL;
  const bool staged = plan.staged;
  const int ksplit = plan.ksplit;
  const int64_t vc = plan.vc;
  const Layout& L = plan.L;
  int sms = 0;
  if ((s = device_info(&sms)) != CCE_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* wsc = static_cast<char*>(ws);

  Operands op;
  if ((s = prepare_operands(H, h_dtype, M, W, L, ws, st, &op)) != CCE_OK) return s;
  const int64_t V = W->V, D = W->D;
  const int64_t cols = ceil_div(V, BN);
  const int64_t n_rt = ceil_div(M, BM);
  const int64_t n_dt = ceil_div(D, BN);
  uint16_t* g = reinterpret_cast<uint16_t*>(wsc + L.g);
  uint8_t* tile_skip = reinterpret_cast<uint8_t*>(wsc + L.tile_skip);
  uint8_t* row_skip = reinterpret_cast<uint8_t*>(wsc + L.row_skip);

  // Plan: rows whose coefficient is 0 everywhere in a tile, and (with the
  // filter and blockmax) vocab blocks the filter would empty.
  {
    const int64_t units = n_rt * cols;
    const int wpb = 8;
    ProfScope ps(PK_SKIP, st);
    skip_plan_kernel<<<int(ceil_div(units, wpb)), wpb * 32, 0, st>>>(
        filter_eps > 0.f ? blockmax : nullptr, lse, labels, coeff, int(M), int(cols),
        int(n_rt), filter_eps, tile_skip, row_skip, skip_stats);
    if (launch_ok() != CCE_OK) return CCE_ERR_CUDA;
  }

  CUtensorMap ma, mb, mg, mw, mgs, md0, md1;
  const int max_pairs = plan.pairs ? device_pairs() : 0;
  const bool pairs = max_pairs > 0;
  if (!make_map(&ma, op.a, op.bf16, op.k, M, op.ld_a, BK, BM)) return CCE_ERR_CUDA;
  if (op.qb) {
    // packed tiles: kGrad as the forward, kDh 64 rows x 256 columns per K step
    if (!make_packed_map(&mb, W, op.qb, 64 * op.qb / 8, BN) ||
        !make_packed_map(&mw, W, op.qb, BN * op.qb / 8, BK))
      return CCE_ERR_CUDA;
  } else if (staged) {
    mb = ma;  // mapped per staged chunk
    mw = ma;
  } else if (!make_map(&mb, op.b, op.bf16, op.k, V, op.ld_b, BK, pairs ? BN / 2 : BN) ||
             !make_map(&mw, op.b, op.bf16, op.ld_b, V, op.ld_b, 64, BK)) {
    return CCE_ERR_CUDA;
  }
  {
    // dH and the K-split partial buffers as [nbuf, M, D] fp32, 32x32 boxes
    const uint64_t dd[3] = {uint64_t(D), uint64_t(M), 1};
    const uint64_t ds[2] = {uint64_t(D) * 4, uint64_t(M) * D * 4};
    const uint32_t db[3] = {32, 32, 1};
    if (!make_map_ex(&md0, dH, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, dd, ds, db,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return CCE_ERR_CUDA;
    md1 = md0;
    if (ksplit > 1) {
      const uint64_t pd[3] = {uint64_t(D), uint64_t(M), uint64_t(ksplit - 1)};
      if (!make_map_ex(&md1, wsc + L.dh_part, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, pd, ds, db,
                       CU_TENSOR_MAP_SWIZZLE_128B))
        return CCE_ERR_CUDA;
    }
  }

  TileArgs a;
  std::memset(&a, 0, sizeof(a));
  a.M = int(M);
  a.n_rt = int(n_rt);
  a.V = int(V);
  a.D = int(D);
  a.fmt = op.bf16 ? 1 : 0;
  a.wait_ns = g_wait_ns.load();
  a.status = status_word(ws);
  a.labels = labels;
  a.lse = lse;
  a.filter_eps = filter_eps;
  a.g_out = g;
  a.g_ld = int(vc);
  a.tile_skip = tile_skip;
  a.skip_ld = int(cols);
  a.row_skip = row_skip;
  a.coeff = coeff;
  a.dh = dH;
  a.dh_part = reinterpret_cast<float*>(wsc + L.dh_part);
  a.ksplit = ksplit;
  a.q_w = static_cast<const uint32_t*>(W->w);
  a.q_scale = static_cast<const uint16_t*>(W->scales);
  a.q_bias = static_cast<const uint16_t*>(W->biases);
  a.group_rt = group_rows(n_rt, op.k);
  a.softcap = W->softcap;
  a.inv_cap = W->softcap > 0.f ? 1.f / W->softcap : 0.f;
  a.n_rt128 = int(n_rt);
  const int64_t n_rt2 = ceil_div(M, 2 * BM);

  // Trainable head: B operand coeff * H and the dW output map.
  CUtensorMap mhg, mdw;
  __nv_bfloat16* hg = reinterpret_cast<__nv_bfloat16*>(wsc + L.hg);
  if (dW != nullptr) {
    {
      ProfScope ps(PK_SPLIT, st);
      if (h_dtype == CCE_F32)
        scale_rows_bf16_kernel<float><<<1184, 256, 0, st>>>(static_cast<const float*>(H), coeff, M,
                                                            int(D), hg);
      else
        scale_rows_bf16_kernel<__nv_bfloat16><<<1184, 256, 0, st>>>(
            static_cast<const __nv_bfloat16*>(H), coeff, M, int(D), hg);
    }
    if (launch_ok() != CCE_OK) return CCE_ERR_CUDA;
    const uint64_t wd[3] = {uint64_t(D), uint64_t(V), 1};
    const uint64_t wsd[2] = {uint64_t(D) * 4, uint64_t(V) * D * 4};
    const uint32_t wb[3] = {32, 32, 1};
    if (!make_map(&mhg, hg, true, D, M, D, 64, BK) ||
        !make_map_ex(&mdw, dW, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, wd, wsd, wb,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return CCE_ERR_CUDA;
  }

  for (int64_t v0 = 0; v0 < V; v0 += vc) {
    const int64_t w = std::min<int64_t>(vc, V - v0);
    const int64_t ct_n = ceil_div(w, BN);
    if (staged) {
      if ((s = stage_chunk(op, W, v0, w, sms, st)) != CCE_OK) return s;
      if (!make_map(&mb, op.b, false, op.k, w, op.ld_b, BK, pairs ? BN / 2 : BN) ||
          !make_map(&mw, op.b, false, op.ld_b, w, op.ld_b, 64, BK))
        return CCE_ERR_CUDA;
    }
    // G' = onehot - softmax for this chunk
    TileArgs ag = a;
    ag.b_shift = staged ? int(v0) : 0;
    ag.n_ct = int(ct_n);
    ag.nk = int(op.k / BK);
    ag.npass = 1;
    ag.b_row0 = int(v0);
    ag.ct_off = int(v0 / BN);
    ag.zero_skip_rows = dW != nullptr ? 1 : 0;
    {
      // G'' store map: [M, chunk columns] 16-bit, 32x32 boxes, 64-byte swizzle
      const uint64_t gd[2] = {uint64_t(ct_n * BN), uint64_t(M)};
      const uint64_t gs[1] = {uint64_t(vc) * 2};
      const uint32_t gb[2] = {32, 32};
      if (!make_map_ex(&mgs, g, op.bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                         : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                       2, gd, gs, gb, CU_TENSOR_MAP_SWIZZLE_64B))
        return CCE_ERR_CUDA;
    }
    {
      ProfScope ps(PK_GRAD, st);
      if (pairs) {
        TileArgs a2 = ag;
        a2.n_rt = int(n_rt2);
        a2.group_rt = std::max(1, ag.group_rt / 2);
        if (launch_tc_pairs<Mode::kGrad>(n_rt2 * ct_n, max_pairs, st, ma, mb, mgs, mgs, a2) !=
            cudaSuccess)
          return CCE_ERR_CUDA;
      } else {
        launch_tc<Mode::kGrad>(op.qb, n_rt * ct_n, sms, st, ma, mb, mgs, mgs, ag);
      }
    }
    if (launch_ok() != CCE_OK) return CCE_ERR_CUDA;
    // dH (+)= coeff * G' . W[chunk]
    if (!make_map(&mg, g, op.bf16, ct_n * BN, M, vc, BK, BM)) return CCE_ERR_CUDA;
    TileArgs ad = a;
    ad.n_ct = int(n_dt);
    ad.nk = int(ct_n * BN / BK);
    ad.npass = op.npass_dh;
    ad.b_pass_off = int(op.d_pass_off);
    ad.b_row0 = int(v0);
    ad.b_shift = staged ? int(v0) : 0;
    ad.first_chunk = v0 == 0 ? 1 : 0;
    {
      ProfScope ps(PK_DH, st);
      if (pairs) {
        TileArgs a2 = ad;
        a2.n_rt = int(n_rt2);
        if (launch_tc_pairs<Mode::kDh>(n_rt2 * n_dt * ksplit, max_pairs, st, mg, mw, md0, md1,
                                       a2) != cudaSuccess)
          return CCE_ERR_CUDA;
      } else {
        launch_tc<Mode::kDh>(op.qb, n_rt * n_dt * ksplit, sms, st, mg, mw, md0, md1, ad);
      }
    }
    if (launch_ok() != CCE_OK) return CCE_ERR_CUDA;
    if (dW != nullptr) {
      // dW[v0 : v0 + w] = -(G''^T . coeff*H): vocab tiles of 128 rows, K = M.
      CUtensorMap mga;
      if (!make_map(&mga, g, true, ct_n * BN, M, vc, 64, BK)) return CCE_ERR_CUDA;
      TileArgs aw = a;
      aw.n_rt = int(ct_n * BN / BM);
      aw.n_ct = int(n_dt);
      aw.nk = int(ceil_div(M, BK));
      aw.npass = 1;
      aw.b_row0 = int(v0);
      aw.ksplit = 1;
      aw.fmt = 1;
      {
        ProfScope ps(PK_DW, st);
        cce_tc_kernel<Mode::kDw, 0><<<grid_for(int64_t(aw.n_rt) * n_dt, sms), NUM_THREADS,
                                      smem_bytes<Mode::kDw>(), st>>>(mga, mhg, mdw, mdw, aw);
      }
      if (launch_ok() != CCE_OK) return CCE_ERR_CUDA;
    }
  }
  if (ksplit > 1) {
    ProfScope ps(PK_DHSUM, st);
    const int64_t n4 = M * D / 4;
    add_parts_kernel<<<std::max<int>(1, std::min<int64_t>(ceil_div(n4, 256), 4 * sms)), 256, 0,
                       st>>>(reinterpret_cast<float4*>(dH),
                             reinterpret_cast<const float4*>(wsc + L.dh_part), ksplit - 1, n4);
    if (launch_ok() != CCE_OK) return CCE_ERR_CUDA;
  }
  return CCE_OK;
}


void cce_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto& r : g_prof) {
    g_ev_pool.push_back(r.a);
    g_ev_pool.push_back(r.b);
  }
  g_prof.clear();
  g_prof_on = on != 0;
}

int cce_profile_read(double* ms, long long* launches, int n) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (int k = 0; k < n && k < PK_N; ++k) {
    if (ms != nullptr) ms[k] = 0.0;
    if (launches != nullptr) launches[k] = 0;
  }
  for (auto& r : g_prof) {
    float t = 0.f;
    if (cudaEventSynchronize(r.b) == cudaSuccess &&
        cudaEventElapsedTime(&t, r.a, r.b) == cudaSuccess && r.kind < n) {
      if (ms != nullptr) ms[r.kind] += t;
      if (launches != nullptr) launches[r.kind] += (r.kind == PK_SPLIT) ? 2 : 1;
    }
    g_ev_pool.push_back(r.a);
    g_ev_pool.push_back(r.b);
  }
  g_prof.clear();
  return PK_N;
}

const char* cce_profile_kind_name(int kind) {
  return (kind >= 0 && kind < PK_N) ? kProfNames[kind] : "unknown";
}

static cce_status prefix_args(int64_t P, int64_t Rc, int64_t Rr, int64_t D) {
  if (P < 1 || Rc < 1 || Rr < 1 || D <= 0) return CCE_ERR_INVALID_ARGUMENT;
  if (P + Rc + Rr > (int64_t(1) << 31) || D > (int64_t(1) << 20)) return CCE_ERR_INVALID_ARGUMENT;
  return CCE_OK;
}

cce_status cce_prefix_gather(const void* H_cat, cce_dtype dtype, int64_t P, int64_t Rc,
                             int64_t Rr, int64_t D, void* H_head, cce_stream_t stream) {
  if (H_cat == nullptr || H_head == nullptr) return CCE_ERR_INVALID_ARGUMENT;
  if (dtype != CCE_F32 && dtype != CCE_BF16) return CCE_ERR_INVALID_ARGUMENT;
  cce_status s = prefix_args(P, Rc, Rr, D);
  if (s != CCE_OK) return s;
  const int64_t row_bytes = D * (dtype == CCE_F32 ? 4 : 2);
  if (row_bytes % 16 != 0 || !aligned16(H_cat) || !aligned16(H_head)) return CCE_ERR_INVALID_ARGUMENT;
  const int64_t M = P + Rc + Rr, row16 = row_bytes / 16;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  ProfScope ps(PK_PREFIX, st);
  prefix_gather_kernel<<<int(std::min<int64_t>(ceil_div(M * row16, 256), 4096)), 256, 0, st>>>(
      static_cast<const uint4*>(H_cat), M, P, Rc, row16, static_cast<uint4*>(H_head));
  return launch_ok();
}

cce_status cce_prefix_scatter(const float* dH_head, int64_t P, int64_t Rc, int64_t Rr, int64_t D,
                              float* dH_cat, cce_stream_t stream) {
  if (dH_head == nullptr || dH_cat == nullptr) return CCE_ERR_INVALID_ARGUMENT;
  cce_status s = prefix_args(P, Rc, Rr, D);
  if (s != CCE_OK) return s;
  if (D % 4 != 0 || !aligned16(dH_head) || !aligned16(dH_cat)) return CCE_ERR_INVALID_ARGUMENT;
  const int64_t M = P + Rc + Rr, row4 = D / 4;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  ProfScope ps(PK_PREFIX, st);
  prefix_scatter_kernel<<<int(std::min<int64_t>(ceil_div(M * row4, 256), 4096)), 256, 0, st>>>(
      reinterpret_cast<const float4*>(dH_head), M, P, Rc, row4, reinterpret_cast<float4*>(dH_cat));
  return launch_ok();
}

cce_status cce_device_status(void* ws, cce_stream_t stream) {
  if (ws == nullptr) return CCE_ERR_INVALID_ARGUMENT;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return CCE_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, ws, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return CCE_ERR_CUDA;
  if (word != 0) {
    const uint32_t zero = 0;
    if (cudaMemcpy(ws, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return CCE_ERR_CUDA;
  }
  if (word & ST_LABEL) return CCE_ERR_LABEL_OUT_OF_RANGE;
  if (word & ST_TIMEOUT) return CCE_ERR_DEVICE_TIMEOUT;
  if (word & ST_EMPTY) return CCE_ERR_EMPTY_SEGMENT;
  if (word & ST_DOMAIN) return CCE_ERR_DOMAIN;
  if (word & ST_FP16) return CCE_ERR_FP16_RANGE;
  return CCE_OK;
}

cce_status cce_selftest_wait_timeout(void* ws, size_t ws_bytes, cce_stream_t stream) {
  if (ws == nullptr || ws_bytes < kStatusBytes || !aligned16(ws)) return CCE_ERR_INVALID_ARGUMENT;
  ProfScope ps(PK_SELFTEST, reinterpret_cast<cudaStream_t>(stream));
  selftest_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      status_word(ws), g_wait_ns.load());
  return launch_ok();
}

}  // extern "C"

// ========================================================================
// Forward without a caller workspace.
//
// Some callers cannot allocate device memory: plugins and plain-C hosts that
// receive only input and output pointers from a framework owning every
// device allocation, and runtimes whose memory budget is fixed at start-up
// and may not grow afterwards.  For them cce_forward_noalloc runs the same
// forward kernels with their scratch (per-block partials, the gathered target
// logits and the status word) in the fixed-size device array below.  The
// array is a module global: every GPU that loads this library holds it until
// the process exits.
namespace {

constexpr size_t kNoallocBytes = size_t(CCE_NOALLOC_SCRATCH_BYTES);
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {};

// Device address of the scratch array on the current device, looked up once
// per device (host code only sees a host-side stand-in for the symbol).
cce_status noalloc_scratch(char** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return CCE_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return CCE_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = static_cast<char*>(g_noalloc_ptr[dev]);
  return CCE_OK;
}

}  // namespace

extern "C" cce_status cce_forward_noalloc(const void* H, int64_t M, const cce_head* W,
                                          const int32_t* labels, float* logp, float* lse,
                                          float* tgt_logit, float* blockmax,
                                          uint32_t* status, cce_stream_t stream) {
  if (H == nullptr || labels == nullptr || logp == nullptr || lse == nullptr)
    return CCE_ERR_INVALID_ARGUMENT;
  if (M <= 0 || M > (int64_t(1) << 30) || !aligned16(H)) return CCE_ERR_INVALID_ARGUMENT;
  cce_status s = check_head(W, CCE_BF16);
  if (s != CCE_OK) return s;
  if (W->format != CCE_W_DENSE) return CCE_ERR_UNSUPPORTED;
  const int64_t V = W->V, D = W->D;
  const int64_t cols = ceil_div(V, BN);
  const int64_t n_rt = ceil_div(M, BM);
  // scratch: status word | part_s [cols, M] | part_m [cols, M] | tgt [M];
  // part_m and tgt take room only when the caller did not pass blockmax or
  // tgt_logit (those outputs are then written directly).
  const size_t o_s = kStatusBytes;
  const size_t o_m = o_s + align_up(size_t(cols) * M * 4);
  const size_t o_t = o_m + (blockmax != nullptr ? 0 : align_up(size_t(cols) * M * 4));
  const size_t need = o_t + (tgt_logit != nullptr ? 0 : align_up(size_t(M) * 4));
  if (need > kNoallocBytes) return CCE_ERR_WORKSPACE_TOO_SMALL;
  int sms = 0;
  if ((s = device_info(&sms)) != CCE_OK) return s;
  char* scr = nullptr;
  if ((s = noalloc_scratch(&scr)) != CCE_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  uint32_t* st_word = status != nullptr ? status : reinterpret_cast<uint32_t*>(scr);
  if (cudaMemsetAsync(st_word, 0, sizeof(uint32_t), st) != cudaSuccess) return CCE_ERR_CUDA;
  float* part_s = reinterpret_cast<float*>(scr + o_s);
  float* part_m = blockmax != nullptr ? blockmax : reinterpret_cast<float*>(scr + o_m);
  float* tgt = tgt_logit != nullptr ? tgt_logit : reinterpret_cast<float*>(scr + o_t);

  CUtensorMap ma, mb;
  if (!make_map(&ma, H, true, D, M, D, BK, BM) || !make_map(&mb, W->w, true, D, V, D, BK, BN))
    return CCE_ERR_CUDA;
  TileArgs a;
  std::memset(&a, 0, sizeof(a));
  a.M = int(M);
  a.n_rt = int(n_rt);
  a.n_ct = int(cols);
  a.nk = int(D / BK);
  a.npass = 1;
  a.V = int(V);
  a.D = int(D);
  a.fmt = 1;
  a.wait_ns = g_wait_ns.load();
  a.status = st_word;
  a.group_rt = int(n_rt);
  a.softcap = W->softcap;
  a.inv_cap = W->softcap > 0.f ? 1.f / W->softcap : 0.f;
  a.labels = labels;
  a.part_m = part_m;
  a.part_s = part_s;
  a.tgt = tgt;
  cce_tc_kernel<Mode::kLse, 0><<<grid_for(n_rt * cols, sms), NUM_THREADS, SMEM_BYTES, st>>>(
      ma, mb, ma, ma, a);
  if (launch_ok() != CCE_OK) return CCE_ERR_CUDA;
  const int rows_per_block = 8;
  merge_lse_kernel<<<int(ceil_div(M, rows_per_block)), rows_per_block * 32, 0, st>>>(
      part_m, part_s, int(cols), int(M), labels, int(V), tgt, logp, lse, st_word);
  return launch_ok();
}
