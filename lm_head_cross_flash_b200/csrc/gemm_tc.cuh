// gemm_tc.cuh — the persistent, warp-specialised tcgen05 GEMM that carries
// the three tensor-core steps of the flash-CCE head, each with its own fused
// epilogue:
//
//   kLse  : S = H . W^T tile (128 rows x 256 vocab) -> online max / sum-exp
//           per row and per vocab block, plus the target-logit gather.
//           (Training design §5.1; ORPO design 0.0.6, fused-head spec,
//           "Forward (online-softmax over vocab tiles)".)
//   kGrad : S recomputed -> G' = onehot - softmax (with the optional coeff
//           filter) for one vocab chunk, stored as 16-bit [M, chunk].
//           (ORPO design 0.0.6, fused-head spec, "Backward".)
//   kDh   : dH[:, d-tile] (+)= coeff * (G'[:, chunk] . W[chunk, d-tile]),
//           fp32 accumulation in TMEM and across chunks.
//   kDw   : dW[chunk rows, d-tile] = -(G'^T . coeff*H) (trainable head),
//           both operands MN-major.
//
// Roles (192 threads): warp 0 issues TMA loads into a 4-stage shared-memory
// ring; warp 1 owns the TMEM allocation and issues tcgen05.mma (M=128,
// N=256, K=16) into one of two 256-column fp32 accumulators; warps 2-5 drain
// the accumulator with tcgen05.ld (warp w reads TMEM lanes 32*(w%4)..+31,
// i.e. one row per thread) and run the epilogue, overlapping the MMA of the
// next tile.  A quantised head (QB = 4 or 8) adds 8 warps that dequantise
// the B half of every stage (3 stages, each also holding the packed B tile).  Tiles are assigned round-robin over a grid of
// at most one CTA per SM, in the order tile_coord gives (below), so the CTAs
// in flight share the operand that should stay in L2.
//
// C2 = true runs the same roles on clusters of two CTAs (one TPC) computing
// a 256x256 tile per pair with tcgen05.mma.cta_group::2 (M=256): each CTA
// loads its own 128 rows of A and one half of B into a 6-stage ring of 32 KB
// stages, both CTAs' copies complete on the leader CTA's full barrier, only
// the leader issues MMAs, and tcgen05.commit with a CTA mask signals both
// CTAs' stage-free and accumulator-full barriers.  Each CTA drains its own
// 128 TMEM lanes; the leader's accumulator-empty barrier counts both CTAs'
// epilogue threads.  No copy is multicast.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace cce {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int NUM_THREADS = 192;     // TMA, MMA, 4 epilogue warps
constexpr int DQ_WARPS = 8;          // dequantisation warps (4-bit head), 2 per SMSP
constexpr int NUM_THREADS_Q4 = NUM_THREADS + 32 * DQ_WARPS;
constexpr int DQ_WARP0 = 6;
constexpr uint32_t TMEM_COLS = 2 * BN;
enum class Mode : int { kLse = 0, kGrad = 1, kDh = 2, kDw = 3 };

// Epilogue staging for TMA stores: per epilogue warp two buffers of
// 32 rows x 32 columns (kGrad: 16-bit G'', 64-byte rows; kDh: fp32 dH,
// 128-byte rows).
template <Mode MODE>
__host__ __device__ constexpr int staging_buf_bytes() {
  return MODE == Mode::kGrad ? 32 * 64 : (MODE == Mode::kDh || MODE == Mode::kDw) ? 32 * 128 : 0;
}
// CTA pairs (cta_group::2): a 256x256 tile per pair, each CTA loads its 128
// rows of A and half (128 columns) of B, so a stage is 32 KB and 6 fit.
constexpr int STAGES2 = 6;
constexpr int B_HALF_BYTES = (BN / 2) * BK * 2;
constexpr int STAGE2_BYTES = A_BYTES + B_HALF_BYTES;
// Quantised heads (QB = 4 or 8) dequantise B in-kernel.  Each of their 3
// stages also holds the packed weights of its B tile, brought in by TMA
// (kLse/kGrad: 256 rows x one group of 64; kDh: 64 rows x 256 columns).
constexpr int STAGES_Q = 3;
template <Mode MODE, int QB>
__host__ __device__ constexpr int pk_bytes() {
  return MODE == Mode::kDh ? BK * (BN * QB / 8) : BN * (64 * QB / 8);
}
template <Mode MODE, bool C2 = false, int QB = 0>
__host__ __device__ constexpr int smem_bytes() {
  return (C2 ? STAGES2 * STAGE2_BYTES
             : QB ? STAGES_Q * (STAGE_BYTES + pk_bytes<MODE, QB>()) : STAGES * STAGE_BYTES) +
         4 * 2 * staging_buf_bytes<MODE>() + 1024 + 256;
}
constexpr int SMEM_BYTES = smem_bytes<Mode::kLse>();
constexpr float LOG2E = 1.4426950408889634f;
// fp16 G'' (4/8-bit heads) is stored times 2^14 so that the probabilities of
// a flat softmax over a large vocabulary (about 5e-6 at V = 128k) stay out of
// fp16 subnormals; |G''| <= 1 keeps it below 16,384.  The dH epilogue takes
// the factor out again in fp32.  bf16 G'' is stored unscaled.
constexpr float G16_SCALE = 16384.f;
constexpr float G16_UNSCALE = 1.f / 16384.f;
constexpr uint64_t DRAIN_LIMIT_NS = 1000000000ull;


struct TileArgs {
  int M;         // rows of A (head rows)
  int n_rt;      // row tiles
  int n_ct;      // column tiles of this launch
  int nk;        // K steps of BK per pass
  int npass;     // passes over K (kDh: hi/lo halves of a split f32 head)
  int b_pass_off;  // kDh: B inner-coordinate offset of pass 1
  int b_row0;    // kLse/kGrad: first vocab row of this launch; kDh: chunk v0
  int b_shift;   // B tensor-map row of vocab row v is v - b_shift (a staged chunk)
  int V;
  int D;
  int fmt;       // operand format: 0 = f16, 1 = bf16
  uint64_t wait_ns;
  uint32_t* status;
  const int32_t* labels;
  // kLse
  float* part_m;  // [cols, M]
  float* part_s;  // [cols, M]
  float* tgt;     // [M]
  int ct_off;     // global vocab-block index of column tile 0
  // kGrad
  const float* lse;
  float filter_eps;
  uint16_t* g_out;  // [M, g_ld] 16-bit
  int g_ld;
  const uint8_t* tile_skip;  // [n_rt_total, skip_ld] or null
  int skip_ld;
  const uint8_t* row_skip;   // [n_rt] or null
  // kDh
  const float* coeff;
  float* dh;       // [M, D]; K-split 0 accumulates here
  float* dh_part;  // K-split s >= 1 accumulates in dh_part + (s-1)*M*D
  int ksplit;      // kDh: the chunk's K range is split in `ksplit` parts
  int first_chunk;
  int group_rt;    // kLse/kGrad: row tiles per raster group
  int zero_skip_rows;  // kGrad: write zeros (not nothing) for row-skipped tiles
  int n_rt128;     // 128-row tiles of A (pairs: n_rt counts 256-row tiles)
  float softcap;   // > 0: logits are cap * tanh(s / cap)
  float inv_cap;
  // 4-bit affine head (group 64): words [V, D/8], scales/biases bf16 [V, D/64]
  const uint32_t* q_w;
  const uint16_t* q_scale;
  const uint16_t* q_bias;
};

// Position, inside its block of 8, at which the dequantiser stores element e
// of the block.  4-bit: the int4 -> fp16 conversion yields the pairs
// (e0,e4), (e1,e5), (e2,e6), (e3,e7); 8-bit: the pairs (e0,e2), (e1,e3) of
// each word.  The hidden rows are stored with the same order along K, so
// every dot product is unchanged.
__host__ __device__ constexpr int q4_pos(int e) { return e < 4 ? 2 * e : 2 * e - 7; }
__host__ __device__ constexpr int q8_pos(int e) {
  return (e & 4) + ((e & 3) == 1 ? 2 : (e & 3) == 2 ? 1 : (e & 3));
}
template <int QB>
__host__ __device__ constexpr int qpos(int e) {
  return QB == 8 ? q8_pos(e) : QB == 4 ? q4_pos(e) : e;
}

// 8-bit variant: 16 packed words (element 4c+j = byte j of word c).
__device__ __forceinline__ void dequant_group64_q8(const uint4 (&wv)[4], uint16_t sbits,
                                                   uint16_t bbits, uint4 (&out)[8]) {
  const __half2 s2 = __float2half2_rn(__uint_as_float(static_cast<uint32_t>(sbits) << 16));
  const __half2 b2 = __float2half2_rn(__uint_as_float(static_cast<uint32_t>(bbits) << 16));
  const __half2 k1024 = __float2half2_rn(1024.f);
  const uint32_t words[16] = {wv[0].x, wv[0].y, wv[0].z, wv[0].w, wv[1].x, wv[1].y,
                              wv[1].z, wv[1].w, wv[2].x, wv[2].y, wv[2].z, wv[2].w,
                              wv[3].x, wv[3].y, wv[3].z, wv[3].w};
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint32_t t[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t x = ((words[2 * c + (i >> 1)] >> (8 * (i & 1))) & 0x00FF00FFu) | 0x64006400u;
      __half2 h = *reinterpret_cast<const __half2*>(&x);
      h = __hfma2(__hsub2(h, k1024), s2, b2);
      t[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    out[c] = make_uint4(t[0], t[1], t[2], t[3]);
  }
}

// Dequantise the 64 weights of one (row, group): w = q * scale + bias, with
// q read from 8 packed words (element 8c+j = bits 4j..4j+3 of word c) and
// the result rounded once to fp16 (fma.rn.f16x2 on q, scale, bias, all exact
// in fp16).  q comes from the bit pattern 0x6400 | q = 1024 + q in fp16.
// out[c] holds the 8 fp16 values of word c in q4_pos order.
__device__ __forceinline__ void dequant_group64(const uint4& wa, const uint4& wb, uint16_t sbits,
                                                uint16_t bbits, uint4 (&out)[8]) {
  const __half2 s2 = __float2half2_rn(__uint_as_float(static_cast<uint32_t>(sbits) << 16));
  const __half2 b2 = __float2half2_rn(__uint_as_float(static_cast<uint32_t>(bbits) << 16));
  const __half2 k1024 = __float2half2_rn(1024.f);
  const uint32_t words[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint32_t t[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t x = ((words[c] >> (4 * i)) & 0x000F000Fu) | 0x64006400u;
      __half2 h = *reinterpret_cast<const __half2*>(&x);
      h = __hfma2(__hsub2(h, k1024), s2, b2);
      t[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    out[c] = make_uint4(t[0], t[1], t[2], t[3]);
  }
}

// Tile t of a launch.  kLse/kGrad: row tiles are taken in groups of
// `group_rt` (sized so a group of H rows stays in L2); inside a group the row
// tile is fastest, so the CTAs in flight share one vocab tile of W, and the
// group sweeps the whole vocabulary before the next group starts.  kDh:
// d-tile fastest, then row tile, then K split, so the CTAs in flight share a
// G'' row tile and one K range of the W chunk.
struct TileCoord {
  int rt, ct, s;
};

template <Mode MODE>
__device__ __forceinline__ TileCoord tile_coord(const TileArgs& a, int t) {
  TileCoord c;
  if (MODE == Mode::kDh || MODE == Mode::kDw) {
    // K split outermost: the tiles in flight stream the same K range of the
    // W chunk (one wave reads 1/ksplit of it), row tiles share G'' rows.
    const int per_s = a.n_ct * a.n_rt;
    c.s = t / per_s;
    const int r = t - c.s * per_s;
    c.ct = r % a.n_ct;
    c.rt = r / a.n_ct;
  } else {
    const int per_group = a.group_rt * a.n_ct;
    const int grp = t / per_group;
    const int r = t - grp * per_group;
    const int g0 = grp * a.group_rt;
    const int gn = min(a.group_rt, a.n_rt - g0);
    c.rt = g0 + r % gn;
    c.ct = r / gn;
    c.s = 0;
  }
  return c;
}

__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }

// 0 = compute, 1 = write zeros only, 2 = nothing.  s: the K split of a kDh
// tile; a split left without K steps (a chunk narrower than the split count)
// only zeroes its buffer on the first chunk.
template <Mode MODE>
__device__ __forceinline__ int tile_kind(const TileArgs& a, int rt, int ct, int s = 0) {
  if (MODE == Mode::kLse || MODE == Mode::kDw) return 0;
  const bool rs = a.row_skip != nullptr && a.row_skip[rt] != 0;
  if (MODE == Mode::kGrad) {
    if (rs) return a.zero_skip_rows ? 1 : 2;
    if (a.tile_skip != nullptr && a.tile_skip[rt * a.skip_ld + a.ct_off + ct]) return 1;
    return 0;
  }
  if (rs || (s + 1) * a.nk / a.ksplit == s * a.nk / a.ksplit) return a.first_chunk ? 1 : 2;
  return 0;
}

// Kind of a pair tile (two 128-row halves): computed when either half is.
template <Mode MODE>
__device__ __forceinline__ int pair_kind(const TileArgs& a, int rt2, int ct, int s) {
  const int k0 = tile_kind<MODE>(a, 2 * rt2, ct, s);
  const int k1 = 2 * rt2 + 1 < a.n_rt128 ? tile_kind<MODE>(a, 2 * rt2 + 1, ct, s) : 2;
  return (k0 == 0 || k1 == 0) ? 0 : 1;
}

template <Mode MODE, bool C2>
__device__ __forceinline__ int launch_kind(const TileArgs& a, int rt, int ct, int s) {
  return C2 ? pair_kind<MODE>(a, rt, ct, s) : tile_kind<MODE>(a, rt, ct, s);
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi, int fmt) {
  if (fmt == 1) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// tanh(x) from one ex2: t = 2^(2 x log2 e), tanh = (t - 1) / (t + 1); |x| is
// clamped at 15, where tanh is 1 to fp32 precision.  Absolute error ~1e-7.
__device__ __forceinline__ float tanh_ex2(float x) {
  x = fminf(fmaxf(x, -15.f), 15.f);
  const float t = ex2_approx(x * (2.f * LOG2E));
  return __fdividef(t - 1.f, t + 1.f);
}

// Softmax probability of logit s given nl = -lse * log2(e).  The block-skip
// planner uses the same expression, so its decisions agree with the filter.
__device__ __forceinline__ float softmax_p(float s, float nl) {
  return ex2_approx(fmaf(s, LOG2E, nl));
}

// G'' = softmax - onehot for the 32 vocabulary columns v0..v0+31 of one row
// (label y, nl = -lse * log2 e), packed to 16 bits (fmt 1: bf16, else fp16).
// Filter: a non-target term with p < eps is dropped.  Columns past V give 0.
// fp16 values are scaled by G16_SCALE.
// With a softcap the logits are cap * tanh(s / cap) and every term carries
// 1 - tanh^2(s / cap).  Called by a whole warp (the fast-path test is
// warp-uniform).  (ORPO design 0.0.6, fused-head spec, "Backward".)
__device__ __forceinline__ void grad_chunk(const uint32_t (&r)[32], int v0, int y, float nl,
                                           float eps, int V, float softcap, float inv_cap,
                                           int fmt, uint32_t (&pk)[16]) {
  const float gs = fmt == 1 ? 1.f : G16_SCALE;
  const int tt = y - v0;
  // Warp-uniform: a chunk inside the vocab with no label of this warp takes
  // the short path (one FFMA + one ex2 per logit).
  const bool slow =
      (v0 + 32 > V) || __any_sync(0xffffffffu, static_cast<unsigned>(tt) < 32u);
  if (softcap > 0.f) {
    // capped logits; each term carries 1 - tanh^2(s / cap)
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
      float g2[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int v = v0 + j + h;
        const float th = tanh_ex2(u2f(r[j + h]) * inv_cap);
        float p = softmax_p(softcap * th, nl);
        const bool tgt = (v == y);
        if (p < eps && !tgt) p = 0.f;
        g2[h] = v < V ? (tgt ? p - 1.f : p) * (1.f - th * th) : 0.f;
      }
      pk[j >> 1] = pack2(g2[0] * gs, g2[1] * gs, fmt);
    }
  } else if (!slow) {
    if (eps > 0.f) {
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        float p0 = softmax_p(u2f(r[j]), nl), p1 = softmax_p(u2f(r[j + 1]), nl);
        p0 = p0 < eps ? 0.f : p0;
        p1 = p1 < eps ? 0.f : p1;
        pk[j >> 1] = pack2(p0 * gs, p1 * gs, fmt);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; j += 2)
        pk[j >> 1] = pack2(softmax_p(u2f(r[j]), nl) * gs, softmax_p(u2f(r[j + 1]), nl) * gs, fmt);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
      float g2[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int v = v0 + j + h;
        float p = softmax_p(u2f(r[j + h]), nl);
        const bool tgt = (v == y);
        if (p < eps && !tgt) p = 0.f;
        g2[h] = v < V ? (tgt ? p - 1.f : p) : 0.f;
      }
      pk[j >> 1] = pack2(g2[0] * gs, g2[1] * gs, fmt);
    }
  }
}

// Drains `nchunks` 32-column chunks of this warp's accumulator lanes through
// two register buffers, so the TMEM load of chunk c+1 overlaps the work on
// chunk c.  f(c, r) receives the 32 fp32 values (as bits) of chunk c.
template <class F>
__device__ __forceinline__ void drain_chunks(uint32_t taddr, int nchunks, F&& f) {
  uint32_t ra[32], rb[32];
  if (nchunks <= 0) return;
  __syncwarp();
  tmem_ld32(taddr, ra);
  tmem_ld_wait(ra);
#pragma unroll 1
  for (int c = 0; c < nchunks; c += 2) {
    const bool more = c + 1 < nchunks;
    if (more) {
      __syncwarp();
      tmem_ld32(taddr + (c + 1) * 32, rb);
    }
    f(c, ra);
    if (more) {
      __syncwarp();
      tmem_ld_wait(rb);
      const bool more2 = c + 2 < nchunks;
      if (more2) tmem_ld32(taddr + (c + 2) * 32, ra);
      f(c + 1, rb);
      if (more2) {
        __syncwarp();
        tmem_ld_wait(ra);
      }
    }
  }
}

template <Mode MODE, int QB = 0, bool C2 = false>
__global__ void __launch_bounds__(QB ? NUM_THREADS_Q4 : NUM_THREADS, 1)
    cce_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                  const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmC,
                  const __grid_constant__ CUtensorMap tmC2, const TileArgs a) {
  static_assert(!(C2 && QB), "quantised heads run single-CTA tiles");
  static_assert(!(C2 && MODE == Mode::kDw), "the dW GEMM runs single-CTA tiles");
  constexpr int NST = C2 ? STAGES2 : (QB ? STAGES_Q : STAGES);
  constexpr int PKB = QB ? pk_bytes<MODE, QB>() : 0;  // packed B tile per stage
  constexpr int SBYTES = C2 ? STAGE2_BYTES : STAGE_BYTES + PKB;
  // With C2 the kernel runs as clusters of two CTAs (a pair on one TPC).
  // rank 0 (the leader) issues the MMAs for both; each CTA loads its own
  // 128 rows of A and its half of B and drains its own 128 TMEM lanes.
  const uint32_t rank = C2 ? cluster_ctarank() : 0u;
  const int tile0 = C2 ? static_cast<int>(cluster_id_x()) : static_cast<int>(blockIdx.x);
  const int tstride = C2 ? static_cast<int>(cluster_count_x()) : static_cast<int>(gridDim.x);
  // tmA/tmB: operand loads.  tmC: kGrad G'' store map [M, chunk] (box 32x32,
  // 64-byte swizzle); kDh dH [1, M, D] (box 1x32x32, 128-byte swizzle).
  // tmC2: kDh partial buffers [ksplit-1, M, D].
  extern __shared__ uint8_t dyn_smem[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = base + NST * SBYTES;
  uint64_t* full =
      reinterpret_cast<uint64_t*>(staging + 4 * 2 * staging_buf_bytes<MODE>());
  uint64_t* empty = full + NST;
  uint64_t* pk_full = empty + NST;  // packed tile landed (quantised heads)
  uint64_t* acc_full = pk_full + NST;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nsplit = (MODE == Mode::kDh || MODE == Mode::kDw) ? a.ksplit : 1;
  const int ntiles = a.n_rt * a.n_ct * nsplit;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], QB ? 1 + DQ_WARPS : 1);
      mbar_init(&empty[s], 1);
      mbar_init(&pk_full[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], (C2 ? 2 : 1) * 4 * 32);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    if constexpr (C2) {
      tmem_alloc2(tmem_slot, TMEM_COLS);
      tmem_relinquish2();
    } else {
      tmem_alloc(tmem_slot, TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (C2) cluster_sync_all();  // barriers of both CTAs initialised
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;
      bool ok = true;
      // H (kLse/kGrad) and the W chunk (kDh) are re-read by many tiles:
      // keep them in L2 ahead of streaming data.
      const uint64_t keep = l2_policy_evict_last();
      for (int t = tile0; t < ntiles && ok; t += tstride) {
        const TileCoord tc = tile_coord<MODE>(a, t);
        if (launch_kind<MODE, C2>(a, tc.rt, tc.ct, tc.s) != 0) continue;
        const int kb = tc.s * a.nk / nsplit, nks = (tc.s + 1) * a.nk / nsplit - kb;
        const int ksteps = nks * a.npass;
        for (int kk = 0; kk < ksteps; ++kk) {
          if (!wait_bounded(&empty[stage], phase ^ 1u, a.wait_ns, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* sA = base + stage * SBYTES;
          uint8_t* sB = sA + A_BYTES;
          const int pass = kk / nks, k = kb + (kk - pass * nks);
          if constexpr (C2) {
            // Both CTAs' copies are counted on the leader's barrier.
            const uint32_t bar = mapa_shared(smem_u32(&full[stage]), 0);
            if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * SBYTES);
            const int arow = (tc.rt * 2 + static_cast<int>(rank)) * BM;
            if (MODE == Mode::kDh) {
              tma_load_2d_pair(sA, &tmA, bar, k * BK, arow, l2_policy_evict_normal());
#pragma unroll
              for (int j = 0; j < BN / 128; ++j)
                tma_load_2d_pair(sB + j * (64 * BK * 2), &tmB, bar,
                                 tc.ct * BN + static_cast<int>(rank) * (BN / 2) + j * 64 +
                                     pass * a.b_pass_off,
                                 a.b_row0 - a.b_shift + k * BK, keep);
            } else {
              tma_load_2d_pair(sA, &tmA, bar, k * BK, arow, keep);
              tma_load_2d_pair(sB, &tmB, bar, k * BK,
                               a.b_row0 - a.b_shift + tc.ct * BN + static_cast<int>(rank) * (BN / 2),
                               l2_policy_evict_normal());
            }
          } else if (QB) {
            // B comes from the dequantisation warps, which read the packed
            // tile (tmB: the packed head as bytes [V, D*QB/8]) from the stage.
            uint8_t* sP = sA + STAGE_BYTES;
            mbar_arrive_expect_tx(&pk_full[stage], PKB);
            if (MODE == Mode::kDh)
              tma_load_2d(sP, &tmB, &pk_full[stage], tc.ct * (BN * QB / 8), a.b_row0 + k * BK);
            else
              tma_load_2d(sP, &tmB, &pk_full[stage], k * (64 * QB / 8),
                          a.b_row0 + tc.ct * BN);
            mbar_arrive_expect_tx(&full[stage], A_BYTES);
            if (MODE == Mode::kDh)
              tma_load_2d(sA, &tmA, &full[stage], k * BK, tc.rt * BM);
            else
              tma_load_2d_hint(sA, &tmA, &full[stage], k * BK, tc.rt * BM, keep);
          } else if (MODE == Mode::kDw) {
            // A = G'' as an MN-major operand (vocab contiguous), two 64x64
            // boxes; B = coeff * H, MN-major (d contiguous), four boxes.
            mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
#pragma unroll
            for (int j = 0; j < BM / 64; ++j)
              tma_load_2d(sA + j * (64 * BK * 2), &tmA, &full[stage], tc.rt * BM + j * 64, k * BK);
#pragma unroll
            for (int j = 0; j < BN / 64; ++j)
              tma_load_2d_hint(sB + j * (64 * BK * 2), &tmB, &full[stage], tc.ct * BN + j * 64,
                               k * BK, keep);
          } else if (MODE == Mode::kDh) {
            mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
            tma_load_2d(sA, &tmA, &full[stage], k * BK, tc.rt * BM);
#pragma unroll
            for (int j = 0; j < BN / 64; ++j)
              tma_load_2d_hint(sB + j * (64 * BK * 2), &tmB, &full[stage],
                               tc.ct * BN + j * 64 + pass * a.b_pass_off,
                               a.b_row0 - a.b_shift + k * BK, keep);
          } else {
            mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
            tma_load_2d_hint(sA, &tmA, &full[stage], k * BK, tc.rt * BM, keep);
            tma_load_2d(sB, &tmB, &full[stage], k * BK, a.b_row0 - a.b_shift + tc.ct * BN);
          }
          issued_mask |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == NST) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        set_status(a.status, ST_TIMEOUT);
        *abort_flag = 1;
      }
      // Let every issued copy land before the CTA can exit (in a pair the
      // leader's barriers also count the other CTA's copies; the final
      // cluster barrier keeps both CTAs alive until then).
      if (!C2 || rank == 0)
        for (int s = 0; s < NST; ++s)
          if (issued_mask & (1u << s)) {
            if (QB)
              wait_bounded(&pk_full[s], (issued_phase >> s) & 1u, DRAIN_LIMIT_NS, nullptr);
            wait_bounded(&full[s], (issued_phase >> s) & 1u, DRAIN_LIMIT_NS,
                         nullptr);
          }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer --
    if (lane == 0 && rank == 0) {
      const uint32_t idesc = idesc_f16(C2 ? 2 * BM : BM, BN, a.fmt, MODE == Mode::kDw,
                                       MODE == Mode::kDh || MODE == Mode::kDw);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      bool ok = true;
      for (int t = tile0; t < ntiles && ok; t += tstride) {
        const TileCoord tc = tile_coord<MODE>(a, t);
        if (launch_kind<MODE, C2>(a, tc.rt, tc.ct, tc.s) != 0) continue;
        const int ksteps =
            ((tc.s + 1) * a.nk / nsplit - tc.s * a.nk / nsplit) * a.npass;
        const int b = acc & 1;
        if (!wait_bounded(&acc_empty[b], ((acc >> 1) & 1) ^ 1u, a.wait_ns,
                          abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * BN;
        for (int kk = 0; kk < ksteps; ++kk) {
          if (!wait_bounded(&full[stage], phase, a.wait_ns, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = smem_u32(base + stage * SBYTES);
          const uint32_t sB = sA + A_BYTES;
#pragma unroll
          for (int j = 0; j < BK / 16; ++j) {
            const uint64_t ad = MODE == Mode::kDw
                                    ? sdesc_sw128(sA + j * 16 * 128, 64 * BK * 2, 1024)
                                    : sdesc_sw128(sA + j * 32, 16, 1024);
            const uint64_t bd =
                (MODE == Mode::kDh || MODE == Mode::kDw)
                    ? sdesc_sw128(sB + j * 16 * 128, 64 * BK * 2, 1024)
                    : sdesc_sw128(sB + j * 32, 16, 1024);
            if constexpr (C2)
              umma_f16_ss2(d_tmem, ad, bd, idesc, (kk | j) != 0 ? 1u : 0u);
            else
              umma_f16_ss(d_tmem, ad, bd, idesc, (kk | j) != 0 ? 1u : 0u);
          }
          // the stage is free in both CTAs once these MMAs have read it
          if constexpr (C2) umma_commit2_mc(&empty[stage], 0x3);
          else umma_commit(&empty[stage]);
          if (++stage == NST) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if constexpr (C2) umma_commit2_mc(&acc_full[b], 0x3);
        else umma_commit(&acc_full[b]);
        ++acc;
      }
      if (!ok) {
        set_status(a.status, ST_TIMEOUT);
        *abort_flag = 1;
      }
      // All MMAs issued by this thread complete before TMEM is released.
      if constexpr (C2) umma_commit2_mc(drain, 0x1);
      else umma_commit(drain);
      wait_bounded(drain, 0, DRAIN_LIMIT_NS, nullptr);
    }
  } else if (QB && warp >= DQ_WARP0) {
    // ------------------------------------------ 4/8-bit dequantisation --
    // 256 threads fill the B half of every stage: 256 (row, group) units of
    // 64 weights per K step, one per thread.  The packed words come from the
    // stage (TMA, pk_full); scale and bias from global memory, fetched one
    // unit ahead (kLse/kGrad: 8 groups of a row at once when rows are 16-byte
    // aligned).  Each unit is dequantised to fp16 and written in the
    // 128-byte-swizzled layout the TMA would produce (16-byte chunk c of row
    // r at c ^ (r & 7)).
    constexpr int QU = 64 * (QB ? QB : 4) / 8;  // packed bytes per unit
    constexpr int NV = QU / 16;
    const int dq = threadIdx.x - DQ_WARP0 * 32;
    const int gpr = a.D / 64;  // groups per head row
    const bool vec8 = MODE != Mode::kDh && (gpr % 8) == 0 &&
                      ((reinterpret_cast<uintptr_t>(a.q_scale) |
                        reinterpret_cast<uintptr_t>(a.q_bias)) & 15u) == 0;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    // unit u of K step k of tile tc: source row, group, offset of its packed
    // words in the stage's packed tile, and of its fp16 output in B.  kDh:
    // the 4 groups of a row are adjacent threads (their scales share a
    // sector).
    auto locate = [&](const TileCoord& tc, int k, int u, int& v, int& g, int& pk, int& off) {
      if (MODE == Mode::kDh) {
        const int r = u >> 2, j = u & 3;
        v = a.b_row0 + k * BK + r;
        g = tc.ct * (BN / 64) + j;
        pk = r * (BN * QB / 8) + j * QU;
        off = j * (64 * BK * 2) + r * 128;
      } else {
        v = a.b_row0 + tc.ct * BN + u;
        g = k;
        pk = u * QU;
        off = u * 128;
      }
    };
    const int r_sw = MODE == Mode::kDh ? (dq >> 2) : dq;  // row for the swizzle
    uint4 sv = make_uint4(0, 0, 0, 0), bv = make_uint4(0, 0, 0, 0);  // 8 groups (vec8)
    int vec_row = -1, vec_g0 = -1;
    auto scale_bias = [&](int v, int g, uint16_t& sc, uint16_t& bi) {
      if (vec8) {
        const int g0 = g & ~7;
        if (v != vec_row || g0 != vec_g0) {
          sv = __ldg(reinterpret_cast<const uint4*>(a.q_scale + static_cast<size_t>(v) * gpr + g0));
          bv = __ldg(reinterpret_cast<const uint4*>(a.q_bias + static_cast<size_t>(v) * gpr + g0));
          vec_row = v;
          vec_g0 = g0;
        }
        const int q = (g & 7) >> 1;
        const uint32_t ws = q == 0 ? sv.x : q == 1 ? sv.y : q == 2 ? sv.z : sv.w;
        const uint32_t wb = q == 0 ? bv.x : q == 1 ? bv.y : q == 2 ? bv.z : bv.w;
        sc = static_cast<uint16_t>((g & 1) ? ws >> 16 : ws & 0xFFFFu);
        bi = static_cast<uint16_t>((g & 1) ? wb >> 16 : wb & 0xFFFFu);
      } else {
        sc = __ldg(a.q_scale + static_cast<size_t>(v) * gpr + g);
        bi = __ldg(a.q_bias + static_cast<size_t>(v) * gpr + g);
      }
    };
    for (int t = tile0; t < ntiles && ok; t += tstride) {
      const TileCoord tc = tile_coord<MODE>(a, t);
      if (tile_kind<MODE>(a, tc.rt, tc.ct, tc.s) != 0) continue;
      const int kb = tc.s * a.nk / nsplit, nks = (tc.s + 1) * a.nk / nsplit - kb;
      for (int kk = 0; kk < nks; ++kk) {
        int v, g, pk, off;
        locate(tc, kb + kk, dq, v, g, pk, off);
        const bool valid = v < a.V && g < gpr;
        uint16_t sc = 0, bi = 0;
        if (valid) scale_bias(v, g, sc, bi);
        if (!wait_bounded(&empty[stage], phase ^ 1u, a.wait_ns, abort_flag) ||
            !wait_bounded(&pk_full[stage], phase, a.wait_ns, abort_flag)) {
          ok = false;
          break;
        }
        uint8_t* sA = base + stage * SBYTES;
        uint8_t* sB = sA + A_BYTES;
        const uint8_t* sP = sA + STAGE_BYTES;
        uint4 out[8];
        if (valid) {
          uint4 w[NV];
#pragma unroll
          for (int i = 0; i < NV; ++i) w[i] = *reinterpret_cast<const uint4*>(sP + pk + 16 * i);
          if constexpr (QB == 8)
            dequant_group64_q8(*reinterpret_cast<const uint4(*)[4]>(w), sc, bi, out);
          else
            dequant_group64(w[0], w[NV - 1], sc, bi, out);
        } else {
#pragma unroll
          for (int c = 0; c < 8; ++c) out[c] = make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(sB + off + ((c ^ (r_sw & 7)) << 4)) = out[c];
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[stage]);
        if (++stage == NST) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok) {
      set_status(a.status, ST_TIMEOUT);
      *abort_flag = 1;
    }
  } else {
    // ---------------------------------------------------------- epilogue --
    const int quad = warp & 3;
    const int rin = quad * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    int acc = 0;
    uint8_t* const stage_base = staging + quad * 2 * staging_buf_bytes<MODE>();
    uint32_t nstore = 0;
    // Leader's acc_empty barriers (a pair's MMA waits for both CTAs).
    uint32_t acc_empty_leader[2] = {0u, 0u};
    if constexpr (C2) {
      acc_empty_leader[0] = mapa_shared(smem_u32(&acc_empty[0]), 0);
      acc_empty_leader[1] = mapa_shared(smem_u32(&acc_empty[1]), 0);
    }
    for (int t = tile0; t < ntiles; t += tstride) {
      const TileCoord tc = tile_coord<MODE>(a, t);
      // this CTA's 128-row tile
      const int rt = C2 ? tc.rt * 2 + static_cast<int>(rank) : tc.rt, ct = tc.ct;
      float* const dh_buf =
          tc.s == 0 ? a.dh : a.dh_part + static_cast<size_t>(tc.s - 1) * a.M * a.D;
      const int kind_launch = launch_kind<MODE, C2>(a, tc.rt, ct, tc.s);
      const int kind = !C2 ? kind_launch
                           : (rt < a.n_rt128 ? tile_kind<MODE>(a, rt, ct, tc.s) : 2);
      const int row = rt * BM + rin;
      const bool live = row < a.M;
      if (C2 && kind_launch == 0 && kind != 0) {
        // The pair computed this tile for the other half: take the
        // accumulator round trip without using it, then do this half's
        // zeros (kind 1) or nothing (kind 2).
        const int b = acc & 1;
        if (!wait_bounded(&acc_full[b], (acc >> 1) & 1, a.wait_ns, abort_flag)) {
          set_status(a.status, ST_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        tc_fence_before();
        mbar_arrive_cluster(acc_empty_leader[b]);
        ++acc;
      }
      if (kind == 2) continue;
      if (kind == 1) {
        if (MODE == Mode::kGrad) {
          if (live) {
            uint4* dst = reinterpret_cast<uint4*>(
                a.g_out + static_cast<size_t>(row) * a.g_ld + ct * BN);
            for (int i = 0; i < BN * 2 / 16; ++i) dst[i] = make_uint4(0, 0, 0, 0);
          }
        } else if (MODE == Mode::kDh) {
          if (live) {
            for (int d0 = ct * BN; d0 < min(a.D, ct * BN + BN); d0 += 4)
              *reinterpret_cast<float4*>(dh_buf + static_cast<size_t>(row) * a.D + d0) =
                  make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
        continue;
      }
      const int b = acc & 1;
      if (!wait_bounded(&acc_full[b], (acc >> 1) & 1, a.wait_ns, abort_flag)) {
        set_status(a.status, ST_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + lane_addr + b * BN;

      if (MODE == Mode::kLse) {
        const int y = live ? a.labels[row] : -1;
        const int vbase = a.b_row0 + ct * BN;
        const int nchunks = min(BN / 32, (a.V - vbase + 31) / 32);
        float m_run = -INFINITY, s_run = 0.f, tval = 0.f;
        bool found = false;
        drain_chunks(taddr, nchunks, [&](int c, const uint32_t (&r)[32]) {
          const int v0 = vbase + c * 32;
          const int nvalid = min(32, a.V - v0);
          float x[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) x[j] = u2f(r[j]);
          if (a.softcap > 0.f) {
#pragma unroll
            for (int j = 0; j < 32; ++j) x[j] = a.softcap * tanh_ex2(x[j] * a.inv_cap);
          }
          float cm = -INFINITY;
          float s0 = 0.f, s1 = 0.f;
          if (nvalid == 32) {
#pragma unroll
            for (int j = 0; j < 32; ++j) cm = fmaxf(cm, x[j]);
            const float mn = fmaxf(m_run, cm);
            const float nb = -mn * LOG2E;
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              s0 += ex2_approx(fmaf(x[j], LOG2E, nb));
              s1 += ex2_approx(fmaf(x[j + 1], LOG2E, nb));
            }
            s_run = s_run * ex2_approx((m_run - mn) * LOG2E) + (s0 + s1);
            m_run = mn;
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < nvalid) cm = fmaxf(cm, x[j]);
            const float mn = fmaxf(m_run, cm);
            const float nb = -mn * LOG2E;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < nvalid) s0 += ex2_approx(fmaf(x[j], LOG2E, nb));
            s_run = s_run * ex2_approx((m_run - mn) * LOG2E) + s0;
            m_run = mn;
          }
          const int tt = y - v0;
          const bool hit = static_cast<unsigned>(tt) < static_cast<unsigned>(nvalid);
          if (__any_sync(0xffffffffu, hit)) {
            if (hit) {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (j == tt) tval = x[j];
              found = true;
            }
            __syncwarp();
          }
        });
        tc_fence_before();
        if constexpr (C2) mbar_arrive_cluster(acc_empty_leader[b]);
        else mbar_arrive(&acc_empty[b]);
        if (live) {
          const size_t o = static_cast<size_t>(a.ct_off + ct) * a.M + row;
          a.part_m[o] = m_run;
          a.part_s[o] = s_run;
          if (found) a.tgt[row] = tval;
        }
      } else if (MODE == Mode::kGrad) {
        // G'' = softmax - onehot (the dH step applies -coeff), 16-bit.
        const int y = live ? a.labels[row] : -1;
        const float nl = live ? -a.lse[row] * LOG2E : 0.f;
        const float eps = a.filter_eps;
        const int vbase = a.b_row0 + ct * BN;
        drain_chunks(taddr, BN / 32, [&](int c, const uint32_t (&r)[32]) {
          uint32_t pk[16];
          grad_chunk(r, vbase + c * 32, y, nl, eps, a.V, a.softcap, a.inv_cap, a.fmt, pk);
          // Stage the 32x32 block in shared memory (64-byte swizzle: 16-byte
          // chunk i of row r sits at chunk i ^ ((r >> 1) & 3)) and let TMA
          // write it; rows past M are clipped by the tensor map.
          uint8_t* sb = stage_base + (nstore & 1) * staging_buf_bytes<MODE>();
          if (lane == 0) bulk_wait_read<1>();
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 4; ++i)
            *reinterpret_cast<uint4*>(sb + lane * 64 + ((i ^ ((lane >> 1) & 3)) << 4)) =
                make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmC, sb, ct * BN + c * 32, rt * BM + quad * 32);
            bulk_commit();
          }
          ++nstore;
        });
        tc_fence_before();
        if constexpr (C2) mbar_arrive_cluster(acc_empty_leader[b]);
        else mbar_arrive(&acc_empty[b]);
      } else {  // kDh: dH (+)= -coeff * (G'' . W);  kDw: dW[chunk] = -(G''^T . coeff*H)
        const float g = MODE == Mode::kDw ? -1.f
                        : live ? -a.coeff[row] * (a.fmt == 1 ? 1.f : G16_UNSCALE)
                               : 0.f;
        const int dbase = ct * BN;
        const int nchunks = min(BN / 32, (a.D - dbase) / 32);
        const CUtensorMap* dmap = tc.s == 0 ? &tmC : &tmC2;
        const int dz = tc.s == 0 ? 0 : tc.s - 1;
        const int orow0 = (MODE == Mode::kDw ? a.b_row0 : 0) + rt * BM + quad * 32;
        const bool store = MODE == Mode::kDw || a.first_chunk;
        drain_chunks(taddr, nchunks, [&](int c, const uint32_t (&r)[32]) {
          // Stage g * acc as a 32x32 fp32 block (128-byte swizzle: chunk i of
          // row r at chunk i ^ (r & 7)); the first vocab chunk stores it, the
          // later ones add it in L2 (one add per element per launch, so the
          // result does not depend on timing).
          uint8_t* sb = stage_base + (nstore & 1) * staging_buf_bytes<MODE>();
          if (lane == 0) bulk_wait_read<1>();
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            // accumulator column of output column j (4-bit heads permute K
            // inside groups of 8, so the dH columns come out permuted too)
            constexpr auto src = [](int j) { return QB ? (j & ~7) + qpos<QB>(j & 7) : j; };
            const float4 o =
                g == 0.f ? make_float4(0.f, 0.f, 0.f, 0.f)
                         : make_float4(g * u2f(r[src(4 * i)]), g * u2f(r[src(4 * i + 1)]),
                                       g * u2f(r[src(4 * i + 2)]), g * u2f(r[src(4 * i + 3)]));
            *reinterpret_cast<float4*>(sb + lane * 128 + ((i ^ (lane & 7)) << 4)) = o;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (store)
              tma_store_3d(dmap, sb, dbase + c * 32, orow0, dz);
            else
              tma_reduce_add_3d(dmap, sb, dbase + c * 32, orow0, dz);
            bulk_commit();
          }
          ++nstore;
        });
        tc_fence_before();
        if constexpr (C2) mbar_arrive_cluster(acc_empty_leader[b]);
        else mbar_arrive(&acc_empty[b]);
      }
      ++acc;
    }
    // Every TMA store / reduction of this warp has completed before exit.
    if (MODE != Mode::kLse && lane == 0) bulk_wait<0>();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  // A pair stays resident until both CTAs are done with each other's shared
  // memory, barriers and tensor memory.
  if constexpr (C2) cluster_sync_all();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if constexpr (C2) tmem_dealloc2(tmem_base, TMEM_COLS);
    else tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace cce
