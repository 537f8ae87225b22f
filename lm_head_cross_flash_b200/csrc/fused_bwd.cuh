// fused_bwd.cuh — the backward of the flash-CCE head as one persistent
// kernel: every vocab tile of the logits is recomputed on the tensor cores,
// turned into the coefficient tile G'' = softmax - onehot straight from the
// TMEM accumulator, and contracted against the same vocab rows of W into a
// dH accumulator that stays in TMEM for a whole sweep over the vocabulary.
// (ORPO design 0.0.6, fused-head implementation spec, "Backward (recompute
// vocab tiles from the saved LSE)": recompute, form g * (onehot - softmax),
// accumulate dh, never form [M, V]; Training design §5.1, tier 4.)
//
// Why a group of CTAs, and what they exchange.  A row tile's dH is
// rows x D fp32: 1 MB for 128 rows at D = 2048, four times a TMEM.  So each
// CTA (or CTA pair) of a group of C = ceil(D / 256) owns the 256 d-columns
// [256 p, 256 p + 256) of dH for the group's row tile, in 256 TMEM columns,
// and the group sweeps the vocabulary in rounds of C vocab tiles.  In a round
// member p recomputes the logits of vocab tile (round * C + p) (K = D), forms
// its G'' tile and publishes it in a small ring of tiles in global memory
// that stays in L2; then every member contracts all C published tiles of the
// round with its own d-columns of W (K = C tiles of vocabulary).  The S GEMM
// of one round is issued before the dH GEMM of the previous one, so the
// exchange has a whole S GEMM to complete in before its tiles are needed
// (what is left of the wait measured about 15 % of a unit at the long pair).
// G'' never exists as a whole: one ring holds DEPTH rounds of tiles per
// group.
//
// Roles (192 threads, as in gemm_tc.cuh): warp 0 loads operand stages by
// TMA (the S phase: H rows and W rows, both K-major; the dH phase: a G''
// tile of the ring, K-major, and W as an MN-major operand); warp 1 issues
// tcgen05.mma into the S accumulator(s) and the dH accumulator; warps 2-5
// drain S, compute G'' (grad_chunk, the same arithmetic as the two-GEMM
// path), stage it for TMA stores into the ring, and at the end of a row
// tile's sweep drain dH, scale each row by -coeff and store it.
//
// C2 = true: clusters of two CTAs computing 256-row tiles with
// tcgen05.mma.cta_group::2 (S: 256 x 256 vocab; dH: 256 x 256 d-columns),
// each CTA loading its own 128 rows of A and half of B (as in gemm_tc.cuh).
// C2 = false: single CTAs on 128-row tiles with 128-column vocab tiles and a
// double-buffered S accumulator (at most one row tile of 128, or CTA pairs
// switched off).
//
// The exchange.  Ring slot (group, unit % DEPTH, member) is filled once per
// DEPTH units.  Publisher: each epilogue warp waits until every member has
// consumed the slot's previous fill (consumed[slot][member] >= fill), writes
// its rows by TMA store, waits for the stores to complete, fences the async
// proxy and adds 1 to ready[slot][half] with release semantics.  Consumer:
// the producer warp waits for ready >= 4 (fill + 1) with acquire semantics,
// fences the async proxy and loads the tile by TMA; once the tile has
// landed (the leader's full barrier counts both CTAs of a pair) the MMA warp
// stores consumed = fill + 1 (relaxed: the tile's reads are complete).  A
// tile that block skip (or the end of the vocabulary) removes is neither
// computed nor loaded, but still advances both counters, so the counts stay
// aligned; its publishers wait for the previous fill to be consumed before
// adding 1, as for a computed tile.  ready counts 4 per fill in total, so
// without that wait a fast warp's count for a skipped fill could stand in
// for a slow warp's count of the fill before it, and the consumer would load
// that fill before the slow warp's rows had landed.  Every wait is bounded; all
// CTAs of the grid are resident at once (at most one CTA per SM, grid no
// larger than the resident count).
//
// Partition of the work.  A unit is (row tile r, round j).  G groups take
// the row tiles in waves (group g: r = w G + g), so that all groups sweep
// the same rounds of W at the same time and W streams from HBM about once
// per wave.  The rem = n_rt mod G row tiles left over are cut into bands of
// rounds (fb_unit) so that concurrent groups still share rounds: a row tile
// split between k groups gives k partial dH slices (buffer 0 is dH itself,
// buffers 1.. are in the workspace) that fused_sum_parts_kernel adds in a
// fixed order.
#pragma once

#include "gemm_tc.cuh"

namespace cce {

// Units in flight in the G'' ring of a group.  Two: a slot is rewritten two
// units after it was filled, soon enough that its lines are still in L2 (a
// three-deep ring had most of its tiles written back to HBM first: 3.3
// against 1.5 GB of DRAM writes per launch at the long pair, 4 % slower).
constexpr int FB_DEPTH = 2;
constexpr int FB_DS = 256;      // dH columns per member
constexpr uint32_t FB_TMEM_COLS = 512;

// BVS: vocab columns of a single-CTA S tile (CTA pairs use 256).  128 is
// the one instantiated: 64-wide tiles at M = 64 halve the W held in L2
// between a round's two reads but double the per-unit exchange overhead,
// and measured slower (0.49 against 0.38 ms).
template <bool C2, int BVS = 128>
struct FusedCfg {
  static constexpr int TH = C2 ? 2 * BM : BM;        // rows of a tile
  static constexpr int BV = C2 ? 256 : BVS;          // vocab columns of an S tile
  static constexpr int SB = C2 ? 1 : 2;              // S accumulators (TMEM columns [0, SB*BV))
  static constexpr int DB = C2 ? FB_DS / 2 : FB_DS;  // d-columns of W each CTA loads (dH phase)
  static constexpr int BR = C2 ? 128 : BV;           // W rows each CTA loads (S phase)
  static constexpr int S_BYTES = A_BYTES + BR * BK * 2;  // H 128 x 64 + W BR x 64
  static constexpr int D_BYTES = A_BYTES + BK * DB * 2;  // G'' 128 x 64 + W 64 x DB
  static constexpr int STAGE = S_BYTES > D_BYTES ? S_BYTES : D_BYTES;
  static constexpr int NST = C2 ? 6 : 4;
  static constexpr int STAGING = 4 * 2 * 32 * 128;   // per epilogue warp two 4 KB blocks
  static constexpr int SMEM = NST * STAGE + STAGING + 1024 + 256;
};
static_assert(FusedCfg<true>::SMEM <= 232448 && FusedCfg<false, 128>::SMEM <= 232448,
              "fused backward exceeds the shared memory of a CTA");

struct FusedArgs {
  int M, V, D;
  int n_rt;       // row tiles of TH rows
  int n_rt128;    // 128-row tiles (block-skip plan granularity)
  int nk;         // K steps of BK over D
  int C;          // members per group (d-slices of 256), at most 32
  int G;          // groups in the waves
  int nb;         // remainder bands: nb * rem groups, band b covering a round
                  // range of every remainder row tile (0: no bands)
  int bw;         // band width in rounds (0: split R evenly over nb bands)
  int lr;         // groups of the leftover (after the bands) or of the whole
                  // remainder when it has fewer units than groups
  int r0;         // first round of the leftover
  int rl;         // rounds of the leftover per remainder row tile
  int ls;         // 1: leftover group l takes remainder row tile l whole (all
                  // leftover groups in step), and only the other rem - lr
                  // tiles are cut into ranges
  int n_vt;       // vocab tiles of BV
  int n_rounds;   // ceil(n_vt / C)
  int waves;      // n_rt / G
  int rem;        // n_rt % G
  int row_rem;    // first row of the remainder (waves * G * TH); partial
                  // buffers hold rows [row_rem, M) only
  uint64_t wait_ns;
  uint32_t* status;
  const int32_t* labels;
  const float* lse;
  const float* coeff;
  float filter_eps;
  const uint8_t* tile_skip;  // [n_rt128, skip_ld], 256-vocab blocks
  int skip_ld;
  const uint8_t* row_skip;   // [n_rt128]
  const uint32_t* unit_mask;  // [n_rt, n_rounds]: fb_mask_of for every unit
  float softcap;
  float inv_cap;
  uint32_t* ready;     // [G * DEPTH * C * 2]
  uint32_t* consumed;  // [G * DEPTH * C * C]
  uint32_t* progress;  // [G]: units member 0 of each group has started
};

// Groups may run at most this many units ahead of the slowest group during
// the waves: the groups then read the same rounds of W within a few units
// of each other and share them in L2 (left alone they drift apart over a
// wave, and each straggler streams W from HBM on its own).  Measured at the
// long pair, three runs each on one box: a lead of 1 unit 13.05-13.24 ms per
// launch, 2 units 13.30-13.44 ms, 4 units 13.39-13.92 ms.
constexpr int FB_LEAD = 1;
constexpr uint64_t FB_LEAD_WAIT_NS = 200000;  // a hint: give up after 0.2 ms

// One unit of group g's sequence: row tile r, round j; first / last unit of
// a segment (a run of units on one row tile), and the dH buffer the segment
// writes.
struct FUnit {
  int r, j;
  bool first, last;
  int buf;
};

// The remainder (rem = n_rt mod G row tiles of R rounds) is cut so that
// groups running at the same time share rounds of W:
//  * nb = G / rem bands of rem groups; the group (b, i) takes remainder row
//    tile i over band b's round range.  The groups of a band read the same
//    rounds at the same time.  With G a multiple of rem the bands split R;
//    otherwise each is bw = floor(rem R / G) rounds wide and
//  * the leftover rounds [r0, R) of every remainder row tile (rem * rl units)
//    go to the lr = G mod rem other groups: leftover group l first takes
//    remainder row tile l's leftover rounds whole, so the lr groups read the
//    same rounds of W at the same time (ls = 1); the leftover rounds of
//    tiles lr .. rem - 1 are then cut into contiguous ranges of the sequence
//    (tile, round), one per leftover group; a tile may be shared by several
//    of them.
//  When the remainder has fewer units than groups, lr = its unit count and
//  every unit is a leftover unit (nb = 0, r0 = 0, rl = R, ls = 0: all of the
//  remainder is cut into ranges).
// A remainder row tile gathers one dH slice per band and one per leftover
// group that touches it: buffer b for band b, nb + k for the k-th leftover
// group on the tile.

// Ranges of the leftover: T units over lr groups, q = T / lr each and one
// more for the first T mod lr groups, so the groups holding units (and the
// groups touching any one row tile) are consecutive.  Group l holds
// [fb_range_lo(l), fb_range_lo(l + 1)).
__host__ __device__ __forceinline__ int64_t fb_range_lo(int64_t l, int64_t T, int lr) {
  const int64_t q = T / lr, r = T % lr;
  return l * q + (l < r ? l : r);
}
// Leftover group holding leftover unit e.
__host__ __device__ __forceinline__ int fb_group_of(int64_t e, int64_t T, int lr) {
  const int64_t q = T / lr, r = T % lr, big = r * (q + 1);
  return static_cast<int>(e < big ? e / (q + 1) : r + (e - big) / q);
}

// Round range [lo, hi) of band b.
__host__ __device__ __forceinline__ void fb_band(const FusedArgs& a, int b, int& lo, int& hi) {
  if (a.bw == 0) {
    lo = b * a.n_rounds / a.nb;
    hi = (b + 1) * a.n_rounds / a.nb;
  } else {
    lo = b * a.bw;
    hi = lo + a.bw;
  }
}

// The leftover's ranged part: tiles [ls ? lr : 0, rem) of rl rounds each.
__host__ __device__ __forceinline__ int fb_ranged_tile0(const FusedArgs& a) {
  return a.ls ? a.lr : 0;
}
__host__ __device__ __forceinline__ int64_t fb_ranged_units(const FusedArgs& a) {
  return static_cast<int64_t>(a.rem - fb_ranged_tile0(a)) * a.rl;
}

__host__ __device__ __forceinline__ int fb_units(const FusedArgs& a, int g) {
  int n = a.waves * a.n_rounds;
  if (a.rem == 0) return n;
  if (g < a.nb * a.rem) {
    int lo, hi;
    fb_band(a, g / a.rem, lo, hi);
    return n + hi - lo;
  }
  const int l = g - a.nb * a.rem;
  if (l < a.lr) {
    const int64_t T = fb_ranged_units(a);
    n += (a.ls ? a.rl : 0) + static_cast<int>(fb_range_lo(l + 1, T, a.lr) - fb_range_lo(l, T, a.lr));
  }
  return n;
}

__host__ __device__ __forceinline__ FUnit fb_unit(const FusedArgs& a, int g, int u) {
  FUnit x;
  const int full = a.waves * a.n_rounds;
  if (u < full) {
    const int w = u / a.n_rounds;
    x.j = u - w * a.n_rounds;
    x.r = w * a.G + g;
    x.first = x.j == 0;
    x.last = x.j == a.n_rounds - 1;
    x.buf = 0;
    return x;
  }
  const int t = u - full;
  if (g < a.nb * a.rem) {
    const int b = g / a.rem;
    int lo, hi;
    fb_band(a, b, lo, hi);
    x.r = a.waves * a.G + (g - b * a.rem);
    x.j = lo + t;
    x.first = t == 0;
    x.last = x.j == hi - 1;
    x.buf = b;
    return x;
  }
  const int l = g - a.nb * a.rem;
  if (a.ls && t < a.rl) {
    // remainder row tile l whole, in step with the other leftover groups
    x.r = a.waves * a.G + l;
    x.j = a.r0 + t;
    x.first = t == 0;
    x.last = t == a.rl - 1;
    x.buf = a.nb;
    return x;
  }
  const int tr = a.ls ? t - a.rl : t;
  const int i0 = fb_ranged_tile0(a);
  const int64_t T = fb_ranged_units(a);
  const int64_t lo = fb_range_lo(l, T, a.lr), hi = fb_range_lo(l + 1, T, a.lr);
  const int64_t e = lo + tr;
  const int i = static_cast<int>(e / a.rl);
  const int jj = static_cast<int>(e - static_cast<int64_t>(i) * a.rl);
  x.r = a.waves * a.G + i0 + i;
  x.j = a.r0 + jj;
  x.first = tr == 0 || jj == 0;
  x.last = (e == hi - 1) || jj == a.rl - 1;
  x.buf = a.nb + l - fb_group_of(static_cast<int64_t>(i) * a.rl, T, a.lr);
  return x;
}

// dH slices a remainder row tile i gathers: one per band, and one per
// leftover group touching it.
__host__ __device__ __forceinline__ int fb_slices(const FusedArgs& a, int i) {
  int k = a.nb;
  if (a.lr > 0) {
    const int i0 = fb_ranged_tile0(a);
    if (i < i0) return k + 1;  // one leftover group takes it whole
    const int64_t T = fb_ranged_units(a);
    i -= i0;
    k += fb_group_of(static_cast<int64_t>(i + 1) * a.rl - 1, T, a.lr) -
         fb_group_of(static_cast<int64_t>(i) * a.rl, T, a.lr) + 1;
  }
  return k;
}

// Tiles of round j with nothing to compute for row tile r, as bits q of a
// mask (vocab tile j*C + q): past the vocabulary, or every 128-row half
// either past M, without a nonzero cotangent, or block-skipped for the
// 256-wide vocabulary block holding the tile.  fused_mask_kernel evaluates
// it once per unit before the backward starts.
template <bool C2, int BV>
__device__ __forceinline__ uint32_t fb_mask_of(const FusedArgs& a, int r, int j) {
  const int v0 = j * a.C;
  uint32_t past = 0;
  for (int q = 0; q < a.C; ++q)
    if (v0 + q >= a.n_vt) past |= 1u << q;
  auto half = [&](int rt) -> uint32_t {
    if (rt >= a.n_rt128 || a.row_skip[rt]) return ~0u;
    if (a.tile_skip == nullptr) return 0u;
    const uint8_t* ts = a.tile_skip + static_cast<size_t>(rt) * a.skip_ld;
    uint32_t m = 0;
    for (int q = 0; q < a.C; ++q) {
      const int v = v0 + q;
      if (v < a.n_vt && ts[v / (256 / BV)] != 0) m |= 1u << q;
    }
    return m;
  };
  return past | (C2 ? (half(2 * r) & half(2 * r + 1)) : half(r));
}

// The skip mask of unit (r, j) for the kernel's roles: one word from the
// table, loaded a unit before it is used.  (Evaluating fb_mask_of in the
// roles themselves chained up to four L2 round trips onto every unit's
// issue path: the long pair ran about 9 % slower with block skip on, even
// when nothing was skipped.)
__device__ __forceinline__ uint32_t fb_mask(const FusedArgs& a, int r, int j) {
  return a.unit_mask[static_cast<size_t>(r) * a.n_rounds + j];
}

// unit_mask[r][j] = fb_mask_of(a, r, j) for every row tile and round.
template <bool C2, int BV>
__global__ void fused_mask_kernel(FusedArgs a, uint32_t* __restrict__ out) {
  const int64_t n = static_cast<int64_t>(a.n_rt) * a.n_rounds;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int r = static_cast<int>(i / a.n_rounds);
    out[i] = fb_mask_of<C2, BV>(a, r, static_cast<int>(i - static_cast<int64_t>(r) * a.n_rounds));
  }
}

template <bool C2, int BVS>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    fused_bwd_kernel(const __grid_constant__ CUtensorMap tmH,   // H [M, D], box 64 x 128
                     const __grid_constant__ CUtensorMap tmWk,  // W [V, D], box 64 x 128
                     const __grid_constant__ CUtensorMap tmWm,  // W [V, D], box 64 x 64 (MN-major B)
                     const __grid_constant__ CUtensorMap tmGl,  // ring [rows, BV], box 64 x 128
                     const __grid_constant__ CUtensorMap tmGs,  // ring [rows, BV], box 32 x 32
                     const __grid_constant__ CUtensorMap tmD0,  // dH [1, M, D] fp32
                     const __grid_constant__ CUtensorMap tmD1,  // partial dH [nbuf-1, M-row_rem, D]
                     const FusedArgs a) {
  using F = FusedCfg<C2, BVS>;
  const uint32_t rank = C2 ? cluster_ctarank() : 0u;
  const int member_id = C2 ? static_cast<int>(cluster_id_x()) : static_cast<int>(blockIdx.x);
  const int g = member_id / a.C, p = member_id - (member_id / a.C) * a.C;

  extern __shared__ uint8_t dyn_smem[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = base + F::NST * F::STAGE;
  uint64_t* full = reinterpret_cast<uint64_t*>(staging + F::STAGING);
  uint64_t* empty = full + F::NST;
  uint64_t* s_full = empty + F::NST;
  uint64_t* s_empty = s_full + 2;
  uint64_t* dh_full = s_empty + 2;
  uint64_t* dh_empty = dh_full + 1;
  uint64_t* drain = dh_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_u = g < a.G ? fb_units(a, g) : 0;
  constexpr int KV = F::BV / BK;  // K steps of one G'' tile in the dH phase

  if (threadIdx.x == 0) {
    for (int s = 0; s < F::NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_empty[b], (C2 ? 2 : 1) * 4 * 32);
    }
    mbar_init(dh_full, 1);
    mbar_init(dh_empty, (C2 ? 2 : 1) * 4 * 32);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
    tma_prefetch_desc(&tmH);
    tma_prefetch_desc(&tmWk);
    tma_prefetch_desc(&tmWm);
    tma_prefetch_desc(&tmGl);
  }
  if (warp == 1) {
    if constexpr (C2) {
      tmem_alloc2(tmem_slot, FB_TMEM_COLS);
      tmem_relinquish2();
    } else {
      tmem_alloc(tmem_slot, FB_TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (C2) cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t tmem_dh = tmem_base + FB_DS;  // columns [256, 512)

  auto slot_of = [&](int u, int q) { return (g * FB_DEPTH + u % FB_DEPTH) * a.C + q; };

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;
      bool ok = true;
      const uint64_t keep = l2_policy_evict_last();
      const uint64_t normal = l2_policy_evict_normal();
      auto next_stage = [&](uint32_t bytes, uint8_t*& sA, uint8_t*& sB, uint32_t& bar) -> bool {
        if (!wait_bounded(&empty[stage], phase ^ 1u, a.wait_ns, abort_flag)) return false;
        sA = base + stage * F::STAGE;
        sB = sA + A_BYTES;
        if constexpr (C2) {
          bar = mapa_shared(smem_u32(&full[stage]), 0);
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * bytes);
        } else {
          bar = smem_u32(&full[stage]);
          mbar_arrive_expect_tx(&full[stage], bytes);
        }
        return true;
      };
      auto advance = [&]() {
        issued_mask |= 1u << stage;
        issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
        if (++stage == F::NST) {
          stage = 0;
          phase ^= 1u;
        }
      };
      uint32_t mk_prev = 0, mk_cur = 0;
      if (n_u > 0) {
        const FUnit x0 = fb_unit(a, g, 0);
        mk_cur = fb_mask(a, x0.r, x0.j);
      }
      for (int u = 0; u <= n_u && ok; ++u) {
        uint32_t mk_next = 0;
        if (u + 1 < n_u) {
          const FUnit xn = fb_unit(a, g, u + 1);
          mk_next = fb_mask(a, xn.r, xn.j);
        }
        if (u < n_u && p == 0 && rank == 0 && u < a.waves * a.n_rounds) {
          st_relaxed_gpu(&a.progress[g], static_cast<uint32_t>(u));
          if (u >= FB_LEAD) {
            const uint32_t need = static_cast<uint32_t>(u - FB_LEAD);
            const uint64_t t0 = globaltimer_ns();
            for (int o = 0; o < a.G; ++o)
              while (ld_relaxed_gpu(&a.progress[o]) < need &&
                     globaltimer_ns() - t0 < FB_LEAD_WAIT_NS)
                __nanosleep(128);
          }
        }
        if (u < n_u) {
          const FUnit x = fb_unit(a, g, u);
          const int v = x.j * a.C + p;
          if (!((mk_cur >> p) & 1u)) {
            const int arow = x.r * F::TH + static_cast<int>(rank) * BM;
            const int brow = v * F::BV + (C2 ? static_cast<int>(rank) * 128 : 0);
            for (int k = 0; k < a.nk; ++k) {
              uint8_t *sA, *sB;
              uint32_t bar;
              if (!next_stage(F::S_BYTES, sA, sB, bar)) {
                ok = false;
                break;
              }
              if constexpr (C2) {
                tma_load_2d_pair(sA, &tmH, bar, k * BK, arow, keep);
                tma_load_2d_pair(sB, &tmWk, bar, k * BK, brow, normal);
              } else {
                tma_load_2d_hint(sA, &tmH, &full[stage], k * BK, arow, keep);
                tma_load_2d_hint(sB, &tmWk, &full[stage], k * BK, brow, normal);
              }
              advance();
            }
          }
        }
        if (u >= 1 && ok) {
          const FUnit x = fb_unit(a, g, u - 1);
          const uint32_t fill = static_cast<uint32_t>((u - 1) / FB_DEPTH);
          for (int q = 0; q < a.C && ok; ++q) {
            const int v = x.j * a.C + q;
            if ((mk_prev >> q) & 1u) continue;
            const int slot = slot_of(u - 1, q);
            if (!wait_flag_geq(&a.ready[slot * 2 + static_cast<int>(rank)], 4u * (fill + 1u),
                               a.wait_ns, abort_flag)) {
              ok = false;
              break;
            }
            fence_proxy_async_global();
            const int grow = slot * F::TH + static_cast<int>(rank) * BM;
            const int dcol = p * FB_DS + (C2 ? static_cast<int>(rank) * (FB_DS / 2) : 0);
            for (int kv = 0; kv < KV; ++kv) {
              uint8_t *sA, *sB;
              uint32_t bar;
              if (!next_stage(F::D_BYTES, sA, sB, bar)) {
                ok = false;
                break;
              }
              if constexpr (C2) {
                tma_load_2d_pair(sA, &tmGl, bar, kv * BK, grow, normal);
#pragma unroll
                for (int jj = 0; jj < F::DB / 64; ++jj)
                  tma_load_2d_pair(sB + jj * (64 * BK * 2), &tmWm, bar, dcol + jj * 64,
                                   v * F::BV + kv * BK, normal);
              } else {
                tma_load_2d(sA, &tmGl, &full[stage], kv * BK, grow);
#pragma unroll
                for (int jj = 0; jj < F::DB / 64; ++jj)
                  tma_load_2d(sB + jj * (64 * BK * 2), &tmWm, &full[stage], dcol + jj * 64,
                              v * F::BV + kv * BK);
              }
              advance();
            }
          }
        }
        mk_prev = mk_cur;
        mk_cur = mk_next;
      }
      if (!ok) {
        set_status(a.status, ST_TIMEOUT);
        *abort_flag = 1;
      }
      if (!C2 || rank == 0)
        for (int s = 0; s < F::NST; ++s)
          if (issued_mask & (1u << s))
            wait_bounded(&full[s], (issued_phase >> s) & 1u, DRAIN_LIMIT_NS, nullptr);
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer --
    if (lane == 0 && rank == 0) {
      const uint32_t idesc_s = idesc_f16(F::TH, F::BV, 1, false, false);
      const uint32_t idesc_d = idesc_f16(F::TH, FB_DS, 1, false, true);
      int stage = 0;
      uint32_t phase = 0;
      int ns = 0, nseg = 0;
      bool ok = true, dh_any = false;
      uint32_t mk_prev = 0, mk_cur = 0;
      if (n_u > 0) {
        const FUnit x0 = fb_unit(a, g, 0);
        mk_cur = fb_mask(a, x0.r, x0.j);
      }
      for (int u = 0; u <= n_u && ok; ++u) {
        uint32_t mk_next = 0;
        if (u + 1 < n_u) {
          const FUnit xn = fb_unit(a, g, u + 1);
          mk_next = fb_mask(a, xn.r, xn.j);
        }
        if (u < n_u) {
          if (!((mk_cur >> p) & 1u)) {
            const int sb = ns % F::SB;
            if (!wait_bounded(&s_empty[sb], ((ns / F::SB) & 1) ^ 1u, a.wait_ns, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + sb * F::BV;
            for (int kk = 0; kk < a.nk; ++kk) {
              if (!wait_bounded(&full[stage], phase, a.wait_ns, abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t sA = smem_u32(base + stage * F::STAGE);
              const uint32_t sB = sA + A_BYTES;
#pragma unroll
              for (int j = 0; j < BK / 16; ++j) {
                const uint64_t ad = sdesc_sw128(sA + j * 32, 16, 1024);
                const uint64_t bd = sdesc_sw128(sB + j * 32, 16, 1024);
                if constexpr (C2) umma_f16_ss2(d_tmem, ad, bd, idesc_s, (kk | j) != 0 ? 1u : 0u);
                else umma_f16_ss(d_tmem, ad, bd, idesc_s, (kk | j) != 0 ? 1u : 0u);
              }
              if constexpr (C2) umma_commit2_mc(&empty[stage], 0x3);
              else umma_commit(&empty[stage]);
              if (++stage == F::NST) {
                stage = 0;
                phase ^= 1u;
              }
            }
            if (!ok) break;
            if constexpr (C2) umma_commit2_mc(&s_full[sb], 0x3);
            else umma_commit(&s_full[sb]);
            ++ns;
          }
        }
        if (u >= 1) {
          const FUnit x = fb_unit(a, g, u - 1);
          const uint32_t fill = static_cast<uint32_t>((u - 1) / FB_DEPTH);
          if (x.first) dh_any = false;
          for (int q = 0; q < a.C && ok; ++q) {
            const int slot = slot_of(u - 1, q);
            uint32_t* cons = &a.consumed[slot * a.C + p];
            if ((mk_prev >> q) & 1u) {
              st_relaxed_gpu(cons, fill + 1u);
              continue;
            }
            if (!dh_any) {
              if (!wait_bounded(dh_empty, (nseg & 1) ^ 1u, a.wait_ns, abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
            }
            for (int kv = 0; kv < KV; ++kv) {
              if (!wait_bounded(&full[stage], phase, a.wait_ns, abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
              // The whole tile has landed (in both CTAs of a pair): its ring
              // slot may be refilled.  The reads are complete, so a relaxed
              // store suffices; a release here would stall this thread, and
              // with it the tensor pipe, on every tile.
              if (kv == KV - 1) st_relaxed_gpu(cons, fill + 1u);
              const uint32_t sA = smem_u32(base + stage * F::STAGE);
              const uint32_t sB = sA + A_BYTES;
#pragma unroll
              for (int j = 0; j < BK / 16; ++j) {
                const uint64_t ad = sdesc_sw128(sA + j * 32, 16, 1024);
                const uint64_t bd = sdesc_sw128(sB + j * 16 * 128, 64 * BK * 2, 1024);
                const uint32_t acc = (dh_any || kv != 0 || j != 0) ? 1u : 0u;
                if constexpr (C2) umma_f16_ss2(tmem_dh, ad, bd, idesc_d, acc);
                else umma_f16_ss(tmem_dh, ad, bd, idesc_d, acc);
              }
              if (kv == 0) dh_any = true;
              if constexpr (C2) umma_commit2_mc(&empty[stage], 0x3);
              else umma_commit(&empty[stage]);
              if (++stage == F::NST) {
                stage = 0;
                phase ^= 1u;
              }
            }
          }
          if (ok && x.last && dh_any) {
            if constexpr (C2) umma_commit2_mc(dh_full, 0x3);
            else umma_commit(dh_full);
            ++nseg;
          }
        }
        mk_prev = mk_cur;
        mk_cur = mk_next;
      }
      if (!ok) {
        set_status(a.status, ST_TIMEOUT);
        *abort_flag = 1;
      }
      if constexpr (C2) umma_commit2_mc(drain, 0x1);
      else umma_commit(drain);
      wait_bounded(drain, 0, DRAIN_LIMIT_NS, nullptr);
    }
  } else {
    // ---------------------------------------------------------- epilogue --
    const int quad = warp & 3;
    const int rin = quad * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    uint8_t* const stage_base = staging + quad * 2 * (32 * 128);
    uint32_t nstore = 0;
    uint32_t s_empty_leader[2] = {0u, 0u}, dh_empty_leader = 0u;
    if constexpr (C2) {
      s_empty_leader[0] = mapa_shared(smem_u32(&s_empty[0]), 0);
      s_empty_leader[1] = mapa_shared(smem_u32(&s_empty[1]), 0);
      dh_empty_leader = mapa_shared(smem_u32(dh_empty), 0);
    }
    int ns = 0, nseg = 0;
    bool ok = true;
    const uint64_t ring_policy = l2_policy_evict_last();  // read by every member, then rewritten
    // Staging per warp: 8 KB, four 2 KB slots for G'' blocks (the TMA store
    // of a block may still be reading its slot while the next three are
    // filled) or two 4 KB slots for fp32 dH blocks during a flush (which
    // drains all pending reads before and after).
    uint32_t ng = 0;
    auto g_buf = [&]() -> uint8_t* {
      uint8_t* sb = stage_base + (ng & 3) * (32 * 64);
      if (lane == 0) bulk_wait_read<3>();
      __syncwarp();
      ++ng;
      return sb;
    };
    auto staging_buf = [&]() -> uint8_t* {
      uint8_t* sb = stage_base + (nstore & 1) * (32 * 128);
      if (lane == 0) bulk_wait_read<1>();
      __syncwarp();
      return sb;
    };
    // dH of a finished segment: -coeff * acc (or zeros when nothing was
    // accumulated) as fp32 32x32 blocks into buffer x.buf.
    auto flush = [&](const FUnit& x, bool any) {
      const int row0 = x.r * F::TH + static_cast<int>(rank) * BM + quad * 32;
      const int row = row0 + lane;
      const float gc = row < a.M ? -a.coeff[row] : 0.f;
      auto put = [&](int c, const uint32_t* r) {
        uint8_t* sb = staging_buf();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float4 o = (r == nullptr || gc == 0.f)
                               ? make_float4(0.f, 0.f, 0.f, 0.f)
                               : make_float4(gc * u2f(r[4 * i]), gc * u2f(r[4 * i + 1]),
                                             gc * u2f(r[4 * i + 2]), gc * u2f(r[4 * i + 3]));
          *reinterpret_cast<float4*>(sb + lane * 128 + ((i ^ (lane & 7)) << 4)) = o;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (x.buf == 0)
            tma_store_3d(&tmD0, sb, p * FB_DS + c * 32, row0, 0);
          else
            tma_store_3d(&tmD1, sb, p * FB_DS + c * 32, row0 - a.row_rem, x.buf - 1);
          bulk_commit();
        }
        ++nstore;
      };
      const int nchunks = min(FB_DS / 32, (a.D - p * FB_DS + 31) / 32);
      if (lane == 0) bulk_wait_read<0>();  // the G'' slots overlap the dH slots
      __syncwarp();
      if (any) {
        if (!wait_bounded(dh_full, nseg & 1, a.wait_ns, abort_flag)) {
          ok = false;
          return;
        }
        tc_fence_after();
        drain_chunks(tmem_dh + lane_addr, nchunks,
                     [&](int c, const uint32_t (&r)[32]) { put(c, r); });
        tc_fence_before();
        if constexpr (C2) mbar_arrive_cluster(dh_empty_leader);
        else mbar_arrive(dh_empty);
        ++nseg;
      } else {
        for (int c = 0; c < nchunks; ++c) put(c, nullptr);
      }
      if (lane == 0) bulk_wait_read<0>();
      __syncwarp();
    };
    bool seg_any = false, prev_any = false;
    FUnit prev{};
    const uint32_t all_c = a.C >= 32 ? ~0u : ((1u << a.C) - 1u);
    uint32_t mk_cur = 0;
    if (n_u > 0) {
      const FUnit x0 = fb_unit(a, g, 0);
      mk_cur = fb_mask(a, x0.r, x0.j);
    }
    for (int u = 0; u < n_u && ok; ++u) {
      uint32_t mk_next = 0;
      if (u + 1 < n_u) {
        const FUnit xn = fb_unit(a, g, u + 1);
        mk_next = fb_mask(a, xn.r, xn.j);
      }
      const FUnit x = fb_unit(a, g, u);
      if (x.first) seg_any = false;
      seg_any = seg_any || (mk_cur & all_c) != all_c;
      const int v = x.j * a.C + p;
      const int slot = slot_of(u, p);
      const uint32_t fill = static_cast<uint32_t>(u / FB_DEPTH);
      uint32_t* rdy = &a.ready[slot * 2 + static_cast<int>(rank)];
      if (!((mk_cur >> p) & 1u)) {
        const int sb = ns % F::SB;
        if (!wait_bounded(&s_full[sb], (ns / F::SB) & 1, a.wait_ns, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // every member is done with this slot's previous fill
        bool w_ok = true;
        if (fill >= 1 && lane == 0) {
          for (int c = 0; c < a.C && w_ok; ++c)
            w_ok = wait_flag_geq(&a.consumed[slot * a.C + c], fill, a.wait_ns, abort_flag);
          fence_proxy_async_global();
        }
        if (!__shfl_sync(0xffffffffu, w_ok ? 1 : 0, 0)) {
          ok = false;
          break;
        }
        const int row = x.r * F::TH + static_cast<int>(rank) * BM + rin;
        const bool live = row < a.M;
        const int y = live ? a.labels[row] : -1;
        const float nl = live ? -a.lse[row] * LOG2E : 0.f;
        const int grow0 = slot * F::TH + static_cast<int>(rank) * BM + quad * 32;
        drain_chunks(tmem_base + lane_addr + sb * F::BV, F::BV / 32,
                     [&](int c, const uint32_t (&r)[32]) {
                       uint32_t pk[16];
                       grad_chunk(r, v * F::BV + c * 32, y, nl, a.filter_eps, a.V, a.softcap,
                                  a.inv_cap, 1, pk);
                       uint8_t* sbuf = g_buf();
#pragma unroll
                       for (int i = 0; i < 4; ++i)
                         *reinterpret_cast<uint4*>(sbuf + lane * 64 +
                                                   ((i ^ ((lane >> 1) & 3)) << 4)) =
                             live ? make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2],
                                               pk[4 * i + 3])
                                  : make_uint4(0, 0, 0, 0);
                       fence_proxy_async_smem();
                       __syncwarp();
                       if (lane == 0) {
                         tma_store_2d_hint(&tmGs, sbuf, c * 32, grow0, ring_policy);
                         bulk_commit();
                       }
                     });
        tc_fence_before();
        if constexpr (C2) mbar_arrive_cluster(s_empty_leader[sb]);
        else mbar_arrive(&s_empty[sb]);
        ++ns;
        if (lane == 0) {
          bulk_wait<0>();  // the tile is in global memory (L2)
          fence_proxy_async_global();
          red_release_gpu_add(rdy, 1u);
        }
      } else {
        // Nothing to publish, but this warp's count for the fill must not
        // reach the slot's consumer before every warp's count for the fill
        // before it: wait, as a publisher does, until that fill is consumed.
        bool w_ok = true;
        if (fill >= 1 && lane == 0)
          for (int c = 0; c < a.C && w_ok; ++c)
            w_ok = wait_flag_geq(&a.consumed[slot * a.C + c], fill, a.wait_ns, abort_flag);
        if (!__shfl_sync(0xffffffffu, w_ok ? 1 : 0, 0)) {
          ok = false;
          break;
        }
        if (lane == 0) red_release_gpu_add(rdy, 1u);
      }
      __syncwarp();
      if (u >= 1 && prev.last) flush(prev, prev_any);
      prev = x;
      prev_any = seg_any;
      mk_cur = mk_next;
    }
    if (ok && n_u > 0) flush(prev, prev_any);
    if (!ok) {
      set_status(a.status, ST_TIMEOUT);
      *abort_flag = 1;
    }
    if (lane == 0) bulk_wait<0>();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if constexpr (C2) cluster_sync_all();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if constexpr (C2) tmem_dealloc2(tmem_base, FB_TMEM_COLS);
    else tmem_dealloc(tmem_base, FB_TMEM_COLS);
  }
}

// dH rows of the remainder row tiles += their partial buffers 1..k-1, in
// buffer order (k = the number of groups that shared the row tile).  The
// partial buffers hold rows [row_rem, M).
__global__ void __launch_bounds__(256) fused_sum_parts_kernel(
    float4* __restrict__ dh, const float4* __restrict__ parts, FusedArgs a, int TH) {
  const int D4 = a.D / 4;
  const int64_t n = static_cast<int64_t>(a.M - a.row_rem) * D4;
  for (int64_t t = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; t < n;
       t += int64_t(gridDim.x) * blockDim.x) {
    const int m = a.row_rem + static_cast<int>(t / D4);
    const int k = fb_slices(a, m / TH - a.waves * a.G);
    const int64_t idx = static_cast<int64_t>(a.row_rem) * D4 + t;
    float4 s = dh[idx];
    for (int b = 1; b < k; ++b) {
      const float4 q = parts[static_cast<size_t>(b - 1) * n + t];
      s.x += q.x;
      s.y += q.y;
      s.z += q.z;
      s.w += q.w;
    }
    dh[idx] = s;
  }
}

}  // namespace cce
