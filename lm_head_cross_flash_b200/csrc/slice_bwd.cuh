// slice_bwd.cuh — the sliced backward for small M (at most 64 head rows,
// dense bf16 heads, D <= 2048): recompute each vocab tile, form the
// coefficient tile and contract it with W into a TMEM-resident dH, reading
// W from HBM once.
//
// What it computes is the fused-head backward ("ORPO training — design"
// 0.0.6, Memory & speed, fused-head implementation spec, "Backward
// (recompute vocab tiles from the saved LSE)"): for every vocab tile,
// s = H W_t^T, G'' = softmax(s) - onehot(label) (filtered, softcapped as in
// the forward), dH -= coeff * (G'' W_t).  Nothing [M, V] is formed.
//
// Why a second fused design: with one row tile the fused kernel of
// fused_bwd.cuh splits D between the members of a group and each member
// recomputes whole S tiles, so every W tile is read twice (once by its S
// owner over all of D, once per d-slice by the dH phase), and at small M the
// groups hold more W between the two reads than L2 keeps.  Here the
// contraction over D is split as well: the Ccl CTAs of a cluster each own
// SL_DS columns of D, compute a PARTIAL logit tile S_c^T = W_t[:, slice] .
// H[:, slice]^T from the same W bytes they later need for their dH slice,
// and sum the partials through distributed shared memory.  Every W byte
// crosses HBM once (the dH phase re-reads its box from L2 a few tiles
// later).
//
// Per tile t of 128 vocab rows, in each CTA c of the cluster:
//  1. MMA: S_c^T[v, m] (128 x 64, fp32, TMEM) over the slice's 256 d.
//  2. Drain thread v reads its row from TMEM and sends it by st.async to the
//     CTA that reduces rows v of the tile (CTA v / R, R = 128 / Ccl rows
//     each).
//  3. That CTA's reducer warps sum the Ccl partials in a fixed order (c = 0,
//     1, ...), form G''[v, m] in bf16, write its R rows into its own G''
//     tile and copy them by cp.async.bulk into the same rows of every other
//     CTA's tile.
//  4. MMA: dH^T[d, m] += W_t[:, slice]^T . G''^T (two 128-row d blocks; W
//     as an MN-major A operand, G'' as an MN-major B operand).
// At the end each CTA scales its dH^T columns by -coeff[m] and writes them
// to the cluster's partial dH; a second kernel sums the clusters' partials
// in a fixed order (the result does not depend on timing).
//
// Roles (384 threads): warp 0 loads the H slice once and streams S-phase W
// boxes ([128 v x 64 d], HBM); warp 1 issues the S MMAs; warp 2 streams
// dH-phase W boxes ([64 v x 64 d] x 2, from L2); warps 3-6 drain S^T (one
// TMEM lane quarter each) and send the partials; warp 7 issues the dH MMAs;
// warps 8-11 reduce the partials and form G''.  The drain of tile k + 1 and
// the reduction of tile k run at the same time.
//
// Cluster protocol (all mbarriers, double-buffered by tile parity b; every
// wait bounded):
//  pfull[b]   partials of a tile received (tx bytes; armed by this CTA)
//  pempty[b]  every reducer warp of every CTA has read this CTA's partials
//             of the tile two back (4 Ccl remote arrivals, relaxed)
//  gfull[b]   G'' tile complete (tx bytes of the peers' rows, plus the dH
//             MMA thread's arm and the four reducer warps' arrivals)
//  gempty[b]  every CTA's dH MMAs of the tile two back are done, so its rows
//             may be overwritten (tcgen05.commit multicast, Ccl arrivals)
// Remote arrivals and copies that nobody would wait for (the last tiles)
// are not issued, and a cluster barrier precedes exit, so no CTA exits
// while a peer can still reach its shared memory.
//
// Measured (D = 2048, V = 262,144, 15 clusters of 8): 0.51 ms for 8 to 64
// rows, about 6,300 cycles per tile for every role.  Shared memory bounds
// the depth: 64 KB S ring, 32 KB dH ring, 32 KB H slice, two 16 KB G''
// tiles and two 32 KB partial buffers fill 224 KB, so each exchange chain
// (send -> reduce everywhere -> release; reduce -> copy -> dH MMAs
// everywhere -> release) spans only two tiles.
#pragma once

#include "ptx.cuh"
#include "gemm_tc.cuh"

namespace cce {

constexpr int SL_DS = 256;     // columns of D per CTA
constexpr int SL_BV = 128;     // vocab rows per tile
constexpr int SL_MP = 64;      // head rows (M <= 64; the rest are zero)
constexpr int SL_MAXC = 8;     // CTAs per cluster (portable limit)
constexpr int SL_NS = 4;       // S-phase stages: one [128 v x 64 d] box each
constexpr int SL_ND = 2;       // dH-phase stages: two [64 v x 64 d] boxes each
constexpr int SL_STAGE = 16384;
constexpr int SL_H = SL_MP * SL_DS * 2;     // H slice: four [64 m x 64 d] boxes
constexpr int SL_G = SL_BV * SL_MP * 2;     // one G'' tile [128 v x 64 m] bf16
constexpr int SL_RECV = SL_BV * SL_MP * 4;  // partial logits received per tile
constexpr int SL_OFF_D = SL_NS * SL_STAGE;
constexpr int SL_OFF_H = SL_OFF_D + SL_ND * SL_STAGE;
constexpr int SL_OFF_G = SL_OFF_H + SL_H;
constexpr int SL_OFF_R = SL_OFF_G + 2 * SL_G;
constexpr int SL_OFF_BAR = SL_OFF_R + 2 * SL_RECV;
constexpr int SL_BAR_BYTES = 256;
constexpr int SL_OFF_ROW = SL_OFF_BAR + SL_BAR_BYTES;  // nl, y, coeff per head row
constexpr int SL_SMEM = SL_OFF_ROW + 3 * SL_MP * 4 + 1024;
constexpr int SL_EPI = 4;      // drain warps, and reducer warps
constexpr int SL_DRAIN0 = 3;   // warps 3-6 drain S^T and send partials (TMEM lane quarters)
constexpr int SL_DHMMA = 7;    // warp 7 issues the dH MMAs
constexpr int SL_RED0 = 8;     // warps 8-11 reduce partials and form G''
constexpr int SL_THREADS = 32 * (SL_RED0 + SL_EPI);
constexpr uint32_t SL_TMEM_COLS = 256;  // S^T buffers [0, 128), dH^T blocks [128, 256)
static_assert(SL_SMEM <= 232448, "sliced backward exceeds the shared memory of a CTA");

struct SliceArgs {
  int M, V, D;
  int Ccl;        // CTAs per cluster (d slices): 1, 2, 4 or 8 (the kernel's CCL)
  int n_cl;       // clusters
  int n_vt;       // vocab tiles of SL_BV rows
  uint64_t wait_ns;
  uint32_t* status;
  const int32_t* labels;
  const float* lse;
  const float* coeff;
  float filter_eps;
  const uint8_t* tile_skip;  // the one row tile's 256-wide vocab blocks; null: none
  const uint8_t* row_skip;   // [1]: the row tile has no nonzero cotangent
  float softcap, inv_cap;
  float* parts;   // [n_cl, M, D] fp32, one partial dH per cluster
};

// First tile >= t of a cluster's sequence (its index, then every n_cl-th
// tile) that is not skipped, or n_vt.  A tile is skipped when no row has a
// cotangent (none = row_skip[0], read once per thread) or block skip proved
// every probability of its 256-wide vocab block below the filter.
__device__ __forceinline__ int sl_next(const SliceArgs& a, int t, bool none) {
  if (none) return a.n_vt;
  for (; t < a.n_vt; t += a.n_cl)
    if (a.tile_skip == nullptr || a.tile_skip[t >> 1] == 0) return t;
  return a.n_vt;
}

// 16 bytes into another CTA's shared memory (shared::cluster address),
// counted on that CTA's mbarrier.
__device__ __forceinline__ void st_async_v4(uint32_t dst, uint32_t bar, uint32_t x, uint32_t y,
                                            uint32_t z, uint32_t w) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, "
      "[%5];" ::"r"(dst),
      "r"(x), "r"(y), "r"(z), "r"(w), "r"(bar)
      : "memory");
}
// Bulk copy of `bytes` (multiple of 16) from this CTA's shared memory into
// another CTA's, counted on that CTA's mbarrier.
__device__ __forceinline__ void bulk_copy_s2c(uint32_t dst, uint32_t src, uint32_t bytes,
                                              uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, "
      "[%3];" ::"r"(dst),
      "r"(src), "r"(bytes), "r"(bar)
      : "memory");
}
// Remote arrive without release semantics.  Used to hand a partial-logit
// buffer back to its writer: the loads it guards have returned (their values
// are consumed before the arrive), and a release here would wait for this
// thread's own outstanding remote stores of the next tile first (about 2,000
// cycles per tile, measured).
__device__ __forceinline__ void mbar_arrive_cluster_relaxed(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
// tcgen05.commit arriving once on the mbarrier at this offset in every CTA
// of `mask` (single-CTA MMAs).
__device__ __forceinline__ void umma_commit_mc(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 "
      "[%0], %1;" ::"r"(smem_u32(bar)),
      "h"(mask)
      : "memory");
}

// G'' of one element (logit s of vocab row vg for a head row with
// nl = -lse * log2 e and label y): the arithmetic of grad_chunk, one value.
__device__ __forceinline__ float sl_grad(float s, int vg, int y, float nl, const SliceArgs& a) {
  if (vg >= a.V) return 0.f;
  const bool tgt = vg == y;
  if (a.softcap > 0.f) {
    const float th = tanh_ex2(s * a.inv_cap);
    float p = softmax_p(a.softcap * th, nl);
    if (p < a.filter_eps && !tgt) p = 0.f;
    return (tgt ? p - 1.f : p) * (1.f - th * th);
  }
  float p = softmax_p(s, nl);
  if (p < a.filter_eps && !tgt) p = 0.f;
  return tgt ? p - 1.f : p;
}

template <int CCL>
__global__ void __launch_bounds__(SL_THREADS, 1)
    slice_bwd_kernel(const __grid_constant__ CUtensorMap tmH,   // H [M, D], box 64 x 64
                     const __grid_constant__ CUtensorMap tmWs,  // W [V, D], box 64 x 128
                     const __grid_constant__ CUtensorMap tmWd,  // W [V, D], box 64 x 64
                     const SliceArgs a) {
  const uint32_t rank = cluster_ctarank();
  const int cl = static_cast<int>(cluster_id_x());
  constexpr int Ccl = CCL;
  constexpr int R = SL_BV / Ccl;  // rows of a tile this CTA reduces
  const int d0 = static_cast<int>(rank) * SL_DS;
  constexpr uint32_t peer_g = static_cast<uint32_t>((Ccl - 1) * R * 128);  // G'' from peers
  constexpr uint16_t all_mask = static_cast<uint16_t>((1u << Ccl) - 1u);

  extern __shared__ uint8_t dyn_smem[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
  uint8_t* s_ring = base;
  uint8_t* d_ring = base + SL_OFF_D;
  uint8_t* hs = base + SL_OFF_H;
  uint8_t* gt = base + SL_OFF_G;                            // G'' tiles [2][128 v][64 m]
  float* recv = reinterpret_cast<float*>(base + SL_OFF_R);  // [2][Ccl][R][64 m]
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + SL_OFF_BAR);
  uint64_t* sfull = bars;               // [SL_NS]
  uint64_t* sempty = sfull + SL_NS;     // [SL_NS]
  uint64_t* dfull = sempty + SL_NS;     // [SL_ND]
  uint64_t* dempty = dfull + SL_ND;     // [SL_ND]
  uint64_t* afull = dempty + SL_ND;     // [2] S^T accumulator written
  uint64_t* aempty = afull + 2;         // [2] S^T accumulator drained
  uint64_t* gfull = aempty + 2;         // [2] G'' tiles k, k + 2, ...
  uint64_t* gempty = gfull + 2;         // [2]
  uint64_t* pfull = gempty + 2;         // [2] partials of tiles b, b + 2, ...
  uint64_t* pempty = pfull + 2;         // [2]
  uint64_t* hfull = pempty + 2;
  uint64_t* dhfull = hfull + 1;
  uint64_t* sdrain = dhfull + 1;
  uint64_t* ddrain = sdrain + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ddrain + 1);
  int* n_slot = reinterpret_cast<int*>(tmem_slot + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);
  float* nl_s = reinterpret_cast<float*>(base + SL_OFF_ROW);
  int* y_s = reinterpret_cast<int*>(nl_s + SL_MP);
  float* cf_s = reinterpret_cast<float*>(y_s + SL_MP);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SL_NS; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], 1);
    }
    for (int s = 0; s < SL_ND; ++s) {
      mbar_init(&dfull[s], 1);
      mbar_init(&dempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&afull[b], 1);
      mbar_init(&aempty[b], SL_EPI);
      mbar_init(&gfull[b], 1 + SL_EPI);
      mbar_init(&gempty[b], static_cast<uint32_t>(Ccl));
      mbar_init(&pfull[b], 1);
      mbar_init(&pempty[b], static_cast<uint32_t>(Ccl * SL_EPI));
    }
    mbar_init(hfull, 1);
    mbar_init(dhfull, 1);
    mbar_init(sdrain, 1);
    mbar_init(ddrain, 1);
    *abort_flag = 0;
    const bool none = a.row_skip[0] != 0;
    int n = 0;
    for (int t = sl_next(a, cl, none); t < a.n_vt; t = sl_next(a, t + a.n_cl, none)) ++n;
    *n_slot = n;
    fence_barrier_init();
    fence_proxy_async_smem();
    // the first tiles' arms: partials and G'' of tiles 0 and 1
    for (int b = 0; b < 2; ++b) {
      mbar_arrive_expect_tx(&pfull[b], SL_RECV);
      mbar_arrive_expect_tx(&gfull[b], peer_g);
    }
    tma_prefetch_desc(&tmH);
    tma_prefetch_desc(&tmWs);
    tma_prefetch_desc(&tmWd);
  }
  if (warp >= SL_RED0) {
    const int m = threadIdx.x - SL_RED0 * 32;
    if (m < SL_MP) {
      const bool live = m < a.M;
      nl_s[m] = live ? -a.lse[m] * LOG2E : 0.f;
      y_s[m] = live ? a.labels[m] : -1;
      cf_s[m] = live ? a.coeff[m] : 0.f;
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, SL_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int n = *n_slot;
  const bool none = a.row_skip[0] != 0;
  const int t_first = sl_next(a, cl, none);
  auto fail = [&]() {
    set_status(a.status, ST_TIMEOUT);
    *abort_flag = 1;
  };

  if (warp == 0) {
    // ------------------------------------------- S-phase loads (HBM) --
    if (lane == 0) {
      bool ok = true;
      mbar_arrive_expect_tx(hfull, SL_H);
      for (int q = 0; q < 4; ++q) tma_load_2d(hs + q * 8192, &tmH, hfull, d0 + 64 * q, 0);
      int st = 0;
      uint32_t ph = 0;
      for (int t = t_first; t < a.n_vt && ok; t = sl_next(a, t + a.n_cl, none)) {
        for (int q = 0; q < 4; ++q) {
          if (!wait_bounded(&sempty[st], ph ^ 1u, a.wait_ns, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sfull[st], SL_STAGE);
          tma_load_2d(s_ring + st * SL_STAGE, &tmWs, &sfull[st], d0 + 64 * q, t * SL_BV);
          if (++st == SL_NS) {
            st = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) fail();
    }
  } else if (warp == 2) {
    // ------------------------------------------- dH-phase loads (L2) --
    if (lane == 0) {
      bool ok = true;
      int st = 0;
      uint32_t ph = 0;
      for (int t = t_first; t < a.n_vt && ok; t = sl_next(a, t + a.n_cl, none)) {
        for (int h = 0; h < 2 && ok; ++h) {
          for (int vh = 0; vh < 2; ++vh) {
            if (!wait_bounded(&dempty[st], ph ^ 1u, a.wait_ns, abort_flag)) {
              ok = false;
              break;
            }
            uint8_t* s = d_ring + st * SL_STAGE;
            mbar_arrive_expect_tx(&dfull[st], SL_STAGE);
            tma_load_2d(s, &tmWd, &dfull[st], d0 + 128 * h, t * SL_BV + 64 * vh);
            tma_load_2d(s + 8192, &tmWd, &dfull[st], d0 + 128 * h + 64, t * SL_BV + 64 * vh);
            if (++st == SL_ND) {
              st = 0;
              ph ^= 1u;
            }
          }
        }
      }
      if (!ok) fail();
    }
  } else if (warp == 1) {
    // ------------------------------------------ S MMA issuer (TMEM) --
    // S_c^T(k) = W_t[:, slice] . H[:, slice]^T into accumulator k & 1
    if (lane == 0) {
      const uint32_t idesc_s = idesc_f16(SL_BV, SL_MP, 1, false, false);
      bool ok = wait_bounded(hfull, 0, a.wait_ns, abort_flag);
      tc_fence_after();
      int st = 0;
      uint32_t ph = 0;
      for (int k = 0; k < n && ok; ++k) {
        const int b = k & 1;
        if (!wait_bounded(&aempty[b], ((k >> 1) & 1) ^ 1u, a.wait_ns, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem_base + static_cast<uint32_t>(b * SL_MP);
        for (int q = 0; q < 4; ++q) {
          if (!wait_bounded(&sfull[st], ph, a.wait_ns, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = smem_u32(s_ring + st * SL_STAGE);
          const uint32_t sB = smem_u32(hs + q * 8192);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            umma_f16_ss(acc, sdesc_sw128(sA + j * 32, 16, 1024), sdesc_sw128(sB + j * 32, 16, 1024),
                        idesc_s, (q | j) != 0 ? 1u : 0u);
          umma_commit(&sempty[st]);
          if (++st == SL_NS) {
            st = 0;
            ph ^= 1u;
          }
        }
        if (ok) umma_commit(&afull[b]);
      }
      if (!ok) fail();
      umma_commit(sdrain);
      wait_bounded(sdrain, 0, DRAIN_LIMIT_NS, nullptr);
    }
  } else if (warp == SL_DHMMA) {
    // ----------------------------------------- dH MMA issuer (TMEM) --
    // dH^T[d, m] += W_t[:, slice]^T . G''(k)^T, two 128-row blocks of d
    if (lane == 0) {
      const uint32_t idesc_d = idesc_f16(128, SL_MP, 1, true, true);
      bool ok = true;
      int st = 0;
      uint32_t ph = 0;
      for (int k = 0; k < n && ok; ++k) {
        const int b = k & 1;
        if (!wait_bounded(&gfull[b], (k >> 1) & 1, a.wait_ns, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t gB = smem_u32(gt + b * SL_G);
        for (int h = 0; h < 2 && ok; ++h) {
          for (int vh = 0; vh < 2; ++vh) {
            if (!wait_bounded(&dfull[st], ph, a.wait_ns, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sA = smem_u32(d_ring + st * SL_STAGE);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              // A: [128 d x 16 v] MN-major, two 64-d atoms 8 KB apart
              const uint64_t ad = sdesc_sw128(sA + j * 16 * 128, 8192, 1024);
              // B: [64 m x 16 v] MN-major, one 64-m atom
              const uint64_t bd = sdesc_sw128(gB + (vh * 64 + j * 16) * 128, 8192, 1024);
              umma_f16_ss(tmem_base + 2 * SL_MP + static_cast<uint32_t>(h * SL_MP), ad, bd,
                          idesc_d, (k | vh | j) != 0 ? 1u : 0u);
            }
            umma_commit(&dempty[st]);
            if (++st == SL_ND) {
              st = 0;
              ph ^= 1u;
            }
          }
        }
        if (ok && k + 2 < n) {
          // tile k + 2 may overwrite this tile in every CTA once the MMAs
          // above are done; then arm this CTA's G'' barrier for it
          umma_commit_mc(&gempty[b], all_mask);
          mbar_arrive_expect_tx(&gfull[b], peer_g);
        }
      }
      if (!ok) fail();
      umma_commit(dhfull);
      umma_commit(ddrain);
      wait_bounded(ddrain, 0, DRAIN_LIMIT_NS, nullptr);
    }
  } else if (warp >= SL_DRAIN0 && warp < SL_DRAIN0 + SL_EPI) {
    // ------------------------------------------- drain and send (TMEM) --
    const int quad = warp & 3;                  // TMEM lanes 32 quad .. 32 quad + 31
    const int v = quad * 32 + lane;             // vocab row of the tile (S^T) / d (dH^T)
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    // where row v's partial goes: reducer v / R, slot [rank][v % R] of its
    // buffer (tile & 1)
    const int red = v / R;
    const int slot = (static_cast<int>(rank) * R + (v - red * R)) * SL_MP;
    const uint32_t p_dst0 = mapa_shared(smem_u32(recv + slot), static_cast<uint32_t>(red));
    const uint32_t p_bar0 = mapa_shared(smem_u32(&pfull[0]), static_cast<uint32_t>(red));
    bool ok = true;
    for (int j = 0; j < n && ok; ++j) {
      const int b = j & 1;
      // this CTA's partial logits of row v for tile j
      ok = __all_sync(0xffffffffu, wait_bounded(&afull[b], (j >> 1) & 1, a.wait_ns, abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint32_t r0[32], r1[32];
      tmem_ld32(tmem_base + lane_addr + static_cast<uint32_t>(b * SL_MP), r0);
      tmem_ld32(tmem_base + lane_addr + static_cast<uint32_t>(b * SL_MP + 32), r1);
      tmem_ld_wait(r0);
      tmem_ld_wait(r1);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&aempty[b]);
      // to the reducer of row v, once every reducer has read tile j - 2
      // out of buffer b
      if (j >= 2 && !wait_bounded(&pempty[b], ((j - 2) >> 1) & 1, a.wait_ns, abort_flag)) {
        ok = false;
        break;
      }
      const uint32_t dst = p_dst0 + static_cast<uint32_t>(b * SL_RECV);
      const uint32_t bar = p_bar0 + static_cast<uint32_t>(b * 8);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        st_async_v4(dst + 16 * i, bar, r0[4 * i], r0[4 * i + 1], r0[4 * i + 2], r0[4 * i + 3]);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        st_async_v4(dst + 128 + 16 * i, bar, r1[4 * i], r1[4 * i + 1], r1[4 * i + 2],
                    r1[4 * i + 3]);
    }
    if (!ok) fail();
    // this cluster's partial dH: thread v holds d = d0 + 128 h + v of block
    // h for all 64 head rows
    if (ok && n > 0 && !wait_bounded(dhfull, 0, a.wait_ns, abort_flag)) fail();
    tc_fence_after();
    float* out = a.parts + static_cast<size_t>(cl) * a.M * a.D;
    for (int h = 0; h < 2; ++h) {
      uint32_t q0[32], q1[32];
      if (n > 0) {
        tmem_ld32(tmem_base + lane_addr + 2 * SL_MP + static_cast<uint32_t>(h * SL_MP), q0);
        tmem_ld32(tmem_base + lane_addr + 2 * SL_MP + static_cast<uint32_t>(h * SL_MP + 32), q1);
        tmem_ld_wait(q0);
        tmem_ld_wait(q1);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) q0[i] = q1[i] = 0u;
      }
      const int d = d0 + 128 * h + v;
      if (d < a.D) {
#pragma unroll
        for (int m = 0; m < 32; ++m)
          if (m < a.M) out[static_cast<size_t>(m) * a.D + d] = -cf_s[m] * u2f(q0[m]);
#pragma unroll
        for (int m = 0; m < 32; ++m)
          if (m + 32 < a.M) out[static_cast<size_t>(m + 32) * a.D + d] = -cf_s[m + 32] * u2f(q1[m]);
      }
    }
  } else if (warp >= SL_RED0) {
    // --------------------------------------------------------- reduce --
    // This warp reduces rows [rank R + e R/4, rank R + (e+1) R/4) of every
    // tile: the Ccl partials summed in a fixed order of c, G'' formed and
    // written into this CTA's tile k & 1 once tile k - 2's MMAs are done
    // everywhere, then copied into the same rows of every other CTA's tile.
    // No barrier spans the four warps: each signals and copies its own rows,
    // so a warp that gives up on a bounded wait only stops itself.
    const int e = warp - SL_RED0;
    constexpr int RW = R / SL_EPI;
    const int row0 = static_cast<int>(rank) * R + e * RW;
    bool ok = true;
    int t = t_first;
    for (int k = 0; k < n; ++k, t = sl_next(a, t + a.n_cl, none)) {
      const int b = k & 1;
      if (!wait_bounded(&pfull[b], (k >> 1) & 1, a.wait_ns, abort_flag) ||
          (k >= 2 && !wait_bounded(&gempty[b], ((k - 2) >> 1) & 1, a.wait_ns, abort_flag))) {
        ok = false;
        break;
      }
      const float* rb = recv + b * (SL_RECV / 4);
      uint8_t* gtile = gt + b * SL_G;
#pragma unroll
      for (int i0 = 0; i0 < RW * 8; i0 += 32) {
        const int i = i0 + lane;
        const int vl = e * RW + (i >> 3), c8 = i & 7;
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.f;
#pragma unroll
        for (int c = 0; c < Ccl; ++c) {
          const float4* src = reinterpret_cast<const float4*>(rb + (c * R + vl) * SL_MP + c8 * 8);
          const float4 x0 = src[0], x1 = src[1];
          acc[0] += x0.x;
          acc[1] += x0.y;
          acc[2] += x0.z;
          acc[3] += x0.w;
          acc[4] += x1.x;
          acc[5] += x1.y;
          acc[6] += x1.z;
          acc[7] += x1.w;
        }
        const int vt = static_cast<int>(rank) * R + vl;
        const int vg = t * SL_BV + vt;
        uint32_t pk[4];
#pragma unroll
        for (int q = 0; q < 8; q += 2) {
          const int m0 = c8 * 8 + q;
          const float g0 = m0 < a.M ? sl_grad(acc[q], vg, y_s[m0], nl_s[m0], a) : 0.f;
          const float g1 =
              m0 + 1 < a.M ? sl_grad(acc[q + 1], vg, y_s[m0 + 1], nl_s[m0 + 1], a) : 0.f;
          pk[q >> 1] = pack2(g0, g1, 1);
        }
        // [128 v x 64 m] MN-major, 128-byte swizzle: chunk c8 of row vt at
        // chunk c8 ^ (vt & 7)
        *reinterpret_cast<uint4*>(gtile + vt * 128 + ((c8 ^ (vt & 7)) << 4)) =
            make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      fence_proxy_async_smem();  // the rows feed tcgen05.mma and cp.async.bulk
      __syncwarp();              // the warp's partials are read, its rows written
      if (k + 2 < n) {
        // buffer b takes tile k + 2: warp 0 arms it before any reducer
        // signal can release a sender
        if (e == 0 && lane == 0) mbar_arrive_expect_tx(&pfull[b], SL_RECV);
        __syncwarp();
        if (lane < Ccl)
          mbar_arrive_cluster_relaxed(
              mapa_shared(smem_u32(&pempty[b]), static_cast<uint32_t>(lane)));
      }
      const uint32_t src = smem_u32(gtile + row0 * 128);
      if (lane < Ccl && lane != static_cast<int>(rank))
        bulk_copy_s2c(mapa_shared(src, static_cast<uint32_t>(lane)), src,
                      static_cast<uint32_t>(RW * 128),
                      mapa_shared(smem_u32(&gfull[b]), static_cast<uint32_t>(lane)));
      if (lane == 0) mbar_arrive(&gfull[b]);
    }
    if (!ok) fail();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, SL_TMEM_COLS);
  }
}

// dH = parts[0] + parts[1] + ... + parts[n_cl - 1] (fixed order); n4 float4
// elements per partial.
__global__ void slice_sum_kernel(float4* __restrict__ dh, const float4* __restrict__ parts,
                                 int n_cl, int64_t n4) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float4 v = parts[i];
    for (int c = 1; c < n_cl; ++c) {
      const float4 q = parts[c * n4 + i];
      v.x += q.x;
      v.y += q.y;
      v.z += q.z;
      v.w += q.w;
    }
    dh[i] = v;
  }
}

}  // namespace cce
