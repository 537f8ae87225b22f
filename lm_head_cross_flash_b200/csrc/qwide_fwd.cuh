// qwide_fwd.cuh — the transposed forward of a 4/8-bit head for up to 256
// head rows (the library chooses it for 129 to 240): S^T[v, m] =
// W_t[v, :] . H[m, :] with the dequantised head tile as the A operand in
// TMEM, as in qsmall_fwd.cuh, but with N up to 256 (M rounded up to 16), so
// one accumulator is as wide as the head rows.
//
// What it computes is the forward of the flash-CCE head (ORPO design 0.0.6,
// fused-head implementation spec, "Forward"; Training design §5.6 for the
// quantised weights): the same per-(256-vocab block, row) partials (max,
// sum of exp), block maxima and target logits as the other forward forms,
// for merge_lse_kernel.
//
// Per CTA: 256-row vocab blocks in turn, each as two 128-row units run one
// after the other (a unit is a K loop over D in groups of 64, starting at
// group b mod (D / 64) and wrapping).  The accumulator of a unit is up to
// 256 TMEM columns, so a block's two units cannot share one K step as in
// the narrower kernel; the epilogue carries each head row's (max, sum)
// from the first unit to the second and writes the block's partials.
// Roles (448 threads): warp 0 loads by TMA the packed rows of the unit's
// group (128 rows) and the group's 64 columns of H (Mp rows); warp 1
// issues the MMAs (4 per K step, 128 x Mp x 16); warps 2-9 dequantise:
// warps 2-5 the first 32 weights of each row's group, warps 6-9 the other
// 32 (one vocab row per thread, 16 TMEM columns each, one tcgen05.st);
// warps 10-13 drain the accumulator, one vocab row per thread.
//
// TMEM (512 columns): A ring of 8 slots x 32 columns, then the accumulator
// from column 256 (single-buffered: the next unit's MMAs wait for the
// drain, about a tenth of a unit).  All waits are bounded; a timeout sets
// the status word.
#pragma once

#include "qsmall_fwd.cuh"

namespace cce {

constexpr int QW_UNIT = 128;       // vocab rows per unit
constexpr int QW_MAXM = 256;       // head rows at most
constexpr int QW_NA = 8;           // TMEM A slots (32 columns each)
constexpr int QW_ACC0 = 256;       // accumulator column
constexpr int QW_MAXC = QW_MAXM / 32;
constexpr int QW_DQ0 = 2;          // dequantisation warps 2-9
constexpr int QW_EP0 = 10;         // epilogue warps 10-13
constexpr int QW_THREADS = 14 * 32;

// Stage: packed [128 rows x QB*8 bytes] then H [Mp rows x 64 fp16] with the
// 128-byte swizzle (1024-aligned).
template <int QB>
struct QwCfg {
  static constexpr int PK = QW_UNIT * QB * 8;
  static constexpr int HB = QW_MAXM * 128;
  static constexpr int STAGE = PK + HB;
  static constexpr int NST = 5;
  static constexpr int RED = 2 * 2 * 4 * QW_MAXM * 4;  // [parity][m|s][warp][row]
  static constexpr int BC = 4 * 32 * 4;
  static constexpr int BARS = 512;
  static constexpr int SMEM = NST * STAGE + RED + BC + BARS + 1024;
};
static_assert(QwCfg<4>::PK % 1024 == 0 && QwCfg<8>::PK % 1024 == 0, "H box alignment");
static_assert(QwCfg<4>::SMEM <= 232448 && QwCfg<8>::SMEM <= 232448,
              "wide small-M forward exceeds the shared memory of a CTA");

// 32 lanes x 16 consecutive 32-bit columns from registers into TMEM.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

// Half of a group: the 32 weights of 4 packed 4-bit words (element 8c+j =
// bits 4j..4j+3 of word c), converted exactly as dequant_group64 does
// (1024 + q from the bits 0x6400 | q, subtract 1024, one fp16 fma with
// scale and bias).  out[c] holds the 8 fp16 of word c in q4_pos order.
__device__ __forceinline__ void qw_dequant_half_q4(const uint4& w, uint16_t sbits, uint16_t bbits,
                                                   uint4 (&out)[4]) {
  const __half2 s2 = __float2half2_rn(__uint_as_float(static_cast<uint32_t>(sbits) << 16));
  const __half2 b2 = __float2half2_rn(__uint_as_float(static_cast<uint32_t>(bbits) << 16));
  const __half2 k1024 = __float2half2_rn(1024.f);
  const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int c = 0; c < 4; ++c) {
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

// Half of a group of an 8-bit head: 8 packed words (element 4c+j = byte j
// of word c), converted as dequant_group64_q8 does; out[c] holds the 8 fp16
// of words 2c and 2c+1 in q8_pos order.
__device__ __forceinline__ void qw_dequant_half_q8(const uint4& wa, const uint4& wb, uint16_t sbits,
                                                   uint16_t bbits, uint4 (&out)[4]) {
  const __half2 s2 = __float2half2_rn(__uint_as_float(static_cast<uint32_t>(sbits) << 16));
  const __half2 b2 = __float2half2_rn(__uint_as_float(static_cast<uint32_t>(bbits) << 16));
  const __half2 k1024 = __float2half2_rn(1024.f);
  const uint32_t words[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
  for (int c = 0; c < 4; ++c) {
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

template <int QB>
__global__ void __launch_bounds__(QW_THREADS, 1)
    qwide_fwd_kernel(const __grid_constant__ CUtensorMap tmP,  // packed bytes, box {QB*8, 128}
                     const __grid_constant__ CUtensorMap tmH,  // fp16 H, box {64, Mp}, SW128
                     const QsArgs a) {
  using F = QwCfg<QB>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  float* red = reinterpret_cast<float*>(base + F::NST * F::STAGE);  // [2][2][4][QW_MAXM]
  float* bc = red + F::RED / 4;                                     // [4][32]
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(bc) + F::BC);
  uint64_t* full = bars;                // [NST] stage landed (TMA bytes)
  uint64_t* empty = full + F::NST;      // [NST] 8 dequant warps read + MMAs done
  uint64_t* afull = empty + F::NST;     // [QW_NA] 8 dequant warps stored
  uint64_t* aempty = afull + QW_NA;     // [QW_NA] MMAs read
  uint64_t* accfull = aempty + QW_NA;   // unit's MMAs done
  uint64_t* accempty = accfull + 1;     // 4 epilogue warps drained
  uint64_t* drain = accempty + 1;
  uint64_t* epibar = drain + 1;         // [2] 4 epilogue warps wrote their pairs
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(epibar + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < F::NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 9);
    }
    for (int s = 0; s < QW_NA; ++s) {
      mbar_init(&afull[s], 8);
      mbar_init(&aempty[s], 1);
    }
    mbar_init(accfull, 1);
    mbar_init(accempty, 4);
    mbar_init(drain, 1);
    mbar_init(&epibar[0], 4);
    mbar_init(&epibar[1], 4);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmP);
    tma_prefetch_desc(&tmH);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, QS_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int nk = a.nk;
  auto fail = [&]() {
    set_status(a.status, ST_TIMEOUT);
    *abort_flag = 1;
  };
  // K step n of the CTA's sequence: stage, stage parity, A slot, slot parity
  auto step_of = [&](uint32_t n, int& s, uint32_t& ph, int& sa, uint32_t& aph) {
    s = static_cast<int>(n % F::NST);
    ph = (n / F::NST) & 1u;
    sa = static_cast<int>(n % QW_NA);
    aph = (n / QW_NA) & 1u;
  };

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      const uint32_t hbytes = static_cast<uint32_t>(a.Mp) * 128u;
      uint32_t n = 0;
      bool ok = true;
      for (int blk = blockIdx.x; blk < a.n_blk && ok; blk += gridDim.x) {
        const int k0 = blk % nk;
        for (int h = 0; h < 2 && ok; ++h) {
          for (int i = 0; i < nk; ++i, ++n) {
            const int k = k0 + i < nk ? k0 + i : k0 + i - nk;
            int s, sa;
            uint32_t ph, aph;
            step_of(n, s, ph, sa, aph);
            if (!wait_bounded(&empty[s], ph ^ 1u, a.wait_ns, abort_flag)) {
              ok = false;
              break;
            }
            uint8_t* st = base + s * F::STAGE;
            mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(F::PK) + hbytes);
            tma_load_2d(st, &tmP, &full[s], k * QB * 8, blk * QS_BLK + h * QW_UNIT);
            tma_load_2d(st + F::PK, &tmH, &full[s], k * 64, 0);
          }
        }
      }
      if (!ok) fail();
      // every copy issued lands before the CTA can exit
      const uint32_t n0 = n > static_cast<uint32_t>(F::NST) ? n - F::NST : 0u;
      for (uint32_t i = n0; i < n; ++i) {
        int s, sa;
        uint32_t ph, aph;
        step_of(i, s, ph, sa, aph);
        wait_bounded(&full[s], ph, DRAIN_LIMIT_NS, nullptr);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      const uint32_t idesc = idesc_f16(128, a.Mp, 0, false, false);
      const uint32_t dcol = tmem_base + QW_ACC0;
      uint32_t n = 0, un = 0;
      bool ok = true;
      for (int blk = blockIdx.x; blk < a.n_blk && ok; blk += gridDim.x) {
        for (int h = 0; h < 2 && ok; ++h, ++un) {
          if (!wait_bounded(accempty, (un & 1u) ^ 1u, a.wait_ns, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int i = 0; i < nk; ++i, ++n) {
            int s, sa;
            uint32_t ph, aph;
            step_of(n, s, ph, sa, aph);
            if (!wait_bounded(&full[s], ph, a.wait_ns, abort_flag) ||
                !wait_bounded(&afull[sa], aph, a.wait_ns, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sH = smem_u32(base + s * F::STAGE + F::PK);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              umma_f16_ts(dcol, tmem_base + static_cast<uint32_t>(sa * 32 + j * 8),
                          sdesc_sw128(sH + j * 32, 16, 1024), idesc, (i | j) != 0 ? 1u : 0u);
            umma_commit(&empty[s]);
            umma_commit(&aempty[sa]);
          }
          if (!ok) break;
          umma_commit(accfull);
        }
      }
      if (!ok) fail();
      // every MMA issued completes before TMEM is released
      umma_commit(drain);
      wait_bounded(drain, 0, DRAIN_LIMIT_NS, nullptr);
    }
  } else if (warp < QW_EP0) {
    // ------------------------------------------------- dequantisation --
    // Thread = vocab row rin of the unit (TMEM lane rin); warps 2-5 take the
    // first half of each group (packed words 0-3 at 4 bits, 0-7 at 8), warps
    // 6-9 the second, into 16 columns each of the A slot.
    const int q4 = warp & 3, hg = (warp - QW_DQ0) >> 2;
    const int rin = q4 * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
    const int gpr = a.D / 64, n8 = gpr / 8;
    uint32_t n = 0;
    bool ok = true;
    for (int blk = blockIdx.x; blk < a.n_blk && ok; blk += gridDim.x) {
      const int k0 = blk % nk;
      const int g8 = k0 >> 3, g8n = g8 + 1 < n8 ? g8 + 1 : 0;
      for (int h = 0; h < 2 && ok; ++h) {
        const int v = blk * QS_BLK + h * QW_UNIT + rin;
        const bool valid = v < a.V;
        const uint4* srow =
            reinterpret_cast<const uint4*>(a.q_scale + static_cast<size_t>(v) * gpr);
        const uint4* brow = reinterpret_cast<const uint4*>(a.q_bias + static_cast<size_t>(v) * gpr);
        uint4 sc = make_uint4(0, 0, 0, 0), bi = sc, sc_n = sc, bi_n = sc;
        if (valid) {
          sc = __ldg(srow + g8);
          bi = __ldg(brow + g8);
          sc_n = __ldg(srow + g8n);
          bi_n = __ldg(brow + g8n);
        }
        for (int i = 0; i < nk; ++i, ++n) {
          const int k = k0 + i < nk ? k0 + i : k0 + i - nk;
          if ((k & 7) == 0 && i > 0) {
            sc = sc_n;
            bi = bi_n;
            const int nx = (k >> 3) + 1 < n8 ? (k >> 3) + 1 : 0;
            if (valid) {
              sc_n = __ldg(srow + nx);
              bi_n = __ldg(brow + nx);
            }
          }
          int s, sa;
          uint32_t ph, aph;
          step_of(n, s, ph, sa, aph);
          if (!__all_sync(0xffffffffu, wait_bounded(&full[s], ph, a.wait_ns, abort_flag))) {
            ok = false;
            break;
          }
          const uint8_t* sP = base + s * F::STAGE + rin * (QB * 8) + hg * (QB * 4);
          uint4 w0 = *reinterpret_cast<const uint4*>(sP), w1 = w0;
          if constexpr (QB == 8) w1 = *reinterpret_cast<const uint4*>(sP + 16);
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[s]);
          const int g = k & 7;
          const uint32_t ws = (g >> 1) == 0 ? sc.x : (g >> 1) == 1 ? sc.y : (g >> 1) == 2 ? sc.z : sc.w;
          const uint32_t wb = (g >> 1) == 0 ? bi.x : (g >> 1) == 1 ? bi.y : (g >> 1) == 2 ? bi.z : bi.w;
          const uint16_t sbits = static_cast<uint16_t>((g & 1) ? ws >> 16 : ws & 0xFFFFu);
          const uint16_t bbits = static_cast<uint16_t>((g & 1) ? wb >> 16 : wb & 0xFFFFu);
          uint4 out[4];
          if (valid) {
            if constexpr (QB == 8)
              qw_dequant_half_q8(w0, w1, sbits, bbits, out);
            else
              qw_dequant_half_q4(w0, sbits, bbits, out);
          } else {
#pragma unroll
            for (int c = 0; c < 4; ++c) out[c] = make_uint4(0, 0, 0, 0);
          }
          uint32_t r[16];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            r[4 * c] = out[c].x;
            r[4 * c + 1] = out[c].y;
            r[4 * c + 2] = out[c].z;
            r[4 * c + 3] = out[c].w;
          }
          if (!__all_sync(0xffffffffu,
                          wait_bounded(&aempty[sa], aph ^ 1u, a.wait_ns, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          tmem_st16(tmem_base + lane_addr + static_cast<uint32_t>(sa * 32 + hg * 16), r);
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&afull[sa]);
        }
      }
    }
    if (!ok) fail();
  } else if (warp < QW_EP0 + 4) {
    // --------------------------------------------------------- epilogue --
    // As in the narrower kernel (qsmall_fwd.cuh): per 32-column chunk the
    // column maxima across the warp's 32 vocab rows, their broadcast, the
    // exponentials and their sums; each warp's (max, sum) per head row runs
    // over the block's two units, and the four warps' pairs are merged per
    // head row behind an mbarrier at the end of the block.
    const int e = warp - QW_EP0;
    const int q4 = warp & 3;
    const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
    const int nch = (a.Mp + 31) / 32;
    float* bcw = bc + e * 32;
    int ylab[QW_MAXC];
#pragma unroll
    for (int c = 0; c < QW_MAXC; ++c) {
      const int m = 32 * c + lane;
      ylab[c] = m < a.M ? a.labels[m] : -1;
    }
    uint32_t un = 0, bn = 0;
    bool ok = true;
    for (int blk = blockIdx.x; blk < a.n_blk && ok; blk += gridDim.x, ++bn) {
      float mw[QW_MAXC], sw[QW_MAXC];
#pragma unroll
      for (int c = 0; c < QW_MAXC; ++c) {
        mw[c] = -INFINITY;
        sw[c] = 0.f;
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (!__all_sync(0xffffffffu, wait_bounded(accfull, un & 1u, a.wait_ns, abort_flag))) {
          ok = false;
          break;
        }
        ++un;
        tc_fence_after();
        const int vq0 = blk * QS_BLK + h * QW_UNIT + q4 * 32;  // vocab row of lane 0
        const bool rvalid = vq0 + lane < a.V;
#pragma unroll
        for (int c = 0; c < QW_MAXC; ++c) {
          if (c >= nch) break;
          uint32_t r[32];
          tmem_ld32(tmem_base + lane_addr + static_cast<uint32_t>(QW_ACC0 + c * 32), r);
          tmem_ld_wait(r);
          float x[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) x[j] = u2f(r[j]);
          if (a.softcap > 0.f) {
#pragma unroll
            for (int j = 0; j < 32; ++j) x[j] = a.softcap * tanh_ex2(x[j] * a.inv_cap);
          }
          if (!rvalid) {
#pragma unroll
            for (int j = 0; j < 32; ++j) x[j] = -INFINITY;
          }
          const int rel = ylab[c] - vq0;
          unsigned hits = __ballot_sync(0xffffffffu, static_cast<unsigned>(rel) < 32u);
          while (hits != 0u) {
            const int j = __ffs(hits) - 1;
            hits &= hits - 1u;
            const int rr = __shfl_sync(0xffffffffu, rel, j);
            if (lane == rr) {
              float val = 0.f;
#pragma unroll
              for (int jj = 0; jj < 32; ++jj)
                if (jj == j) val = x[jj];
              a.tgt[32 * c + j] = val;
            }
          }
          float t[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) t[j] = x[j];
          const float cm = qs_reduce_scatter(t, lane, QsMax());
          __syncwarp();
          bcw[lane] = cm == -INFINITY ? 0.f : -cm * LOG2E;
          __syncwarp();
#pragma unroll
          for (int j4 = 0; j4 < 8; ++j4) {
            const float4 nb = reinterpret_cast<const float4*>(bcw)[j4];
            t[4 * j4] = ex2_approx(fmaf(x[4 * j4], LOG2E, nb.x));
            t[4 * j4 + 1] = ex2_approx(fmaf(x[4 * j4 + 1], LOG2E, nb.y));
            t[4 * j4 + 2] = ex2_approx(fmaf(x[4 * j4 + 2], LOG2E, nb.z));
            t[4 * j4 + 3] = ex2_approx(fmaf(x[4 * j4 + 3], LOG2E, nb.w));
          }
          const float cs = qs_reduce_scatter(t, lane, QsAdd());
          if (h == 0) {
            mw[c] = cm;
            sw[c] = cs;
          } else {
            qs_combine(mw[c], sw[c], cm, cs);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(accempty);
      }
      if (!ok) break;
      const int par = static_cast<int>(bn & 1u);
      float* rm = red + (par * 2 + 0) * 4 * QW_MAXM;
      float* rs = red + (par * 2 + 1) * 4 * QW_MAXM;
#pragma unroll
      for (int c = 0; c < QW_MAXC; ++c)
        if (c < nch) {
          rm[e * QW_MAXM + 32 * c + lane] = mw[c];
          rs[e * QW_MAXM + 32 * c + lane] = sw[c];
        }
      __syncwarp();
      if (lane == 0) mbar_arrive(&epibar[par]);
      if (!__all_sync(0xffffffffu,
                      wait_bounded(&epibar[par], (bn >> 1) & 1u, a.wait_ns, abort_flag))) {
        ok = false;
        break;
      }
      // head rows e*32 + lane + 128 i, i = 0, 1 (up to 256 rows over 128 threads)
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int m = e * 32 + lane + 128 * i;
        if (m < a.M) {
          float M0 = -INFINITY, S0 = 0.f;
#pragma unroll
          for (int qq = 0; qq < 4; ++qq)
            qs_combine(M0, S0, rm[qq * QW_MAXM + m], rs[qq * QW_MAXM + m]);
          const size_t o = static_cast<size_t>(blk) * a.M + m;
          a.part_m[o] = M0;
          a.part_s[o] = S0;
        }
      }
    }
    if (!ok) fail();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, QS_TMEM_COLS);
  }
}

}  // namespace cce
