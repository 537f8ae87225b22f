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
//
// Roles (192 threads): warp 0 issues TMA loads into a 4-stage shared-memory
// ring; warp 1 owns the TMEM allocation and issues tcgen05.mma (M=128,
// N=256, K=16) into one of two 256-column fp32 accumulators; warps 2-5 drain
// the accumulator with tcgen05.ld (warp w reads TMEM lanes 32*(w%4)..+31,
// i.e. one row per thread) and run the epilogue, overlapping the MMA of the
// next tile.  Tiles are assigned round-robin over a grid of at most one CTA
// per SM; consecutive tile ids share the column tile (vocab or d), so the CTAs
// in flight stream the same W tiles from L2.
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
constexpr int NUM_THREADS = 192;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
constexpr float LOG2E = 1.4426950408889634f;
constexpr uint64_t DRAIN_LIMIT_NS = 1000000000ull;

enum class Mode : int { kLse = 0, kGrad = 1, kDh = 2 };

struct TileArgs {
  int M;         // rows of A (head rows)
  int n_rt;      // row tiles
  int n_ct;      // column tiles of this launch
  int nk;        // K steps of BK per pass
  int npass;     // passes over K (kDh: hi/lo halves of a split f32 head)
  int b_pass_off;  // kDh: B inner-coordinate offset of pass 1
  int b_row0;    // kLse/kGrad: first vocab row of this launch; kDh: chunk v0
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
  float* dh;  // [M, D]
  int first_chunk;
};

__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }

// 0 = compute, 1 = write zeros only, 2 = nothing.
template <Mode MODE>
__device__ __forceinline__ int tile_kind(const TileArgs& a, int rt, int ct) {
  if (MODE == Mode::kLse) return 0;
  const bool rs = a.row_skip != nullptr && a.row_skip[rt] != 0;
  if (MODE == Mode::kGrad) {
    if (rs) return 2;
    if (a.tile_skip != nullptr && a.tile_skip[rt * a.skip_ld + a.ct_off + ct]) return 1;
    return 0;
  }
  if (rs) return a.first_chunk ? 1 : 2;
  return 0;
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi, int fmt) {
  if (fmt == 1) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Softmax probability of logit s given nl = -lse * log2(e).  The block-skip
// planner uses the same expression, so its decisions agree with the filter.
__device__ __forceinline__ float softmax_p(float s, float nl) {
  return ex2_approx(fmaf(s, LOG2E, nl));
}

template <Mode MODE>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    cce_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                  const __grid_constant__ CUtensorMap tmB, const TileArgs a) {
  extern __shared__ uint8_t dyn_smem[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(base + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int ntiles = a.n_rt * a.n_ct;
  const int ksteps = a.nk * a.npass;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4 * 32);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        const int rt = t % a.n_rt, ct = t / a.n_rt;
        if (tile_kind<MODE>(a, rt, ct) != 0) continue;
        for (int kk = 0; kk < ksteps; ++kk) {
          if (!wait_bounded(&empty[stage], phase ^ 1u, a.wait_ns, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* sA = base + stage * STAGE_BYTES;
          uint8_t* sB = sA + A_BYTES;
          mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
          const int pass = kk / a.nk, k = kk - pass * a.nk;
          tma_load_2d(sA, &tmA, &full[stage], k * BK, rt * BM);
          if (MODE == Mode::kDh) {
#pragma unroll
            for (int j = 0; j < BN / 64; ++j)
              tma_load_2d(sB + j * (64 * BK * 2), &tmB, &full[stage],
                          ct * BN + j * 64 + pass * a.b_pass_off,
                          a.b_row0 + k * BK);
          } else {
            tma_load_2d(sB, &tmB, &full[stage], k * BK, a.b_row0 + ct * BN);
          }
          issued_mask |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        set_status(a.status, ST_TIMEOUT);
        *abort_flag = 1;
      }
      // Let every issued copy land before the CTA can exit.
      for (int s = 0; s < STAGES; ++s)
        if (issued_mask & (1u << s))
          wait_bounded(&full[s], (issued_phase >> s) & 1u, DRAIN_LIMIT_NS,
                       nullptr);
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      const uint32_t idesc =
          idesc_f16(BM, BN, a.fmt, false, MODE == Mode::kDh);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        const int rt = t % a.n_rt, ct = t / a.n_rt;
        if (tile_kind<MODE>(a, rt, ct) != 0) continue;
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
          const uint32_t sA = smem_u32(base + stage * STAGE_BYTES);
          const uint32_t sB = sA + A_BYTES;
#pragma unroll
          for (int j = 0; j < BK / 16; ++j) {
            const uint64_t ad = sdesc_sw128(sA + j * 32, 16, 1024);
            const uint64_t bd =
                MODE == Mode::kDh
                    ? sdesc_sw128(sB + j * 16 * 128, 64 * BK * 2, 1024)
                    : sdesc_sw128(sB + j * 32, 16, 1024);
            umma_f16_ss(d_tmem, ad, bd, idesc, (kk | j) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&acc_full[b]);
        ++acc;
      }
      if (!ok) {
        set_status(a.status, ST_TIMEOUT);
        *abort_flag = 1;
      }
      // All MMAs issued by this thread complete before TMEM is released.
      umma_commit(drain);
      wait_bounded(drain, 0, DRAIN_LIMIT_NS, nullptr);
    }
  } else {
    // ---------------------------------------------------------- epilogue --
    const int quad = warp & 3;
    const int rin = quad * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    int acc = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
      const int rt = t % a.n_rt, ct = t / a.n_rt;
      const int kind = tile_kind<MODE>(a, rt, ct);
      const int row = rt * BM + rin;
      const bool live = row < a.M;
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
              *reinterpret_cast<float4*>(a.dh + static_cast<size_t>(row) * a.D + d0) =
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
        float m_run = -INFINITY, s_run = 0.f, tval = 0.f;
        bool found = false;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          const int v0 = vbase + c * 32;
          const int nvalid = min(32, a.V - v0);
          if (nvalid <= 0) break;
          __syncwarp();
          uint32_t r[32];
          tmem_ld32(taddr + c * 32, r);
          tmem_ld_wait();
          float cm = -INFINITY;
          if (nvalid == 32) {
#pragma unroll
            for (int j = 0; j < 32; ++j) cm = fmaxf(cm, u2f(r[j]));
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < nvalid) cm = fmaxf(cm, u2f(r[j]));
          }
          const float mn = fmaxf(m_run, cm);
          const float nb = -mn * LOG2E;
          float s0 = 0.f, s1 = 0.f;
          if (nvalid == 32) {
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              s0 += ex2_approx(fmaf(u2f(r[j]), LOG2E, nb));
              s1 += ex2_approx(fmaf(u2f(r[j + 1]), LOG2E, nb));
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < nvalid) s0 += ex2_approx(fmaf(u2f(r[j]), LOG2E, nb));
          }
          s_run = s_run * ex2_approx((m_run - mn) * LOG2E) + (s0 + s1);
          m_run = mn;
          const int tt = y - v0;
          const bool hit = static_cast<unsigned>(tt) < static_cast<unsigned>(nvalid);
          if (__any_sync(0xffffffffu, hit)) {
            if (hit) {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (j == tt) tval = u2f(r[j]);
              found = true;
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&acc_empty[b]);
        if (live) {
          const size_t o = static_cast<size_t>(a.ct_off + ct) * a.M + row;
          a.part_m[o] = m_run;
          a.part_s[o] = s_run;
          if (found) a.tgt[row] = tval;
        }
      } else if (MODE == Mode::kGrad) {
        const int y = live ? a.labels[row] : -1;
        const float nl = live ? -a.lse[row] * LOG2E : 0.f;
        const float eps = a.filter_eps;
        const int vbase = a.b_row0 + ct * BN;
        uint16_t* gdst = a.g_out + static_cast<size_t>(live ? row : 0) * a.g_ld + ct * BN;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          const int v0 = vbase + c * 32;
          __syncwarp();
          uint32_t r[32];
          tmem_ld32(taddr + c * 32, r);
          tmem_ld_wait();
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            float g2[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int v = v0 + j + h;
              float p = softmax_p(u2f(r[j + h]), nl);
              const bool tgt = (v == y);
              if (p < eps && !tgt) p = 0.f;
              g2[h] = v < a.V ? (tgt ? 1.f - p : -p) : 0.f;
            }
            pk[j >> 1] = pack2(g2[0], g2[1], a.fmt);
          }
          if (live) {
            uint4* dst = reinterpret_cast<uint4*>(gdst + c * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          }
        }
        tc_fence_before();
        mbar_arrive(&acc_empty[b]);
      } else {  // kDh
        const float g = live ? a.coeff[row] : 0.f;
        const int dbase = ct * BN;
        float* drow = a.dh + static_cast<size_t>(live ? row : 0) * a.D;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          const int d0 = dbase + c * 32;
          if (d0 >= a.D) break;
          __syncwarp();
          uint32_t r[32];
          tmem_ld32(taddr + c * 32, r);
          tmem_ld_wait();
          if (live) {
            float4* dst = reinterpret_cast<float4*>(drow + d0);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              float4 o;
              o.x = g == 0.f ? 0.f : g * u2f(r[4 * i + 0]);
              o.y = g == 0.f ? 0.f : g * u2f(r[4 * i + 1]);
              o.z = g == 0.f ? 0.f : g * u2f(r[4 * i + 2]);
              o.w = g == 0.f ? 0.f : g * u2f(r[4 * i + 3]);
              if (!a.first_chunk) {
                const float4 p = dst[i];
                o.x += p.x;
                o.y += p.y;
                o.z += p.z;
                o.w += p.w;
              }
              dst[i] = o;
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&acc_empty[b]);
      }
      ++acc;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace cce
