// qsmall_fwd.cuh — the forward of a 4/8-bit head at small M (at most 128
// head rows): the logits computed transposed, S^T[v, m] = W_t[v, :] . H[m, :],
// with the dequantised head tile as the tensor cores' A operand in TMEM.
//
// What it computes is the forward of the flash-CCE head (ORPO design 0.0.6,
// fused-head implementation spec, "Forward": online softmax over the vocab
// tiles, the target logit captured on the way; Training design §5.6,
// quantised base: w = q * scale + bias per group of 64 along D), producing
// the same per-(256-vocab block, row) partials (max, sum of exp) and target
// logits as the GEMM forward, for merge_lse_kernel.
//
// Why transposed.  With few head rows the head itself is the stream: every
// weight is dequantised once, and the MMA's N dimension is the head rows.
// In the GEMM kernel (gemm_tc.cuh) the dequantisation warps write the fp16
// head tile into shared memory (the B operand), fence the async proxy and
// signal the MMA; those stores, the fence and the warps' arithmetic measured
// as the bound (0.27 ms for the 4-bit long-context head at M = 64, 0.16 of
// the HBM rate on its packed bytes).  Here the head tile is the A operand,
// which tcgen05.mma can read from TMEM: each dequantisation thread owns one
// vocab row (one TMEM lane), converts its 64 weights of a group and writes
// them with one tcgen05.st (32 columns, two fp16 per column, K pairs in the
// order the converter produces them; H is permuted to match, as for the
// GEMM kernel).  H, the small operand, comes by TMA into shared memory.
//
// Per CTA: 256-row vocab blocks in turn (block b, then b + grid, ...), each
// as two 128-row halves that share every K step's H slices; the K loop runs
// over D in steps of KG groups of 64 (QsCfg), starting for block b at step
// b mod (D / (64 KG)) and wrapping.  Every CTA reads the same small H, so with one K order for all
// the SMs would fetch the same H slice from L2 at the same moment and a few
// L2 slices would serve the whole GPU; rotated, they spread over all of H.
// Roles (480 threads): warp 0 loads by TMA the packed rows of every K step
// (256 rows of KG groups) and the matching 64-column slices of H; warps 1
// and 14 issue the MMAs, one 128-row half each (4 per group: K = 16 each); warps
// 2-9 dequantise, one vocab row per thread, into a ring of TMEM A slots;
// warps 10-13 drain the accumulators (one vocab row per thread), reduce
// each head row's maximum and sum of exponentials over the block's 256
// vocab rows and write the block's partials.
//
// TMEM (512 columns): A ring of NA slots x (2 halves x KG groups x 32
// columns); from column 256 the accumulators, 2 halves x Mp columns, two
// buffers when Mp <= 64.  Shared-memory traffic per group: packed 8 KB
// (4-bit) written by TMA and read once by the dequantisers, the H slice (Mp
// x 128 bytes) written once and read by 8 MMAs; no operand stores by
// threads.  Two groups per K step (4-bit heads) halve the hand-offs between the roles
// (waits, commits, stores), which bound the one-group form.
//
// All waits are bounded; a timeout sets the status word.
#pragma once

#include "ptx.cuh"
#include "gemm_tc.cuh"

namespace cce {

constexpr int QS_BLK = 256;          // vocab rows per block (two MMA halves)
constexpr int QS_MAXM = 128;         // head rows at most
constexpr int QS_ACC0 = 256;         // first accumulator column (the A ring below it)
constexpr uint32_t QS_TMEM_COLS = 512;
constexpr int QS_DQ0 = 2;            // first dequantisation warp (8 of them)
constexpr int QS_EP0 = 10;           // first epilogue warp (4 of them)
constexpr int QS_ISS1 = 14;          // the second MMA issuer (half 1; warp 1 issues half 0)
constexpr int QS_THREADS = 15 * 32;
constexpr int QS_MAXC = QS_MAXM / 32;  // 32-column chunks of the accumulator

// KG groups of 64 weights per K step: 2 for 4-bit heads (half the
// hand-offs between the roles per weight; 15 % faster at N = 64), 1 for
// 8-bit heads, where two groups measured 10-15 % slower: with 3 stages of
// 64 KB, and also with 4 of 48 KB when the H slots were sized for N <= 64
// (which left 4-bit heads unchanged with 6 stages instead of 4).
// Stage: packed [256 rows x KG*QB*8 bytes], then per group H [Mp rows x
// 64 fp16] with the 128-byte swizzle (1024-aligned, HG bytes apart).  TMEM
// A ring below column 256: NA slots of 2 halves x KG groups x 32 columns.
template <int QB>
struct QsCfg {
  static constexpr int KG = QB == 4 ? 2 : 1;
  static constexpr int SLOT = 2 * KG * 32;
  static constexpr int NA = QS_ACC0 / SLOT;
  static constexpr int PK = QS_BLK * QB * 8 * KG;
  static constexpr int HG = QS_MAXM * 128;
  static constexpr int HB = KG * HG;
  static constexpr int STAGE = PK + HB;
  static constexpr int NST = QB == 4 ? 4 : 6;
  static constexpr int RED = 2 * 2 * 4 * QS_MAXM * 4;  // [parity][m|s][quarter][row]
  static constexpr int BC = 4 * 32 * 4;                // per epilogue warp broadcast row
  static constexpr int BARS = 512;
  static constexpr int SMEM = NST * STAGE + RED + BC + BARS + 1024;
};
static_assert(QsCfg<4>::PK % 1024 == 0 && QsCfg<8>::PK % 1024 == 0, "H box alignment");
static_assert(QsCfg<4>::SMEM <= 232448 && QsCfg<8>::SMEM <= 232448,
              "small-M forward exceeds the shared memory of a CTA");

struct QsArgs {
  int M, Mp;       // head rows; rounded up to a multiple of 16 (the MMA's N)
  int V, D;
  int nk;          // K steps over D (QsCfg<QB>::KG groups of 64 each in qsmall_fwd.cuh,
                   // one in qwide_fwd.cuh)
  int n_blk;       // 256-row vocab blocks
  int nacc;        // accumulator buffers (2 when Mp <= 64)
  uint64_t wait_ns;
  uint32_t* status;
  const int32_t* labels;
  const uint16_t* q_scale;  // bf16 [V, D/64], 16-byte aligned rows (D % 512 == 0)
  const uint16_t* q_bias;
  float softcap, inv_cap;
  float* part_m;   // [n_blk, M]
  float* part_s;
  float* tgt;      // [M]
};

// tcgen05.mma with A read from TMEM (kind::f16, single CTA).
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns from registers into TMEM: thread
// i of the warp writes row (lane base + i), columns [col, col + 32).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Lane i of the warp ends with op over the 32 lanes of column i of v (each
// lane's v[j] is its value in column j): five exchange rounds, each halving
// the columns a lane keeps (31 shuffles in all, instead of 32 x 5).  v is
// overwritten.
template <class Op>
__device__ __forceinline__ float qs_reduce_scatter(float (&v)[32], int lane, Op op) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool up = (lane & s) != 0;
#pragma unroll
    for (int j = 0; j < s; ++j) {
      const float send = up ? v[j] : v[j + s];
      const float keep = up ? v[j + s] : v[j];
      v[j] = op(keep, __shfl_xor_sync(0xffffffffu, send, s));
    }
  }
  return v[0];
}

struct QsMax {
  __device__ __forceinline__ float operator()(float a, float b) const { return fmaxf(a, b); }
};
struct QsAdd {
  __device__ __forceinline__ float operator()(float a, float b) const { return a + b; }
};

// (m, s) of exp-sums: the pair for the union of two sets, each given as its
// maximum and its sum of exp(x - maximum); an empty set is (-inf, 0).
__device__ __forceinline__ void qs_combine(float& m, float& s, float m2, float s2) {
  const float mn = fmaxf(m, m2);
  if (mn == -INFINITY) return;
  s = s * ex2_approx((m - mn) * LOG2E) + s2 * ex2_approx((m2 - mn) * LOG2E);
  m = mn;
}

// Status of a block's K step n (a global counter shared by every role):
// stage, stage parity, A slot, A slot parity.
struct QsStep {
  int s, a;
  uint32_t ph, aph;
};
template <int NST, int NA>
__device__ __forceinline__ QsStep qs_step(uint32_t n) {
  QsStep r;
  r.s = static_cast<int>(n % NST);
  r.ph = (n / NST) & 1u;
  r.a = static_cast<int>(n % NA);
  r.aph = (n / NA) & 1u;
  return r;
}

template <int QB>
__global__ void __launch_bounds__(QS_THREADS, 1)
    qsmall_fwd_kernel(const __grid_constant__ CUtensorMap tmP,  // packed bytes, box {QB*8, 256}
                      const __grid_constant__ CUtensorMap tmH,  // fp16 H, box {64, Mp}, SW128
                      const QsArgs a) {
  using F = QsCfg<QB>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  float* red = reinterpret_cast<float*>(base + F::NST * F::STAGE);  // [2][2][4][QS_MAXM]
  float* bc = red + F::RED / 4;                                     // [4][32]
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(bc) + F::BC);
  uint64_t* full = bars;                   // [NST] stage landed (TMA bytes)
  uint64_t* empty = full + F::NST;         // [NST] 8 dequant warps read + MMAs done
  uint64_t* afull = empty + F::NST;        // [NA] 8 dequant warps stored
  uint64_t* aempty = afull + F::NA;        // [NA] MMAs read
  uint64_t* accfull = aempty + F::NA;      // [2]
  uint64_t* accempty = accfull + 2;        // [2] 4 epilogue warps drained
  uint64_t* drain = accempty + 2;          // [2] one per MMA issuer
  uint64_t* epibar = drain + 2;            // [2] 4 epilogue warps wrote their pairs
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(epibar + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < F::NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 10);
    }
    for (int s = 0; s < F::NA; ++s) {
      mbar_init(&afull[s], 8);
      mbar_init(&aempty[s], 2);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 2);
      mbar_init(&accempty[b], 4);
      mbar_init(&epibar[b], 4);
    }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
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

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      const uint32_t hbytes = static_cast<uint32_t>(a.Mp) * 128u;
      uint32_t n = 0;
      bool ok = true;
      for (int blk = blockIdx.x; blk < a.n_blk && ok; blk += gridDim.x) {
        const int k0 = blk % nk;
        for (int i = 0; i < nk; ++i, ++n) {
          const int k = k0 + i < nk ? k0 + i : k0 + i - nk;
          const QsStep q = qs_step<F::NST, F::NA>(n);
          if (!wait_bounded(&empty[q.s], q.ph ^ 1u, a.wait_ns, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* st = base + q.s * F::STAGE;
          mbar_arrive_expect_tx(&full[q.s], static_cast<uint32_t>(F::PK) + F::KG * hbytes);
          tma_load_2d(st, &tmP, &full[q.s], k * F::KG * QB * 8, blk * QS_BLK);
#pragma unroll
          for (int g = 0; g < F::KG; ++g)
            tma_load_2d(st + F::PK + g * F::HG, &tmH, &full[q.s], (k * F::KG + g) * 64, 0);
        }
      }
      if (!ok) fail();
      // Every copy issued lands before the CTA can exit: the last NST
      // steps' stages (earlier ones were consumed, hence landed).
      const uint32_t n0 = n > static_cast<uint32_t>(F::NST) ? n - F::NST : 0u;
      for (uint32_t i = n0; i < n; ++i) {
        const QsStep q = qs_step<F::NST, F::NA>(i);
        wait_bounded(&full[q.s], q.ph, DRAIN_LIMIT_NS, nullptr);
      }
    }
  } else if (warp == 1 || warp == QS_ISS1) {
    // ------------------------------------------------------ MMA issuers --
    // One thread per 128-row half: a single thread's tcgen05.mma issue
    // measured about 100 cycles per 128 x 64 x 16 MMA with the tensor pipe
    // mostly idle, and two issuers each take half of the MMAs.  Every
    // barrier the MMAs release counts one commit from each.
    if (lane == 0) {
      const int h = warp == 1 ? 0 : 1;
      const uint32_t idesc = idesc_f16(128, a.Mp, 0, false, false);
      uint32_t n = 0, accn = 0;
      bool ok = true;
      for (int blk = blockIdx.x; blk < a.n_blk && ok; blk += gridDim.x, ++accn) {
        const int buf = a.nacc == 2 ? static_cast<int>(accn & 1u) : 0;
        const uint32_t use = a.nacc == 2 ? accn >> 1 : accn;
        if (!wait_bounded(&accempty[buf], (use & 1u) ^ 1u, a.wait_ns, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dcol = tmem_base + QS_ACC0 + static_cast<uint32_t>(buf * 2 * a.Mp);
        for (int i = 0; i < nk; ++i, ++n) {
          const QsStep q = qs_step<F::NST, F::NA>(n);
          if (!wait_bounded(&full[q.s], q.ph, a.wait_ns, abort_flag) ||
              !wait_bounded(&afull[q.a], q.aph, a.wait_ns, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sH = smem_u32(base + q.s * F::STAGE + F::PK);
#pragma unroll
          for (int g = 0; g < F::KG; ++g)
#pragma unroll
            for (int j = 0; j < 4; ++j)
              umma_f16_ts(dcol + static_cast<uint32_t>(h * a.Mp),
                          tmem_base + static_cast<uint32_t>(q.a * F::SLOT + h * F::KG * 32 +
                                                            g * 32 + j * 8),
                          sdesc_sw128(sH + g * F::HG + j * 32, 16, 1024), idesc,
                          (i | g | j) != 0 ? 1u : 0u);
          umma_commit(&empty[q.s]);
          umma_commit(&aempty[q.a]);
        }
        if (!ok) break;
        umma_commit(&accfull[buf]);
      }
      if (!ok) fail();
      // Every MMA issued completes before TMEM is released.
      umma_commit(&drain[h]);
      wait_bounded(&drain[h], 0, DRAIN_LIMIT_NS, nullptr);
    }
  } else if (warp < QS_EP0) {
    // ------------------------------------------------- dequantisation --
    // Thread = vocab row rin of the block (TMEM lane rin % 128 of half
    // rin / 128).  Per K step: the row's packed words of KG groups from
    // the stage, their scales and biases (8 groups per 16-byte load, the
    // next 8 fetched while these are used), 64 fp16 weights per group into
    // the A slot (one tcgen05.st each).
    const int q4 = warp & 3, h = (warp - QS_DQ0) >> 2;
    const int rin = h * 128 + q4 * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
    constexpr int NV = QB * 8 / 16;  // 16-byte words of packed data per row and group
    const int gpr = a.D / 64;
    uint32_t n = 0;
    bool ok = true;
    for (int blk = blockIdx.x; blk < a.n_blk && ok; blk += gridDim.x) {
      const int v = blk * QS_BLK + rin;
      const bool valid = v < a.V;
      const uint4* srow = reinterpret_cast<const uint4*>(a.q_scale + static_cast<size_t>(v) * gpr);
      const uint4* brow = reinterpret_cast<const uint4*>(a.q_bias + static_cast<size_t>(v) * gpr);
      // the K loop starts at step k0 and wraps (as the producer's); group
      // gi = k * KG + g of step k; scales and biases 8 groups per load,
      // the next 8 fetched while these are used
      const int k0 = blk % nk, n8 = gpr / 8;
      const int g8 = (k0 * F::KG) >> 3, g8n = g8 + 1 < n8 ? g8 + 1 : 0;
      uint4 sc = make_uint4(0, 0, 0, 0), bi = sc, sc_n = sc, bi_n = sc;
      if (valid) {
        sc = __ldg(srow + g8);
        bi = __ldg(brow + g8);
        sc_n = __ldg(srow + g8n);
        bi_n = __ldg(brow + g8n);
      }
      for (int i = 0; i < nk; ++i, ++n) {
        const int k = k0 + i < nk ? k0 + i : k0 + i - nk;
        const QsStep q = qs_step<F::NST, F::NA>(n);
        if (!__all_sync(0xffffffffu, wait_bounded(&full[q.s], q.ph, a.wait_ns, abort_flag))) {
          ok = false;
          break;
        }
        uint4 w[F::KG][NV];
        const uint8_t* sP = base + q.s * F::STAGE + rin * (F::KG * QB * 8);
#pragma unroll
        for (int g = 0; g < F::KG; ++g)
#pragma unroll
          for (int t = 0; t < NV; ++t)
            w[g][t] = *reinterpret_cast<const uint4*>(sP + g * (QB * 8) + 16 * t);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[q.s]);
#pragma unroll
        for (int g = 0; g < F::KG; ++g) {
          const int gi = k * F::KG + g;
          if ((gi & 7) == 0 && (i | g) != 0) {
            sc = sc_n;
            bi = bi_n;
            const int nx = (gi >> 3) + 1 < n8 ? (gi >> 3) + 1 : 0;
            if (valid) {
              sc_n = __ldg(srow + nx);
              bi_n = __ldg(brow + nx);
            }
          }
          const int gg = gi & 7;
          const uint32_t ws = (gg >> 1) == 0 ? sc.x : (gg >> 1) == 1 ? sc.y : (gg >> 1) == 2 ? sc.z : sc.w;
          const uint32_t wb = (gg >> 1) == 0 ? bi.x : (gg >> 1) == 1 ? bi.y : (gg >> 1) == 2 ? bi.z : bi.w;
          const uint16_t sbits = static_cast<uint16_t>((gg & 1) ? ws >> 16 : ws & 0xFFFFu);
          const uint16_t bbits = static_cast<uint16_t>((gg & 1) ? wb >> 16 : wb & 0xFFFFu);
          uint4 out[8];
          if (valid) {
            if constexpr (QB == 8)
              dequant_group64_q8(*reinterpret_cast<const uint4(*)[4]>(w[g]), sbits, bbits, out);
            else
              dequant_group64(w[g][0], w[g][NV - 1], sbits, bbits, out);
          } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) out[c] = make_uint4(0, 0, 0, 0);
          }
          uint32_t r[32];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            r[4 * c] = out[c].x;
            r[4 * c + 1] = out[c].y;
            r[4 * c + 2] = out[c].z;
            r[4 * c + 3] = out[c].w;
          }
          if (g == 0) {
            if (!__all_sync(0xffffffffu,
                            wait_bounded(&aempty[q.a], q.aph ^ 1u, a.wait_ns, abort_flag))) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
          tmem_st32(tmem_base + lane_addr +
                        static_cast<uint32_t>(q.a * F::SLOT + h * F::KG * 32 + g * 32),
                    r);
        }
        if (!ok) break;
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&afull[q.a]);
      }
    }
    if (!ok) fail();
  } else if (warp < QS_EP0 + 4) {
    // --------------------------------------------------------- epilogue --
    // Thread = vocab row (lane quarter q4 of each half); a 32-column chunk
    // of the accumulator holds 32 head rows.  Per chunk the warp reduces,
    // for each head row, the maximum over its 32 vocab rows (lane i ends
    // with column i), broadcasts it, sums the exponentials and reduces them
    // the same way; the warp's (max, sum) per head row runs over the
    // block's two halves, and the four warps' pairs are merged in shared
    // memory at the end of the block.  The target logit of head row m is
    // taken by the thread whose vocab row is labels[m].
    const int e = warp - QS_EP0;
    const int q4 = warp & 3;
    const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
    const int nch = (a.Mp + 31) / 32;
    float* bcw = bc + e * 32;
    int ylab[QS_MAXC];
#pragma unroll
    for (int c = 0; c < QS_MAXC; ++c) {
      const int m = 32 * c + lane;
      ylab[c] = m < a.M ? a.labels[m] : -1;
    }
    uint32_t accn = 0;
    bool ok = true;
    for (int blk = blockIdx.x; blk < a.n_blk; blk += gridDim.x, ++accn) {
      const int buf = a.nacc == 2 ? static_cast<int>(accn & 1u) : 0;
      const uint32_t use = a.nacc == 2 ? accn >> 1 : accn;
      if (!__all_sync(0xffffffffu, wait_bounded(&accfull[buf], use & 1u, a.wait_ns, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float mw[QS_MAXC], sw[QS_MAXC];
#pragma unroll
      for (int c = 0; c < QS_MAXC; ++c) {
        mw[c] = -INFINITY;
        sw[c] = 0.f;
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int vq0 = blk * QS_BLK + h * 128 + q4 * 32;  // vocab row of lane 0
        const bool rvalid = vq0 + lane < a.V;
#pragma unroll
        for (int c = 0; c < QS_MAXC; ++c) {
          if (c >= nch) break;
          uint32_t r[32];
          tmem_ld32(tmem_base + lane_addr +
                        static_cast<uint32_t>(QS_ACC0 + buf * 2 * a.Mp + h * a.Mp + c * 32),
                    r);
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
          // target logits in this chunk's head rows and this warp's vocab rows
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
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[buf]);
      // the four warps' pairs, merged per head row (parity-buffered: a warp
      // two blocks ahead has passed the next block's barrier, which every
      // warp reaches only after its reads here; the barrier is an mbarrier
      // so that a timed-out warp cannot leave the others waiting)
      const int par = static_cast<int>(accn & 1u);
      float* rm = red + (par * 2 + 0) * 4 * QS_MAXM;
      float* rs = red + (par * 2 + 1) * 4 * QS_MAXM;
#pragma unroll
      for (int c = 0; c < QS_MAXC; ++c)
        if (c < nch) {
          rm[e * QS_MAXM + 32 * c + lane] = mw[c];
          rs[e * QS_MAXM + 32 * c + lane] = sw[c];
        }
      __syncwarp();
      if (lane == 0) mbar_arrive(&epibar[par]);
      if (!__all_sync(0xffffffffu,
                      wait_bounded(&epibar[par], (accn >> 1) & 1u, a.wait_ns, abort_flag))) {
        ok = false;
        break;
      }
      const int m = e * 32 + lane;
      if (m < a.M) {
        float M0 = -INFINITY, S0 = 0.f;
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) qs_combine(M0, S0, rm[qq * QS_MAXM + m], rs[qq * QS_MAXM + m]);
        const size_t o = static_cast<size_t>(blk) * a.M + m;
        a.part_m[o] = M0;
        a.part_s[o] = S0;
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
