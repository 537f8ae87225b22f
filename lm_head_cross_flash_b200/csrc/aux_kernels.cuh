// aux_kernels.cuh — the small, bandwidth- or latency-bound steps of the head:
// the cross-block LSE merge, the ORPO epilogue (loss and cotangent), the
// block-skip planner, operand preparation, and the timeout self-test.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "gemm_tc.cuh"

namespace cce {

// ------------------------------------------------------------ LSE merge --
// lse[m] = max_b part_m[b,m] + log(sum_b part_s[b,m] exp(part_m[b,m] - max));
// logp[m] = tgt[m] - lse[m] for 0 <= y < V, else 0.  (Cross-block merge of
// the per-block partials; Training design §5.1, "Vocab-parallel grid":
// the merge is a cheap reduction of (blockMax, block sum-exp) partials.)
// One warp per row: lanes stride over the blocks, then a shuffle reduction.
__global__ void __launch_bounds__(256) merge_lse_kernel(
    const float* __restrict__ part_m, const float* __restrict__ part_s,
    int cols, int M, const int32_t* __restrict__ labels, int V,
    const float* __restrict__ tgt, float* __restrict__ logp,
    float* __restrict__ lse, uint32_t* status) {
  const int warps = blockDim.x >> 5;
  const int row = blockIdx.x * warps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  float m = -INFINITY, s = 0.f;
  for (int b = lane; b < cols; b += 32) {
    const float mb = part_m[static_cast<size_t>(b) * M + row];
    const float sb = part_s[static_cast<size_t>(b) * M + row];
    const float mn = fmaxf(m, mb);
    s = s * expf(m - mn) + sb * expf(mb - mn);
    m = mn;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float mo = __shfl_xor_sync(0xffffffffu, m, off);
    const float so = __shfl_xor_sync(0xffffffffu, s, off);
    const float mn = fmaxf(m, mo);
    const float a = (m == -INFINITY) ? 0.f : s * expf(m - mn);
    const float bb = (mo == -INFINITY) ? 0.f : so * expf(mo - mn);
    s = a + bb;
    m = mn;
  }
  if (lane == 0) {
    const float l = m + logf(s);
    lse[row] = l;
    const int y = labels[row];
    if (y >= V) set_status(status, ST_LABEL);
    logp[row] = (y >= 0 && y < V) ? tgt[row] - l : 0.f;
  }
}

// ------------------------------------------------------- ORPO epilogue --
struct OrpoArgs {
  int64_t pb, pe, cb, ce, rb, re;  // layout
  double lambda;
  int scope;                       // 0 full, 1 response
  int want_coeff;
  int kind;                        // 0 ORPO, 1 SimPO, 2 ORPO + SimPO margin
  double beta, gamma;              // SimPO scale and target margin
  // Row-sharded pairs: sums_out != null -> write the local segment sums
  // (sum and count of logp per segment) and stop; sums_in != null -> take
  // the segment sums from there (all-reduced over the shards) instead of
  // summing the local rows.
  const double* sums_in;
  double* sums_out;
};

// log(1 - e^x), x < 0: two-branch form (Maechler 2012), fp64.
__device__ __forceinline__ double log1mexp_d(double x) {
  return x > -0.6931471805599453 ? log(-expm1(x)) : log1p(-exp(x));
}

__device__ __forceinline__ double softplus_d(double x) {
  return fmax(x, 0.0) + log1p(exp(-fabs(x)));
}

// One block: fp64 segment sums (warp shuffles + shared memory), then thread 0
// forms lw, lr, pm, NLL, z, L_OR, L (Training design §1) and, in coefficient
// mode, every thread writes dL/dlogp for its rows.
__global__ void __launch_bounds__(1024) orpo_kernel(
    const float* __restrict__ logp, const int32_t* __restrict__ labels,
    int64_t M, OrpoArgs o, double* __restrict__ out8,
    float* __restrict__ coeff, uint32_t* status) {
  double s[3] = {0.0, 0.0, 0.0};
  double n[3] = {0.0, 0.0, 0.0};
  for (int64_t m = threadIdx.x; o.sums_in == nullptr && m < M; m += blockDim.x) {
    if (labels[m] < 0) continue;
    const double v = static_cast<double>(logp[m]);
    if (m >= o.pb && m < o.pe) { s[0] += v; n[0] += 1.0; }
    if (m >= o.cb && m < o.ce) { s[1] += v; n[1] += 1.0; }
    if (m >= o.rb && m < o.re) { s[2] += v; n[2] += 1.0; }
  }
#pragma unroll
  for (int i = 0; i < 3; ++i) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      s[i] += __shfl_xor_sync(0xffffffffu, s[i], off);
      n[i] += __shfl_xor_sync(0xffffffffu, n[i], off);
    }
  }
  __shared__ double red[32][6];
  __shared__ double sc[8];  // c_prompt, c_chosen, c_rejected, ok
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0)
    for (int i = 0; i < 3; ++i) { red[warp][i] = s[i]; red[warp][3 + i] = n[i]; }
  __syncthreads();
  if (threadIdx.x == 0) {
    double t[6] = {0, 0, 0, 0, 0, 0};
    const int nw = (blockDim.x + 31) >> 5;
    if (o.sums_in != nullptr) {
      for (int i = 0; i < 6; ++i) t[i] = o.sums_in[i];
    } else {
      for (int w = 0; w < nw; ++w)
        for (int i = 0; i < 6; ++i) t[i] += red[w][i];
    }
    if (o.sums_out != nullptr) {
      for (int i = 0; i < 6; ++i) o.sums_out[i] = t[i];
      return;
    }
    const double sP = t[0], sC = t[1], sR = t[2];
    const double nP = t[3], nC = t[4], nR = t[5];
    double res[8];
    const double qnan = __longlong_as_double(0x7ff8000000000000ll);
    double cP = 0.0, cC = 0.0, cR = 0.0;
    bool ok = true;
    if (nC == 0.0 || nR == 0.0) {
      set_status(status, ST_EMPTY);
      ok = false;
    }
    const double lw = ok ? sC / nC : qnan;
    const double lr = ok ? sR / nR : qnan;
    if (ok && o.kind == 0 && !(lw < 0.0 && lr < 0.0)) {
      set_status(status, ST_DOMAIN);
      ok = false;
    }
    if (ok && o.kind != 0) {
      // SimPO term softplus(-u), u = beta (lw - lr) - gamma; ORPO + margin
      // adds it, weighted by lambda, to the NLL term.
      const double pm = nP > 0.0 ? sP / nP : 0.0;
      const double nll = o.scope == 0 ? -(sP + sC) / (nP + nC) : -lw;
      const double u = o.beta * (lw - lr) - o.gamma;
      const double term = softplus_d(-u);
      const double sig = u >= 0.0 ? 1.0 / (1.0 + exp(-u)) : exp(u) / (1.0 + exp(u));
      const double w = o.kind == 1 ? 1.0 : o.lambda;
      res[0] = o.kind == 1 ? term : nll + o.lambda * term;
      res[1] = nll;
      res[2] = term;
      res[3] = lw;
      res[4] = lr;
      res[5] = pm;
      res[6] = u;
      res[7] = sig;
      const double d = w * (sig - 1.0) * o.beta;
      const double sNll = o.kind == 1 ? 0.0 : (o.scope == 0 ? -1.0 / (nP + nC) : -1.0 / nC);
      cP = (o.kind == 1 || o.scope == 1) ? 0.0 : sNll;
      cC = d / nC + sNll;
      cR = -d / nR;
    } else if (ok) {
      const double pm = nP > 0.0 ? sP / nP : 0.0;
      const double nll = o.scope == 0 ? -(sP + sC) / (nP + nC) : -lw;
      const double z = (lw - lr) - (log1mexp_d(lw) - log1mexp_d(lr));
      const double lor = softplus_d(-z);
      const double sig = z >= 0.0 ? 1.0 / (1.0 + exp(-z)) : exp(z) / (1.0 + exp(z));
      res[0] = nll + o.lambda * lor;
      res[1] = nll;
      res[2] = lor;
      res[3] = lw;
      res[4] = lr;
      res[5] = pm;
      res[6] = z;
      res[7] = sig;
      const double aw = 1.0 / (-expm1(lw));
      const double ar = 1.0 / (-expm1(lr));
      const double dz = sig - 1.0;
      const double sNll = o.scope == 0 ? -1.0 / (nP + nC) : -1.0 / nC;
      cP = o.scope == 0 ? sNll : 0.0;
      cC = o.lambda * dz * aw / nC + sNll;
      cR = -o.lambda * dz * ar / nR;
    } else {
      for (int i = 0; i < 8; ++i) res[i] = qnan;
    }
    if (out8 != nullptr)
      for (int i = 0; i < 8; ++i) out8[i] = res[i];
    sc[0] = cP;
    sc[1] = cC;
    sc[2] = cR;
  }
  if (!o.want_coeff || o.sums_out != nullptr) return;
  __syncthreads();
  const float cP = static_cast<float>(sc[0]);
  const float cC = static_cast<float>(sc[1]);
  const float cR = static_cast<float>(sc[2]);
  for (int64_t m = threadIdx.x; m < M; m += blockDim.x) {
    float c = 0.f;
    if (labels[m] >= 0) {
      if (m >= o.pb && m < o.pe) c = cP;
      else if (m >= o.cb && m < o.ce) c = cC;
      else if (m >= o.rb && m < o.re) c = cR;
    }
    coeff[m] = c;
  }
}

// ----------------------------------------------------- block-skip planner --
// tile_skip[rt, b] = 1 when, for every row m of row tile rt with coeff != 0,
// the block's largest softmax probability exp(blockmax[b,m] - lse[m]) is
// below eps and y_m is not in block b: every term of that tile would be
// dropped by the coefficient filter.  row_skip[rt] = 1 when every row of the
// tile has coeff == 0.  One warp per (rt, b).
__global__ void __launch_bounds__(256) skip_plan_kernel(
    const float* __restrict__ blockmax, const float* __restrict__ lse,
    const int32_t* __restrict__ labels, const float* __restrict__ coeff,
    int M, int cols, int n_rt, float eps, uint8_t* __restrict__ tile_skip,
    uint8_t* __restrict__ row_skip, unsigned long long* stats) {
  const int64_t unit = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (unit >= static_cast<int64_t>(n_rt) * cols) return;
  const int rt = static_cast<int>(unit / cols);
  const int b = static_cast<int>(unit - static_cast<int64_t>(rt) * cols);
  bool all_zero = true, skip = true;
  for (int i = lane; i < BM; i += 32) {
    const int m = rt * BM + i;
    if (m >= M) continue;
    const float c = coeff[m];
    if (c == 0.f) continue;
    all_zero = false;
    const int y = labels[m];
    if (y >= b * BN && y < (b + 1) * BN) skip = false;
    if (blockmax == nullptr) { skip = false; continue; }
    const float p = softmax_p(blockmax[static_cast<size_t>(b) * M + m], -lse[m] * LOG2E);
    if (!(p < eps)) skip = false;
  }
  all_zero = __all_sync(0xffffffffu, all_zero);
  skip = __all_sync(0xffffffffu, skip) && !all_zero;
  if (lane == 0) {
    tile_skip[unit] = skip ? 1 : 0;
    if (b == 0) row_skip[rt] = all_zero ? 1 : 0;
    if (stats != nullptr) {
      if (skip || all_zero) atomicAdd(&stats[0], 1ull);
      atomicAdd(&stats[1], 1ull);
    }
  }
}

// ------------------------------------------------------ operand preparation --
// Split an fp32 matrix [rows, D] into bf16 parts so that three bf16 products
// reproduce an fp32 product to ~2^-16: x = hi + lo, hi = bf16(x),
// lo = bf16(x - hi).  dst is [rows, 3*D]; `order` selects the part written to
// each third: 0 -> (hi, hi, lo) for the left operand, 1 -> (hi, lo, hi) for
// the right operand, so that the K-concatenated product is
// hi*hi + hi*lo + lo*hi.
__global__ void split_f32_kernel(const float* __restrict__ src, int64_t rows,
                                 int D, int order,
                                 __nv_bfloat16* __restrict__ dst) {
  const int64_t n = rows * D;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / D;
    const int d = static_cast<int>(i - r * D);
    const float x = src[i];
    const __nv_bfloat16 hi = __float2bfloat16_rn(x);
    const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
    __nv_bfloat16* o = dst + r * (3 * static_cast<int64_t>(D));
    o[d] = hi;
    o[D + d] = order == 0 ? hi : lo;
    o[2 * D + d] = order == 0 ? lo : hi;
  }
}

// fp16 copy of bf16 rows [rows, D] for a quantised head, with element e of
// every block of 8 columns stored at position qpos<QB>(e) (the order in which
// the dequantiser lays out the weights along K).  n8 = rows*D/8.
template <int QB>
__global__ void h_to_f16_perm_kernel(const uint4* __restrict__ src, int64_t n8,
                                     uint4* __restrict__ dst, uint32_t* status) {
  bool over = false;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 v = src[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    __half h[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint32_t bits = (w[e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
      const float x = __uint_as_float(bits << 16);
      // a finite bf16 value beyond the largest fp16 would become inf
      over = over || (fabsf(x) > 65504.f && fabsf(x) <= 3.4e38f);
      h[qpos<QB>(e)] = __float2half_rn(x);
    }
    dst[i] = *reinterpret_cast<const uint4*>(h);
  }
  if (__any_sync(0xffffffffu, over) && (threadIdx.x & 31) == 0) set_status(status, ST_FP16);
}

// Scales and biases of a 4/8-bit head feed fp16 arithmetic, which holds a
// bf16 value exactly only inside the fp16 normal range: report any nonzero
// one with |x| < 2^-14 or |x| > 65504 (one pass over both arrays).
__global__ void sb_range_kernel(const uint16_t* __restrict__ scales,
                                const uint16_t* __restrict__ biases, int64_t n,
                                uint32_t* status) {
  bool bad = false;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float s = fabsf(__uint_as_float(static_cast<uint32_t>(scales[i]) << 16));
    const float b = fabsf(__uint_as_float(static_cast<uint32_t>(biases[i]) << 16));
    bad = bad || (s != 0.f && (s < 6.103515625e-05f || s > 65504.f)) ||
          (b != 0.f && (b < 6.103515625e-05f || b > 65504.f));
  }
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) set_status(status, ST_FP16);
}

// ---------------------------------------------- staged dequantisation --
// fp16 rows [rows, D] of a 4- or 8-bit affine head, vocab rows v0 .. v0+rows,
// in natural column order: w = q * scale + bias per group of 64 along D.  The
// values are those the in-kernel dequantiser produces (the same fp16 ops on
// the same bits: 0x6400 | q is 1024 + q, subtract 1024, one fma), only laid
// out in order.  One thread per 8 weights (one 4-bit word or two 8-bit
// words): a warp reads 128 or 256 contiguous bytes and writes 512.
template <int QB>
__global__ void dequant_rows_f16_kernel(const uint32_t* __restrict__ qw,
                                        const uint16_t* __restrict__ scales,
                                        const uint16_t* __restrict__ biases, int64_t v0,
                                        int64_t rows, int D, uint4* __restrict__ out) {
  static_assert(QB == 4 || QB == 8, "4- or 8-bit heads");
  using Word = typename std::conditional<QB == 4, uint32_t, uint2>::type;
  constexpr int U = 4;  // units per thread in flight (loads issued before use)
  const int64_t n8 = rows * (D / 8);  // 8-weight units
  const int upr = D / 8, gpr = D / 64;
  const __half2 k1024 = __float2half2_rn(1024.f);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i0 = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i0 < n8;
       i0 += U * stride) {
    Word w[U];
    uint16_t sb[U], bb[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t i = i0 + u * stride;
      if (i < n8) {
        const int64_t r = i / upr;
        const int c8 = static_cast<int>(i - r * upr);
        const int64_t v = v0 + r;
        const size_t gi = static_cast<size_t>(v) * gpr + c8 / 8;
        w[u] = __ldg(reinterpret_cast<const Word*>(qw + static_cast<size_t>(v) * (D / (32 / QB))) + c8);
        sb[u] = __ldg(scales + gi);
        bb[u] = __ldg(biases + gi);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t i = i0 + u * stride;
      if (i >= n8) break;
      const __half2 s2 = __float2half2_rn(__uint_as_float(static_cast<uint32_t>(sb[u]) << 16));
      const __half2 b2 = __float2half2_rn(__uint_as_float(static_cast<uint32_t>(bb[u]) << 16));
      uint32_t t[4];
      if constexpr (QB == 4) {
        // element j = bits 4j..4j+3: the half pairs come out as (e_k, e_k+4)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t x = ((w[u] >> (4 * k)) & 0x000F000Fu) | 0x64006400u;
          __half2 h = __hfma2(__hsub2(*reinterpret_cast<const __half2*>(&x), k1024), s2, b2);
          t[k] = *reinterpret_cast<uint32_t*>(&h);
        }
        out[i] = make_uint4(__byte_perm(t[0], t[1], 0x5410), __byte_perm(t[2], t[3], 0x5410),
                            __byte_perm(t[0], t[1], 0x7632), __byte_perm(t[2], t[3], 0x7632));
      } else {
        // element j of a word = byte j: pairs (e0,e2) (e1,e3) per word
        const uint32_t ws[2] = {w[u].x, w[u].y};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t x = ((ws[k >> 1] >> (8 * (k & 1))) & 0x00FF00FFu) | 0x64006400u;
          __half2 h = __hfma2(__hsub2(*reinterpret_cast<const __half2*>(&x), k1024), s2, b2);
          t[k] = *reinterpret_cast<uint32_t*>(&h);
        }
        out[i] = make_uint4(__byte_perm(t[0], t[1], 0x5410), __byte_perm(t[0], t[1], 0x7632),
                            __byte_perm(t[2], t[3], 0x5410), __byte_perm(t[2], t[3], 0x7632));
      }
    }
  }
}

// ---------------------------------------------------- trainable head --
// hg[m, d] = bf16(coeff[m] * H[m, d]): the B operand of the dW GEMM (the row
// cotangent enters along K, so it is folded into the rows of H).
template <typename T>
__global__ void scale_rows_bf16_kernel(const T* __restrict__ H, const float* __restrict__ coeff,
                                       int64_t M, int D, __nv_bfloat16* __restrict__ out) {
  const int64_t n = M * D;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = i / D;
    float h;
    if constexpr (sizeof(T) == 4) h = H[i];
    else h = __bfloat162float(H[i]);
    out[i] = __float2bfloat16_rn(coeff[m] * h);
  }
}

// ----------------------------------------------- prefix-shared ORPO pair --
// Source row of head row m (Training design §5.4): m - 1 for m >= 1 except
// the first rejected row m = P + Rc, which reads P - 1; head row 0 reads 0.
__device__ __forceinline__ int64_t prefix_src(int64_t m, int64_t P, int64_t Rc) {
  return m == 0 ? 0 : (m == P + Rc ? P - 1 : m - 1);
}

// H_head[m] = H_cat[prefix_src(m)], rows of `row_bytes` (multiple of 16).
__global__ void prefix_gather_kernel(const uint4* __restrict__ src, int64_t M, int64_t P,
                                     int64_t Rc, int64_t row16, uint4* __restrict__ dst) {
  const int64_t n = M * row16;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = i / row16, c = i - m * row16;
    dst[i] = src[prefix_src(m, P, Rc) * row16 + c];
  }
}

// Adjoint: dH_cat[r] = sum over head rows m with prefix_src(m) == r of
// dH_head[m], added in increasing m (deterministic).  Rows P + Rc - 1 and
// M - 1 receive nothing.
__global__ void prefix_scatter_kernel(const float4* __restrict__ dh, int64_t M, int64_t P,
                                      int64_t Rc, int64_t row4, float4* __restrict__ out) {
  const int64_t n = M * row4;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / row4, c = i - r * row4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    auto add = [&](int64_t m) {
      const float4 v = dh[m * row4 + c];
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    };
    if (r == 0) add(0);
    if (r + 1 < M && r + 1 != P + Rc) add(r + 1);
    if (r == P - 1) add(P + Rc);
    out[i] = acc;
  }
}

// ------------------------------------------------- K-split partial sums --
// dH += parts[0] + parts[1] + ... (fixed order, so the result is
// deterministic); n4 = M*D/4 float4 elements per buffer.
__global__ void add_parts_kernel(float4* __restrict__ dh, const float4* __restrict__ parts,
                                 int nparts, int64_t n4) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float4 v = dh[i];
    for (int p = 0; p < nparts; ++p) {
      const float4 q = parts[p * n4 + i];
      v.x += q.x;
      v.y += q.y;
      v.z += q.z;
      v.w += q.w;
    }
    dh[i] = v;
  }
}

// ------------------------------------------------------ timeout self-test --
__global__ void selftest_timeout_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Nothing ever arrives on `bar`: the wait must run out.
    if (!wait_bounded(&bar, 0, limit_ns, nullptr)) set_status(status, ST_TIMEOUT);
  }
}

}  // namespace cce
