// quant_pack.cuh -- per-token activation quantisation and the weight packers.
//
// Activation quantisation follows the BitNet b1.58 activation_quant of the
// "BitNet 1-Bit LLM" blog (section "Absmean quantization function"):
// gamma = max |x| per token, q = clamp(round(x * 127 / (gamma + 1e-5)), -128, 127),
// rounded half to even, with the product and the quotient evaluated as IEEE
// fp32 (x * 127 is exact for bf16 x).
//
// Weight quantisation follows weight_quant_ternary on the same page (absmean
// over the whole matrix, W / (alpha + 1e-5) rounded half to even, clamped to
// [-1, 1]) and the 2B4T report's section 5.1 (four ternary values per byte);
// the 2-bit code map is bitnet.cpp's I2_S map (-1 -> 00, 0 -> 01, +1 -> 10).
// The N:M mask follows the Sparse-BitNet review, section 3.2: the n largest
// |W| of each block of m consecutive k are kept (ties to the lower k), and the
// mask is applied after ternarisation.
#pragma once
#include "ptx.cuh"

namespace bl {

constexpr float kEps = 1e-5f;
constexpr float kQb = 127.0f;

// ----------------------------------------------------------------- helpers

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

// Ternary value of one latent weight: clamp(rne(w / d), -1, 1).
__device__ __forceinline__ int32_t ternary_of(float w, float d) {
  int32_t c = __float2int_rn(__fdiv_rn(w, d));
  return max(-1, min(1, c));
}

template <typename T, typename Op>
__device__ __forceinline__ T block_reduce(T v, Op op, T* red /* >= 32 entries */, T identity) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  const int nw = (blockDim.x + 31) >> 5;
  v = lane < nw ? red[lane] : identity;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

struct AddD {
  __device__ double operator()(double a, double b) const { return a + b; }
};

// Exact round-half-to-even of RN(t / d), t = RN(v * 127), for |t / d| < 128,
// without a division per element.  With c = RN(127 * RN(1 / d)), the exact
// product v * c differs from t / d by at most 2 * 2^-24 relative (bf16 v: t is
// exact), i.e. by less than 1.6e-5 absolute, and RN(t / d) lies within 7.6e-6
// of t / d.  One fused multiply-add, r' = RN(v * c + 1.5 * 2^23), rounds the
// exact product to the nearest integer r (the sum's last place is 1, ties to
// even) and leaves the two's-complement code in the low byte; a second,
// e = RN(v * c - r), gives the distance to it within 2^-25.  Unless some |e| of
// a group exceeds 1/2 - 2^-14, RN(t / d) is nearer than 1/2 to r and rounds to
// it; such a group is recomputed with the exact quotient.
constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23

// Codes of 8 consecutive activations (the first or second half of a 16-group).  b[e] holds the code of
// element e in its low byte.
__device__ __forceinline__ void codes8(const uint32_t (&raw)[4], float c, float d, uint32_t (&b)[8]) {
  float emax = 0.0f;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float v = __uint_as_float((e & 1) ? (raw[e >> 1] & 0xFFFF0000u) : (raw[e >> 1] << 16));
    const float sm = __fmaf_rn(v, c, kMagic);
    emax = fmaxf(emax, fabsf(__fmaf_rn(v, c, -__fsub_rn(sm, kMagic))));
    b[e] = __float_as_uint(sm);
  }
  if (emax > 0.5f - 6.103515625e-05f) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float v = __uint_as_float((e & 1) ? (raw[e >> 1] & 0xFFFF0000u) : (raw[e >> 1] << 16));
      b[e] = 0x4B400000u + static_cast<uint32_t>(__float2int_rn(__fdiv_rn(__fmul_rn(v, kQb), d)));
    }
  }
}

// codes8 for fp32 values (RMSNorm outputs): the same rounding argument holds
// with t = RN(v * 127) no longer exact, since |v * c - RN(t / d)| stays below
// 4 * 2^-24 * 127 < 2^-14; the fallback recomputes RN(RN(v * 127) / d).
__device__ __forceinline__ void codes8f(const float* v, float c, float d, uint32_t (&b)[8]) {
  float emax = 0.0f;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float sm = __fmaf_rn(v[e], c, kMagic);
    emax = fmaxf(emax, fabsf(__fmaf_rn(v[e], c, -__fsub_rn(sm, kMagic))));
    b[e] = __float_as_uint(sm);
  }
  if (emax > 0.5f - 6.103515625e-05f) {
#pragma unroll
    for (int e = 0; e < 8; ++e)
      b[e] = 0x4B400000u + static_cast<uint32_t>(__float2int_rn(__fdiv_rn(__fmul_rn(v[e], kQb), d)));
  }
}

// 8 bf16 values of a row from k0 as 4 words (zero past K).
__device__ __forceinline__ void load8_raw(const uint16_t* row, int k0, int K, bool vec_ok, uint32_t (&r)[4]) {
  if (vec_ok && k0 + 8 <= K) {
    const uint4 a = *reinterpret_cast<const uint4*>(row + k0);
    r[0] = a.x; r[1] = a.y; r[2] = a.z; r[3] = a.w;
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t lo = (k0 + 2 * i < K) ? row[k0 + 2 * i] : 0u;
      const uint32_t hi = (k0 + 2 * i + 1 < K) ? row[k0 + 2 * i + 1] : 0u;
      r[i] = lo | (hi << 16);
    }
  }
}

// ----------------------------------------------------------------- quant_act
// A token row is handled by wpr warps of a 256-thread CTA (wpr = 1, 2, 4 or 8,
// 8 / wpr rows per CTA).  A lane owns the 16-wide k-groups
// g = sub * 32 + lane + j * 32 * wpr of its row; when the row fits (K % 8 == 0,
// at most G groups per lane) every load of the row is issued at once into
// registers, so each element is read from memory once and all of a CTA's
// reads are in flight together.  quant_shape picks the smallest wpr that
// leaves at most three groups per lane (short per-warp chains, many warps in
// flight; the kernel is bound by latency, not by issue) and G, a compile-time
// register count of 2, 3 or 8.  With RMSNorm and enough rows to give every SM
// a CTA of eight (M >= 8 * SMs), a row of up to 256 groups stays in one warp:
// at M = 2048, K = 2560 that measured faster than two warps joined by the
// barriers of the fp64 sum, the maximum and the code sum, while for a few rows
// the shorter per-warp chains of the split win.  With fewer rows than about
// 24 warps per SM would take, each row is split further (up to eight warps):
// at M = 256 and M = 16, K = 2560, eight warps a row took 2.9 and 2.5 us
// against 4.0 and 3.3 us for two, while at M = 2048 two stayed fastest.  gamma is an integer warp max of the
// |x| bit patterns (then across the row's warps), and the 16 codes of a group
// come from the division-free exact rounding of codes8.  Longer or unaligned
// rows take a two-pass loop (the second pass re-reads from L1/L2).
// kPermute = false writes natural-order codes [M, ldq] (ldq = K, or K rounded
// up to 16 with zeros past K, as the structured-sparse MMA reads them);
// kPermute = true writes the contraction order [M, ldq] with ldq = K rounded
// up to 16 (zeros past K).  kNorm = true first applies RMSNorm with weight gnorm
// ([b158] BitLinear_b158.forward normalises x before activation_quant):
// r = RN32(1 / sqrt(RN32(sum x^2 / K) + eps)) with the sum, the root and the
// quotient in fp64, xn = RN(RN(x * r) * g) in fp32, and quantises xn.  Both write gamma and, when asked, the sum of the row's
// codes.  The first CTA also clears the split-K arrival counters, and CTAs
// past the rows (blockIdx >= qblocks) clear the split-K sums, of the GEMMs that
// read these codes.
constexpr int kQuantWarps = 8;

struct QuantShape {
  int wpr;  // warps per token row
  int G;    // k-groups per lane held in registers (template argument: 2, 3 or 8)
};

__host__ __device__ __forceinline__ QuantShape quant_shape(int M, int K, bool norm, int sm_count) {
  const int groups = (K + 15) / 16;
  int wpr = 1;
  if (!(norm && groups <= 8 * 32 && M >= kQuantWarps * sm_count))
    while (wpr < kQuantWarps && groups > 3 * 32 * wpr) wpr *= 2;
  // few rows: split them over more warps until about 24 warps per SM are in flight
  while (wpr < kQuantWarps && M * wpr < 24 * sm_count && !(norm && M >= kQuantWarps * sm_count)) wpr *= 2;
  const int need = (groups + 32 * wpr - 1) / (32 * wpr);
  return {wpr, need <= 2 ? 2 : need <= 3 ? 3 : 8};
}

// 16 codes of one k-group (raw: the group's 16 bf16 as 8 words) in the
// requested order; adds their sum to *sum.
template <bool kPermute>
__device__ __forceinline__ uint4 pack_group(const uint32_t (&b0)[8], const uint32_t (&b1)[8], int32_t& sum) {
  uint32_t w[4];
  if (kPermute) {
    // byte 4j + b <- k0 + 4b + j
#pragma unroll
    for (int j = 0; j < 4; ++j)
      w[j] = __byte_perm(__byte_perm(b0[j], b0[4 + j], 0x0040), __byte_perm(b1[j], b1[4 + j], 0x0040), 0x5410);
  } else {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      w[j] = __byte_perm(__byte_perm(b0[4 * j], b0[4 * j + 1], 0x0040), __byte_perm(b0[4 * j + 2], b0[4 * j + 3], 0x0040),
                         0x5410);
      w[2 + j] = __byte_perm(__byte_perm(b1[4 * j], b1[4 * j + 1], 0x0040),
                             __byte_perm(b1[4 * j + 2], b1[4 * j + 3], 0x0040), 0x5410);
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) sum = __dp4a(static_cast<int>(w[j]), 0x01010101, sum);
  return make_uint4(w[0], w[1], w[2], w[3]);
}

template <bool kPermute>
__device__ __forceinline__ uint4 group_codes(const uint32_t (&r0)[4], const uint32_t (&r1)[4], float c, float d,
                                             int32_t& sum) {
  uint32_t b0[8], b1[8];
  codes8(r0, c, d, b0);  // elements past K are zero and give code 0
  codes8(r1, c, d, b1);
  return pack_group<kPermute>(b0, b1, sum);
}

// 16 normalised values of a group: xn = RN(RN(x * r) * g) (zero past K, where g is not read).
__device__ __forceinline__ void norm16(const uint32_t (&r0)[4], const uint32_t (&r1)[4], const float* __restrict__ g,
                                       int k0, int K, float r, float (&xn)[16]) {
  float gv[16];
  if (k0 + 16 <= K && (reinterpret_cast<uintptr_t>(g + k0) & 15u) == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 t = reinterpret_cast<const float4*>(g + k0)[i];
      gv[4 * i] = t.x; gv[4 * i + 1] = t.y; gv[4 * i + 2] = t.z; gv[4 * i + 3] = t.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) gv[i] = k0 + i < K ? g[k0 + i] : 0.0f;
  }
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const uint32_t w = e < 8 ? r0[e >> 1] : r1[(e - 8) >> 1];
    const float xv = __uint_as_float((e & 1) ? (w & 0xFFFF0000u) : (w << 16));
    xn[e] = __fmul_rn(__fmul_rn(xv, r), gv[e]);
  }
}

__device__ __forceinline__ double sumsq8(const uint32_t (&w)[4], double acc) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const double lo = static_cast<double>(__uint_as_float(w[i] << 16));
    const double hi = static_cast<double>(__uint_as_float(w[i] & 0xFFFF0000u));
    acc = __fma_rn(lo, lo, acc);
    acc = __fma_rn(hi, hi, acc);
  }
  return acc;
}

__device__ __forceinline__ float absmax8(const uint32_t (&w)[4], float mx) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
    mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(w[i] << 16)), fabsf(__uint_as_float(w[i] & 0xFFFF0000u))));
  return mx;
}

// Four CTAs per SM for G <= 3 (at most 64 registers a thread), so that one
// wave holds 2048 tokens split over two warps each; two for G = 8.
template <bool kPermute, bool kNorm, int G>
__global__ void __launch_bounds__(32 * kQuantWarps, G <= 3 ? 4 : 2) quant_act_kernel(const uint16_t* __restrict__ x, int M, int K,
                                                                     int ldq, int8_t* __restrict__ q,
                                                                     float* __restrict__ gamma,
                                                                     int32_t* __restrict__ rowsum,
                                                                     uint32_t* __restrict__ cnt, int ncnt,
                                                                     float* __restrict__ zbuf, size_t zvec4,
                                                                     int qblocks, int wpr,
                                                                     const float* __restrict__ gnorm, float eps) {
  __shared__ float s_mx[kQuantWarps];
  __shared__ int32_t s_sum[kQuantWarps];
  __shared__ double s_ss[kQuantWarps];
  pdl_wait_primary();
  pdl_launch_dependents();
  // split-K arrival counters and sums of the GEMMs that follow start from zero
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < ncnt; i += blockDim.x) cnt[i] = 0u;
  if (static_cast<int>(blockIdx.x) >= qblocks) {
    const size_t stride = static_cast<size_t>(gridDim.x - qblocks) * blockDim.x;
    for (size_t i = static_cast<size_t>(blockIdx.x - qblocks) * blockDim.x + threadIdx.x; i < zvec4; i += stride)
      reinterpret_cast<float4*>(zbuf)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    return;
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rloc = warp / wpr, sub = warp - rloc * wpr;
  const int row = blockIdx.x * (kQuantWarps / wpr) + rloc;
  const bool active = row < M;  // inactive warps still reach the CTA barriers
  const uint16_t* xr = x + static_cast<size_t>(active ? row : 0) * K;
  const bool vec_ok = (K % 8) == 0 && (reinterpret_cast<uintptr_t>(x) & 15u) == 0;
  const int groups = (K + 15) / 16;
  const int gstride = 32 * wpr;
  const int g0 = sub * 32 + lane;
  const bool in_regs = vec_ok && groups <= G * gstride;

  // Calls f(g, r0, r1) for each of this lane's groups with the group's raw
  // bf16 words: from registers (unrolled, static indices) or loaded again.
  uint32_t v[G][8];
  auto for_groups = [&](auto&& f) {
    if (in_regs) {
#pragma unroll
      for (int j = 0; j < G; ++j) {
        const int g = g0 + j * gstride;
        if (g < groups) {
          uint32_t r0[4], r1[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            r0[i] = v[j][i];
            r1[i] = v[j][4 + i];
          }
          f(g, r0, r1);
        }
      }
    } else {
      for (int g = g0; g < groups; g += gstride) {
        uint32_t r0[4], r1[4];
        load8_raw(xr, 16 * g, K, vec_ok, r0);
        load8_raw(xr, 16 * g + 8, K, vec_ok, r1);
        f(g, r0, r1);
      }
    }
  };
  if (active && in_regs) {
#pragma unroll
    for (int j = 0; j < G; ++j) {
      const int k0 = 16 * (g0 + j * gstride);
      uint4 a = make_uint4(0u, 0u, 0u, 0u), b = make_uint4(0u, 0u, 0u, 0u);
      if (k0 + 8 <= K) a = *reinterpret_cast<const uint4*>(xr + k0);
      if (k0 + 16 <= K) b = *reinterpret_cast<const uint4*>(xr + k0 + 8);
      v[j][0] = a.x; v[j][1] = a.y; v[j][2] = a.z; v[j][3] = a.w;
      v[j][4] = b.x; v[j][5] = b.y; v[j][6] = b.z; v[j][7] = b.w;
    }
  }

  // RMSNorm: r = RN32(1 / sqrt(RN32(sum x^2 / K) + eps)), sums in fp64
  float rn = 1.0f;
  if (kNorm) {
    double ss = 0.0;
    if (active) for_groups([&](int, const uint32_t (&r0)[4], const uint32_t (&r1)[4]) { ss = sumsq8(r1, sumsq8(r0, ss)); });
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (wpr > 1) {
      if (lane == 0) s_ss[warp] = ss;
      __syncthreads();
      ss = 0.0;
      for (int i = 0; i < wpr; ++i) ss += s_ss[rloc * wpr + i];
    }
    const float ms = __double2float_rn(__ddiv_rn(ss, static_cast<double>(K)));
    rn = __double2float_rn(__ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(static_cast<double>(ms), static_cast<double>(eps)))));
  }

  float mx = 0.0f;
  if (active)
    for_groups([&](int g, const uint32_t (&r0)[4], const uint32_t (&r1)[4]) {
      if (kNorm) {
        float xn[16];
        norm16(r0, r1, gnorm, 16 * g, K, rn, xn);
#pragma unroll
        for (int e = 0; e < 16; ++e) mx = fmaxf(mx, fabsf(xn[e]));
      } else {
        mx = absmax8(r1, absmax8(r0, mx));
      }
    });
  // |x| >= 0, whose bit patterns order like the values: integer maxima
  mx = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(mx)));
  if (wpr > 1) {
    if (lane == 0) s_mx[warp] = mx;
    __syncthreads();
    for (int i = 0; i < wpr; ++i) mx = fmaxf(mx, s_mx[rloc * wpr + i]);
  }
  const float d = __fadd_rn(mx, kEps);
  const float c = __fmul_rn(kQb, __frcp_rn(d));

  int32_t sum = 0;
  if (active) {
    int8_t* qr = q + static_cast<size_t>(row) * ldq;
    const bool qvec = ((reinterpret_cast<uintptr_t>(q) & 15u) == 0) && (ldq % 16) == 0;
    for_groups([&](int g, const uint32_t (&r0)[4], const uint32_t (&r1)[4]) {
      const int k0 = 16 * g;
      uint4 w;
      if (kNorm) {
        float xn[16];
        norm16(r0, r1, gnorm, k0, K, rn, xn);
        uint32_t b0[8], b1[8];
        codes8f(xn, c, d, b0);
        codes8f(xn + 8, c, d, b1);
        w = pack_group<kPermute>(b0, b1, sum);
      } else {
        w = group_codes<kPermute>(r0, r1, c, d, sum);
      }
      if (kPermute || (qvec && k0 + 16 <= ldq)) {
        *reinterpret_cast<uint4*>(qr + k0) = w;
      } else {
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
        for (int i = 0; i < 16 && k0 + i < K; ++i) qr[k0 + i] = static_cast<int8_t>(ww[i >> 2] >> (8 * (i & 3)));
      }
    });
  }
  sum = __reduce_add_sync(0xffffffffu, sum);
  if (wpr > 1) {
    if (lane == 0) s_sum[warp] = sum;
    __syncthreads();
    sum = 0;
    for (int i = 0; i < wpr; ++i) sum += s_sum[rloc * wpr + i];
  }
  if (active && sub == 0 && lane == 0) {
    if (gamma) gamma[row] = mx;
    if (rowsum) rowsum[row] = sum;
  }
}

// ----------------------------------------------------------------- absmean
// Stage 1: per-CTA fp64 partial sums of |W| (grid-stride, fixed grid).
__global__ void __launch_bounds__(256) absmean_partial_kernel(const float* __restrict__ W, int64_t count,
                                                              double* __restrict__ partial) {
  __shared__ double red[32];
  double s = 0.0;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < count; i += stride)
    s += fabs(static_cast<double>(W[i]));
  s = block_reduce(s, AddD(), red, 0.0);
  if (threadIdx.x == 0) partial[blockIdx.x] = s;
}

// Stage 2: one CTA adds the partials in a fixed order; alpha = RN32(sum / count).
__global__ void __launch_bounds__(256) absmean_final_kernel(const double* __restrict__ partial, int nparts,
                                                            int64_t count, float* __restrict__ alpha) {
  __shared__ double red[32];
  double s = 0.0;
  for (int i = threadIdx.x; i < nparts; i += blockDim.x) s += partial[i];
  s = block_reduce(s, AddD(), red, 0.0);
  if (threadIdx.x == 0) *alpha = static_cast<float>(s / static_cast<double>(count));
}

// ----------------------------------------------------------------- dense pack
// One thread per 16-byte unit (64 weights) of a packed row.  Source is either a
// latent fp32 matrix (ternarised with alpha) or an int8 ternary matrix.
template <bool kFromLatent>
__global__ void __launch_bounds__(256) pack_dense_kernel(const float* __restrict__ W, const int8_t* __restrict__ Wt,
                                                         int N, int K, int64_t ld, const float* __restrict__ alpha,
                                                         uint8_t* __restrict__ codes) {
  const int64_t units_per_row = ld / 16;
  const int64_t u = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (u >= units_per_row * N) return;
  const int64_t r = u / units_per_row;
  const int k0 = static_cast<int>(u % units_per_row) * 64;
  float d = 0.0f;
  if (kFromLatent) d = __fadd_rn(*alpha, kEps);
  uint32_t w[4];
#pragma unroll
  for (int wi = 0; wi < 4; ++wi) {
    uint32_t acc = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int k = k0 + wi * 16 + i;
      int32_t t = 0;
      if (k < K) {
        if (kFromLatent)
          t = ternary_of(W[r * K + k], d);
        else
          t = max(-1, min(1, static_cast<int32_t>(Wt[r * K + k])));
      }
      acc |= static_cast<uint32_t>(t + 1) << (2 * i);
    }
    w[wi] = acc;
  }
  *reinterpret_cast<uint4*>(codes + r * ld + (k0 / 4)) = make_uint4(w[0], w[1], w[2], w[3]);
}

__global__ void write_alpha_kernel(float* alpha_out, float a) {
  if (threadIdx.x == 0 && blockIdx.x == 0) *alpha_out = a;
}

// ----------------------------------------------------------------- N:M pack
// One thread per span of 64 blocks of one row.  Writes the span's kept codes
// (16 * n bytes) and metadata (32 bytes for 2:4, 64 for n:8), clipped to the
// row strides; positions past the row's last block keep code 01 / meta 0.
__global__ void __launch_bounds__(128) pack_nm_kernel(const float* __restrict__ W, int N, int K, int n, int m,
                                                      int64_t ldv, int64_t ldm, const float* __restrict__ alpha,
                                                      uint8_t* __restrict__ values, uint8_t* __restrict__ meta) {
  const int blocks_per_row = K / m;
  const int spans = (blocks_per_row + 63) / 64;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= static_cast<int64_t>(spans) * N) return;
  const int64_t r = t / spans;
  const int s = static_cast<int>(t % spans);
  const float d = __fadd_rn(*alpha, kEps);

  uint8_t vb[112];  // up to 16 * 7 bytes of kept codes
  uint8_t mb[64];
  const int vbytes = 16 * n, mbytes = (m == 4) ? 32 : 64;
  for (int i = 0; i < vbytes; ++i) vb[i] = 0x55;
  for (int i = 0; i < mbytes; ++i) mb[i] = 0;

  int out = 0;  // kept-code index inside the span
  for (int bi = 0; bi < 64; ++bi) {
    const int b = s * 64 + bi;
    if (b >= blocks_per_row) break;
    const float* w = W + r * K + static_cast<int64_t>(b) * m;
    float a[8];
    for (int j = 0; j < m; ++j) a[j] = fabsf(w[j]);
    uint32_t keep = 0;
    for (int j = 0; j < m; ++j) {
      int rank = 0;
      for (int i = 0; i < m; ++i) rank += (a[i] > a[j]) || (a[i] == a[j] && i < j);
      if (rank < n) keep |= 1u << j;
    }
    int kept = 0;
    uint32_t nib = 0;
    for (int j = 0; j < m; ++j) {
      if (!((keep >> j) & 1u)) continue;
      const uint32_t code = static_cast<uint32_t>(ternary_of(w[j], d) + 1);
      const int pos = out++;
      vb[pos >> 2] = static_cast<uint8_t>((vb[pos >> 2] & ~(3u << (2 * (pos & 3)))) | (code << (2 * (pos & 3))));
      if (m == 4) nib |= static_cast<uint32_t>(j) << (2 * kept);
      ++kept;
    }
    if (m == 4)
      mb[bi >> 1] |= static_cast<uint8_t>(nib << (4 * (bi & 1)));
    else
      mb[bi] = static_cast<uint8_t>(keep);
  }
  const int64_t v0 = static_cast<int64_t>(s) * vbytes, m0 = static_cast<int64_t>(s) * mbytes;
  for (int i = 0; i < vbytes && v0 + i < ldv; ++i) values[r * ldv + v0 + i] = vb[i];
  for (int i = 0; i < mbytes && m0 + i < ldm; ++i) meta[r * ldm + m0 + i] = mb[i];
}

}  // namespace bl
