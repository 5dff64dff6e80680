// hbit.cuh -- the activation side of H-BitLinear: an online Hadamard transform
// of each token row, then 4-bit absmax codes.
//
// The "BitNet v2" page (brain.hanbit.co.kr; the paragraphs on the H-BitLinear
// module and on native 4-bit activations) describes the module as a Hadamard
// transform of the activations applied on the fly, a 4-bit quantisation, then
// the ternary linear map.  It gives no size, normalisation or evaluation order
// for the transform and no formula for the 4-bit quantiser; the readings here
// are the ones the oracle states:
//   - B = the largest power of two dividing K; each B-block of a row is
//     multiplied by the Sylvester-order Walsh-Hadamard matrix, formed by the
//     in-place fast transform in fp32: stage h = 1, 2, 4, ..., B/2 replaces
//     every pair (j, j + h) with bit h of j clear by (a + b, a - b), one
//     rounding each; then one fp32 multiply by RN32(1 / sqrt(B)).
//   - gamma = max |xh|, q = clamp(rne(RN(xh * 7) / RN(gamma + 1e-5)), -8, 7),
//     and the rescale divides by 7 instead of 127.
// Every element's value after each stage is one IEEE add or subtract of two
// values of the previous stage, so the order in which threads visit the pairs
// does not matter: the transformed row, and so the codes, are bit-identical to
// a sequential evaluation.  The codes are held in int8 and feed the unchanged
// kind::i8 tensor-core GEMM (tcgen05 has no 4-bit integer kind).
#pragma once
#include "quant_pack.cuh"

namespace bl {

constexpr int kHbitThreads = 256;
constexpr int kHbitMaxK = 16384;  // the row is transformed in shared memory (64 KB of fp32)
constexpr float kQb4 = 7.0f;

__host__ __device__ constexpr int hbit_block(int K) {
  int b = 1;
  while (K % (2 * b) == 0 && 2 * b <= K) b *= 2;
  return b;
}

// One CTA per token row (blocks past M clear the split-K sums and blockIdx 0
// the arrival counters of the GEMMs that follow, as quant_act_kernel does).
// kPermute: codes in contraction order [M, ldq], ldq = K rounded up to 16
// (zeros past K); otherwise natural order with ldq = K.
template <bool kPermute>
__global__ void __launch_bounds__(kHbitThreads) hbit_quant_kernel(const uint16_t* __restrict__ x, int M, int K,
                                                                  int B, float scale, int ldq, int8_t* __restrict__ q,
                                                                  float* __restrict__ gamma,
                                                                  int32_t* __restrict__ rowsum,
                                                                  uint32_t* __restrict__ cnt, int ncnt,
                                                                  float* __restrict__ zbuf, size_t zvec4) {
  extern __shared__ float s_v[];  // [K]: the row, transformed in place
  __shared__ uint32_t s_max[kHbitThreads / 32];
  __shared__ int32_t s_sum[kHbitThreads / 32];
  pdl_wait_primary();
  pdl_launch_dependents();
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < ncnt; i += blockDim.x) cnt[i] = 0u;
  if (static_cast<int>(blockIdx.x) >= M) {
    const size_t stride = static_cast<size_t>(gridDim.x - M) * blockDim.x;
    for (size_t i = static_cast<size_t>(blockIdx.x - M) * blockDim.x + threadIdx.x; i < zvec4; i += stride)
      reinterpret_cast<float4*>(zbuf)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    return;
  }
  const int row = blockIdx.x;
  const uint16_t* xr = x + static_cast<size_t>(row) * K;
  for (int k = threadIdx.x; k < K; k += blockDim.x) s_v[k] = bf16_bits_to_f32(xr[k]);
  __syncthreads();

  // fast Walsh-Hadamard butterflies, stage by stage over the whole row
  // (blocks start at multiples of B >= 2h, so a pair never leaves its block)
  const int half = K >> 1;
  for (int h = 1, lh = 0; h < B; h <<= 1, ++lh) {
    for (int p = threadIdx.x; p < half; p += blockDim.x) {
      const int j = ((p >> lh) << (lh + 1)) | (p & (h - 1));  // the p-th index with bit h clear
      const float a = s_v[j], b = s_v[j + h];
      s_v[j] = __fadd_rn(a, b);
      s_v[j + h] = __fsub_rn(a, b);
    }
    __syncthreads();
  }

  // orthonormal scale, then gamma = max |xh| (integer max of the |xh| bit patterns)
  uint32_t mx = 0u;
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    const float v = __fmul_rn(s_v[k], scale);
    s_v[k] = v;
    mx = max(mx, __float_as_uint(fabsf(v)));
  }
  mx = __reduce_max_sync(0xffffffffu, mx);
  if ((threadIdx.x & 31) == 0) s_max[threadIdx.x >> 5] = mx;
  __syncthreads();
  mx = 0u;
#pragma unroll
  for (int w = 0; w < kHbitThreads / 32; ++w) mx = max(mx, s_max[w]);
  const float g = __uint_as_float(mx);
  const float d = __fadd_rn(g, kEps);

  // 4-bit codes, one 16-wide k-group per thread and step
  int32_t sum = 0;
  int8_t* qr = q + static_cast<size_t>(row) * ldq;
  const int groups = (K + 15) / 16;
  for (int gi = threadIdx.x; gi < groups; gi += blockDim.x) {
    uint32_t c[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int k = 16 * gi + i;
      int32_t v = 0;
      if (k < K) {
        v = __float2int_rn(__fdiv_rn(__fmul_rn(s_v[k], kQb4), d));
        v = max(-8, min(7, v));
      }
      sum += v;
      c[i] = static_cast<uint32_t>(v) & 0xFFu;
    }
    if (kPermute) {
      // byte 4j + b <- k = 16 gi + 4b + j
      uint4 w;
      w.x = c[0] | (c[4] << 8) | (c[8] << 16) | (c[12] << 24);
      w.y = c[1] | (c[5] << 8) | (c[9] << 16) | (c[13] << 24);
      w.z = c[2] | (c[6] << 8) | (c[10] << 16) | (c[14] << 24);
      w.w = c[3] | (c[7] << 8) | (c[11] << 16) | (c[15] << 24);
      *reinterpret_cast<uint4*>(qr + 16 * gi) = w;
    } else {
      for (int i = 0; i < 16 && 16 * gi + i < K; ++i) qr[16 * gi + i] = static_cast<int8_t>(c[i]);
    }
  }
  sum = __reduce_add_sync(0xffffffffu, sum);
  if ((threadIdx.x & 31) == 0) s_sum[threadIdx.x >> 5] = sum;
  __syncthreads();
  if (threadIdx.x == 0) {
    int32_t t = 0;
#pragma unroll
    for (int w = 0; w < kHbitThreads / 32; ++w) t += s_sum[w];
    if (gamma) gamma[row] = g;
    if (rowsum) rowsum[row] = t;
  }
}

}  // namespace bl
