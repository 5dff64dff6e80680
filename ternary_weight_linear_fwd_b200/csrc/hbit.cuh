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

// 4-bit codes of 16 fp32 values without a division per element: with
// c = RN(7 * RN(1 / d)) the exact product v * c lies within 2e-6 of
// RN(RN(v * 7) / d) (|q| <= 7: two roundings in c, one in RN(v * 7), one in
// the quotient, each at most 2^-24 relative), so one fused multiply-add with
// 1.5 * 2^23 rounds v * c to the nearest integer r (ties to even) and a second
// gives v * c - r; unless some |v * c - r| of the group exceeds 1/2 - 2^-14,
// RN(RN(v * 7) / d) is nearer than 1/2 to r and rounds to it.  Otherwise the
// group is recomputed with the exact quotient.  Codes clamp to [-8, 7].
__device__ __forceinline__ void codes16_q7(const float (&v)[16], float c, float d, int32_t (&q)[16]) {
  float emax = 0.0f;
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const float sm = __fmaf_rn(v[e], c, kMagic);
    emax = fmaxf(emax, fabsf(__fmaf_rn(v[e], c, -__fsub_rn(sm, kMagic))));
    q[e] = static_cast<int32_t>(__float_as_uint(sm) - 0x4B400000u);
  }
  if (emax > 0.5f - 6.103515625e-05f) {
#pragma unroll
    for (int e = 0; e < 16; ++e) q[e] = __float2int_rn(__fdiv_rn(__fmul_rn(v[e], kQb4), d));
  }
#pragma unroll
  for (int e = 0; e < 16; ++e) q[e] = max(-8, min(7, q[e]));
}

// The butterflies of one tile of 32 * V consecutive elements held V per lane
// (lane l owns elements l * V .. l * V + V - 1).  A tile is one block when
// B >= 32 (V = B / 32: stages h < V inside a lane, h >= V between lanes
// l and l ^ (h / V)); when B < 32 each lane owns whole blocks (V = B, every
// stage inside the lane).  Stage order and arithmetic are those of the
// in-place transform: the lower element of each pair becomes a + b, the upper
// a - b, one IEEE rounding each.
template <int V>
__device__ __forceinline__ void hadamard_tile(float (&v)[V], int B, int lane) {
#pragma unroll
  for (int h = 1; h < V; h <<= 1)
#pragma unroll
    for (int i = 0; i < V; ++i)
      if ((i & h) == 0) {
        const float a = v[i], b = v[i + h];
        v[i] = __fadd_rn(a, b);
        v[i + h] = __fsub_rn(a, b);
      }
  for (int h = V; h < B; h <<= 1) {
    const int lm = h / V;  // partner lane distance
    const bool upper = (lane & lm) != 0;
#pragma unroll
    for (int i = 0; i < V; ++i) {
      const float o = __shfl_xor_sync(0xffffffffu, v[i], lm);
      v[i] = upper ? __fsub_rn(o, v[i]) : __fadd_rn(v[i], o);
    }
  }
}

// One CTA (kHbitThreads) per token row; blocks past M clear the split-K sums
// and blockIdx 0 the arrival counters of the GEMMs that follow, as
// quant_act_kernel does.  kPermute: codes in contraction order [M, ldq],
// ldq = K rounded up to 16 (zeros past K); otherwise natural order, ldq = K
// or K rounded up to 16 (then zeros past K as well).
// V > 0: the transform runs in registers, warps taking the row's tiles of
// 32 * V elements in turn; V = 0 (blocks of more than 2048): stage by stage
// over the row in shared memory, with a CTA barrier between stages.  Either
// way the transformed, scaled row lands in shared memory, gamma is the CTA
// maximum, and each thread turns 16-groups of it into codes.
template <bool kPermute, int V>
__global__ void __launch_bounds__(kHbitThreads) hbit_quant_kernel(const uint16_t* __restrict__ x, int M, int K,
                                                                  int B, float scale, int ldq, int8_t* __restrict__ q,
                                                                  float* __restrict__ gamma,
                                                                  int32_t* __restrict__ rowsum,
                                                                  uint32_t* __restrict__ cnt, int ncnt,
                                                                  float* __restrict__ zbuf, size_t zvec4) {
  extern __shared__ float s_v[];  // [K]: the transformed row
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
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint16_t* xr = x + static_cast<size_t>(row) * K;
  const bool vec_ok = (K % 8) == 0 && (reinterpret_cast<uintptr_t>(x) & 15u) == 0;
  uint32_t mx = 0u;  // max of the |xh| bit patterns (they order like the values)
  if constexpr (V > 0) {
    const int tile = 32 * V;
    const int tiles = (K + tile - 1) / tile;  // a partial last tile only when B < 32 (whole blocks per lane)
    for (int t = warp; t < tiles; t += kHbitThreads / 32) {
      const int k0 = t * tile + lane * V;
      float v[V];
      if constexpr (V % 8 == 0) {
        // B >= 256: K is a multiple of the tile, so the whole tile is in the row
        if (vec_ok) {
#pragma unroll
          for (int i = 0; i < V; i += 8) {
            const uint4 u = *reinterpret_cast<const uint4*>(xr + k0 + i);
            const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              v[i + 2 * e] = __uint_as_float(uw[e] << 16);
              v[i + 2 * e + 1] = __uint_as_float(uw[e] & 0xFFFF0000u);
            }
          }
        } else {
#pragma unroll
          for (int i = 0; i < V; ++i) v[i] = bf16_bits_to_f32(xr[k0 + i]);
        }
      } else {
#pragma unroll
        for (int i = 0; i < V; ++i) v[i] = k0 + i < K ? bf16_bits_to_f32(xr[k0 + i]) : 0.0f;
      }
      hadamard_tile<V>(v, B, lane);
#pragma unroll
      for (int i = 0; i < V; ++i) {
        v[i] = __fmul_rn(v[i], scale);
        if (k0 + i < K) mx = max(mx, __float_as_uint(fabsf(v[i])));
      }
      if constexpr (V % 4 == 0) {
        if (k0 < K)  // whole lane chunks: K is a multiple of B = 32 V here, or V = B < 32 divides K
#pragma unroll
          for (int i = 0; i < V; i += 4)
            *reinterpret_cast<float4*>(s_v + k0 + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
      } else {
#pragma unroll
        for (int i = 0; i < V; ++i)
          if (k0 + i < K) s_v[k0 + i] = v[i];
      }
    }
  } else {
    for (int k = threadIdx.x; k < K; k += blockDim.x) s_v[k] = bf16_bits_to_f32(xr[k]);
    __syncthreads();
    // stage by stage over the whole row (blocks start at multiples of B >= 2h,
    // so a pair never leaves its block)
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
    for (int k = threadIdx.x; k < K; k += blockDim.x) {
      const float h = __fmul_rn(s_v[k], scale);
      s_v[k] = h;
      mx = max(mx, __float_as_uint(fabsf(h)));
    }
  }
  mx = __reduce_max_sync(0xffffffffu, mx);
  if (lane == 0) s_max[warp] = mx;
  __syncthreads();
  mx = 0u;
#pragma unroll
  for (int w = 0; w < kHbitThreads / 32; ++w) mx = max(mx, s_max[w]);
  const float g = __uint_as_float(mx);
  const float d = __fadd_rn(g, kEps);
  const float c = __fmul_rn(kQb4, __frcp_rn(d));

  // 4-bit codes, one 16-wide k-group per thread and step
  int32_t sum = 0;
  int8_t* qr = q + static_cast<size_t>(row) * ldq;
  const int groups = (K + 15) / 16;
  for (int gi = threadIdx.x; gi < groups; gi += blockDim.x) {
    float v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = 16 * gi + i < K ? s_v[16 * gi + i] : 0.0f;
    int32_t cq[16];
    codes16_q7(v, c, d, cq);
    uint32_t cb[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      sum += cq[i];
      cb[i] = static_cast<uint32_t>(cq[i]) & 0xFFu;
    }
    if (kPermute) {
      // byte 4j + b <- k = 16 gi + 4b + j
      uint4 w;
      w.x = cb[0] | (cb[4] << 8) | (cb[8] << 16) | (cb[12] << 24);
      w.y = cb[1] | (cb[5] << 8) | (cb[9] << 16) | (cb[13] << 24);
      w.z = cb[2] | (cb[6] << 8) | (cb[10] << 16) | (cb[14] << 24);
      w.w = cb[3] | (cb[7] << 8) | (cb[11] << 16) | (cb[15] << 24);
      *reinterpret_cast<uint4*>(qr + 16 * gi) = w;
    } else if (16 * gi + 16 <= ldq && ((reinterpret_cast<uintptr_t>(qr) | (16u * gi)) & 15u) == 0) {
      uint4 w;
      w.x = cb[0] | (cb[1] << 8) | (cb[2] << 16) | (cb[3] << 24);
      w.y = cb[4] | (cb[5] << 8) | (cb[6] << 16) | (cb[7] << 24);
      w.z = cb[8] | (cb[9] << 8) | (cb[10] << 16) | (cb[11] << 24);
      w.w = cb[12] | (cb[13] << 8) | (cb[14] << 16) | (cb[15] << 24);
      *reinterpret_cast<uint4*>(qr + 16 * gi) = w;
    } else {
      for (int i = 0; i < 16 && 16 * gi + i < K; ++i) qr[16 * gi + i] = static_cast<int8_t>(cb[i]);
    }
  }
  sum = __reduce_add_sync(0xffffffffu, sum);
  if (lane == 0) s_sum[warp] = sum;
  __syncthreads();
  if (threadIdx.x == 0) {
    int32_t t = 0;
#pragma unroll
    for (int w = 0; w < kHbitThreads / 32; ++w) t += s_sum[w];
    if (gamma) gamma[row] = g;
    if (rowsum) rowsum[row] = t;
  }
}

// Register tile of a block size: V values per lane (0: shared-memory stages).
__host__ __device__ constexpr int hbit_vals_per_lane(int B) { return B < 32 ? B : (B <= 2048 ? B / 32 : 0); }

}  // namespace bl
