// gemv.cuh -- decode-regime (one token) BitLinear: a streaming GEMV over the
// 2-bit packed weights with the activation quantisation fused in.
//
// The 2B4T report (section 5.1, GPU Inference) moves packed ternary weights
// from HBM on chip, unpacks them and combines them with 8-bit activations;
// for one token the contraction is bound by those weight bytes.  Here every
// CTA quantises the single activation row into shared memory (gamma, codes
// in contraction order, their sum), while the weight loads it issued first
// are in flight.  A lane owns a fixed set of 64-weight chunks of a row; its
// activation codes for those chunks stay in registers for every row it
// visits.  With code = W_t + 1:
//     acc = sum_k q_k * W_t,k = sum_k q_k * code_k - sum_k q_k
// and sum_k q_k * code_k is formed four bytes at a time with an unsigned x
// signed dp4a on (word & (3 << 2j) per byte), whose partial sums carry a
// factor 4^j that is removed exactly at the end (every term is a multiple).
#pragma once
#include "quant_pack.cuh"

namespace bl {

constexpr int kGemvThreads = 256;

struct GemvArgs {
  const uint8_t* codes;  // dense codes, or N:M kept values
  const uint8_t* meta;   // N:M metadata (N:M kernel only)
  int64_t ld;            // row stride of codes/values (bytes)
  int64_t ld_meta;       // row stride of meta (bytes)
  int N, K;
  int C;                 // dense: 16-byte chunks per row; N:M: 128-weight units per row
  int nm_n, nm_m;
  const uint16_t* x;     // one bf16 row [K]
  const float* alpha;
  uint16_t* y;           // [N]
  int32_t* acc;          // [N] or null
  int tpr_log2;          // lanes per row = 1 << tpr_log2
  int passes;            // chunk passes (C > CPT << tpr_log2)
  int rows_base, rows_rem;  // CTA b owns rows_base (+1 if b < rows_rem) consecutive rows
};

// Exact round-half-to-even of RN(t / d) for |t / d| < 128, given inv = RN(1 / d):
// y = RN(t * inv) is within 2.3e-5 of RN(t / d); unless y sits within 2^-15 of
// a half-integer both round to the same integer, otherwise the quotient is
// formed exactly.
__device__ __forceinline__ int32_t act_code_fast(float v, float d, float inv) {
  const float t = __fmul_rn(v, kQb);
  const float yq = __fmul_rn(t, inv);
  const float fr = yq - floorf(yq);
  int32_t c;
  if (fabsf(fr - 0.5f) < 3.0517578125e-05f)
    c = __float2int_rn(__fdiv_rn(t, d));
  else
    c = __float2int_rn(yq);
  return max(-128, min(127, c));
}

// Quantises the activation row into shared memory (contraction order, 4 * C16
// entries of 16 codes, zero past K) and returns gamma and sum(q) to every thread.
__device__ __forceinline__ void gemv_quantise_row(const uint16_t* __restrict__ x, int K, int groups_alloc,
                                                  uint4* s_act, float* red_f, int32_t* red_i, float& gamma_out,
                                                  int32_t& qsum_out) {
  const bool vec_ok = (K % 8) == 0;
  float mx = 0.0f;
  if (vec_ok) {
    for (int k = threadIdx.x * 8; k < K; k += blockDim.x * 8) {
      const uint4 a = *reinterpret_cast<const uint4*>(x + k);
      const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        mx = fmaxf(mx, fabsf(__uint_as_float(w[i] << 16)));
        mx = fmaxf(mx, fabsf(__uint_as_float(w[i] & 0xFFFF0000u)));
      }
    }
  } else {
    for (int k = threadIdx.x; k < K; k += blockDim.x) mx = fmaxf(mx, fabsf(bf16_bits_to_f32(x[k])));
  }
  mx = block_reduce(mx, MaxOp(), red_f, 0.0f);
  const float d = __fadd_rn(mx, kEps);
  const float inv = __frcp_rn(d);
  int32_t sum = 0;
  const int groups = (K + 15) / 16;
  for (int g = threadIdx.x; g < groups_alloc; g += blockDim.x) {
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    if (g < groups) {
      const int k0 = g * 16;
      float v[16];
      load16_bf16(x, k0, K, vec_ok, v);
      int32_t c[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        c[i] = (k0 + i < K) ? act_code_fast(v[i], d, inv) : 0;
        sum += c[i];
      }
      permute16(c, w);
    }
    s_act[g] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  sum = block_reduce(sum, AddI(), red_i, 0);  // also orders the s_act stores before their reads
  gamma_out = mx;
  qsum_out = sum;
}

__device__ __forceinline__ void gemv_store(const GemvArgs& a, int row, int32_t total, float s) {
  if (a.acc) a.acc[row] = total;
  const __nv_bfloat16 h = __float2bfloat16_rn(__fmul_rn(static_cast<float>(total), s));
  a.y[row] = *reinterpret_cast<const uint16_t*>(&h);
}

__device__ __forceinline__ int32_t group_sum(int32_t v, int tpr) {
  for (int o = tpr >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Dot of one packed 32-bit weight word (16 codes) with its 4 activation words.
__device__ __forceinline__ void dot_word(uint32_t wd, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         int32_t& s0, int32_t& s1, int32_t& s2, int32_t& s3) {
  s0 = dp4a_us(wd & 0x03030303u, a0, s0);
  s1 = dp4a_us(wd & 0x0C0C0C0Cu, a1, s1);
  s2 = dp4a_us(wd & 0x30303030u, a2, s2);
  s3 = dp4a_us(wd & 0xC0C0C0C0u, a3, s3);
}

// ------------------------------------------------------------------ dense M = 1
template <int CPT, int RMAX>
__global__ void __launch_bounds__(kGemvThreads) gemv_m1_kernel(const GemvArgs a) {
  extern __shared__ uint4 s_act[];  // 4 * C entries
  __shared__ float red_f[32];
  __shared__ int32_t red_i[32];
  pdl_launch_dependents();
  const int tpr = 1 << a.tpr_log2;
  const int sub = threadIdx.x & (tpr - 1);
  const int grp = threadIdx.x >> a.tpr_log2;
  const int ngrp = blockDim.x >> a.tpr_log2;
  const int b = blockIdx.x;
  const int r0 = b * a.rows_base + min(b, a.rows_rem);
  const int nrows = a.rows_base + (b < a.rows_rem ? 1 : 0);

  // Weight loads of the first pass go out before anything else.
  uint4 w[RMAX][CPT];
  auto load_pass = [&](int pass) {
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
      const int lr = grp + r * ngrp;
#pragma unroll
      for (int c = 0; c < CPT; ++c) {
        const int ch = pass * CPT * tpr + sub + c * tpr;
        if (lr < nrows && ch < a.C)
          w[r][c] = ldg_stream_v4(a.codes + static_cast<int64_t>(r0 + lr) * a.ld + static_cast<int64_t>(ch) * 16);
        else
          w[r][c] = make_uint4(0x55555555u, 0x55555555u, 0x55555555u, 0x55555555u);
      }
    }
  };
  load_pass(0);

  pdl_wait_primary();  // x may come from the preceding kernel
  float gamma;
  int32_t qsum;
  gemv_quantise_row(a.x, a.K, 4 * a.C, s_act, red_f, red_i, gamma, qsum);
  const float s = __fdiv_rn(__fmul_rn(*a.alpha, gamma), kQb);

  int32_t part[RMAX];
#pragma unroll
  for (int r = 0; r < RMAX; ++r) part[r] = 0;
  for (int pass = 0; pass < a.passes; ++pass) {
    if (pass > 0) load_pass(pass);
    uint32_t A[CPT][16];
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      const int ch = pass * CPT * tpr + sub + c * tpr;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 v = ch < a.C ? s_act[4 * ch + i] : make_uint4(0u, 0u, 0u, 0u);
        A[c][4 * i + 0] = v.x;
        A[c][4 * i + 1] = v.y;
        A[c][4 * i + 2] = v.z;
        A[c][4 * i + 3] = v.w;
      }
    }
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
      int32_t s0 = 0, s1 = 0, s2 = 0, s3 = 0;
#pragma unroll
      for (int c = 0; c < CPT; ++c) {
        dot_word(w[r][c].x, A[c][0], A[c][1], A[c][2], A[c][3], s0, s1, s2, s3);
        dot_word(w[r][c].y, A[c][4], A[c][5], A[c][6], A[c][7], s0, s1, s2, s3);
        dot_word(w[r][c].z, A[c][8], A[c][9], A[c][10], A[c][11], s0, s1, s2, s3);
        dot_word(w[r][c].w, A[c][12], A[c][13], A[c][14], A[c][15], s0, s1, s2, s3);
      }
      part[r] += s0 + (s1 >> 2) + (s2 >> 4) + (s3 >> 6);
    }
  }
#pragma unroll
  for (int r = 0; r < RMAX; ++r) {
    const int v = group_sum(part[r], tpr);
    const int lr = grp + r * ngrp;
    if (sub == 0 && lr < nrows) gemv_store(a, r0 + lr, v - qsum, s);
  }
}

// ------------------------------------------------------------------ N:M M = 1
// Expands kept codes + metadata of 16 dense weights into one dense 2-bit code
// word (pruned positions get code 01, the zero weight).
__device__ __forceinline__ uint32_t nm24_dense_word(uint32_t meta16, uint32_t vals16) {
  uint32_t dense = 0x55555555u;
#pragma unroll
  for (int t = 0; t < 4; ++t) {  // four 2:4 blocks
    const uint32_t nib = (meta16 >> (4 * t)) & 0xFu;
    const uint32_t i0 = nib & 3u, i1 = nib >> 2;
    const uint32_t c0 = (vals16 >> (4 * t)) & 3u, c1 = (vals16 >> (4 * t + 2)) & 3u;
    dense ^= ((c0 ^ 1u) << (8 * t + 2 * i0)) ^ ((c1 ^ 1u) << (8 * t + 2 * i1));
  }
  return dense;
}

// One n:8 block: inserts code 01 at every pruned position, in increasing order.
__device__ __forceinline__ uint32_t n8_dense_block(uint32_t mask8, uint32_t kept) {
  uint32_t x = kept;
  uint32_t pr = (~mask8) & 0xFFu;
  while (pr) {
    const int j = __ffs(pr) - 1;
    pr &= pr - 1;
    const uint32_t lowm = (1u << (2 * j)) - 1u;
    const uint32_t low = x & lowm;
    x = low | (1u << (2 * j)) | ((x ^ low) << 2);
  }
  return x & 0xFFFFu;
}

// nbits (<= 32) bits starting at an even bit offset of a 16-byte aligned row;
// the following word is read only when the field straddles it.
__device__ __forceinline__ uint32_t load_bits(const uint8_t* base, int64_t bit, int nbits) {
  const int64_t wi = bit >> 5;
  const int sh = static_cast<int>(bit & 31);
  const uint32_t* p = reinterpret_cast<const uint32_t*>(base);
  const uint32_t lo = __ldg(p + wi);
  if (sh == 0) return lo;
  uint32_t v = lo >> sh;
  if (sh + nbits > 32) v |= __ldg(p + wi + 1) << (32 - sh);
  return v;
}

// A lane owns 128-weight units (2:4: 32 blocks, n:8: 16 blocks) of a row.
__global__ void __launch_bounds__(kGemvThreads) gemv_nm_m1_kernel(const GemvArgs a) {
  extern __shared__ uint4 s_act[];
  __shared__ float red_f[32];
  __shared__ int32_t red_i[32];
  pdl_launch_dependents();
  const int tpr = 1 << a.tpr_log2;
  const int sub = threadIdx.x & (tpr - 1);
  const int grp = threadIdx.x >> a.tpr_log2;
  const int ngrp = blockDim.x >> a.tpr_log2;
  const int b = blockIdx.x;
  const int r0 = b * a.rows_base + min(b, a.rows_rem);
  const int nrows = a.rows_base + (b < a.rows_rem ? 1 : 0);

  pdl_wait_primary();
  float gamma;
  int32_t qsum;
  gemv_quantise_row(a.x, a.K, 8 * a.C, s_act, red_f, red_i, gamma, qsum);
  const float s = __fdiv_rn(__fmul_rn(*a.alpha, gamma), kQb);
  const int n = a.nm_n, m = a.nm_m;
  const int blocks_per_row = a.K / m;

  const int iters = (nrows + ngrp - 1) / ngrp;
  for (int it = 0; it < iters; ++it) {
    const int lr = grp + it * ngrp;
    const bool valid = lr < nrows;
    int32_t s0 = 0, s1 = 0, s2 = 0, s3 = 0;
    if (valid) {
      const int64_t row = r0 + lr;
      const uint8_t* vrow = a.codes + row * a.ld;
      const uint8_t* mrow = a.meta + row * a.ld_meta;
      for (int u = sub; u < a.C; u += tpr) {
        // 8 groups of 16 dense weights per unit
        const uint4 mq = *reinterpret_cast<const uint4*>(mrow + static_cast<int64_t>(u) * 16);
        const uint32_t mw[4] = {mq.x, mq.y, mq.z, mq.w};
#pragma unroll
        for (int gi = 0; gi < 8; ++gi) {
          const int g = u * 8 + gi;  // 16-weight group index in the row
          uint32_t dense;
          if (m == 4) {
            // group gi: blocks 4gi .. 4gi+3, meta nibbles 4gi.., kept codes 8gi..
            dense = 0x55555555u;
            if (g * 4 < blocks_per_row) {  // K is a multiple of 4, so a group is whole or absent
              const uint32_t meta16 = (mw[gi >> 1] >> (16 * (gi & 1))) & 0xFFFFu;
              const uint32_t vals16 = load_bits(vrow, static_cast<int64_t>(g) * 16, 16) & 0xFFFFu;
              dense = nm24_dense_word(meta16, vals16);
            }
          } else {
            // group gi: blocks 2gi, 2gi+1, meta bytes 2gi, 2gi+1, kept codes n per block
            const int blk = g * 2;
            const uint32_t m0 = (mw[gi >> 1] >> (16 * (gi & 1))) & 0xFFu;
            const uint32_t m1 = (mw[gi >> 1] >> (16 * (gi & 1) + 8)) & 0xFFu;
            const uint32_t fmask = (1u << (2 * n)) - 1u;
            dense = 0x55555555u;
            if (blk + 1 < blocks_per_row) {
              const uint32_t kv = load_bits(vrow, static_cast<int64_t>(blk) * n * 2, 4 * n);
              dense = n8_dense_block(m0, kv & fmask) | (n8_dense_block(m1, (kv >> (2 * n)) & fmask) << 16);
            } else if (blk < blocks_per_row) {
              const uint32_t kv = load_bits(vrow, static_cast<int64_t>(blk) * n * 2, 2 * n);
              dense = n8_dense_block(m0, kv & fmask) | (0x5555u << 16);
            }
          }
          const uint4 av = s_act[g];
          dot_word(dense, av.x, av.y, av.z, av.w, s0, s1, s2, s3);
        }
      }
    }
    int32_t part = s0 + (s1 >> 2) + (s2 >> 4) + (s3 >> 6);
    part = group_sum(part, tpr);
    if (valid && sub == 0) gemv_store(a, r0 + lr, part - qsum, s);
  }
}

}  // namespace bl
