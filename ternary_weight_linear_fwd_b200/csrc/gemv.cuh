// gemv.cuh -- decode-regime (one token) BitLinear: a streaming GEMV over the
// 2-bit packed weights with the activation quantisation fused in.
//
// The 2B4T report (section 5.1, GPU Inference) moves packed ternary weights
// from HBM on chip, unpacks them and combines them with 8-bit activations;
// for one token the contraction is bound by those weight bytes.  Here every
// CTA first hands its contiguous weight rows to the tensor-copy engine (TMA
// tile loads into shared memory, issued before griddepcontrol.wait, so under
// programmatic dependent launch the copy overlaps the preceding kernel), then
// quantises the single activation row into shared memory (gamma, codes in
// contraction order, per-chunk code sums) while the copy lands, and finally
// splits the (64-weight chunk, row) products evenly over all its threads.
// With code = W_t + 1:
//     acc = sum_k q_k * W_t,k = sum_k q_k * code_k - sum_k q_k
// and sum_k q_k * code_k is formed four bytes at a time with an unsigned x
// signed dp4a on (word & (3 << 2j) per byte), whose partial sums carry a
// factor 4^j that is removed exactly at the end (every term is a multiple).
#pragma once
#include "quant_pack.cuh"

namespace bl {

constexpr int kGemvThreads = 512;

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
  int32_t* status;       // device status word
};

// Quantises the single activation row into shared memory: s_act[slot(g)]
// holds the 16 codes of k-group g in contraction order (byte 4j + b <- k =
// 16g + 4b + j), for g < groups_alloc (zero past K), where
// slot(g) = (g % 4) * (groups_alloc / 4) + g / 4 puts the four groups of one
// 64-weight chunk a quarter of the array apart, so lanes reading consecutive
// chunks hit consecutive 16-byte words; s_hsum[h] is the sum of the 8 codes of
// half h (chunk_sum adds the eight of a chunk).  Each thread handles 8-element
// halves h = tid, tid + nthr, ...: one 16-byte load, 8 codes, four 16-bit
// stores (bytes 2*(h%2), 2*(h%2)+1 of words 0..3) and its code sum.  One
// barrier publishes the per-warp maxima, one the codes.  Returns gamma = max |x|.
constexpr int kHalvesInRegs = 2;  // halves per thread kept in registers (K <= 8192 at 512 threads)

__device__ __forceinline__ float quantise_row_smem(const uint16_t* __restrict__ x, int K, int groups_alloc,
                                                   uint4* s_act, int32_t* s_hsum, float* s_red) {
  const bool vec_ok = (K % 8) == 0;
  const int nthr = blockDim.x;
  const int halves = (K + 7) / 8;
  const int halves_alloc = 2 * groups_alloc;
  const int trips = (halves_alloc + nthr - 1) / nthr;
  uint32_t v[kHalvesInRegs][4];
  float mx = 0.0f;
#pragma unroll
  for (int j = 0; j < kHalvesInRegs; ++j) {
    const int h = threadIdx.x + j * nthr;
    if (h < halves) {
      load8_raw(x, h * 8, K, vec_ok, v[j]);
    } else {
      v[j][0] = v[j][1] = v[j][2] = v[j][3] = 0u;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
      mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(v[j][i] << 16)), fabsf(__uint_as_float(v[j][i] & 0xFFFF0000u))));
  }
  for (int h = threadIdx.x + kHalvesInRegs * nthr; h < halves; h += nthr) {
    uint32_t t[4];
    load8_raw(x, h * 8, K, vec_ok, t);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(t[i] << 16)), fabsf(__uint_as_float(t[i] & 0xFFFF0000u))));
  }
  // |x| >= 0, whose bit patterns order like the values: one integer warp reduction
  mx = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(mx)));
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = mx;
  __syncthreads();
  mx = (threadIdx.x & 31) < (nthr >> 5) ? s_red[threadIdx.x & 31] : 0.0f;
  mx = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(mx)));
  const float d = __fadd_rn(mx, kEps);
  const float c = __fmul_rn(kQb, __frcp_rn(d));
  const int quarter = groups_alloc >> 2;
  auto emit = [&](const uint32_t (&raw)[4], int h) {
    uint32_t b[8];
    codes8(raw, c, d, b);
    const uint32_t lo = __byte_perm(b[0], b[1], 0x0040), hi = __byte_perm(b[2], b[3], 0x0040);
    const uint32_t lo2 = __byte_perm(b[4], b[5], 0x0040), hi2 = __byte_perm(b[6], b[7], 0x0040);
    const uint32_t p0 = __byte_perm(lo, hi, 0x5410), p1 = __byte_perm(lo2, hi2, 0x5410);  // codes 0..3, 4..7
    if (h < halves_alloc) {
      s_hsum[h] = __dp4a(static_cast<int>(p1), 0x01010101, __dp4a(static_cast<int>(p0), 0x01010101, 0));
      const int g = h >> 1, half = h & 1;
      const int sl = (g & 3) * quarter + (g >> 2);
      uint16_t* dst = reinterpret_cast<uint16_t*>(s_act + sl) + half;
      // word j gets codes j and j + 4 of this half in its bytes 2*half, 2*half + 1
      dst[0] = static_cast<uint16_t>(__byte_perm(b[0], b[4], 0x0040));
      dst[2] = static_cast<uint16_t>(__byte_perm(b[1], b[5], 0x0040));
      dst[4] = static_cast<uint16_t>(__byte_perm(b[2], b[6], 0x0040));
      dst[6] = static_cast<uint16_t>(__byte_perm(b[3], b[7], 0x0040));
    }
  };
#pragma unroll
  for (int j = 0; j < kHalvesInRegs; ++j)
    if (j < trips) emit(v[j], threadIdx.x + j * nthr);
  for (int j = kHalvesInRegs; j < trips; ++j) {
    const int h = threadIdx.x + j * nthr;
    uint32_t raw[4] = {0u, 0u, 0u, 0u};
    if (h < halves) load8_raw(x, h * 8, K, vec_ok, raw);
    emit(raw, h);
  }
  __syncthreads();
  return mx;
}

__device__ __forceinline__ void gemv_store(uint16_t* y, int32_t* acc, int row, int32_t total, float s) {
  if (acc) acc[row] = total;
  const __nv_bfloat16 h = __float2bfloat16_rn(__fmul_rn(static_cast<float>(total), s));
  y[row] = *reinterpret_cast<const uint16_t*>(&h);
}

// Sum of the 64 codes of chunk ch (eight half sums; s_hsum 16-byte aligned).
__device__ __forceinline__ int32_t chunk_sum(const int32_t* s_hsum, int ch) {
  const int4 a = reinterpret_cast<const int4*>(s_hsum)[2 * ch];
  const int4 b = reinterpret_cast<const int4*>(s_hsum)[2 * ch + 1];
  return (a.x + a.y) + (a.z + a.w) + ((b.x + b.y) + (b.z + b.w));
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
// A CTA owns a contiguous range of rows.  One thread issues one TMA tile load
// per 128-byte stripe of those rows (box {128 bytes, rows}) with the 128-byte
// swizzle, so chunk ch of row r sits at stripe ch / 8, line r, 16-byte slot
// (ch % 8) ^ (r % 8): lanes reading one chunk of consecutive rows never share
// a bank.  The contraction is a flat list of (chunk, row pair) units, row pair
// fastest, spread evenly over all threads; a unit is one 64-weight chunk of
// two rows and adds its partial sums (minus the chunk's share of sum(q)) into
// the rows' shared accumulators.

__host__ __device__ __forceinline__ int gemv_stripes(int64_t ld) { return static_cast<int>((ld + 127) / 128); }
__host__ __device__ __forceinline__ int gemv_stripe_bytes(int rows_box) { return (rows_box * 128 + 1023) & ~1023; }

__host__ __device__ __forceinline__ size_t gemv_smem_bytes(int rows_box, int64_t ld, int C) {
  return 1024 /* alignment */ + static_cast<size_t>(gemv_stripes(ld)) * gemv_stripe_bytes(rows_box) +
         static_cast<size_t>(C) * 4 * 16 + static_cast<size_t>(C) * 8 * 4 + static_cast<size_t>(rows_box) * 4;
}

// Weight chunk ch of local row r in the swizzled stripes.
__device__ __forceinline__ uint4 gemv_wchunk(const uint8_t* s_w, int stripe_bytes, int r, int ch) {
  return *reinterpret_cast<const uint4*>(s_w + (ch >> 3) * stripe_bytes + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
}

// Up to kGemvGroup matrices that multiply the same activation row (and have
// the same K) run in one launch: CTAs [cta_begin, next cta_begin) belong to
// one matrix.  Each CTA quantises x for itself, so grouping saves the launches
// and the repeated quantisation, and changes no result.
constexpr int kGemvGroup = 4;

struct GemvMat {
  const float* alpha;
  uint16_t* y;       // [N]
  int32_t* acc;      // [N] or null
  int rows_base, rows_rem;  // local CTA b owns rows_base (+1 if b < rows_rem) consecutive rows
  int cta_begin;
};

struct GemvDense {
  GemvMat mat[kGemvGroup];
  const uint16_t* x;  // one bf16 row [K]
  int32_t* status;
  int64_t ld;
  int K, C, rows_box, count;
};

// The tensor maps (per matrix: uint8 [N, ld], box {128, rows_box}, 128-byte
// swizzle) are separate kernel parameters, and every parameter is read at a
// fixed offset: the matrix of this CTA is selected into registers.
__global__ void __launch_bounds__(kGemvThreads) gemv_dense_kernel(const __grid_constant__ CUtensorMap map0,
                                                                  const __grid_constant__ CUtensorMap map1,
                                                                  const __grid_constant__ CUtensorMap map2,
                                                                  const __grid_constant__ CUtensorMap map3,
                                                                  const GemvDense g) {
  extern __shared__ uint8_t s_raw[];
  __shared__ uint64_t s_bar;
  __shared__ float s_red[32];
  int mi = 0;
#pragma unroll
  for (int i = 1; i < kGemvGroup; ++i)
    if (i < g.count && static_cast<int>(blockIdx.x) >= g.mat[i].cta_begin) mi = i;
  GemvMat mt = g.mat[0];
#pragma unroll
  for (int i = 1; i < kGemvGroup; ++i)
    if (i == mi) mt = g.mat[i];
  const CUtensorMap* map = mi == 0 ? &map0 : mi == 1 ? &map1 : mi == 2 ? &map2 : &map3;
  const int b = blockIdx.x - mt.cta_begin;
  const int r0 = b * mt.rows_base + min(b, mt.rows_rem);
  const int nrows = mt.rows_base + (b < mt.rows_rem ? 1 : 0);
  const int C = g.C;
  const int rows_box = g.rows_box;
  const int stripes = gemv_stripes(g.ld);
  const int stripe_bytes = gemv_stripe_bytes(rows_box);
  // offset arithmetic on the shared array keeps every derived pointer in the shared window
  uint8_t* s_w = s_raw + ((1024u - (smem_u32(s_raw) & 1023u)) & 1023u);
  uint4* s_act = reinterpret_cast<uint4*>(s_w + static_cast<size_t>(stripes) * stripe_bytes);
  int32_t* s_hsum = reinterpret_cast<int32_t*>(s_act + 4 * C);  // 8 * C half sums
  int32_t* s_acc = s_hsum + 8 * C;

  // The weights (and alpha, which belongs to them) do not depend on the
  // preceding kernel: their copies start first.
  if (threadIdx.x == 0) {
    mbar_init(&s_bar, 1);
    fence_mbar_init();
    tma_prefetch_desc(map);
    mbar_arrive_expect_tx(&s_bar, static_cast<uint32_t>(stripes) * 128u * static_cast<uint32_t>(rows_box));
    const uint64_t pol = l2_policy_evict_first();
    for (int st = 0; st < stripes; ++st) tma_load_2d_hint(s_w + st * stripe_bytes, map, st * 128, r0, &s_bar, pol);
  }
  const float alpha = *mt.alpha;
  for (int r = threadIdx.x; r < nrows; r += blockDim.x) s_acc[r] = 0;
  __syncthreads();

  pdl_wait_primary();  // x may come from the preceding kernel
  const float gamma = quantise_row_smem(g.x, g.K, 4 * C, s_act, s_hsum, s_red);
  // The next kernel may start now: its weight copies then stream while this
  // one contracts, and no longer delay this kernel's read of x.
  pdl_launch_dependents();
  const float s = __fdiv_rn(__fmul_rn(alpha, gamma), kQb);
  const bool landed = mbar_wait(&s_bar, 0);
  if (!landed && threadIdx.x == 0) *g.status = kDevTimeoutProducer;

  if (landed) {
    // units (chunk, row pair), row pair fastest: the lanes of a warp read one
    // activation chunk (one shared-memory broadcast) for up to 64 rows
    const int nthr = blockDim.x;
    const int half = (nrows + 1) >> 1;  // pair p covers rows p and p + half
    const int total = half * C;
    const int dq = nthr / half, dr = nthr % half;
    int ch = threadIdx.x / half, p = threadIdx.x % half;
    for (int u = threadIdx.x; u < total; u += nthr) {
      const int r2 = p + half < nrows ? p + half : p;  // an odd last pair reads row p twice
      const uint4 wa = gemv_wchunk(s_w, stripe_bytes, p, ch);
      const uint4 wb = gemv_wchunk(s_w, stripe_bytes, r2, ch);
      const uint4 q0 = s_act[ch], q1 = s_act[C + ch], q2 = s_act[2 * C + ch], q3 = s_act[3 * C + ch];
      const int32_t cs = chunk_sum(s_hsum, ch);
      int32_t a0 = 0, a1 = 0, a2 = 0, a3 = 0, b0 = 0, b1 = 0, b2 = 0, b3 = 0;
      dot_word(wa.x, q0.x, q0.y, q0.z, q0.w, a0, a1, a2, a3);
      dot_word(wb.x, q0.x, q0.y, q0.z, q0.w, b0, b1, b2, b3);
      dot_word(wa.y, q1.x, q1.y, q1.z, q1.w, a0, a1, a2, a3);
      dot_word(wb.y, q1.x, q1.y, q1.z, q1.w, b0, b1, b2, b3);
      dot_word(wa.z, q2.x, q2.y, q2.z, q2.w, a0, a1, a2, a3);
      dot_word(wb.z, q2.x, q2.y, q2.z, q2.w, b0, b1, b2, b3);
      dot_word(wa.w, q3.x, q3.y, q3.z, q3.w, a0, a1, a2, a3);
      dot_word(wb.w, q3.x, q3.y, q3.z, q3.w, b0, b1, b2, b3);
      // every partial sum s_j is a multiple of 4^j, so the shifts are exact
      atomicAdd(&s_acc[p], a0 + (a1 >> 2) + (a2 >> 4) + (a3 >> 6) - cs);
      if (p + half < nrows) atomicAdd(&s_acc[p + half], b0 + (b1 >> 2) + (b2 >> 4) + (b3 >> 6) - cs);
      p += dr;
      ch += dq;
      if (p >= half) {
        p -= half;
        ++ch;
      }
    }
  }
  __syncthreads();
  if (landed)
    for (int rr = threadIdx.x; rr < nrows; rr += blockDim.x) gemv_store(mt.y, mt.acc, r0 + rr, s_acc[rr], s);
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
  extern __shared__ uint4 s_dyn[];
  uint4* s_act = s_dyn;                                            // 8 * C entries
  int32_t* s_hsum = reinterpret_cast<int32_t*>(s_dyn + 8 * a.C);   // 16 * C half sums
  __shared__ float s_red[32];
  pdl_launch_dependents();
  const int tpr = 1 << a.tpr_log2;
  const int sub = threadIdx.x & (tpr - 1);
  const int grp = threadIdx.x >> a.tpr_log2;
  const int ngrp = blockDim.x >> a.tpr_log2;
  const int b = blockIdx.x;
  const int r0 = b * a.rows_base + min(b, a.rows_rem);
  const int nrows = a.rows_base + (b < a.rows_rem ? 1 : 0);

  pdl_wait_primary();
  const float gamma = quantise_row_smem(a.x, a.K, 8 * a.C, s_act, s_hsum, s_red);
  const float s = __fdiv_rn(__fmul_rn(*a.alpha, gamma), kQb);
  int32_t qsum = 0;  // this lane's share of sum(q): the two 64-weight chunks of each of its units
  for (int u = sub; u < a.C; u += tpr) qsum += chunk_sum(s_hsum, 2 * u) + chunk_sum(s_hsum, 2 * u + 1);
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
          const uint4 av = s_act[(g & 3) * (2 * a.C) + (g >> 2)];
          dot_word(dense, av.x, av.y, av.z, av.w, s0, s1, s2, s3);
        }
      }
    }
    int32_t part = s0 + (s1 >> 2) + (s2 >> 4) + (s3 >> 6) - qsum;
    part = group_sum(part, tpr);
    if (valid && sub == 0) gemv_store(a.y, a.acc, r0 + lr, part, s);
  }
}

}  // namespace bl
