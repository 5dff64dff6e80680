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
// contraction order, their sum) while the copy lands, and finally splits the
// (64-weight chunk, row) products evenly over all its threads.
// With code = W_t + 1:
//     acc = sum_k q_k * W_t,k = sum_k q_k * code_k - sum_k q_k
// where sum_k q_k is the same for every row (formed once, with the codes),
// and sum_k q_k * code_k is formed four bytes at a time with an unsigned x
// signed dp4a on (word & (3 << 2j) per byte), whose partial sums carry a
// factor 4^j that is removed exactly at the end (every term is a multiple).
#pragma once
#include "quant_pack.cuh"

namespace bl {

constexpr int kGemvThreads = 512;


// Quantises the single activation row into shared memory: s_act[slot(g)]
// holds the 16 codes of k-group g in contraction order (byte 4j + b <- k =
// 16g + 4b + j), for g < groups_alloc (zero past K), where
// slot(g) = (g % 4) * (groups_alloc / 4) + g / 4 puts the four groups of one
// 64-weight chunk a quarter of the array apart, so lanes reading consecutive
// chunks hit consecutive 16-byte words.  *s_qsum (zeroed by the caller before
// a barrier that precedes this call) receives the sum of all codes.  Each
// thread handles 8-element halves h = tid, tid + nthr, ...: one 16-byte load,
// 8 codes and four 16-bit stores (bytes 2*(h%2), 2*(h%2)+1 of words 0..3).
// One barrier publishes the per-warp maxima, one the codes and their sum.
// Returns gamma = max |x|.
constexpr int kHalvesInRegs = 2;  // halves per thread kept in registers (K <= 8192 at 512 threads)

__device__ __forceinline__ float quantise_row_smem(const uint16_t* __restrict__ x, int K, int groups_alloc,
                                                   uint4* s_act, int32_t* s_qsum, float* s_red) {
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
  int32_t qsum = 0;
  auto emit = [&](const uint32_t (&raw)[4], int h) {
    uint32_t b[8];
    codes8(raw, c, d, b);
    const uint32_t lo = __byte_perm(b[0], b[1], 0x0040), hi = __byte_perm(b[2], b[3], 0x0040);
    const uint32_t lo2 = __byte_perm(b[4], b[5], 0x0040), hi2 = __byte_perm(b[6], b[7], 0x0040);
    const uint32_t p0 = __byte_perm(lo, hi, 0x5410), p1 = __byte_perm(lo2, hi2, 0x5410);  // codes 0..3, 4..7
    if (h < halves_alloc) {
      qsum = __dp4a(static_cast<int>(p1), 0x01010101, __dp4a(static_cast<int>(p0), 0x01010101, qsum));
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
  qsum = __reduce_add_sync(0xffffffffu, qsum);
  if ((threadIdx.x & 31) == 0) atomicAdd(s_qsum, qsum);
  __syncthreads();
  return mx;
}

// quantise_row_smem with RMSNorm first (weight s_g[K] already in shared
// memory): r = RN32(1 / sqrt(RN32(sum x^2 / K) + eps)) with the sum (one
// fixed-order reduction over the CTA), the root and the quotient in fp64;
// the codes are those of xn = RN(RN(x * r) * g), which is never stored.
__device__ __forceinline__ float quantise_row_smem_norm(const uint16_t* __restrict__ x, int K, int groups_alloc,
                                                        uint4* s_act, int32_t* s_qsum, float* s_red, double* s_redd,
                                                        const float* s_g, float eps) {
  const bool vec_ok = (K % 8) == 0;
  const int nthr = blockDim.x;
  const int halves = (K + 7) / 8;
  const int halves_alloc = 2 * groups_alloc;
  const int trips = (halves_alloc + nthr - 1) / nthr;
  uint32_t v[kHalvesInRegs][4];
  double ss = 0.0;
#pragma unroll
  for (int j = 0; j < kHalvesInRegs; ++j) {
    const int h = threadIdx.x + j * nthr;
    if (h < halves) {
      load8_raw(x, h * 8, K, vec_ok, v[j]);
    } else {
      v[j][0] = v[j][1] = v[j][2] = v[j][3] = 0u;
    }
    ss = sumsq8(v[j], ss);
  }
  for (int h = threadIdx.x + kHalvesInRegs * nthr; h < halves; h += nthr) {
    uint32_t t[4];
    load8_raw(x, h * 8, K, vec_ok, t);
    ss = sumsq8(t, ss);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) s_redd[threadIdx.x >> 5] = ss;
  __syncthreads();
  ss = 0.0;
  for (int w = 0; w < (nthr >> 5); ++w) ss += s_redd[w];
  const float ms = __double2float_rn(__ddiv_rn(ss, static_cast<double>(K)));
  const float rn = __double2float_rn(__ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(static_cast<double>(ms), static_cast<double>(eps)))));
  // xn of half h (zero past K)
  auto norm8 = [&](const uint32_t (&raw)[4], int h, float (&xn)[8]) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int k = 8 * h + e;
      const float xv = __uint_as_float((e & 1) ? (raw[e >> 1] & 0xFFFF0000u) : (raw[e >> 1] << 16));
      xn[e] = k < K ? __fmul_rn(__fmul_rn(xv, rn), s_g[k]) : 0.0f;
    }
  };
  float mx = 0.0f;
#pragma unroll
  for (int j = 0; j < kHalvesInRegs; ++j) {
    const int h = threadIdx.x + j * nthr;
    if (h < halves) {
      float xn[8];
      norm8(v[j], h, xn);
#pragma unroll
      for (int e = 0; e < 8; ++e) mx = fmaxf(mx, fabsf(xn[e]));
    }
  }
  for (int h = threadIdx.x + kHalvesInRegs * nthr; h < halves; h += nthr) {
    uint32_t t[4];
    load8_raw(x, h * 8, K, vec_ok, t);
    float xn[8];
    norm8(t, h, xn);
#pragma unroll
    for (int e = 0; e < 8; ++e) mx = fmaxf(mx, fabsf(xn[e]));
  }
  mx = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(mx)));
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = mx;
  __syncthreads();
  mx = (threadIdx.x & 31) < (nthr >> 5) ? s_red[threadIdx.x & 31] : 0.0f;
  mx = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(mx)));
  const float d = __fadd_rn(mx, kEps);
  const float c = __fmul_rn(kQb, __frcp_rn(d));
  const int quarter = groups_alloc >> 2;
  int32_t qsum = 0;
  auto emit = [&](const uint32_t (&raw)[4], int h) {
    float xn[8];
    norm8(raw, h, xn);
    uint32_t b[8];
    codes8f(xn, c, d, b);
    const uint32_t lo = __byte_perm(b[0], b[1], 0x0040), hi = __byte_perm(b[2], b[3], 0x0040);
    const uint32_t lo2 = __byte_perm(b[4], b[5], 0x0040), hi2 = __byte_perm(b[6], b[7], 0x0040);
    const uint32_t p0 = __byte_perm(lo, hi, 0x5410), p1 = __byte_perm(lo2, hi2, 0x5410);
    if (h < halves_alloc) {
      qsum = __dp4a(static_cast<int>(p1), 0x01010101, __dp4a(static_cast<int>(p0), 0x01010101, qsum));
      const int g = h >> 1, half = h & 1;
      const int sl = (g & 3) * quarter + (g >> 2);
      uint16_t* dst = reinterpret_cast<uint16_t*>(s_act + sl) + half;
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
  qsum = __reduce_add_sync(0xffffffffu, qsum);
  if ((threadIdx.x & 31) == 0) atomicAdd(s_qsum, qsum);
  __syncthreads();
  return mx;
}

// CTA-wide barrier that also settles a timed-out wait for the weight copies
// (one barrier, phase 0).  Returns true when some thread of the CTA gave up:
// then thread 0 records kDevTimeoutProducer and waits once more (bounded) for
// the copies still in flight, so that the CTA's shared memory is not released
// under them, and the CTA writes no output.
__device__ __forceinline__ bool gemv_gave_up(bool landed, uint64_t* bar, int32_t* status) {
  if (!__syncthreads_or(!landed)) return false;
  if (threadIdx.x == 0) {
    *status = kDevTimeoutProducer;
    if (!mbar_wait(bar, 0)) *status = kDevTimeoutDrain;
  }
  return true;
}

__device__ __forceinline__ void gemv_store(uint16_t* y, int32_t* acc, int row, int32_t total, float s) {
  if (acc) acc[row] = total;
  const __nv_bfloat16 h = __float2bfloat16_rn(__fmul_rn(static_cast<float>(total), s));
  y[row] = *reinterpret_cast<const uint16_t*>(&h);
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
// two rows and adds its partial sums of q * code into the rows' shared
// accumulators, from which the store subtracts sum(q) once.

__host__ __device__ __forceinline__ int gemv_stripes(int64_t ld) { return static_cast<int>((ld + 127) / 128); }
__host__ __device__ __forceinline__ int gemv_stripe_bytes(int rows_box) { return (rows_box * 128 + 1023) & ~1023; }

__host__ __device__ __forceinline__ size_t gemv_smem_bytes(int rows_box, int64_t ld, int C) {
  return 1024 /* alignment */ + static_cast<size_t>(gemv_stripes(ld)) * gemv_stripe_bytes(rows_box) +
         static_cast<size_t>(C) * 4 * 16 + 16 /* code sum */ + static_cast<size_t>(rows_box) * 4;
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
  const uint16_t* x;      // one bf16 row [K]
  const float* gnorm;     // RMSNorm weight [K] (norm kernel variant only)
  float eps;
  int32_t* status;
  int64_t ld;
  int K, C, rows_box, count;
};

// The tensor maps (per matrix: uint8 [N, ld], box {128, rows_box}, 128-byte
// swizzle) are separate kernel parameters, and every parameter is read at a
// fixed offset: the matrix of this CTA is selected into registers.
template <bool kNorm>
__global__ void __launch_bounds__(kGemvThreads) gemv_dense_kernel(const __grid_constant__ CUtensorMap map0,
                                                                  const __grid_constant__ CUtensorMap map1,
                                                                  const __grid_constant__ CUtensorMap map2,
                                                                  const __grid_constant__ CUtensorMap map3,
                                                                  const GemvDense g) {
  extern __shared__ uint8_t s_raw[];
  __shared__ uint64_t s_bar;
  __shared__ float s_red[32];
  uint64_t tl[8] = {tl_now(), 0ull, 0ull, 0ull, 0ull, 0ull, 0ull, 0ull};  // test-build phase stamps (tl_now)
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
  int32_t* s_qsum = reinterpret_cast<int32_t*>(s_act + 4 * C);  // sum of the codes (one 16-byte slot)
  int32_t* s_acc = s_qsum + 4;
  float* s_g = reinterpret_cast<float*>(s_acc + rows_box);        // norm variant: RMSNorm weight [K]
  __shared__ double s_redd[32];

  // The weights (and alpha, which belongs to them) do not depend on the
  // preceding kernel: their copies start first.
  if (threadIdx.x == 0) {
    mbar_init(&s_bar, 1);
    fence_mbar_init();
    tma_prefetch_desc(map);
    mbar_arrive_expect_tx(&s_bar,
                          static_cast<uint32_t>(stripes) * 128u * static_cast<uint32_t>(rows_box) + test_extra_tx());
    const uint64_t pol = l2_policy_evict_first();
    for (int st = 0; st < stripes; ++st) tma_load_2d_hint(s_w + st * stripe_bytes, map, st * 128, r0, &s_bar, pol);
  }
  const float alpha = *mt.alpha;
  for (int r = threadIdx.x; r < nrows; r += blockDim.x) s_acc[r] = 0;
  if (threadIdx.x == 0) *s_qsum = 0;
  if (kNorm)  // the norm weight, like the matrix, does not depend on the preceding kernel
    for (int k = threadIdx.x; k < g.K; k += blockDim.x) s_g[k] = g.gnorm[k];
  __syncthreads();

  pdl_wait_primary();  // x may come from the preceding kernel
  if (kTimeline) tl[1] = tl_now();
  float gamma;
  if (kNorm)
    gamma = quantise_row_smem_norm(g.x, g.K, 4 * C, s_act, s_qsum, s_red, s_redd, s_g, g.eps);
  else
    gamma = quantise_row_smem(g.x, g.K, 4 * C, s_act, s_qsum, s_red);
  if (kTimeline) tl[2] = tl_now();
  // The next kernel may start now: its weight copies then stream while this
  // one contracts, and no longer delay this kernel's read of x.
  pdl_launch_dependents();
  const float s = __fdiv_rn(__fmul_rn(alpha, gamma), kQb);
  const bool landed = mbar_wait(&s_bar, 0);
  if (kTimeline) tl[3] = tl_now();

  if (landed) {
    // Thread (seg, p) takes row pair p (rows p and p + half) over the chunks of
    // segment seg and keeps the partial sums in registers; consecutive threads
    // take consecutive pairs of one segment, so a warp's lanes read one
    // activation chunk (a shared-memory broadcast) and conflict-free weight
    // slots.  Each partial sum s_j carries the factor 4^j of its bit plane and
    // stays below 2 * 64 * 127 * K / 4 < 2^31, so the final shifts are exact.
    const int half = (nrows + 1) >> 1;  // rows_box <= 256: at most 128 pairs, at least 4 segments
    const int nseg = blockDim.x / half;
    const int seg = threadIdx.x / half, p = threadIdx.x - seg * half;
    if (seg < nseg) {
      const int c_beg = seg * C / nseg, c_end = (seg + 1) * C / nseg;
      const int r2 = p + half < nrows ? p + half : p;  // an odd last pair reads row p twice
      int32_t a0 = 0, a1 = 0, a2 = 0, a3 = 0, b0 = 0, b1 = 0, b2 = 0, b3 = 0;
      for (int ch = c_beg; ch < c_end; ++ch) {
        const uint4 wa = gemv_wchunk(s_w, stripe_bytes, p, ch);
        const uint4 wb = gemv_wchunk(s_w, stripe_bytes, r2, ch);
        const uint4 q0 = s_act[ch], q1 = s_act[C + ch], q2 = s_act[2 * C + ch], q3 = s_act[3 * C + ch];
        dot_word(wa.x, q0.x, q0.y, q0.z, q0.w, a0, a1, a2, a3);
        dot_word(wb.x, q0.x, q0.y, q0.z, q0.w, b0, b1, b2, b3);
        dot_word(wa.y, q1.x, q1.y, q1.z, q1.w, a0, a1, a2, a3);
        dot_word(wb.y, q1.x, q1.y, q1.z, q1.w, b0, b1, b2, b3);
        dot_word(wa.z, q2.x, q2.y, q2.z, q2.w, a0, a1, a2, a3);
        dot_word(wb.z, q2.x, q2.y, q2.z, q2.w, b0, b1, b2, b3);
        dot_word(wa.w, q3.x, q3.y, q3.z, q3.w, a0, a1, a2, a3);
        dot_word(wb.w, q3.x, q3.y, q3.z, q3.w, b0, b1, b2, b3);
      }
      if (c_end > c_beg) {
        atomicAdd(&s_acc[p], a0 + (a1 >> 2) + (a2 >> 4) + (a3 >> 6));
        if (p + half < nrows) atomicAdd(&s_acc[p + half], b0 + (b1 >> 2) + (b2 >> 4) + (b3 >> 6));
      }
    }
  }
  if (gemv_gave_up(landed, &s_bar, g.status)) return;
  if (kTimeline) tl[4] = tl_now();
  const int32_t qsum = *s_qsum;
  for (int rr = threadIdx.x; rr < nrows; rr += blockDim.x) gemv_store(mt.y, mt.acc, r0 + rr, s_acc[rr] - qsum, s);
  if (kTimeline && threadIdx.x == 0) tl_commit_now(1, (static_cast<uint64_t>(g.K) << 32) | (blockIdx.x << 16) | gridDim.x, tl, 5);
}

// ------------------------------------------------------------------ FFN gate/up with squared ReLU, M = 1
// The FFN of BitNet b1.58 2B4T uses squared ReLU (2B4T report summary,
// section 2, Architecture).  With the block's gate and up projections (two
// BitLinears of one x, outputs g and u in bf16) the result is taken as
//     h = RN_bf16(RN_bf16(max(g, 0)^2) * u)
// elementwise; both products are exact in fp32 (8-bit significands), so each
// step rounds once, as the bf16 operations would.
__device__ __forceinline__ uint16_t relu2_glu_bf16(uint16_t gb, uint16_t ub) {
  const float gv = __uint_as_float(static_cast<uint32_t>(gb) << 16);
  const float r = gv > 0.0f ? gv : 0.0f;
  const __nv_bfloat16 sq = __float2bfloat16_rn(__fmul_rn(r, r));
  const __nv_bfloat16 h = __float2bfloat16_rn(
      __fmul_rn(__bfloat162float(sq), __uint_as_float(static_cast<uint32_t>(ub) << 16)));
  return *reinterpret_cast<const uint16_t*>(&h);
}

// One token: each CTA owns the same rows of both matrices.  Its stripes hold
// the gate rows at lines 0.. and the up rows at lines rows_box.. (rows_box a
// multiple of 8, so both boxes keep the 128-byte swizzle phase), and thread
// (segment, p) contracts gate row p and up row p over its segment; the store
// forms y_gate and y_up as the single-matrix GEMV would and writes h only.
struct GemvGlu {
  const float* alpha_g;
  const float* alpha_u;
  uint16_t* h;        // [N]
  const uint16_t* x;  // one bf16 row [K]
  int32_t* status;
  int64_t ld;
  int K, C, rows_box, rows_base, rows_rem;
};

__host__ __device__ __forceinline__ size_t gemv_glu_smem_bytes(int rows_box, int64_t ld, int C) {
  return 1024 + static_cast<size_t>(gemv_stripes(ld)) * gemv_stripe_bytes(2 * rows_box) +
         static_cast<size_t>(C) * 4 * 16 + 16 + static_cast<size_t>(2 * rows_box) * 4;
}

__global__ void __launch_bounds__(kGemvThreads) gemv_glu_kernel(const __grid_constant__ CUtensorMap map_g,
                                                                const __grid_constant__ CUtensorMap map_u,
                                                                const GemvGlu g) {
  extern __shared__ uint8_t s_raw[];
  __shared__ uint64_t s_bar;
  __shared__ float s_red[32];
  const int b = blockIdx.x;
  const int r0 = b * g.rows_base + min(b, g.rows_rem);
  const int nrows = g.rows_base + (b < g.rows_rem ? 1 : 0);
  const int C = g.C;
  const int rows_box = g.rows_box;
  const int stripes = gemv_stripes(g.ld);
  const int stripe_bytes = gemv_stripe_bytes(2 * rows_box);
  uint8_t* s_w = s_raw + ((1024u - (smem_u32(s_raw) & 1023u)) & 1023u);
  uint4* s_act = reinterpret_cast<uint4*>(s_w + static_cast<size_t>(stripes) * stripe_bytes);
  int32_t* s_qsum = reinterpret_cast<int32_t*>(s_act + 4 * C);
  int32_t* s_acc = s_qsum + 4;  // [2 * rows_box]: gate rows, then up rows

  if (threadIdx.x == 0) {
    mbar_init(&s_bar, 1);
    fence_mbar_init();
    tma_prefetch_desc(&map_g);
    tma_prefetch_desc(&map_u);
    mbar_arrive_expect_tx(&s_bar,
                          static_cast<uint32_t>(stripes) * 256u * static_cast<uint32_t>(rows_box) + test_extra_tx());
    const uint64_t pol = l2_policy_evict_first();
    for (int st = 0; st < stripes; ++st) {
      tma_load_2d_hint(s_w + st * stripe_bytes, &map_g, st * 128, r0, &s_bar, pol);
      tma_load_2d_hint(s_w + st * stripe_bytes + rows_box * 128, &map_u, st * 128, r0, &s_bar, pol);
    }
  }
  const float alpha_g = *g.alpha_g, alpha_u = *g.alpha_u;
  for (int r = threadIdx.x; r < 2 * rows_box; r += blockDim.x) s_acc[r] = 0;
  if (threadIdx.x == 0) *s_qsum = 0;
  __syncthreads();

  pdl_wait_primary();  // x may come from the preceding kernel
  const float gamma = quantise_row_smem(g.x, g.K, 4 * C, s_act, s_qsum, s_red);
  pdl_launch_dependents();
  const float sg = __fdiv_rn(__fmul_rn(alpha_g, gamma), kQb);
  const float su = __fdiv_rn(__fmul_rn(alpha_u, gamma), kQb);
  const bool landed = mbar_wait(&s_bar, 0);

  if (landed && nrows > 0) {
    // as gemv_dense_kernel, with the pair (gate row p, up row p): consecutive threads take consecutive
    // rows of one segment, so a warp reads one activation chunk (broadcast) and conflict-free weight slots
    const int nseg = blockDim.x / nrows;  // rows_box <= 128: at least 4 segments
    const int seg = threadIdx.x / nrows, p = threadIdx.x - seg * nrows;
    if (seg < nseg) {
      const int c_beg = seg * C / nseg, c_end = (seg + 1) * C / nseg;
      int32_t a0 = 0, a1 = 0, a2 = 0, a3 = 0, b0 = 0, b1 = 0, b2 = 0, b3 = 0;
      for (int ch = c_beg; ch < c_end; ++ch) {
        const uint4 wa = gemv_wchunk(s_w, stripe_bytes, p, ch);
        const uint4 wb = gemv_wchunk(s_w, stripe_bytes, rows_box + p, ch);
        const uint4 q0 = s_act[ch], q1 = s_act[C + ch], q2 = s_act[2 * C + ch], q3 = s_act[3 * C + ch];
        dot_word(wa.x, q0.x, q0.y, q0.z, q0.w, a0, a1, a2, a3);
        dot_word(wb.x, q0.x, q0.y, q0.z, q0.w, b0, b1, b2, b3);
        dot_word(wa.y, q1.x, q1.y, q1.z, q1.w, a0, a1, a2, a3);
        dot_word(wb.y, q1.x, q1.y, q1.z, q1.w, b0, b1, b2, b3);
        dot_word(wa.z, q2.x, q2.y, q2.z, q2.w, a0, a1, a2, a3);
        dot_word(wb.z, q2.x, q2.y, q2.z, q2.w, b0, b1, b2, b3);
        dot_word(wa.w, q3.x, q3.y, q3.z, q3.w, a0, a1, a2, a3);
        dot_word(wb.w, q3.x, q3.y, q3.z, q3.w, b0, b1, b2, b3);
      }
      if (c_end > c_beg) {
        atomicAdd(&s_acc[p], a0 + (a1 >> 2) + (a2 >> 4) + (a3 >> 6));
        atomicAdd(&s_acc[rows_box + p], b0 + (b1 >> 2) + (b2 >> 4) + (b3 >> 6));
      }
    }
  }
  if (gemv_gave_up(landed, &s_bar, g.status)) return;
  const int32_t qsum = *s_qsum;
  for (int rr = threadIdx.x; rr < nrows; rr += blockDim.x) {
    const __nv_bfloat16 yg = __float2bfloat16_rn(__fmul_rn(static_cast<float>(s_acc[rr] - qsum), sg));
    const __nv_bfloat16 yu = __float2bfloat16_rn(__fmul_rn(static_cast<float>(s_acc[rows_box + rr] - qsum), su));
    g.h[r0 + rr] = relu2_glu_bf16(*reinterpret_cast<const uint16_t*>(&yg), *reinterpret_cast<const uint16_t*>(&yu));
  }
}

// Many tokens: h from the two BitLinear outputs (bf16 bits), 8 per thread and
// step when the three arrays are 16-byte aligned.
__global__ void __launch_bounds__(256) relu2_glu_kernel(const uint16_t* __restrict__ yg,
                                                        const uint16_t* __restrict__ yu, uint16_t* __restrict__ h,
                                                        size_t count, bool vec) {
  pdl_wait_primary();
  pdl_launch_dependents();
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (vec) {
    for (; 8 * i + 8 <= count; i += stride) {
      const uint4 a = reinterpret_cast<const uint4*>(yg)[i], b = reinterpret_cast<const uint4*>(yu)[i];
      const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        o[j] = relu2_glu_bf16(static_cast<uint16_t>(aw[j]), static_cast<uint16_t>(bw[j])) |
               (static_cast<uint32_t>(relu2_glu_bf16(static_cast<uint16_t>(aw[j] >> 16),
                                                     static_cast<uint16_t>(bw[j] >> 16))) << 16);
      reinterpret_cast<uint4*>(h)[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    // the tail (count % 8 elements) by the first threads
    const size_t tail0 = count / 8 * 8;
    const size_t t = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (tail0 + t < count) h[tail0 + t] = relu2_glu_bf16(yg[tail0 + t], yu[tail0 + t]);
  } else {
    for (; i < count; i += stride) h[i] = relu2_glu_bf16(yg[i], yu[i]);
  }
}

// ------------------------------------------------------------------ dense M = 1, lookup tables
// The TL2 lookup idea of bitnet.cpp ("BitNet 1-Bit LLM" blog, section "I2_S
// kernel internals"): two consecutive ternary weights index a table of the
// nine sums +-a0 +-a1 of their two activations.  Here the index is the pair's
// 4-bit nibble of I2_S codes (c0 | c1 << 2, 9 of 16 entries used), the table
// entry is (c0 - 1) q0 + (c1 - 1) q1 (int16) for the pair's int8 codes, and
// one table of 16 entries per pair is built in shared memory after the
// quantisation.  A unit (64-weight chunk, row) then costs 32 lookups and adds
// instead of 16 masked dp4a: this kernel exists to measure that trade against
// gemv_dense_kernel (same weights, same staging, same results).
__host__ __device__ __forceinline__ size_t gemv_lut_smem_bytes(int rows_box, int64_t ld, int C) {
  return gemv_smem_bytes(rows_box, ld, C) + static_cast<size_t>(C) * 32 * 16 * 2 + 16;
}

__global__ void __launch_bounds__(kGemvThreads) gemv_lut_kernel(const __grid_constant__ CUtensorMap map0,
                                                                const GemvDense g) {
  extern __shared__ uint8_t s_raw[];
  __shared__ uint64_t s_bar;
  __shared__ float s_red[32];
  const GemvMat mt = g.mat[0];
  const int b = blockIdx.x;
  const int r0 = b * mt.rows_base + min(b, mt.rows_rem);
  const int nrows = mt.rows_base + (b < mt.rows_rem ? 1 : 0);
  const int C = g.C;
  const int rows_box = g.rows_box;
  const int stripes = gemv_stripes(g.ld);
  const int stripe_bytes = gemv_stripe_bytes(rows_box);
  uint8_t* s_w = s_raw + ((1024u - (smem_u32(s_raw) & 1023u)) & 1023u);
  uint4* s_act = reinterpret_cast<uint4*>(s_w + static_cast<size_t>(stripes) * stripe_bytes);
  int32_t* s_qsum = reinterpret_cast<int32_t*>(s_act + 4 * C);  // filled, not needed: the tables carry W_t
  int32_t* s_acc = s_qsum + 4;
  int16_t* s_lut = reinterpret_cast<int16_t*>(s_acc + rows_box + 3 - ((rows_box + 3) & 3));  // [pairs][16]

  if (threadIdx.x == 0) {
    mbar_init(&s_bar, 1);
    fence_mbar_init();
    tma_prefetch_desc(&map0);
    mbar_arrive_expect_tx(&s_bar,
                          static_cast<uint32_t>(stripes) * 128u * static_cast<uint32_t>(rows_box) + test_extra_tx());
    const uint64_t pol = l2_policy_evict_first();
    for (int st = 0; st < stripes; ++st) tma_load_2d_hint(s_w + st * stripe_bytes, &map0, st * 128, r0, &s_bar, pol);
  }
  const float alpha = *mt.alpha;
  for (int r = threadIdx.x; r < nrows; r += blockDim.x) s_acc[r] = 0;
  if (threadIdx.x == 0) *s_qsum = 0;
  __syncthreads();

  pdl_wait_primary();
  const float gamma = quantise_row_smem(g.x, g.K, 4 * C, s_act, s_qsum, s_red);
  pdl_launch_dependents();
  // tables: pair p covers k = 2p, 2p + 1; code of k sits in group k / 16, word k % 4, byte (k % 16) / 4
  const int pairs = 32 * C;  // 64-weight chunks of 32 pairs (codes past K are 0)
  const int quarter = C;     // s_act slot stride (groups_alloc / 4)
  for (int p = threadIdx.x; p < pairs; p += blockDim.x) {
    int32_t qv[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int k = 2 * p + t, gi = k >> 4;
      const uint32_t* w = reinterpret_cast<const uint32_t*>(s_act + (gi & 3) * quarter + (gi >> 2));
      qv[t] = static_cast<int8_t>(w[k & 3] >> (8 * ((k & 15) >> 2)));
    }
#pragma unroll
    for (int n = 0; n < 16; ++n)
      s_lut[16 * p + n] = static_cast<int16_t>(((n & 3) - 1) * qv[0] + ((n >> 2) - 1) * qv[1]);
  }
  __syncthreads();
  const float s = __fdiv_rn(__fmul_rn(alpha, gamma), kQb);
  const bool landed = mbar_wait(&s_bar, 0);

  if (landed) {
    const int total = nrows * C;  // units (chunk, row), row fastest
    for (int u = threadIdx.x; u < total; u += blockDim.x) {
      const int ch = u / nrows, r = u - ch * nrows;
      const uint4 wv = gemv_wchunk(s_w, stripe_bytes, r, ch);
      const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
      const int16_t* lut = s_lut + 16 * 32 * ch;
      int32_t acc = 0;
#pragma unroll
      for (int wi = 0; wi < 4; ++wi)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc += lut[16 * (8 * wi + i) + ((ww[wi] >> (4 * i)) & 0xFu)];
      atomicAdd(&s_acc[r], acc);
    }
  }
  if (gemv_gave_up(landed, &s_bar, g.status)) return;
  for (int rr = threadIdx.x; rr < nrows; rr += blockDim.x) gemv_store(mt.y, mt.acc, r0 + rr, s_acc[rr], s);
}

// ------------------------------------------------------------------ N:M helpers
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

// ------------------------------------------------------------------ N:M, M = 1
// Same structure as the dense kernel: each CTA's rows of kept values and of
// metadata arrive by TMA tile loads (128-byte swizzle) issued before the
// dependency wait, x is quantised into shared memory, and a flat list of
// (128-weight unit, row pair) units is spread over all threads.  A unit
// rebuilds the dense 2-bit code words of its 128 weights (pruned positions get
// code 01, weight 0) and runs the dense dot on them, so Σ q * code - Σ q over
// the unit gives the exact partial sum.
//   2:4: per block the 4-bit metadata (i0 | i1 << 2) and the block's two kept
//        codes (4 bits) index a 256-entry table of dense code bytes; each lane
//        reads its own bank-private copy (entry e of lane l at word e * 32 + l).
//   n:8: the pruned positions of each 8-block are inserted one by one
//        (n8_dense_block); the values of a unit are 4n bytes.
constexpr int kNmLutWords = 256 * 32;

struct GemvNmArgs {
  const uint16_t* x;   // one bf16 row [K]
  const float* alpha;
  uint16_t* y;         // [N]
  int32_t* acc;        // [N] or null
  int32_t* status;
  int64_t ld_v, ld_m;  // row strides of values / metadata (bytes)
  int K, C;            // C = ceil(K / 128) units per row
  int rows_base, rows_rem, rows_box;
};

__host__ __device__ __forceinline__ int nm_unit_value_bytes(int n) { return n == 0 ? 16 : 4 * n; }  // n = 0: 2:4

__host__ __device__ __forceinline__ size_t gemv_nm_smem_bytes(int rows_box, int64_t ld_v, int64_t ld_m, int C, bool lut) {
  return 1024 + static_cast<size_t>(gemv_stripes(ld_v) + gemv_stripes(ld_m)) * gemv_stripe_bytes(rows_box) +
         (lut ? static_cast<size_t>(kNmLutWords) * 4 : 0) + static_cast<size_t>(C) * 8 * 16 /* codes */ +
         16 /* code sum */ + static_cast<size_t>(rows_box) * 4;
}

// 32-bit word at byte offset off (a multiple of 4) of local row r in swizzled 128-byte stripes.
__device__ __forceinline__ uint32_t sw_word(const uint8_t* base, int stripe_bytes, int r, int off) {
  const int w = off & 127;
  return *reinterpret_cast<const uint32_t*>(base + (off >> 7) * stripe_bytes + r * 128 +
                                            ((((w >> 4) ^ (r & 7)) << 4) | (w & 15)));
}

// Fills the 2:4 table (all threads of the CTA): entry e = (i0 | i1 << 2) |
// (c0 | c1 << 2) << 4 holds the dense code byte of a block, lane l's copy at
// word e * 32 + l.
__device__ __forceinline__ void nm24_fill_lut(uint32_t* s_lut) {
  for (int i = threadIdx.x; i < kNmLutWords; i += blockDim.x) {
    const uint32_t e = static_cast<uint32_t>(i) >> 5;
    const uint32_t i0 = e & 3u, i1 = (e >> 2) & 3u, c0 = (e >> 4) & 3u, c1 = (e >> 6) & 3u;
    s_lut[i] = (0x55u ^ ((c0 ^ 1u) << (2 * i0)) ^ ((c1 ^ 1u) << (2 * i1))) & 0xFFu;
  }
}

// Dense code word of 16 weights (4 blocks) of a 2:4 row from 16 bits of
// metadata and 16 bits of kept codes, through the lane's table copy.
__device__ __forceinline__ uint32_t nm24_word_lut(const uint32_t* lut_lane, uint32_t meta16, uint32_t vals16) {
  // spread the four nibbles of each into the low nibbles of four bytes
  uint32_t m = (meta16 | (meta16 << 8)) & 0x00FF00FFu;
  m = (m | (m << 4)) & 0x0F0F0F0Fu;
  uint32_t v = (vals16 | (vals16 << 8)) & 0x00FF00FFu;
  v = (v | (v << 4)) & 0x0F0F0F0Fu;
  const uint32_t idx = m | (v << 4);  // byte t: block t's table index
  const uint32_t d0 = lut_lane[(idx & 0xFFu) << 5];
  const uint32_t d1 = lut_lane[((idx >> 8) & 0xFFu) << 5];
  const uint32_t d2 = lut_lane[((idx >> 16) & 0xFFu) << 5];
  const uint32_t d3 = lut_lane[(idx >> 24) << 5];
  return __byte_perm(__byte_perm(d0, d1, 0x0040), __byte_perm(d2, d3, 0x0040), 0x5410);
}

// Dense code words of the 8 groups of unit u of local row r.
template <int NMN>
__device__ __forceinline__ void nm_unit_words(const uint8_t* s_v, const uint8_t* s_m, int stripe_bytes, int r, int u,
                                              const uint32_t* lut_lane, uint32_t (&dw)[8]) {
  uint32_t mw[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) mw[i] = sw_word(s_m, stripe_bytes, r, 16 * u + 4 * i);
  if (NMN == 0) {
    uint32_t vw[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) vw[i] = sw_word(s_v, stripe_bytes, r, 16 * u + 4 * i);
#pragma unroll
    for (int g = 0; g < 8; ++g)
      dw[g] = nm24_word_lut(lut_lane, (mw[g >> 1] >> (16 * (g & 1))) & 0xFFFFu, (vw[g >> 1] >> (16 * (g & 1))) & 0xFFFFu);
  } else {
    constexpr int n = NMN;
    uint32_t vw[n + 1];
#pragma unroll
    for (int i = 0; i < n; ++i) vw[i] = sw_word(s_v, stripe_bytes, r, 4 * n * u + 4 * i);
    vw[n] = 0u;
    constexpr uint32_t fmask = (1u << (2 * n)) - 1u;
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      const int bit = 4 * n * g;  // two blocks of n kept codes
      const int wi = bit >> 5, sh = bit & 31;
      const uint32_t kv = sh == 0 ? vw[wi] : __funnelshift_r(vw[wi], vw[wi + 1], sh);
      const uint32_t m0 = (mw[g >> 1] >> (16 * (g & 1))) & 0xFFu, m1 = (mw[g >> 1] >> (16 * (g & 1) + 8)) & 0xFFu;
      dw[g] = n8_dense_block(m0, kv & fmask) | (n8_dense_block(m1, (kv >> (2 * n)) & fmask) << 16);
    }
  }
}

template <int NMN>
__global__ void __launch_bounds__(kGemvThreads) gemv_nm_kernel(const __grid_constant__ CUtensorMap map_v,
                                                               const __grid_constant__ CUtensorMap map_m,
                                                               const GemvNmArgs a) {
  extern __shared__ uint8_t s_raw[];
  __shared__ uint64_t s_bar;
  __shared__ float s_red[32];
  const int b = blockIdx.x;
  const int r0 = b * a.rows_base + min(b, a.rows_rem);
  const int nrows = a.rows_base + (b < a.rows_rem ? 1 : 0);
  const int C = a.C;
  const int rows_box = a.rows_box;
  const int stripes_v = gemv_stripes(a.ld_v), stripes_m = gemv_stripes(a.ld_m);
  const int stripe_bytes = gemv_stripe_bytes(rows_box);
  // offset arithmetic on the shared array keeps every derived pointer in the shared window
  uint8_t* s_v = s_raw + ((1024u - (smem_u32(s_raw) & 1023u)) & 1023u);
  uint8_t* s_m = s_v + static_cast<size_t>(stripes_v) * stripe_bytes;
  uint32_t* s_lut = reinterpret_cast<uint32_t*>(s_m + static_cast<size_t>(stripes_m) * stripe_bytes);
  uint4* s_act = reinterpret_cast<uint4*>(s_lut + (NMN == 0 ? kNmLutWords : 0));
  int32_t* s_qsum = reinterpret_cast<int32_t*>(s_act + 8 * C);  // sum of the codes (one 16-byte slot)
  int32_t* s_acc = s_qsum + 4;

  if (threadIdx.x == 0) {
    mbar_init(&s_bar, 1);
    fence_mbar_init();
    tma_prefetch_desc(&map_v);
    tma_prefetch_desc(&map_m);
    mbar_arrive_expect_tx(&s_bar, static_cast<uint32_t>(stripes_v + stripes_m) * 128u * static_cast<uint32_t>(rows_box) +
                                      test_extra_tx());
    const uint64_t pol = l2_policy_evict_first();
    for (int st = 0; st < stripes_v; ++st) tma_load_2d_hint(s_v + st * stripe_bytes, &map_v, st * 128, r0, &s_bar, pol);
    for (int st = 0; st < stripes_m; ++st) tma_load_2d_hint(s_m + st * stripe_bytes, &map_m, st * 128, r0, &s_bar, pol);
  }
  if (NMN == 0) nm24_fill_lut(s_lut);
  const float alpha = *a.alpha;
  for (int r = threadIdx.x; r < nrows; r += blockDim.x) s_acc[r] = 0;
  if (threadIdx.x == 0) *s_qsum = 0;
  __syncthreads();

  pdl_wait_primary();  // x may come from the preceding kernel
  const float gamma = quantise_row_smem(a.x, a.K, 8 * C, s_act, s_qsum, s_red);
  pdl_launch_dependents();
  const float s = __fdiv_rn(__fmul_rn(alpha, gamma), kQb);
  const bool landed = mbar_wait(&s_bar, 0);

  if (landed) {
    const uint32_t* lut_lane = s_lut + (threadIdx.x & 31);
    const int nthr = blockDim.x;
    const int half = (nrows + 1) >> 1;
    const int total = half * C;
    const int dq = nthr / half, dr = nthr % half;
    int u = threadIdx.x / half, p = threadIdx.x % half;
    const int quarter = 2 * C;  // s_act slot stride: group g sits at (g % 4) * 2C + g / 4
    for (int it = threadIdx.x; it < total; it += nthr) {
      const int r2 = p + half < nrows ? p + half : p;
      uint32_t da[8], db[8];
      nm_unit_words<NMN>(s_v, s_m, stripe_bytes, p, u, lut_lane, da);
      nm_unit_words<NMN>(s_v, s_m, stripe_bytes, r2, u, lut_lane, db);
      int32_t a0 = 0, a1 = 0, a2 = 0, a3 = 0, b0 = 0, b1 = 0, b2 = 0, b3 = 0;
#pragma unroll
      for (int gi = 0; gi < 8; ++gi) {
        const int g = 8 * u + gi;
        const uint4 q = s_act[(g & 3) * quarter + (g >> 2)];
        dot_word(da[gi], q.x, q.y, q.z, q.w, a0, a1, a2, a3);
        dot_word(db[gi], q.x, q.y, q.z, q.w, b0, b1, b2, b3);
      }
      atomicAdd(&s_acc[p], a0 + (a1 >> 2) + (a2 >> 4) + (a3 >> 6));
      if (p + half < nrows) atomicAdd(&s_acc[p + half], b0 + (b1 >> 2) + (b2 >> 4) + (b3 >> 6));
      p += dr;
      u += dq;
      if (p >= half) {
        p -= half;
        ++u;
      }
    }
  }
  if (gemv_gave_up(landed, &s_bar, a.status)) return;
  const int32_t qsum = *s_qsum;
  for (int rr = threadIdx.x; rr < nrows; rr += blockDim.x) gemv_store(a.y, a.acc, r0 + rr, s_acc[rr] - qsum, s);
}

}  // namespace bl
