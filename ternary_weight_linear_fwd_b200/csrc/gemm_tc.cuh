// gemm_tc.cuh -- many-token BitLinear on the 5th-generation tensor cores.
//
// The 2B4T report (section 5.1) stages packed ternary weights on chip,
// unpacks them and multiplies them with 8-bit activations.  On sm_100a that
// becomes a persistent tcgen05 kind::i8 GEMM:
//
//   D[128 weight rows, BN tokens] (int32, TMEM) += A * B^T over K, where
//   A = the weight rows' 2-bit codes (0, 1, 2) expanded to u8 and written
//       straight into tensor memory by the unpack warps (tcgen05.st), so the
//       expanded weights never pass through shared memory;
//   B = the tokens' int8 codes, TMA-loaded into 128-byte-swizzled shared
//       memory (K-major).
//
// With code = W_t + 1 the contraction gives sum q * code, and the epilogue
// subtracts the token's sum of codes: acc = D - rowsum (exact in int32).
// Both operands are in natural K order: the activation codes as the
// quantisation writes them, the weights after a 4 x 4 byte transpose of the
// masked 2-bit fields (codes_word_natural).
//
// One CTA per SM walks a static list of (weight-row tile, token tile, K slice)
// units.  When the tiles alone would leave SMs idle (few tokens, or few
// weight rows), each tile's K range is split into slices; every slice adds its
// partial sums into one fp32 [M, N] buffer with vector atomic adds, and the
// slice that arrives last (an atomic counter per tile) reads the sums, runs
// the epilogue and clears them.  The sums are exact: every partial and total
// of q * code is an integer of magnitude at most 254 * K <= 254 * 65536 < 2^24.
// Warp roles (16 warps): warp 0 lane 0 issues TMA loads, warp 1 lane 0 issues
// the MMAs, warp 2 owns the TMEM allocation, warps 4..11 unpack weights (two
// groups of four, for the even and the odd stages), warps 12..15 run the epilogue.  Warp
// w reaches TMEM lanes 32 * (w % 4) .. + 31.  A mbarrier ring (4 to 8 stages of
// 256 k for dense weights, 128 k for N:M; as many as TMEM has A slots for) couples
// the producer, unpackers and MMA issuer (full: TMA bytes landed, aready: A
// slot written, empty: the MMAs that read the stage completed); two TMEM
// accumulators (accfull / accempty) let the epilogue of one tile overlap the
// main loop of the next.  Every wait is bounded; a role that gives up records
// a status code and unwinds.
//
// N:M weights (Sparse-BitNet, section 3.2): n:8 rows, and 2:4 rows on request,
// are expanded from kept values + metadata into the same dense code words
// before the tcgen05.st, so the MMA is the dense one.  By default 2:4 rows
// run on the structured-sparse MMA (NM = 3, the sparse tensor-core path of
// the Sparse-BitNet review, section 4): the unpack warps turn the kept codes
// into signed int8 weights (W_t itself, so no code-sum correction) in the
// 128-byte-swizzled K-major layout of a shared-memory A operand holding only
// the kept values, copy the packed metadata unchanged into TMEM (its nibble
// i0 | i1 << 2 per block of four is the instruction's metadata format), and
// tcgen05.mma.sp kind::i8 multiplies them with activation codes in natural K
// order: 64 K per instruction, half the instructions of the dense MMA.
#pragma once
#include "gemv.cuh"
#include "hbit.cuh"

namespace bl {

constexpr int kTcMaxStages = 8;
constexpr int kTcSubK = 128;    // K elements of one 128-byte swizzle row of the activation tile
constexpr int kTcRows = 128;    // weight rows per tile (MMA M)
constexpr int kTcThreads = 512;
constexpr int kTcEpiWarp0 = 12;  // first epilogue warp

// K elements per stage: dense and 2:4 weights with token tiles up to 128 take
// two 128-wide sub-tiles (eight MMAs per barrier round trip, which halves the
// fixed cost of a stage per MAC); wider tiles and n:8 weights keep one.
__host__ __device__ constexpr int tc_ksub(int NM, int BN) { return (NM != 2 && BN <= 128) ? 2 : 1; }
__host__ __device__ constexpr int tc_bk(int NM, int BN) { return kTcSubK * tc_ksub(NM, BN); }

struct TcArgs {
  int M, N, K;
  int kblocks;            // ceil(K / tc_bk(NM))
  int row_tiles, tok_tiles;
  int ksplit;             // K slices per tile (1: no split)
  int kbs;                // k-blocks per slice, ceil(kblocks / ksplit)
  float* part;            // ksplit > 1: fp32 [M][N] sums of the slices, zero on entry and left zero
  uint32_t* cnt;          // ksplit > 1: [row_tiles * tok_tiles] arrival counters, zero on entry and left zero
  const float* gamma;     // [M] per-token absmax
  const float* alpha;     // the matrix's absmean scale (device)
  const int32_t* rowsum;  // [M] sum of the token's codes
  uint16_t* y;            // [M, N] bf16 bits
  int32_t* acc;           // [M, N] or null
  int vec_store;          // y / acc rows are 16-byte aligned and N % 8 == 0
  int nm_n;               // kept per 8-block (n:8 mode)
  int vbox;               // n:8: bytes of the values box per row
  float qb;               // Q_b of the activation codes: 127 (8-bit), 7 (H-BitLinear 4-bit)
  int32_t* status;        // device status word
};

template <int NM, int BN>
struct TcStageBytes {
  // packed A bytes per stage (TMA box bytes, rows = 128)
  static __host__ __device__ constexpr int a_values(int vbox) {
    return NM == 0 ? kTcRows * 32 * tc_ksub(0, BN) : (NM != 2 ? kTcRows * 16 * tc_ksub(NM, BN) : kTcRows * vbox);
  }
  static __host__ __device__ constexpr int a_meta() { return NM == 0 ? 0 : kTcRows * 16 * tc_ksub(NM, BN); }
};

__host__ __device__ constexpr int tc_dcols(int BN) { return BN < 32 ? 32 : BN; }  // TMEM columns of one accumulator
// TMEM columns of one stage: the expanded A codes (32 per 128 k), or for the
// sparse MMA the metadata (4 bits per 4 k: 4 columns per 128 k)
__host__ __device__ constexpr int tc_slot_cols(int NM, int BN) { return (NM == 3 ? 4 : 32) * tc_ksub(NM, BN); }
constexpr int kTcSmemMax = 232448;  // dynamic shared memory a CTA may opt into
// Compressed int8 A of one sparse-MMA stage: 128 rows x (stage K / 2) bytes.
__host__ __device__ constexpr int tc_sp_a_bytes(int BN) { return kTcRows * 64 * tc_ksub(3, BN); }
// Shared memory of one stage's A: the TMA box(es) of packed weights; for the
// sparse MMA the compressed operand, which the packed values and metadata
// (half its size) land in and are unpacked over.
__host__ __device__ constexpr int tc_a_stage_bytes(int NM, int BN, int vbox) {
  return NM == 3 ? tc_sp_a_bytes(BN)
                 : ((NM == 0 ? kTcRows * 32 * tc_ksub(0, BN) : (NM != 2 ? kTcRows * 16 * tc_ksub(NM, BN) : kTcRows * vbox)) +
                    (NM == 0 ? 0 : kTcRows * 16 * tc_ksub(NM, BN)) + 1023) / 1024 * 1024;
}
__host__ __device__ constexpr int tc_fixed_smem(int BN, int NM) {
  return 1024 /* alignment slack */ + (NM == 1 ? kNmLutWords * 4 : 0) /* 2:4 expansion table, one copy per lane */ +
         4 * 32 * 33 * 4 /* epilogue staging */ + 2 * BN * 8 /* scales, code sums */ + 256 /* barriers */;
}
// Shared memory of one pipeline stage.
__host__ __device__ constexpr int tc_stage_smem(int BN, int NM, int vbox) {
  return BN * 128 * tc_ksub(NM, BN) + tc_a_stage_bytes(NM, BN, vbox);
}
__host__ __device__ constexpr int tc_min3(int a, int b, int c) { return a < b ? (a < c ? a : c) : (b < c ? b : c); }
// Pipeline stages: as many as TMEM has slots for beside the two accumulators,
// at most 8; the sparse MMA's stages are bounded by shared memory instead.
__host__ __device__ constexpr int tc_stages(int BN, int NM) {
  return tc_min3(kTcMaxStages, (512 - 2 * tc_dcols(BN)) / tc_slot_cols(NM, BN),
                 NM == 3 ? (kTcSmemMax - tc_fixed_smem(BN, 3)) / tc_stage_smem(BN, 3, 0) : kTcMaxStages);
}

template <int BN, int NM>
struct TcCols {
  static constexpr int kDcols = tc_dcols(BN);                      // one accumulator
  static constexpr int kAcol0 = 2 * kDcols;                        // A slots after both accumulators
  static constexpr int kNeed = kAcol0 + tc_stages(BN, NM) * tc_slot_cols(NM, BN);
  static constexpr int kAlloc = kNeed <= 256 ? 256 : 512;
  static_assert(kNeed <= 512, "TMEM budget");
};

__host__ __device__ constexpr int tc_smem_bytes(int BN, int NM, int vbox) {
  return tc_fixed_smem(BN, NM) + tc_stages(BN, NM) * tc_stage_smem(BN, NM, vbox);
}

// Dense code word of 16 weights (group gi of the stage) of an n:8 row: two
// blocks of n kept codes starting at bit rem * 8 + gi * 4n of the values.
__device__ __forceinline__ uint32_t tc_n8_group_word(const uint8_t* arow, const uint8_t* mrow, int gi, int n,
                                                     int rem) {
  const uint32_t m0 = mrow[2 * gi], m1 = mrow[2 * gi + 1];
  const int bit = rem * 8 + gi * 4 * n;
  const uint32_t* p = reinterpret_cast<const uint32_t*>(arow);
  const int wi = bit >> 5, sh = bit & 31;
  uint32_t kv = p[wi] >> sh;
  if (sh != 0 && sh + 4 * n > 32) kv |= p[wi + 1] << (32 - sh);
  const uint32_t fmask = (1u << (2 * n)) - 1u;
  return n8_dense_block(m0, kv & fmask) | (n8_dense_block(m1, (kv >> (2 * n)) & fmask) << 16);
}

// Rescales and stores the first ntok (<= 32) tokens of one warp's 32
// accumulator rows, as read from TMEM (v[j] = D[row][tokb + j], lane = row),
// tokens past M skipped: for each token the 32 lanes
// write its 32 consecutive outputs, 64 contiguous bytes of y (128 of acc)
// per store, straight from the lane layout.  scl / rsm: the tokens' scales and
// code sums (broadcast reads from shared memory).
__device__ __forceinline__ void tc_store_token_rows(const uint32_t (&v)[32], const float* scl, const int32_t* rsm,
                                                    int row, int tokb, int ntok, const TcArgs& a) {
  if (row >= a.N) return;
  if (ntok > a.M - tokb) ntok = a.M - tokb;
  uint16_t* yr = a.y + static_cast<size_t>(tokb) * a.N + row;
  int32_t* ar = a.acc ? a.acc + static_cast<size_t>(tokb) * a.N + row : nullptr;
  if (ntok == 32) {
    // a full chunk: scales and sums as 16-byte broadcast reads, then 32 independent stores
    float sc[32];
    int32_t rs[32];
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
      const float4 f = *reinterpret_cast<const float4*>(scl + j);
      const int4 r = *reinterpret_cast<const int4*>(rsm + j);
      sc[j] = f.x; sc[j + 1] = f.y; sc[j + 2] = f.z; sc[j + 3] = f.w;
      rs[j] = r.x; rs[j + 1] = r.y; rs[j + 2] = r.z; rs[j + 3] = r.w;
    }
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int32_t tv = static_cast<int32_t>(v[j]) - rs[j];
      const __nv_bfloat16 h = __float2bfloat16_rn(__fmul_rn(static_cast<float>(tv), sc[j]));
      yr[static_cast<size_t>(j) * a.N] = *reinterpret_cast<const uint16_t*>(&h);
      if (ar) ar[static_cast<size_t>(j) * a.N] = tv;
    }
    return;
  }
#pragma unroll
  for (int j = 0; j < 32; ++j) {  // static indices keep v in registers
    if (j >= ntok) break;
    const int32_t tv = static_cast<int32_t>(v[j]) - rsm[j];
    const __nv_bfloat16 h = __float2bfloat16_rn(__fmul_rn(static_cast<float>(tv), scl[j]));
    yr[static_cast<size_t>(j) * a.N] = *reinterpret_cast<const uint16_t*>(&h);
    if (ar) ar[static_cast<size_t>(j) * a.N] = tv;
  }
}

// The 16 codes of one dense code word (weight k of the 16-group at bits
// 2k .. 2k + 1) as bytes in natural k order: o[m] byte b = code of weight
// 4m + b.  (w >> 2j) & 0x03030303 gives byte b = code of weight 4b + j; the
// byte permutes transpose that 4 x 4 arrangement.
__device__ __forceinline__ void codes_word_natural(uint32_t w, uint32_t* o) {
  const uint32_t s0 = w & 0x03030303u, s1 = (w >> 2) & 0x03030303u;
  const uint32_t s2 = (w >> 4) & 0x03030303u, s3 = (w >> 6) & 0x03030303u;
  const uint32_t t0 = __byte_perm(s0, s1, 0x5140), t1 = __byte_perm(s0, s1, 0x7362);
  const uint32_t t2 = __byte_perm(s2, s3, 0x5140), t3 = __byte_perm(s2, s3, 0x7362);
  o[0] = __byte_perm(t0, t2, 0x5410);
  o[1] = __byte_perm(t0, t2, 0x7632);
  o[2] = __byte_perm(t1, t3, 0x5410);
  o[3] = __byte_perm(t1, t3, 0x7632);
}

template <int BN, int NM>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap mapB, const __grid_constant__ CUtensorMap mapA,
                   const __grid_constant__ CUtensorMap mapMeta, const TcArgs a) {
  constexpr int S = tc_stages(BN, NM);
  constexpr int KSUB = tc_ksub(NM, BN);
  constexpr int SLOT = tc_slot_cols(NM, BN);
  constexpr int DCOLS = TcCols<BN, NM>::kDcols;
  constexpr int A_COL0 = TcCols<BN, NM>::kAcol0;
  constexpr int NCOLS = TcCols<BN, NM>::kAlloc;
  constexpr bool SP = NM == 3;  // 2:4 rows on the structured-sparse MMA
  static_assert(!SP || KSUB == 2, "the sparse stage is one 128-byte swizzle row of kept values");
  constexpr uint32_t IDESC = SP ? idesc_i8_sp_s8s8(kTcRows, BN) : idesc_i8_u8s8(kTcRows, BN);

  constexpr int B_SUB = BN * 128;         // one 128-wide K sub-tile of the activations
  constexpr int B_STAGE = B_SUB * KSUB;

  extern __shared__ uint8_t smem_raw[];
  // offset arithmetic on the shared array keeps every derived pointer in the shared window
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int a_val_bytes = TcStageBytes<NM, BN>::a_values(a.vbox);
  const int a_meta_bytes = TcStageBytes<NM, BN>::a_meta();
  const int a_stage = tc_a_stage_bytes(NM, BN, a.vbox);
  uint8_t* sB = base;
  uint8_t* sA = base + S * B_STAGE;
  // sparse MMA: stage s of sA is the compressed operand [128 rows][128 B] once unpacked
  uint32_t* s_lut = reinterpret_cast<uint32_t*>(sA + S * a_stage);     // expanded 2:4 only: [256][32] code bytes
  uint32_t* s_stage = s_lut + (NM == 1 ? kNmLutWords : 0);               // 4 warps x 32 x 33 words
  float* s_scale = reinterpret_cast<float*>(s_stage + 4 * 32 * 33);     // [2][BN]
  int32_t* s_rowsum = reinterpret_cast<int32_t*>(s_scale + 2 * BN);     // [2][BN]
  uint64_t* full = reinterpret_cast<uint64_t*>(s_rowsum + 2 * BN);
  uint64_t* empty = full + S;
  uint64_t* aready = empty + S;
  uint64_t* accfull = aready + S;   // [2]
  uint64_t* accempty = accfull + 2; // [2]
  uint64_t* drain = accempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* s_last = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = a.kbs;  // k-blocks per unit
  const int nunits = a.row_tiles * a.tok_tiles * a.ksplit;
  const int my_tiles = blockIdx.x < nunits ? (nunits - 1 - blockIdx.x) / gridDim.x + 1 : 0;  // units of this CTA
  const int total_kb = my_tiles * KB;  // k-blocks this CTA streams
  const uint32_t tx_bytes = static_cast<uint32_t>(B_STAGE + a_val_bytes + a_meta_bytes);
  // unit t of this CTA -> (row tile, token tile, K slice), slice fastest, then token tile
  auto unit_of = [&](int t, int& rt, int& tt, int& ks) {
    const int g = blockIdx.x + t * gridDim.x;
    const int tile = g / a.ksplit;
    ks = g - tile * a.ksplit;
    rt = tile / a.tok_tiles;
    tt = tile - rt * a.tok_tiles;
  };
  // absolute k-block of the i-th k-block this CTA streams (slices past K read zeros)
  auto kblock_of = [&](int i, int& rt, int& tt) {
    int ks;
    unit_of(i / KB, rt, tt, ks);
    return ks * KB + i % KB;
  };

  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&aready[s], 4);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], 4);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&mapB);
    tma_prefetch_desc(&mapA);
    if (NM != 0) tma_prefetch_desc(&mapMeta);
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, NCOLS);
    tmem_relinquish();
  }
  if (NM == 1) nm24_fill_lut(s_lut);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0 && total_kb > 0) {
      // ------------------------------------------------------------ producer
      auto load_a = [&](int row0, int kb, int s) {
        uint8_t* dst = sA + s * a_stage;
        if (NM == 0) {
          tma_load_2d(dst, &mapA, kb * 32 * KSUB, row0, &full[s]);
        } else if (NM == 1 || NM == 3) {
          tma_load_2d(dst, &mapA, kb * 16 * KSUB, row0, &full[s]);
          tma_load_2d(dst + a_val_bytes, &mapMeta, kb * 16 * KSUB, row0, &full[s]);
        } else {
          tma_load_2d(dst, &mapA, (kb * 4 * a.nm_n) & ~15, row0, &full[s]);
          tma_load_2d(dst + a_val_bytes, &mapMeta, kb * 16, row0, &full[s]);
        }
      };
      const int pre = total_kb < S ? total_kb : S;
      // Weights do not depend on the preceding kernel: start them first.
      for (int i = 0; i < pre; ++i) {
        int rt, tt;
        const int kb = kblock_of(i, rt, tt);
        mbar_arrive_expect_tx(&full[i], tx_bytes);
        load_a(rt * kTcRows, kb, i);
      }
      pdl_wait_primary();
      for (int i = 0; i < pre; ++i) {
        int rt, tt;
        const int kb = kblock_of(i, rt, tt);
        for (int sub = 0; sub < KSUB; ++sub)
          tma_load_2d(sB + i * B_STAGE + sub * B_SUB, &mapB, (kb * KSUB + sub) * kTcSubK, tt * BN, &full[i]);
      }
      bool ok = true;
      int i = pre;
      for (; i < total_kb; ++i) {
        const int s = i % S;
        if (!mbar_wait(&empty[s], ((i / S) - 1) & 1)) {
          *a.status = kDevTimeoutProducer;
          ok = false;
          break;
        }
        int rt, tt;
        const int kb = kblock_of(i, rt, tt);
        mbar_arrive_expect_tx(&full[s], tx_bytes);
        load_a(rt * kTcRows, kb, s);
        for (int sub = 0; sub < KSUB; ++sub)
          tma_load_2d(sB + s * B_STAGE + sub * B_SUB, &mapB, (kb * KSUB + sub) * kTcSubK, tt * BN, &full[s]);
      }
      if (!ok) {
        // Let the copies already issued land before the CTA exits.
        for (int j = (i - S > 0 ? i - S : 0); j < i; ++j)
          if (!mbar_wait(&full[j % S], (j / S) & 1)) *a.status = kDevTimeoutDrain;
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && total_kb > 0) {
      // ------------------------------------------------------------ MMA issuer
      bool issued = false, ok = true;
      for (int t = 0; t < my_tiles && ok; ++t) {
        const int buf = t & 1;
        if (t >= 2 && !mbar_wait(&accempty[buf], ((t >> 1) - 1) & 1)) {
          *a.status = kDevTimeoutMma;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dcol = tmem + buf * DCOLS;
        for (int kb = 0; kb < KB; ++kb) {
          const int i = t * KB + kb;
          const int s = i % S;
          const uint32_t par = (i / S) & 1;
          if (!mbar_wait(&full[s], par) || !mbar_wait(&aready[s], par)) {
            *a.status = kDevTimeoutMma;
            ok = false;
            break;
          }
          tc_fence_after();
          if (SP) {
            // four instructions of 64 k: 32 bytes of kept values, two metadata columns, 64 bytes of B each
            const uint64_t adesc = smem_desc_sw128_kmajor(smem_u32(sA + s * a_stage));
#pragma unroll
            for (int kk = 0; kk < 2 * KSUB; ++kk) {
              const uint64_t bdesc = smem_desc_sw128_kmajor(smem_u32(sB + s * B_STAGE + (kk >> 1) * B_SUB));
              tc_mma_sp_i8_ss(dcol, adesc + static_cast<uint64_t>(kk * 2), bdesc + static_cast<uint64_t>((kk & 1) * 4),
                              tmem + A_COL0 + s * SLOT + kk * 2, IDESC, (kb | kk) != 0 ? 1u : 0u);
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < 4 * KSUB; ++kk) {
              const uint64_t bdesc = smem_desc_sw128_kmajor(smem_u32(sB + s * B_STAGE + (kk >> 2) * B_SUB));
              tc_mma_i8_ts(dcol, tmem + A_COL0 + s * SLOT + kk * 8, bdesc + static_cast<uint64_t>((kk & 3) * 2),
                           IDESC, (kb | kk) != 0 ? 1u : 0u);
            }
          }
          tc_commit(&empty[s]);
          issued = true;
        }
        if (ok) tc_commit(&accfull[buf]);
      }
      if (!ok && issued) {
        tc_commit(drain);
        if (!mbar_wait(drain, 0)) *a.status = kDevTimeoutDrain;
      }
    }
  } else if (warp >= 4 && warp < kTcEpiWarp0) {
    // -------------------------------------------------------------- unpack (two groups)
    // A group takes every use of the stages of its parity, so its parity waits on a
    // stage never skip a phase.  (Alternating k-blocks would, with an odd stage
    // count, hand each stage to the two groups in turn, and a group could pass
    // the wait on a phase that completed two uses earlier.)
    const int grp = (warp - 4) >> 2;       // 0: even stages, 1: odd stages
    const int q = warp & 3;                // TMEM lane quarter
    const int r = q * 32 + lane;           // weight row inside the tile
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    for (int i = 0; i < total_kb; ++i) {
      const int s = i % S;
      if ((s & 1) != grp) continue;
      int rt_u, tt_u;
      const int kb = kblock_of(i, rt_u, tt_u);
      bool landed = mbar_wait(&full[s], (i / S) & 1);
      // sparse MMA: the group's four warps unpack over a shared buffer, so they give up together
      if (SP) landed = bar_red_and(landed, 2 + grp, 128);
      if (!landed) {
        *a.status = kDevTimeoutUnpack;
        break;
      }
      uint8_t* st = sA + s * a_stage;
      if (SP) {
        // 32 bytes of kept codes (128 kept values, 256 k) and 32 of metadata for this row; every
        // row of the group is read before any is overwritten by the compressed operand
        const uint4* vp = reinterpret_cast<const uint4*>(st + r * 32);
        const uint4* mp = reinterpret_cast<const uint4*>(st + a_val_bytes + r * 32);
        const uint4 v0 = vp[0], v1 = vp[1], m0 = mp[0], m1 = mp[1];
        const uint32_t vw[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        const uint32_t mw[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
        bar_sync_n(2 + grp, 128);
        uint8_t* arow_s = st + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          // 16 kept codes (32 k) -> 16 int8 weights W_t = code - 1 in kept order: the 16-byte chunk c
          // of the row's 128-byte swizzle row
          uint32_t sj[4];
#pragma unroll
          for (int j = 0; j < 4; ++j)  // byte b of sj[j]: kept value 4b + j, as 0x80 + code - 1
            sj[j] = (((vw[c] >> (2 * j)) & 0x03030303u) | 0x80808080u) - 0x01010101u;
          const uint32_t t0 = __byte_perm(sj[0], sj[1], 0x5140), t1 = __byte_perm(sj[0], sj[1], 0x7362);
          const uint32_t t2 = __byte_perm(sj[2], sj[3], 0x5140), t3 = __byte_perm(sj[2], sj[3], 0x7362);
          const uint4 o = make_uint4(__byte_perm(t0, t2, 0x5410) ^ 0x80808080u, __byte_perm(t0, t2, 0x7632) ^ 0x80808080u,
                                     __byte_perm(t1, t3, 0x5410) ^ 0x80808080u, __byte_perm(t1, t3, 0x7632) ^ 0x80808080u);
          *reinterpret_cast<uint4*>(arow_s + ((c ^ (r & 7)) << 4)) = o;
        }
        tc_st_32x32b_x8(tmem + lane_base + A_COL0 + s * SLOT, mw);
        fence_proxy_async_smem();  // the compressed A is read by the tensor cores
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&aready[s]);
        continue;
      }
      const uint8_t* arow;
      const uint8_t* mrow = st + a_val_bytes + r * 16 * KSUB;
      int rem = 0;
      if (NM == 0)
        arow = st + r * 32 * KSUB;
      else if (NM == 1)
        arow = st + r * 16 * KSUB;
      else {
        arow = st + r * a.vbox;
        rem = (kb * 4 * a.nm_n) & 15;
      }
#pragma unroll
      for (int sub = 0; sub < KSUB; ++sub) {
        uint32_t dw[8];
        if (NM == 0) {
          const uint4 lo = reinterpret_cast<const uint4*>(arow)[2 * sub];
          const uint4 hi = reinterpret_cast<const uint4*>(arow)[2 * sub + 1];
          dw[0] = lo.x; dw[1] = lo.y; dw[2] = lo.z; dw[3] = lo.w;
          dw[4] = hi.x; dw[5] = hi.y; dw[6] = hi.z; dw[7] = hi.w;
        } else if (NM == 1) {
          // 16 bytes of kept codes and 16 of metadata per row and sub-tile: 8 groups of 16 weights
          const uint4 vv = reinterpret_cast<const uint4*>(arow)[sub];
          const uint4 mm = reinterpret_cast<const uint4*>(mrow)[sub];
          const uint32_t vw[4] = {vv.x, vv.y, vv.z, vv.w}, mw[4] = {mm.x, mm.y, mm.z, mm.w};
          const uint32_t* lut_lane = s_lut + lane;
#pragma unroll
          for (int gi = 0; gi < 8; ++gi)
            dw[gi] = nm24_word_lut(lut_lane, (mw[gi >> 1] >> (16 * (gi & 1))) & 0xFFFFu,
                                   (vw[gi >> 1] >> (16 * (gi & 1))) & 0xFFFFu);
        } else {
#pragma unroll
          for (int gi = 0; gi < 8; ++gi) dw[gi] = tc_n8_group_word(arow, mrow, gi, a.nm_n, rem);
        }
        uint32_t outw[32];
#pragma unroll
        for (int gi = 0; gi < 8; ++gi) codes_word_natural(dw[gi], outw + 4 * gi);
        tc_st_32x32b_x32(tmem + lane_base + A_COL0 + s * SLOT + sub * 32, outw);
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&aready[s]);
    }
  } else if (warp >= kTcEpiWarp0) {
    // -------------------------------------------------------------- epilogue
    const int q = warp - kTcEpiWarp0;       // TMEM lane quarter = 32-row block of the tile
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    uint32_t* stg = s_stage + q * 32 * 33;
    const float alpha = *a.alpha;
    pdl_wait_primary();
    for (int t = 0; t < my_tiles; ++t) {
      const int buf = t & 1;
      int rt, tt, ks;
      unit_of(t, rt, tt, ks);
      const int row0 = rt * kTcRows + q * 32;
      const int tok0 = tt * BN;
      float* scl = s_scale + buf * BN;
      int32_t* rsm = s_rowsum + buf * BN;
      if (a.ksplit > 1) {
        // ---- K slice: add the partial sums into the tile's fp32 sums; the last slice finishes the tile
        if (!mbar_wait(&accfull[buf], (t >> 1) & 1)) {
          *a.status = kDevTimeoutEpilogue;
          break;
        }
        tc_fence_after();
        const bool vec = (a.N % 4) == 0 && row0 + 32 <= a.N;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 32) {
          uint32_t v[32];
          tc_ld_32x32b_x32(tmem + lane_base + buf * DCOLS + c0, v);
          tc_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) stg[j * 33 + lane] = v[j];
          __syncwarp();
          const int tcol = c0 + lane;  // lane l now holds token c0 + l, rows row0 .. row0 + 31
          const int tok = tok0 + tcol;
          if (tcol < BN && tok < a.M && row0 < a.N) {
            float* dst = a.part + static_cast<size_t>(tok) * a.N + row0;
            const uint32_t* src = stg + lane * 33;
            if (vec) {
#pragma unroll
              for (int e = 0; e < 32; e += 4)
                red_add_v4_f32(dst + e, static_cast<float>(static_cast<int32_t>(src[e])),
                               static_cast<float>(static_cast<int32_t>(src[e + 1])),
                               static_cast<float>(static_cast<int32_t>(src[e + 2])),
                               static_cast<float>(static_cast<int32_t>(src[e + 3])));
            } else {
              for (int e = 0; e < 32 && row0 + e < a.N; ++e)
                atomicAdd(dst + e, static_cast<float>(static_cast<int32_t>(src[e])));
            }
          }
          __syncwarp();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&accempty[buf]);
        __threadfence();
        const int tile = rt * a.tok_tiles + tt;
        for (int j = threadIdx.x - kTcEpiWarp0 * 32; j < BN; j += 128) {
          const int tok = tok0 + j;
          scl[j] = tok < a.M ? __fdiv_rn(__fmul_rn(alpha, a.gamma[tok]), a.qb) : 0.0f;  // RN(RN(alpha gamma) / Q_b)
          rsm[j] = (tok < a.M && a.rowsum) ? a.rowsum[tok] : 0;
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (threadIdx.x == kTcEpiWarp0 * 32)
          *s_last = (atomicAdd(&a.cnt[tile], 1u) == static_cast<uint32_t>(a.ksplit - 1)) ? 1 : 0;
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (*s_last) {
          __threadfence();
          if (threadIdx.x == kTcEpiWarp0 * 32) a.cnt[tile] = 0u;  // left zero for the next GEMM
#pragma unroll 1
          for (int c0 = 0; c0 < BN; c0 += 32) {
            const int tcol = c0 + lane;
            const int tok = tok0 + tcol;
            if (tcol < BN && tok < a.M && row0 < a.N) {
              float* srcp = a.part + static_cast<size_t>(tok) * a.N + row0;
              const float sc = scl[tcol];
              const int32_t rs = rsm[tcol];
              const size_t o = static_cast<size_t>(tok) * a.N + row0;
              if (vec) {
                int32_t tv[32];
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                  const float4 f = __ldcg(reinterpret_cast<const float4*>(srcp + e));
                  tv[e] = __float2int_rn(f.x) - rs;
                  tv[e + 1] = __float2int_rn(f.y) - rs;
                  tv[e + 2] = __float2int_rn(f.z) - rs;
                  tv[e + 3] = __float2int_rn(f.w) - rs;
                  __stcg(reinterpret_cast<float4*>(srcp + e), make_float4(0.f, 0.f, 0.f, 0.f));
                }
                if (a.vec_store) {
                  uint32_t hb[16];
#pragma unroll
                  for (int e = 0; e < 32; e += 2) {
                    const __nv_bfloat16 h0 = __float2bfloat16_rn(__fmul_rn(static_cast<float>(tv[e]), sc));
                    const __nv_bfloat16 h1 = __float2bfloat16_rn(__fmul_rn(static_cast<float>(tv[e + 1]), sc));
                    hb[e >> 1] = static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(&h0)) |
                                 (static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(&h1)) << 16);
                  }
                  uint4* dy = reinterpret_cast<uint4*>(a.y + o);
#pragma unroll
                  for (int e = 0; e < 4; ++e) dy[e] = make_uint4(hb[4 * e], hb[4 * e + 1], hb[4 * e + 2], hb[4 * e + 3]);
                  if (a.acc) {
                    uint4* da = reinterpret_cast<uint4*>(a.acc + o);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                      da[e] = make_uint4(static_cast<uint32_t>(tv[4 * e]), static_cast<uint32_t>(tv[4 * e + 1]),
                                         static_cast<uint32_t>(tv[4 * e + 2]), static_cast<uint32_t>(tv[4 * e + 3]));
                  }
                } else {
#pragma unroll
                  for (int e = 0; e < 32; ++e) {
                    if (a.acc) a.acc[o + e] = tv[e];
                    const __nv_bfloat16 h = __float2bfloat16_rn(__fmul_rn(static_cast<float>(tv[e]), sc));
                    a.y[o + e] = *reinterpret_cast<const uint16_t*>(&h);
                  }
                }
              } else {
                for (int e = 0; e < 32 && row0 + e < a.N; ++e) {
                  const int32_t tv = __float2int_rn(__ldcg(srcp + e)) - rs;
                  __stcg(srcp + e, 0.0f);
                  if (a.acc) a.acc[o + e] = tv;
                  const __nv_bfloat16 h = __float2bfloat16_rn(__fmul_rn(static_cast<float>(tv), sc));
                  a.y[o + e] = *reinterpret_cast<const uint16_t*>(&h);
                }
              }
            }
          }
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");  // s_last and the scales are read before the next unit
        continue;
      }
      for (int j = threadIdx.x - kTcEpiWarp0 * 32; j < BN; j += 128) {
        const int tok = tok0 + j;
        scl[j] = tok < a.M ? __fdiv_rn(__fmul_rn(alpha, a.gamma[tok]), a.qb) : 0.0f;  // RN(RN(alpha gamma) / Q_b)
        rsm[j] = (tok < a.M && a.rowsum) ? a.rowsum[tok] : 0;
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (!mbar_wait(&accfull[buf], (t >> 1) & 1)) {
        *a.status = kDevTimeoutEpilogue;
        break;
      }
      tc_fence_after();
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t v[32];
        tc_ld_32x32b_x32(tmem + lane_base + buf * DCOLS + c0, v);
        tc_wait_ld();
        tc_store_token_rows(v, scl + c0, rsm + c0, row0 + lane, tok0 + c0, BN - c0 < 32 ? BN - c0 : 32, a);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[buf]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, NCOLS);
  }
}


}  // namespace bl
