// gemm_tc.cuh -- many-token BitLinear on the 5th-generation tensor cores.
//
// The 2B4T report (section 5.1) stages packed ternary weights on chip,
// unpacks them and multiplies them with 8-bit activations.  On sm_100a that
// becomes one tcgen05 kind::i8 contraction per CTA tile:
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
// Both operands use the same K order inside each 16-wide group (byte 4j + b
// holds k = 4b + j), which is the order (w >> 2j) & 0x03030303 produces.
//
// Roles (256 threads): warp 0 lane 0 issues TMA loads, warp 1 lane 0 issues
// the MMAs, warp 2 owns the TMEM allocation, warps 4..7 unpack weights and
// run the epilogue (warp w reaches TMEM lanes 32 * (w % 4) .. + 31).
// A four-stage mbarrier ring couples them: full (TMA bytes landed), aready
// (A slot written), empty (MMAs that read the stage completed).  Every wait is
// bounded; a role that gives up records a status code and unwinds.
//
// N:M weights (Sparse-BitNet, section 3.2) are expanded from kept values +
// metadata into the same dense code words before the tcgen05.st, so the MMA
// is the dense one.
#pragma once
#include "gemv.cuh"

namespace bl {

constexpr int kTcStages = 4;
constexpr int kTcBK = 128;      // K elements per stage (one 128-byte swizzle row)
constexpr int kTcRows = 128;    // weight rows per CTA (MMA M)
constexpr int kTcThreads = 256;

struct TcArgs {
  int M, N, K;
  int kblocks;            // ceil(K / 128)
  const float* scale;     // [M] per-token rescale RN(RN(alpha * gamma) / 127)
  const int32_t* rowsum;  // [M] sum of the token's codes
  uint16_t* y;            // [M, N] bf16 bits
  int32_t* acc;           // [M, N] or null
  int nm_n;               // kept per 8-block (n:8 mode)
  int vbox;               // n:8: bytes of the values box per row
  int32_t* status;        // device status word
};

template <int NM>
struct TcStageBytes {
  // packed A bytes per stage (TMA box bytes, rows = 128)
  static __host__ __device__ constexpr int a_values(int vbox) {
    return NM == 0 ? kTcRows * 32 : (NM == 1 ? kTcRows * 16 : kTcRows * vbox);
  }
  static __host__ __device__ constexpr int a_meta() { return NM == 0 ? 0 : kTcRows * 16; }
};

template <int BN>
struct TcCols {
  static constexpr int kAcol0 = BN < 32 ? 32 : BN;
  static constexpr int kNeed = kAcol0 + kTcStages * 32;
  static constexpr int kAlloc = kNeed <= 128 ? 128 : (kNeed <= 256 ? 256 : 512);
};

__host__ __device__ constexpr int tc_smem_bytes(int BN, int NM, int vbox) {
  const int a_bytes = (NM == 0 ? kTcRows * 32 : (NM == 1 ? kTcRows * 16 : kTcRows * vbox)) + (NM == 0 ? 0 : kTcRows * 16);
  const int a_stage = (a_bytes + 1023) / 1024 * 1024;
  return 1024 /* alignment slack */ + kTcStages * (BN * 128 + a_stage) + 1024 /* barriers, scales */ + BN * 8;
}

// Dense code word of 16 weights for the current stage and group, per mode.
template <int NM>
__device__ __forceinline__ uint32_t tc_group_word(const uint8_t* arow, const uint8_t* mrow, int gi, int n,
                                                  int rem) {
  if (NM == 0) {
    return reinterpret_cast<const uint32_t*>(arow)[gi];
  } else if (NM == 1) {
    const uint32_t meta16 = reinterpret_cast<const uint16_t*>(mrow)[gi];
    const uint32_t vals16 = reinterpret_cast<const uint16_t*>(arow)[gi];
    return nm24_dense_word(meta16, vals16);
  } else {
    const uint32_t m0 = mrow[2 * gi], m1 = mrow[2 * gi + 1];
    const int bit = rem * 8 + gi * 4 * n;  // two blocks of n kept codes
    const uint32_t* p = reinterpret_cast<const uint32_t*>(arow);
    const int wi = bit >> 5, sh = bit & 31;
    uint32_t kv = p[wi] >> sh;
    if (sh != 0 && sh + 4 * n > 32) kv |= p[wi + 1] << (32 - sh);
    const uint32_t fmask = (1u << (2 * n)) - 1u;
    return n8_dense_block(m0, kv & fmask) | (n8_dense_block(m1, (kv >> (2 * n)) & fmask) << 16);
  }
}

template <int BN, int NM>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap mapB, const __grid_constant__ CUtensorMap mapA,
                   const __grid_constant__ CUtensorMap mapMeta, const TcArgs a) {
  constexpr int S = kTcStages;
  constexpr int A_COL0 = TcCols<BN>::kAcol0;
  constexpr int NCOLS = TcCols<BN>::kAlloc;
  constexpr uint32_t IDESC = idesc_i8_u8s8(kTcRows, BN);
  constexpr int B_STAGE = BN * 128;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int a_val_bytes = TcStageBytes<NM>::a_values(a.vbox);
  const int a_meta_bytes = TcStageBytes<NM>::a_meta();
  const int a_stage = (a_val_bytes + a_meta_bytes + 1023) / 1024 * 1024;
  uint8_t* sB = base;
  uint8_t* sA = base + S * B_STAGE;
  uint8_t* misc = sA + S * a_stage;
  uint64_t* full = reinterpret_cast<uint64_t*>(misc);
  uint64_t* empty = full + S;
  uint64_t* aready = empty + S;
  uint64_t* accfull = aready + S;
  uint64_t* drain = accfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  float* s_scale = reinterpret_cast<float*>(misc + 256);
  int32_t* s_rowsum = reinterpret_cast<int32_t*>(s_scale + BN);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * kTcRows;
  const int tok0 = blockIdx.y * BN;
  const int KB = a.kblocks;
  const uint32_t tx_bytes = static_cast<uint32_t>(B_STAGE + a_val_bytes + a_meta_bytes);

  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&aready[s], 4);
    }
    mbar_init(accfull, 1);
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- producer
      auto load_a = [&](int kb, int s) {
        uint8_t* dst = sA + s * a_stage;
        if (NM == 0) {
          tma_load_2d(dst, &mapA, kb * 32, row0, &full[s]);
        } else if (NM == 1) {
          tma_load_2d(dst, &mapA, kb * 16, row0, &full[s]);
          tma_load_2d(dst + a_val_bytes, &mapMeta, kb * 16, row0, &full[s]);
        } else {
          const int x0 = (kb * 4 * a.nm_n) & ~15;
          tma_load_2d(dst, &mapA, x0, row0, &full[s]);
          tma_load_2d(dst + a_val_bytes, &mapMeta, kb * 16, row0, &full[s]);
        }
      };
      const int pre = KB < S ? KB : S;
      // Weights do not depend on the preceding kernel: start them first.
      for (int kb = 0; kb < pre; ++kb) {
        mbar_arrive_expect_tx(&full[kb], tx_bytes);
        load_a(kb, kb);
      }
      pdl_wait_primary();
      for (int kb = 0; kb < pre; ++kb) tma_load_2d(sB + kb * B_STAGE, &mapB, kb * kTcBK, tok0, &full[kb]);
      bool ok = true;
      int kb = pre;
      for (; kb < KB; ++kb) {
        const int s = kb % S, round = kb / S;
        if (!mbar_wait(&empty[s], (round - 1) & 1)) {
          *a.status = kDevTimeoutProducer;
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[s], tx_bytes);
        load_a(kb, s);
        tma_load_2d(sB + s * B_STAGE, &mapB, kb * kTcBK, tok0, &full[s]);
      }
      if (!ok) {
        // Let the copies already issued land before the CTA exits.
        for (int j = (kb - S > 0 ? kb - S : 0); j < kb; ++j)
          if (!mbar_wait(&full[j % S], (j / S) & 1)) *a.status = kDevTimeoutDrain;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      bool issued = false, ok = true;
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % S;
        const uint32_t par = (kb / S) & 1;
        if (!mbar_wait(&full[s], par) || !mbar_wait(&aready[s], par)) {
          *a.status = kDevTimeoutMma;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t bdesc = smem_desc_sw128_kmajor(smem_u32(sB + s * B_STAGE));
#pragma unroll
        for (int kk = 0; kk < kTcBK / 32; ++kk) {
          tc_mma_i8_ts(tmem, tmem + A_COL0 + s * 32 + kk * 8, bdesc + static_cast<uint64_t>(kk * 2), IDESC,
                       (kb | kk) != 0 ? 1u : 0u);
        }
        tc_commit(&empty[s]);
        issued = true;
      }
      if (ok) {
        tc_commit(accfull);
      } else if (issued) {
        tc_commit(drain);
        if (!mbar_wait(drain, 0)) *a.status = kDevTimeoutDrain;
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ unpack
    const int q = warp - 4;               // TMEM lane quarter
    const int r = q * 32 + lane;          // weight row inside the tile
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    pdl_wait_primary();
    for (int t = threadIdx.x - 128; t < BN; t += 128) {
      const int tok = tok0 + t;
      s_scale[t] = tok < a.M ? a.scale[tok] : 0.0f;
      s_rowsum[t] = tok < a.M ? a.rowsum[tok] : 0;
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    bool ok = true;
    for (int kb = 0; kb < KB; ++kb) {
      const int s = kb % S;
      const uint32_t par = (kb / S) & 1;
      if (!mbar_wait(&full[s], par)) {
        *a.status = kDevTimeoutUnpack;
        ok = false;
        break;
      }
      const uint8_t* st = sA + s * a_stage;
      const uint8_t* arow;
      const uint8_t* mrow = st + a_val_bytes + r * 16;
      int rem = 0;
      if (NM == 0)
        arow = st + r * 32;
      else if (NM == 1)
        arow = st + r * 16;
      else {
        arow = st + r * a.vbox;
        rem = (kb * 4 * a.nm_n) & 15;
      }
      uint32_t outw[32];
      uint32_t dw[8];
      if (NM == 0) {
        const uint4 lo = reinterpret_cast<const uint4*>(arow)[0];
        const uint4 hi = reinterpret_cast<const uint4*>(arow)[1];
        dw[0] = lo.x; dw[1] = lo.y; dw[2] = lo.z; dw[3] = lo.w;
        dw[4] = hi.x; dw[5] = hi.y; dw[6] = hi.z; dw[7] = hi.w;
      } else {
#pragma unroll
        for (int gi = 0; gi < 8; ++gi) dw[gi] = tc_group_word<NM>(arow, mrow, gi, a.nm_n, rem);
      }
#pragma unroll
      for (int gi = 0; gi < 8; ++gi) {
#pragma unroll
        for (int j = 0; j < 4; ++j) outw[4 * gi + j] = (dw[gi] >> (2 * j)) & 0x03030303u;
      }
      tc_st_32x32b_x32(tmem + lane_base + A_COL0 + s * 32, outw);
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&aready[s]);
    }
    // ------------------------------------------------------------ epilogue
    if (ok) {
      if (!mbar_wait(accfull, 0)) {
        *a.status = kDevTimeoutEpilogue;
        ok = false;
      }
    }
    tc_fence_after();
    if (ok) {
      const int row = row0 + r;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t v[32];
        tc_ld_32x32b_x32(tmem + lane_base + c0, v);
        tc_wait_ld();
        if (row < a.N) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int t = c0 + j;
            const int tok = tok0 + t;
            if (t < BN && tok < a.M) {
              const int32_t total = static_cast<int32_t>(v[j]) - s_rowsum[t];
              const size_t o = static_cast<size_t>(tok) * a.N + row;
              if (a.acc) a.acc[o] = total;
              const __nv_bfloat16 h = __float2bfloat16_rn(__fmul_rn(static_cast<float>(total), s_scale[t]));
              a.y[o] = *reinterpret_cast<const uint16_t*>(&h);
            }
          }
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, NCOLS);
  }
}

}  // namespace bl
