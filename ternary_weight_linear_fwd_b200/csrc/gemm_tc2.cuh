// gemm_tc2.cuh -- many-token BitLinear on pairs of SMs (tcgen05 cta_group::2).
//
// The persistent GEMM of gemm_tc.cuh reads, for every 128-row weight tile, the
// whole activation tile of its tokens from L2: at 128 x 128 tiles the
// activations are four fifths of the bytes a stage moves, and a copy of the
// kernel that skipped both the MMAs and the unpacking still took four fifths
// of the full kernel's time (2048 -> 11008 at M = 4096).  Here two CTAs of a
// cluster share one MMA of M = 256 weight rows: each CTA holds its own 128
// weight rows (expanded codes in its TMEM or shared memory for dense and n:8
// weights, the compressed kept values in its shared memory for 2:4 weights)
// and HALF of the BN tokens' activation tile, so the activation bytes per MAC
// halve.
//
//   D[256 rows, BN tokens] += A[256 rows, K] * B[BN tokens, K]^T
//   CTA r of the pair: rows 128 r .. 128 r + 127 of A and D (its own TMEM),
//                      tokens BN/2 r .. BN/2 r + BN/2 - 1 of B (its own shared memory).
// Token tiles: BN = 128, 160, 192 or 224, picked on the host by how many rounds of
// pairs a shape takes.  Narrower tiles did less work per k-block in nearly the
// same time (the k-block's cost is mostly per MMA instruction and per
// hand-off).  Dense weights at BN = 128 keep their expanded codes in TMEM
// (the MMA's A from TMEM, 512-k stages); wider tiles leave TMEM no room for
// operand slots beside two accumulators, so there the codes go to shared
// memory like the 2:4 kept values (A from shared memory, 256-k stages).  An
// A operand in shared memory is read again by every MMA; a wider token tile
// spreads that read over more tokens.
//
// Two rings: S copy stages in shared memory (the CTA's half of the activation
// tile and its packed weights) and R operand slots (expanded codes in TMEM, or
// compressed kept values in shared memory plus metadata in TMEM).  A copy
// stage is freed when the MMAs that read its activations complete, an operand
// slot likewise (one commit per k-block serves both); S > R lets the copies
// run further ahead of the MMAs than the operand slots alone would allow.
//
// Every copy is an ordinary one-CTA TMA load signalling the CTA's own
// barrier.  The unpack warps of both CTAs wait for their CTA's stage (weights
// and activations landed), unpack, and arrive on the MMA barrier of the pair's
// rank-0 CTA (tcgen05 / async-proxy fences first, then a CTA-scope release
// arrive: a cluster-scope release cost about 1500 cycles per arrive and made
// the unpacking the bottleneck); rank 0's MMA thread waits there (acquire at
// cluster scope), issues the pair MMAs and commits them to the stage's "empty"
// barrier of both CTAs at once (multicast commit), which frees the stage for
// both producers.  The accumulators work the same way: the commit of a tile
// reaches both CTAs' epilogues, and both epilogues arrive on rank 0's
// "accumulator free" barrier.  Each CTA's epilogue stores its own 128 rows.
// Every wait is bounded; a role that gives up records a status and unwinds,
// and neither CTA leaves before the other (final cluster barrier), so no
// remote arrive or multicast commit reaches an exited CTA.
#pragma once
#include "gemm_tc.cuh"

namespace bl {

constexpr int kT2Rows = 256;     // weight rows of a pair tile (the MMA's M)

// n:8 expansion.  Selectors of the two byte permutes that turn the spread
// kept codes of one 8-block (bytes 0 .. n-1: kept codes in k order, byte 7:
// code 1) into its eight codes: output byte p takes kept code j when p is the
// j-th set bit of the mask, byte 7 (code 1, weight 0) when p is pruned.
// Low 16 bits: positions 0..3; high 16 bits: positions 4..7.
__device__ __forceinline__ uint32_t n8_perm_selectors(uint32_t mask) {
  uint32_t sel = 0u, j = 0u;
  for (int p = 0; p < 8; ++p) {
    uint32_t nib = 7u;
    if ((mask >> p) & 1u) nib = j < 7u ? j++ : 7u;
    sel |= nib << (4 * p);
  }
  return sel;
}

// One weight row of an n:8 stage (SUBS x 128 k) into its operand slot: u8
// codes in natural k order, either to TMEM (four stores of 128 k) or to the
// 128-byte-swizzled shared-memory operand (orow: the row's line in the first
// 128-k column; chunk g of a column at g ^ (r % 8)).  The row's kept codes
// (4 SUBS n bytes, 2 n bits per 8-block, blocks in k order) are read with
// 16-byte loads into registers, the masks (one byte per 8-block) 16 bytes per
// 128 k.  n is a compile-time constant, so every block's bit offset is one.
template <int NK, int SUBS, bool SMEM>
__device__ __forceinline__ void n8_unpack_row(const uint8_t* vals, const uint8_t* masks, int r, const uint32_t* s_sel,
                                              uint32_t taddr, uint8_t* orow);

// The eight codes of one 8-block (natural k order, one byte each) from its
// kept codes (2 bits each, k order from bit 0, at most 7) and its selectors.
__device__ __forceinline__ void n8_block_codes(uint32_t kept, uint32_t sel, uint32_t& lo_out, uint32_t& hi_out) {
  uint32_t lo = kept & 0xFFu, hi = (kept >> 8) & 0xFFu;
  lo = (lo | (lo << 12)) & 0x000F000Fu;  // codes 0, 1 | codes 2, 3 sixteen bits up
  lo = (lo | (lo << 6)) & 0x03030303u;   // one code per byte
  hi = (hi | (hi << 12)) & 0x000F000Fu;
  hi = ((hi | (hi << 6)) & 0x03030303u) | 0x01000000u;  // byte 7: code 1 (n <= 7, so no kept code there)
  lo_out = __byte_perm(lo, hi, sel & 0xFFFFu);
  hi_out = __byte_perm(lo, hi, sel >> 16);
}

template <int NK, int SUBS, bool SMEM>
__device__ __forceinline__ void n8_unpack_row(const uint8_t* vals, const uint8_t* masks, int r, const uint32_t* s_sel,
                                              uint32_t taddr, uint8_t* orow) {
  constexpr int VW = SUBS * NK;  // 32-bit words of kept codes in the row's stage
  if constexpr (VW % 4 != 0) {   // rows not 16-byte aligned: never launched (the host keeps odd n at 512 k)
    return;
  } else {
    uint32_t v[VW];
#pragma unroll
    for (int i = 0; i < VW / 4; ++i) {
      const uint4 t = reinterpret_cast<const uint4*>(vals + r * 4 * VW)[i];
      v[4 * i] = t.x; v[4 * i + 1] = t.y; v[4 * i + 2] = t.z; v[4 * i + 3] = t.w;
    }
    constexpr uint32_t fmask = (1u << (2 * NK)) - 1u;
#pragma unroll
    for (int sub = 0; sub < SUBS; ++sub) {
      const uint4 mq = reinterpret_cast<const uint4*>(masks + r * 16 * SUBS)[sub];
      const uint32_t mw[4] = {mq.x, mq.y, mq.z, mq.w};
      uint32_t outw[32];
#pragma unroll
      for (int jb = 0; jb < 16; ++jb) {
        constexpr int kBits = 2 * NK;
        const int bit = (sub * 16 + jb) * kBits;  // compile-time after unrolling
        const int wi = bit >> 5, sh = bit & 31;
        uint32_t kv = v[wi] >> sh;
        if (sh + kBits > 32) kv |= v[wi + 1] << (32 - sh);
        const uint32_t sel = s_sel[(mw[jb >> 2] >> (8 * (jb & 3))) & 0xFFu];
        n8_block_codes(kv & fmask, sel, outw[2 * jb], outw[2 * jb + 1]);
      }
      if constexpr (SMEM) {
#pragma unroll
        for (int g = 0; g < 8; ++g)
          *reinterpret_cast<uint4*>(orow + sub * (kTcRows * 128) + ((g ^ (r & 7)) << 4)) =
              make_uint4(outw[4 * g], outw[4 * g + 1], outw[4 * g + 2], outw[4 * g + 3]);
      } else {
        tc_st_32x32b_x32(taddr + sub * 32, outw);
      }
    }
  }
}

// Dense at BN = 128: 512-k stages, 4 copy stages of 48 KB, 2 operand slots of
// 128 TMEM columns beside two 128-column accumulators.  Dense, wider: 256-k
// stages, 4 copy stages, 2 slots of 32 KB expanded codes in shared memory.
// 2:4: 256-k stages, 4 to 6 copy stages (by BN) and 4 slots of 16 KB
// compressed operand (+ 8 metadata columns each).  n:8 (NM = 2): as dense,
// the stage holding the kept codes (2 n bits per 8 k) and the masks (one byte
// per 8 k) instead of the packed codes; wider tiles than 128 only for even n
// (a 256-k stage's 8 n bytes of kept codes must start 16-byte aligned).
// BN: tokens of a pair tile (the MMA's N, a multiple of 32), BN / 2 per CTA.
template <int NM, int BN>
struct T2 {
  static_assert(NM == 0 || NM == 2 || NM == 3, "pair GEMM: dense, n:8 expanded, or 2:4 on the sparse MMA");
  static_assert(BN % 32 == 0 && BN >= 64 && BN <= 224, "pair token tile");
  static constexpr bool SP = NM == 3;
  static constexpr bool N8 = NM == 2;
  static constexpr bool OPS = SP || BN > 128;  // A operand in shared memory
  static constexpr int KSUB = OPS ? 2 : 4;     // k-block: 512 k with A in TMEM (16 MMAs per hand-off), else 256 k
  static constexpr int HALF = BN / 2;
  static constexpr int B_SUB = HALF * 128;  // a whole number of 8-row swizzle atoms
  static constexpr int B_STAGE = B_SUB * KSUB;
  // TMA bytes of values and of metadata per stage (n:8: room for n = 7, 2 n bits and one mask bit per 8 k)
  static constexpr int A_VAL = N8 ? kTcRows * 28 * KSUB : kTcRows * (SP ? 16 : 32) * KSUB;
  static constexpr int A_META = SP || N8 ? kTcRows * 16 * KSUB : 0;
  static constexpr int STAGE = B_STAGE + A_VAL + A_META;             // one copy stage
  // operand slot in shared memory: 2:4 compressed (128 B a row), dense codes (256 B a row: two swizzle columns)
  static constexpr int OPA = SP ? kTcRows * 128 : OPS ? kTcRows * 256 : 0;
  static constexpr int SLOT = SP ? 8 : OPS ? 0 : 32 * KSUB;          // TMEM columns per operand slot
  static constexpr int DCOLS = BN > 128 ? 256 : BN;  // accumulator 1's first column (256 for wide tiles)
  static constexpr int R = SP ? 4 : OPS ? 2 : (512 - 2 * BN) / SLOT;  // operand slots (TMEM: as it holds)
  // no alignment slack: the dynamic shared memory is declared 1024-byte aligned (checked at run time)
  // scales, code sums, barriers (n:8: selectors; test builds: the phase stamps)
  static constexpr int FIXED = 2 * BN * 8 + 256 + (N8 ? 1024 : 0) + (kTimeline ? 64 : 0);
  static constexpr int S = tc_min3(kTcMaxStages, (kTcSmemMax - FIXED - R * OPA) / STAGE, 64) & ~1;  // even
  static constexpr int SMEM = FIXED + S * STAGE + R * OPA;
  static constexpr int A_COL0 = DCOLS + BN;         // operand slots after accumulator 1
  static_assert(A_COL0 + R * SLOT <= 512, "TMEM budget");
  static_assert(S >= R, "copy ring at least as deep as the operand ring");
  static constexpr uint32_t IDESC = SP ? idesc_i8_sp_s8s8(kT2Rows, BN) : idesc_i8_u8s8(kT2Rows, BN);
};

// Launched in clusters of two CTAs (an even grid); a.row_tiles counts 256-row
// pair tiles here; no K split (a.ksplit == 1).
template <int NM, int BN>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc2_gemm_kernel(const __grid_constant__ CUtensorMap mapB, const __grid_constant__ CUtensorMap mapA,
                    const __grid_constant__ CUtensorMap mapMeta, const TcArgs a) {
  using C = T2<NM, BN>;
  constexpr int S = C::S;
  constexpr bool SP = C::SP;
  constexpr int KSUB = C::KSUB;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint64_t t_entry = tl_now();
  // both CTAs see the same offset, so both leave here together (before any cluster barrier)
  if ((smem_u32(smem_raw) & 1023u) != 0u) {
    if (threadIdx.x == 0) *a.status = kDevBadSmemAlign;
    return;
  }
  uint8_t* base = smem_raw;
  constexpr int R = C::R;
  uint8_t* sStage = base;                        // [S][B half | packed values | metadata]
  uint8_t* sOp = base + S * C::STAGE;            // 2:4: [R][128 rows][128 B] compressed operand
  float* s_scale = reinterpret_cast<float*>(sOp + R * C::OPA);  // [2][BN]
  int32_t* s_rowsum = reinterpret_cast<int32_t*>(s_scale + 2 * BN);  // [2][BN]
  uint64_t* full = reinterpret_cast<uint64_t*>(s_rowsum + 2 * BN);
  uint64_t* empty = full + S;
  uint64_t* aready = empty + S;     // [R] rank 0's: both CTAs' unpack warps
  uint64_t* accfull = aready + R;   // [2]
  uint64_t* accempty = accfull + 2; // [2] rank 0's: both CTAs' epilogue warps
  uint64_t* drain = accempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  // n:8: byte-permute selectors of the 256 masks, after the 256 bytes of barriers
  uint32_t* s_sel = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(s_rowsum + 2 * BN) + 256);
  // test builds: phase stamps (0 entry, 1 set-up done, 2 producer past the dependency wait, 3 first stage
  // landed, 4 first tile's MMAs issued, 5 first accumulator ready, 6 last epilogue done, 7 end)
  uint64_t* s_tl = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(s_rowsum + 2 * BN) + 256 +
                                               (C::N8 ? 1024 : 0));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int KB = a.kbs;
  // dense codes into TMEM (A from TMEM): both unpack groups take every k-block, group g the half of its
  // 512 k in subs 2g, 2g + 1, so a slot is refilled in half the time after its release
  constexpr bool kSplit = !SP && !C::OPS && !C::N8;
  const int nunits = a.row_tiles * a.tok_tiles;
  const int my_tiles = pair < nunits ? (nunits - 1 - pair) / npairs + 1 : 0;
  const int total_kb = my_tiles * KB;
  const uint32_t tx_bytes =
      static_cast<uint32_t>(C::B_STAGE + (C::N8 ? kTcRows * (4 * KSUB * a.nm_n + 16 * KSUB) : C::A_VAL + C::A_META));
  auto unit_of = [&](int t, int& rt, int& tt) {  // token tile fastest: neighbouring pairs share weight rows
    const int g = pair + t * npairs;
    rt = g / a.tok_tiles;
    tt = g - rt * a.tok_tiles;
  };

  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int j = 0; j < R; ++j) mbar_init(&aready[j], kSplit ? 16 : 8);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], 8);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&mapB);
    tma_prefetch_desc(&mapA);
    if (SP) tma_prefetch_desc(&mapMeta);
  }
  if (warp == 2) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  if (C::N8)
    for (int m = threadIdx.x; m < 256; m += blockDim.x) s_sel[m] = n8_perm_selectors(static_cast<uint32_t>(m));
  if (kTimeline && threadIdx.x < 8) s_tl[threadIdx.x] = threadIdx.x == 0 ? t_entry : 0ull;
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers exist before any remote arrive or multicast commit
  tc_fence_after();
  if (kTimeline && threadIdx.x == 0) s_tl[1] = tl_now();
  const uint32_t tmem = *tmem_slot;
  const uint32_t aready0 = mapa_shared(smem_u32(aready), 0);
  const uint32_t accempty0 = mapa_shared(smem_u32(accempty), 0);

  if (warp == 0) {
    if (lane == 0 && total_kb > 0) {
      // ------------------------------------------------------------ producer (both CTAs)
      auto load_a = [&](int rt, int kb, int s) {
        uint8_t* dst = sStage + s * C::STAGE + C::B_STAGE;
        const int row0 = rt * kT2Rows + static_cast<int>(rank) * kTcRows;
        if (SP) {
          tma_load_2d(dst, &mapA, kb * 16 * KSUB, row0, &full[s]);
          tma_load_2d(dst + C::A_VAL, &mapMeta, kb * 16 * KSUB, row0, &full[s]);
        } else if (C::N8) {
          tma_load_2d(dst, &mapA, kb * 4 * KSUB * a.nm_n, row0, &full[s]);  // kept codes: 2 n bits per 8 k
          tma_load_2d(dst + C::A_VAL, &mapMeta, kb * 16 * KSUB, row0, &full[s]);  // masks: one byte per 8 k
        } else {
          tma_load_2d(dst, &mapA, kb * 32 * KSUB, row0, &full[s]);
        }
      };
      auto load_b = [&](int tt, int kb, int s) {
        const int tok0 = tt * BN + static_cast<int>(rank) * C::HALF;
        for (int sub = 0; sub < KSUB; ++sub)
          tma_load_2d(sStage + s * C::STAGE + sub * C::B_SUB, &mapB, (kb * KSUB + sub) * kTcSubK, tok0, &full[s]);
      };
      const int pre = total_kb < S ? total_kb : S;
      for (int i = 0; i < pre; ++i) {  // weights do not depend on the preceding kernel
        int rt, tt;
        unit_of(i / KB, rt, tt);
        mbar_arrive_expect_tx(&full[i], tx_bytes);
        load_a(rt, i % KB, i);
      }
      pdl_wait_primary();
      if (kTimeline) s_tl[2] = tl_now();
      for (int i = 0; i < pre; ++i) {
        int rt, tt;
        unit_of(i / KB, rt, tt);
        load_b(tt, i % KB, i);
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
        unit_of(i / KB, rt, tt);
        mbar_arrive_expect_tx(&full[s], tx_bytes);
        load_a(rt, i % KB, s);
        load_b(tt, i % KB, s);
      }
      if (!ok) {
        for (int j = (i - S > 0 ? i - S : 0); j < i; ++j)
          if (!mbar_wait(&full[j % S], (j / S) & 1)) *a.status = kDevTimeoutDrain;
      }
    }
  } else if (warp == 1) {
    if (rank == 0 && lane == 0 && total_kb > 0) {
      // ------------------------------------------------------------ MMA issuer (rank 0 only)
      bool issued = false, ok = true;
      for (int t = 0; t < my_tiles && ok; ++t) {
        const int buf = t & 1;
        if (t >= 2 && !mbar_wait_cluster(&accempty[buf], ((t >> 1) - 1) & 1)) {
          *a.status = kDevTimeoutMma;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dcol = tmem + buf * C::DCOLS;
        for (int kb = 0; kb < KB; ++kb) {
          const int i = t * KB + kb;
          const int s = i % S, j = i % R;
          // both CTAs' unpack warps arrived: both stages landed and both operands are written
          if (!mbar_wait_cluster(&aready[j], (i / R) & 1)) {
            *a.status = kDevTimeoutMma;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint8_t* sB = sStage + s * C::STAGE;
          if (SP) {
            const uint64_t adesc = smem_desc_sw128_kmajor(smem_u32(sOp + j * C::OPA));
#pragma unroll
            for (int kk = 0; kk < 2 * KSUB; ++kk) {
              const uint64_t bdesc = smem_desc_sw128_kmajor(smem_u32(sB + (kk >> 1) * C::B_SUB));
              tc_mma_sp_i8_ss_pair(dcol, adesc + static_cast<uint64_t>(kk * 2),
                                   bdesc + static_cast<uint64_t>((kk & 1) * 4), tmem + C::A_COL0 + j * C::SLOT + kk * 2,
                                   C::IDESC, (kb | kk) != 0 ? 1u : 0u);
            }
          } else if (C::OPS) {
#pragma unroll
            for (int kk = 0; kk < 4 * KSUB; ++kk) {  // A: 128-byte swizzle columns of 128 k, like B
              const uint64_t adesc = smem_desc_sw128_kmajor(smem_u32(sOp + j * C::OPA + (kk >> 2) * (kTcRows * 128)));
              const uint64_t bdesc = smem_desc_sw128_kmajor(smem_u32(sB + (kk >> 2) * C::B_SUB));
              tc_mma_i8_ss_pair(dcol, adesc + static_cast<uint64_t>((kk & 3) * 2),
                                bdesc + static_cast<uint64_t>((kk & 3) * 2), C::IDESC, (kb | kk) != 0 ? 1u : 0u);
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < 4 * KSUB; ++kk) {
              const uint64_t bdesc = smem_desc_sw128_kmajor(smem_u32(sB + (kk >> 2) * C::B_SUB));
              tc_mma_i8_ts_pair(dcol, tmem + C::A_COL0 + j * C::SLOT + kk * 8,
                                bdesc + static_cast<uint64_t>((kk & 3) * 2), C::IDESC, (kb | kk) != 0 ? 1u : 0u);
            }
          }
          tc_commit_pair_mc(&empty[s], 0x3);  // frees copy stage s, and operand slot j for k-block i + R
          issued = true;
        }
        if (ok) tc_commit_pair_mc(&accfull[buf], 0x3);
        if (kTimeline && t == 0) s_tl[4] = tl_now();
      }
      if (!ok && issued) {
        tc_commit_pair(drain);
        if (!mbar_wait(drain, 0)) *a.status = kDevTimeoutDrain;
      }
    }
  } else if (warp >= 4 && warp < kTcEpiWarp0) {
    // -------------------------------------------------------------- unpack (both CTAs)
    // Group g takes the k-blocks of parity g (with kSplit: every k-block, its
    // half of the k): with S and R even it sees every use of its copy stages
    // and operand slots, so no parity wait skips a phase.  The operand slot of
    // k-block i is free once the MMAs of k-block i - R have completed: the
    // commit that frees copy stage (i - R) % S says so.
    const int grp = (warp - 4) >> 2;
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    for (int i = kSplit ? 0 : grp; i < total_kb; i += kSplit ? 1 : 2) {
      const int s = i % S, j = i % R;
      if (!mbar_wait(&full[s], (i / S) & 1) || (i >= R && !mbar_wait(&empty[(i - R) % S], ((i - R) / S) & 1))) {
        *a.status = kDevTimeoutUnpack;
        break;
      }
      if (kTimeline && i == 0 && warp == 4 && lane == 0) s_tl[3] = tl_now();
      const uint8_t* st = sStage + s * C::STAGE + C::B_STAGE;
      if (SP) {
        const uint4* vp = reinterpret_cast<const uint4*>(st + r * 32);
        const uint4* mp = reinterpret_cast<const uint4*>(st + C::A_VAL + r * 32);
        const uint4 v0 = vp[0], v1 = vp[1], m0 = mp[0], m1 = mp[1];
        const uint32_t vw[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        const uint32_t mw[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
        uint8_t* arow_s = sOp + j * C::OPA + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t sj[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) sj[j] = (((vw[c] >> (2 * j)) & 0x03030303u) | 0x80808080u) - 0x01010101u;
          const uint32_t t0 = __byte_perm(sj[0], sj[1], 0x5140), t1 = __byte_perm(sj[0], sj[1], 0x7362);
          const uint32_t t2 = __byte_perm(sj[2], sj[3], 0x5140), t3 = __byte_perm(sj[2], sj[3], 0x7362);
          const uint4 o = make_uint4(__byte_perm(t0, t2, 0x5410) ^ 0x80808080u, __byte_perm(t0, t2, 0x7632) ^ 0x80808080u,
                                     __byte_perm(t1, t3, 0x5410) ^ 0x80808080u, __byte_perm(t1, t3, 0x7632) ^ 0x80808080u);
          *reinterpret_cast<uint4*>(arow_s + ((c ^ (r & 7)) << 4)) = o;
        }
        tc_st_32x32b_x8(tmem + lane_base + C::A_COL0 + j * C::SLOT, mw);
        fence_proxy_async_smem();
      } else if (C::OPS && !C::N8) {
        // the packed row (64 bytes) landed 64-byte-swizzled: its 16-byte chunk c sits at chunk c ^ ((r / 2) % 4),
        // so the 8 rows a quarter-warp reads at once fall in 8 different bank groups; the codes of 128 k
        // go to one 128-byte-swizzled row of the operand (chunk g at g ^ (r % 8))
        const uint8_t* arow = st + r * 64;
        uint8_t* orow = sOp + j * C::OPA + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
        for (int sub = 0; sub < KSUB; ++sub) {
          const uint4 lo = *reinterpret_cast<const uint4*>(arow + (((2 * sub) ^ ((r >> 1) & 3)) << 4));
          const uint4 hi = *reinterpret_cast<const uint4*>(arow + (((2 * sub + 1) ^ ((r >> 1) & 3)) << 4));
          const uint32_t dw[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
          for (int gi = 0; gi < 8; ++gi) {
            uint32_t o[4];
            codes_word_natural(dw[gi], o);
            *reinterpret_cast<uint4*>(orow + sub * (kTcRows * 128) + ((gi ^ (r & 7)) << 4)) =
                make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
        fence_proxy_async_smem();
      } else if (C::N8) {
        const uint32_t taddr = tmem + lane_base + C::A_COL0 + j * C::SLOT;
        uint8_t* orow = sOp + j * C::OPA + (r >> 3) * 1024 + (r & 7) * 128;
        switch (a.nm_n) {  // odd n never runs wide tiles (the host keeps them at 128 tokens)
          case 2: n8_unpack_row<2, KSUB, C::OPS>(st, st + C::A_VAL, r, s_sel, taddr, orow); break;
          case 4: n8_unpack_row<4, KSUB, C::OPS>(st, st + C::A_VAL, r, s_sel, taddr, orow); break;
          case 6: n8_unpack_row<6, KSUB, C::OPS>(st, st + C::A_VAL, r, s_sel, taddr, orow); break;
          case 1: n8_unpack_row<1, KSUB, C::OPS>(st, st + C::A_VAL, r, s_sel, taddr, orow); break;
          case 3: n8_unpack_row<3, KSUB, C::OPS>(st, st + C::A_VAL, r, s_sel, taddr, orow); break;
          case 5: n8_unpack_row<5, KSUB, C::OPS>(st, st + C::A_VAL, r, s_sel, taddr, orow); break;
          default: n8_unpack_row<7, KSUB, C::OPS>(st, st + C::A_VAL, r, s_sel, taddr, orow); break;
        }
        if (C::OPS) fence_proxy_async_smem();
      } else {
        // the packed row (128 bytes) landed 128-byte-swizzled: its 16-byte chunk c sits at chunk c ^ (r % 8),
        // so the 8 rows a quarter-warp reads at once fall in 8 different bank groups
        static_assert(SP || C::OPS || C::N8 || 32 * KSUB == 128, "one swizzle row of packed codes per weight row");
        const uint8_t* arow = st + r * 128;
#pragma unroll
        for (int hs = 0; hs < (kSplit ? KSUB / 2 : KSUB); ++hs) {
          const int sub = kSplit ? grp * (KSUB / 2) + hs : hs;
          const uint4 lo = *reinterpret_cast<const uint4*>(arow + (((2 * sub) ^ (r & 7)) << 4));
          const uint4 hi = *reinterpret_cast<const uint4*>(arow + (((2 * sub + 1) ^ (r & 7)) << 4));
          const uint32_t dw[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
          uint32_t outw[32];
#pragma unroll
          for (int gi = 0; gi < 8; ++gi) codes_word_natural(dw[gi], outw + 4 * gi);
          tc_st_32x32b_x32(tmem + lane_base + C::A_COL0 + j * C::SLOT + sub * 32, outw);
        }
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote_cta(aready0 + static_cast<uint32_t>(j * 8));
    }
  } else if (warp >= kTcEpiWarp0) {
    // -------------------------------------------------------------- epilogue (both CTAs, own rows)
    const int q = warp - kTcEpiWarp0;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const float alpha = *a.alpha;
    pdl_wait_primary();
    for (int t = 0; t < my_tiles; ++t) {
      const int buf = t & 1;
      int rt, tt;
      unit_of(t, rt, tt);
      const int row0 = rt * kT2Rows + static_cast<int>(rank) * kTcRows + q * 32;
      const int tok0 = tt * BN;
      float* scl = s_scale + buf * BN;
      int32_t* rsm = s_rowsum + buf * BN;
      for (int j = threadIdx.x - kTcEpiWarp0 * 32; j < BN; j += 128) {
        const int tok = tok0 + j;
        scl[j] = tok < a.M ? __fdiv_rn(__fmul_rn(alpha, a.gamma[tok]), a.qb) : 0.0f;  // RN(RN(alpha gamma) / Q_b)
        rsm[j] = (tok < a.M && a.rowsum) ? a.rowsum[tok] : 0;
      }
      bar_sync_n(1, 128);
      if (!mbar_wait(&accfull[buf], (t >> 1) & 1)) {
        *a.status = kDevTimeoutEpilogue;
        break;
      }
      if (kTimeline && t == 0 && q == 0 && lane == 0) s_tl[5] = tl_now();
      tc_fence_after();
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t v[32];
        tc_ld_32x32b_x32(tmem + lane_base + buf * C::DCOLS + c0, v);
        tc_wait_ld();
        tc_store_token_rows(v, scl + c0, rsm + c0, row0 + lane, tok0 + c0, 32, a);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote_cta(accempty0 + static_cast<uint32_t>(buf * 8));
      if (kTimeline && q == 0 && lane == 0) s_tl[6] = tl_now();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (kTimeline && threadIdx.x == 0) {
    uint64_t t8[8];
    for (int i = 0; i < 7; ++i) t8[i] = s_tl[i];
    t8[7] = tl_now();
    tl_commit(2, (static_cast<uint64_t>(a.M) << 32) | (static_cast<uint64_t>(blockIdx.x) << 16) | gridDim.x, t8);
  }
  cluster_sync_all();  // no remote arrive or multicast commit is left in flight towards either CTA
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace bl
