// gemm_skinny.cuh -- BitLinear for a few tokens (M <= 64) on the tensor cores
// in one launch: activation quantisation, contraction and rescale fused, K
// split across the CTAs of a thread-block cluster and reduced through
// distributed shared memory.
//
// With few tokens the call is bound by the weight bytes and by latency, not by
// the tensor cores.  So every CTA of a cluster owns one 128-row weight tile
// and one slice of K, and
//   1. hands all of its packed weight chunks (128 rows x 128 k, 4 KB each) to
//      the tensor-copy engine at once, before waiting on the preceding kernel;
//   2. quantises its K slice of every token: the slice's per-token maximum is
//      stored into every CTA of the cluster (st.shared::cluster), then, after
//      one cluster-scope fence, a remote mbarrier arrive; each CTA waits on its own
//      barrier, takes gamma = the maximum over the cluster and writes the codes
//      straight into the 128-byte-swizzled K-major B operand in shared memory
//      (contraction order inside each 16-group, as the A unpack produces);
//   3. expands each weight chunk to u8 codes in tensor memory (three groups of
//      four unpack warps, one chunk each in turn; a ring of A slots) and issues
//      the chunk's four tcgen05.mma kind::i8 (M = 128 weight rows, N = BN
//      tokens, K = 32) into one int32 accumulator;
//   4. reads its accumulator (tcgen05.ld), subtracts its slice's code sums and
//      stores each row into the CTA that owns the row's band (rows are split
//      in bands, one per CTA), then arrives remotely on that CTA's barrier;
//      each CTA waits for its band from every CTA of the cluster, sums the
//      slices in its own shared memory, rescales by RN(RN(alpha gamma) / 127)
//      and stores bf16 (and int32 on request).
// Only point-to-point signals cross CTAs (no cluster-wide barrier after the
// start), every wait is a bounded mbarrier wait, and no CTA reads another's
// shared memory, so a CTA may leave once its own band is done.  A CTA whose
// role gave up on a wait sends a flag with its rows; a band that received one
// is not stored.  The result equals the persistent GEMM's bit for bit: the
// same codes, an exact integer contraction, the same rescale.
#pragma once
#include "gemm_tc.cuh"

namespace bl {

constexpr int kSkThreads = 512;
constexpr int kSkChunkBytes = kTcRows * 32;  // packed weights of one 128-k chunk of a 128-row tile
constexpr int kSkMaxChunks = 24;             // weight chunks per CTA, all resident in shared memory
constexpr int kSkMaxCluster = 8;             // portable cluster size
constexpr int kSkGroups = 3;                 // unpack groups of four warps (warps 4 .. 15)
constexpr int kSkTmemCols = 256;
// Dynamic shared memory of at least this many bytes keeps one CTA per SM, so
// the 256 TMEM columns a CTA allocates are always available to it.
constexpr size_t kSkMinSmem = 116 * 1024;

__host__ __device__ constexpr int sk_dcols(int BN) { return BN <= 32 ? 32 : 64; }  // accumulator columns
__host__ __device__ constexpr int sk_aslots(int BN) { return (kSkTmemCols - sk_dcols(BN)) / 32; }
// Rows of the tile each CTA of a cluster of cs reduces and stores (a multiple of 4).
__host__ __device__ constexpr int sk_band(int cs) { return ((kTcRows + cs - 1) / cs + 3) & ~3; }
__host__ __device__ constexpr int sk_band_rows(int cs, int rank) {
  return rank * sk_band(cs) >= kTcRows ? 0
         : (kTcRows - rank * sk_band(cs) < sk_band(cs) ? kTcRows - rank * sk_band(cs) : sk_band(cs));
}

__host__ __device__ constexpr size_t sk_fixed_bytes(int BN) {
  return 1024 /* alignment */ + static_cast<size_t>(160) * BN * 4 /* band staging: cs * band <= 160 rows */ +
         kSkMaxCluster * BN * 4 /* partial maxima */ + BN * 8 /* code sums, scales */ + 768 /* flags, barriers */;
}
__host__ __device__ constexpr size_t sk_chunk_bytes(int BN) { return kSkChunkBytes + static_cast<size_t>(BN) * 128; }
__host__ __device__ constexpr size_t sk_smem_bytes(int BN, int per) {
  return sk_fixed_bytes(BN) + static_cast<size_t>(per) * sk_chunk_bytes(BN);
}

struct SkArgs {
  const uint16_t* x;  // [M, K] bf16 bits
  int M, N, K;
  int kchunks;        // ceil(K / 128)
  int per;            // chunks per K slice: cluster rank r owns [r * per, min((r + 1) * per, kchunks))
  int cs;             // CTAs per cluster (K slices)
  const float* alpha;
  uint16_t* y;        // [M, N]
  int32_t* acc;       // [M, N] or null
  int32_t* status;
};

template <int BN>
__global__ void __launch_bounds__(kSkThreads, 1) skinny_kernel(const __grid_constant__ CUtensorMap mapW,
                                                              const SkArgs a) {
  constexpr int DC = sk_dcols(BN);
  constexpr int SA = sk_aslots(BN);
  constexpr uint32_t IDESC = idesc_i8_u8s8(kTcRows, BN);
  constexpr int TPT = kSkThreads / BN;  // threads per token in the quantisation (32, 16 or 8 lanes)
  constexpr int B_CHUNK = BN * 128;     // one chunk of the B operand (BN rows x 128 bytes)
  static_assert(DC + SA * 32 <= kSkTmemCols, "TMEM budget");
  static_assert(B_CHUNK % 1024 == 0, "B chunks keep the 1024-byte swizzle alignment");

  extern __shared__ uint8_t smem_raw[];
  // offset arithmetic on the shared array keeps every derived pointer in the shared window
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int per = a.per;
  const int cs = a.cs;
  const int band = sk_band(cs);
  uint8_t* sB = base;                                                     // [per][B_CHUNK]
  uint8_t* sW = sB + static_cast<size_t>(per) * B_CHUNK;                  // [per][128 rows x 32 B]
  int32_t* sStage = reinterpret_cast<int32_t*>(sW + static_cast<size_t>(per) * kSkChunkBytes);  // [cs][band][BN]
  uint32_t* sPmax = reinterpret_cast<uint32_t*>(sStage + 160 * BN);     // [kSkMaxCluster][BN]
  int32_t* sQsum = reinterpret_cast<int32_t*>(sPmax + kSkMaxCluster * BN);  // [BN]
  float* sScale = reinterpret_cast<float*>(sQsum + BN);                   // [BN]
  uint32_t* sFailIn = reinterpret_cast<uint32_t*>(sScale + BN);           // [kSkMaxCluster]
  uint64_t* full = reinterpret_cast<uint64_t*>(sFailIn + kSkMaxCluster);  // [kSkMaxChunks]
  uint64_t* aready = full + kSkMaxChunks;                                 // [SA]
  uint64_t* afree = aready + SA;                                          // [SA]
  uint64_t* accfull = afree + SA;
  uint64_t* maxbar = accfull + 1;  // every CTA's per-token maxima have arrived
  uint64_t* redbar = maxbar + 1;   // every CTA's rows of this CTA's band have arrived
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(redbar + 1);
  uint32_t* s_fail = tmem_slot + 1;  // nonzero: a wait of this CTA gave up

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int row0 = static_cast<int>(blockIdx.x / cs) * kTcRows;
  const int c0 = static_cast<int>(rank) * per;
  const int nch = max(0, min(per, a.kchunks - c0));
  const int my_rows = sk_band_rows(cs, static_cast<int>(rank));

  if (threadIdx.x == 0) {
    for (int c = 0; c < nch; ++c) mbar_init(&full[c], 1);
    for (int i = 0; i < SA; ++i) {
      mbar_init(&aready[i], 4);
      mbar_init(&afree[i], 1);
    }
    mbar_init(accfull, 1);
    mbar_init(maxbar, static_cast<uint32_t>(cs * BN));
    mbar_init(redbar, static_cast<uint32_t>(cs * (my_rows > 0 ? my_rows : 1)));
    *s_fail = 0u;
    fence_mbar_init();
    tma_prefetch_desc(&mapW);
    // the weights do not depend on the preceding kernel: every chunk of the slice now
    const uint64_t pol = l2_policy_evict_first();
    for (int c = 0; c < nch; ++c) {
      mbar_arrive_expect_tx(&full[c], static_cast<uint32_t>(kSkChunkBytes) + test_extra_tx());
      tma_load_2d_hint(sW + c * kSkChunkBytes, &mapW, (c0 + c) * 32, row0, &full[c], pol);
    }
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, kSkTmemCols);
    tmem_relinquish();
  }
  const float alpha = *a.alpha;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The first access to another CTA's shared memory must follow a cluster
  // barrier (every CTA of the cluster running, its barriers initialised); its
  // wait comes just before that access.
  cluster_arrive_relaxed();

  // ------------------------------------------------ quantisation of this CTA's K slice
  pdl_wait_primary();  // x may come from the preceding kernel
  const int t = threadIdx.x / TPT, sub = threadIdx.x % TPT;
  const bool active = t < a.M;
  const uint16_t* xr = a.x + static_cast<size_t>(active ? t : 0) * a.K;
  const bool vec_ok = (a.K % 8) == 0;
  const int gbeg = c0 * 8;                                    // first 16-group of the slice
  const int gend = min((a.K + 15) / 16, (c0 + nch) * 8);      // groups holding some k < K
  float mx = 0.0f;
  if (active)
    for (int g = gbeg + sub; g < gend; g += TPT) {
      uint32_t r0[4], r1[4];
      load8_raw(xr, 16 * g, a.K, vec_ok, r0);
      load8_raw(xr, 16 * g + 8, a.K, vec_ok, r1);
      mx = absmax8(r1, absmax8(r0, mx));
    }
  uint32_t mb = __float_as_uint(mx);  // |x| >= 0: bit patterns order like the values
#pragma unroll
  for (int o = TPT / 2; o > 0; o >>= 1) mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, o));
  cluster_wait();
  if (sub == 0) {
    // all stores, one cluster-scope fence, then the arrives (each arrive with its
    // own release would wait for the stores once per destination)
    const uint32_t lmax = smem_u32(&sPmax[rank * BN + t]), lbar = smem_u32(maxbar);
    for (int p = 0; p < cs; ++p) st_cluster_u32(mapa_shared(lmax, static_cast<uint32_t>(p)), mb);
    fence_cluster();
    for (int p = 0; p < cs; ++p) mbar_arrive_remote_relaxed(mapa_shared(lbar, static_cast<uint32_t>(p)));
  }
  if (!mbar_wait_cluster(maxbar, 0)) *s_fail = 1u;
  uint32_t gb = 0u;
  for (int p = 0; p < cs; ++p) gb = max(gb, sPmax[p * BN + t]);
  const float gamma = __uint_as_float(gb);
  const float d = __fadd_rn(gamma, kEps);
  const float cq = __fmul_rn(kQb, __frcp_rn(d));
  int32_t qs = 0;
  for (int g = gbeg + sub; g < gbeg + nch * 8; g += TPT) {
    uint4 w = make_uint4(0u, 0u, 0u, 0u);  // past K and for absent tokens: code 0
    if (active && g < gend) {
      uint32_t r0[4], r1[4];
      load8_raw(xr, 16 * g, a.K, vec_ok, r0);
      load8_raw(xr, 16 * g + 8, a.K, vec_ok, r1);
      w = group_codes<true>(r0, r1, cq, d, qs);
    }
    const int gl = g - gbeg;
    const int ch = gl >> 3, j16 = gl & 7;  // chunk, 16-byte column of the token's 128-byte row
    *reinterpret_cast<uint4*>(sB + ch * B_CHUNK + (t >> 3) * 1024 + (t & 7) * 128 + ((j16 ^ (t & 7)) << 4)) = w;
  }
#pragma unroll
  for (int o = TPT / 2; o > 0; o >>= 1) qs += __shfl_xor_sync(0xffffffffu, qs, o);
  if (sub == 0) {
    sQsum[t] = qs;  // this slice's share of the token's code sum
    sScale[t] = active ? __fdiv_rn(__fmul_rn(alpha, gamma), kQb) : 0.0f;  // RN(RN(alpha gamma) / 127)
  }
  fence_proxy_async_smem();  // the B tile is read by the tensor cores
  __syncthreads();
  pdl_launch_dependents();

  // ------------------------------------------------ roles
  if (warp == 1) {
    if (lane == 0) {
      // MMA issuer
      for (int c = 0; c < nch; ++c) {
        const int sl = c % SA;
        if (!mbar_wait(&aready[sl], (c / SA) & 1)) {
          *a.status = kDevTimeoutMma;
          *s_fail = 1u;
          break;
        }
        tc_fence_after();
        const uint64_t bdesc = smem_desc_sw128_kmajor(smem_u32(sB + c * B_CHUNK));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma_i8_ts(tmem, tmem + DC + sl * 32 + kk * 8, bdesc + static_cast<uint64_t>(kk * 2), IDESC,
                       (c | kk) != 0 ? 1u : 0u);
        tc_commit(&afree[sl]);
      }
      tc_commit(accfull);  // completes once every MMA issued above has (also after a give-up)
    }
  } else if (warp >= 4) {
    // unpack: group grp expands chunks grp, grp + 3, ... for the 32 rows of its lane quarter
    const int grp = (warp - 4) >> 2;
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    for (int c = grp; c < nch; c += kSkGroups) {
      const int sl = c % SA;
      if ((c >= SA && !mbar_wait(&afree[sl], ((c / SA) - 1) & 1)) || !mbar_wait(&full[c], 0)) {
        *a.status = kDevTimeoutUnpack;
        *s_fail = 1u;
        break;
      }
      const uint4 lo = *reinterpret_cast<const uint4*>(sW + c * kSkChunkBytes + r * 32);
      const uint4 hi = *reinterpret_cast<const uint4*>(sW + c * kSkChunkBytes + r * 32 + 16);
      const uint32_t dw[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
      uint32_t outw[32];
#pragma unroll
      for (int gi = 0; gi < 8; ++gi)
#pragma unroll
        for (int j = 0; j < 4; ++j) outw[4 * gi + j] = (dw[gi] >> (2 * j)) & 0x03030303u;
      tc_st_32x32b_x32(tmem + lane_base + DC + sl * 32, outw);
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&aready[sl]);
    }
    if (warp < 8) {
      // epilogue part 1: row r of this CTA's partial tile, minus the slice's code
      // sums, goes to the CTA whose band holds the row
      if (!mbar_wait(accfull, 0)) {
        *a.status = kDevTimeoutEpilogue;
        *s_fail = 1u;
      }
      tc_fence_after();
      const int p = r / band;
      const uint32_t dst = mapa_shared(smem_u32(sStage + (static_cast<int>(rank) * band + (r - p * band)) * BN),
                                       static_cast<uint32_t>(p));
#pragma unroll
      for (int cb = 0; cb < (BN + 31) / 32; ++cb) {
        uint32_t v[32];
        tc_ld_32x32b_x32(tmem + lane_base + cb * 32, v);
        tc_wait_ld();
#pragma unroll
        for (int j = 0; j < 32 && cb * 32 + j < BN; j += 4)
          st_cluster_v4(dst + (cb * 32 + j) * 4, v[j] - sQsum[cb * 32 + j], v[j + 1] - sQsum[cb * 32 + j + 1],
                        v[j + 2] - sQsum[cb * 32 + j + 2], v[j + 3] - sQsum[cb * 32 + j + 3]);
      }
      st_cluster_u32(mapa_shared(smem_u32(&sFailIn[rank]), static_cast<uint32_t>(p)), *s_fail);
      mbar_arrive_remote(mapa_shared(smem_u32(redbar), static_cast<uint32_t>(p)));
    }
  }

  // ------------------------------------------------ this CTA's band: sum the slices, rescale, store
  bool ok = my_rows > 0 && mbar_wait_cluster(redbar, 0);
  if (!ok && my_rows > 0) *a.status = kDevTimeoutEpilogue;
  for (int p = 0; p < cs && ok; ++p) ok = sFailIn[p] == 0u;
  if (ok) {
    const int rb = static_cast<int>(rank) * band;
    for (int it = threadIdx.x; it < my_rows * a.M; it += kSkThreads) {
      const int lr = it / a.M, tok = it - lr * a.M;
      int32_t acc = 0;
      for (int p = 0; p < cs; ++p) acc += sStage[(p * band + lr) * BN + tok];
      const int n = row0 + rb + lr;
      if (n >= a.N) continue;
      const size_t o = static_cast<size_t>(tok) * a.N + n;
      if (a.acc) a.acc[o] = acc;
      const __nv_bfloat16 h = __float2bfloat16_rn(__fmul_rn(static_cast<float>(acc), sScale[tok]));
      a.y[o] = *reinterpret_cast<const uint16_t*>(&h);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, kSkTmemCols);
  }
}

}  // namespace bl
