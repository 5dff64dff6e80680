/*
 * bitlinear.h -- C ABI of the B200 (sm_100a) BitLinear forward library.
 *
 * The operation (BitNet b1.58 / Sparse-BitNet BitLinear, forward only):
 *
 *   alpha   = mean |W|                       over the whole latent matrix W [N, K]
 *   W_t     = clamp(round(W / (alpha + 1e-5)), -1, 1)
 *   gamma_m = max_k |x_mk|                    per token (row of x [M, K])
 *   q       = clamp(round(127 x / (gamma + 1e-5)), -128, 127)   (int8)
 *   acc     = q W_t^T                         int32 [M, N]
 *   y       = acc * alpha * gamma_m / 127     bf16  [M, N]
 *
 * Sources, cited by page title and section:
 *  - "BitNet 1-Bit LLM" blog (youngju.dev), section "BitNet b1.58 / Absmean
 *    quantization function": weight_quant_ternary, activation_quant and the
 *    BitLinear_b158 forward (integer matmul, then rescale).
 *  - "BitNet b1.58 2B4T Technical Report" summary, section 2 Architecture
 *    (absmean ternary weights, per-token absmax 8-bit activations) and
 *    section 5.1 GPU Inference (four ternary weights packed per int8, moved
 *    from HBM to on-chip memory, unpacked, combined with 8-bit activations).
 *  - "BitNet 1-Bit LLM" blog, section "bitnet.cpp / Architecture overview":
 *    the I2_S code map -1 -> 00, 0 -> 01, +1 -> 10.
 *  - "Sparse-BitNet" review, section 3.2 (N:M mask from the latent
 *    magnitudes, applied after ternarisation) and section 4 (6:8 and 2:4).
 *
 * Readings where the pages are silent or disagree: Q_b = 127 in both the
 * quantisation and the rescale (the blog prints 2**(bits-1) = 128; this
 * library uses 127 throughout); round-half-to-even everywhere; scale divisions in
 * IEEE fp32 (RN(x * 127) / RN(gamma + 1e-5)); alpha summed in fp64 and
 * rounded once to fp32; the rescale as RN(RN(alpha * gamma) / 127) applied
 * with one fp32 multiply before the bf16 rounding; N:M blocks run along K
 * inside one output row, ties in |W| go to the lower position.
 *
 * Packed layouts (all device memory, caller-owned):
 *  dense  codes: row n is ld = 16 * ceil(K / 64) bytes; weight k sits in
 *         byte k / 4, bits 2*(k % 4) .. +1, code = W_t + 1 (00 = -1,
 *         01 = 0, 10 = +1, 11 unused); tail positions hold code 01.
 *  N:M    values: per row the n kept codes of every block in increasing k,
 *         same 2-bit packing, row stride 16 * ceil(K * n / m / 64) bytes.
 *         meta (2:4): per block a nibble i0 | i1 << 2 (kept positions,
 *         i0 < i1), block b in byte b / 2, low nibble first.
 *         meta (n:8): per block one byte, bit j = position j kept.
 *         meta row stride 16 * ceil(K / 128) bytes.
 *
 * Conventions for every call:
 *  - Pointers marked "device" are CUDA device pointers owned by the caller;
 *    "host" pointers are ordinary host memory.  The library allocates no
 *    memory in any call.
 *  - stream is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Work is enqueued asynchronously; argument errors are returned before
 *    anything is enqueued.  A kernel that gives up on an internal wait
 *    (about one second) writes a code to the device status word instead of
 *    trapping; read it with bitlinear_device_status().
 *  - No CPU fallback exists.  Unsupported shapes return BITLINEAR_ERR_SHAPE.
 *  - bf16 values are passed as their 16-bit patterns (uint16_t).
 */
#ifndef BITLINEAR_H_
#define BITLINEAR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum bitlinear_status {
  BITLINEAR_OK = 0,
  BITLINEAR_ERR_NULL = 1,           /* a required pointer is NULL */
  BITLINEAR_ERR_SHAPE = 2,          /* M, N or K out of the supported range */
  BITLINEAR_ERR_ALIGN = 3,          /* a pointer misses its 16-byte alignment */
  BITLINEAR_ERR_PATTERN = 4,        /* N:M pattern other than dense, 2:4 or n:8 (1 <= n <= 7) */
  BITLINEAR_ERR_WORKSPACE = 5,      /* workspace NULL or smaller than required */
  BITLINEAR_ERR_CUDA = 6,           /* a CUDA runtime/driver call failed */
  BITLINEAR_ERR_DEVICE = 7,         /* current device is not sm_100 */
  BITLINEAR_ERR_FLAGS = 8           /* unknown flag, or a path flag the shape cannot take */
} bitlinear_status;

/* Limits checked by every call. */
#define BITLINEAR_LAYOUT_VERSION 1
#define BITLINEAR_MAX_K 65536       /* keeps every int32 partial sum exact */
#define BITLINEAR_MAX_N (1 << 24)
#define BITLINEAR_MAX_M (1 << 24)
#define BITLINEAR_MAX_GROUP 4       /* matrices per bitlinear_forward_group call */

/* Flags of bitlinear_forward / bitlinear_forward_nm. */
#define BITLINEAR_FLAG_PDL 0x1u       /* launch as a programmatic dependent: the
                                         kernel may start reading w->codes,
                                         w->meta and *w->alpha before the
                                         preceding kernel on the stream finishes.
                                         The caller asserts that this preceding
                                         kernel does not write those buffers.
                                         x, y and acc are touched only after it
                                         ends. */
#define BITLINEAR_FLAG_PATH_GEMV 0x2u /* force the M = 1 streaming GEMV (needs M == 1) */
#define BITLINEAR_FLAG_PATH_TC 0x4u   /* force the tensor-core path at any M */
#define BITLINEAR_FLAG_PATH_PERSISTENT 0x10u /* tensor-core path: take the persistent GEMM (separate
                                        * quantisation launch, K split through a workspace) even
                                        * where the fused few-token kernel applies; same results */
#define BITLINEAR_FLAG_NM24_EXPAND 0x20u /* tensor-core path, 2:4 weights: expand the kept values
                                        * to dense codes and run the dense MMA instead of the
                                        * structured-sparse tcgen05.mma.sp (the Sparse-BitNet
                                        * review, section 4: 2:4 on sparse tensor cores); same
                                        * results.  A comparison path, not the default. */
#define BITLINEAR_FLAG_DECODE_LUT 0x8u /* M = 1, dense weights: run the decode GEMV with
                                        * per-pair lookup tables (the TL2 idea of the
                                        * "BitNet 1-Bit LLM" blog, section "I2_S kernel
                                        * internals") instead of dp4a; same results.  A
                                        * comparison path, not the default. */

/* Packed weights.  All pointers device, caller-owned. */
typedef struct bitlinear_weights {
  int32_t N;              /* output features (rows of W) */
  int32_t K;              /* input features */
  int32_t nm_n;           /* kept per block: 0 for dense */
  int32_t nm_m;           /* block length: 0 for dense, 4 (with n = 2) or 8 */
  const uint8_t* codes;   /* dense codes, or the N:M kept values (16-byte aligned) */
  const uint8_t* meta;    /* N:M metadata (16-byte aligned); NULL for dense */
  const float* alpha;     /* one fp32: the absmean scale of the dense latent W */
} bitlinear_weights;

/* Byte sizes of the packed buffers.  ld_codes / ld_meta are row strides in
 * bytes; meta outputs are 0 for dense.  Any output pointer may be NULL.
 * Pure host computation.  Errors: SHAPE (N, K out of range or K % m != 0),
 * PATTERN. */
bitlinear_status bitlinear_packed_layout(int32_t N, int32_t K, int32_t nm_n, int32_t nm_m,
                                         int64_t* ld_codes, int64_t* ld_meta,
                                         size_t* codes_bytes, size_t* meta_bytes);

/* Workspace bytes needed by bitlinear_pack_weights for an N x K matrix. */
size_t bitlinear_pack_workspace_bytes(int32_t N, int32_t K);

/* Quantises and packs a latent fp32 matrix.
 * W        device, fp32 [N, K] row-major (read only).
 * nm_n/m   0,0 dense; 2,4; or n,8 with 1 <= n <= 7 (mask of |W| per block
 *          of m consecutive k, applied after ternarisation; alpha still comes
 *          from the dense W).
 * codes    device, out: codes_bytes (dense) or the kept values (N:M).
 * meta     device, out: meta_bytes (N:M only; ignored for dense).
 * alpha    device, out: one fp32.
 * workspace, workspace_bytes: device scratch of bitlinear_pack_workspace_bytes().
 * Errors: NULL, SHAPE, PATTERN, ALIGN (codes/meta not 16-byte aligned),
 *         WORKSPACE, CUDA. */
bitlinear_status bitlinear_pack_weights(const float* W, int32_t N, int32_t K, int32_t nm_n, int32_t nm_m,
                                        uint8_t* codes, uint8_t* meta, float* alpha,
                                        void* workspace, size_t workspace_bytes, void* stream);

/* Packs an already-ternary matrix (values in {-1, 0, 1}) with a given scale,
 * for weights drawn directly in ternary form.  Dense layout only.
 * Wt       device, int8 [N, K] row-major; values outside {-1,0,1} are clamped.
 * alpha    host value, written to alpha_out (device, one fp32).
 * Errors: NULL, SHAPE, ALIGN, CUDA. */
bitlinear_status bitlinear_pack_ternary(const int8_t* Wt, int32_t N, int32_t K, float alpha,
                                        uint8_t* codes, float* alpha_out, void* stream);

/* Per-token absmax int8 quantisation.
 * x        device, bf16 bits [M, K] row-major (16-byte aligned).
 * q        device, out: int8 [M, K] row-major codes in natural k order.
 * gamma    device, out: fp32 [M] = max_k |x_mk|.
 * rowsum   device, out (may be NULL): int32 [M] = sum_k q_mk.
 * Errors: NULL, SHAPE, ALIGN, CUDA. */
bitlinear_status bitlinear_quant_act(const uint16_t* x, int32_t M, int32_t K, int8_t* q, float* gamma,
                                     int32_t* rowsum, void* stream);

/* RMSNorm followed by the per-token absmax int8 quantisation, in one kernel.
 * The page's BitLinear normalises its input with an RMSNorm (per-feature
 * weight g) before the activation quantisation ("BitNet 1-Bit LLM" blog,
 * section "BitNet b1.58: Absmean quantization function", BitLinear_b158.forward).
 * Per row: ms = RN32(sum_k x_k^2 / K) and r = RN32(1 / sqrt(ms + eps)), the sum,
 * root and quotient in fp64; xn_k = RN32(RN32(x_k * r) * g_k) (not rounded to
 * bf16); then gamma = max |xn| and q = clamp(rne(RN32(xn * 127) / RN32(gamma +
 * 1e-5)), -128, 127) as in bitlinear_quant_act.
 * x        device, bf16 bits [M, K] (16-byte aligned).
 * g        device, fp32 [K] (4-byte aligned).
 * eps      0 <= eps <= 1 (with eps = 0 an all-zero row is undefined).
 * q, gamma, rowsum: as bitlinear_quant_act (natural k order; rowsum may be NULL).
 * Errors: NULL, SHAPE (also eps out of range), ALIGN, DEVICE, CUDA. */
bitlinear_status bitlinear_rmsnorm_quant_act(const uint16_t* x, int32_t M, int32_t K, const float* g, float eps,
                                             int8_t* q, float* gamma, int32_t* rowsum, void* stream);

/* y = BitLinear(RMSNorm(x)) as the page's BitLinear_b158.forward computes it
 * (see bitlinear_rmsnorm_quant_act for the normalisation).  For M == 1 and
 * dense weights every CTA of the decode GEMV normalises and quantises the
 * token itself (no workspace is used); otherwise the normalisation is fused
 * into the activation quantisation kernel, which writes the codes into the
 * workspace, and the tensor-core GEMM follows.
 * w        dense or N:M weights.
 * g, eps   as bitlinear_rmsnorm_quant_act.
 * workspace, workspace_bytes: bitlinear_forward_workspace_bytes(M, N, K,
 *          BITLINEAR_FLAG_PATH_TC).
 * flags    BITLINEAR_FLAG_PDL; BITLINEAR_FLAG_PATH_TC forces the tensor-core
 *          GEMM at M == 1 (BITLINEAR_FLAG_PATH_GEMV is not accepted).
 * Errors: as bitlinear_forward; SHAPE also for eps out of range. */
bitlinear_status bitlinear_forward_norm(const bitlinear_weights* w, const uint16_t* x, int32_t M, const float* g,
                                        float eps, uint16_t* y, int32_t* acc, void* workspace, size_t workspace_bytes,
                                        uint32_t flags, void* stream);

/* H-BitLinear ("BitNet v2" page, brain.hanbit.co.kr: the paragraphs on the
 * H-BitLinear module and on native 4-bit activations): an online Hadamard
 * transform of the activations, then 4-bit quantisation, then the ternary
 * linear map.  The page fixes neither the transform's size, normalisation and
 * evaluation order nor the 4-bit quantiser; this library takes, per token row:
 *   B  = the largest power of two dividing K (2560 -> 512, 6912 -> 256,
 *        odd K -> 1, no transform);
 *   xh = each B-block times the Sylvester-order Walsh-Hadamard matrix, by the
 *        fast butterflies in fp32 (stage h = 1, 2, ..., B/2: every pair
 *        (j, j + h) with bit h of j clear becomes (a + b, a - b), one rounding
 *        each), then one fp32 multiply by RN32(1 / sqrt(B));
 *   gamma = max_k |xh_k|, q = clamp(rne(RN32(xh * 7) / RN32(gamma + 1e-5)),
 *        -8, 7) (held in int8), and y = acc * alpha * gamma / 7 with the
 *        rescale s = RN(RN(alpha * gamma) / 7).
 * The weights are the ternary matrix as given (no transform at run time). */
#define BITLINEAR_HBIT_MAX_K 16384  /* the row is transformed in shared memory */

/* Hadamard transform and 4-bit codes of each token row (natural k order).
 * x device, bf16 bits [M, K] (2-byte aligned); q device out int8 [M, K] in
 * [-8, 7]; gamma device out fp32 [M] = max |xh|; rowsum device out (may be
 * NULL) int32 [M] = sum of the row's codes.  Errors: NULL, SHAPE (K above
 * BITLINEAR_HBIT_MAX_K), ALIGN, DEVICE, CUDA. */
bitlinear_status bitlinear_hadamard_quant_act4(const uint16_t* x, int32_t M, int32_t K, int8_t* q, float* gamma,
                                               int32_t* rowsum, void* stream);

/* y = H-BitLinear(x): the transform and 4-bit codes above, then the
 * tensor-core GEMM with dense or N:M weights (every M, M = 1 included).
 * Arguments as bitlinear_forward; workspace_bytes at least
 * bitlinear_forward_workspace_bytes(M, N, K, BITLINEAR_FLAG_PATH_TC).
 * flags: BITLINEAR_FLAG_PDL (BITLINEAR_FLAG_PATH_TC is accepted, and implied).
 * Errors: as bitlinear_forward; SHAPE also for K above BITLINEAR_HBIT_MAX_K. */
bitlinear_status bitlinear_forward_hbit(const bitlinear_weights* w, const uint16_t* x, int32_t M, uint16_t* y,
                                        int32_t* acc, void* workspace, size_t workspace_bytes, uint32_t flags,
                                        void* stream);

/* y = BitLinear for activations already quantised: the int8 codes, gamma and
 * code sums of x as bitlinear_quant_act writes them ("BitNet b1.58 2B4T
 * Technical Report", section 2 Architecture, BitLinear: activation_quant then
 * the ternary contraction and the rescale by alpha * gamma / Q_b), so that a
 * producer that quantises once (for example bitlinear_rmsnorm_quant_act)
 * feeds several matrices, and so that the contraction can be timed on its
 * own.  Dense or N:M weights; always the tensor-core GEMM (any M >= 1); the
 * same bits as bitlinear_forward / bitlinear_forward_nm on the x the codes came
 * from.
 * q        device, int8 [M, ldq]: codes in natural K order; ldq >= K and a
 *          multiple of 16 (bitlinear_quant_act writes ldq = K, so K % 16 == 0
 *          there, or copy into a padded buffer); bytes K .. ldq - 1 of every
 *          row zero; 16-byte aligned.
 * gamma    device, fp32 [M];  rowsum  device, int32 [M] (sum of each row's codes).
 * y, acc   as bitlinear_forward.
 * workspace, workspace_bytes: device scratch of at least
 *          bitlinear_forward_q8_workspace_bytes(M, N, K) (0 when the GEMM does
 *          not split K; then NULL is accepted).
 * flags    BITLINEAR_FLAG_PDL (the GEMM is always launched as a programmatic
 *          dependent), BITLINEAR_FLAG_PATH_TC (accepted), BITLINEAR_FLAG_NM24_EXPAND.
 * Errors: NULL, SHAPE (also ldq < K or not a multiple of 16), ALIGN, PATTERN,
 *         WORKSPACE, FLAGS, DEVICE, CUDA. */
bitlinear_status bitlinear_forward_q8(const bitlinear_weights* w, const int8_t* q, int32_t ldq, const float* gamma,
                                      const int32_t* rowsum, int32_t M, uint16_t* y, int32_t* acc, void* workspace,
                                      size_t workspace_bytes, uint32_t flags, void* stream);
size_t bitlinear_forward_q8_workspace_bytes(int32_t M, int32_t N, int32_t K);

/* Workspace bytes needed by bitlinear_forward / bitlinear_forward_nm.  0 when
 * the call takes the M = 1 GEMV path (which quantises in-kernel).  The
 * tensor-core path needs the int8 codes, gamma and code sums of x and, when it
 * splits K across SMs (few tokens or few weight rows), ksplit int32 [M, N]
 * partial-sum slabs; the size depends on the current device's SM count.  The
 * workspace holds no state between calls. */
size_t bitlinear_forward_workspace_bytes(int32_t M, int32_t N, int32_t K, uint32_t flags);

/* y = BitLinear(x) for dense packed weights.
 * w        host struct describing device buffers; w->nm_n == w->nm_m == 0.
 * x        device, bf16 bits [M, K] (16-byte aligned).
 * y        device, out: bf16 bits [M, N].
 * acc      device, out (may be NULL): int32 [M, N], the exact accumulator.
 * workspace, workspace_bytes: device scratch (may be NULL when 0 is needed).
 * flags    BITLINEAR_FLAG_*.
 * Path: M == 1 takes the streaming GEMV.  2 <= M <= 64 (or M == 1 with
 * BITLINEAR_FLAG_PATH_TC) takes the fused few-token tensor-core kernel: one
 * launch that quantises, contracts on tcgen05 with K split over the CTAs of a
 * thread-block cluster and reduced through distributed shared memory, and
 * rescales; it needs no workspace (and reads none it is given) when K fits
 * eight slices of resident weights (K <= 8 * 24 * 128 for up to 32 tokens).
 * Larger M, longer K, or BITLINEAR_FLAG_PATH_PERSISTENT take the persistent
 * tcgen05 GEMM after a quantisation launch.  Every path gives the same bits.
 * Errors: NULL, SHAPE, ALIGN, PATTERN, WORKSPACE, FLAGS, DEVICE, CUDA. */
bitlinear_status bitlinear_forward(const bitlinear_weights* w, const uint16_t* x, int32_t M, uint16_t* y,
                                   int32_t* acc, void* workspace, size_t workspace_bytes, uint32_t flags,
                                   void* stream);

/* Same as bitlinear_forward for N:M packed weights (w->nm_n/nm_m = 2,4 or n,8).
 * Path: M == 1 takes the N:M streaming GEMV; otherwise (or with
 * BITLINEAR_FLAG_PATH_TC) a quantisation launch and the persistent tcgen05
 * GEMM.  There 2:4 weights run on the structured-sparse MMA
 * (tcgen05.mma.sp kind::i8: the kept values as signed int8, the packed
 * metadata unchanged, activation codes in natural K order), the Sparse-BitNet
 * review's sparse tensor-core path (section 4); n:8 weights, and 2:4 with
 * BITLINEAR_FLAG_NM24_EXPAND, are expanded to dense codes for the dense MMA.
 * Every path gives the same bits. */
bitlinear_status bitlinear_forward_nm(const bitlinear_weights* w, const uint16_t* x, int32_t M, uint16_t* y,
                                      int32_t* acc, void* workspace, size_t workspace_bytes, uint32_t flags,
                                      void* stream);

/* Several BitLinear layers applied to the same input, e.g. the gate and up
 * projections of one feed-forward block, or q, k and v.  The method defines
 * each layer on its own ("BitNet b1.58 2B4T Technical Report", section 2
 * Architecture, BitLinear; the activation quantisation depends on x alone),
 * so quantising x once for all of them changes no result: every y[i] equals
 * bitlinear_forward /
 * bitlinear_forward_nm of w[i] on x, bit for bit.  Only the launches and the
 * repeated quantisation are saved.
 * w        host array of count structs (1 <= count <= BITLINEAR_MAX_GROUP),
 *          dense or N:M, all with the same K.
 * x        device, bf16 bits [M, K] (16-byte aligned).
 * y        host array of count device pointers, out: bf16 bits [M, w[i].N].
 * acc      NULL, or a host array of count device pointers (each may be NULL):
 *          int32 [M, w[i].N].
 * workspace, workspace_bytes: at least bitlinear_forward_workspace_bytes(M, w[i].N, K,
 *          flags) for every i.
 * flags    as for bitlinear_forward; PDL applies to the first kernel the call
 *          launches (the later ones follow kernels of the same call).
 * Path: M == 1 runs the dense matrices in one GEMV launch (CTAs split among
 * them by rows) and each N:M matrix in its own; 2 <= M <= 64 with dense
 * weights runs the fused few-token kernel once per matrix (see
 * bitlinear_forward); otherwise the call quantises once and runs one
 * persistent tensor-core GEMM per matrix.
 * Errors: as bitlinear_forward; SHAPE also for count out of range or unequal K. */
bitlinear_status bitlinear_forward_group(const bitlinear_weights* w, int32_t count, const uint16_t* x, int32_t M,
                                         uint16_t* const* y, int32_t* const* acc, void* workspace,
                                         size_t workspace_bytes, uint32_t flags, void* stream);

/* ---------------------------------------------------------------------------
 * FFN gate/up pair with squared ReLU.
 *
 * Source: BitNet b1.58 2B4T technical report summary (greeksharifa.github.io
 * page), section 2 "Architecture": the FFN sublayer uses squared ReLU, the
 * rectified activation squared.  With the block's gate and up projections
 * (two BitLinears of the same x) the result is taken as, elementwise,
 *     h = RN_bf16( RN_bf16( max(g, 0)^2 ) * u ),
 * g = BitLinear_gate(x) and u = BitLinear_up(x) in bf16 exactly as
 * bitlinear_forward returns them, each bf16 operation rounded once.
 *
 * w_gate, w_up: packed weights of the same N and K (dense or N:M), device.
 * x: bf16 bits [M, K], device, 16-byte aligned.  h: bf16 bits [M, N], device.
 * workspace: device scratch of at least
 * bitlinear_forward_relu2_glu_workspace_bytes(M, N, K, flags) bytes, 16-byte
 * aligned (g and u for M > 1, then the forward's own workspace); may be NULL
 * when M = 1, both matrices are dense, K <= 22528 (the rows of both matrices
 * fit one CTA's shared memory) and BITLINEAR_FLAG_PATH_TC is not set: then one
 * launch computes both BitLinears and h.  Otherwise the pair runs as
 * bitlinear_forward_group into the workspace and h is formed by one more
 * launch.  flags: as bitlinear_forward (BITLINEAR_FLAG_DECODE_LUT rejected).
 * Errors: NULL, SHAPE (N or K differ, M out of range), ALIGN, FLAGS,
 * WORKSPACE, PATTERN, DEVICE, CUDA; h is then unspecified.
 * ------------------------------------------------------------------------- */
size_t bitlinear_forward_relu2_glu_workspace_bytes(int32_t M, int32_t N, int32_t K, uint32_t flags);
bitlinear_status bitlinear_forward_relu2_glu(const bitlinear_weights* w_gate, const bitlinear_weights* w_up,
                                             const uint16_t* x, int32_t M, uint16_t* h, void* workspace,
                                             size_t workspace_bytes, uint32_t flags, void* stream);

/* Largest scratch, in bytes, that bitlinear_forward_noalloc can use. */
#define BITLINEAR_NOALLOC_SCRATCH_BYTES (8u << 20)

/* bitlinear_forward / bitlinear_forward_nm (chosen by w->nm_m) for callers
 * that cannot allocate device memory: the call needs no workspace argument
 * and performs no allocation of any kind.  The papers have no counterpart to
 * this entry point; it exists for integration only.
 *
 * Who needs it: a host that hands the library only its input and output
 * buffers and owns no allocator -- for example a plugin inside an inference
 * server or an embedded deployment whose device memory budget is reserved at
 * start-up -- and latency-critical callers that may not call cudaMalloc /
 * cudaFree on their hot path, because those calls can synchronise the whole
 * device and take unbounded time.
 *
 * How: the scratch the tensor-core path needs (quantised activations, per-
 * token scales and code sums) lives in one fixed device array of
 * BITLINEAR_NOALLOC_SCRATCH_BYTES inside the library; every GPU that loads
 * the library holds that array until the process exits.  The first call on
 * each device looks the array's device address up (with that device
 * current); make that first call before any stream capture.
 *
 * Limits: the one test is bitlinear_forward_workspace_bytes(M, N, K, flags)
 * <= BITLINEAR_NOALLOC_SCRATCH_BYTES; larger shapes are rejected with
 * BITLINEAR_ERR_WORKSPACE and nothing is enqueued.  For example M = 2048
 * tokens fits up to K = 4080 when the tensor-core plan does not split K
 * (enough weight rows, e.g. N >= 2048); with few weight rows the K split adds
 * M * N fp32 partial sums, so the same M and K may not fit.  All calls on a device share the one array and
 * it keeps the previous call's contents, which this call overwrites before
 * reading; two calls whose work overlaps on the GPU (different streams, no
 * ordering between them) race on it and may return wrong results.
 * Arguments, outputs and the other errors are those of bitlinear_forward. */
bitlinear_status bitlinear_forward_noalloc(const bitlinear_weights* w, const uint16_t* x, int32_t M, uint16_t* y,
                                           int32_t* acc, uint32_t flags, void* stream);

/* Synchronises stream and reads the current device's status word into *code
 * (0 = no kernel gave up on a wait).  If clear != 0 the word is reset.
 * Codes: 1 weight/activation copies, 2 weight unpacking, 3 MMA issue, 4
 * epilogue (the role whose wait ran out); 5 the wait for copies or MMAs
 * already issued ran out as well; 6 a kernel found its dynamic shared memory
 * misaligned and did nothing.  Outputs of a call that set a code are
 * undefined. */
bitlinear_status bitlinear_device_status(void* stream, int32_t* code, int32_t clear);

/* Name of the kernel variant the last successful call on this host thread
 * enqueued (a static string; "" before the first call).  With the environment
 * variable BITLINEAR_LOG set to a non-empty value other than "0" when the
 * library is first used, every such call also writes "bitlinear: <name>" on
 * a line of stderr. */
const char* bitlinear_last_kernel(void);

/* BITLINEAR_LAYOUT_VERSION of the compiled library: the version of the packed
 * layouts described at the top of this header.  Buffers packed under another
 * version must be packed again from the latent (or ternary) weights. */
int32_t bitlinear_layout_version(void);

/* Human-readable name of a status code (static string). */
const char* bitlinear_status_string(bitlinear_status s);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_H_ */
