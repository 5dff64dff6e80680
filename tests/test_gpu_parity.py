"""Parity of the CUDA path (through the C ABI) with the oracle, on seeded inputs.

Integer results (activation codes, gamma, packed bytes, alpha, N:M metadata,
int32 accumulators) must match bit for bit.  bf16 outputs must lie within one
bf16 ulp of the oracle's: the oracle rounds acc * alpha * gamma / 127 once
from fp64, the kernels form RN(RN(alpha * gamma) / 127) and one fp32 multiply
(relative error below 2 fp32 ulp) before the bf16 rounding, so the two can
differ only where that product sits next to a bf16 rounding boundary.

Workloads follow the pages' layer shapes (BitNet b1.58 2B4T: 2560 / 6912 /
640; Qwen2.5-3B MLP: 2048 / 11008).  Small cases are checked in full; the
full-size prefill cases run the kernel at full size and check sampled tokens
(every output of those tokens), since the oracle is a plain triple loop.
"""
import numpy as np
import pytest

import oracle
from ternary_weight_linear_fwd_b200 import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import ternary_weight_linear_fwd_b200 as bl  # noqa: E402

DEV = torch.device("cuda:0")
BF16_ULP_TOL = 1


@pytest.fixture(scope="module", autouse=True)
def _built():
    from ternary_weight_linear_fwd_b200 import build as b
    b.build()
    oracle.build()
    yield
    torch.cuda.synchronize()
    assert bl.device_status() == 0


def to_dev_bf16(x_bits):
    return torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).to(DEV).view(torch.bfloat16)


def bf16_bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def assert_bf16_close(got_bits, ref_bits):
    d = np.abs(got_bits.astype(np.int32) - ref_bits.astype(np.int32))
    # same sign everywhere (acc is exact on both sides), so the bit distance is the ulp distance
    assert d.max() <= BF16_ULP_TOL, f"max bf16 ulp distance {d.max()} at {np.unravel_index(d.argmax(), d.shape)}"
    assert (d > 0).mean() < 0.01


# ---------------------------------------------------------------- activation quantisation

@pytest.mark.parametrize("M,K", [(8, 256), (5, 200), (3, 203), (1, 6912), (64, 11008), (2048, 2560), (2, 40000)])
def test_quant_act_bit_exact(M, K):
    x = synth.activations(M, K, seed=M + K)
    q, g, rs = bl.quant_act(to_dev_bf16(x))
    qo, go, rso = oracle.quant_act(x)
    np.testing.assert_array_equal(q.cpu().numpy(), qo)
    np.testing.assert_array_equal(g.cpu().numpy(), go)
    np.testing.assert_array_equal(rs.cpu().numpy(), rso)


def test_quant_act_zero_and_constant_rows():
    x = synth.activations(4, 320, seed=9)
    x[1] = 0
    x[2] = synth.to_bf16_bits(np.full(320, -3.5, np.float32))
    q, g, rs = bl.quant_act(to_dev_bf16(x))
    qo, go, rso = oracle.quant_act(x)
    np.testing.assert_array_equal(q.cpu().numpy(), qo)
    np.testing.assert_array_equal(g.cpu().numpy(), go)
    assert not qo[1].any() and np.all(qo[2] == -127)


# ---------------------------------------------------------------- weight packing

@pytest.mark.parametrize("N,K", [(512, 256), (33, 200), (7, 3), (6912, 2560), (2560, 6912)])
def test_pack_dense_bit_exact(N, K):
    W = synth.latent_weights(N, K, seed=3)
    ref = oracle.pack_weights(W)
    w = bl.pack_weights(torch.from_numpy(W).to(DEV))
    assert float(w.alpha.cpu()[0]) == float(ref["alpha"])
    np.testing.assert_array_equal(w.codes.cpu().numpy(), ref["codes"])


def test_pack_ternary_bit_exact():
    T = synth.ternary_weights(6912, 2560, seed=1)
    a = synth.alpha_uniform(1)
    w = bl.pack_ternary(torch.from_numpy(T).to(DEV), float(a))
    np.testing.assert_array_equal(w.codes.cpu().numpy(), oracle.pack_dense(T))
    assert float(w.alpha.cpu()[0]) == float(a)


@pytest.mark.parametrize("n,m", [(2, 4), (6, 8), (7, 8), (5, 8), (3, 8), (2, 8), (1, 8)])
@pytest.mark.parametrize("N,K", [(40, 256), (24, 1032), (11008, 2048), (2048, 11008)])
def test_pack_nm_bit_exact(n, m, N, K):
    if N * K > 1_000_000 and (n, m) not in ((2, 4), (6, 8)):
        pytest.skip("full-size shapes only for the 2:4 and 6:8 patterns")
    if K % m:
        pytest.skip("K must be a multiple of m")
    W = synth.latent_weights(N, K, seed=5)
    W[0, :16] = 0.01  # tie-heavy blocks exercise the lower-position rule
    ref = oracle.pack_weights(W, n, m)
    w = bl.pack_weights(torch.from_numpy(W).to(DEV), n, m)
    assert float(w.alpha.cpu()[0]) == float(ref["alpha"])
    np.testing.assert_array_equal(w.codes.cpu().numpy(), ref["values"])
    np.testing.assert_array_equal(w.meta.cpu().numpy(), ref["meta"])


# ---------------------------------------------------------------- forward helpers

def _dense_case(M, K, N, seed, ternary=False):
    x = synth.activations(M, K, seed=seed)
    if ternary:
        T = synth.ternary_weights(N, K, seed=seed)
        a = synth.alpha_uniform(seed)
        w = bl.pack_ternary(torch.from_numpy(T).to(DEV), float(a))
        return x, T, np.float32(a), w
    W = synth.latent_weights(N, K, seed=seed)
    ref = oracle.pack_weights(W)
    w = bl.pack_weights(torch.from_numpy(W).to(DEV))
    return x, ref["Wt"], ref["alpha"], w


def _check_rows(x, Wt, alpha, y, acc, rows):
    yo, acco, *_ = oracle.forward(x[rows], Wt, alpha)
    np.testing.assert_array_equal(acc.cpu().numpy()[rows], acco)
    assert_bf16_close(bf16_bits(y)[rows], yo)


# ---------------------------------------------------------------- dense forward

@pytest.mark.parametrize("M,K,N", [(1, 256, 512), (1, 2560, 6912), (1, 6912, 2560), (1, 2560, 640),
                                   (1, 200, 33), (1, 11008, 2048), (1, 20480, 96)])
def test_forward_gemv_m1(M, K, N):
    x, Wt, a, w = _dense_case(M, K, N, seed=K + N, ternary=(K, N) in ((2560, 6912), (6912, 2560)))
    y, acc = bl.forward(w, to_dev_bf16(x), want_acc=True)
    assert bl.last_kernel() == "gemv_m1_dense"
    _check_rows(x, Wt, a, y, acc, np.arange(M))


# Decode GEMV row splits and chunk counts: 47 rows per CTA with an odd number
# of 64-weight chunks (K = 2624), 64 rows with a ragged last chunk (K = 2600),
# 64- and 65-row CTAs in one launch, 32 rows with a single chunk (K = 64), 94
# rows (the grouped gate+up shape), and the RMSNorm variant on 2560 -> 6912.
@pytest.mark.parametrize("K,N", [(2624, 6956), (2600, 9472), (2600, 9477), (64, 4736), (1024, 13912)])
def test_forward_gemv_row_splits(K, N):
    x, Wt, a, w = _dense_case(1, K, N, seed=K + 3 * N)
    y, acc = bl.forward(w, to_dev_bf16(x), want_acc=True)
    assert bl.last_kernel() == "gemv_m1_dense"
    _check_rows(x, Wt, a, y, acc, np.arange(1))


def test_forward_norm_gemv_gate_shape():
    K, N = 2560, 6912
    x, Wt, a, w = _dense_case(1, K, N, seed=41)
    g = _norm_weight(K, 5)
    y, acc = bl.forward_norm(w, to_dev_bf16(x), torch.from_numpy(g).to(DEV), 1e-5, want_acc=True)
    assert bl.last_kernel() == "gemv_m1_dense"
    yo, acco, *_ = oracle.forward_norm(x, g, 1e-5, Wt, a)
    np.testing.assert_array_equal(acc.cpu().numpy(), acco)
    assert_bf16_close(bf16_bits(y), yo)


@pytest.mark.parametrize("M,K,N", [(8, 256, 512), (2, 256, 512), (16, 2560, 640), (20, 203, 130), (300, 1000, 400),
                                   (1, 2560, 6912), (130, 384, 256), (64, 128, 128), (13, 256, 9600)])
def test_forward_tc_full(M, K, N):
    x, Wt, a, w = _dense_case(M, K, N, seed=M * 7 + K)
    y, acc = bl.forward(w, to_dev_bf16(x), want_acc=True, flags=bl.FLAG_PATH_TC)
    assert bl.last_kernel().startswith(("tc_gemm_dense", "tc_skinny"))
    _check_rows(x, Wt, a, y, acc, np.arange(M))
    y2, acc2 = bl.forward(w, to_dev_bf16(x), want_acc=True, flags=bl.FLAG_PATH_TC | bl.FLAG_PATH_PERSISTENT)
    assert bl.last_kernel().startswith(("tc_gemm_dense", "tc2_gemm_dense"))
    assert torch.equal(acc, acc2) and torch.equal(y.view(torch.int16), y2.view(torch.int16))


# The fused few-token kernel: token tiles of 16, 32 and 64; one to eight K slices per cluster (2560 -> 6912:
# two; 6912 -> 2560: seven or fewer; 11008 -> 2048: eight); a ragged K (203: a partial 16-group and chunk)
# and N (130, 1, 33); the forced tensor-core path at M = 1.  Every output is checked against the oracle and
# against the persistent GEMM bit for bit.
@pytest.mark.parametrize("M,K,N", [(2, 256, 512), (16, 2560, 6912), (16, 6912, 2560), (16, 2560, 640),
                                   (32, 2560, 2560), (64, 2560, 6912), (33, 203, 130), (5, 11008, 2048),
                                   (64, 2048, 11008), (9, 1000, 1), (17, 384, 33), (1, 2560, 6912)])
def test_forward_skinny(M, K, N):
    x, Wt, a, w = _dense_case(M, K, N, seed=M * 11 + K + N, ternary=(K, N) in ((2560, 6912), (6912, 2560)))
    xd = to_dev_bf16(x)
    y, acc = bl.forward(w, xd, want_acc=True, flags=bl.FLAG_PATH_TC if M == 1 else 0)
    assert bl.last_kernel().startswith("tc_skinny"), bl.last_kernel()
    _check_rows(x, Wt, a, y, acc, np.arange(M))
    y2, acc2 = bl.forward(w, xd, want_acc=True, flags=bl.FLAG_PATH_TC | bl.FLAG_PATH_PERSISTENT)
    assert torch.equal(acc, acc2) and torch.equal(y.view(torch.int16), y2.view(torch.int16))
    y3 = bl.forward(w, xd, flags=bl.FLAG_PDL | (bl.FLAG_PATH_TC if M == 1 else 0))  # no acc, programmatic launch
    assert torch.equal(y.view(torch.int16), y3.view(torch.int16))


def test_forward_skinny_zero_and_outlier_tokens():
    """A zero token, a single huge outlier and a constant token in one few-token call."""
    M, K, N = 12, 2560, 640
    x = synth.activations(M, K, seed=13)
    x[3] = 0
    x[5, 1234] = synth.to_bf16_bits(np.array([3.0e4], np.float32))[0]
    x[7] = synth.to_bf16_bits(np.full(K, -0.75, np.float32))
    W = synth.latent_weights(N, K, seed=13)
    ref = oracle.pack_weights(W)
    w = bl.pack_weights(torch.from_numpy(W).to(DEV))
    y, acc = bl.forward(w, to_dev_bf16(x), want_acc=True)
    assert bl.last_kernel().startswith("tc_skinny")
    _check_rows(x, ref["Wt"], ref["alpha"], y, acc, np.arange(M))
    assert not bf16_bits(y)[3].any()


@pytest.mark.parametrize("K,N", [(2560, 6912), (6912, 2560), (2560, 2560), (2560, 640)])
def test_forward_tc_prefill_2b4t_sampled(K, N):
    """Prefill workload (M = 2048 tokens) at full size; 48 sampled tokens checked in full."""
    M = 2048
    x, Wt, a, w = _dense_case(M, K, N, seed=3)
    y, acc = bl.forward(w, to_dev_bf16(x), want_acc=True)
    rows = np.unique(np.concatenate([[0, 255, 256, M - 1], synth.splitmix64(3, 77, 44) % M])).astype(np.int64)
    _check_rows(x, Wt, a, y, acc, rows)


@pytest.mark.parametrize("M", [16, 256])
def test_forward_layer_sweep_shapes(M):
    """The seven 2B4T layer matrices at M = 16 and 256 (sampled tokens)."""
    for name, (K, N) in synth.B2B4T_LAYER.items():
        x, Wt, a, w = _dense_case(M, K, N, seed=4)
        y, acc = bl.forward(w, to_dev_bf16(x), want_acc=True)
        rows = np.arange(M) if M <= 16 else np.unique(synth.splitmix64(4, 5, 24) % M).astype(np.int64)
        _check_rows(x, Wt, a, y, acc, rows)


def test_forward_layer_sweep_m4096_sampled():
    """The seven 2B4T layer matrices at M = 4096 tokens through bitlinear_forward's default path (the
    largest configuration of the layer sweep): the kernels run at full size, 20 sampled tokens (the
    first, the last, the edges of the 128-token tiles around the middle and 15 drawn at random) are
    checked against the oracle on every output."""
    M = 4096
    rows = np.unique(np.concatenate([[0, 127, 128, 2047, 2048, M - 1], synth.splitmix64(4096, 6, 15) % M]))
    rows = rows.astype(np.int64)
    for name, (K, N) in synth.B2B4T_LAYER.items():
        x, Wt, a, w = _dense_case(M, K, N, seed=4)
        y, acc = bl.forward(w, to_dev_bf16(x), want_acc=True)
        assert bl.last_kernel().startswith(("tc_gemm_dense", "tc2_gemm_dense")), (name, bl.last_kernel())
        _check_rows(x, Wt, a, y, acc, rows)


def test_forward_stale_workspace():
    """A caller workspace full of 0xFF bytes gives the same results as a fresh one: every byte the GEMM
    reads is written (codes, scales, code sums) or cleared (split-K sums and counters) by the call itself.
    Shapes: a K-split GEMM (few row tiles), then a tile-parallel one, then the split one again."""
    cases = [(16, 2560, 640), (300, 1000, 2048), (16, 2560, 640)]
    ws = torch.full((max(bl.forward_workspace_bytes(M, N, K) for M, K, N in cases),), 0xFF, dtype=torch.uint8,
                    device=DEV)
    for M, K, N in cases:
        x, Wt, a, w = _dense_case(M, K, N, seed=M + N)
        y, acc = bl.forward(w, to_dev_bf16(x), want_acc=True, workspace=ws, flags=bl.FLAG_PATH_PERSISTENT)
        assert bl.last_kernel().startswith(("tc_gemm_dense", "tc2_gemm_dense"))
        _check_rows(x, Wt, a, y, acc, np.arange(M))
        ws.fill_(0xFF)


def test_pack_dense_exact_ties():
    """Latent weights at exactly +-0.5 * d and +-1.5 * d, d = RN(alpha + 1e-5), ternarise to 0 and to +-1
    (round half to even, then the clamp), and the next float above 0.5 * d to +-1, on the GPU as in the
    oracle.  alpha depends on the tie entries themselves, so they are placed by a fixed-point iteration:
    alpha of the final matrix is the alpha the ties were computed from (the sums of fp32 magnitudes are
    exact in fp64 here, so the kernel's summation order cannot change it)."""
    N, K = 96, 520
    W = synth.latent_weights(N, K, seed=44)
    rows = [0, 1, 47, 95]
    for _ in range(50):
        a = oracle.absmean(W)
        d = np.float32(a + np.float32(1e-5))
        h = np.float32(d * np.float32(0.5))
        t = np.float32(np.float32(3) * h)
        above = np.nextafter(h, np.float32(1))
        vals = [h, -h, above, -above]
        if np.float64(t) == 3.0 * np.float64(h):  # 1.5 d is representable: include that tie as well
            vals += [t, -t]
        for r in rows:
            W[r, 3:3 + len(vals)] = vals
        if oracle.absmean(W) == a:
            break
    else:
        pytest.fail("no fixed point for alpha")
    expect = [0, 0, 1, -1] + ([1, -1] if len(vals) == 6 else [])
    ref = oracle.pack_weights(W)
    for r in rows:
        np.testing.assert_array_equal(ref["Wt"][r, 3:3 + len(vals)], expect)
    w = bl.pack_weights(torch.from_numpy(W).to(DEV))
    assert float(w.alpha.cpu()[0]) == float(ref["alpha"])
    np.testing.assert_array_equal(w.codes.cpu().numpy(), ref["codes"])
    for n, m in ((2, 4), (6, 8)):
        refn = oracle.pack_weights(W, n, m)
        wn = bl.pack_weights(torch.from_numpy(W).to(DEV), n, m)
        np.testing.assert_array_equal(wn.codes.cpu().numpy(), refn["values"])
        np.testing.assert_array_equal(wn.meta.cpu().numpy(), refn["meta"])


def test_forward_zero_and_outlier_rows():
    M, K, N = 6, 512, 256
    x = synth.activations(M, K, seed=12)
    x[2] = 0
    x[4, 7] = synth.to_bf16_bits(np.array([3.0e4], np.float32))[0]
    W = synth.latent_weights(N, K, seed=12)
    ref = oracle.pack_weights(W)
    w = bl.pack_weights(torch.from_numpy(W).to(DEV))
    y, acc = bl.forward(w, to_dev_bf16(x), want_acc=True)
    _check_rows(x, ref["Wt"], ref["alpha"], y, acc, np.arange(M))
    assert not bf16_bits(y)[2].any()
    y1, acc1 = bl.forward(w, to_dev_bf16(x[2:3]), want_acc=True)
    assert not acc1.cpu().numpy().any() and not bf16_bits(y1).any()


def test_forward_pdl_flag_same_result():
    x, Wt, a, w = _dense_case(33, 640, 300, seed=21)
    xd = to_dev_bf16(x)
    y0, acc0 = bl.forward(w, xd, want_acc=True)
    y1, acc1 = bl.forward(w, xd, want_acc=True, flags=bl.FLAG_PDL)
    assert torch.equal(acc0, acc1) and torch.equal(y0.view(torch.int16), y1.view(torch.int16))
    x1 = to_dev_bf16(x[:1])
    ya = bl.forward(w, x1)
    yb = bl.forward(w, x1, flags=bl.FLAG_PDL)
    assert torch.equal(ya.view(torch.int16), yb.view(torch.int16))


# ---------------------------------------------------------------- N:M forward

def _nm_case(M, K, N, n, m, seed):
    x = synth.activations(M, K, seed=seed)
    W = synth.latent_weights(N, K, seed=seed)
    ref = oracle.pack_weights(W, n, m)
    w = bl.pack_weights(torch.from_numpy(W).to(DEV), n, m)
    return x, ref["Wt"], ref["alpha"], w


@pytest.mark.parametrize("n,m", [(2, 4), (6, 8), (7, 8), (3, 8), (1, 8)])
@pytest.mark.parametrize("M,K,N", [(1, 256, 40), (1, 1032, 24), (1, 2048, 11008), (1, 11008, 2048),
                                   (5, 1032, 140), (70, 256, 300)])
def test_forward_nm(n, m, M, K, N):
    if K % m:
        pytest.skip("K must be a multiple of m")
    if N * K > 1_000_000 and (n, m) not in ((2, 4), (6, 8)):
        pytest.skip("full-size shapes only for the 2:4 and 6:8 patterns")
    x, Wt, a, w = _nm_case(M, K, N, n, m, seed=5)
    y, acc = bl.forward_nm(w, to_dev_bf16(x), want_acc=True)
    _check_rows(x, Wt, a, y, acc, np.arange(M))


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 6, 7])
def test_forward_nm_gemv_every_n8(n):
    """Decode GEMV for every n:8 pattern on a ragged shape (K not a multiple of the 128-weight unit)."""
    x, Wt, a, w = _nm_case(1, 1032, 37, n, 8, seed=40 + n)
    y, acc = bl.forward_nm(w, to_dev_bf16(x), want_acc=True)
    assert bl.last_kernel() == "gemv_m1_n8"
    _check_rows(x, Wt, a, y, acc, np.arange(1))


@pytest.mark.parametrize("n,m", [(2, 4), (6, 8)])
@pytest.mark.parametrize("K,N", [(2048, 11008), (11008, 2048)])
def test_forward_nm_prefill_qwen_sampled(n, m, K, N):
    """Qwen2.5-3B MLP shapes at M = 4096 tokens; 24 sampled tokens checked in full."""
    M = 4096
    x, Wt, a, w = _nm_case(M, K, N, n, m, seed=5)
    y, acc = bl.forward_nm(w, to_dev_bf16(x), want_acc=True)
    rows = np.unique(np.concatenate([[0, M - 1], synth.splitmix64(5, 78, 22) % M])).astype(np.int64)
    _check_rows(x, Wt, a, y, acc, rows)


def test_forward_nm_m1_forced_tc_matches_gemv():
    x, Wt, a, w = _nm_case(1, 2048, 1000, 6, 8, seed=8)
    xd = to_dev_bf16(x)
    y0, acc0 = bl.forward_nm(w, xd, want_acc=True)
    y1, acc1 = bl.forward_nm(w, xd, want_acc=True, flags=bl.FLAG_PATH_TC)
    assert torch.equal(acc0, acc1)
    _check_rows(x, Wt, a, y1, acc1, np.arange(1))


# ---------------------------------------------------------------- 2:4 on the structured-sparse MMA

@pytest.mark.parametrize("M,K,N", [(2, 256, 128), (37, 1032, 300), (300, 2048, 520), (128, 4100, 257),
                                   (1, 768, 130), (2048, 2048, 1100)])
def test_forward_nm24_sparse_mma_matches_expanded_and_oracle(M, K, N):
    """2:4 weights on tcgen05.mma.sp (kept values as int8, packed metadata in TMEM, natural-order codes)
    against the expanded dense MMA of the same call (bit for bit) and the oracle (every token)."""
    x, Wt, a, w = _nm_case(M, K, N, 2, 4, seed=K + N)
    xd = to_dev_bf16(x)
    y, acc = bl.forward_nm(w, xd, want_acc=True, flags=bl.FLAG_PATH_TC if M == 1 else 0)
    assert bl.last_kernel().startswith(("tc_gemm_sp24", "tc2_gemm_sp24")), bl.last_kernel()
    ye, acce = bl.forward_nm(w, xd, want_acc=True, flags=bl.FLAG_NM24_EXPAND | (bl.FLAG_PATH_TC if M == 1 else 0))
    assert bl.last_kernel().startswith("tc_gemm_nm24"), bl.last_kernel()
    assert torch.equal(acc, acce) and torch.equal(y.view(torch.int16), ye.view(torch.int16))
    _check_rows(x, Wt, a, y, acc, np.arange(M))


def test_forward_nm24_sparse_mma_tie_decides_kept_pair():
    """Blocks whose latent magnitudes tie (all four equal, or three equal largest): the mask rule decides which
    two positions are kept, the pack must keep the same pair as the oracle, and the sparse MMA must then
    contract exactly those positions (acc bit-exact against the oracle on every token)."""
    M, K, N = 96, 512, 160
    W = synth.latent_weights(N, K, seed=91)
    base = np.float32(3 * np.abs(W).mean())
    for r in range(0, N, 3):
        for b in range(r % 7, K // 4, 5):
            k0 = 4 * b
            if (r + b) % 2:
                W[r, k0:k0 + 4] = np.array([1, -1, 1, -1], np.float32) * base          # all four tie
            else:
                W[r, k0:k0 + 4] = np.array([0.5, 1, -1, 1], np.float32) * base         # three tie for two places
    ref = oracle.pack_weights(W, 2, 4)
    w = bl.pack_weights(torch.from_numpy(W).to(DEV), 2, 4)
    np.testing.assert_array_equal(w.codes.cpu().numpy(), ref["values"])
    np.testing.assert_array_equal(w.meta.cpu().numpy(), ref["meta"])
    x = synth.activations(M, K, seed=92)
    y, acc = bl.forward_nm(w, to_dev_bf16(x), want_acc=True)
    assert bl.last_kernel().startswith(("tc_gemm_sp24", "tc2_gemm_sp24"))
    _check_rows(x, ref["Wt"], ref["alpha"], y, acc, np.arange(M))


def test_forward_group_all_nm24_uses_sparse_mma():
    """A group of 2:4 matrices quantises once in natural order and runs each on the sparse MMA; a group
    mixing dense and 2:4 keeps the contraction order and the expanded MMA.  Both match single calls."""
    M, K = 40, 1024
    x = synth.activations(M, K, seed=93)
    xd = to_dev_bf16(x)
    specs = [(300, 2, 4), (200, 2, 4)]
    ws, refs = [], []
    for i, (N, n, m) in enumerate(specs):
        W = synth.latent_weights(N, K, seed=94 + i)
        refs.append(oracle.pack_weights(W, n, m))
        ws.append(bl.pack_weights(torch.from_numpy(W).to(DEV), n, m))
    outs = bl.forward_group(ws, xd, want_acc=True)
    assert bl.last_kernel().startswith(("tc_gemm_sp24", "tc2_gemm_sp24"))
    for w, ref, (y, acc) in zip(ws, refs, outs):
        y1, acc1 = bl.forward_nm(w, xd, want_acc=True)
        assert torch.equal(acc, acc1) and torch.equal(y.view(torch.int16), y1.view(torch.int16))
        _check_rows(x, ref["Wt"], ref["alpha"], y, acc, np.arange(M))
    Wd = synth.latent_weights(130, K, seed=97)
    refd = oracle.pack_weights(Wd)
    wd = bl.pack_weights(torch.from_numpy(Wd).to(DEV))
    outs = bl.forward_group([ws[0], wd], xd, want_acc=True, flags=bl.FLAG_PATH_PERSISTENT)
    for ref, (y, acc) in zip([refs[0], refd], outs):
        _check_rows(x, ref["Wt"], ref["alpha"], y, acc, np.arange(M))


# ---------------------------------------------------------------- pairs of SMs (cta_group::2)

def _check_pair_kernel(prefix, bn):
    """The pair GEMM ran, with the token tile the host picks on a 148-SM B200."""
    if torch.cuda.get_device_properties(0).multi_processor_count == 148:
        assert bl.last_kernel() == f"{prefix}_bn{bn}", bl.last_kernel()
    else:
        assert bl.last_kernel().startswith(prefix), bl.last_kernel()


# Shapes whose plan is 128-token tiles without a K split (at least 75 tiles of 128 x 128), so the GEMM
# runs on CTA pairs sharing one M = 256 MMA: ragged M (a last tile of 1 or 44 tokens), ragged N (the
# last pair tile's second CTA partly or wholly past N), K not a multiple of the 256-k stage.
# The token tile (128 to 224 tokens a pair) follows the rounds of pairs a shape takes on 148 SMs: codes in
# TMEM at 128 tokens, in shared memory for the wider tiles.
@pytest.mark.parametrize("M,K,N,bn", [(1000, 2560, 2000, 128), (4096, 1032, 640, 192), (300, 2048, 11008, 128),
                                      (129, 6912, 9000, 128), (4736, 512, 256, 128), (2048, 2560, 2560, 160),
                                      (4000, 1032, 11000, 224)])
def test_forward_pair_gemm_dense(M, K, N, bn):
    x, Wt, a, w = _dense_case(M, K, N, seed=M + K + N)
    y, acc = bl.forward(w, to_dev_bf16(x), want_acc=True)
    _check_pair_kernel("tc2_gemm_dense", bn)
    edges = [0, bn // 2 - 1, bn // 2, bn - 1, bn, M - 1]  # each CTA's token half
    rows = np.arange(M) if M * N <= 3_000_000 else np.unique(np.concatenate(
        [[t for t in edges if t < M], synth.splitmix64(M, 7, 18) % M])).astype(np.int64)
    _check_rows(x, Wt, a, y, acc, rows)


# The wide tiles run here with a ragged last token tile, ragged N and K off the 256-k stage.
@pytest.mark.parametrize("M,K,N,bn", [(1000, 2048, 2000, 128), (129, 4096, 9000, 128), (2048, 11008, 2048, 128),
                                      (4736, 512, 256, 128), (2048, 2560, 2560, 160), (3001, 1544, 2050, 192),
                                      (4000, 1032, 11000, 224), (4096, 2048, 11008, 224)])
def test_forward_pair_gemm_sparse24(M, K, N, bn):
    """2:4 weights on the pair's structured-sparse MMA, against the expanded one-CTA kernel (bit for bit)
    and the oracle (sampled tokens)."""
    x, Wt, a, w = _nm_case(M, K, N, 2, 4, seed=M + K)
    xd = to_dev_bf16(x)
    y, acc = bl.forward_nm(w, xd, want_acc=True)
    _check_pair_kernel("tc2_gemm_sp24", bn)
    ye, acce = bl.forward_nm(w, xd, want_acc=True, flags=bl.FLAG_NM24_EXPAND)
    assert torch.equal(acc, acce) and torch.equal(y.view(torch.int16), ye.view(torch.int16))
    edges = [t for t in (0, bn // 2 - 1, bn // 2, bn - 1, bn, M - 1) if t < M]  # each CTA's token half
    rows = np.unique(np.concatenate([edges, synth.splitmix64(M, 8, 12) % M])).astype(np.int64)
    _check_rows(x, Wt, a, y, acc, rows)


# n:8 weights on the pair GEMM: kept codes and masks expanded to dense codes (in TMEM at 128-token tiles,
# in shared memory at wider ones, even n only), checked bit for bit against the same pruned ternary matrix
# packed dense, and against the oracle.
@pytest.mark.parametrize("M,K,N,n,bn", [(1000, 2048, 2000, 6, 128), (1000, 2048, 2000, 1, 128),
                                        (1000, 2048, 2000, 3, 128), (1000, 2048, 2000, 7, 128),
                                        (4096, 1032, 640, 6, 192), (300, 2048, 11008, 6, 128),
                                        (2048, 2560, 2560, 5, 128), (4000, 1032, 11000, 6, 224),
                                        (2048, 6912, 2560, 6, 160), (3001, 1544, 2050, 2, 192),
                                        (2048, 2560, 6912, 4, 224)])
def test_forward_pair_gemm_n8(M, K, N, n, bn):
    x, Wt, a, w = _nm_case(M, K, N, n, 8, seed=M + K + n)
    xd = to_dev_bf16(x)
    y, acc = bl.forward_nm(w, xd, want_acc=True)
    _check_pair_kernel("tc2_gemm_n8", bn)
    wd = bl.pack_ternary(torch.from_numpy(np.ascontiguousarray(Wt, dtype=np.int8)).to(DEV), float(w.alpha.item()))
    yd, accd = bl.forward(wd, xd, want_acc=True)
    assert torch.equal(acc, accd) and torch.equal(y.view(torch.int16), yd.view(torch.int16))
    edges = [0, bn // 2 - 1, bn // 2, bn - 1, bn, M - 1]  # each CTA's token half
    rows = np.unique(np.concatenate([[t for t in edges if t < M], synth.splitmix64(M, 9, 12) % M])).astype(np.int64)
    _check_rows(x, Wt, a, y, acc, rows)


# ---------------------------------------------------------------- codes-in entry (the GEMM alone)

@pytest.mark.parametrize("n,m", [(0, 0), (2, 4), (6, 8)])
@pytest.mark.parametrize("M,K,N", [(1, 256, 300), (37, 1024, 640), (300, 2048, 1100), (2048, 2560, 2560)])
def test_forward_q8_matches_forward(n, m, M, K, N):
    """bitlinear_forward_q8 on the codes, gamma and code sums of bitlinear_quant_act gives the bits of
    bitlinear_forward / bitlinear_forward_nm on x (same plan, same kernels after the quantisation)."""
    x = synth.activations(M, K, seed=M + N)
    W = synth.latent_weights(N, K, seed=K + N)
    w = bl.pack_weights(torch.from_numpy(W).to(DEV), n, m)
    ref = oracle.pack_weights(W, n, m)
    xd = to_dev_bf16(x)
    q, g, rs = bl.quant_act(xd)
    y, acc = bl.forward_q8(w, q, g, rs, want_acc=True)
    fn = bl.forward_nm if m else bl.forward
    y1, acc1 = fn(w, xd, want_acc=True, flags=bl.FLAG_PATH_TC)
    assert torch.equal(acc, acc1) and torch.equal(y.view(torch.int16), y1.view(torch.int16))
    rows = np.arange(M) if M <= 300 else np.unique(np.concatenate([[0, M - 1], synth.splitmix64(M, 3, 10) % M]))
    _check_rows(x, ref["Wt"], ref["alpha"], y, acc, rows.astype(np.int64))


def test_forward_q8_padded_rows():
    """Codes in a row stride above K (K = 1000 padded to 1008, zeros past K)."""
    M, K, N = 96, 1000, 512
    x = synth.activations(M, K, seed=61)
    W = synth.latent_weights(N, K, seed=62)
    w = bl.pack_weights(torch.from_numpy(W).to(DEV))
    ref = oracle.pack_weights(W)
    q, g, rs = bl.quant_act(to_dev_bf16(x))
    qp = torch.zeros((M, 1008), dtype=torch.int8, device=DEV)
    qp[:, :K] = q
    y, acc = bl.forward_q8(w, qp, g, rs, want_acc=True)
    _check_rows(x, ref["Wt"], ref["alpha"], y, acc, np.arange(M))


# ---------------------------------------------------------------- grouped forward

@pytest.mark.parametrize("M", [1, 37])
@pytest.mark.parametrize("shapes", [((2560, 6912), (2560, 6912)), ((640, 1000), (640, 33), (640, 512), (640, 2048)),
                                    ((6912, 2560),)])
def test_forward_group_dense_matches_single_and_oracle(M, shapes):
    """gate + up of the 2B4T FFN (and a ragged 4-matrix group): each output equals the single-matrix call
    bit for bit and the oracle within the bf16 tolerance."""
    K = shapes[0][0]
    x = synth.activations(M, K, seed=31)
    xd = to_dev_bf16(x)
    cases = []
    for i, (_, N) in enumerate(shapes):
        T = synth.ternary_weights(N, K, seed=40 + i)
        a = synth.alpha_uniform(40 + i)
        cases.append((T, np.float32(a), bl.pack_ternary(torch.from_numpy(T).to(DEV), float(a))))
    rows = np.arange(M)
    # at M = 37 both the fused few-token launches and the quantise-once persistent path
    for flags in ((0,) if M == 1 else (0, bl.FLAG_PATH_PERSISTENT)):
        outs = bl.forward_group([c[2] for c in cases], xd, want_acc=True, flags=flags)
        if M == 1:
            assert bl.last_kernel() == "gemv_m1_dense"
        else:
            assert bl.last_kernel().startswith("tc_gemm_dense" if flags else "tc_skinny"), bl.last_kernel()
        for (T, a, w), (y, acc) in zip(cases, outs):
            y1, acc1 = bl.forward(w, xd, want_acc=True)
            assert torch.equal(acc, acc1) and torch.equal(y.view(torch.int16), y1.view(torch.int16))
            _check_rows(x, T, a, y, acc, rows)


def test_forward_group_mixed_dense_nm():
    K = 1024
    x = synth.activations(1, K, seed=33)
    xd = to_dev_bf16(x)
    specs = [(300, 0, 0), (200, 2, 4), (130, 6, 8)]
    ws, refs = [], []
    for i, (N, n, m) in enumerate(specs):
        W = synth.latent_weights(N, K, seed=50 + i)
        refs.append(oracle.pack_weights(W, n, m))
        ws.append(bl.pack_weights(torch.from_numpy(W).to(DEV), n, m))
    for flags in (0, bl.FLAG_PDL, bl.FLAG_PATH_TC):
        outs = bl.forward_group(ws, xd, want_acc=True, flags=flags)
        for ref, (y, acc) in zip(refs, outs):
            _check_rows(x, ref["Wt"], ref["alpha"], y, acc, np.arange(1))


def test_forward_group_prefill_sampled():
    """gate + up at M = 2048 through one quantisation and two tensor-core GEMMs (sampled tokens)."""
    M, K, N = 2048, 2560, 6912
    x = synth.activations(M, K, seed=34)
    xd = to_dev_bf16(x)
    cases = []
    for i in range(2):
        T = synth.ternary_weights(N, K, seed=60 + i)
        a = synth.alpha_uniform(60 + i)
        cases.append((T, np.float32(a), bl.pack_ternary(torch.from_numpy(T).to(DEV), float(a))))
    outs = bl.forward_group([c[2] for c in cases], xd, want_acc=True)
    rows = np.unique(np.concatenate([[0, M - 1], synth.splitmix64(34, 9, 14) % M])).astype(np.int64)
    for (T, a, w), (y, acc) in zip(cases, outs):
        _check_rows(x, T, a, y, acc, rows)


# ---------------------------------------------------------------- lookup-table decode (comparison path)

@pytest.mark.parametrize("K,N", [(256, 512), (2560, 6912), (6912, 2560), (200, 33), (1032, 300)])
def test_forward_decode_lut_matches(K, N):
    """The TL2-style lookup-table GEMV gives the dp4a GEMV's results bit for bit, and the oracle's."""
    x, Wt, a, w = _dense_case(1, K, N, seed=K + 3 * N, ternary=True)
    xd = to_dev_bf16(x)
    y, acc = bl.forward(w, xd, want_acc=True, flags=bl.FLAG_DECODE_LUT)
    assert bl.last_kernel() == "gemv_m1_dense_lut"
    y0, acc0 = bl.forward(w, xd, want_acc=True)
    assert torch.equal(acc, acc0) and torch.equal(y.view(torch.int16), y0.view(torch.int16))
    _check_rows(x, Wt, a, y, acc, np.arange(1))


# ---------------------------------------------------------------- RMSNorm before the quantisation

def _norm_weight(K, seed):
    return (0.5 + synth.uniform(seed, 11, K)).astype(np.float32)


@pytest.mark.parametrize("M,K", [(8, 256), (5, 200), (3, 203), (1, 6912), (64, 11008), (2048, 2560), (2, 20480),
                                 (1, 40000)])
def test_rmsnorm_quant_act_bit_exact(M, K):
    x = synth.activations(M, K, seed=M + K)
    g = _norm_weight(K, K)
    q, gm, rs = bl.rmsnorm_quant_act(to_dev_bf16(x), torch.from_numpy(g).to(DEV), 1e-6)
    xn = oracle.rmsnorm(x, g, 1e-6)
    qo, go, ro = oracle.quant_act_f32(xn)
    np.testing.assert_array_equal(q.cpu().numpy(), qo)
    np.testing.assert_array_equal(gm.cpu().numpy(), go)
    np.testing.assert_array_equal(rs.cpu().numpy(), ro)
    assert bl.last_kernel() == "rmsnorm_quant_act"


# Every launch shape of the quantisation kernel (warps per token row, k-groups
# per lane held in registers): K = 1536 (1 warp, 3 groups), 1544 (2, 2, a
# half-filled last group), 2048 (2, 2), 4096 (4, 2), 16384 (8, 8 in registers),
# 40008 (8, the streaming loop), each in natural order, with RMSNorm, and in
# contraction order through the tensor-core forward with and without the norm.
# (With the norm and at least eight rows per SM, rows of up to 256 groups stay
# in one warp: test_rmsnorm_quant_act_bit_exact and test_forward_norm at
# M = 2048 run that shape.)
@pytest.mark.parametrize("K", [1536, 1544, 2048, 4096, 16384, 40008])
def test_quant_every_launch_shape(K):
    M, N = 3, 40
    x, Wt, a, w = _dense_case(M, K, N, seed=K)
    q, gm, rs = bl.quant_act(to_dev_bf16(x))
    qo, go, ro = oracle.quant_act(x)
    np.testing.assert_array_equal(q.cpu().numpy(), qo)
    np.testing.assert_array_equal(gm.cpu().numpy(), go)
    np.testing.assert_array_equal(rs.cpu().numpy(), ro)
    g = _norm_weight(K, K + 1)
    gd = torch.from_numpy(g).to(DEV)
    q, gm, rs = bl.rmsnorm_quant_act(to_dev_bf16(x), gd, 1e-6)
    qo, go, ro = oracle.quant_act_f32(oracle.rmsnorm(x, g, 1e-6))
    np.testing.assert_array_equal(q.cpu().numpy(), qo)
    np.testing.assert_array_equal(gm.cpu().numpy(), go)
    np.testing.assert_array_equal(rs.cpu().numpy(), ro)
    y, acc = bl.forward(w, to_dev_bf16(x), want_acc=True, flags=bl.FLAG_PATH_TC)
    _check_rows(x, Wt, a, y, acc, np.arange(M))
    y, acc = bl.forward_norm(w, to_dev_bf16(x), gd, 1e-6, want_acc=True)
    yo, acco, *_ = oracle.forward_norm(x, g, 1e-6, Wt, a)
    np.testing.assert_array_equal(acc.cpu().numpy(), acco)
    assert_bf16_close(bf16_bits(y), yo)


@pytest.mark.parametrize("n,m", [(0, 0), (2, 4), (6, 8)])
@pytest.mark.parametrize("M,K,N", [(1, 2560, 640), (16, 1024, 300), (300, 512, 1000), (2048, 2560, 96)])
def test_forward_norm(n, m, M, K, N):
    x = synth.activations(M, K, seed=7 + M)
    W = synth.latent_weights(N, K, seed=7 + N)
    ref = oracle.pack_weights(W, n, m)
    w = bl.pack_weights(torch.from_numpy(W).to(DEV), n, m)
    g = _norm_weight(K, 3)
    y, acc = bl.forward_norm(w, to_dev_bf16(x), torch.from_numpy(g).to(DEV), 1e-5, want_acc=True)
    if M == 1 and m == 0:
        assert bl.last_kernel() == "gemv_m1_dense"  # the decode GEMV on the normalised codes
    yo, acco, *_ = oracle.forward_norm(x, g, 1e-5, ref["Wt"], ref["alpha"])
    np.testing.assert_array_equal(acc.cpu().numpy(), acco)
    assert_bf16_close(bf16_bits(y), yo)
    if M == 1:
        y2, acc2 = bl.forward_norm(w, to_dev_bf16(x), torch.from_numpy(g).to(DEV), 1e-5, want_acc=True,
                                   flags=bl.FLAG_PATH_TC)
        assert torch.equal(acc2, acc) and torch.equal(y2.view(torch.int16), y.view(torch.int16))


def test_status_word_clean():
    torch.cuda.synchronize()
    assert bl.device_status(clear=False) == 0


# ---------------------------------------------------------------- FFN gate/up with squared ReLU

def _check_relu2_glu(x, cases, wg, wu, xd, h, rows):
    """h against the oracle: exactly the oracle's squared-ReLU product of the device's own g and u (each
    the BitLinear output, identical to bitlinear_forward), and exactly the oracle's h wherever the device's
    g and u equal the oracle's (elsewhere they differ by the documented bf16 ulp of the rescale)."""
    (Wg, ag), (Wu, au) = cases
    fwd = lambda w: bl.forward_nm(w, xd) if w.nm_m else bl.forward(w, xd)  # noqa: E731
    yg, yu = bf16_bits(fwd(wg))[rows], bf16_bits(fwd(wu))[rows]
    hb = bf16_bits(h)[rows]
    np.testing.assert_array_equal(hb, oracle.relu2_glu(yg, yu))
    ygo, yuo = oracle.forward(x[rows], Wg, ag)[0], oracle.forward(x[rows], Wu, au)[0]
    assert_bf16_close(yg, ygo)
    assert_bf16_close(yu, yuo)
    same = (yg == ygo) & (yu == yuo)
    np.testing.assert_array_equal(hb[same], oracle.relu2_glu(ygo, yuo)[same])


@pytest.mark.parametrize("M,K,N,flags,kernel", [
    (1, 2560, 6912, 0, "gemv_m1_relu2_glu"), (1, 6912, 2560, 0, "gemv_m1_relu2_glu"),
    (1, 1032, 37, 0, "gemv_m1_relu2_glu"), (1, 200, 333, 0, "gemv_m1_relu2_glu"),
    (1, 2560, 6912, 0x4, "relu2_glu"), (1, 24576, 130, 0, "relu2_glu"),  # K past the one-launch kernel
    (5, 1032, 300, 0, "relu2_glu"), (70, 2560, 640, 0, "relu2_glu"),
    (300, 2048, 2000, 0, "relu2_glu")])
def test_forward_relu2_glu(M, K, N, flags, kernel):
    x, Wg, ag, wg = _dense_case(M, K, N, seed=M + K + N)
    _, Wu, au, wu = _dense_case(M, K, N, seed=M + K + N + 1)
    xd = to_dev_bf16(x)
    h = bl.forward_relu2_glu(wg, wu, xd, flags=flags)
    assert bl.last_kernel() == kernel, bl.last_kernel()
    assert torch.equal(h.view(torch.int16), bl.forward_relu2_glu(wg, wu, xd, flags=flags).view(torch.int16))
    _check_relu2_glu(x, [(Wg, ag), (Wu, au)], wg, wu, xd, h, np.arange(M))


def test_forward_relu2_glu_nm_and_prefill_sampled():
    """6:8 weights at one token (grouped N:M GEMVs, then h), and the 2B4T gate/up at M = 2048 on sampled
    tokens (pair GEMMs, then h)."""
    x, Wg, ag, wg = _nm_case(1, 2048, 1000, 6, 8, seed=21)
    _, Wu, au, wu = _nm_case(1, 2048, 1000, 6, 8, seed=22)
    xd = to_dev_bf16(x)
    h = bl.forward_relu2_glu(wg, wu, xd)
    _check_relu2_glu(x, [(Wg, ag), (Wu, au)], wg, wu, xd, h, np.arange(1))
    M, K, N = 2048, 2560, 6912
    x, Wg, ag, wg = _dense_case(M, K, N, seed=31, ternary=True)
    _, Wu, au, wu = _dense_case(M, K, N, seed=32, ternary=True)
    xd = to_dev_bf16(x)
    h = bl.forward_relu2_glu(wg, wu, xd)
    rows = np.unique(np.concatenate([[0, 127, 128, M - 1], synth.splitmix64(M, 5, 10) % M])).astype(np.int64)
    _check_relu2_glu(x, [(Wg, ag), (Wu, au)], wg, wu, xd, h, rows)
