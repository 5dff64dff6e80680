"""Pins for the oracle: hand-worked examples from the pages, closed forms,
invariants, brute force and special cases.  None of these re-types the
oracle's own formula; each would fail on a dropped term, a wrong sign, a
wrong index or a transposed operand somewhere in the oracle.

CPU only (no GPU marker)."""
import math

import numpy as np
import pytest

import oracle
from ternary_weight_linear_fwd_b200 import synth


def _ints(tok):
    return np.array([int(t) for t in tok], dtype=np.int64)


def _floats(tok):
    return np.array([float(t) for t in tok], dtype=np.float32)


# ---------------------------------------------------------------- worked examples

def test_tl2_worked_example_acc(golden):
    g = golden("tl2_worked_example.txt")
    w = _ints(g["weights"][0]).astype(np.int8)
    q = _ints(g["q"][0]).astype(np.int8)
    acc = oracle.matmul_i32(q[None, :], w[None, :])
    assert int(acc[0, 0]) == int(g["acc"][0][0])


def test_tl2_lookup_identity(golden):
    """The 9-entry pair table of the TL2 scheme gives the same dot product as
    the direct sum, for every pair code and for the page's weight vector."""
    g = golden("tl2_worked_example.txt")
    w = _ints(g["weights"][0])
    idx = [(w[i] + 1) * 3 + (w[i + 1] + 1) for i in range(0, 8, 2)]
    assert idx == [int(t) for t in g["tl2_pair_index"][0]]
    rng = np.random.default_rng(0)
    for _ in range(50):
        a = rng.integers(-127, 128, size=8)
        lut_sum = 0
        for i in range(0, 8, 2):
            a0, a1 = a[i], a[i + 1]
            lut = [-(a0 + a1), -a0, -a0 + a1, -a1, 0, a1, a0 - a1, a0, a0 + a1]
            lut_sum += lut[idx[i // 2]]
        acc = oracle.matmul_i32(a.astype(np.int8)[None, :], w.astype(np.int8)[None, :])
        assert int(acc[0, 0]) == int(lut_sum)


def test_i2s_packed_bytes(golden):
    g = golden("tl2_worked_example.txt")
    w = _ints(g["weights"][0]).astype(np.int8)[None, :]
    expect = np.array([int(t, 16) for t in g["packed_row_hex"][0]], dtype=np.uint8)
    got = oracle.pack_dense(w)
    assert got.shape == (1, 16)
    np.testing.assert_array_equal(got[0], expect)
    np.testing.assert_array_equal(oracle.unpack_dense(got, 1, 8), w)


def test_quant_act_hand(golden):
    g = golden("quant_act_hand.txt")
    x = synth.to_bf16_bits(_floats(g["x"][0]))[None, :]
    for key, qb in (("q_qb127", 127), ("q_qb128", 128)):
        q, gam, rs = oracle.quant_act(x, qb)
        np.testing.assert_array_equal(q[0], _ints(g[key][0]))
        assert float(gam[0]) == float(g["gamma"][0][0])
        assert int(rs[0]) == int(_ints(g[key][0]).sum())


def test_dequant_hand(golden):
    for acc, alpha, gamma, hexbits in golden("dequant_hand.txt")["case"]:
        y = oracle.dequant(np.array([[int(acc)]], np.int32), np.array([float(gamma)], np.float32),
                           np.float32(float(alpha)))
        assert int(y[0, 0]) == int(hexbits, 16), (acc, alpha, gamma)


def test_ternarize_hand(golden):
    g = golden("ternarize_hand.txt")
    W = _floats(g["W"][0])[None, :]
    a = oracle.absmean(W)
    assert a == np.float32(float(g["alpha"][0][0]))
    np.testing.assert_array_equal(oracle.ternarize(W, a)[0], _ints(g["Wt"][0]))


def test_nm_mask_hand(golden):
    g = golden("nm_mask_hand.txt")
    cases = (("w24", "keep24", "meta24", 2, 4), ("w68", "keep68", "meta68", 6, 8),
             ("w68tie", "keep68tie", "meta68tie", 6, 8))
    for wk, kk, mk, n, m in cases:
        W = _floats(g[wk][0])[None, :]
        mask = oracle.nm_mask(W, n, m)
        np.testing.assert_array_equal(mask[0], _ints(g[kk][0]))
        Wt = oracle.ternarize(W, oracle.absmean(W))
        _, meta = oracle.pack_nm(oracle.apply_mask(Wt, mask), mask, n, m)
        assert int(meta[0, 0]) == int(g[mk][0][0])


# ---------------------------------------------------------------- special cases

def test_ternarize_ties_round_half_to_even():
    """r = W / RN(alpha + eps) exactly +-0.5 rounds to 0 and +-1.5 to +-2 -> clamp +-1;
    the next float above 0.5 gives +-1.  d is formed by an independent fp32 add."""
    alpha = np.float32(0.75) - np.float32(1e-5)
    d = np.float32(alpha + np.float32(1e-5))
    half = np.float32(d * np.float32(0.5))  # exact: scaling by a power of two
    assert np.float32(half / d) == np.float32(0.5)
    above = np.nextafter(half, np.float32(1))
    W = np.array([[half, -half, np.float32(3) * half, -np.float32(3) * half, above, -above, 0.0, -0.0]],
                 dtype=np.float32)
    got = oracle.ternarize(W, alpha)[0]
    np.testing.assert_array_equal(got, [0, 0, 1, -1, 1, -1, 0, 0])


def test_bf16_rounding_matches_independent_fp32_path():
    """For values exactly representable in fp32, rounding from fp64 to bf16 must
    agree with numpy's fp32 -> bf16 bit rounding (an independent implementation)."""
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.standard_normal(2000) * 10 ** rng.uniform(-30, 30, 2000),
                        [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 2 ** -130, 2 ** -133 * 1.5]])
    v32 = v.astype(np.float32)
    ref = synth.to_bf16_bits(v32)
    got = np.array([oracle.bf16_from_f64(float(x)) for x in v32], dtype=np.uint16)
    np.testing.assert_array_equal(got, ref)


def test_zero_input_gives_zero():
    x = np.zeros((3, 64), np.uint16)
    W = synth.latent_weights(16, 64, seed=7)
    p = oracle.pack_weights(W)
    y, acc, q, g, rs = oracle.forward(x, p["Wt"], p["alpha"])
    assert not q.any() and not acc.any() and not g.any() and not rs.any()
    assert not y.any()


def test_argmax_maps_to_127():
    x = synth.activations(16, 512, seed=3)
    q, g, _ = oracle.quant_act(x)
    xf = synth.bf16_bits_to_f32(x)
    am = np.abs(xf).argmax(axis=1)
    assert np.all(np.abs(q[np.arange(16), am]) == 127)
    assert np.all(np.abs(q.astype(np.int32)) <= 127)
    assert np.all(g == np.abs(xf).max(axis=1))


def test_hand_2x8_closed_form():
    """x = +-c with c >> eps gives q = +-127 exactly (127c/(c+1e-5) > 126.5 for
    c > 2.54e-3), so acc is 127 times a signed count and y = acc * alpha * c / 127."""
    c = 0.75
    signs = np.array([[1, -1, 1, 1, -1, -1, 1, -1], [-1, -1, -1, 1, 1, 1, 1, 1]])
    x = synth.to_bf16_bits((signs * c).astype(np.float32))
    Wt = np.array([[1, 0, -1, 1, 0, 0, -1, 1], [0, 0, 0, 0, 0, 0, 0, 0], [1, 1, 1, 1, 1, 1, 1, 1]],
                  dtype=np.int8)
    alpha = np.float32(0.5)
    y, acc, q, g, _ = oracle.forward(x, Wt, alpha)
    np.testing.assert_array_equal(q, 127 * signs)
    expect_acc = 127 * (signs @ Wt.T.astype(np.int64))
    np.testing.assert_array_equal(acc, expect_acc)
    for i in range(2):
        for j in range(3):
            assert y[i, j] == oracle.bf16_from_f64(expect_acc[i, j] * 0.5 * c / 127)


def test_qb128_reading_clamps():
    x = synth.activations(4, 256, seed=11)
    q, _, _ = oracle.quant_act(x, 128)
    assert q.min() >= -128 and q.max() <= 127
    assert (np.abs(q.astype(np.int32)) >= 127).sum() >= 4


# ---------------------------------------------------------------- closed forms

def test_absmean_constant_magnitude_exact():
    W = (np.where(synth.uniform(5, 9, 4096) < 0.5, -1.0, 1.0) * 0.037).astype(np.float32).reshape(64, 64)
    assert oracle.absmean(W) == np.float32(0.037)


def test_absmean_and_zero_fraction_closed_form():
    """For W ~ N(0, s): alpha -> s*sqrt(2/pi) and P(W_t = 0) -> 2*Phi(0.5*sqrt(2/pi)) - 1 = 0.3101."""
    N, K, s = 512, 256, 0.02
    W = synth.latent_weights(N, K, seed=0)
    a = float(oracle.absmean(W))
    mu = s * math.sqrt(2 / math.pi)
    se = s * math.sqrt(1 - 2 / math.pi) / math.sqrt(N * K)
    assert abs(a - mu) < 5 * se
    Wt = oracle.ternarize(W, a)
    p0 = (Wt == 0).mean()
    z = 0.5 * (a + 1e-5) / s
    expect = math.erf(z / math.sqrt(2))  # = 2*Phi(z) - 1
    assert abs(expect - 0.3101) < 0.002
    assert abs(p0 - expect) < 4 * math.sqrt(expect * (1 - expect) / (N * K))
    assert set(np.unique(Wt).tolist()) <= {-1, 0, 1}


def test_pack_recovers_scaled_ternary():
    """W = c * T (T drawn with P(0) = 0.42) has alpha = c * (1 - p0_emp); every nonzero
    scales to +-1/(1 - p0) > 1.5 and therefore ternarises back to T exactly."""
    T = synth.ternary_weights(96, 512, seed=1)
    c = np.float32(0.03125)
    W = (T.astype(np.float32) * c)
    p = oracle.pack_weights(W)
    np.testing.assert_array_equal(p["Wt"], T)
    frac_nz = (T != 0).mean()
    assert abs(float(p["alpha"]) - float(c) * frac_nz) < 1e-7
    assert abs((T == 0).mean() - 0.42) < 4 * math.sqrt(0.42 * 0.58 / T.size)


# ---------------------------------------------------------------- invariants

@pytest.mark.parametrize("N,K", [(512, 256), (33, 200), (7, 3)])
def test_dense_pack_roundtrip_and_codes(N, K):
    W = synth.latent_weights(N, K, seed=N + K)
    p = oracle.pack_weights(W)
    codes = p["codes"]
    assert codes.shape == (N, 16 * ((K + 63) // 64))
    np.testing.assert_array_equal(oracle.unpack_dense(codes, N, K), p["Wt"])
    c = np.stack([(codes >> s) & 3 for s in (0, 2, 4, 6)], axis=-1).reshape(N, -1)
    assert not (c == 3).any()
    assert np.all(c[:, K:] == 1)  # padding positions hold the zero code
    np.testing.assert_array_equal(c[:, :K].astype(np.int8) - 1, p["Wt"])


@pytest.mark.parametrize("n,m", [(2, 4), (6, 8), (7, 8), (5, 8), (3, 8), (2, 8), (1, 8)])
def test_nm_mask_is_topn_and_roundtrips(n, m):
    N, K = 40, 256
    W = synth.latent_weights(N, K, seed=5)
    W[3, :16] = 0.01  # tie-heavy blocks
    W[4, :8] = -0.0
    mask = oracle.nm_mask(W, n, m)
    blocks = mask.reshape(N, K // m, m)
    assert np.all(blocks.sum(-1) == n)
    # brute force: a stable library sort of -|W| inside each block
    mag = np.abs(W.reshape(N, K // m, m)).astype(np.float64)
    order = np.argsort(-mag, axis=-1, kind="stable")
    ref = np.zeros_like(blocks)
    np.put_along_axis(ref, order[..., :n], 1, axis=-1)
    np.testing.assert_array_equal(blocks, ref)
    p = oracle.pack_weights(W, n, m)
    assert p["alpha"] == oracle.absmean(W)  # alpha from the dense latent matrix
    dense_t = oracle.ternarize(W, oracle.absmean(W))
    np.testing.assert_array_equal(p["Wt"], dense_t * mask)  # quant, then mask
    back = oracle.unpack_nm(p["values"], p["meta"], N, K, n, m)
    np.testing.assert_array_equal(back, p["Wt"])
    assert p["values"].shape[1] == 16 * ((K * n // m + 63) // 64)


def test_nm_rejects_bad_pattern():
    W = synth.latent_weights(4, 64, seed=1)
    with pytest.raises(ValueError):
        oracle.pack_nm(np.zeros((4, 64), np.int8), np.ones((4, 64), np.uint8), 3, 4)


# ---------------------------------------------------------------- brute force

def test_matmul_matches_float64_library_matmul():
    x = synth.activations(8, 256, seed=0)
    W = synth.latent_weights(512, 256, seed=0)
    p = oracle.pack_weights(W)
    q, _, _ = oracle.quant_act(x)
    acc = oracle.matmul_i32(q, p["Wt"])
    ref = q.astype(np.float64) @ p["Wt"].astype(np.float64).T
    np.testing.assert_array_equal(acc, ref.astype(np.int64))


def test_forward_within_quantisation_error_bound():
    """|y - x . (alpha W_t)| <= alpha/127 * (|acc| (d - gamma) + d * 0.50001 * sum|W_t|) + |y| 2^-8,
    d = RN(gamma + eps): the codes are within half a step of 127 x / d, and y is rounded to bf16."""
    M, K, N = 8, 256, 512
    x = synth.activations(M, K, seed=0)
    W = synth.latent_weights(N, K, seed=0)
    p = oracle.pack_weights(W)
    y, acc, q, g, _ = oracle.forward(x, p["Wt"], p["alpha"])
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    a = float(p["alpha"])
    ref = xf @ (a * p["Wt"].astype(np.float64)).T
    yf = synth.bf16_bits_to_f32(y).astype(np.float64)
    d = (g.astype(np.float32) + np.float32(1e-5)).astype(np.float64)
    l1 = np.abs(p["Wt"]).sum(axis=1).astype(np.float64)
    bound = a / 127 * (np.abs(acc) * (d - g)[:, None] + d[:, None] * 0.50001 * l1[None, :]) \
        + np.abs(yf) * 2.0 ** -8 + 1e-12
    assert np.all(np.abs(yf - ref) <= bound)
    # the bound sits below the signal, and the typical error is far smaller still
    assert np.median(bound) < np.median(np.abs(ref))
    assert np.sqrt(np.mean((yf - ref) ** 2)) < 0.05 * np.sqrt(np.mean(ref ** 2))


def test_third_restatement_torch_cpu():
    """The blog's PyTorch BitLinear_b158 formulas (Qb = 127) in torch CPU fp32."""
    torch = pytest.importorskip("torch")
    M, K, N = 8, 256, 512
    x = synth.activations(M, K, seed=0)
    W = synth.latent_weights(N, K, seed=0)
    p = oracle.pack_weights(W)
    wt = torch.from_numpy(W)
    wq = torch.clamp(torch.round(wt / (torch.tensor(float(p["alpha"]), dtype=torch.float32) + 1e-5)), -1, 1)
    np.testing.assert_array_equal(wq.numpy().astype(np.int8), p["Wt"])
    xt = torch.from_numpy(synth.bf16_bits_to_f32(x).copy())
    gam = xt.abs().max(dim=-1, keepdim=True).values
    xq = torch.clamp(torch.round(xt * 127 / (gam + 1e-5)), -128, 127)
    q, g, _ = oracle.quant_act(x)
    np.testing.assert_array_equal(xq.numpy().astype(np.int8), q)
    out = torch.nn.functional.linear(xq.double(), wq.double()) * (float(p["alpha"]) * gam.double()) / 127
    ref = out.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    y, *_ = oracle.forward(x, p["Wt"], p["alpha"])
    diff = np.abs(y.astype(np.int32) - ref.astype(np.int32))
    assert diff.max() <= 1


# ---------------------------------------------------------------- RMSNorm before the activation quantisation
# [b158] BitLinear_b158.forward normalises x with nn.RMSNorm (per-feature weight g) before activation_quant.

def _bf16(vals):
    return synth.to_bf16_bits(np.asarray(vals, np.float32))


def test_rmsnorm_hand_worked():
    """x = (3, 4): ms = 12.5, xn = (3, 4) / sqrt(12.5); gamma = 4 r; codes 127 * (3/4) = 95.25 -> 95 and 127.
    With g = (2, 0.5): xn = (6 r, 2 r), codes 127 and 127/3 = 42.33 -> 42."""
    x = _bf16([[3.0, 4.0]])
    r = np.float32(1.0 / np.sqrt(12.5))
    xn = oracle.rmsnorm(x, np.array([1.0, 1.0], np.float32), 0.0)
    assert xn[0, 0] == np.float32(np.float32(3.0) * r) and xn[0, 1] == np.float32(np.float32(4.0) * r)
    q, g, rs = oracle.quant_act_f32(xn)
    assert list(q[0]) == [95, 127] and rs[0] == 222 and g[0] == xn[0, 1]
    xn2 = oracle.rmsnorm(x, np.array([2.0, 0.5], np.float32), 0.0)
    q2, g2, _ = oracle.quant_act_f32(xn2)
    assert list(q2[0]) == [127, 42] and g2[0] == xn2[0, 0]


def test_rmsnorm_unit_mean_square():
    """g = 1, eps = 0: mean(xn^2) = 1 up to fp32 rounding, for any row."""
    x = synth.activations(6, 1000, seed=21)
    xn = oracle.rmsnorm(x, np.ones(1000, np.float32), 0.0).astype(np.float64)
    np.testing.assert_allclose((xn ** 2).mean(axis=1), 1.0, rtol=1e-6)


def test_rmsnorm_scale_invariance():
    """eps = 0: scaling x by a power of two leaves xn unchanged bit for bit; doubling g doubles xn and leaves
    the codes and code sums unchanged."""
    x = synth.activations(4, 300, seed=22)
    xf = synth.bf16_bits_to_f32(x)
    x4 = synth.to_bf16_bits(xf * np.float32(4.0))
    g = (1.0 + 0.25 * synth.uniform(22, 9, 300)).astype(np.float32)
    a = oracle.rmsnorm(x, g, 0.0)
    np.testing.assert_array_equal(oracle.rmsnorm(x4, g, 0.0), a)
    b = oracle.rmsnorm(x, g * np.float32(2.0), 0.0)
    np.testing.assert_array_equal(b, a * np.float32(2.0))
    qa, ga, ra = oracle.quant_act_f32(a)
    qb, gb, rb = oracle.quant_act_f32(b)
    np.testing.assert_array_equal(qa, qb)
    np.testing.assert_array_equal(ra, rb)
    np.testing.assert_array_equal(gb, ga * np.float32(2.0))


def test_rmsnorm_constant_and_zero_rows():
    """A constant row of a power of two normalises to +-1 exactly with eps = 0 (codes +-127, gamma 1); with
    eps > 0 a zero row gives zeros (with eps = 0 it is 0 / 0, left undefined)."""
    x = _bf16([[0.5] * 8, [-2.0] * 8])
    xn = oracle.rmsnorm(x, np.ones(8, np.float32), 0.0)
    assert (xn[0] == 1.0).all() and (xn[1] == -1.0).all()
    q, g, rs = oracle.quant_act_f32(xn)
    assert (q[0] == 127).all() and (q[1] == -127).all()
    assert list(g) == [1.0, 1.0] and list(rs) == [1016, -1016]
    xe = oracle.rmsnorm(_bf16([[0.0] * 8]), np.ones(8, np.float32), 1e-6)
    assert not xe.any()
    qe, ge, re_ = oracle.quant_act_f32(xe)
    assert not qe.any() and ge[0] == 0.0 and re_[0] == 0


def test_rmsnorm_eps_lowers_scale():
    """eps > 0 can only shrink xn: |xn(eps)| <= |xn(0)| elementwise."""
    x = synth.activations(3, 64, seed=23)
    g = np.ones(64, np.float32)
    assert (np.abs(oracle.rmsnorm(x, g, 1e-2)) <= np.abs(oracle.rmsnorm(x, g, 0.0))).all()


def test_quant_act_f32_matches_bf16_path_on_bf16_values():
    """On rows whose values are bf16 numbers, the fp32-input quantisation is the bf16 one."""
    x = synth.activations(5, 200, seed=24)
    q1, g1, r1 = oracle.quant_act(x)
    q2, g2, r2 = oracle.quant_act_f32(synth.bf16_bits_to_f32(x))
    np.testing.assert_array_equal(q1, q2)
    np.testing.assert_array_equal(g1, g2)
    np.testing.assert_array_equal(r1, r2)


# ---------------------------------------------------------------- N:M packed bytes, worked by hand

def test_nm_packed_bytes_hand():
    """Sparse-BitNet review, section 3.2 (top-n |W| per block of m along k, quant then mask), with the
    I2_S 2-bit codes of the 2B4T report (section 5.1) and the layout: kept codes in increasing k,
    LSB first, tail code 01; 2:4 meta a nibble i0 | i1 << 2 per block, low nibble first; n:8 meta
    one bitmask byte per block.

    2:4, W = (0.9, 0.1, 0.05, -0.8 | 0.02, 0.7, -0.6, 0.01): alpha = 3.18 / 8 = 0.3975, W / alpha
    rounds to (1, 0, 0, -1 | 0, 1, -1, 0) (-0.6 / 0.3975 = -1.51 -> -2 -> -1).  Kept k = 0, 3 | 5, 6:
    meta = 12 | 9 << 4 = 0x9C; codes (2, 0, 2, 0) -> 0x22.
    3:8, W = (0.1, -0.5, 0.05, 0.3, -0.35, 0.2, 0.01, 0.45): alpha = 1.96 / 8 = 0.245, W_t =
    (0, -1, 0, 1, -1, 1, 0, 1); kept k = 1, 4, 7 (|W| 0.5, 0.35, 0.45): meta 0b10010010 = 0x92;
    codes (0, 0, 2) and one tail code 01 -> 0x60; the masked matrix drops W_t = 1 at k = 3 and 5."""
    cases = (
        ([0.9, 0.1, 0.05, -0.8, 0.02, 0.7, -0.6, 0.01], 2, 4, 0.3975, [1, 0, 0, -1, 0, 1, -1, 0], 0x22, 0x9C,
         [1, 0, 0, -1, 0, 1, -1, 0]),
        ([0.1, -0.5, 0.05, 0.3, -0.35, 0.2, 0.01, 0.45], 3, 8, 0.245, [0, -1, 0, 1, -1, 1, 0, 1], 0x60, 0x92,
         [0, -1, 0, 0, -1, 0, 0, 1]),
    )
    for w, n, m, alpha, wt, vbyte, mbyte, weff in cases:
        W = np.array([w], np.float32)
        p = oracle.pack_weights(W, n, m)
        assert p["alpha"] == np.float32(alpha)
        np.testing.assert_array_equal(oracle.ternarize(W, p["alpha"])[0], wt)
        np.testing.assert_array_equal(p["Wt"][0], weff)
        assert p["values"].shape == (1, 16) and p["meta"].shape == (1, 16)
        assert int(p["values"][0, 0]) == vbyte and int(p["meta"][0, 0]) == mbyte
        assert (p["values"][0, 1:] == 0x55).all()  # tail codes 01


# ---------------------------------------------------------------- RMSNorm composed with the forward

def test_forward_norm_reduces_to_forward_on_unit_rows():
    """Rows of +-1 have mean square 1, so with g = 1 and eps = 0 the normalised row is the row itself
    and forward_norm equals forward bit for bit; with g = 2 every xn doubles, the codes stay and gamma
    doubles, so y doubles exactly (a rescale that used gamma of x instead of xn would not)."""
    M, K, N = 4, 128, 96
    signs = np.where(synth.uniform(31, 3, M * K) < 0.5, -1.0, 1.0).reshape(M, K).astype(np.float32)
    x = synth.to_bf16_bits(signs)
    W = synth.latent_weights(N, K, seed=31)
    p = oracle.pack_weights(W)
    y0, acc0, *_ = oracle.forward(x, p["Wt"], p["alpha"])
    y1, acc1, *_ = oracle.forward_norm(x, np.ones(K, np.float32), 0.0, p["Wt"], p["alpha"])
    np.testing.assert_array_equal(acc1, acc0)
    np.testing.assert_array_equal(y1, y0)
    y2, acc2, *_ = oracle.forward_norm(x, np.full(K, 2.0, np.float32), 0.0, p["Wt"], p["alpha"])
    np.testing.assert_array_equal(acc2, acc0)
    np.testing.assert_array_equal(synth.bf16_bits_to_f32(y2), 2.0 * synth.bf16_bits_to_f32(y0))
    assert np.abs(acc0).max() > 0


def test_threaded_contraction_equals_plain_loop():
    """The benchmark's all-cores leg splits the output columns over threads; every element is the same
    loop, so the accumulators must equal the single-threaded ones (and the float64 library matmul)."""
    T = synth.ternary_weights(301, 777, seed=12)
    x = synth.activations(5, 777, seed=13)
    q, _, _ = oracle.quant_act(x)
    a1 = oracle.matmul_i32(q, T)
    for th in (2, 3, 8, 400):
        np.testing.assert_array_equal(oracle.matmul_i32_threads(q, T, th), a1)
    np.testing.assert_array_equal(a1, (q.astype(np.float64) @ T.astype(np.float64).T).astype(np.int64))


# ---------------------------------------------------------------- squared-ReLU gate/up (FFN of the 2B4T model)

def _f32_of_bf16(bits):
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32)


def test_relu2_glu_nonpositive_gate_is_signed_zero():
    """ReLU of a non-positive gate is 0, so h is a zero carrying the sign of u (IEEE 0 * u)."""
    g = _bf16([-2.5, -0.0, 0.0, -1e-3, -300.0])
    u = _bf16([3.0, 1.5, -7.0, -2.0, 0.25])
    h = oracle.relu2_glu(g, u)
    assert [int(v) for v in h] == [0x0000, 0x0000, 0x8000, 0x8000, 0x0000]


def test_relu2_glu_powers_of_two_exact():
    """g = 2^a > 0, u = +-2^b: h = +-2^(2a + b) exactly (no rounding anywhere)."""
    rng = np.random.default_rng(3)
    a = rng.integers(-20, 20, 64)
    b = rng.integers(-20, 20, 64)
    s = rng.choice([-1.0, 1.0], 64)
    g = _bf16([2.0 ** int(v) for v in a])
    u = _bf16([float(sv) * 2.0 ** int(v) for sv, v in zip(s, b)])
    h = _f32_of_bf16(oracle.relu2_glu(g, u))
    assert np.array_equal(h, (s * 2.0 ** (2 * a + b)).astype(np.float32))


def test_relu2_glu_hand_rounding():
    """Worked by hand.  g = 1 + 2^-7 squares to 1 + 2^-6 + 2^-14, which bf16 (8 significant bits,
    spacing 2^-7 on [1, 2)) rounds to 1 + 2^-6 = 1.015625.  Times u = 3: 3.046875 = 1.5234375 * 2,
    exact in bf16 (0x4043).  Times u = 1.25: 1.26953125, exactly half-way between 1.265625 and
    1.2734375, so ties-to-even gives 1.265625 (0x3FA2) -- whereas rounding g^2 u only once
    (1.26960754...) would give 1.2734375 (0x3FA3): the squared gate is rounded first.
    g = 1.5, u = 2: 2.25 * 2 = 4.5 (0x4090)."""
    g = _bf16([1.0 + 2.0 ** -7, 1.0 + 2.0 ** -7, 1.5])
    u = _bf16([3.0, 1.25, 2.0])
    assert [int(v) for v in oracle.relu2_glu(g, u)] == [0x4043, 0x3FA2, 0x4090]


def test_relu2_glu_odd_in_u_and_within_two_roundings():
    """h(g, -u) = -h(g, u); and |h - max(g, 0)^2 u| <= (2^-8 + 2^-8 + 2^-16) |max(g, 0)^2 u| for
    normal results (two roundings to 8 significant bits)."""
    rng = np.random.default_rng(11)
    gv = rng.normal(0, 3, 4096)
    uv = rng.normal(0, 3, 4096)
    g, u = _bf16(gv), _bf16(uv)
    h = oracle.relu2_glu(g, u)
    hn = oracle.relu2_glu(g, _bf16(-_f32_of_bf16(u).astype(np.float64)))
    assert np.array_equal(_f32_of_bf16(hn), -_f32_of_bf16(h))
    ex = np.maximum(_f32_of_bf16(g).astype(np.float64), 0.0) ** 2 * _f32_of_bf16(u).astype(np.float64)
    hv = _f32_of_bf16(h).astype(np.float64)
    big = np.abs(ex) > 1e-30
    assert np.all(np.abs(hv[big] - ex[big]) <= (2.0 ** -7 + 2.0 ** -16) * np.abs(ex[big]))
    assert np.all(hv[~big] == 0.0)
