"""Pins for the H-BitLinear oracle ("BitNet v2" page of brain.hanbit.co.kr, the paragraphs on the
H-BitLinear module and on native 4-bit activations: an online Hadamard transform of the activations,
4-bit activation quantisation, then the ternary linear map).  Closed
forms of the Sylvester Hadamard matrix, its orthogonality, hand-worked codes, the reduction to the
plain 4-bit BitLinear for odd K, and the quantisation error bound against a float64 reference.

CPU only (no GPU marker)."""
import numpy as np
import pytest

import oracle
from ternary_weight_linear_fwd_b200 import synth


def _sylvester(B):
    """H_B[i, j] = (-1)^popcount(i & j), the Sylvester construction written out entrywise."""
    i = np.arange(B)[:, None]
    j = np.arange(B)[None, :]
    bits = np.vectorize(lambda v: bin(int(v)).count("1"))(i & j)
    return np.where(bits % 2 == 0, 1.0, -1.0)


def test_block_size_is_largest_power_of_two_dividing_k():
    for K, B in ((2560, 512), (6912, 256), (2048, 2048), (11008, 256), (200, 8), (203, 1), (96, 32), (1, 1)):
        assert oracle.hadamard_block(K) == B
        assert K % B == 0 and (K // B) % 2 == 1 or K == B


@pytest.mark.parametrize("B", [2, 4, 8, 16, 64, 512])
def test_one_hot_rows_give_hadamard_columns(B):
    """The transform of e_j is column j of H_B / sqrt(B): (-1)^popcount(i & j) * RN32(1 / sqrt(B))."""
    x = synth.to_bf16_bits(np.eye(B, dtype=np.float32))
    xh = oracle.hadamard(x, B)
    s = np.float32(1.0 / np.sqrt(B))
    np.testing.assert_array_equal(xh, (_sylvester(B) * s).astype(np.float32).T)


def test_blocks_are_independent_and_in_place():
    """K = 3 blocks of 8: each block transforms alone (a transposed or misplaced block index fails)."""
    rng = np.random.default_rng(3)
    vals = rng.integers(-9, 10, size=(2, 24)).astype(np.float32)
    xh = oracle.hadamard(synth.to_bf16_bits(vals), 8)
    H = _sylvester(8) / np.sqrt(8)
    ref = np.concatenate([vals[:, 8 * b:8 * b + 8] @ H.T for b in range(3)], axis=1)
    np.testing.assert_allclose(xh, ref, rtol=0, atol=1e-5)


def test_involution_exact_for_power_of_four():
    """H_16 / 4 is orthogonal and symmetric, so applying it twice returns the input; with small integer
    inputs every intermediate is a multiple of 1/4 below 2^7 and the round trip through bf16 is exact."""
    rng = np.random.default_rng(4)
    vals = rng.integers(-8, 9, size=(5, 32)).astype(np.float32)
    x = synth.to_bf16_bits(vals)
    once = oracle.hadamard(x, 16)
    assert np.all(once * 4 == np.round(once * 4))
    twice = oracle.hadamard(synth.to_bf16_bits(once), 16)
    np.testing.assert_array_equal(twice, vals)


def test_parseval():
    x = synth.activations(6, 2560, seed=51)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    xh = oracle.hadamard(x).astype(np.float64)
    np.testing.assert_allclose((xh ** 2).sum(axis=1), (xf ** 2).sum(axis=1), rtol=1e-5)


def test_hand_worked_codes_and_output():
    """B = 4: x = (1,1,1,1) -> (2,0,0,0); (1,-1,1,-1) -> (0,2,0,0); (3,1,0,0) -> H x / 2 = (2,1,2,1).
    gamma = 2, codes rne(7 v / 2.00001): 2 -> 7, 1 -> 3.49998 -> 3.  With W_t = (1, 0, -1, 1) and
    alpha = 0.5: acc = 7, 0, 7 - 7 + 3 = 3, and y = 3 * 0.5 * 2 / 7 = 0.428571... -> bf16 0x3EDB."""
    x = synth.to_bf16_bits(np.array([[1, 1, 1, 1], [1, -1, 1, -1], [3, 1, 0, 0]], np.float32))
    xh = oracle.hadamard(x)
    np.testing.assert_array_equal(xh, [[2, 0, 0, 0], [0, 2, 0, 0], [2, 1, 2, 1]])
    q, g, rs = oracle.quant_act4(xh)
    np.testing.assert_array_equal(q, [[7, 0, 0, 0], [0, 7, 0, 0], [7, 3, 7, 3]])
    np.testing.assert_array_equal(g, [2, 2, 2])
    np.testing.assert_array_equal(rs, [7, 7, 20])
    y, acc, q2, g2 = oracle.forward_hbit(x, np.array([[1, 0, -1, 1]], np.int8), np.float32(0.5))
    np.testing.assert_array_equal(acc[:, 0], [7, 0, 3])
    assert int(y[2, 0]) == 0x3EDB and int(y[1, 0]) == 0


def test_four_bit_codes_range_and_argmax():
    x = synth.activations(8, 512, seed=52)
    q, g, _ = oracle.quant_act4(oracle.hadamard(x))
    assert q.min() >= -7 and q.max() <= 7  # |v| <= gamma keeps the -8 end unreachable, as -128 is at 8 bits
    xh = oracle.hadamard(x)
    am = np.abs(xh).argmax(axis=1)
    assert np.all(np.abs(q[np.arange(8), am]) == 7)


def test_odd_k_reduces_to_plain_four_bit_bitlinear():
    """For odd K the block is 1 (the identity, scale 1), so H-BitLinear is BitLinear with Q_b = 7: the
    codes equal the bf16-input quantiser's at Q_b = 7 and the outputs its forward's."""
    x = synth.activations(4, 203, seed=53)
    W = synth.latent_weights(40, 203, seed=53)
    p = oracle.pack_weights(W)
    y, acc, q, g = oracle.forward_hbit(x, p["Wt"], p["alpha"])
    q7, g7, _ = oracle.quant_act(x, 7)
    np.testing.assert_array_equal(q, q7)
    np.testing.assert_array_equal(g, g7)
    y7, acc7, *_ = oracle.forward(x, p["Wt"], p["alpha"], 7)
    np.testing.assert_array_equal(acc, acc7)
    np.testing.assert_array_equal(y, y7)


def test_within_four_bit_quantisation_error_bound():
    """|y - (H x) . (alpha W_t)| <= alpha / 7 * (|acc| (d - gamma) + d * 0.50001 * sum |W_t|) + |y| 2^-8
    (+ the fp32 rounding of the transform), d = RN(gamma + eps): each code is within half a step of
    7 xh / d; the float reference uses a float64 Hadamard product written entrywise."""
    M, K, N = 4, 512, 64
    x = synth.activations(M, K, seed=54)
    W = synth.latent_weights(N, K, seed=54)
    p = oracle.pack_weights(W)
    y, acc, q, g = oracle.forward_hbit(x, p["Wt"], p["alpha"])
    B = oracle.hadamard_block(K)
    H = _sylvester(B) / np.sqrt(B)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    xr = np.concatenate([xf[:, b:b + B] @ H.T for b in range(0, K, B)], axis=1)
    a = float(p["alpha"])
    ref = xr @ (a * p["Wt"].astype(np.float64)).T
    yf = synth.bf16_bits_to_f32(y).astype(np.float64)
    d = (g.astype(np.float32) + np.float32(1e-5)).astype(np.float64)
    l1 = np.abs(p["Wt"]).sum(axis=1).astype(np.float64)
    bound = a / 7 * (np.abs(acc) * (d - g)[:, None] + d[:, None] * 0.50001 * l1[None, :]) \
        + np.abs(yf) * 2.0 ** -8 + 1e-5 * a * l1[None, :] * np.abs(xr).max()
    assert np.all(np.abs(yf - ref) <= bound)
