"""H-BitLinear on the GPU against the oracle ("BitNet v2" page of brain.hanbit.co.kr: an online
Hadamard transform of the activations, 4-bit quantisation, then the ternary linear map; the transform
size, normalisation and order, and the 4-bit quantiser, are the readings stated in include/bitlinear.h).

The transformed codes, gamma and the code sums must match bit for bit (every butterfly is one IEEE add
or subtract in the oracle's stage order, the code decision one IEEE multiply and divide); accumulators
bit for bit; bf16 outputs within one ulp (the rescale RN(RN(alpha gamma) / 7) and one multiply against
the oracle's single fp64 rounding).  Shapes: the 2B4T widths (2560 -> B = 512, 6912 -> B = 256), the
Qwen2.5 MLP width 2048 (B = 2048), an odd K (B = 1: no transform), a K with B = 8, and the largest K
the kernel takes."""
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


@pytest.fixture(scope="module", autouse=True)
def _built():
    from ternary_weight_linear_fwd_b200 import build as b
    b.build()
    oracle.build()
    yield
    torch.cuda.synchronize()
    assert bl.device_status() == 0


def _dev(x_bits):
    return torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).to(DEV).view(torch.bfloat16)


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("M,K", [(1, 2560), (3, 6912), (5, 203), (64, 2048), (2048, 2560), (2, 16384), (4, 1000)])
def test_hadamard_quant_act4_bit_exact(M, K):
    x = synth.activations(M, K, seed=M * 3 + K)
    q, g, rs = bl.hadamard_quant_act4(_dev(x))
    assert bl.last_kernel() == "hadamard_quant_act4"
    qo, go, ro = oracle.quant_act4(oracle.hadamard(x))
    np.testing.assert_array_equal(q.cpu().numpy(), qo)
    np.testing.assert_array_equal(g.cpu().numpy(), go)
    np.testing.assert_array_equal(rs.cpu().numpy(), ro)
    assert qo.min() >= -8 and qo.max() <= 7


def _check(x, Wt, alpha, y, acc, rows):
    yo, acco, _, _ = oracle.forward_hbit(x[rows], Wt, alpha)
    np.testing.assert_array_equal(acc.cpu().numpy()[rows], acco)
    d = np.abs(_bits(y)[rows].astype(np.int32) - yo.astype(np.int32))
    assert d.max() <= 1, f"max bf16 ulp distance {d.max()}"
    assert (d > 0).mean() < 0.01


@pytest.mark.parametrize("M,K,N", [(1, 2560, 6912), (1, 6912, 2560), (7, 203, 130), (300, 2560, 640),
                                   (16, 2048, 1000), (33, 1000, 96)])
def test_forward_hbit(M, K, N):
    x = synth.activations(M, K, seed=M + N)
    W = synth.latent_weights(N, K, seed=K + N)
    ref = oracle.pack_weights(W)
    w = bl.pack_weights(torch.from_numpy(W).to(DEV))
    y, acc = bl.forward_hbit(w, _dev(x), want_acc=True)
    assert bl.last_kernel().startswith("tc_gemm_dense")
    _check(x, ref["Wt"], ref["alpha"], y, acc, np.arange(M))


@pytest.mark.parametrize("n,m", [(2, 4), (6, 8)])
def test_forward_hbit_nm(n, m):
    M, K, N = 9, 1032, 140
    x = synth.activations(M, K, seed=n * m)
    W = synth.latent_weights(N, K, seed=n + m)
    ref = oracle.pack_weights(W, n, m)
    w = bl.pack_weights(torch.from_numpy(W).to(DEV), n, m)
    y, acc = bl.forward_hbit(w, _dev(x), want_acc=True)
    _check(x, ref["Wt"], ref["alpha"], y, acc, np.arange(M))


@pytest.mark.parametrize("K,N", [(2560, 6912), (6912, 2560)])
def test_forward_hbit_prefill_sampled(K, N):
    """The 2B4T FFN shapes at M = 2048 tokens; 16 sampled tokens checked on every output."""
    M = 2048
    x = synth.activations(M, K, seed=11)
    T = synth.ternary_weights(N, K, seed=12)
    a = np.float32(synth.alpha_uniform(12))
    w = bl.pack_ternary(torch.from_numpy(T).to(DEV), float(a))
    y, acc = bl.forward_hbit(w, _dev(x), want_acc=True)
    rows = np.unique(np.concatenate([[0, M - 1], synth.splitmix64(11, 3, 14) % M])).astype(np.int64)
    _check(x, T, a, y, acc, rows)
