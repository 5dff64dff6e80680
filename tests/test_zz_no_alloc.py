"""bitlinear_forward_noalloc: the forward for hosts that cannot allocate device
memory (plugins with a fixed memory budget, latency-critical callers that may
not call cudaMalloc / cudaFree on their hot path).  Its scratch is one fixed
array inside the library, so its results must equal those of
bitlinear_forward with a caller-provided workspace -- on consecutive calls too,
since each call reuses the array the previous one left behind.

The file name sorts after every other test file, so pytest collects it last:
a run that stops at the first failure has then already run every other test,
and the test also runs after the others have left the library's state (the
scratch array's contents) behind, as well as alone in a fresh process."""
import ctypes

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


def _lib():
    from ternary_weight_linear_fwd_b200 import build as b
    b.build()
    L = bl.lib()
    fn = L.bitlinear_forward_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.POINTER(bl._Weights), ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.c_uint32, ctypes.c_void_p]
    return L


def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _case(M, K, N, seed, n=0, m=0):
    x = synth.activations(M, K, seed=seed)
    W = synth.latent_weights(N, K, seed=seed)
    ref = oracle.pack_weights(W, n, m)
    w = bl.pack_weights(torch.from_numpy(W).to(DEV), n, m)
    xd = torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16)
    return w, xd, x, ref


def _noalloc(L, w, xd, flags=0):
    M = xd.shape[0]
    y = torch.empty((M, w.N), dtype=torch.bfloat16, device=DEV)
    acc = torch.empty((M, w.N), dtype=torch.int32, device=DEV)
    ws = w.c_struct()
    st = L.bitlinear_forward_noalloc(ctypes.byref(ws), xd.data_ptr(), M, y.data_ptr(), acc.data_ptr(), flags,
                                     torch.cuda.current_stream().cuda_stream)
    assert st == 0, L.bitlinear_status_string(st)
    return y, acc


def _check(L, fwd, M, K, N, seed, n, m, flags):
    """The no-allocation call equals the workspace call bit for bit (same kernels, same inputs) and the
    oracle within the parity tolerance (accumulators exact, outputs within one bf16 ulp)."""
    w, xd, x, ref = _case(M, K, N, seed, n, m)
    y_ref, acc_ref = fwd(w, xd, want_acc=True, flags=flags)
    y, acc = _noalloc(L, w, xd, flags)
    torch.cuda.synchronize()
    assert torch.equal(acc, acc_ref)
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
    yo, acco, *_ = oracle.forward(x, ref["Wt"], ref["alpha"])
    np.testing.assert_array_equal(acc.cpu().numpy(), acco)
    d = np.abs(_bits(y).astype(np.int32) - yo.astype(np.int32))
    assert d.max() <= 1  # one bf16 ulp, the tolerance of every forward parity test


# Calls in a row with different inputs and shapes, each reusing the scratch the previous call left
# behind: a K-split persistent tensor-core GEMM (few weight-row tiles), a tile-parallel one with a
# different M x N, the K-split one again, the fused few-token kernel and the M = 1 decode GEMV (these
# two use no scratch).
P = bl.FLAG_PATH_PERSISTENT


@pytest.mark.parametrize("n,m", [(0, 0), (6, 8)])
def test_noalloc_matches_workspace_forward_twice(n, m):
    L = _lib()
    fwd = bl.forward_nm if m else bl.forward
    for (M, K, N, seed, flags) in ((64, 2560, 640, 2, P), (300, 512, 2048, 1, P), (64, 2560, 640, 3, P),
                                   (16, 2560, 640, 5, 0), (1, 2560, 1000, 4, 0)):
        _check(L, fwd, M, K, N, seed, n, m, flags)
    assert bl.device_status() == 0


def test_noalloc_rejects_oversized_scratch():
    L = _lib()
    w, xd, _, _ = _case(2, 4096, 64, 3)
    big_m = 2048  # 2048 x 4096 int8 codes + scales exceed the fixed 8 MiB array
    assert bl.forward_workspace_bytes(big_m, 64, 4096) > bl.NOALLOC_SCRATCH_BYTES
    ws = w.c_struct()
    st = L.bitlinear_forward_noalloc(ctypes.byref(ws), xd.data_ptr(), big_m, xd.data_ptr(), None, 0,
                                     torch.cuda.current_stream().cuda_stream)
    assert st == 5  # BITLINEAR_ERR_WORKSPACE, nothing enqueued
