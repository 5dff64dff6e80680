"""The device status word: a kernel that gives up on a bounded wait records a
code there, writes no output, lets its in-flight copies land and exits, and
the context stays usable for the next call (bitlinear.h, conventions).

The give-up is provoked without any fault, in the test build of the library
(libbitlinear_testhooks.so, include/bitlinear_test_hooks.h): the decode GEMVs
are told to expect a few more copy bytes than they issue, so every issued
copy lands but the barrier never completes, and the wait limit is cut to a
few milliseconds.  Then the hooks are reset and the same call must match the
oracle again with a clean status word."""
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
PRODUCT_WAIT_NS = 1_000_000_000
SHORT_WAIT_NS = 2_000_000  # 2 ms


@pytest.fixture(scope="module")
def T():
    """The test build, bound with the entry points this file calls."""
    from ternary_weight_linear_fwd_b200 import build as b
    L = ctypes.CDLL(b.build_test_hooks())
    P, i32, u32, u64, st = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_int
    W = ctypes.POINTER(bl._Weights)
    for name, res, args in [
        ("bitlinear_test_set_wait_fault", st, [u64, u32]),
        ("bitlinear_pack_ternary", st, [P, i32, i32, ctypes.c_float, P, P, P]),
        ("bitlinear_pack_weights", st, [P, i32, i32, i32, i32, P, P, P, P, ctypes.c_size_t, P]),
        ("bitlinear_forward", st, [W, P, i32, P, P, P, ctypes.c_size_t, u32, P]),
        ("bitlinear_forward_nm", st, [W, P, i32, P, P, P, ctypes.c_size_t, u32, P]),
        ("bitlinear_device_status", st, [P, ctypes.POINTER(i32), i32]),
        ("bitlinear_pack_workspace_bytes", ctypes.c_size_t, [i32, i32]),
    ]:
        fn = getattr(L, name)
        fn.restype, fn.argtypes = res, args
    yield L
    assert L.bitlinear_test_set_wait_fault(PRODUCT_WAIT_NS, 0) == 0


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _status(L):
    v = ctypes.c_int32()
    assert L.bitlinear_device_status(_stream(), ctypes.byref(v), 1) == 0
    return v.value


def _pack(L, W, n, m):
    N, K = W.shape
    ldc, ldm, _, _ = bl.packed_layout(N, K, n, m)
    codes = torch.empty((N, ldc), dtype=torch.uint8, device=DEV)
    meta = torch.empty((N, ldm), dtype=torch.uint8, device=DEV) if m else None
    alpha = torch.empty(1, dtype=torch.float32, device=DEV)
    ws = torch.empty(L.bitlinear_pack_workspace_bytes(N, K), dtype=torch.uint8, device=DEV)
    Wd = torch.from_numpy(W).to(DEV)
    assert L.bitlinear_pack_weights(Wd.data_ptr(), N, K, n, m, codes.data_ptr(),
                                    None if meta is None else meta.data_ptr(), alpha.data_ptr(), ws.data_ptr(),
                                    ws.numel(), _stream()) == 0
    torch.cuda.synchronize()
    return bl.PackedWeights(N, K, n, m, codes, meta, alpha)


def _call(L, w, xd, flags=0):
    M, N = xd.shape[0], w.N
    y = torch.full((M, N), -1, dtype=torch.int16, device=DEV)  # 0xFFFF: a NaN pattern no output has
    acc = torch.full((M, N), -(2 ** 31), dtype=torch.int32, device=DEV)
    ws = w.c_struct()
    fn = L.bitlinear_forward_nm if w.nm_m else L.bitlinear_forward
    assert fn(ctypes.byref(ws), xd.data_ptr(), M, y.data_ptr(), acc.data_ptr(), None, 0, flags, _stream()) == 0
    torch.cuda.synchronize()
    return y.cpu().numpy().view(np.uint16), acc.cpu().numpy()


@pytest.mark.parametrize("n,m,flags", [(0, 0, 0), (0, 0, bl.FLAG_DECODE_LUT), (2, 4, 0), (6, 8, 0)])
def test_gemv_gives_up_records_status_and_recovers(T, n, m, flags):
    K, N = 1024, 700
    x = synth.activations(1, K, seed=70 + n)
    W = synth.latent_weights(N, K, seed=70 + n)
    ref = oracle.pack_weights(W, n, m)
    y_ref, acc_ref, *_ = oracle.forward(x, ref["Wt"], ref["alpha"])
    w = _pack(T, W, n, m)
    xd = torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16)
    assert _status(T) == 0

    assert T.bitlinear_test_set_wait_fault(SHORT_WAIT_NS, 16) == 0
    y, acc = _call(T, w, xd, flags)
    code = _status(T)
    assert code in (1, 5), code  # gave up on the weight copies (5: the drain wait ran out as well)
    assert np.all(y == 0xFFFF) and np.all(acc == -(2 ** 31))  # no CTA wrote an output

    assert T.bitlinear_test_set_wait_fault(PRODUCT_WAIT_NS, 0) == 0
    y, acc = _call(T, w, xd, flags)
    assert _status(T) == 0
    np.testing.assert_array_equal(acc, acc_ref)
    d = np.abs(y.astype(np.int32) - y_ref.astype(np.int32))
    assert d.max() <= 1


def test_few_token_kernel_gives_up_records_status_and_recovers(T):
    """The fused few-token tensor-core kernel (K split over a cluster): its weight chunks are told to
    expect more bytes than arrive, the unpack warps and the MMA issuer give up, every CTA still passes
    the cluster barriers, and since some CTA of each cluster gave up none stores a result."""
    M, K, N = 8, 2560, 700
    x = synth.activations(M, K, seed=77)
    W = synth.latent_weights(N, K, seed=78)
    ref = oracle.pack_weights(W)
    y_ref, acc_ref, *_ = oracle.forward(x, ref["Wt"], ref["alpha"])
    w = _pack(T, W, 0, 0)
    xd = torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16)
    assert _status(T) == 0

    assert T.bitlinear_test_set_wait_fault(SHORT_WAIT_NS, 16) == 0
    y, acc = _call(T, w, xd)
    code = _status(T)
    assert code in (2, 3, 4, 5), code
    assert np.all(y == 0xFFFF) and np.all(acc == -(2 ** 31))

    assert T.bitlinear_test_set_wait_fault(PRODUCT_WAIT_NS, 0) == 0
    y, acc = _call(T, w, xd)
    assert _status(T) == 0
    np.testing.assert_array_equal(acc, acc_ref)
    d = np.abs(y.astype(np.int32) - y_ref.astype(np.int32))
    assert d.max() <= 1
