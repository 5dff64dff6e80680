"""B200 (sm_100a) BitLinear forward: thin Python binding over ``libbitlinear.so``.

Every step of the forward pass runs in the library's CUDA kernels; this module
only marshals torch tensors (device memory, the current stream) into the C ABI
of ``include/bitlinear.h``.  There is no CPU fallback: if the library is not
built, or the device is not sm_100, the calls raise.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

__all__ = [
    "BitLinearError", "PackedWeights", "lib", "packed_layout", "pack_weights", "pack_ternary",
    "quant_act", "rmsnorm_quant_act", "forward", "forward_nm", "forward_group", "forward_norm",
    "forward_workspace_bytes", "device_status", "last_kernel", "layout_version", "hadamard_quant_act4",
    "forward_hbit", "HBIT_MAX_K", "forward_q8", "forward_q8_workspace_bytes", "forward_relu2_glu",
    "forward_relu2_glu_workspace_bytes",
    "FLAG_PDL", "FLAG_PATH_GEMV", "FLAG_PATH_TC", "FLAG_DECODE_LUT", "FLAG_PATH_PERSISTENT", "FLAG_NM24_EXPAND",
]

FLAG_PDL = 0x1
MAX_GROUP = 4
FLAG_PATH_GEMV = 0x2
FLAG_PATH_TC = 0x4
FLAG_DECODE_LUT = 0x8
FLAG_PATH_PERSISTENT = 0x10
FLAG_NM24_EXPAND = 0x20

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libbitlinear.so")


class BitLinearError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {lib().bitlinear_status_string(status).decode()} (status {status})")
        self.status = status


class _Weights(ctypes.Structure):
    _fields_ = [
        ("N", ctypes.c_int32), ("K", ctypes.c_int32), ("nm_n", ctypes.c_int32), ("nm_m", ctypes.c_int32),
        ("codes", ctypes.c_void_p), ("meta", ctypes.c_void_p), ("alpha", ctypes.c_void_p),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded C-ABI library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"{_LIB_PATH} is missing: build the CUDA library first "
                "(python -m ternary_weight_linear_fwd_b200.build)")
        L = ctypes.CDLL(_LIB_PATH)
        P, i32, i64, u32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32, ctypes.c_size_t
        st = ctypes.c_int
        sig = {
            "bitlinear_packed_layout": (st, [i32, i32, i32, i32, P, P, P, P]),
            "bitlinear_pack_workspace_bytes": (sz, [i32, i32]),
            "bitlinear_pack_weights": (st, [P, i32, i32, i32, i32, P, P, P, P, sz, P]),
            "bitlinear_pack_ternary": (st, [P, i32, i32, ctypes.c_float, P, P, P]),
            "bitlinear_quant_act": (st, [P, i32, i32, P, P, P, P]),
            "bitlinear_forward_workspace_bytes": (sz, [i32, i32, i32, u32]),
            "bitlinear_forward": (st, [ctypes.POINTER(_Weights), P, i32, P, P, P, sz, u32, P]),
            "bitlinear_forward_nm": (st, [ctypes.POINTER(_Weights), P, i32, P, P, P, sz, u32, P]),
            "bitlinear_forward_group": (st, [ctypes.POINTER(_Weights), i32, P, i32, P, P, P, sz, u32, P]),
            "bitlinear_rmsnorm_quant_act": (st, [P, i32, i32, P, ctypes.c_float, P, P, P, P]),
            "bitlinear_forward_norm": (st, [ctypes.POINTER(_Weights), P, i32, P, ctypes.c_float, P, P, P, sz, u32, P]),
            "bitlinear_hadamard_quant_act4": (st, [P, i32, i32, P, P, P, P]),
            "bitlinear_forward_hbit": (st, [ctypes.POINTER(_Weights), P, i32, P, P, P, sz, u32, P]),
            "bitlinear_forward_q8": (st, [ctypes.POINTER(_Weights), P, i32, P, P, i32, P, P, P, sz, u32, P]),
            "bitlinear_forward_q8_workspace_bytes": (sz, [i32, i32, i32]),
            "bitlinear_forward_relu2_glu": (st, [ctypes.POINTER(_Weights), ctypes.POINTER(_Weights), P, i32, P, P, sz,
                                                 u32, P]),
            "bitlinear_forward_relu2_glu_workspace_bytes": (sz, [i32, i32, i32, u32]),
            "bitlinear_device_status": (st, [P, ctypes.POINTER(i32), i32]),
            "bitlinear_last_kernel": (ctypes.c_char_p, []),
            "bitlinear_layout_version": (i32, []),
            "bitlinear_status_string": (ctypes.c_char_p, [st]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(status: int, what: str):
    if status != 0:
        raise BitLinearError(status, what)


def _stream(stream=None) -> int:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _check_out(t, shape, dtype, device, what: str):
    """A caller-supplied output must be a contiguous tensor of exactly the shape, dtype and device the
    kernels write: they take only its address, so anything smaller would be overrun."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype or t.device != device or not t.is_contiguous():
        raise ValueError(f"{what}: expected a contiguous {dtype} tensor of shape {tuple(shape)} on {device}, "
                         f"got {tuple(t.shape)} {t.dtype} on {t.device}"
                         f"{'' if t.is_contiguous() else ' (not contiguous)'}")


def _check_workspace(t, device):
    if t is not None and (t.device != device or not t.is_contiguous()):
        raise ValueError(f"workspace: expected a contiguous tensor on {device}, got one on {t.device}")


def packed_layout(N: int, K: int, n: int = 0, m: int = 0):
    """(ld_codes, ld_meta, codes_bytes, meta_bytes) of the packed layout."""
    a, b = ctypes.c_int64(), ctypes.c_int64()
    c, d = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().bitlinear_packed_layout(N, K, n, m, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c),
                                         ctypes.byref(d)), "packed_layout")
    return a.value, b.value, c.value, d.value


@dataclass
class PackedWeights:
    N: int
    K: int
    nm_n: int
    nm_m: int
    codes: "object"           # torch.uint8 [N, ld_codes] on the device
    meta: "object"            # torch.uint8 [N, ld_meta] or None
    alpha: "object"           # torch.float32 [1]

    def c_struct(self) -> _Weights:
        return _Weights(self.N, self.K, self.nm_n, self.nm_m, _ptr(self.codes), _ptr(self.meta), _ptr(self.alpha))

    @property
    def nbytes(self) -> int:
        return self.codes.numel() + (0 if self.meta is None else self.meta.numel())


def _alloc_packed(N, K, n, m, device):
    import torch
    ldc, ldm, _, _ = packed_layout(N, K, n, m)
    codes = torch.empty((N, ldc), dtype=torch.uint8, device=device)
    meta = torch.empty((N, ldm), dtype=torch.uint8, device=device) if m else None
    alpha = torch.empty(1, dtype=torch.float32, device=device)
    return codes, meta, alpha


def pack_weights(W, n: int = 0, m: int = 0, stream=None) -> PackedWeights:
    """Absmean-ternarise and pack a latent fp32 [N, K] CUDA matrix (optionally N:M)."""
    import torch
    assert W.is_cuda and W.dtype == torch.float32 and W.is_contiguous() and W.dim() == 2
    N, K = W.shape
    codes, meta, alpha = _alloc_packed(N, K, n, m, W.device)
    ws = torch.empty(lib().bitlinear_pack_workspace_bytes(N, K), dtype=torch.uint8, device=W.device)
    _check(lib().bitlinear_pack_weights(_ptr(W), N, K, n, m, _ptr(codes), _ptr(meta), _ptr(alpha), _ptr(ws),
                                        ws.numel(), _stream(stream)), "pack_weights")
    return PackedWeights(N, K, n, m, codes, meta, alpha)


def pack_ternary(Wt, alpha: float, stream=None) -> PackedWeights:
    """Pack an int8 [N, K] CUDA matrix with values in {-1, 0, 1} and a given scale."""
    import torch
    assert Wt.is_cuda and Wt.dtype == torch.int8 and Wt.is_contiguous() and Wt.dim() == 2
    N, K = Wt.shape
    codes, _, a = _alloc_packed(N, K, 0, 0, Wt.device)
    _check(lib().bitlinear_pack_ternary(_ptr(Wt), N, K, float(alpha), _ptr(codes), _ptr(a), _stream(stream)),
           "pack_ternary")
    return PackedWeights(N, K, 0, 0, codes, None, a)


def quant_act(x, rowsum: bool = True, stream=None):
    """Per-token int8 codes of a bf16 [M, K] CUDA matrix: (q, gamma, rowsum or None)."""
    import torch
    assert x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous() and x.dim() == 2
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    g = torch.empty(M, dtype=torch.float32, device=x.device)
    rs = torch.empty(M, dtype=torch.int32, device=x.device) if rowsum else None
    _check(lib().bitlinear_quant_act(_ptr(x), M, K, _ptr(q), _ptr(g), _ptr(rs), _stream(stream)), "quant_act")
    return q, g, rs


def rmsnorm_quant_act(x, g, eps: float, rowsum: bool = True, stream=None):
    """RMSNorm (weight g, fp32 [K]) then per-token int8 codes of a bf16 [M, K] CUDA matrix:
    (q, gamma, rowsum or None)."""
    import torch
    assert x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous() and x.dim() == 2
    assert g.is_cuda and g.dtype == torch.float32 and g.is_contiguous() and g.numel() == x.shape[1]
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    gm = torch.empty(M, dtype=torch.float32, device=x.device)
    rs = torch.empty(M, dtype=torch.int32, device=x.device) if rowsum else None
    _check(lib().bitlinear_rmsnorm_quant_act(_ptr(x), M, K, _ptr(g), float(eps), _ptr(q), _ptr(gm), _ptr(rs),
                                             _stream(stream)), "rmsnorm_quant_act")
    return q, gm, rs


HBIT_MAX_K = 16384


def hadamard_quant_act4(x, rowsum: bool = True, stream=None):
    """H-BitLinear activations of a bf16 [M, K] CUDA matrix: the per-row Hadamard transform and 4-bit
    codes (natural k order): (q int8 in [-8, 7], gamma, rowsum or None)."""
    import torch
    assert x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous() and x.dim() == 2
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    g = torch.empty(M, dtype=torch.float32, device=x.device)
    rs = torch.empty(M, dtype=torch.int32, device=x.device) if rowsum else None
    _check(lib().bitlinear_hadamard_quant_act4(_ptr(x), M, K, _ptr(q), _ptr(g), _ptr(rs), _stream(stream)),
           "hadamard_quant_act4")
    return q, g, rs


def forward_hbit(w: PackedWeights, x, want_acc: bool = False, flags: int = 0, workspace=None, out=None,
                 acc_out=None, stream=None):
    """y = H-BitLinear(x): Hadamard transform, 4-bit codes, ternary contraction on the tensor cores,
    rescale by alpha * gamma / 7."""
    import torch
    assert x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous() and x.dim() == 2 and x.shape[1] == w.K
    M = x.shape[0]
    _check_out(out, (M, w.N), torch.bfloat16, x.device, "out")
    _check_out(acc_out, (M, w.N), torch.int32, x.device, "acc_out")
    _check_workspace(workspace, x.device)
    y = out if out is not None else torch.empty((M, w.N), dtype=torch.bfloat16, device=x.device)
    acc = acc_out if acc_out is not None else (
        torch.empty((M, w.N), dtype=torch.int32, device=x.device) if want_acc else None)
    if workspace is None:
        workspace = torch.empty(forward_workspace_bytes(M, w.N, w.K, FLAG_PATH_TC), dtype=torch.uint8,
                                device=x.device)
    ws = w.c_struct()
    _check(lib().bitlinear_forward_hbit(ctypes.byref(ws), _ptr(x), M, _ptr(y), _ptr(acc), _ptr(workspace),
                                        workspace.numel() * workspace.element_size(), flags, _stream(stream)),
           "forward_hbit")
    return (y, acc) if want_acc else y


def forward_q8_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib().bitlinear_forward_q8_workspace_bytes(M, N, K))


def forward_q8(w: PackedWeights, q, gamma, rowsum, want_acc: bool = False, flags: int = 0, workspace=None, out=None,
               acc_out=None, stream=None):
    """y = BitLinear from activations already quantised (q int8 [M, ldq] natural k order with ldq >= K a
    multiple of 16 and zeros past K, gamma fp32 [M], rowsum int32 [M], e.g. from quant_act): the
    tensor-core GEMM alone, dense or N:M weights."""
    import torch
    assert q.is_cuda and q.dtype == torch.int8 and q.dim() == 2 and q.stride(1) == 1 and q.shape[1] >= w.K
    M = q.shape[0]
    assert gamma.dtype == torch.float32 and gamma.numel() == M and gamma.is_contiguous()
    assert rowsum.dtype == torch.int32 and rowsum.numel() == M and rowsum.is_contiguous()
    _check_out(out, (M, w.N), torch.bfloat16, q.device, "out")
    _check_out(acc_out, (M, w.N), torch.int32, q.device, "acc_out")
    _check_workspace(workspace, q.device)
    y = out if out is not None else torch.empty((M, w.N), dtype=torch.bfloat16, device=q.device)
    acc = acc_out if acc_out is not None else (
        torch.empty((M, w.N), dtype=torch.int32, device=q.device) if want_acc else None)
    need = forward_q8_workspace_bytes(M, w.N, w.K)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_n = 0 if workspace is None else workspace.numel() * workspace.element_size()
    ws = w.c_struct()
    _check(lib().bitlinear_forward_q8(ctypes.byref(ws), _ptr(q), q.stride(0), _ptr(gamma), _ptr(rowsum), M, _ptr(y),
                                      _ptr(acc), _ptr(workspace), ws_n, flags, _stream(stream)), "forward_q8")
    return (y, acc) if want_acc else y


def forward_workspace_bytes(M: int, N: int, K: int, flags: int = 0) -> int:
    return int(lib().bitlinear_forward_workspace_bytes(M, N, K, flags))


def _forward(fn, what, w: PackedWeights, x, want_acc, flags, workspace, out, acc_out, stream):
    import torch
    assert x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous() and x.dim() == 2 and x.shape[1] == w.K
    M = x.shape[0]
    _check_out(out, (M, w.N), torch.bfloat16, x.device, "out")
    _check_out(acc_out, (M, w.N), torch.int32, x.device, "acc_out")
    _check_workspace(workspace, x.device)
    y = out if out is not None else torch.empty((M, w.N), dtype=torch.bfloat16, device=x.device)
    acc = acc_out if acc_out is not None else (
        torch.empty((M, w.N), dtype=torch.int32, device=x.device) if want_acc else None)
    need = forward_workspace_bytes(M, w.N, w.K, flags)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_n = 0 if workspace is None else workspace.numel() * workspace.element_size()
    ws = w.c_struct()
    _check(fn(ctypes.byref(ws), _ptr(x), M, _ptr(y), _ptr(acc), _ptr(workspace), ws_n, flags, _stream(stream)), what)
    return (y, acc) if want_acc else y


def forward(w: PackedWeights, x, want_acc: bool = False, flags: int = 0, workspace=None, out=None, acc_out=None,
            stream=None):
    """y = BitLinear(x) (bf16 [M, N]); with want_acc also the int32 accumulator."""
    return _forward(lib().bitlinear_forward, "forward", w, x, want_acc, flags, workspace, out, acc_out, stream)


def forward_nm(w: PackedWeights, x, want_acc: bool = False, flags: int = 0, workspace=None, out=None, acc_out=None,
               stream=None):
    """Same as forward for N:M packed weights."""
    return _forward(lib().bitlinear_forward_nm, "forward_nm", w, x, want_acc, flags, workspace, out, acc_out, stream)


def forward_group(ws, x, want_acc: bool = False, flags: int = 0, workspace=None, outs=None, stream=None):
    """BitLinear of several matrices (same K) on one input x: a list of y
    (with want_acc, a list of (y, acc)), each identical to forward /
    forward_nm of that matrix."""
    import torch
    assert x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous() and x.dim() == 2
    count = len(ws)
    M = x.shape[0]
    if outs is not None:
        if len(outs) != count:
            raise ValueError(f"forward_group: {count} matrices but {len(outs)} outputs")
        for i, (o, w) in enumerate(zip(outs, ws)):
            _check_out(o, (M, w.N), torch.bfloat16, x.device, f"outs[{i}]")
    _check_workspace(workspace, x.device)
    ys = outs if outs is not None else [torch.empty((M, w.N), dtype=torch.bfloat16, device=x.device) for w in ws]
    accs = [torch.empty((M, w.N), dtype=torch.int32, device=x.device) for w in ws] if want_acc else None
    need = max((forward_workspace_bytes(M, w.N, w.K, flags) for w in ws), default=0)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_n = 0 if workspace is None else workspace.numel() * workspace.element_size()
    arr = (_Weights * max(count, 1))(*[w.c_struct() for w in ws])
    yp = (ctypes.c_void_p * max(count, 1))(*[_ptr(y) for y in ys])
    ap = (ctypes.c_void_p * max(count, 1))(*[_ptr(a) for a in accs]) if want_acc else None
    _check(lib().bitlinear_forward_group(arr, count, _ptr(x), M, yp, ap, _ptr(workspace), ws_n, flags,
                                         _stream(stream)), "forward_group")
    return list(zip(ys, accs)) if want_acc else ys


def forward_relu2_glu_workspace_bytes(M: int, N: int, K: int, flags: int = 0) -> int:
    return int(lib().bitlinear_forward_relu2_glu_workspace_bytes(M, N, K, flags))


def forward_relu2_glu(w_gate: PackedWeights, w_up: PackedWeights, x, flags: int = 0, workspace=None, out=None,
                      stream=None):
    """h = RN(RN(max(g, 0)^2) * u) with g, u the BitLinear outputs of the FFN's gate and up projections
    on x (same N and K): the 2B4T FFN's squared ReLU on the gate, times the up projection."""
    import torch
    assert x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous() and x.dim() == 2 and x.shape[1] == w_gate.K
    if (w_up.N, w_up.K) != (w_gate.N, w_gate.K):
        raise ValueError("forward_relu2_glu: gate and up must have the same N and K")
    M = x.shape[0]
    _check_out(out, (M, w_gate.N), torch.bfloat16, x.device, "out")
    _check_workspace(workspace, x.device)
    h = out if out is not None else torch.empty((M, w_gate.N), dtype=torch.bfloat16, device=x.device)
    need = forward_relu2_glu_workspace_bytes(M, w_gate.N, w_gate.K, flags)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_n = 0 if workspace is None else workspace.numel() * workspace.element_size()
    wg, wu = w_gate.c_struct(), w_up.c_struct()
    _check(lib().bitlinear_forward_relu2_glu(ctypes.byref(wg), ctypes.byref(wu), _ptr(x), M, _ptr(h),
                                             _ptr(workspace), ws_n, flags, _stream(stream)), "forward_relu2_glu")
    return h


def forward_norm(w: PackedWeights, x, g, eps: float, want_acc: bool = False, flags: int = 0, workspace=None,
                 out=None, acc_out=None, stream=None):
    """y = BitLinear(RMSNorm(x)) with the normalisation fused into the activation quantisation."""
    import torch
    assert x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous() and x.dim() == 2 and x.shape[1] == w.K
    assert g.is_cuda and g.dtype == torch.float32 and g.is_contiguous() and g.numel() == w.K
    M = x.shape[0]
    _check_out(out, (M, w.N), torch.bfloat16, x.device, "out")
    _check_out(acc_out, (M, w.N), torch.int32, x.device, "acc_out")
    _check_workspace(workspace, x.device)
    y = out if out is not None else torch.empty((M, w.N), dtype=torch.bfloat16, device=x.device)
    acc = acc_out if acc_out is not None else (
        torch.empty((M, w.N), dtype=torch.int32, device=x.device) if want_acc else None)
    need = forward_workspace_bytes(M, w.N, w.K, FLAG_PATH_TC)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_n = workspace.numel() * workspace.element_size()
    ws = w.c_struct()
    _check(lib().bitlinear_forward_norm(ctypes.byref(ws), _ptr(x), M, _ptr(g), float(eps), _ptr(y), _ptr(acc),
                                        _ptr(workspace), ws_n, flags, _stream(stream)), "forward_norm")
    return (y, acc) if want_acc else y


def device_status(clear: bool = True, stream=None) -> int:
    v = ctypes.c_int32()
    _check(lib().bitlinear_device_status(_stream(stream), ctypes.byref(v), 1 if clear else 0), "device_status")
    return v.value


def last_kernel() -> str:
    return lib().bitlinear_last_kernel().decode()


def layout_version() -> int:
    """Version of the packed weight layouts the library reads and writes."""
    return int(lib().bitlinear_layout_version())


NOALLOC_SCRATCH_BYTES = 8 << 20


def forward_noalloc(w: PackedWeights, x, out=None, acc_out=None, want_acc: bool = False, flags: int = 0,
                    stream=None):
    """BitLinear forward that allocates nothing inside the library: the scratch
    of the tensor-core path comes from one fixed array per device, shared by
    all calls (so calls running concurrently on different streams race).
    For hosts that can hand over only inputs and outputs.  Raises
    BitLinearError (status 5) when the shape needs more than
    NOALLOC_SCRATCH_BYTES of scratch."""
    import torch
    L = lib()
    fn = L.bitlinear_forward_noalloc
    if fn.argtypes is None:
        fn.restype = ctypes.c_int
        fn.argtypes = [ctypes.POINTER(_Weights), ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                       ctypes.c_uint32, ctypes.c_void_p]
    assert x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous() and x.dim() == 2 and x.shape[1] == w.K
    M = x.shape[0]
    _check_out(out, (M, w.N), torch.bfloat16, x.device, "out")
    _check_out(acc_out, (M, w.N), torch.int32, x.device, "acc_out")
    y = out if out is not None else torch.empty((M, w.N), dtype=torch.bfloat16, device=x.device)
    acc = acc_out if acc_out is not None else (
        torch.empty((M, w.N), dtype=torch.int32, device=x.device) if want_acc else None)
    ws = w.c_struct()
    _check(fn(ctypes.byref(ws), _ptr(x), M, _ptr(y), _ptr(acc), flags, _stream(stream)), "forward_noalloc")
    return (y, acc) if (want_acc or acc_out is not None) else y
