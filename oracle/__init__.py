"""Oracle for the BitLinear forward: ctypes wrapper around ``oracle.c``.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import this package.  The CUDA
library never imports, links or loads it, and this package never imports the
CUDA library.

Every function takes and returns numpy arrays and follows the definitions
in ``oracle.c`` (BitNet b1.58 weight/activation quantisation, the I2_S code
map, Sparse-BitNet N:M masks); see the citations there.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

QB = 127  # the product's Q_b; the oracle also accepts 128 (the blog's literal 2**(bits-1))


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` with gcc into ``liboracle.so`` (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=gnu11", "-fPIC", "-shared", "-pthread", "-ffp-contract=off",
             "-fno-fast-math", "-fno-builtin", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i32, i64, f32 = ctypes.c_int, ctypes.c_int64, ctypes.c_float
        sig = {
            "orc_absmean": (f32, [P, i64]),
            "orc_ternarize": (None, [P, i64, f32, P]),
            "orc_nm_mask": (None, [P, i32, i32, i32, i32, P]),
            "orc_apply_mask": (None, [P, P, i64]),
            "orc_dense_ld": (i64, [i32]),
            "orc_nm_values_ld": (i64, [i32, i32, i32]),
            "orc_nm_meta_ld": (i64, [i32]),
            "orc_pack_dense": (None, [P, i32, i32, P]),
            "orc_unpack_dense": (None, [P, i32, i32, P]),
            "orc_pack_nm": (i32, [P, P, i32, i32, i32, i32, P, P]),
            "orc_unpack_nm": (i32, [P, P, i32, i32, i32, i32, P]),
            "orc_quant_act": (None, [P, i32, i32, i32, P, P, P]),
            "orc_rmsnorm": (None, [P, P, i32, i32, f32, P]),
            "orc_quant_act_f32": (None, [P, i32, i32, i32, P, P, P]),
            "orc_matmul_i32": (i32, [P, P, i32, i32, i32, P]),
            "orc_matmul_i32_threads": (i32, [P, P, i32, i32, i32, P, i32]),
            "orc_online_cpus": (i32, []),
            "orc_dequant": (None, [P, P, f32, i32, i32, i32, P]),
            "orc_bf16_from_f64": (ctypes.c_uint16, [ctypes.c_double]),
            "orc_hadamard_block": (i32, [i32]),
            "orc_hadamard_rows": (None, [P, i32, i32, i32, P]),
            "orc_quant_act4": (None, [P, i32, i32, P, P, P]),
            "orc_forward_hbit": (i32, [P, i32, i32, P, i32, f32, P, P, P, P]),
            "orc_relu2_glu": (None, [P, P, i64, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def absmean(W: np.ndarray) -> np.float32:
    """alpha = mean |W| (fp64 sum in storage order, rounded once to fp32)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    return np.float32(_load().orc_absmean(_ptr(W), W.size))


def ternarize(W: np.ndarray, alpha) -> np.ndarray:
    """W_t = clamp(rne(W / RN(alpha + 1e-5)), -1, 1) in fp32."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    out = np.empty(W.shape, dtype=np.int8)
    _load().orc_ternarize(_ptr(W), W.size, float(np.float32(alpha)), _ptr(out))
    return out


def nm_mask(W: np.ndarray, n: int, m: int) -> np.ndarray:
    """Top-n of |W| in each block of m consecutive k (ties to the lower k)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    assert K % m == 0
    out = np.empty((N, K), dtype=np.uint8)
    _load().orc_nm_mask(_ptr(W), N, K, n, m, _ptr(out))
    return out


def apply_mask(Wt: np.ndarray, mask: np.ndarray) -> np.ndarray:
    out = np.ascontiguousarray(Wt, dtype=np.int8).copy()
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    _load().orc_apply_mask(_ptr(out), _ptr(mask), out.size)
    return out


def dense_ld(K: int) -> int:
    return int(_load().orc_dense_ld(K))


def nm_values_ld(K: int, n: int, m: int) -> int:
    return int(_load().orc_nm_values_ld(K, n, m))


def nm_meta_ld(K: int) -> int:
    return int(_load().orc_nm_meta_ld(K))


def pack_dense(Wt: np.ndarray) -> np.ndarray:
    """Dense 2-bit I2_S-coded matrix, shape [N, dense_ld(K)] uint8."""
    Wt = np.ascontiguousarray(Wt, dtype=np.int8)
    N, K = Wt.shape
    out = np.empty((N, dense_ld(K)), dtype=np.uint8)
    _load().orc_pack_dense(_ptr(Wt), N, K, _ptr(out))
    return out


def unpack_dense(codes: np.ndarray, N: int, K: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    assert codes.size >= N * dense_ld(K)
    out = np.empty((N, K), dtype=np.int8)
    _load().orc_unpack_dense(_ptr(codes), N, K, _ptr(out))
    return out


def pack_nm(Wt: np.ndarray, mask: np.ndarray, n: int, m: int):
    """(values [N, nm_values_ld], meta [N, nm_meta_ld]) of the masked matrix."""
    Wt = np.ascontiguousarray(Wt, dtype=np.int8)
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    N, K = Wt.shape
    vals = np.empty((N, nm_values_ld(K, n, m)), dtype=np.uint8)
    meta = np.empty((N, nm_meta_ld(K)), dtype=np.uint8)
    rc = _load().orc_pack_nm(_ptr(Wt), _ptr(mask), N, K, n, m, _ptr(vals), _ptr(meta))
    if rc != 0:
        raise ValueError("oracle pack_nm: unsupported pattern or mask count")
    return vals, meta


def unpack_nm(vals: np.ndarray, meta: np.ndarray, N: int, K: int, n: int, m: int) -> np.ndarray:
    vals = np.ascontiguousarray(vals, dtype=np.uint8)
    meta = np.ascontiguousarray(meta, dtype=np.uint8)
    out = np.empty((N, K), dtype=np.int8)
    rc = _load().orc_unpack_nm(_ptr(vals), _ptr(meta), N, K, n, m, _ptr(out))
    if rc != 0:
        raise ValueError("oracle unpack_nm: unsupported pattern")
    return out


def quant_act(x_bf16: np.ndarray, Qb: int = QB):
    """(q int8 [M,K], gamma fp32 [M], rowsum int32 [M]) from bf16 bits [M,K]."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    M, K = x.shape
    q = np.empty((M, K), dtype=np.int8)
    g = np.empty(M, dtype=np.float32)
    rs = np.empty(M, dtype=np.int32)
    _load().orc_quant_act(_ptr(x), M, K, Qb, _ptr(q), _ptr(g), _ptr(rs))
    return q, g, rs


def rmsnorm(x_bf16: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """fp32 [M,K]: RN(RN(x * r) * g), r = RN32(1 / sqrt(RN32(mean x^2) + eps)) in fp64."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    M, K = x.shape
    g = np.ascontiguousarray(g, dtype=np.float32)
    assert g.shape == (K,)
    xn = np.empty((M, K), dtype=np.float32)
    _load().orc_rmsnorm(_ptr(x), _ptr(g), M, K, eps, _ptr(xn))
    return xn


def quant_act_f32(xn: np.ndarray, Qb: int = QB):
    """(q int8 [M,K], gamma fp32 [M], rowsum int32 [M]) from fp32 rows."""
    xn = np.ascontiguousarray(xn, dtype=np.float32)
    M, K = xn.shape
    q = np.empty((M, K), dtype=np.int8)
    gm = np.empty(M, dtype=np.float32)
    rs = np.empty(M, dtype=np.int32)
    _load().orc_quant_act_f32(_ptr(xn), M, K, Qb, _ptr(q), _ptr(gm), _ptr(rs))
    return q, gm, rs


def forward_norm(x_bf16: np.ndarray, g: np.ndarray, eps: float, Wt: np.ndarray, alpha, Qb: int = QB):
    """BitLinear with RMSNorm first: (y bf16 bits, acc int32, q, gamma, rowsum)."""
    xn = rmsnorm(x_bf16, g, eps)
    q, gm, rs = quant_act_f32(xn, Qb)
    acc = matmul_i32(q, Wt)
    y = dequant(acc, gm, alpha, Qb)
    return y, acc, q, gm, rs


def matmul_i32(q: np.ndarray, Wt: np.ndarray) -> np.ndarray:
    """acc[m, n] = sum_k q[m, k] * Wt[n, k] (int32, checked in int64)."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    Wt = np.ascontiguousarray(Wt, dtype=np.int8)
    M, K = q.shape
    N, K2 = Wt.shape
    assert K == K2
    acc = np.empty((M, N), dtype=np.int32)
    if _load().orc_matmul_i32(_ptr(q), _ptr(Wt), M, N, K, _ptr(acc)) != 0:
        raise OverflowError("accumulator left int32")
    return acc


def matmul_i32_threads(q: np.ndarray, Wt: np.ndarray, threads: int) -> np.ndarray:
    """matmul_i32 with the output columns split over `threads` POSIX threads (same loop per element)."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    Wt = np.ascontiguousarray(Wt, dtype=np.int8)
    M, K = q.shape
    N, K2 = Wt.shape
    assert K == K2
    acc = np.empty((M, N), dtype=np.int32)
    if _load().orc_matmul_i32_threads(_ptr(q), _ptr(Wt), M, N, K, _ptr(acc), int(threads)) != 0:
        raise OverflowError("accumulator left int32 (or a thread could not start)")
    return acc


def online_cpus() -> int:
    """Host threads the system reports online."""
    return int(_load().orc_online_cpus())


def dequant(acc: np.ndarray, gamma: np.ndarray, alpha, Qb: int = QB) -> np.ndarray:
    """bf16 bits of acc * alpha * gamma / Qb (fp64, one rounding)."""
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    gamma = np.ascontiguousarray(gamma, dtype=np.float32)
    M, N = acc.shape
    y = np.empty((M, N), dtype=np.uint16)
    _load().orc_dequant(_ptr(acc), _ptr(gamma), float(np.float32(alpha)), M, N, Qb, _ptr(y))
    return y


def bf16_from_f64(v: float) -> int:
    return int(_load().orc_bf16_from_f64(float(v)))


def relu2_glu(g_bf16: np.ndarray, u_bf16: np.ndarray) -> np.ndarray:
    """h = RN_bf16(RN_bf16(max(g, 0)^2) * u) elementwise on bf16 bits (the 2B4T FFN's squared ReLU on
    the gate, times the up projection)."""
    g = np.ascontiguousarray(g_bf16, dtype=np.uint16)
    u = np.ascontiguousarray(u_bf16, dtype=np.uint16)
    assert g.shape == u.shape
    h = np.empty(g.shape, dtype=np.uint16)
    _load().orc_relu2_glu(_ptr(g), _ptr(u), g.size, _ptr(h))
    return h


def forward(x_bf16: np.ndarray, Wt: np.ndarray, alpha, Qb: int = QB, threads: int = 1):
    """Full forward on a dense ternary matrix: returns (y bf16 bits, acc, q, gamma, rowsum).
    threads > 1 runs the contraction on that many host threads (same result)."""
    q, g, rs = quant_act(x_bf16, Qb)
    acc = matmul_i32(q, Wt) if threads <= 1 else matmul_i32_threads(q, Wt, threads)
    y = dequant(acc, g, alpha, Qb)
    return y, acc, q, g, rs


def pack_weights(W: np.ndarray, n: int = 0, m: int = 0):
    """Latent fp32 [N,K] -> dict(alpha, Wt (effective, masked), codes | values+meta, mask)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    alpha = absmean(W)
    Wt = ternarize(W, alpha)
    if n == 0 and m == 0:
        return {"alpha": alpha, "Wt": Wt, "codes": pack_dense(Wt)}
    mask = nm_mask(W, n, m)
    Weff = apply_mask(Wt, mask)
    vals, meta = pack_nm(Weff, mask, n, m)
    return {"alpha": alpha, "Wt": Weff, "values": vals, "meta": meta, "mask": mask}


# ---------------------------------------------------------------- H-BitLinear ("BitNet v2" page, brain.hanbit.co.kr:
# the H-BitLinear module and native 4-bit activation paragraphs)

def hadamard_block(K: int) -> int:
    """Size of the Hadamard blocks along K: the largest power of two dividing K."""
    return int(_load().orc_hadamard_block(int(K)))


def hadamard(x_bf16: np.ndarray, B: int = None) -> np.ndarray:
    """fp32 [M, K]: each B-block of each bf16 row times the orthonormal Sylvester
    Hadamard matrix (fast butterflies in fp32, then one multiply by RN32(1/sqrt(B)))."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    M, K = x.shape
    if B is None:
        B = hadamard_block(K)
    assert B >= 1 and (B & (B - 1)) == 0 and K % B == 0
    xh = np.empty((M, K), dtype=np.float32)
    _load().orc_hadamard_rows(_ptr(x), M, K, int(B), _ptr(xh))
    return xh


def quant_act4(xh: np.ndarray):
    """(q int8 in [-8, 7], gamma fp32 [M], rowsum int32 [M]) of fp32 rows, Q_b = 7."""
    xh = np.ascontiguousarray(xh, dtype=np.float32)
    M, K = xh.shape
    q = np.empty((M, K), dtype=np.int8)
    g = np.empty(M, dtype=np.float32)
    rs = np.empty(M, dtype=np.int32)
    _load().orc_quant_act4(_ptr(xh), M, K, _ptr(q), _ptr(g), _ptr(rs))
    return q, g, rs


def forward_hbit(x_bf16: np.ndarray, Wt: np.ndarray, alpha):
    """H-BitLinear: Hadamard transform, 4-bit codes, ternary contraction, y = acc * alpha * gamma / 7.
    Returns (y bf16 bits, acc, q, gamma)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    Wt = np.ascontiguousarray(Wt, dtype=np.int8)
    M, K = x.shape
    N = Wt.shape[0]
    y = np.empty((M, N), dtype=np.uint16)
    q = np.empty((M, K), dtype=np.int8)
    acc = np.empty((M, N), dtype=np.int32)
    g = np.empty(M, dtype=np.float32)
    if _load().orc_forward_hbit(_ptr(x), M, K, _ptr(Wt), N, float(np.float32(alpha)), _ptr(y), _ptr(q), _ptr(acc),
                                _ptr(g)) != 0:
        raise OverflowError("accumulator left int32")
    return y, acc, q, g
