"""C-ABI checks that need no GPU: the library builds and loads, exports every
entry point declared in include/bitlinear.h, agrees with the oracle on the
packed layout sizes (two independent implementations of the written format),
and rejects bad arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest

import oracle
from ternary_weight_linear_fwd_b200 import build as blbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bitlinear.h")


@pytest.fixture(scope="module")
def L():
    blbuild.build()
    import ternary_weight_linear_fwd_b200 as bl
    return bl.lib()


HOOKS_HEADER = os.path.join(ROOT, "include", "bitlinear_test_hooks.h")


def _declared(header=HEADER):
    src = open(header).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bitlinear_[a-z_0-9]+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = _declared()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n


def test_headers_cover_every_header_file():
    """include/ holds the product header and the test-hook header, nothing else."""
    assert sorted(os.listdir(os.path.join(ROOT, "include"))) == ["bitlinear.h", "bitlinear_test_hooks.h"]


def test_test_hooks_only_in_the_test_build(L):
    """The test build exports the product ABI plus the hooks; the product library has no hook."""
    hooks = _declared(HOOKS_HEADER)
    assert hooks == ["bitlinear_test_set_wait_fault", "bitlinear_test_timeline"]
    T = ctypes.CDLL(blbuild.build_test_hooks())
    for n in _declared() + hooks:
        assert hasattr(T, n), n
    for n in hooks:
        assert not hasattr(L, n), n


def test_status_strings(L):
    for code in range(0, 9):
        assert L.bitlinear_status_string(code)
    assert L.bitlinear_status_string(0) == b"ok"


@pytest.mark.parametrize("N,K,n,m", [(512, 256, 0, 0), (7, 3, 0, 0), (33, 200, 0, 0), (6912, 2560, 0, 0),
                                     (11008, 2048, 2, 4), (2048, 11008, 6, 8), (24, 1032, 7, 8),
                                     (40, 256, 1, 8), (5, 8, 3, 8), (3, 12, 2, 4)])
def test_layout_matches_oracle(N, K, n, m):
    import ternary_weight_linear_fwd_b200 as bl
    ldc, ldm, cb, mb = bl.packed_layout(N, K, n, m)
    if m == 0:
        assert ldc == oracle.dense_ld(K) and ldm == 0 and mb == 0
    else:
        assert ldc == oracle.nm_values_ld(K, n, m) and ldm == oracle.nm_meta_ld(K)
        assert mb == N * ldm
    assert cb == N * ldc


@pytest.mark.parametrize("n,m", [(3, 4), (8, 8), (0, 8), (2, 0), (4, 16)])
def test_layout_rejects_patterns(n, m):
    import ternary_weight_linear_fwd_b200 as bl
    with pytest.raises(bl.BitLinearError) as e:
        bl.packed_layout(64, 256, n, m)
    assert e.value.status == 4


def test_layout_rejects_shapes():
    import ternary_weight_linear_fwd_b200 as bl
    for N, K, n, m in [(0, 64, 0, 0), (64, 0, 0, 0), (64, 65537, 0, 0), (64, 100, 6, 8)]:
        with pytest.raises(bl.BitLinearError) as e:
            bl.packed_layout(N, K, n, m)
        assert e.value.status == 2


def _w(L, N=64, K=256, n=0, m=0, codes=0x10000, meta=None, alpha=0x20000):
    import ternary_weight_linear_fwd_b200 as bl
    return bl._Weights(N, K, n, m, codes, meta, alpha)


def test_forward_host_checks(L):
    """Argument errors come back before any device work (fake, never dereferenced addresses)."""
    fw = L.bitlinear_forward
    x, y = 0x30000, 0x40000
    assert fw(None, x, 1, y, None, None, 0, 0, None) == 1
    w = _w(L)
    assert fw(ctypes.byref(w), None, 1, y, None, None, 0, 0, None) == 1
    assert fw(ctypes.byref(w), x, 0, y, None, None, 0, 0, None) == 2
    assert fw(ctypes.byref(_w(L, K=70000)), x, 1, y, None, None, 0, 0, None) == 2
    assert fw(ctypes.byref(_w(L, codes=0x10008)), x, 1, y, None, None, 0, 0, None) == 3
    assert fw(ctypes.byref(w), x + 4, 1, y, None, None, 0, 0, None) == 3
    assert fw(ctypes.byref(w), x, 1, y, None, None, 0, 0x80, None) == 8          # unknown flag
    assert fw(ctypes.byref(w), x, 2, y, None, None, 0, 0x2, None) == 8           # GEMV path needs M == 1
    assert fw(ctypes.byref(w), x, 1, y, None, None, 0, 0x6, None) == 8           # both path flags
    assert fw(ctypes.byref(w), x, 2, y, None, None, 0, 0x8, None) == 8           # lookup-table decode needs M == 1
    assert fw(ctypes.byref(w), x, 1, y, None, None, 0, 0xC, None) == 8           # ... and the GEMV path
    nmw = _w(L, n=6, m=8, meta=0x50000)
    assert fw(ctypes.byref(nmw), x, 1, y, None, None, 0, 0, None) == 4          # dense entry, N:M weights
    assert L.bitlinear_forward_nm(ctypes.byref(w), x, 1, y, None, None, 0, 0, None) == 4
    assert L.bitlinear_forward_nm(ctypes.byref(_w(L, n=6, m=8)), x, 1, y, None, None, 0, 0, None) == 1
    assert L.bitlinear_forward_nm(ctypes.byref(_w(L, n=3, m=4, meta=0x50000)), x, 1, y, None, None, 0, 0,
                                  None) == 4


def test_pack_and_quant_host_checks(L):
    assert L.bitlinear_pack_weights(None, 64, 256, 0, 0, 0x1000, None, 0x2000, 0x3000, 8192, None) == 1
    assert L.bitlinear_pack_weights(0x1000, 64, 256, 3, 4, 0x1000, 0x4000, 0x2000, 0x3000, 8192, None) == 4
    assert L.bitlinear_pack_weights(0x1000, 64, 256, 0, 0, 0x1008, None, 0x2000, 0x3000, 8192, None) == 3
    assert L.bitlinear_pack_weights(0x1000, 64, 256, 0, 0, 0x1000, None, 0x2000, 0x3000, 16, None) == 5
    assert L.bitlinear_quant_act(None, 4, 64, 0x1000, 0x2000, None, None) == 1
    assert L.bitlinear_quant_act(0x1000, 0, 64, 0x1000, 0x2000, None, None) == 2
    assert L.bitlinear_quant_act(0x1002, 4, 64, 0x1000, 0x2000, None, None) == 3
    assert L.bitlinear_pack_ternary(None, 4, 64, 0.5, 0x1000, 0x2000, None) == 1


def test_workspace_sizes(L):
    assert L.bitlinear_forward_workspace_bytes(1, 6912, 2560, 0) == 0          # GEMV quantises in-kernel
    assert L.bitlinear_forward_workspace_bytes(1, 6912, 2560, 0x4) >= 2560     # forced tensor-core path
    assert L.bitlinear_forward_workspace_bytes(2048, 6912, 2560, 0) >= 2048 * 2560 + 2 * 4 * 2048
    assert L.bitlinear_pack_workspace_bytes(6912, 2560) >= 8 * 1024


def test_forward_group_host_checks(L):
    """Group-specific argument errors (fake, never dereferenced addresses)."""
    import ternary_weight_linear_fwd_b200 as bl
    fg = L.bitlinear_forward_group
    x = 0x30000
    ws = (bl._Weights * 5)(*[_w(L) for _ in range(5)])
    ys = (ctypes.c_void_p * 5)(*[0x40000 + 0x1000 * i for i in range(5)])
    assert fg(None, 1, x, 1, ys, None, None, 0, 0, None) == 1
    assert fg(ws, 1, x, 1, None, None, None, 0, 0, None) == 1
    assert fg(ws, 0, x, 1, ys, None, None, 0, 0, None) == 2                      # empty group
    assert fg(ws, 5, x, 1, ys, None, None, 0, 0, None) == 2                      # above MAX_GROUP
    bad_k = (bl._Weights * 2)(_w(L), _w(L, K=512))
    assert fg(bad_k, 2, x, 1, ys, None, None, 0, 0, None) == 2                   # unequal K
    bad_a = (bl._Weights * 2)(_w(L), _w(L, codes=0x10008))
    assert fg(bad_a, 2, x, 1, ys, None, None, 0, 0, None) == 3
    bad_p = (bl._Weights * 2)(_w(L), _w(L, n=3, m=4, meta=0x50000))
    assert fg(bad_p, 2, x, 1, ys, None, None, 0, 0, None) == 4
    nometa = (bl._Weights * 2)(_w(L), _w(L, n=2, m=4))
    assert fg(nometa, 2, x, 1, ys, None, None, 0, 0, None) == 1
    assert fg(ws, 2, x, 2, ys, None, None, 0, 0x2, None) == 8                    # GEMV path needs M == 1


def test_rmsnorm_entry_points_host_checks(L):
    """RMSNorm entry points reject bad arguments before any device work (fake addresses)."""
    x, g, q, gm = 0x30000, 0x40000, 0x50000, 0x60000
    f = L.bitlinear_rmsnorm_quant_act
    assert f(None, 4, 64, g, 1e-6, q, gm, None, None) == 1
    assert f(x, 4, 64, None, 1e-6, q, gm, None, None) == 1
    assert f(x, 0, 64, g, 1e-6, q, gm, None, None) == 2
    assert f(x, 4, 64, g, -1.0, q, gm, None, None) == 2           # eps out of range
    assert f(x, 4, 64, g, float("nan"), q, gm, None, None) == 2
    assert f(x + 2, 4, 64, g, 1e-6, q, gm, None, None) == 3
    assert f(x, 4, 64, g + 2, 1e-6, q, gm, None, None) == 3
    fn = L.bitlinear_forward_norm
    w = _w(L)
    y = 0x70000
    assert fn(ctypes.byref(w), x, 1, None, 1e-6, y, None, None, 0, 0, None) == 1
    assert fn(ctypes.byref(w), x, 1, g, 2.0, y, None, None, 0, 0, None) == 2
    assert fn(ctypes.byref(w), x, 1, g, 1e-6, y, None, None, 0, 0x2, None) == 8   # the GEMV path is not offered
    assert fn(ctypes.byref(_w(L, codes=0x10008)), x, 1, g, 1e-6, y, None, None, 0, 0, None) == 3


def test_binding_rejects_bad_outputs():
    """Caller-supplied outputs must have exactly the shape, dtype and device the kernels write (they
    receive only an address); the checks run before any library call, so CPU tensors exercise them."""
    torch = pytest.importorskip("torch")
    import ternary_weight_linear_fwd_b200 as bl
    dev = torch.device("cpu")
    good = torch.empty((3, 5), dtype=torch.bfloat16)
    bl._check_out(good, (3, 5), torch.bfloat16, dev, "out")
    bl._check_out(None, (3, 5), torch.bfloat16, dev, "out")
    bad = [torch.empty((3, 4), dtype=torch.bfloat16),            # too narrow: would be overrun
           torch.empty((2, 5), dtype=torch.bfloat16),            # too few rows
           torch.empty((3, 5), dtype=torch.float32),             # wrong dtype
           torch.empty((5, 3), dtype=torch.bfloat16).t(),        # right shape, not contiguous
           torch.empty((3, 10), dtype=torch.bfloat16)[:, ::2]]   # strided view
    for t in bad:
        with pytest.raises(ValueError):
            bl._check_out(t, (3, 5), torch.bfloat16, dev, "out")
    with pytest.raises(ValueError):
        bl._check_out(good, (3, 5), torch.bfloat16, torch.device("meta"), "out")
    bl._check_workspace(torch.empty(64, dtype=torch.uint8), dev)
    with pytest.raises(ValueError):
        bl._check_workspace(torch.empty((8, 16), dtype=torch.uint8)[:, ::2], dev)


def test_layout_version_matches_header(L):
    m = re.search(r"#define BITLINEAR_LAYOUT_VERSION (\d+)", open(HEADER).read())
    assert m is not None
    L.bitlinear_layout_version.restype = ctypes.c_int32
    assert L.bitlinear_layout_version() == int(m.group(1))
    import ternary_weight_linear_fwd_b200 as bl
    assert bl.layout_version() == int(m.group(1))


def test_hbit_host_checks(L):
    """H-BitLinear argument errors come back before any device work (fake addresses)."""
    fh = L.bitlinear_forward_hbit
    x, y = 0x30000, 0x40000
    assert fh(None, x, 1, y, None, None, 0, 0, None) == 1
    assert fh(ctypes.byref(_w(L, K=16385)), x, 1, y, None, None, 0, 0, None) == 2   # above the transform limit
    assert fh(ctypes.byref(_w(L)), x, 0, y, None, None, 0, 0, None) == 2
    assert fh(ctypes.byref(_w(L)), x + 4, 1, y, None, None, 0, 0, None) == 3
    assert fh(ctypes.byref(_w(L)), x, 1, y, None, None, 0, 0x2, None) == 8          # no GEMV path
    hq = L.bitlinear_hadamard_quant_act4
    assert hq(None, 4, 64, 0x1000, 0x2000, None, None) == 1
    assert hq(0x1000, 4, 16385, 0x1000, 0x2000, None, None) == 2
    assert hq(0x1001, 4, 64, 0x1000, 0x2000, None, None) == 3


def test_flag_values_match_header():
    """Every BITLINEAR_FLAG_* of the header has the same value in the binding, and no two flags share a bit."""
    import ternary_weight_linear_fwd_b200 as bl
    flags = dict(re.findall(r"#define BITLINEAR_(FLAG_\w+) (0x[0-9a-fA-F]+)u", open(HEADER).read()))
    assert "FLAG_NM24_EXPAND" in flags and len(flags) >= 6
    for name, val in flags.items():
        assert getattr(bl, name) == int(val, 16), name
    vals = [int(v, 16) for v in flags.values()]
    assert all(v and (v & (v - 1)) == 0 for v in vals) and len(set(vals)) == len(vals)


def test_forward_q8_host_checks(L):
    """Codes-in entry: argument errors before any device work (fake addresses)."""
    import ternary_weight_linear_fwd_b200 as bl
    f = L.bitlinear_forward_q8
    f.restype = ctypes.c_int
    P, i32 = ctypes.c_void_p, ctypes.c_int32
    f.argtypes = [ctypes.POINTER(bl._Weights), P, i32, P, P, i32, P, P, P, ctypes.c_size_t, ctypes.c_uint32, P]
    q, g, rs, y = 0x10000, 0x20000, 0x30000, 0x40000
    w = _w(L)
    assert f(None, q, 256, g, rs, 4, y, None, None, 0, 0, None) == 1
    assert f(ctypes.byref(w), None, 256, g, rs, 4, y, None, None, 0, 0, None) == 1
    assert f(ctypes.byref(w), q, 256, g, None, 4, y, None, None, 0, 0, None) == 1
    assert f(ctypes.byref(w), q, 250, g, rs, 4, y, None, None, 0, 0, None) == 2   # ldq < K
    assert f(ctypes.byref(w), q, 264, g, rs, 0, y, None, None, 0, 0, None) == 2   # M = 0
    assert f(ctypes.byref(w), q + 8, 256, g, rs, 4, y, None, None, 0, 0, None) == 3
    assert f(ctypes.byref(w), q, 256, g, rs, 4, y, None, None, 0, 0x2, None) == 8  # no GEMV path


def test_relu2_glu_host_checks(L):
    """Gate/up with squared ReLU: argument errors come back before any device work (fake addresses)."""
    f = L.bitlinear_forward_relu2_glu
    f.restype = ctypes.c_int
    x, h = 0x30000, 0x40000
    wg, wu = _w(L), _w(L)
    assert f(None, ctypes.byref(wu), x, 1, h, None, 0, 0, None) == 1
    assert f(ctypes.byref(wg), None, x, 1, h, None, 0, 0, None) == 1
    assert f(ctypes.byref(wg), ctypes.byref(wu), None, 1, h, None, 0, 0, None) == 1
    assert f(ctypes.byref(wg), ctypes.byref(wu), x, 1, None, None, 0, 0, None) == 1
    other_n = _w(L, N=96)
    assert f(ctypes.byref(wg), ctypes.byref(other_n), x, 1, h, None, 0, 0, None) == 2   # N differs
    other_k = _w(L, K=512)
    assert f(ctypes.byref(wg), ctypes.byref(other_k), x, 1, h, None, 0, 0, None) == 2   # K differs
    assert f(ctypes.byref(wg), ctypes.byref(wu), x, 0, h, None, 0, 0, None) == 2        # M = 0
    assert f(ctypes.byref(wg), ctypes.byref(wu), x + 8, 1, h, None, 0, 0, None) == 3    # x not 16-byte aligned
    bad_p = _w(L, n=3, m=4, meta=0x50000)
    assert f(ctypes.byref(wg), ctypes.byref(bad_p), x, 1, h, None, 0, 0, None) == 4
    assert f(ctypes.byref(wg), ctypes.byref(wu), x, 1, h, None, 0, 0x100, None) == 8    # unknown flag
    assert f(ctypes.byref(wg), ctypes.byref(wu), x, 1, h, None, 0, 0x8, None) == 8      # no lookup-table path


def test_relu2_glu_workspace_bytes(L):
    q = L.bitlinear_forward_relu2_glu_workspace_bytes
    q.restype = ctypes.c_size_t
    q.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_uint32]
    assert q(0, 64, 256, 0) == 0
    for M, N, K in ((1, 6912, 2560), (2048, 6912, 2560), (300, 2000, 1032)):
        assert q(M, N, K, 0) >= 2 * M * N * 2 + L.bitlinear_forward_workspace_bytes(M, N, K, 0)
