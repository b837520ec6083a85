"""C-ABI checks that need no GPU: the library loads, exports every entry
point ``include/fp8fg.h`` declares, the Python binding uses the same names,
and argument validation answers synchronously before any CUDA work.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8fg.h")


def declared_functions():
    text = open(HEADER, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fp8_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    from fp8_fine_grained_online_b200 import _lib
    return _lib.lib


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("fp8_quantize_act_1x128", "fp8_quantize_weight_128x128", "fp8_blockscaled_gemm",
              "fp8_grouped_gemm", "fp8_dequantize", "fp8_status_string", "fp8_get_device_error"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_binding_covers_every_declared_symbol():
    import fp8_fine_grained_online_b200 as fp8
    from fp8_fine_grained_online_b200 import _lib
    for name in declared_functions():
        assert name in _lib.SIGNATURES, name
        assert callable(getattr(fp8, name)), name


def test_library_exports_nothing_else(L):
    """Hidden visibility: only the C ABI is exported."""
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", L._name], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert exported == set(declared_functions())


def test_status_strings(L):
    for code in range(10):
        s = L.fp8_status_string(code).decode()
        assert s.startswith("FP8_")
    assert L.fp8_status_string(99).decode() == "unknown fp8_status_t"


P = ctypes.c_void_p
A16 = P(0x10000)          # an aligned, never-dereferenced address
A8 = P(0x10008)


def act(L, x=A16, xt=0, M=4, K=128, ldx=128, q=A16, ldq=128, sa=A16, sm=1, skb=4):
    return L.fp8_quantize_act_1x128(x, xt, M, K, ldx, q, ldq, sa, sm, skb, None)


def test_act_argument_errors(L):
    assert act(L, xt=7) == 5                       # DTYPE
    assert act(L, K=100, ldx=128) == 2             # SHAPE: K % 128
    assert act(L, M=-1) == 2
    assert act(L, M=0, x=None, q=None, sa=None) == 0   # empty: no-op
    assert act(L, K=0, x=None, q=None, sa=None) == 0
    assert act(L, x=None) == 1                     # NULL
    assert act(L, sa=None) == 1
    assert act(L, ldx=64) == 4                     # LAYOUT: ldx < K
    assert act(L, skb=-1) == 4
    assert act(L, x=A8) == 3                       # ALIGN
    assert act(L, q=A8) == 3
    assert act(L, ldx=132) == 3                    # 132 bf16 = 264 B, not 16-B multiple
    assert act(L, ldq=136) == 3
    assert act(L, sa=P(0x10002)) == 3


def test_weight_argument_errors(L):
    def w(**kw):
        a = dict(w=A16, wt=0, K=128, N=256, ldw=256, q=A16, tr=1, ldq=128, sb=A16, skb=2, snb=1)
        a.update(kw)
        return L.fp8_quantize_weight_128x128(a["w"], a["wt"], a["K"], a["N"], a["ldw"], a["q"],
                                             a["tr"], a["ldq"], a["sb"], a["skb"], a["snb"], None)
    assert w(N=200, ldw=256) == 2
    assert w(K=0, w=None) == 0
    assert w(q=None) == 1
    assert w(tr=1, ldq=64) == 4                    # transposed q is [N, K]: ldq >= K
    assert w(tr=0, ldq=128) == 4                   # [K, N]: ldq >= N
    assert w(w=A8) == 3
    assert w(wt=3) == 5


def gemm(L, **kw):
    a = dict(a=A16, lda=256, sa=A16, sam=1, sakb=128, b=A16, ldb=256, bk=1, sb=A16, sbkb=2,
             sbnb=1, c=A16, ct=1, ldc=256, M=128, N=256, K=256)
    a.update(kw)
    return L.fp8_blockscaled_gemm(a["a"], a["lda"], a["sa"], a["sam"], a["sakb"], a["b"],
                                  a["ldb"], a["bk"], a["sb"], a["sbkb"], a["sbnb"], a["c"],
                                  a["ct"], a["ldc"], a["M"], a["N"], a["K"], None)


def test_gemm_argument_errors(L):
    assert gemm(L, ct=4) == 5
    assert gemm(L, K=200) == 2
    assert gemm(L, N=100) == 2
    assert gemm(L, M=0, a=None) == 0
    assert gemm(L, bk=0) == 4                      # only K-major B
    assert gemm(L, sb=None) == 1
    assert gemm(L, lda=128) == 4
    assert gemm(L, a=A8) == 3
    assert gemm(L, ldb=264) == 3
    assert gemm(L, ldc=260) == 3                   # 260 bf16 = 520 B


def test_grouped_argument_errors(L):
    def g(**kw):
        a = dict(a=A16, lda=256, sa=A16, sam=1, sakb=64, b=A16, ldb=256, sb=A16, sbg=4,
                 sbkb=2, sbnb=1, c=A16, ct=1, ldc=256, off=A16, G=4, M=64, N=256, K=256)
        a.update(kw)
        return L.fp8_grouped_gemm(a["a"], a["lda"], a["sa"], a["sam"], a["sakb"], a["b"],
                                  a["ldb"], a["sb"], a["sbg"], a["sbkb"], a["sbnb"], a["c"],
                                  a["ct"], a["ldc"], a["off"], a["G"], a["M"], a["N"], a["K"],
                                  None)
    assert g(G=0) == 2
    assert g(G=1025) == 2
    assert g(M=0) == 0
    assert g(off=None) == 1
    assert g(off=P(0x10001)) == 3
    assert g(sbg=-1) == 4


def test_valid_arguments_without_gpu_report_device_error(L):
    """With every argument valid, the next check is the device: no GPU here."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is visible")
    assert act(L) == 6
    assert gemm(L) == 6
    code = ctypes.c_int(0)
    assert L.fp8_get_device_error(None, ctypes.byref(code)) == 6
    assert L.fp8_set_wait_limit(0) == 6


def test_dequantize_argument_errors(L):
    vp = ctypes.c_void_p
    buf = ctypes.create_string_buffer(4096 + 16)
    base = (ctypes.addressof(buf) + 15) // 16 * 16
    p = vp(base)
    # q, rows, cols, ldq, s, s_r, s_c, tile_rows, out, out_type, ldo, stream
    assert L.fp8_dequantize(p, 4, 128, 128, p, 1, 1, 1, p, 5, 128, None) == 5      # dtype
    assert L.fp8_dequantize(p, 4, 100, 128, p, 1, 1, 1, p, 0, 128, None) == 2      # cols % 128
    assert L.fp8_dequantize(p, 4, 128, 128, p, 1, 1, 64, p, 0, 128, None) == 2     # tile_rows
    assert L.fp8_dequantize(p, -1, 128, 128, p, 1, 1, 1, p, 0, 128, None) == 2     # rows < 0
    assert L.fp8_dequantize(p, 0, 128, 128, None, 1, 1, 1, None, 0, 128, None) == 0  # empty: no-op
    assert L.fp8_dequantize(None, 4, 128, 128, p, 1, 1, 1, p, 0, 128, None) == 1   # null
    assert L.fp8_dequantize(p, 4, 128, 64, p, 1, 1, 1, p, 0, 128, None) == 4       # ldq < cols
    assert L.fp8_dequantize(p, 4, 128, 136, p, 1, 1, 1, p, 0, 128, None) == 3      # ldq % 16
    assert L.fp8_dequantize(vp(base + 8), 4, 128, 128, p, 1, 1, 1, p, 0, 128, None) == 3


def test_gemm_quant_argument_errors(L):
    vp = ctypes.c_void_p
    buf = ctypes.create_string_buffer(4096 + 16)
    base = (ctypes.addressof(buf) + 15) // 16 * 16
    p = vp(base)

    def call(qc=p, ldqc=128, sc=p, c=None, ldc=0, M=4, N=128, K=128):
        # a, lda, sa, sa_m, sa_kb, b, ldb, sb, sb_kb, sb_nb, qc, ldqc, sc, sc_m, sc_nb, c, ldc, M, N, K
        return L.fp8_blockscaled_gemm_quant(p, 128, p, 1, 1, p, 128, p, 1, 1, qc, ldqc, sc, 1, 1,
                                            c, ldc, M, N, K, None)
    assert call(N=100) == 2                 # N % 128
    assert call(K=0) == 2                   # empty contraction not supported here
    assert call(M=0, qc=None, sc=None) == 0  # empty: no-op
    assert call(qc=None) == 1
    assert call(sc=None) == 1
    assert call(ldqc=64) == 4               # ldqc < N
    assert call(ldqc=136) == 3              # ldqc % 16
    assert call(c=p, ldc=64) == 4           # ldc < N
    assert call(c=vp(base + 2), ldc=128) == 3


def test_gather_quant_argument_errors(L):
    vp = ctypes.c_void_p
    buf = ctypes.create_string_buffer(4096 + 16)
    base = (ctypes.addressof(buf) + 15) // 16 * 16
    p = vp(base)

    # x, x_type, src_rows, K, ldx, rows, R, q, ldq, sa, sa_m, sa_kb, stream
    def call(x=p, xt=0, T=4, K=128, ldx=128, rows=p, R=4, q=p, ldq=128, sa=p):
        return L.fp8_quantize_act_1x128_gather(x, xt, T, K, ldx, rows, R, q, ldq, sa, 1, 1, None)
    assert call(xt=7) == 5
    assert call(K=100) == 2
    assert call(R=-1) == 2
    assert call(R=0, x=None, rows=None, q=None, sa=None) == 0
    assert call(rows=None) == 1
    assert call(ldq=64) == 4
    assert call(ldx=132) == 3          # ldx * 2 bytes % 16
    assert call(rows=vp(base + 2)) == 3


def test_scatter_quant_argument_errors(L):
    vp = ctypes.c_void_p
    buf = ctypes.create_string_buffer(4096 + 32)
    base = (ctypes.addressof(buf) + 31) // 32 * 32
    p = vp(base)

    # x, x_type, T, K, ldx, dest, topk, q, R, ldq, sa, sa_m, sa_kb, stream
    def call(x=p, xt=0, T=4, K=128, ldx=128, dest=p, topk=2, q=p, R=8, ldq=128, sa=p, sm=1):
        return L.fp8_quantize_act_1x128_scatter(x, xt, T, K, ldx, dest, topk, q, R, ldq, sa, sm,
                                                1, None)
    assert call(xt=7) == 5
    assert call(xt=1) == 5                  # bf16 input only
    assert call(K=100) == 2
    assert call(T=-1) == 2
    assert call(topk=-1) == 2
    assert call(T=0, x=None, dest=None) == 0   # empty: no-op
    assert call(topk=0, dest=None) == 0
    assert call(dest=None) == 1
    assert call(q=None) == 1
    assert call(ldq=64) == 4
    assert call(ldx=64) == 4
    assert call(sm=-1) == 4
    assert call(q=vp(base + 16)) == 3       # codes leave as 32-byte stores
    assert call(ldq=144) == 3               # ldq % 32
    assert call(dest=vp(base + 2)) == 3
    assert call(x=vp(base + 8)) == 3


def test_act_128x1_argument_errors(L):
    # x, x_type, M, K, ldx, qt, ldq, st, st_k, st_mb, stream
    def call(x=A16, xt=0, M=256, K=128, ldx=128, qt=A16, ldq=256, st=A16, sk=2, smb=1):
        return L.fp8_quantize_act_128x1(x, xt, M, K, ldx, qt, ldq, st, sk, smb, None)
    assert call(xt=7) == 5
    assert call(M=200) == 2                        # M % 128 (the tile runs along M)
    assert call(K=100, ldx=128) == 2
    assert call(M=0, x=None, qt=None, st=None) == 0
    assert call(xt=1) == 5                         # bf16 input only
    assert call(qt=None) == 1
    assert call(ldq=128) == 4                      # qt is [K, M]: ldq >= M
    assert call(ldx=64) == 4
    assert call(smb=-1) == 4
    assert call(x=A8) == 3
    assert call(ldq=264) == 3
    assert call(st=P(0x10002)) == 3


def test_gemm_colscale_argument_errors(L):
    # a, lda, sa, sa_m, sa_kb, b, ldb, sb, sb_kb, c, c_type, ldc, M, N, K, stream
    def call(a=A16, sa=A16, b=A16, sb=A16, sbkb=256, c=A16, ct=1, ldc=256, M=128, N=256,
             K=256):
        return L.fp8_blockscaled_gemm_colscale(a, 256, sa, 2, 1, b, 256, sb, sbkb, c, ct, ldc, M,
                                               N, K, None)
    assert call(ct=4) == 5
    assert call(N=100) == 2
    assert call(K=200) == 2
    assert call(M=0, a=None) == 0
    assert call(sb=None) == 1
    assert call(sbkb=128) == 4                     # sb rows hold N values
    assert call(sbkb=258) == 3                     # 16-byte pieces of a row: stride % 4
    if not __import__("torch").cuda.is_available():
        assert call(sbkb=1, K=128) == 6            # one chunk: the row stride is unused
    assert call(sb=P(0x10004)) == 3
    assert call(ldc=260) == 3
