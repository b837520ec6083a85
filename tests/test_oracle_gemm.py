"""Pins for the oracle's block-scaled GEMM references (CPU only).

Pins: brute force against numpy's fp64 matmul of the dequantized operands
(an independent library routine), an integer closed form compared bit for
bit, the single-chunk case reducing to one scaled plain GEMM, and
consistency of the entry-sampled and grouped forms with the full one.
"""
import numpy as np
import pytest
import torch

from synth import normal, scale_outliers


def quantized_pair(orc, M, N, K, seed, b_kmajor=True):
    x = normal((M, K), 1.0, seed, "cpu", torch.float32)
    scale_outliers(x, 0.02, 50.0, seed + 1)
    w = normal((K, N), 0.02, seed + 2, "cpu", torch.float32)
    x, w = x.numpy(), w.numpy()
    qa, sa = orc.quantize_act_1x128(x)
    qb, sb = orc.quantize_weight_128x128(w, transpose_out=b_kmajor)
    return x, w, qa, sa, qb, sb


@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (5, 256, 256), (130, 128, 384),
                                   (64, 384, 256)])
@pytest.mark.parametrize("b_kmajor", [True, False])
def test_gemm_ref_brute_force(orc, M, N, K, b_kmajor):
    x, w, qa, sa, qb, sb = quantized_pair(orc, M, N, K, 1000 + M + N + K, b_kmajor)
    C, T = orc.gemm_ref(qa, sa, qb, sb, b_kmajor=b_kmajor)
    A = orc.dequantize(qa, sa, 1, 128)
    Bkn = orc.dequantize(qb.T if b_kmajor else qb, sb, 128, 128)
    ref = A @ Bkn
    assert np.all(np.abs(C - ref) <= 1e-12 * T)
    assert np.allclose(T, np.abs(A) @ np.abs(Bkn), rtol=1e-12, atol=0)
    assert np.all(T >= np.abs(C))


def test_gemm_ref_integer_closed_form_bit_exact(orc):
    """Every tile holds +448 and small integers that are E4M3 codes, so all
    scales are 1 and every product and sum is an exact integer."""
    rng = np.random.default_rng(3)
    M, N, K = 40, 256, 384
    a = rng.integers(-8, 9, size=(M, K)).astype(np.float32)
    b = rng.integers(-8, 9, size=(K, N)).astype(np.float32)
    a[:, ::128] = 448.0
    for kb in range(K // 128):
        for nb in range(N // 128):
            b[kb * 128, nb * 128] = 448.0
    qa, sa = orc.quantize_act_1x128(a)
    qb, sb = orc.quantize_weight_128x128(b, transpose_out=True)
    assert np.all(sa == 1.0) and np.all(sb == 1.0)
    C, _ = orc.gemm_ref(qa, sa, qb, sb, want_t=False)
    exact = a.astype(np.int64) @ b.astype(np.int64)
    assert np.array_equal(C, exact.astype(np.float64))


def test_gemm_ref_single_chunk_is_scaled_plain_gemm(orc):
    """K = 128: C = sa[m] * sb[nb] * (dec(qa) @ dec(qb))."""
    x, w, qa, sa, qb, sb = quantized_pair(orc, 16, 256, 128, 77)
    C, T = orc.gemm_ref(qa, sa, qb, sb)
    P = orc.e4m3_decode(qa) @ orc.e4m3_decode(qb).T          # exact: integers x 2^-18
    scale = sa[:, 0:1].astype(np.float64) * np.repeat(sb[0].astype(np.float64), 128)[None, :]
    # fp64 rounding of 128 products and sums: far below 1e-13 of sum |terms|
    assert np.all(np.abs(C - scale * P) <= 1e-13 * T)


def test_gemm_ref_scale_indexing_dgrad_orientation(orc):
    """B stored [K][N] with its scales read transposed ([nb][kb]) gives the same
    result as the [N][K] copy with scales [kb][nb]."""
    x, w, qa, sa, qb, sb = quantized_pair(orc, 8, 256, 384, 88, b_kmajor=False)
    C0, _ = orc.gemm_ref(qa, sa, qb, sb, b_kmajor=False)
    C1, _ = orc.gemm_ref(qa, sa, np.ascontiguousarray(qb.T), sb, b_kmajor=True)
    C2, _ = orc.gemm_ref(qa, sa, np.ascontiguousarray(qb.T), np.ascontiguousarray(sb.T),
                         b_kmajor=True, sb_transposed=True)
    assert np.array_equal(C0, C1) and np.array_equal(C1, C2)


def test_gemm_ref_entries_match_full(orc):
    x, w, qa, sa, qb, sb = quantized_pair(orc, 50, 256, 256, 99)
    C, T = orc.gemm_ref(qa, sa, qb, sb)
    rng = np.random.default_rng(0)
    rows = rng.integers(0, 50, 300)
    cols = rng.integers(0, 256, 300)
    c, t = orc.gemm_ref_entries(qa, sa, qb, sb, rows, cols)
    assert np.array_equal(c, C[rows, cols]) and np.array_equal(t, T[rows, cols])


def test_grouped_ref_matches_per_group(orc):
    rng = np.random.default_rng(1)
    G, N, K = 5, 128, 256
    sizes = [3, 0, 130, 1, 0]
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    total = int(off[-1])
    x = normal((total, K), 1.0, 555, "cpu", torch.float32).numpy()
    qa, sa = orc.quantize_act_1x128(x)
    qbs, sbs = [], []
    for g in range(G):
        w = normal((K, N), 0.02, 600 + g, "cpu", torch.float32).numpy()
        q, s = orc.quantize_weight_128x128(w, transpose_out=True)
        qbs.append(q)
        sbs.append(s)
    qb, sb = np.stack(qbs), np.stack(sbs)
    C, T = orc.grouped_gemm_ref(qa, sa, qb, sb, off)
    for g in range(G):
        r0, r1 = off[g], off[g + 1]
        if r1 == r0:
            continue
        Cg, Tg = orc.gemm_ref(qa[r0:r1], sa[r0:r1], qb[g], sb[g])
        assert np.array_equal(C[r0:r1], Cg) and np.array_equal(T[r0:r1], Tg)


def test_gemm_exact_matches_numpy(orc):
    x = normal((20, 300), 1.0, 5, "cpu", torch.float32).numpy()
    w = normal((300, 70), 1.0, 6, "cpu", torch.float32).numpy()
    E = orc.gemm_exact(x, w)
    assert np.allclose(E, x.astype(np.float64) @ w.astype(np.float64), rtol=1e-12, atol=1e-12)
    xb = normal((7, 256), 1.0, 7, "cpu", torch.bfloat16)
    bits = xb.view(torch.int16).numpy().view(np.uint16)
    E2 = orc.gemm_exact(bits, w[:256])
    assert np.allclose(E2, xb.double().numpy() @ w[:256].astype(np.float64), rtol=1e-12)


def test_quantized_gemm_close_to_exact(orc):
    """Sanity: fine-grained FP8 keeps the product within a few percent."""
    x, w, qa, sa, qb, sb = quantized_pair(orc, 64, 256, 512, 123)
    C, _ = orc.gemm_ref(qa, sa, qb, sb, want_t=False)
    E = orc.gemm_exact(x, w)
    rel = np.linalg.norm(C - E) / np.linalg.norm(E)
    assert rel < 0.05


def test_colscale_reduces_to_block_scales(orc):
    """Per-column B scales that are equal within each 128-column block give
    the block-scaled reference (a pinned function)."""
    rng = np.random.default_rng(21)
    I, N, K = 64, 256, 384
    qa = rng.integers(0, 0x7E, (I, K)).astype(np.uint8)
    qb = rng.integers(0, 0x7E, (N, K)).astype(np.uint8)
    sa = rng.uniform(0.5, 2, (I, K // 128)).astype(np.float32)
    sb_blk = rng.uniform(0.5, 2, (K // 128, N // 128)).astype(np.float32)
    sb_cols = np.repeat(sb_blk.T, 128, axis=0)              # [N, K/128]
    C1, T1 = orc.gemm_ref_colscale(qa, sa, qb, sb_cols)
    C2, T2 = orc.gemm_ref(qa, sa, qb, sb_blk)
    np.testing.assert_allclose(C1, C2, rtol=0, atol=1e-9 * np.max(T2))
    np.testing.assert_allclose(T1, T2, rtol=1e-12)


def test_colscale_closed_form_integers(orc):
    """E4M3 small integers with power-of-two scales: every product and sum is
    an exact integer multiple of a power of two, so C is known exactly."""
    I, N, K = 8, 256, 256
    codes = {1.0: 0x38, 2.0: 0x40, 3.0: 0x44, -1.0: 0xB8}
    rng = np.random.default_rng(22)
    va = rng.choice(list(codes), (I, K))
    vb = rng.choice(list(codes), (N, K))
    qa = np.vectorize(codes.get)(va).astype(np.uint8)
    qb = np.vectorize(codes.get)(vb).astype(np.uint8)
    sa = np.exp2(rng.integers(-3, 3, (I, K // 128))).astype(np.float32)
    sb = np.exp2(rng.integers(-3, 3, (N, K // 128))).astype(np.float32)
    C, _ = orc.gemm_ref_colscale(qa, sa, qb, sb)
    ref = np.zeros((I, N))
    for kb in range(K // 128):
        blk = slice(kb * 128, (kb + 1) * 128)
        ref += (va[:, blk] * sa[:, kb:kb + 1]) @ (vb[:, blk] * sb[:, kb:kb + 1]).T
    assert np.array_equal(C, ref)
