"""Pins for the CPU oracle: checks against what the pages and mathematics fix.

Each ``check_*`` takes the oracle as a namespace ``o`` so that
``test_oracle_pins.py`` can run it on the real oracle and on mutants with a
planted mistake (a dropped term, a wrong sign, a transposed operand); every
mutant must fail at least one check. None of these checks re-types the
oracle's own formula: they use brute-force loops, closed forms, invariants,
hand-worked examples and independent library routines.
"""
from __future__ import annotations

import itertools
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(*k):
    return np.random.default_rng(list(k) + [7])


# ------------------------------------------------------------------ helpers
def read_band_golden():
    rows = []
    with open(os.path.join(GOLDEN, "band_sizes.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            nums = [int(t) for t in line.split()]
            rows.append((nums[0], nums[1], nums[2:]))
    return rows


def brute_force_bands(L, G):
    """All compositions of L into G positive parts that are as equal as possible
    (max - min <= 1) with the larger parts first; the rule admits exactly one."""
    found = []
    for cuts in itertools.combinations(range(1, L), G - 1):
        edges = (0,) + cuts + (L,)
        sizes = [edges[i + 1] - edges[i] for i in range(G)]
        if max(sizes) - min(sizes) <= 1 and all(sizes[i] >= sizes[i + 1] for i in range(G - 1)):
            found.append(sizes)
    return found


def band_sizes_by_counting(L, G):
    """Same rule, computed without division: deal layers one by one to the band
    that currently holds the fewest (earliest band on ties), then sort."""
    counts = [0] * G
    for _ in range(L):
        b = min(range(G), key=lambda j: (counts[j], j))
        counts[b] += 1
    return counts


def raises(fn, exc=Exception):
    try:
        fn()
    except exc:
        return True
    return False


# --------------------------------------------------------------- round_to
def check_round(o):
    import torch
    rng = _rng(1)
    x32 = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(2000) * 1e-38).astype(np.float32),  # f32 subnormal / bf16 tiny
        (rng.standard_normal(2000) * 1e37).astype(np.float32),
        np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 2 ** -133, 3 * 2 ** -134,
                  3.3895314e38, 0.0, -0.0], dtype=np.float32),
    ])
    ref = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()
    got = o.round_to(x32.astype(np.float64), "bf16")
    assert np.array_equal(got, ref, equal_nan=True), "bf16 rounding differs from torch"
    # hand-worked ties: 1 + 2^-8 sits halfway between 1 and 1 + 2^-7 -> even (1.0)
    assert o.round_to(np.array([1 + 2 ** -8]), "bf16")[0] == 1.0
    assert o.round_to(np.array([1 + 3 * 2 ** -8]), "bf16")[0] == 1 + 2 ** -6
    x64 = np.concatenate([rng.standard_normal(20000), rng.standard_normal(1000) * 1e-42])
    assert np.array_equal(o.round_to(x64, "f32"), x64.astype(np.float32).astype(np.float64))


# --------------------------------------------------------------- bands
def check_bands(o):
    for L, G, sizes in read_band_golden():
        assert list(o.band_sizes(L, G)) == sizes, (L, G)
    for L in range(1, 13):
        for G in range(1, L + 1):
            bf = brute_force_bands(L, G)
            assert len(bf) == 1
            assert list(o.band_sizes(L, G)) == bf[0] == band_sizes_by_counting(L, G), (L, G)
    for L, G in [(26, 4), (60, 15), (26, 7), (60, 7), (4, 2)]:
        sizes = list(o.band_sizes(L, G))
        assert sum(sizes) == L and max(sizes) - min(sizes) <= 1
        assert sizes == sorted(sizes, reverse=True)
        assert sizes == band_sizes_by_counting(L, G)
        bol, start = o.band_index(L, G)
        assert list(start) == [0] + list(itertools.accumulate(sizes))
        assert all(start[bol[i]] <= i < start[bol[i] + 1] for i in range(L))
        assert list(bol) == sorted(bol)
    for L, G in [(4, 0), (4, 5), (0, 1), (3, -1)]:
        assert raises(lambda: o.band_sizes(L, G), ValueError), (L, G)


# --------------------------------------------------------------- band mean
def check_band_mean(o):
    rng = _rng(2)
    L, O, I = 7, 3, 5
    w = rng.standard_normal((L, O, I))
    for G in (1, 2, 3, 7):
        sizes = brute_force_bands(L, G)[0]
        got = o.band_mean(w, G)
        first = 0
        for b, n in enumerate(sizes):
            for r in range(O):
                for c in range(I):
                    acc = 0.0
                    for layer in range(first, first + n):
                        acc += float(w[layer, r, c])
                    assert math.isclose(got[b, r, c], acc / n, rel_tol=1e-13, abs_tol=1e-15)
            first += n
    # passthrough: one layer per band returns the weights bit for bit
    assert np.array_equal(o.band_mean(w, L), w)
    w32 = rng.standard_normal((L, O, I)).astype(np.float32).astype(np.float64)
    assert np.array_equal(o.band_mean(w32, L, "f32"), w32)
    # linearity and the all-equal case
    assert np.allclose(o.band_mean(3.0 * w, 2), 3.0 * o.band_mean(w, 2), rtol=1e-14, atol=0)
    same = np.broadcast_to(w[0], (L, O, I))
    assert np.allclose(o.band_mean(same, 3), np.broadcast_to(w[0], (3, O, I)), rtol=1e-15, atol=0)


# --------------------------------------------------------------- row scale
def check_row_scale(o):
    rng = _rng(3)
    O, I = 6, 9
    w = rng.standard_normal((O, I))
    W0 = rng.standard_normal((O, I))
    s = o.row_scale(w, W0)
    for r in range(O):
        ls = np.linalg.lstsq(W0[r][:, None], w[r], rcond=None)[0][0]
        assert math.isclose(s[r], ls, rel_tol=1e-12)
        best = np.sum((w[r] - s[r] * W0[r]) ** 2)
        for d in (1e-3, -1e-3, 1e-1, -1e-1):
            assert np.sum((w[r] - (s[r] + d) * W0[r]) ** 2) >= best
    # scale covariance: W0 -> c W0 gives s -> s / c
    assert np.allclose(o.row_scale(w, 4.0 * W0), s / 4.0, rtol=1e-13, atol=0)
    # exact multiple and passthrough
    assert np.allclose(o.row_scale(2.5 * W0, W0), 2.5, rtol=1e-14, atol=0)
    assert np.all(o.row_scale(w, w) == 1.0)
    # hand example: w = (1, 2), W0 = (1, 1) -> (1 + 2) / (1 + 1) = 1.5
    assert o.row_scale(np.array([[1.0, 2.0]]), np.array([[1.0, 1.0]]))[0] == 1.5
    # a zero row of W0 gets s = 0 (minimum-norm least squares)
    W0z = W0.copy()
    W0z[2] = 0
    sz = o.row_scale(w, W0z)
    assert sz[2] == 0.0 and np.allclose(np.delete(sz, 2), np.delete(s, 2), rtol=1e-15, atol=0)
    pinv = np.linalg.pinv(W0z[2][:, None]) @ w[2]
    assert pinv[0] == 0.0


# --------------------------------------------------------------- residual
def check_residual(o):
    rng = _rng(4)
    O, I = 5, 8
    w = rng.standard_normal((O, I))
    W0 = rng.standard_normal((O, I))
    s = o.row_scale(w, W0)
    R = o.residual(w, W0, s)
    # normal equation: the residual is orthogonal to its W0 row
    for r in range(O):
        assert abs(np.dot(R[r], W0[r])) <= 1e-12 * np.linalg.norm(w[r]) * np.linalg.norm(W0[r])
    # w = diag(s) W0 + R
    back = np.diag(s) @ W0 + R
    assert np.allclose(back, w, rtol=0, atol=1e-14)
    # hand example: w = (1, 2), W0 = (1, 0), s = 1 -> R = (0, 2)
    assert np.array_equal(o.residual(np.array([[1.0, 2.0]]), np.array([[1.0, 0.0]]), np.array([1.0])),
                          np.array([[0.0, 2.0]]))
    # passthrough: zero exactly
    assert np.all(o.residual(w, w, o.row_scale(w, w)) == 0.0)


# --------------------------------------------------------------- reconstruct
def check_reconstruct(o):
    rng = _rng(5)
    O, I, r = 4, 6, 3
    s = rng.standard_normal(O)
    W0 = rng.standard_normal((O, I))
    U = rng.standard_normal((O, r))
    V = rng.standard_normal((I, r))
    got = o.reconstruct(s, W0, U, V)
    for a in range(O):
        for b in range(I):
            acc = s[a] * W0[a, b]
            for j in range(r):
                acc += U[a, j] * V[b, j]
            assert math.isclose(got[a, b], acc, rel_tol=1e-12, abs_tol=1e-13)
    # rank 0: a pure scaled shared block
    z = o.reconstruct(s, W0, np.zeros((O, 0)), np.zeros((I, 0)))
    assert np.allclose(z, np.diag(s) @ W0, rtol=1e-15, atol=0)
    # passthrough: s = 1, U = V = 0 returns the weight bit for bit
    assert np.array_equal(o.reconstruct(np.ones(O), W0, np.zeros((O, r)), np.zeros((I, r))), W0)


# --------------------------------------------------------------- frobenius
def check_frob(o):
    rng = _rng(6)
    A = rng.standard_normal((7, 5))
    assert o.frob_error(A, A) == 0.0
    assert math.isclose(o.frob_error(A, np.zeros_like(A)), 1.0, rel_tol=1e-15)
    for eps in (1e-3, -0.25, 2.0):
        assert math.isclose(o.frob_error(A, (1 + eps) * A), abs(eps), rel_tol=1e-12)
    # hand example: A = [[1,2],[2,1]], B = [[1,2],[2,2]] -> 1 / sqrt(10)
    assert math.isclose(o.frob_error(np.array([[1.0, 2.0], [2.0, 1.0]]),
                                     np.array([[1.0, 2.0], [2.0, 2.0]])), 1 / math.sqrt(10), rel_tol=1e-15)
    # not symmetric in its arguments: normalised by the original
    assert math.isclose(o.frob_error(np.array([[3.0, 4.0]]), np.array([[0.0, 0.0]])), 1.0)
    assert math.isclose(o.frob_error(np.array([[6.0, 8.0]]), np.array([[3.0, 4.0]])), 0.5)
    # the degenerate original
    Z = np.zeros((2, 2))
    assert o.frob_error(Z, Z) == 0.0
    assert o.frob_error(Z, np.ones((2, 2))) == float("inf")


def check_frob_partials(o):
    """The two sums a row-sharded error combines: hand values, the ratio they
    give is frob_error's, and row blocks add up exactly on integer data."""
    assert o.frob_partials(np.array([[3.0, 4.0]]), np.array([[0.0, 0.0]])) == (25.0, 25.0)
    assert o.frob_partials(np.array([[1.0, 2.0], [2.0, 1.0]]), np.array([[1.0, 2.0], [2.0, 2.0]])) == (1.0, 10.0)
    assert o.frob_partials(np.array([[6.0, 8.0]]), np.array([[3.0, 4.0]])) == (25.0, 100.0)
    rng = _rng(16)
    A = rng.standard_normal((9, 6))
    B = A + 0.1 * rng.standard_normal((9, 6))
    assert o.frob_from_partials(*o.frob_partials(A, B)) == o.frob_error(A, B)
    assert o.frob_from_partials(0.0, 0.0) == 0.0 and o.frob_from_partials(2.0, 0.0) == float("inf")
    # brute-force sums of squares by loops
    num = sum((A[i, j] - B[i, j]) ** 2 for i in range(9) for j in range(6))
    den = sum(A[i, j] ** 2 for i in range(9) for j in range(6))
    n2, d2 = o.frob_partials(A, B)
    assert math.isclose(n2, num, rel_tol=1e-14) and math.isclose(d2, den, rel_tol=1e-14)
    # small integers: every partial sum is exact, so any split of the rows
    # into blocks adds up to the whole bit for bit
    Ai = rng.integers(-50, 50, size=(11, 7)).astype(np.float64)
    Bi = rng.integers(-50, 50, size=(11, 7)).astype(np.float64)
    whole = o.frob_partials(Ai, Bi)
    for cuts in ([5], [1, 8], [3, 4, 9]):
        blocks = np.split(np.arange(11), cuts)
        parts = [o.frob_partials(Ai[b], Bi[b]) for b in blocks]
        assert (sum(p[0] for p in parts), sum(p[1] for p in parts)) == whole


# --------------------------------------------------------------- forward
def check_forward(o):
    import torch
    rng = _rng(7)
    M, O, I, r = 3, 4, 5, 2
    X = rng.standard_normal((M, I))
    s = rng.standard_normal(O)
    W0 = rng.standard_normal((O, I))
    U = rng.standard_normal((O, r))
    V = rng.standard_normal((I, r))
    Y = o.linear_forward(X, W0, s, U, V)
    for m in range(M):
        for n in range(O):
            acc = 0.0
            for k in range(I):
                wk = s[n] * W0[n, k]
                for j in range(r):
                    wk += U[n, j] * V[k, j]
                acc += X[m, k] * wk
            assert math.isclose(Y[m, n], acc, rel_tol=1e-12, abs_tol=1e-12)
    # equals the projection by the explicitly rebuilt weight (torch's linear)
    Wr = np.diag(s) @ W0 + U @ V.T
    ref = torch.nn.functional.linear(torch.from_numpy(X), torch.from_numpy(Wr)).numpy()
    assert np.allclose(Y, ref, rtol=1e-12, atol=1e-12)
    # s = 1, rank 0: the textbook X W^T
    Y0 = o.linear_forward(X, W0, np.ones(O), np.zeros((O, 0)), np.zeros((I, 0)))
    ref0 = torch.nn.functional.linear(torch.from_numpy(X), torch.from_numpy(W0)).numpy()
    assert np.allclose(Y0, ref0, rtol=1e-13, atol=1e-13)
    # a large rank term: each part matters on its own
    U2, V2 = 10 * U, 10 * V
    Ya = o.linear_forward(X, W0, s, U2, V2)
    Yb = o.linear_forward(X, W0, s, np.zeros_like(U2), np.zeros_like(V2))
    assert np.allclose(Ya - Yb, X @ (U2 @ V2.T).T, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------- svd
def check_svd(o):
    rng = _rng(8)
    O, I = 9, 7
    R = rng.standard_normal((O, I))
    eig = np.sort(np.linalg.eigvalsh(R.T @ R))[::-1]  # squared singular values
    for r in (0, 1, 3, 7):
        U, V = o.truncated_svd(R, r)
        assert U.shape == (O, r) and V.shape == (I, r)
        err2 = np.sum((R - U @ V.T) ** 2)
        assert math.isclose(err2, float(np.sum(eig[r:])), rel_tol=1e-9, abs_tol=1e-10)
        if r:
            assert np.allclose(V.T @ V, np.eye(r), atol=1e-12)          # orthonormal right factor
            assert np.allclose(np.sum(U ** 2, axis=0), eig[:r], rtol=1e-9)  # U absorbs sigma
    U, V = o.truncated_svd(R, I)
    assert np.allclose(U @ V.T, R, atol=1e-12)


def check_randomized_svd(o):
    """randomized_svd: exact on matrices of rank <= r; with a square test
    matrix (k = min(O, I)) it is the truncated SVD, so Eckart-Young fixes its
    error; on a decaying spectrum two subspace iterations land within 1% of
    the optimum; V is orthonormal and U's column norms are B's singular
    values; rank 0 gives empty factors."""
    rng = _rng(21)
    O, I, r = 40, 30, 5
    # exact rank r: recovered to rounding whatever the draw
    R = rng.standard_normal((O, r)) @ rng.standard_normal((r, I))
    omega = rng.standard_normal((r + 4, I))
    U, V = o.randomized_svd(R, r, omega)
    assert U.shape == (O, r) and V.shape == (I, r)
    assert np.allclose(U @ V.T, R, atol=1e-10 * np.abs(R).max())
    # k = I: the sample spans everything, so the result is the truncated SVD
    R = rng.standard_normal((O, I))
    eig = np.sort(np.linalg.eigvalsh(R.T @ R))[::-1]
    U, V = o.randomized_svd(R, r, rng.standard_normal((I, I)))
    err2 = np.sum((R - U @ V.T) ** 2)
    assert math.isclose(err2, float(np.sum(eig[r:])), rel_tol=1e-9)
    assert np.allclose(V.T @ V, np.eye(r), atol=1e-12)
    assert np.allclose(np.sum(U ** 2, axis=0), eig[:r], rtol=1e-9)
    # decaying spectrum, k = r + 6, two power iterations: near-optimal
    A, _ = np.linalg.qr(rng.standard_normal((O, I)))
    Bq, _ = np.linalg.qr(rng.standard_normal((I, I)))
    sig = 0.7 ** np.arange(I)
    R = (A * sig) @ Bq.T
    U, V = o.randomized_svd(R, r, rng.standard_normal((r + 6, I)), power_iters=2)
    opt = float(np.sum(sig[r:] ** 2))
    err2 = float(np.sum((R - U @ V.T) ** 2))
    assert opt <= err2 * (1 + 1e-9) and err2 <= 1.01 * opt
    U0, V0 = o.randomized_svd(R, 0, rng.standard_normal((4, I)))
    assert U0.shape == (O, 0) and V0.shape == (I, 0)


def check_nvfp4(o):
    """NVFP4: the E2M1 and E4M3 grids, round-to-nearest-even with saturation
    (E4M3 against torch's float8_e4m3fn cast), exact round trip for weights on
    the grid, the error bound, zero blocks, packing order and the byte count."""
    import torch
    e2, e4 = o.e2m1_values(), o.e4m3_values()
    assert list(e2) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert len(e4) == 127 and e4[126] == 448.0 and e4[1] == 2.0 ** -9 and e4[56] == 1.0 and e4[8] == 2.0 ** -6
    # E4M3 rounding of in-range values equals torch's cast (RNE), ties included
    x = np.concatenate([np.linspace(0, 448, 20001), e4[1:] * (1 + 2.0 ** -4), (e4[1:] + e4[:-1]) / 2])
    x = x[x <= 448].astype(np.float32)
    codes = o._grid_round(x, e4) if hasattr(o, "_grid_round") else None
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert codes is not None and np.array_equal(e4[codes], ref)
    # E2M1 ties go to the even code; above 6 saturates
    xs = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, 100.0, 0.26, 0.74], dtype=np.float32)
    assert list(e2[o._grid_round(xs, e2)]) == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, 6.0, 6.0, 0.5, 0.5]
    rng = _rng(31)
    # weights on the grid come back exactly: every block holds its max 6*s*g
    g = np.float32(2.0 ** -12)
    O, I = 3, 64
    sq = rng.integers(8, 127, size=(O, I // 16))
    sq[0, 0] = 126  # the tensor max sets g
    q = e2[rng.integers(0, 8, size=(O, I))] * rng.choice([-1.0, 1.0], size=(O, I))
    q[:, ::16] = 6.0
    W = (q * np.repeat(e4[sq], 16, axis=1) * g).astype(np.float32)
    c, sc, gg = o.nvfp4_quantize(W)
    assert gg == g and np.array_equal(sc, sq.astype(np.uint8))
    assert np.array_equal(o.nvfp4_dequantize(c, sc, gg), W.astype(np.float64))
    assert c.shape == (O, I // 2) and c.dtype == np.uint8
    assert (c[0, 0] & 15) == 7 and (int(q[0, 1] < 0) << 3 | int(np.where(e2 == abs(q[0, 1]))[0][0])) == c[0, 0] >> 4
    # random weights: each element within a quarter of its block's max
    W = (rng.standard_normal((8, 128)) * 0.02).astype(np.float32)
    W[2, 16:32] = 0.0
    c, sc, gg = o.nvfp4_quantize(W)
    D = o.nvfp4_dequantize(c, sc, gg)
    bmax = np.repeat(np.abs(W).reshape(8, 8, 16).max(axis=2), 16, axis=1)
    assert np.all(np.abs(D - W) <= 0.25 * bmax + 1e-30)
    assert np.all(D[2, 16:32] == 0) and sc[2, 1] == 0
    assert (c.nbytes + sc.nbytes) / W.size == 0.5625  # 3.56x fewer bytes than bf16
    z, zs, zg = o.nvfp4_quantize(np.zeros((2, 32), np.float32))
    assert zg == 0 and not z.any() and not zs.any()
    # the forward with an NVFP4 shared block is the forward with its dequantized values
    X = rng.standard_normal((3, 128))
    s_, U, V = rng.standard_normal(8), rng.standard_normal((8, 4)), rng.standard_normal((128, 4))
    assert np.allclose(o.linear_forward_nvfp4(X, c, sc, gg, s_, U, V), o.linear_forward(X, D, s_, U, V),
                       rtol=1e-13, atol=1e-13)


# --------------------------------------------------------------- pipeline
def check_decompose(o):
    rng = _rng(9)
    L, O, I = 4, 6, 10
    w = (rng.standard_normal((O, I)) * 0.02 + rng.standard_normal((L, O, I)) * 0.005)
    w = w.astype(np.float32).astype(np.float64)
    # passthrough G = L: W0 = weight, s = 1, residual = 0, reconstruction exact
    d = o.decompose_family(w, L, 2, "f32")
    assert np.array_equal(d["W0"], w)
    assert np.all(d["s"] == 1.0) and np.all(d["R"] == 0.0)
    for layer in range(L):
        rec = o.reconstruct(d["s"][layer], d["W0"][layer], d["U"][layer], d["V"][layer], "f32")
        assert np.array_equal(rec, w[layer])
        assert o.frob_error(w[layer], rec) == 0.0
    # G < L with full rank rebuilds each layer (fp64)
    d = o.decompose_family(w, 2, min(O, I))
    for layer in range(L):
        b = d["band_of_layer"][layer]
        rec = o.reconstruct(d["s"][layer], d["W0"][b], d["U"][layer], d["V"][layer])
        assert o.frob_error(w[layer], rec) < 1e-12


def check_frob_statistics(o):
    """Sanity of the weight model: at G=1, rank 0, the error is close to
    0.005 * sqrt(1 - 1/L) / sqrt(0.02^2 + 0.005^2) (about 0.238 at L=26),
    slightly less because s absorbs part of the noise."""
    rng = np.random.default_rng(11)
    L, O, I = 26, 48, 256
    base = rng.standard_normal((O, I)) * 0.02
    w = base + rng.standard_normal((L, O, I)) * 0.005
    d = o.decompose_family(w, 1, 0)
    errs = [o.frob_error(w[i], o.reconstruct(d["s"][i], d["W0"][0], d["U"][i], d["V"][i]))
            for i in range(L)]
    expect = 0.005 * math.sqrt(1 - 1 / L) / math.sqrt(0.02 ** 2 + 0.005 ** 2)
    assert 0.9 * expect < float(np.mean(errs)) <= expect * 1.01


def check_gelu(o):
    """gelu_tanh: torch's tanh-form GELU, the odd-part identity
    gelu(x) - gelu(-x) = x, its limits, and closeness to the erf form."""
    import torch
    from scipy.special import erf
    x = np.linspace(-8.0, 8.0, 4001)
    g = o.gelu_tanh(x)
    ref = torch.nn.functional.gelu(torch.from_numpy(x), approximate="tanh").numpy()
    assert np.allclose(g, ref, rtol=1e-12, atol=1e-13)
    assert np.allclose(g - o.gelu_tanh(-x), x, rtol=0, atol=1e-12)
    assert o.gelu_tanh(np.array([0.0]))[0] == 0.0
    assert abs(o.gelu_tanh(np.array([30.0]))[0] - 30.0) < 1e-12
    assert abs(o.gelu_tanh(np.array([-30.0]))[0]) < 1e-12
    exact = 0.5 * x * (1.0 + erf(x / np.sqrt(2.0)))
    assert np.max(np.abs(g - exact)) < 1e-3  # the approximation's known accuracy
    assert np.max(np.abs(g - exact)) > 1e-5  # ... and it is the tanh form, not the erf one


def check_gate_up(o):
    """gate_up_forward against loops over the explicitly rebuilt weights and
    torch's tanh-form GELU: gelu(X·W_gateᵀ) ⊙ (X·W_upᵀ)."""
    import torch
    rng = _rng(11)
    M, O, I, r = 3, 4, 5, 2
    X = rng.standard_normal((M, I))
    gate = (rng.standard_normal((O, I)), rng.standard_normal(O), rng.standard_normal((O, r)),
            rng.standard_normal((I, r)))
    up = (rng.standard_normal((O, I)), rng.standard_normal(O), rng.standard_normal((O, r)),
          rng.standard_normal((I, r)))
    Y = o.gate_up_forward(X, gate, up)
    Wg = np.diag(gate[1]) @ gate[0] + gate[2] @ gate[3].T
    Wu = np.diag(up[1]) @ up[0] + up[2] @ up[3].T
    for m in range(M):
        for n in range(O):
            g = sum(X[m, k] * Wg[n, k] for k in range(I))
            u = sum(X[m, k] * Wu[n, k] for k in range(I))
            act = torch.nn.functional.gelu(torch.tensor(g, dtype=torch.float64), approximate="tanh").item()
            assert math.isclose(Y[m, n], act * u, rel_tol=1e-12, abs_tol=1e-12)
    # the activation applies to the gate only: swapping the roles changes Y
    assert not np.allclose(Y, o.gate_up_forward(X, up, gate))


ALL_CHECKS = [check_gelu, check_gate_up, check_randomized_svd, check_nvfp4, check_round, check_bands, check_band_mean, check_row_scale, check_residual,
              check_reconstruct, check_frob, check_frob_partials, check_forward, check_svd, check_decompose,
              check_frob_statistics]
