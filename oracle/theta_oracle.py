"""Plain fp64 CPU oracle for the theta-bundle projection path.

TEST INFRASTRUCTURE ONLY. This module is the independent checker for the GPU
library: only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline leg may import it. The product path never calls it, and it shares no
code with the CUDA implementation (it imports neither torch nor the library).

Every function is the definition from the pages written out with numpy in
float64, no blocking, no fusion, no reordering beyond what the definition
states. Inputs arrive as float32 arrays whose values are exact in their
storage dtype (f32 or bf16); they are upcast exactly to float64. Results that
the GPU stores in a narrower dtype are rounded once, round-to-nearest-even,
by ``round_to``.

Sources (page title -- section):
  * "Banded sharing" -- How layers map to bands: G contiguous bands, as equal
    as possible, earlier bands take the remainder.
  * "The theta bundle" -- table of components (W0 [out,in], s [out],
    U [out,rank], V [in,rank]); the approximation weight ~ diag(s)·W0 + U·Vᵀ;
    Analytic decomposition (Shared block, Per-row scale, Low-rank residual);
    reconstruct_weight / relative_frobenius_error.
  * "Quality" -- Native-equivalent at passthrough (G = num_layers rebuilds the
    weight exactly); Reconstruction error (relative Frobenius error).

Readings where the pages are silent:
  * G outside [1, num_layers] is rejected.
  * W0 is the fp64 mean, rounded once to the storage dtype.
  * s is fitted against the *stored* (rounded) W0, the block the forward uses.
  * A row whose W0·W0 is zero gets s = 0 (minimum-norm least squares).
  * relative_frobenius_error = ||A - B||_F / ||A||_F; 0/0 -> 0, x/0 -> inf.
  * The forward has no bias term; its output dtype is the activations' dtype.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
against closed forms, brute force on tiny inputs, library routines and the
passthrough invariant. None is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

F64 = np.float64

# significand bits and smallest quantum exponent of each storage dtype
_FORMATS = {"f32": (24, -149), "bf16": (8, -133)}
_MAX_FINITE_EXP = 128  # both f32 and bf16 overflow at 2**128


# ------------------------------------------------------------------ rounding
def round_to(x, dtype: str) -> np.ndarray:
    """Round float64 values to the nearest value of ``dtype`` (ties to even).

    A value with binary exponent e (2**(e-1) <= |x| < 2**e) has quantum
    2**(e - p) in a format with p significand bits; subnormals share the
    smallest quantum. np.rint rounds half to even.
    """
    a = np.asarray(x, dtype=F64)
    if dtype == "f64":
        return a.copy()
    p, qmin = _FORMATS[dtype]
    _, e = np.frexp(a)
    q = np.maximum(e - p, qmin)
    y = np.ldexp(np.rint(np.ldexp(a, -q)), q)
    over = np.abs(y) >= 2.0 ** _MAX_FINITE_EXP
    if np.any(over):
        y = np.where(over, np.copysign(np.inf, a), y)
    return y


# ------------------------------------------------------------- banded sharing
def band_sizes(num_layers: int, G: int) -> list[int]:
    """Sizes of the G contiguous bands ("Banded sharing" -- How layers map to bands).

    As equal as possible: every band holds num_layers // G layers, and the
    num_layers % G leftover layers go one each to the earliest bands.
    """
    if not (isinstance(num_layers, int) and isinstance(G, int)):
        raise TypeError("num_layers and G must be int")
    if num_layers < 1 or G < 1 or G > num_layers:
        raise ValueError(f"need 1 <= G <= num_layers, got G={G}, num_layers={num_layers}")
    base, extra = divmod(num_layers, G)
    return [base + 1 if b < extra else base for b in range(G)]


def band_index(num_layers: int, G: int):
    """(band_of_layer[num_layers], band_start[G + 1]) as int32 arrays."""
    sizes = band_sizes(num_layers, G)
    start = np.zeros(G + 1, dtype=np.int32)
    start[1:] = np.cumsum(sizes)
    band_of_layer = np.empty(num_layers, dtype=np.int32)
    for b in range(G):
        band_of_layer[start[b]:start[b + 1]] = b
    return band_of_layer, start


# ---------------------------------------------------------- decomposition
def band_mean(weights, G: int, out_dtype: str = "f64") -> np.ndarray:
    """W0[b] = mean of the band's layer weights ("The theta bundle" -- Shared block).

    weights: [L, O, I]. Returns [G, O, I] rounded to ``out_dtype``.
    """
    w = np.asarray(weights, dtype=F64)
    _, start = band_index(w.shape[0], G)
    out = np.empty((G,) + w.shape[1:], dtype=F64)
    for b in range(G):
        out[b] = w[start[b]:start[b + 1]].mean(axis=0)
    return round_to(out, out_dtype)


def row_scale(weight, W0) -> np.ndarray:
    """s_r = (w_r · W0_r) / (W0_r · W0_r) per output row r
    ("The theta bundle" -- Per-row scale). Rows with W0_r = 0 get s_r = 0.
    """
    w = np.asarray(weight, dtype=F64)
    w0 = np.asarray(W0, dtype=F64)
    num = np.einsum("oi,oi->o", w, w0)
    den = np.einsum("oi,oi->o", w0, w0)
    s = np.zeros_like(num)
    nz = den != 0
    s[nz] = num[nz] / den[nz]
    return s


def residual(weight, W0, s, out_dtype: str = "f64") -> np.ndarray:
    """weight - diag(s)·W0 ("The theta bundle" -- Low-rank residual)."""
    w = np.asarray(weight, dtype=F64)
    w0 = np.asarray(W0, dtype=F64)
    sc = np.asarray(s, dtype=F64)
    return round_to(w - sc[:, None] * w0, out_dtype)


def truncated_svd(R, rank: int):
    """Rank-r factors of the residual with U absorbing the singular values
    ("The theta bundle" -- Low-rank residual). Full LAPACK SVD, for small
    matrices only. Returns (U [O, r], V [I, r]) with U·Vᵀ ~ R.
    """
    Rm = np.asarray(R, dtype=F64)
    if rank == 0:
        return np.zeros((Rm.shape[0], 0)), np.zeros((Rm.shape[1], 0))
    Uf, sig, Vt = np.linalg.svd(Rm, full_matrices=False)
    return Uf[:, :rank] * sig[:rank], Vt[:rank].T.copy()


def randomized_svd(R, rank: int, omega, power_iters: int = 0):
    """Rank-r factors of a large residual by the randomized algorithm the pages
    name ("The theta bundle" -- Low-rank residual: Halko et al., 2009, for
    large matrices; U absorbs the singular values). The steps follow Halko,
    Martinsson and Tropp: sample the range, Y = R·Ωᵀ, and orthonormalize it
    (Q); optionally refine by subspace iteration (Q ← orth(R·orth(Rᵀ·Q)),
    power_iters times); project, B = Qᵀ·R; take the SVD of the small B; and
    lift back, U = Q·Ũ[:, :r]·diag(σ[:r]), V = W[:, :r].

    omega [k, I] holds the Gaussian test matrix (k = r + oversampling), passed
    in so that the GPU and this function see the same draw. Returns
    (U [O, r], V [I, r]).
    """
    Rm = np.asarray(R, dtype=F64)
    Om = np.asarray(omega, dtype=F64)
    if rank == 0:
        return np.zeros((Rm.shape[0], 0)), np.zeros((Rm.shape[1], 0))
    Q, _ = np.linalg.qr(Rm @ Om.T)
    for _ in range(power_iters):
        Z, _ = np.linalg.qr(Rm.T @ Q)
        Q, _ = np.linalg.qr(Rm @ Z)
    B = Q.T @ Rm
    Ub, sig, Wt = np.linalg.svd(B, full_matrices=False)
    return (Q @ Ub[:, :rank]) * sig[:rank], Wt[:rank].T.copy()


# ----------------------------------------------------------------- NVFP4
# The pages name NVFP4 for weight bytes ("Quality" -- What NVFP4 quantization
# costs; 3.18x smaller weights) without defining it. Published NVFP4: 4-bit
# E2M1 elements, one FP8 E4M3 scale per 16 consecutive elements of a row,
# and one FP32 scale per tensor. Every rounding decision below is taken in
# fp32 with round-to-nearest-even, as the GPU takes it.
F32 = np.float32


def _grid_round(x, values):
    """Round non-negative fp32 x to the nearest entry of `values` (ascending,
    index = code), ties to the even code; above the top: the top (saturate)."""
    x = np.asarray(x, dtype=F64)
    v = np.asarray(values, dtype=F64)
    hi = np.clip(np.searchsorted(v, x, side="left"), 1, len(v) - 1)
    lo = hi - 1
    dl, dh = x - v[lo], v[hi] - x
    pick_hi = (dh < dl) | ((dh == dl) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(x >= v[-1], len(v) - 1, code)
    return code.astype(np.int64)


def e2m1_values() -> np.ndarray:
    """Non-negative E2M1 magnitudes by code 0..7: 1 sign, 2 exponent (bias 1), 1 mantissa bit."""
    return np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e4m3_values() -> np.ndarray:
    """Non-negative finite FP8 E4M3 values by code 0..126 (bias 7, 3 mantissa
    bits, subnormals below 2^-6, largest 448; code 127 is NaN)."""
    out = []
    for c in range(127):
        e, m = c >> 3, c & 7
        out.append(m / 8.0 * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7))
    return np.array(out)


def nvfp4_quantize(W):
    """W [O, I] (I a multiple of 16) -> (codes uint8 [O, I/2], element 2j in
    the low nibble of byte j; scales uint8 [O, I/16], E4M3 codes; g fp32).

    amax over the tensor; g = amax / (6 * 448); per block of 16: the block
    scale b = blockmax / 6 relative to g, rounded to E4M3; the element scale
    is E4M3(b) * g, and each element w * (1 / scale) is rounded to E2M1 with
    its sign. A zero block (or tensor) gets zero codes.
    """
    w = np.asarray(W, dtype=F32)
    O, I = w.shape
    amax = F32(np.max(np.abs(w))) if w.size else F32(0)
    g = F32(amax / F32(2688.0))
    blk = np.abs(w).reshape(O, I // 16, 16).max(axis=2).astype(F32)
    sb = (blk / F32(6.0)).astype(F32)
    ratio = (sb / g).astype(F32) if g > 0 else np.zeros_like(sb)
    sq = _grid_round(ratio, e4m3_values())
    scale = (e4m3_values()[sq].astype(F32) * g).astype(F32)
    inv = np.where(scale > 0, (F32(1.0) / np.where(scale > 0, scale, F32(1.0))).astype(F32), F32(0.0)).astype(F32)
    x = (w.reshape(O, I // 16, 16) * inv[:, :, None]).astype(F32)
    mag = _grid_round(np.abs(x), e2m1_values())
    code = (mag | np.where((x < 0) & (mag > 0), 8, 0)).reshape(O, I).astype(np.uint8)
    codes = (code[:, 0::2] | (code[:, 1::2] << 4)).astype(np.uint8)
    return codes, sq.astype(np.uint8), g


def nvfp4_dequantize(codes, scales, g) -> np.ndarray:
    """The fp64 weights an NVFP4 encoding stands for: E2M1(code) * E4M3(scale) * g."""
    c = np.asarray(codes, dtype=np.uint8)
    O = c.shape[0]
    el = np.empty((O, c.shape[1] * 2), dtype=np.int64)
    el[:, 0::2], el[:, 1::2] = c & 15, c >> 4
    mag = e2m1_values()[el & 7] * np.where(el & 8, -1.0, 1.0)
    sc = e4m3_values()[np.asarray(scales, dtype=np.int64)]
    return mag * np.repeat(sc, 16, axis=1) * F64(g)


def linear_forward_nvfp4(X, codes, scales, g, s, U, V, out_dtype: str = "f64") -> np.ndarray:
    """The theta forward with W0 given in NVFP4: the projection by the
    dequantized shared block, s ⊙ (X·Ŵ0ᵀ) + (X·V)·Uᵀ."""
    return linear_forward(X, nvfp4_dequantize(codes, scales, g), s, U, V, out_dtype)


def reconstruct(s, W0, U, V, out_dtype: str = "f64") -> np.ndarray:
    """reconstruct_weight(s, W0, U, V) = diag(s)·W0 + U·Vᵀ
    ("The theta bundle" -- the approximation formula and Key layout)."""
    sc = np.asarray(s, dtype=F64)
    w0 = np.asarray(W0, dtype=F64)
    Um = np.asarray(U, dtype=F64).reshape(w0.shape[0], -1)
    Vm = np.asarray(V, dtype=F64).reshape(w0.shape[1], -1)
    return round_to(sc[:, None] * w0 + Um @ Vm.T, out_dtype)


def frob_error(original, reconstructed) -> float:
    """relative_frobenius_error = ||A - B||_F / ||A||_F ("Quality" --
    Reconstruction error). 0 when both norms are 0, +inf when only ||A|| is."""
    A = np.asarray(original, dtype=F64)
    B = np.asarray(reconstructed, dtype=F64)
    num = np.sqrt(np.sum((A - B) ** 2))
    den = np.sqrt(np.sum(A ** 2))
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return float(num / den)


def frob_partials(original, reconstructed):
    """The two sums behind relative_frobenius_error ("Quality" --
    Reconstruction error): (sum of (A - B)^2, sum of A^2) in fp64. Both are
    plain sums over the elements, so a split of the rows into blocks gives
    per-block sums that add up to these; the ratio of their square roots is
    frob_error."""
    A = np.asarray(original, dtype=F64)
    B = np.asarray(reconstructed, dtype=F64)
    return float(np.sum((A - B) ** 2)), float(np.sum(A ** 2))


def frob_from_partials(num, den) -> float:
    """sqrt(num) / sqrt(den), with the same 0/0 -> 0 and x/0 -> +inf cases as
    frob_error."""
    n, d = np.sqrt(F64(num)), np.sqrt(F64(den))
    if d == 0.0:
        return 0.0 if n == 0.0 else float("inf")
    return float(n / d)


# ----------------------------------------------------------------- forward
def linear_forward(X, W0, s, U, V, out_dtype: str = "f64") -> np.ndarray:
    """Y = X·(diag(s)·W0 + U·Vᵀ)ᵀ = s ⊙ (X·W0ᵀ) + (X·V)·Uᵀ.

    The projection applies the rebuilt weight of "The theta bundle" to the
    activations without forming it; X [M, I] -> Y [M, O].
    """
    Xm = np.asarray(X, dtype=F64)
    w0 = np.asarray(W0, dtype=F64)
    sc = np.asarray(s, dtype=F64)
    Um = np.asarray(U, dtype=F64).reshape(w0.shape[0], -1)
    Vm = np.asarray(V, dtype=F64).reshape(w0.shape[1], -1)
    Y = sc[None, :] * (Xm @ w0.T) + (Xm @ Vm) @ Um.T
    return round_to(Y, out_dtype)


def gelu_tanh(x) -> np.ndarray:
    """GELU in its tanh form, 0.5·x·(1 + tanh(√(2/π)·(x + 0.044715·x³))).

    "Quality" — Native-equivalent at passthrough: the MLP takes its
    activation from the model config, and Gemma 3 and Gemma 4 name gelu_tanh.
    The formula is the published tanh approximation of GELU (Hendrycks and
    Gimpel, 2016); the pages name the function, not the formula.
    """
    x = np.asarray(x, dtype=F64)
    return 0.5 * x * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (x + 0.044715 * x ** 3)))


def gate_up_forward(X, gate, up, out_dtype: str = "f64") -> np.ndarray:
    """Y = gelu_tanh(G) ⊙ P for an MLP's gate and up projections on the same
    activations, each the theta forward of its own (W0, s, U, V): the product
    that follows the two projections in the MLP ("Quality" — What quantizing
    attention costs: the fused MLP). G and P are kept in fp64; the product is
    rounded once.
    """
    G = linear_forward(X, *gate)
    P = linear_forward(X, *up)
    return round_to(gelu_tanh(G) * P, out_dtype)


# -------------------------------------------------------- whole decomposition
def decompose_family(weights, G: int, rank: int, dtype: str = "f64"):
    """Analytic decomposition of one projection family, in the pages' order:
    band means, then per layer the row scale against its band's stored W0, the
    residual, and its rank-r truncated SVD. Returns a dict with W0 [G,O,I],
    s [L,O], R [L,O,I], U [L,O,r], V [L,I,r], band_of_layer [L].
    """
    w = np.asarray(weights, dtype=F64)
    L = w.shape[0]
    band_of_layer, _ = band_index(L, G)
    W0 = band_mean(w, G, dtype)
    s = np.empty((L, w.shape[1]))
    R = np.empty_like(w)
    Us, Vs = [], []
    for layer in range(L):
        w0 = W0[band_of_layer[layer]]
        s[layer] = row_scale(w[layer], w0)
        R[layer] = residual(w[layer], w0, s[layer], dtype)
        U, V = truncated_svd(R[layer], rank)
        Us.append(U)
        Vs.append(V)
    return {"W0": W0, "s": s, "R": R, "U": np.stack(Us), "V": np.stack(Vs),
            "band_of_layer": band_of_layer}
