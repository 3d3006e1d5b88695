"""The oracle against its pins, and planted mistakes against the pins (CPU only).

A mutant is a copy of the oracle with one plausible mistake; every mutant must
be caught by at least one check, which shows the pins can see that mistake.
"""
import types

import numpy as np
import pytest

import oracle
import oracle_checks as oc


@pytest.mark.parametrize("check", oc.ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(check):
    check(oracle)


# --------------------------------------------------------------- mutants
def _ns(**override):
    ns = types.SimpleNamespace(**{k: v for k, v in vars(oracle).items() if not k.startswith("_")})
    for k, v in override.items():
        setattr(ns, k, v)
    return ns


def _m_round_truncate(x, dtype):
    a = np.asarray(x, dtype=np.float64)
    if dtype == "f64":
        return a
    p, qmin = {"f32": (24, -149), "bf16": (8, -133)}[dtype]
    _, e = np.frexp(a)
    q = np.maximum(e - p, qmin)
    return np.ldexp(np.trunc(np.ldexp(a, -q)), q)


def _m_bands_late_remainder(L, G):
    if L < 1 or G < 1 or G > L:
        raise ValueError
    q, r = divmod(L, G)
    return [q + 1 if b >= G - r else q for b in range(G)]


def _m_bands_first_takes_all(L, G):
    if L < 1 or G < 1 or G > L:
        raise ValueError
    q, r = divmod(L, G)
    return [q + r] + [q] * (G - 1)


def _m_band_mean_divide_by_L(weights, G, out_dtype="f64"):
    w = np.asarray(weights, dtype=np.float64)
    _, start = oracle.band_index(w.shape[0], G)
    out = np.stack([w[start[b]:start[b + 1]].sum(0) / w.shape[0] for b in range(G)])
    return oracle.round_to(out, out_dtype)


def _m_band_mean_off_by_one(weights, G, out_dtype="f64"):
    w = np.asarray(weights, dtype=np.float64)
    _, start = oracle.band_index(w.shape[0], G)
    out = np.stack([w[start[b]:max(start[b + 1] - 1, start[b] + 1)].mean(0) for b in range(G)])
    return oracle.round_to(out, out_dtype)


def _m_row_scale_swapped(weight, W0):
    return oracle.row_scale(W0, weight)


def _m_row_scale_wrong_norm(weight, W0):
    w, w0 = np.asarray(weight, np.float64), np.asarray(W0, np.float64)
    return np.einsum("oi,oi->o", w, w0) / np.einsum("oi,oi->o", w, w)


def _m_residual_sign(weight, W0, s, out_dtype="f64"):
    return oracle.round_to(np.asarray(weight) + np.asarray(s)[:, None] * np.asarray(W0), out_dtype)


def _m_reconstruct_v_layout(s, W0, U, V, out_dtype="f64"):
    # reads V [in, rank] as if it were stored [rank, in]
    w0 = np.asarray(W0, np.float64)
    Vm = np.asarray(V, np.float64)
    Vwrong = Vm.reshape(Vm.shape[1], Vm.shape[0])
    return oracle.round_to(np.asarray(s)[:, None] * w0 + np.asarray(U) @ Vwrong, out_dtype)


def _m_reconstruct_unscaled(s, W0, U, V, out_dtype="f64"):
    return oracle.reconstruct(np.ones_like(np.asarray(s, np.float64)), W0, U, V, out_dtype)


def _m_frob_by_recon(A, B):
    A, B = np.asarray(A, np.float64), np.asarray(B, np.float64)
    den = np.sqrt(np.sum(B ** 2))
    return float(np.sqrt(np.sum((A - B) ** 2)) / den) if den else 0.0


def _m_frob_squared(A, B):
    e = oracle.frob_error(A, B)
    return e * e


def _m_frob_partials_den_from_recon(A, B):
    A, B = np.asarray(A, np.float64), np.asarray(B, np.float64)
    return float(np.sum((A - B) ** 2)), float(np.sum(B ** 2))


def _m_frob_partials_norms(A, B):
    A, B = np.asarray(A, np.float64), np.asarray(B, np.float64)
    return float(np.sqrt(np.sum((A - B) ** 2))), float(np.sqrt(np.sum(A ** 2)))


def _m_forward_no_rank(X, W0, s, U, V, out_dtype="f64"):
    return oracle.linear_forward(X, W0, s, np.zeros_like(np.asarray(U, np.float64)),
                                 np.zeros_like(np.asarray(V, np.float64)), out_dtype)


def _m_forward_scale_all(X, W0, s, U, V, out_dtype="f64"):
    Xm, w0, sc = (np.asarray(a, np.float64) for a in (X, W0, s))
    Y = sc[None, :] * (Xm @ w0.T + (Xm @ np.asarray(V)) @ np.asarray(U).T)
    return oracle.round_to(Y, out_dtype)


def _m_forward_scale_rows(X, W0, s, U, V, out_dtype="f64"):
    Xm, w0, sc = (np.asarray(a, np.float64) for a in (X, W0, s))
    Y = (Xm @ w0.T) * sc[: Xm.shape[0], None] if Xm.shape[0] <= sc.shape[0] else Xm @ w0.T
    return oracle.round_to(Y + (Xm @ np.asarray(V)) @ np.asarray(U).T, out_dtype)


def _m_svd_no_sigma(R, rank):
    Uf, sig, Vt = np.linalg.svd(np.asarray(R, np.float64), full_matrices=False)
    return Uf[:, :rank], Vt[:rank].T


def _m_gelu_erf(x):
    from scipy.special import erf
    x = np.asarray(x, np.float64)
    return 0.5 * x * (1.0 + erf(x / np.sqrt(2.0)))


def _m_gelu_constant(x):
    x = np.asarray(x, np.float64)
    return 0.5 * x * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (x + 0.0447 * x ** 3)))


def _m_gate_up_activates_up(X, gate, up, out_dtype="f64"):
    return oracle.round_to(oracle.linear_forward(X, *gate) * oracle.gelu_tanh(oracle.linear_forward(X, *up)),
                           out_dtype)


def _m_gate_up_no_activation(X, gate, up, out_dtype="f64"):
    return oracle.round_to(oracle.linear_forward(X, *gate) * oracle.linear_forward(X, *up), out_dtype)


def _m_rsvd_unorthonormalized(R, rank, omega, power_iters=0):
    Rm, Om = np.asarray(R, np.float64), np.asarray(omega, np.float64)
    Q = Rm @ Om.T  # the sample used as if it were an orthonormal basis
    Ub, sig, Wt = np.linalg.svd(Q.T @ Rm, full_matrices=False)
    return (Q @ Ub[:, :rank]) * sig[:rank], Wt[:rank].T.copy()


def _m_rsvd_sigma_in_v(R, rank, omega, power_iters=0):
    U, V = oracle.randomized_svd(R, rank, omega, power_iters)
    n = np.linalg.norm(U, axis=0)
    return U / np.where(n == 0, 1, n), V * n


def _m_nvfp4_high_nibble_first(W):
    c, sc, g = oracle.nvfp4_quantize(W)
    return ((c >> 4) | (c << 4)).astype(np.uint8), sc, g


def _m_nvfp4_ties_away(x, values):
    v = np.asarray(values, np.float64)
    x = np.asarray(x, np.float64)
    hi = np.clip(np.searchsorted(v, x, side="left"), 1, len(v) - 1)
    lo = hi - 1
    code = np.where(v[hi] - x <= x - v[lo], hi, lo)
    return np.where(x >= v[-1], len(v) - 1, code).astype(np.int64)


def _m_nvfp4_no_global_scale(codes, scales, g):
    return oracle.nvfp4_dequantize(codes, scales, 1.0)


MUTANTS = {
    "nvfp4_high_nibble_first": dict(nvfp4_quantize=_m_nvfp4_high_nibble_first),
    "nvfp4_ties_away_from_zero": dict(_grid_round=_m_nvfp4_ties_away),
    "nvfp4_drops_global_scale": dict(nvfp4_dequantize=_m_nvfp4_no_global_scale),
    "rsvd_sample_not_orthonormalized": dict(randomized_svd=_m_rsvd_unorthonormalized),
    "rsvd_sigma_in_v": dict(randomized_svd=_m_rsvd_sigma_in_v),
    "gelu_erf_form": dict(gelu_tanh=_m_gelu_erf),
    "gelu_wrong_constant": dict(gelu_tanh=_m_gelu_constant),
    "gate_up_activates_up": dict(gate_up_forward=_m_gate_up_activates_up),
    "gate_up_without_activation": dict(gate_up_forward=_m_gate_up_no_activation),
    "round_truncates": dict(round_to=_m_round_truncate),
    "bands_late_remainder": dict(band_sizes=_m_bands_late_remainder),
    "bands_first_takes_all": dict(band_sizes=_m_bands_first_takes_all),
    "band_mean_divides_by_L": dict(band_mean=_m_band_mean_divide_by_L),
    "band_mean_drops_last_layer": dict(band_mean=_m_band_mean_off_by_one),
    "row_scale_swapped_operands": dict(row_scale=_m_row_scale_swapped),
    "row_scale_wrong_norm": dict(row_scale=_m_row_scale_wrong_norm),
    "residual_wrong_sign": dict(residual=_m_residual_sign),
    "reconstruct_transposed_factor": dict(reconstruct=_m_reconstruct_v_layout),
    "reconstruct_drops_scale": dict(reconstruct=_m_reconstruct_unscaled),
    "frob_normalised_by_reconstruction": dict(frob_error=_m_frob_by_recon),
    "frob_squared": dict(frob_error=_m_frob_squared),
    "frob_partials_normalised_by_reconstruction": dict(frob_partials=_m_frob_partials_den_from_recon),
    "frob_partials_as_norms": dict(frob_partials=_m_frob_partials_norms),
    "forward_drops_rank_term": dict(linear_forward=_m_forward_no_rank),
    "forward_scales_rank_term": dict(linear_forward=_m_forward_scale_all),
    "forward_scale_on_wrong_axis": dict(linear_forward=_m_forward_scale_rows),
    "svd_u_without_sigma": dict(truncated_svd=_m_svd_no_sigma),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    ns = _ns(**MUTANTS[name])
    failures = []
    for check in oc.ALL_CHECKS:
        try:
            check(ns)
        except AssertionError:
            failures.append(check.__name__)
    assert failures, f"mutant {name} passed every pin"
