"""GPU randomized SVD of a residual against the CPU oracle's randomized SVD
(same Gaussian test matrix) and against what the mathematics fixes: exact
recovery of a matrix of rank <= r, orthonormal V, U's column norms = the
singular values in descending order, and the same approximation error as the
oracle on the pages' kind of residual (a flat spectrum)."""
import numpy as np
import pytest

import oracle
import synthetic as syn
from gpu_helpers import dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


def gpu_svd(lib, torch, R, rank, omega, power_iters, dt):
    O, I = R.shape
    samples = omega.shape[0]
    Rd = dev(R, dt)
    U = torch.empty(O, rank, dtype=Rd.dtype, device="cuda")
    V = torch.empty(I, rank, dtype=Rd.dtype, device="cuda")
    nb = lib.theta_workspace_size(lib.THETA_OP_RESIDUAL_SVD, samples, O, I, rank, Rd)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    lib.theta_residual_svd(Rd, rank, dev(np.asarray(omega, np.float32), "f32"), U, V, ws, power_iters=power_iters)
    lib.theta_device_status()
    return host(U).astype(np.float64), host(V).astype(np.float64)


def decaying(O, I, n, decay, seed):
    rng = np.random.default_rng(seed)
    A, _ = np.linalg.qr(rng.standard_normal((O, n)))
    B, _ = np.linalg.qr(rng.standard_normal((I, n)))
    sig = decay ** np.arange(n)
    return (A * sig) @ B.T, sig


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("O,I,r0,r,k", [(200, 136, 3, 8, 16), (1024, 1152, 16, 16, 24), (97, 300, 5, 5, 5)])
def test_exact_low_rank_is_recovered(lib, torch, dt, O, I, r0, r, k):
    rng = np.random.default_rng(O + I)
    R = rng.standard_normal((O, r0)) @ rng.standard_normal((r0, I)) * 0.01
    R = oracle.round_to(R, dt)  # the GPU reads the stored values
    U, V = gpu_svd(lib, torch, R, r, rng.standard_normal((k, I)), 1, dt)
    err = np.linalg.norm(R - U @ V.T) / np.linalg.norm(R)
    assert err < (1e-5 if dt == "f32" else 1.5e-2), err  # bf16: the stored U, V carry 8 bits


@pytest.mark.parametrize("power_iters", [0, 1, 2])
@pytest.mark.parametrize("O,I,r,k", [(300, 200, 8, 14), (1152, 6912, 32, 42), (513, 257, 1, 4), (256, 192, 40, 40)])
def test_matches_oracle_on_a_decaying_spectrum(lib, torch, O, I, r, k, power_iters):
    R, sig = decaying(O, I, min(O, I), 0.8, O * 7 + I)
    omega = np.random.default_rng(r + k).standard_normal((k, I))
    U, V = gpu_svd(lib, torch, R, r, omega, power_iters, "f32")
    Uo, Vo = oracle.randomized_svd(R, r, omega, power_iters)
    scale = np.linalg.norm(R)
    assert np.linalg.norm(U @ V.T - Uo @ Vo.T) <= 1e-4 * scale
    assert np.allclose(V.T @ V, np.eye(r), atol=1e-4)
    nrm = np.linalg.norm(U, axis=0)
    assert np.all(np.diff(nrm) <= 1e-5 * nrm[0])  # descending singular values
    assert np.allclose(nrm, np.linalg.norm(Uo, axis=0), rtol=1e-4, atol=1e-6 * scale)


@pytest.mark.parametrize("power_iters", [0, 2])
@pytest.mark.parametrize("O,I,r,k", [(1152, 6912, 32, 42), (300, 200, 8, 14), (513, 264, 1, 4), (264, 392, 40, 40),
                                     (2056, 1160, 64, 74)])
def test_bf16_residual_matches_oracle(lib, torch, O, I, r, k, power_iters):
    """A bf16 residual (I a multiple of 8): the products with R run on tensor
    cores, the fp32 factor in three bf16 parts. Against the oracle on the
    same stored R; U and V come back in bf16, so the bound is bf16's."""
    R, sig = decaying(O, I, min(O, I), 0.8, O * 5 + I)
    R = oracle.round_to(R * 0.02, "bf16")
    omega = np.random.default_rng(r + k + 1).standard_normal((k, I))
    U, V = gpu_svd(lib, torch, R, r, omega, power_iters, "bf16")
    Uo, Vo = oracle.randomized_svd(R, r, omega, power_iters)
    scale = np.linalg.norm(Uo @ Vo.T)
    assert np.linalg.norm(U @ V.T - Uo @ Vo.T) <= 1e-2 * scale
    nrm, nrm_o = np.linalg.norm(U, axis=0), np.linalg.norm(Uo, axis=0)
    assert np.allclose(nrm, nrm_o, rtol=1e-2, atol=1e-3 * nrm_o[0])


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_flat_spectrum_residual_error_matches_oracle(lib, torch, dt):
    """The pages' kind of residual (no spectral knee): a Gemma-3-1B gate layer
    minus its scaled band mean, rank 32, 10 extra samples, two iterations."""
    L, O, I, r, k = 3, 6912, 1152, 32, 42
    w = syn.host_family_weights(L, O, I, seed=4, family="svd", dtype=dt)
    ref = oracle.decompose_family(w, 1, 0, dt)
    R = ref["R"][0]
    omega = syn.host_normal((k, I), 1.0, 4, "omega", O, I)
    U, V = gpu_svd(lib, torch, R, r, omega, 2, dt)
    Uo, Vo = oracle.randomized_svd(R, r, omega, 2)
    nR = np.linalg.norm(R)
    e_gpu = np.linalg.norm(R - U @ V.T) / nR
    e_ora = np.linalg.norm(R - Uo @ Vo.T) / nR
    assert abs(e_gpu - e_ora) < (1e-4 if dt == "f32" else 2e-3), (e_gpu, e_ora)
    Ue, Ve = oracle.truncated_svd(R, r)  # Eckart-Young: nothing beats the exact truncation
    assert e_gpu >= np.linalg.norm(R - Ue @ Ve.T) / nR - 1e-6


def test_zero_residual_gives_zero_factors(lib, torch):
    R = np.zeros((64, 80))
    U, V = gpu_svd(lib, torch, R, 4, np.random.default_rng(0).standard_normal((8, 80)), 1, "f32")
    assert np.all(U == 0) and np.all(np.isfinite(V))
