"""GPU parity at the full sizes of the benchmark workloads, on sampled outputs.

The inputs are drawn on the GPU (too large to draw on the host quickly); the
sampled rows of every input are copied to the host and the CPU oracle
computes the same rows of every output from them. Every output row depends
only on the same row of W / W0 / U / s (and on all of X and V), so the oracle
can check rows one by one. Launch configurations are those bench.py times:
Gemma-3-1B-shaped families (26 layers, G = 26 and G = 1, rank 32,
M = 1, 16, 256) and Gemma-4-31B-shaped projections (rank 64, M = 1, 64, 2048).
"""
import numpy as np
import pytest

import oracle
import synthetic as syn
from gpu_helpers import assert_close, assert_close_chain, assert_residual_step, assert_scalar_close, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


def sample_rows(O, n, seed):
    rng = np.random.default_rng(seed)
    rows = rng.choice(O, size=min(n, O), replace=False)
    rows[:2] = [0, O - 1]  # always include the first and the last row (edge tiles)
    return np.unique(rows)


@pytest.mark.parametrize("fam", ["gate", "down", "k"])
def test_gemma3_1b_family_all_stages(lib, torch, fam):
    O, I = syn.GEMMA3_1B.shapes[fam]
    L, r = syn.GEMMA3_1B.num_layers, 32
    W = syn.device_family_weights(L, O, I, seed=0, family=fam)
    rows = sample_rows(O, 48, 1)
    w_rows = np.stack([host(W[l][rows]) for l in range(L)])       # [L, n, I]
    U = [syn.device_normal((O, r), 0.01, 0, "U", fam, l) for l in range(L)]
    V = [syn.device_normal((I, r), 0.01, 0, "V", fam, l) for l in range(L)]
    for G in (26, 1):
        W0 = [torch.empty(O, I, dtype=torch.bfloat16, device="cuda") for _ in range(G)]
        s = [torch.empty(O, dtype=torch.float32, device="cuda") for _ in range(L)]
        R = [torch.empty(O, I, dtype=torch.bfloat16, device="cuda") for _ in range(L)]
        lib.theta_decompose_prelude(W, G, W0, s, R)
        ref = oracle.decompose_family(w_rows, G, 0, "bf16")
        band = ref["band_of_layer"]
        for b in range(G):
            assert_close(host(W0[b][rows]), ref["W0"][b], "bf16", f"W0[{b}] G={G}")
        for l in (0, 7, L - 1):
            assert_close(host(s[l][rows]), ref["s"][l], "f32", f"s[{l}] G={G}")
            assert_close_chain(host(R[l][rows]), ref["R"][l], "bf16", f"R[{l}] G={G}")
            if G == L:
                assert torch.equal(W0[l], W[l]) and bool((s[l] == 1).all()) and bool((R[l] == 0).all())
        # reconstruct + frob for two layers (frob over the whole matrix)
        fws = torch.empty(lib.theta_workspace_size(lib.THETA_OP_FROB_ERROR, 1, 1, 1, 0, 1), dtype=torch.uint8,
                          device="cuda")
        out = torch.empty(1, dtype=torch.float64, device="cuda")
        for l in (3, L - 2):
            rec = torch.empty(O, I, dtype=torch.bfloat16, device="cuda")
            lib.theta_reconstruct(s[l], W0[band[l]], U[l], V[l], rec)
            s_h, w0_h = host(s[l][rows]), host(W0[band[l]][rows])
            rec_ref = oracle.reconstruct(s_h, w0_h, host(U[l][rows]), host(V[l]), "bf16")
            assert_close(host(rec[rows]), rec_ref, "bf16", f"reconstruct[{l}] G={G}")
            lib.theta_frob_error(W[l], rec, out, fws)
            full_ref = oracle.frob_error(host(W[l]), host(rec))
            assert_scalar_close(out.item(), full_ref, 1e-5, f"frob[{l}] G={G}")
        # forward at the three token counts, sampled output columns
        for m in (1, 16, 256):
            X = syn.device_normal((m, I), 1.0, 0, "X", m, I)
            Y = torch.empty(m, O, dtype=torch.bfloat16, device="cuda")
            ws = torch.empty(lib.theta_workspace_size(lib.THETA_OP_LINEAR_FORWARD, m, O, I, r, 1),
                             dtype=torch.uint8, device="cuda")
            l = 11
            lib.theta_linear_forward(X, W0[band[l]], s[l], U[l], V[l], Y, ws)
            lib.theta_device_status()
            Y_ref = oracle.linear_forward(host(X), host(W0[band[l]][rows]), host(s[l][rows]), host(U[l][rows]),
                                          host(V[l]))
            assert_close(host(Y[:, rows]), Y_ref, "bf16", f"Y m={m} G={G}")


@pytest.mark.parametrize("fam,M", [("gate", 1), ("gate", 4), ("gate", 64), ("gate", 2048), ("k", 1), ("k", 2), ("q", 2),
                                   ("down", 1), ("down", 3), ("down", 16), ("down", 2048), ("o", 256)])
def test_gemma4_31b_forward(lib, torch, fam, M):
    O, I = syn.GEMMA4_31B.shapes[fam]
    r = 64
    W0 = syn.device_normal((O, I), 0.02, 0, "W0", fam)
    s = 1.0 + syn.device_normal((O,), 0.05, 0, "s", fam, dtype="f32")
    U = syn.device_normal((O, r), 0.01, 0, "U", fam)
    V = syn.device_normal((I, r), 0.01, 0, "V", fam)
    X = syn.device_normal((M, I), 1.0, 0, "X", M, I)
    Y = torch.empty(M, O, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(lib.theta_workspace_size(lib.THETA_OP_LINEAR_FORWARD, M, O, I, r, 1), dtype=torch.uint8,
                     device="cuda")
    lib.theta_linear_forward(X, W0, s, U, V, Y, ws)
    lib.theta_device_status()
    rows = sample_rows(O, 40, 2)
    Y_ref = oracle.linear_forward(host(X), host(W0[rows]), host(s[rows]), host(U[rows]), host(V))
    assert_close(host(Y[:, rows]), Y_ref, "bf16", f"Y {fam} M={M}")


def test_gemma4_31b_decomposition(lib, torch):
    O, I = syn.GEMMA4_31B.shapes["gate"]
    L, r = 4, 64
    W = syn.device_family_weights(L, O, I, seed=0, family="gate31")
    rows = sample_rows(O, 24, 3)
    w_rows = np.stack([host(W[l][rows]) for l in range(L)])
    for G in (1, 4):
        W0 = [torch.empty(O, I, dtype=torch.bfloat16, device="cuda") for _ in range(G)]
        s = [torch.empty(O, dtype=torch.float32, device="cuda") for _ in range(L)]
        R = [torch.empty(O, I, dtype=torch.bfloat16, device="cuda") for _ in range(L)]
        lib.theta_decompose_prelude(W, G, W0, s, R)
        ref = oracle.decompose_family(w_rows, G, 0, "bf16")
        for b in range(G):
            assert_close(host(W0[b][rows]), ref["W0"][b], "bf16", f"W0[{b}]")
        for l in range(L):
            assert_close(host(s[l][rows]), ref["s"][l], "f32", f"s[{l}]")
            assert_close_chain(host(R[l][rows]), ref["R"][l], "bf16", f"R[{l}]")
    U = syn.device_normal((O, r), 0.01, 0, "U31")
    V = syn.device_normal((I, r), 0.01, 0, "V31")
    rec = torch.empty(O, I, dtype=torch.bfloat16, device="cuda")
    lib.theta_reconstruct(s[1], W0[1], U, V, rec)
    lib.theta_device_status()
    rec_ref = oracle.reconstruct(host(s[1][rows]), host(W0[1][rows]), host(U[rows]), host(V), "bf16")
    assert_close(host(rec[rows]), rec_ref, "bf16", "reconstruct")


def test_gemma4_31b_sixty_layer_bands(lib, torch):
    """The decomposition sweep's long bands at full size (60 x [21504, 5376]
    bf16, G = 1 and G = 4, the launch configuration the bench times):
    sampled rows of W0, s and R against the oracle on those rows."""
    O, I = syn.GEMMA4_31B.shapes["gate"]
    L = 60
    W = syn.device_family_weights(L, O, I, seed=1, family="gate31-sweep")
    rows = sample_rows(O, 16, 5)
    w_rows = np.stack([host(W[l][rows]) for l in range(L)])
    R = [torch.empty(O, I, dtype=torch.bfloat16, device="cuda") for _ in range(L)]
    s = [torch.empty(O, dtype=torch.float32, device="cuda") for _ in range(L)]
    for G in (1, 4):
        W0 = [torch.empty(O, I, dtype=torch.bfloat16, device="cuda") for _ in range(G)]
        lib.theta_decompose_prelude(W, G, W0, s, R)
        lib.theta_device_status()
        ref = oracle.decompose_family(w_rows, G, 0, "bf16")
        for b in range(G):
            assert_close(host(W0[b][rows]), ref["W0"][b], "bf16", f"G={G} W0[{b}]")
        for l in range(0, L, 7):
            assert_close(host(s[l][rows]), ref["s"][l], "f32", f"G={G} s[{l}]")
            assert_residual_step(host(R[l][rows]), w_rows[l], host(W0[ref["band_of_layer"][l]][rows]),
                                 host(s[l][rows]), "bf16", f"G={G} R[{l}]")
            assert_close_chain(host(R[l][rows]), ref["R"][l], "bf16", f"G={G} R[{l}] (chain)")
