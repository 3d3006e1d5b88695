"""GPU parity of the fused gate/up forward (Y = gelu_tanh(gate) * up, each a
theta forward) against the CPU oracle, to the bf16 bound of a product (the
forward's 2e-2 of the RMS plus the one rounding of each element): ragged tiles, rank 0 and ranks that
are not a multiple of the MMA K step, several token tiles, split-K across a
cluster and whole tiles (both launch policies), a rank term as large as the
main term, and a Gemma-4-31B-sized layer checked on sampled rows."""
import numpy as np
import pytest

import oracle
import synthetic as syn
from gpu_helpers import assert_close_product, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


def projection(O, I, r, seed, tag, uv_std=0.01):
    W0 = syn.host_normal((O, I), 0.02, seed, "W0", tag, O, I, dtype="bf16")
    s = (1.0 + syn.host_normal((O,), 0.05, seed, "s", tag, O)).astype(np.float32)
    U = syn.host_normal((O, r), uv_std, seed, "U", tag, O, r, dtype="bf16")
    V = syn.host_normal((I, r), uv_std, seed, "V", tag, I, r, dtype="bf16")
    return W0, s, U, V


def run_gate_up(lib, torch, X, gate, up):
    M, I = X.shape
    O, r = gate[0].shape[0], gate[2].shape[1]
    to_dev = lambda p: (dev(p[0], "bf16"), dev(p[1], "f32"), dev(p[2], "bf16") if r else None,  # noqa: E731
                        dev(p[3], "bf16") if r else None)
    Y = torch.empty(M, O, dtype=torch.bfloat16, device="cuda")
    nb = lib.theta_workspace_size(lib.THETA_OP_GATE_UP_FORWARD, M, O, I, r, lib.THETA_BF16)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda") if nb else None
    lib.theta_linear_gate_up_forward(dev(X, "bf16"), to_dev(gate), to_dev(up), Y, ws)
    lib.theta_device_status()
    return host(Y)


CASES = [
    # (M, O, I, r)
    (1, 256, 1152, 32),
    (5, 392, 328, 8),
    (16, 6912, 1152, 32),    # the Gemma-3-1B gate/up shape
    (37, 264, 392, 64),
    (130, 136, 520, 24),     # two token tiles, ragged
    (300, 136, 520, 16),     # three token tiles
    (64, 1024, 1152, 0),     # rank 0
    (3, 1024, 6912, 16),     # deep K: split across a cluster
    (128, 392, 1160, 256),   # maximum rank
    # more than 256 tokens: under the throughput policy CTA pairs share
    # 256-row x 128-token tiles (ragged rows past O, tokens past M, K not a
    # multiple of 64, rank 0, the largest rank)
    (257, 264, 392, 40),
    (600, 392, 1160, 256),
    (520, 1032, 264, 0),
    (1100, 520, 1096, 16),
]


@pytest.mark.parametrize("policy", ["latency", "throughput"])
@pytest.mark.parametrize("M,O,I,r", CASES)
def test_gate_up(lib, torch, M, O, I, r, policy):
    seed = M + O + I + r
    X = syn.host_activations(M, I, seed=seed, tag=f"gu{M}x{I}", dtype="bf16")
    gate, up = projection(O, I, r, seed, "gate"), projection(O, I, r, seed, "up")
    ref = oracle.gate_up_forward(X, gate, up)
    lib.theta_set_policy(lib.THETA_POLICY_THROUGHPUT if policy == "throughput" else lib.THETA_POLICY_LATENCY)
    try:
        got = run_gate_up(lib, torch, X, gate, up)
    finally:
        lib.theta_set_policy(lib.THETA_POLICY_LATENCY)
    assert_close_product(got, ref, f"Y {M}x{O}x{I} r{r}")


def test_gate_up_large_rank_term(lib, torch):
    """U, V ~ N(0, 0.1): the rank terms are as large as the main terms."""
    M, O, I, r = 24, 512, 1152, 64
    X = syn.host_activations(M, I, seed=9, tag="gularge", dtype="bf16")
    gate, up = projection(O, I, r, 9, "gate", 0.1), projection(O, I, r, 9, "up", 0.1)
    ref = oracle.gate_up_forward(X, gate, up)
    z = lambda p: (p[0], p[1], p[2] * 0, p[3] * 0)  # noqa: E731
    main = oracle.gate_up_forward(X, z(gate), z(up))
    assert np.sqrt(np.mean((ref - main) ** 2)) > 0.3 * np.sqrt(np.mean(ref ** 2))
    assert_close_product(run_gate_up(lib, torch, X, gate, up), ref, "Y")


@pytest.mark.parametrize("M", [2, 64, 512])
def test_gate_up_gemma4_31b(lib, torch, M):
    """A Gemma-4-31B gate/up pair [21504, 5376], r = 64, drawn on the device;
    sampled output rows against the oracle."""
    O, I = syn.GEMMA4_31B.shapes["gate"]
    r = 64
    dv = lambda tag: (syn.device_normal((O, I), 0.02, 0, "W0", tag),  # noqa: E731
                      1.0 + syn.device_normal((O,), 0.05, 0, "s", tag, dtype="f32"),
                      syn.device_normal((O, r), 0.01, 0, "U", tag), syn.device_normal((I, r), 0.01, 0, "V", tag))
    gate, up = dv("gate31"), dv("up31")
    X = syn.device_normal((M, I), 1.0, 0, "X", M, I)
    Y = torch.empty(M, O, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(lib.theta_workspace_size(lib.THETA_OP_GATE_UP_FORWARD, M, O, I, r, lib.THETA_BF16),
                     dtype=torch.uint8, device="cuda")
    lib.theta_linear_gate_up_forward(X, gate, up, Y, ws)
    lib.theta_device_status()
    rows = np.sort(np.random.default_rng(5).choice(O, 40, replace=False))
    hg = (host(gate[0][rows]), host(gate[1][rows]), host(gate[2][rows]), host(gate[3]))
    hu = (host(up[0][rows]), host(up[1][rows]), host(up[2][rows]), host(up[3]))
    ref = oracle.gate_up_forward(host(X), hg, hu)
    assert_close_product(host(Y[:, rows]), ref, f"Y M={M}")
