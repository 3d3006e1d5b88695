"""Grouped decode forward on the GPU: every problem's Y against the oracle's
forward (bf16 bound), for groups mixing shapes, ranks (0 included) and
problems sharing one X; a whole Gemma-3-1B-shaped layer set (7 families x 3
layers) on sampled rows; the result equal, up to fp32 summation order, to
one theta_linear_forward call per problem."""
import numpy as np
import pytest

import oracle
import synthetic as syn
from gpu_helpers import assert_close, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


def oracle_args(X, W0, s, U, V):
    """The oracle's forward takes zero-width factors at rank 0."""
    O, I = W0.shape
    return (X, W0, s, np.zeros((O, 0)) if U is None else U, np.zeros((I, 0)) if V is None else V)


def host_problem(M, O, I, r, seed, X=None):
    W0 = syn.host_normal((O, I), 0.02, seed, "W0g", O, I, dtype="bf16")
    s = (1.0 + syn.host_normal((O,), 0.05, seed, "sg", O)).astype(np.float32)
    U = syn.host_normal((O, r), 0.01, seed, "Ug", O, r, dtype="bf16") if r else None
    V = syn.host_normal((I, r), 0.01, seed, "Vg", I, r, dtype="bf16") if r else None
    if X is None:
        X = syn.host_activations(M, I, seed=seed, tag="grouped", dtype="bf16")
    return X, W0, s, U, V


def run_group(lib, torch, hosts, M):
    probs, Ys = [], []
    xdev = {}
    for X, W0, s, U, V in hosts:
        key = id(X)
        if key not in xdev:
            xdev[key] = dev(X, "bf16")
        Y = torch.full((M, W0.shape[0]), float("nan"), dtype=torch.bfloat16, device="cuda")
        probs.append((xdev[key], dev(W0, "bf16"), dev(s, "f32"), dev(U, "bf16") if U is not None else None,
                      dev(V, "bf16") if V is not None else None, Y))
        Ys.append(Y)
    group = lib.ForwardGroup(probs)
    nb = group.workspace_size()
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda") if nb else None
    lib.theta_linear_forward_grouped(group, ws)
    lib.theta_device_status()
    return group, [host(Y) for Y in Ys]


@pytest.mark.parametrize("M", [1, 2])
def test_mixed_group_matches_oracle(lib, torch, M):
    shared = syn.host_activations(M, 1152, seed=5, tag="grouped-shared", dtype="bf16")
    hosts = [host_problem(M, 256, 1152, 32, 1, X=shared), host_problem(M, 1024, 1152, 0, 2, X=shared),
             host_problem(M, 40, 64, 8, 3), host_problem(M, 1152, 2048, 64, 4), host_problem(M, 8, 8, 8, 5),
             host_problem(M, 392, 320, 256, 6), host_problem(M, 6912, 1152, 32, 7, X=shared)]
    _, Ys = run_group(lib, torch, hosts, M)
    for k, ((X, W0, s, U, V), Y) in enumerate(zip(hosts, Ys)):
        ref = oracle.linear_forward(*oracle_args(X, W0, s, U, V))
        assert_close(Y, ref, "bf16", f"problem {k} M={M}")


def test_single_problem_and_max_count(lib, torch):
    hosts = [host_problem(1, 64, 128, 8, 10)]
    _, Ys = run_group(lib, torch, hosts, 1)
    assert_close(Ys[0], oracle.linear_forward(*oracle_args(*hosts[0])), "bf16", "one problem")
    X = syn.host_activations(1, 64, seed=11, tag="grouped-many", dtype="bf16")
    hosts = [host_problem(1, 8 * (1 + k % 5), 64, 8 * (k % 3), 100 + k, X=X) for k in range(256)]
    _, Ys = run_group(lib, torch, hosts, 1)
    for k, ((X_, W0, s, U, V), Y) in enumerate(zip(hosts, Ys)):
        assert_close(Y, oracle.linear_forward(*oracle_args(X_, W0, s, U, V)), "bf16", f"problem {k} of 256")


@pytest.mark.parametrize("M", [1, 2])
def test_gemma3_1b_layers(lib, torch, M):
    """7 families x 3 layers at the Gemma-3-1B shapes, rank 32, on the device;
    sampled rows of every Y against the oracle, and every Y against one
    theta_linear_forward call per problem."""
    shapes = syn.GEMMA3_1B.shapes
    r = 32
    xs = {I: syn.device_normal((M, I), 1.0, 0, "Xg", M, I) for I in sorted({I for (_, I) in shapes.values()})}
    probs, meta = [], []
    for fam, (O, I) in shapes.items():
        for l in range(3):
            W0 = syn.device_normal((O, I), 0.02, l, "W0", fam)
            s = 1.0 + syn.device_normal((O,), 0.05, l, "s", fam, dtype="f32")
            U = syn.device_normal((O, r), 0.01, l, "U", fam)
            V = syn.device_normal((I, r), 0.01, l, "V", fam)
            Y = torch.empty(M, O, dtype=torch.bfloat16, device="cuda")
            probs.append((xs[I], W0, s, U, V, Y))
    group = lib.ForwardGroup(probs)
    ws = torch.empty(group.workspace_size(), dtype=torch.uint8, device="cuda")
    lib.theta_linear_forward_grouped(group, ws)
    lib.theta_device_status()
    rng = np.random.default_rng(7)
    fws = torch.empty(1 << 22, dtype=torch.uint8, device="cuda")
    for k, (X, W0, s, U, V, Y) in enumerate(probs):
        O = W0.shape[0]
        rows = np.sort(rng.choice(O, min(O, 48), replace=False))
        ref = oracle.linear_forward(host(X), host(W0[rows]), host(s[rows]), host(U[rows]), host(V))
        assert_close(host(Y[:, rows]), ref, "bf16", f"problem {k} sampled rows")
        Y1 = torch.empty_like(Y)
        lib.theta_linear_forward(X, W0, s, U, V, Y1, fws)
        d = (Y.float() - Y1.float()).abs().max().item()
        assert d <= 2 ** -7 * Y1.float().abs().max().item(), f"problem {k}: grouped vs single {d}"


def test_max_count_two_tokens(lib, torch):
    """256 problems of two tokens, widths 8..40 rows, ranks 0/8/16."""
    X = syn.host_activations(2, 64, seed=12, tag="grouped-many2", dtype="bf16")
    hosts = [host_problem(2, 8 * (1 + k % 5), 64, 8 * (k % 3), 300 + k, X=X) for k in range(256)]
    _, Ys = run_group(lib, torch, hosts, 2)
    for k, ((X_, W0, s, U, V), Y) in enumerate(zip(hosts, Ys)):
        assert_close(Y, oracle.linear_forward(*oracle_args(X_, W0, s, U, V)), "bf16", f"problem {k} of 256, M=2")
