"""GPU parity of the theta forward and reconstruct_weight against the CPU oracle.

Sizes span several tiles with ragged tails (M, O, I not multiples of the tile
sizes), rank 0 and ranks that are not a multiple of the MMA K step, decode-
sized M (split-K paths) and prefill-sized M. A large-U,V variant makes the
rank-r term as large as the main term, so a dropped or mis-scaled correction
cannot hide under the bf16 tolerance.
"""
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


def bundle(M, O, I, r, dt, seed=0, uv_std=0.01):
    """Seeded (X, W0, s, U, V): W0 from the weight model, s near 1."""
    X = syn.host_activations(M, I, seed=seed, tag=f"{M}x{I}", dtype=dt)
    W0 = syn.host_normal((O, I), 0.02, seed, "W0", O, I, dtype=dt)
    s = (1.0 + syn.host_normal((O,), 0.05, seed, "s", O)).astype(np.float32)
    U = syn.host_normal((O, r), uv_std, seed, "U", O, r, dtype=dt)
    V = syn.host_normal((I, r), uv_std, seed, "V", I, r, dtype=dt)
    return X, W0, s, U, V


def run_forward(lib, torch, X, W0, s, U, V, dt):
    M, I = X.shape
    O, r = W0.shape[0], U.shape[1]
    Xd, W0d, sd = dev(X, dt), dev(W0, dt), dev(s, "f32")
    Ud = dev(U, dt) if r else None
    Vd = dev(V, dt) if r else None
    Y = torch.empty(M, O, dtype=Xd.dtype, device="cuda")
    nbytes = lib.theta_workspace_size(lib.THETA_OP_LINEAR_FORWARD, M, O, I, r, Xd)
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device="cuda") if nbytes else None
    lib.theta_linear_forward(Xd, W0d, sd, Ud, Vd, Y, ws)
    lib.theta_device_status()
    return host(Y)


FORWARD_CASES = [
    # (M, O, I, r)
    (16, 256, 256, 8),       # the tiny workload's shape
    (1, 392, 328, 8),
    (3, 136, 72, 0),
    (16, 392, 328, 32),
    (37, 256, 1152, 64),
    (64, 1024, 1152, 32),
    (65, 392, 328, 24),
    (130, 136, 1160, 16),
    (256, 1152, 1024, 32),
    (300, 392, 328, 64),
    (1, 8, 8, 8),
    (5, 2056, 200, 8),
    (600, 256, 1152, 32),    # three 256-token tiles
    (40, 256, 264, 128),     # rank variants of the T = X.V kernel
    (8, 136, 200, 192),
    (130, 264, 392, 256),
    (3, 1024, 6912, 16),     # deep K: split across a cluster
    # one or two tokens (the CUDA-core sweep): ragged row ranges per CTA,
    # long rows, maximum rank; three and four tokens take the tile path
    (2, 4104, 1152, 64),
    (4, 1000, 200, 8),
    (2, 1000, 8200, 24),
    (4, 304, 16392, 0),
    (1, 24, 64, 8),
    (3, 2056, 200, 256),
    (4, 136, 24, 16),
]


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("M,O,I,r", FORWARD_CASES)
def test_forward(lib, torch, dt, M, O, I, r):
    X, W0, s, U, V = bundle(M, O, I, r, dt, seed=M + O + I + r)
    got = run_forward(lib, torch, X, W0, s, U, V, dt)
    ref = oracle.linear_forward(X, W0, s, U, V)
    assert_close(got, ref, dt, f"Y {M}x{O}x{I} r{r}")


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("M,O,I,r", [(16, 392, 328, 32), (200, 256, 1152, 64), (1, 1024, 1152, 64),
                                     (4, 1024, 1152, 64), (2, 520, 9000, 32)])
def test_forward_large_rank_term(lib, torch, dt, M, O, I, r):
    """U, V ~ N(0, 0.1): the rank term is comparable to the main term."""
    X, W0, s, U, V = bundle(M, O, I, r, dt, seed=7, uv_std=0.1)
    got = run_forward(lib, torch, X, W0, s, U, V, dt)
    ref = oracle.linear_forward(X, W0, s, U, V)
    main = oracle.linear_forward(X, W0, s, U * 0, V * 0)
    assert np.sqrt(np.mean((ref - main) ** 2)) > 0.3 * np.sqrt(np.mean(ref ** 2))
    assert_close(got, ref, dt, "Y")


@pytest.mark.parametrize("M,O,I,r", [(3, 1024, 6912, 16), (16, 392, 328, 32), (64, 1024, 1152, 32),
                                     (600, 256, 1152, 32), (40, 256, 264, 128)])
def test_forward_throughput_policy(lib, torch, M, O, I, r):
    """Without split-K (every CTA owns a whole tile) the result is the same."""
    X, W0, s, U, V = bundle(M, O, I, r, "bf16", seed=5)
    ref = oracle.linear_forward(X, W0, s, U, V)
    lib.theta_set_policy(lib.THETA_POLICY_THROUGHPUT)
    try:
        got = run_forward(lib, torch, X, W0, s, U, V, "bf16")
    finally:
        lib.theta_set_policy(lib.THETA_POLICY_LATENCY)
    assert_close(got, ref, "bf16", "Y")


# More than 256 tokens with a whole tile per CTA: pairs of SMs share 256 x 256
# tiles (the even CTA's MMAs read both CTAs' halves of W0 and X). Ragged row
# pairs (the odd CTA's rows partly or wholly past O), ragged token tiles (the
# odd CTA's tokens wholly past M), K not a multiple of 64, rank 0 and the
# largest rank.
PAIR_CASES = [
    (600, 392, 328, 64),     # 1.5 row pairs, 2.3 token tiles
    (257, 264, 1160, 40),    # one token in the second tile
    (520, 1032, 264, 0),     # rank 0: no D2
    (300, 264, 392, 256),    # four rank blocks, hi and lo parts each
    (2100, 520, 1096, 16),
    (200, 264, 1160, 40),    # 129-256 tokens: one pair tile, the odd CTA's tokens partly past M
    (256, 1152, 1024, 32),
    (129, 392, 328, 8),
]


@pytest.mark.parametrize("M,O,I,r", PAIR_CASES)
def test_forward_pair_tiles(lib, torch, M, O, I, r):
    X, W0, s, U, V = bundle(M, O, I, r, "bf16", seed=M + O)
    ref = oracle.linear_forward(X, W0, s, U, V)
    lib.theta_set_policy(lib.THETA_POLICY_THROUGHPUT)
    try:
        got = run_forward(lib, torch, X, W0, s, U, V, "bf16")
    finally:
        lib.theta_set_policy(lib.THETA_POLICY_LATENCY)
    assert_close(got, ref, "bf16", f"Y {M}x{O}x{I} r{r}")


def test_forward_pair_tiles_fill_the_gpu_under_latency_policy(lib, torch):
    """Under the latency policy the pair path is taken once the 128 x 256
    tiles alone fill the GPU (here 26 x 6 = 156 tiles)."""
    M, O, I, r = 1300, 3208, 1160, 40
    X, W0, s, U, V = bundle(M, O, I, r, "bf16", seed=13)
    got = run_forward(lib, torch, X, W0, s, U, V, "bf16")
    rows = np.r_[0:8, 120:136, 250:262, 1500:1530, 3190:3208]
    ref = oracle.linear_forward(X, W0[rows], s[rows], U[rows], V)
    assert_close(got[:, rows], ref, "bf16", "Y")


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_forward_rank0_is_scaled_shared_block(lib, torch, dt):
    X, W0, s, U, V = bundle(9, 264, 520, 0, dt, seed=3)
    got = run_forward(lib, torch, X, W0, s, U, V, dt)
    assert_close(got, oracle.linear_forward(X, W0, s, U, V), dt, "Y")


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_forward_equals_rebuilt_weight_projection(lib, torch, dt):
    """Y equals X . reconstruct(s, W0, U, V)^T (the weight the forward never forms)."""
    M, O, I, r = 24, 256, 392, 16
    X, W0, s, U, V = bundle(M, O, I, r, dt, seed=11)
    got = run_forward(lib, torch, X, W0, s, U, V, dt)
    Wr = oracle.reconstruct(s, W0, U, V)
    assert_close(got, X.astype(np.float64) @ Wr.T, dt, "Y vs X.W^T")


# ---------------------------------------------------------------- reconstruct
RECON_CASES = [(256, 256, 8), (392, 328, 32), (136, 1160, 64), (1024, 1152, 32), (40, 24, 0), (8, 8, 8),
               (2056, 200, 24), (200, 136, 128), (64, 520, 192), (72, 264, 256), (128, 64, 64)]


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("O,I,r", RECON_CASES)
def test_reconstruct(lib, torch, dt, O, I, r):
    _, W0, s, U, V = bundle(1, O, I, r, dt, seed=O * 3 + I + r)
    out = torch.empty(O, I, dtype=dev(W0[:1], dt).dtype, device="cuda")
    lib.theta_reconstruct(dev(s, "f32"), dev(W0, dt), dev(U, dt) if r else None, dev(V, dt) if r else None, out)
    lib.theta_device_status()
    assert_close(host(out), oracle.reconstruct(s, W0, U, V, dt), dt, "W_rec")


BAND_CASES = [("bf16", 4, 256, 264, 16), ("bf16", 7, 300, 1152, 32), ("bf16", 15, 1024, 5376, 64),
              ("bf16", 3, 130, 200, 128), ("bf16", 70, 64, 256, 8), ("bf16", 2, 40, 64, 0),
              ("bf16", 5, 2056, 136, 64), ("f32", 3, 72, 96, 16)]


@pytest.mark.parametrize("dt,n,O,I,r", BAND_CASES)
def test_reconstruct_band(lib, torch, dt, n, O, I, r):
    """theta_reconstruct_band over the n layers of one band: each output
    equals theta_reconstruct of that layer element for element, and the
    oracle's reconstruct within the tolerance (bands of more than 64 layers
    take two launches; rank 0 and fp32 take one call per layer)."""
    W0 = syn.host_normal((O, I), 0.02, n + O, "W0-band", dtype=dt)
    s = [1.0 + syn.host_normal((O,), 0.05, n + O, "s-band", l) for l in range(n)]
    U = [syn.host_normal((O, r), 0.05, n + O, "U-band", l, dtype=dt) for l in range(n)]
    V = [syn.host_normal((I, r), 0.05, n + O, "V-band", l, dtype=dt) for l in range(n)]
    d_s = [dev(x, "f32") for x in s]
    d_U = [dev(x, dt) for x in U] if r else None
    d_V = [dev(x, dt) for x in V] if r else None
    d_W0 = dev(W0, dt)
    outs = [torch.full((O, I), float("nan"), dtype=d_W0.dtype, device="cuda") for _ in range(n)]
    lib.theta_reconstruct_band(d_s, d_W0, d_U, d_V, outs)
    one = torch.empty_like(outs[0])
    for l in range(n):
        lib.theta_reconstruct(d_s[l], d_W0, d_U[l] if r else None, d_V[l] if r else None, one)
        assert torch.equal(outs[l], one), f"layer {l}: differs from theta_reconstruct"
        if l in (0, n // 2, n - 1):
            assert_close(host(outs[l]), oracle.reconstruct(s[l], W0, U[l], V[l], dt), dt, f"W_rec[{l}]")
    lib.theta_device_status()


def test_tiny_workload_end_to_end(lib, torch):
    """The tiny workload: 4 layers [256, 256] fp32, G = 2, rank 8 from the
    oracle's SVD of each residual, X [16, 256]; the GPU runs the prelude,
    reconstruct, Frobenius error and the forward, each checked element-wise."""
    L, G, O, I, r, M = 4, 2, 256, 256, 8, 16
    w = syn.host_family_weights(L, O, I, seed=0, family="tiny", dtype="f32")
    X = syn.host_activations(M, I, seed=0, tag="tiny")
    ws = [dev(w[i]) for i in range(L)]
    W0 = [torch.empty(O, I, device="cuda") for _ in range(G)]
    s = [torch.empty(O, device="cuda") for _ in range(L)]
    R = [torch.empty(O, I, device="cuda") for _ in range(L)]
    lib.theta_decompose_prelude(ws, G, W0, s, R)
    ref = oracle.decompose_family(w, G, r, "f32")
    frob_ws = torch.empty(lib.theta_workspace_size(0, 1, 1, 1, 0, 0), dtype=torch.uint8, device="cuda")
    out = torch.empty(1, dtype=torch.float64, device="cuda")
    for layer in range(L):
        b = ref["band_of_layer"][layer]
        assert_close(host(W0[b]), ref["W0"][b], "f32", "W0")
        assert_close(host(s[layer]), ref["s"][layer], "f32", "s")
        assert_close(host(R[layer]), ref["R"][layer], "f32", "R")
        U = oracle.round_to(ref["U"][layer], "f32").astype(np.float32)
        V = oracle.round_to(ref["V"][layer], "f32").astype(np.float32)
        s32 = oracle.round_to(ref["s"][layer], "f32").astype(np.float32)
        W0_32 = ref["W0"][b].astype(np.float32)
        rec = torch.empty(O, I, device="cuda")
        lib.theta_reconstruct(dev(s32), dev(W0_32), dev(U), dev(V), rec)
        rec_ref = oracle.reconstruct(s32, W0_32, U, V, "f32")
        assert_close(host(rec), rec_ref, "f32", "reconstruct")
        lib.theta_frob_error(ws[layer], rec, out, frob_ws)
        fe = oracle.frob_error(w[layer], rec_ref)
        assert abs(out.item() - fe) <= 1e-5 * fe
        Y = run_forward(lib, torch, X, W0_32, s32, U, V, "f32")
        assert_close(Y, oracle.linear_forward(X, W0_32, s32, U, V), "f32", "Y")
