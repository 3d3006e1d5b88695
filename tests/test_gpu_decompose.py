"""GPU parity of the decomposition and checking kernels against the CPU oracle:
band mean, row scale, residual, the fused prelude, relative Frobenius error.
"""
import numpy as np
import pytest

import oracle
import synthetic as syn
from gpu_helpers import assert_close, assert_close_chain, assert_residual_step, assert_scalar_close, dev, host, TOL

pytestmark = pytest.mark.gpu

DTYPES = ["f32", "bf16"]


@pytest.fixture(scope="module")
def torch():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


def weights(L, O, I, dt, seed=0, fam="w"):
    return syn.host_family_weights(L, O, I, seed=seed, family=fam, dtype=dt)


# ---------------------------------------------------------------- band mean
@pytest.mark.parametrize("dt", DTYPES)
@pytest.mark.parametrize("n,O,I", [(1, 64, 256), (2, 256, 256), (3, 37, 1152), (7, 5, 13), (26, 24, 1000),
                                   (60, 8, 5376), (5, 3, 7)])
def test_band_mean(lib, torch, dt, n, O, I):
    w = weights(n, O, I, dt, seed=n)
    ws = [dev(w[i], dt) for i in range(n)]
    W0 = torch.empty_like(ws[0])
    lib.theta_band_mean(ws, W0)
    ref = oracle.band_mean(w, 1, dt)[0]
    assert_close(host(W0), ref, dt, "W0")


@pytest.mark.parametrize("dt", DTYPES)
def test_band_mean_single_layer_is_bitwise_copy(lib, torch, dt):
    w = weights(1, 33, 264, dt)
    W = dev(w[0], dt)
    W0 = torch.empty_like(W)
    lib.theta_band_mean([W], W0)
    assert torch.equal(W0, W)


# ---------------------------------------------------------------- row scale
# row lengths chosen to exercise every (threads per row, vectors per thread)
# variant and the scalar path for lengths that are not a vector multiple
ROW_LENGTHS = [8, 64, 256, 1000, 1024, 1152, 2056, 5376, 6912, 13, 21504]


@pytest.mark.parametrize("dt", DTYPES)
@pytest.mark.parametrize("I", ROW_LENGTHS)
def test_row_scale(lib, torch, dt, I):
    O = 37
    w = weights(3, O, I, dt, seed=I)
    W0 = oracle.band_mean(w, 1, dt)[0]
    s = torch.empty(O, dtype=torch.float32, device="cuda")
    lib.theta_row_scale(dev(w[1], dt), dev(W0, dt), s)
    ref = oracle.row_scale(w[1], W0)
    assert_close(host(s), ref, "f32", "s")


@pytest.mark.parametrize("dt", DTYPES)
@pytest.mark.parametrize("I", [256, 1152, 13, 5376])
def test_residual(lib, torch, dt, I):
    O = 29
    w = weights(2, O, I, dt, seed=I + 1)
    W0 = oracle.band_mean(w, 1, dt)[0]
    s = oracle.round_to(oracle.row_scale(w[0], W0), "f32")
    R = torch.empty_like(dev(w[0], dt))
    lib.theta_residual(dev(w[0], dt), dev(W0, dt), dev(s, "f32"), R)
    assert_close(host(R), oracle.residual(w[0], W0, s, dt), dt, "R")
    assert_residual_step(host(R), w[0], W0, s, dt, "R")


def test_zero_w0_row_gives_zero_scale(lib, torch):
    O, I = 8, 64
    w = weights(1, O, I, "f32")[0]
    W0 = w.copy() * 0.5
    W0[3] = 0.0
    s = torch.empty(O, dtype=torch.float32, device="cuda")
    lib.theta_row_scale(dev(w), dev(W0), s)
    sh = host(s)
    assert sh[3] == 0.0
    assert_close(sh, oracle.row_scale(w, W0), "f32", "s")
    R = torch.empty(O, I, device="cuda")
    lib.theta_residual(dev(w), dev(W0), s, R)
    assert np.array_equal(host(R)[3], w[3].astype(np.float64))


# ---------------------------------------------------------------- prelude
@pytest.mark.parametrize("dt,L,G,O,I", [("f32", 4, 2, 256, 256),     # the tiny workload
                                        ("bf16", 7, 3, 40, 264),
                                        ("bf16", 26, 4, 24, 1152),
                                        ("f32", 5, 2, 17, 13),
                                        ("bf16", 6, 1, 9, 5376),
                                        ("bf16", 8, 2, 33, 5376),     # one-pass prelude, 4-layer bands
                                        ("bf16", 2, 2, 20, 21504),    # one-pass prelude, widest rows
                                        ("f32", 3, 1, 21, 1000),
                                        # bands of more than 4 layers: two-pass prelude, else
                                        # band mean + row pass
                                        ("f32", 9, 2, 19, 1000),
                                        ("bf16", 60, 1, 3, 5376),
                                        ("bf16", 11, 2, 130, 1152),
                                        ("bf16", 12, 1, 5, 21504),     # rows too long: band mean + row pass
                                        ("f32", 30, 1, 7, 5376),
                                        ("bf16", 26, 1, 40, 6912),     # the 1B down projection at G = 1
                                        ("bf16", 60, 4, 261, 5376),    # ragged 15-layer bands
                                        ("bf16", 60, 1, 300, 5376)])   # 60-layer band, many rows
def test_decompose_prelude(lib, torch, dt, L, G, O, I):
    w = weights(L, O, I, dt, seed=L * G)
    ws = [dev(w[i], dt) for i in range(L)]
    W0 = [torch.empty_like(ws[0]) for _ in range(G)]
    s = [torch.empty(O, dtype=torch.float32, device="cuda") for _ in range(L)]
    R = [torch.empty_like(ws[0]) for _ in range(L)]
    lib.theta_decompose_prelude(ws, G, W0, s, R)
    ref = oracle.decompose_family(w, G, 0, dt)
    for b in range(G):
        assert_close(host(W0[b]), ref["W0"][b], dt, f"W0[{b}]")
    for layer in range(L):
        b = ref["band_of_layer"][layer]
        # s and R against the oracle given the GPU's stored W0 (one input, the
        # oracle's own arithmetic), and against the pure oracle chain
        w0_gpu = host(W0[b])
        assert_close(host(s[layer]), oracle.row_scale(w[layer], w0_gpu), "f32", f"s[{layer}]")
        assert_close(host(s[layer]), ref["s"][layer], "f32", f"s[{layer}] (chain)")
        # R: the step on the GPU's own W0 and s exactly, the chain within one ulp
        assert_residual_step(host(R[layer]), w[layer], w0_gpu, host(s[layer]), dt, f"R[{layer}]")
        assert_close_chain(host(R[layer]), ref["R"][layer], dt, f"R[{layer}] (chain)")


@pytest.mark.parametrize("dt", DTYPES)
def test_prelude_without_residual(lib, torch, dt):
    L, G, O, I = 4, 2, 16, 64
    w = weights(L, O, I, dt)
    ws = [dev(w[i], dt) for i in range(L)]
    W0 = [torch.empty_like(ws[0]) for _ in range(G)]
    s = [torch.empty(O, dtype=torch.float32, device="cuda") for _ in range(L)]
    lib.theta_decompose_prelude(ws, G, W0, s, None)
    ref = oracle.decompose_family(w, G, 0, dt)
    for layer in range(L):
        assert_close(host(s[layer]), ref["s"][layer], "f32", "s")


@pytest.mark.parametrize("dt,L,O,I", [("bf16", 26, 40, 6912), ("f32", 30, 9, 5376)])
def test_long_band_prelude_without_residual(lib, torch, dt, L, O, I):
    w = weights(L, O, I, dt, seed=7)
    ws = [dev(w[i], dt) for i in range(L)]
    W0 = [torch.empty_like(ws[0])]
    s = [torch.empty(O, dtype=torch.float32, device="cuda") for _ in range(L)]
    lib.theta_decompose_prelude(ws, 1, W0, s, None)
    ref = oracle.decompose_family(w, 1, 0, dt)
    assert_close(host(W0[0]), ref["W0"][0], dt, "W0")
    for layer in range(L):
        assert_close(host(s[layer]), ref["s"][layer], "f32", f"s[{layer}]")


@pytest.mark.parametrize("dt,L,I", [("bf16", 60, 5376), ("bf16", 26, 6912), ("bf16", 12, 21504)])
def test_identical_layers_give_exact_scale_in_a_long_band(lib, torch, dt, L, I):
    """Every layer of a long band equal (bf16 weights; two-pass and band mean +
    row pass routes): the mean is that weight exactly -- up to 256 copies of
    an 8-bit significand sum exactly in fp32 -- and the two dot products of
    each row use one operation order, so s == 1 and the residual is 0 bit for
    bit. (fp32 weights have no such guarantee: k copies of a 24-bit
    significand already round at k = 3.)"""
    O = 24
    one = weights(1, O, I, dt, seed=9)[0]
    ws = [dev(one, dt) for _ in range(L)]
    W0 = [torch.empty_like(ws[0])]
    s = [torch.empty(O, dtype=torch.float32, device="cuda") for _ in range(L)]
    R = [torch.full_like(ws[0], 7.0) for _ in range(L)]
    lib.theta_decompose_prelude(ws, 1, W0, s, R)
    assert torch.equal(W0[0], ws[0])
    for layer in range(L):
        assert bool((s[layer] == 1.0).all()), layer
        assert bool((R[layer] == 0).all()), layer


@pytest.mark.parametrize("dt", DTYPES)
def test_passthrough_is_exact(lib, torch, dt):
    """G = num_layers: W0 is the layer's own weight, s == 1, residual == 0, and
    the rebuilt weight equals the original bit for bit ("Banded sharing";
    "Quality" -- Native-equivalent at passthrough)."""
    L, O, I = 4, 48, 1152
    w = weights(L, O, I, dt, seed=5)
    ws = [dev(w[i], dt) for i in range(L)]
    W0 = [torch.empty_like(ws[0]) for _ in range(L)]
    s = [torch.empty(O, dtype=torch.float32, device="cuda") for _ in range(L)]
    R = [torch.empty_like(ws[0]) for _ in range(L)]
    lib.theta_decompose_prelude(ws, L, W0, s, R)
    ws_frob = torch.empty(lib.theta_workspace_size(lib.THETA_OP_FROB_ERROR, 1, 1, 1, 0, 0) // 4 + 4,
                          dtype=torch.float32, device="cuda")
    out = torch.empty(1, dtype=torch.float64, device="cuda")
    for layer in range(L):
        assert torch.equal(W0[layer], ws[layer])
        assert bool((s[layer] == 1.0).all())
        assert bool((R[layer] == 0).all())
        rec = torch.empty_like(ws[0])
        lib.theta_reconstruct(s[layer], W0[layer], None, None, rec)          # rank 0
        assert torch.equal(rec, ws[layer])
        U = torch.zeros(O, 8, dtype=ws[0].dtype, device="cuda")
        V = torch.zeros(I, 8, dtype=ws[0].dtype, device="cuda")
        lib.theta_reconstruct(s[layer], W0[layer], U, V, rec)                # U = V = 0
        assert torch.equal(rec, ws[layer])
        lib.theta_frob_error(ws[layer], rec, out, ws_frob)
        assert out.item() == 0.0


# ---------------------------------------------------------------- frobenius
@pytest.mark.parametrize("dt", DTYPES)
@pytest.mark.parametrize("n", [1, 7, 4096, 1000003, 6912 * 1152])
def test_frob_error(lib, torch, dt, n):
    a = syn.host_normal((n,), 0.02, 1, "A", n, dtype=dt)
    b = syn.as_dtype_values(a + syn.host_normal((n,), 0.005, 1, "B", n), dt)
    out = torch.empty(1, dtype=torch.float64, device="cuda")
    ws = torch.empty(lib.theta_workspace_size(lib.THETA_OP_FROB_ERROR, 1, 1, 1, 0, 0), dtype=torch.uint8,
                     device="cuda")
    lib.theta_frob_error(dev(a, dt), dev(b, dt), out, ws)
    assert_scalar_close(out.item(), oracle.frob_error(a, b), 1e-5, "frob")


def test_frob_error_degenerate_and_closed_forms(lib, torch):
    ws = torch.empty(lib.theta_workspace_size(lib.THETA_OP_FROB_ERROR, 1, 1, 1, 0, 0), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty(1, dtype=torch.float64, device="cuda")
    z = torch.zeros(1000, device="cuda")
    lib.theta_frob_error(z, z, out, ws)
    assert out.item() == 0.0
    lib.theta_frob_error(z, torch.ones_like(z), out, ws)
    assert out.item() == float("inf")
    a = dev(syn.host_normal((5000,), 1.0, 3, "A"))
    lib.theta_frob_error(a, torch.zeros_like(a), out, ws)
    assert abs(out.item() - 1.0) < 1e-6
    lib.theta_frob_error(a, a * 1.25, out, ws)
    assert abs(out.item() - 0.25) < 1e-6
    empty = torch.empty(0, device="cuda")
    lib.theta_frob_error(empty, empty, out, ws)
    assert out.item() == 0.0
    # a second call over the same workspace gives the same bits (fixed order)
    b = a * 1.001
    lib.theta_frob_error(a, b, out, ws)
    first = out.item()
    lib.theta_frob_error(a, b, out, ws)
    assert out.item() == first


@pytest.mark.parametrize("dt", DTYPES)
@pytest.mark.parametrize("n", [1, 7, 1000003, 6912 * 1152])
def test_frob_partials(lib, torch, dt, n):
    """The two sums against the oracle's; their ratio is theta_frob_error's
    result bit for bit (same kernels, one IEEE sqrt and division each)."""
    import math
    a = syn.host_normal((n,), 0.02, 2, "A", n, dtype=dt)
    b = syn.as_dtype_values(a + syn.host_normal((n,), 0.005, 2, "B", n), dt)
    ws = torch.empty(lib.theta_workspace_size(lib.THETA_OP_FROB_ERROR, 1, 1, 1, 0, 0), dtype=torch.uint8,
                     device="cuda")
    p = torch.full((2,), float("nan"), dtype=torch.float64, device="cuda")
    out = torch.empty(1, dtype=torch.float64, device="cuda")
    A, B = dev(a, dt), dev(b, dt)
    lib.theta_frob_partials(A, B, p, ws)
    lib.theta_frob_error(A, B, out, ws)
    num, den = oracle.frob_partials(a, b)
    g = p.cpu().tolist()
    assert_scalar_close(g[0], num, 1e-5, "sum (A-B)^2")
    assert_scalar_close(g[1], den, 1e-5, "sum A^2")
    assert math.sqrt(g[0]) / math.sqrt(g[1]) == out.item()


def test_frob_partials_of_row_blocks_add_up(lib, torch):
    """Rows split into uneven blocks (as across GPUs): the blocks' sums add up
    to the whole matrix's, and the error formed from them matches the oracle's
    error of the whole matrix."""
    O, I = 1000, 1152
    a = syn.host_normal((O, I), 0.02, 4, "A", dtype="bf16")
    b = syn.as_dtype_values(a + syn.host_normal((O, I), 0.005, 4, "B"), "bf16")
    A, B = dev(a, "bf16"), dev(b, "bf16")
    ws = torch.empty(lib.theta_workspace_size(lib.THETA_OP_FROB_ERROR, 1, 1, 1, 0, 0), dtype=torch.uint8,
                     device="cuda")
    whole = torch.empty(2, dtype=torch.float64, device="cuda")
    lib.theta_frob_partials(A, B, whole, ws)
    tot = torch.zeros(2, dtype=torch.float64, device="cuda")
    for o0, o1 in ((0, 336), (336, 672), (672, 1000)):
        part = torch.empty(2, dtype=torch.float64, device="cuda")
        lib.theta_frob_partials(A[o0:o1], B[o0:o1], part, ws)
        tot += part
    w, t = whole.cpu().tolist(), tot.cpu().tolist()
    assert abs(w[0] - t[0]) <= 1e-12 * w[0] and abs(w[1] - t[1]) <= 1e-12 * w[1]
    assert_scalar_close(oracle.frob_from_partials(*t), oracle.frob_error(a, b), 1e-5, "frob from blocks")
