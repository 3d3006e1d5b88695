"""NVFP4 shared block on the GPU: the encoder's codes, block scales and tensor
scale bit-exact against the oracle's encoder (every decision in fp32,
round-to-nearest-even -- blocks of very different magnitude exercise
subnormal E4M3 scales, zero blocks and values that round to zero); the
decode forward against the oracle's forward by the dequantized block; a
Gemma-4-31B-sized gate checked on sampled rows."""
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


def encode(lib, torch, W0d):
    O, I = W0d.shape
    codes = torch.empty(O, I // 2, dtype=torch.uint8, device="cuda")
    scales = torch.empty(O, I // 16, dtype=torch.uint8, device="cuda")
    g = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = torch.empty(lib.theta_workspace_size(lib.THETA_OP_NVFP4_QUANTIZE, 1, O, I, 0, lib.THETA_BF16),
                     dtype=torch.uint8, device="cuda")
    lib.theta_nvfp4_quantize(W0d, codes, scales, g, ws)
    lib.theta_device_status()
    return codes, scales, g


def varied_weights(O, I, seed):
    """bf16 weights whose 16-element blocks span six decades of magnitude,
    with a zero block and tiny negatives that round to zero."""
    rng = np.random.default_rng(seed)
    W = rng.standard_normal((O, I)) * 0.02
    W *= np.repeat(10.0 ** rng.uniform(-6, 0, size=(O, I // 16)), 16, axis=1)
    W[0, :16] = 0.0
    W[-1, 16:32] = -1e-7
    return oracle.round_to(W, "bf16").astype(np.float32)


@pytest.mark.parametrize("O,I", [(24, 64), (130, 1152), (1000, 4096)])
def test_encoder_is_bit_exact(lib, torch, O, I):
    W = varied_weights(O, I, O + I)
    codes, scales, g = encode(lib, torch, dev(W, "bf16"))
    c_ref, s_ref, g_ref = oracle.nvfp4_quantize(W)
    assert host(g)[0] == g_ref
    assert np.array_equal(host(scales), s_ref)
    assert np.array_equal(host(codes), c_ref)


@pytest.mark.parametrize("M,O,I,r", [(1, 256, 1152, 32), (2, 392, 320, 8), (1, 6912, 1152, 32), (2, 1024, 4096, 0),
                                     (1, 24, 64, 64)])
def test_forward_matches_oracle(lib, torch, M, O, I, r):
    seed = M + O + I + r
    W0 = oracle.round_to(syn.host_normal((O, I), 0.02, seed, "W0q", O, I), "bf16").astype(np.float32)
    X = syn.host_activations(M, I, seed=seed, tag="nvfp4", dtype="bf16")
    s = (1.0 + syn.host_normal((O,), 0.05, seed, "s", O)).astype(np.float32)
    U = syn.host_normal((O, r), 0.01, seed, "U", O, r, dtype="bf16")
    V = syn.host_normal((I, r), 0.01, seed, "V", I, r, dtype="bf16")
    codes, scales, g = encode(lib, torch, dev(W0, "bf16"))
    Y = torch.empty(M, O, dtype=torch.bfloat16, device="cuda")
    nb = lib.theta_workspace_size(lib.THETA_OP_LINEAR_FORWARD_NVFP4, M, O, I, r, lib.THETA_BF16)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda") if nb else None
    lib.theta_linear_forward_nvfp4(dev(X, "bf16"), codes, scales, g, dev(s, "f32"), dev(U, "bf16") if r else None,
                                   dev(V, "bf16") if r else None, Y, ws)
    lib.theta_device_status()
    ref = oracle.linear_forward_nvfp4(X, host(codes), host(scales), host(g)[0], s, U, V)
    assert_close(host(Y), ref, "bf16", f"Y {M}x{O}x{I} r{r}")
    # and the encoding stays within NVFP4's error of the bf16 forward
    exact = oracle.linear_forward(X, W0, s, U, V)
    assert np.sqrt(np.mean((ref - exact) ** 2)) < 0.15 * np.sqrt(np.mean(exact ** 2))


@pytest.mark.parametrize("M", [1, 2])
def test_gemma4_31b_gate(lib, torch, M):
    O, I = syn.GEMMA4_31B.shapes["gate"]
    r = 64
    W0 = syn.device_normal((O, I), 0.02, 0, "W0", "nv31")
    s = 1.0 + syn.device_normal((O,), 0.05, 0, "s", "nv31", dtype="f32")
    U = syn.device_normal((O, r), 0.01, 0, "U", "nv31")
    V = syn.device_normal((I, r), 0.01, 0, "V", "nv31")
    X = syn.device_normal((M, I), 1.0, 0, "X", M, I)
    codes, scales, g = encode(lib, torch, W0)
    assert host(g)[0] == np.float32(np.float32(W0.abs().max().float().item()) / np.float32(2688.0))
    Y = torch.empty(M, O, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(lib.theta_workspace_size(lib.THETA_OP_LINEAR_FORWARD_NVFP4, M, O, I, r, lib.THETA_BF16),
                     dtype=torch.uint8, device="cuda")
    lib.theta_linear_forward_nvfp4(X, codes, scales, g, s, U, V, Y, ws)
    lib.theta_device_status()
    rows = np.sort(np.random.default_rng(3).choice(O, 40, replace=False))
    hw = host(W0[rows]).astype(np.float64)
    D = oracle.nvfp4_dequantize(host(codes[rows]), host(scales[rows]), host(g)[0])
    bmax = np.repeat(np.abs(hw).reshape(40, I // 16, 16).max(axis=2), 16, axis=1)
    assert np.all(np.abs(D - hw) <= 0.25 * bmax + 1e-30)
    ref = oracle.linear_forward(host(X), D, host(s[rows]), host(U[rows]), host(V))
    assert_close(host(Y[:, rows]), ref, "bf16", f"Y M={M}")


@pytest.mark.parametrize("xs", [1e-30, 1e-3, 1e25])
def test_forward_token_scales(lib, torch, xs):
    """Tokens far from unit size (and two of very different size in one
    call): X is rescaled per token by a power of two before the packed fp16
    sums, so the result must follow the oracle at any scale bf16 holds."""
    M, O, I, r = 2, 512, 2048, 16
    seed = 77
    W0 = oracle.round_to(syn.host_normal((O, I), 0.02, seed, "W0q", O, I), "bf16").astype(np.float32)
    X = syn.host_activations(M, I, seed=seed, tag="nvfp4s", dtype="bf16").astype(np.float64)
    X[0] *= xs
    X = oracle.round_to(X, "bf16")
    s = (1.0 + syn.host_normal((O,), 0.05, seed, "s", O)).astype(np.float32)
    U = syn.host_normal((O, r), 0.01, seed, "U", O, r, dtype="bf16")
    V = syn.host_normal((I, r), 0.01, seed, "V", I, r, dtype="bf16")
    codes, scales, g = encode(lib, torch, dev(W0, "bf16"))
    Y = torch.empty(M, O, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(lib.theta_workspace_size(lib.THETA_OP_LINEAR_FORWARD_NVFP4, M, O, I, r, lib.THETA_BF16),
                     dtype=torch.uint8, device="cuda")
    lib.theta_linear_forward_nvfp4(dev(X, "bf16"), codes, scales, g, dev(s, "f32"), dev(U, "bf16"), dev(V, "bf16"),
                                   Y, ws)
    lib.theta_device_status()
    ref = oracle.linear_forward_nvfp4(X, host(codes), host(scales), host(g)[0], s, U, V)
    for m in range(M):  # each token against its own scale
        assert_close(host(Y)[m:m + 1].astype(np.float64), ref[m:m + 1], "bf16", f"token {m} x{xs:g}")


@pytest.mark.parametrize("M,I", [(1, 101376), (2, 50176)])
def test_forward_at_shared_memory_limit(lib, torch, M, I):
    """The widest rows the sweep takes: X in fp16 for M tokens fills 200 KB
    of shared memory (M * ceil(I / 1024) = 99 or 98 groups)."""
    O, r = 64, 8
    W0 = syn.host_normal((O, I), 0.02, 9, "W0wide", O, I, dtype="bf16")
    X = syn.host_activations(M, I, seed=9, tag="nvfp4wide", dtype="bf16")
    s = (1.0 + syn.host_normal((O,), 0.05, 9, "s", O)).astype(np.float32)
    U = syn.host_normal((O, r), 0.01, 9, "U", O, r, dtype="bf16")
    V = syn.host_normal((I, r), 0.01, 9, "V", I, r, dtype="bf16")
    codes, scales, g = encode(lib, torch, dev(W0, "bf16"))
    Y = torch.empty(M, O, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(lib.theta_workspace_size(lib.THETA_OP_LINEAR_FORWARD_NVFP4, M, O, I, r, lib.THETA_BF16),
                     dtype=torch.uint8, device="cuda")
    lib.theta_linear_forward_nvfp4(dev(X, "bf16"), codes, scales, g, dev(s, "f32"), dev(U, "bf16"), dev(V, "bf16"),
                                   Y, ws)
    lib.theta_device_status()
    ref = oracle.linear_forward_nvfp4(X, host(codes), host(scales), host(g)[0], s, U, V)
    assert_close(host(Y), ref, "bf16", f"Y M={M} I={I}")


def test_forward_past_shared_memory_limit_is_refused(lib, torch):
    """One group more than shared memory holds: THETA_ERR_UNSUPPORTED before
    any launch, and the device stays clean."""
    M, O, I = 1, 8, 102400
    codes = torch.zeros(O, I // 2, dtype=torch.uint8, device="cuda")
    scales = torch.zeros(O, I // 16, dtype=torch.uint8, device="cuda")
    g = torch.ones(1, dtype=torch.float32, device="cuda")
    X = torch.zeros(M, I, dtype=torch.bfloat16, device="cuda")
    s = torch.ones(O, dtype=torch.float32, device="cuda")
    Y = torch.empty(M, O, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.ThetaError) as err:
        lib.theta_linear_forward_nvfp4(X, codes, scales, g, s, None, None, Y, None)
    assert err.value.status == -2
    lib.theta_device_status()
