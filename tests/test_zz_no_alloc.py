"""theta_linear_forward_noalloc: the forward for callers that cannot allocate.

Some users of the library may not call cudaMalloc: serving engines whose
device memory is all handed out by their own fixed pool, and plugins that are
given only their input and output buffers. For them the library offers a
forward whose scratch memory is a fixed array built into the library.

These tests call it through the C ABI and check that it gives the same result
as theta_linear_forward with a caller-supplied workspace, on two calls in a
row (the second call reuses the built-in scratch the first one left behind),
and that a request larger than the built-in scratch is refused up front. Both
entry points run the same kernels on the same inputs in the same launch
configuration, so the results must be equal bit for bit (the oracle parity of
that forward is checked elsewhere). The cases cover the one- and two-token
CUDA-core sweep (its scratch holds partial sums of T = X.V), the tensor-core
tile path, and the fp32 path.

The file is named so that pytest collects it after every other test file.
"""
import ctypes

import pytest

import synthetic as syn
from gpu_helpers import assert_close, dev


def _inputs(M, O, I, r, dt, seed):
    X = syn.host_activations(M, I, seed=seed, tag="noalloc", dtype=dt)
    W0 = syn.host_normal((O, I), 0.02, seed, "W0-noalloc", dtype=dt)
    s = (1.0 + syn.host_normal((O,), 0.05, seed, "s-noalloc"))
    U = syn.host_normal((O, r), 0.05, seed, "U-noalloc", dtype=dt)
    V = syn.host_normal((I, r), 0.05, seed, "V-noalloc", dtype=dt)
    return dev(X, dt), dev(W0, dt), dev(s, "f32"), dev(U, dt), dev(V, dt)


@pytest.mark.gpu
@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("M,O,I,r", [(1, 1032, 1152, 32), (2, 6912, 1152, 64), (16, 392, 328, 32),
                                     (256, 1024, 1152, 64)])
def test_noalloc_forward_matches_workspace_forward(lib, dt, M, O, I, r):
    import torch
    for call, seed in enumerate((1, 2)):  # two calls in a row over the same scratch
        X, W0, s, U, V = _inputs(M, O, I, r, dt, seed)
        ref = torch.empty(M, O, dtype=X.dtype, device="cuda")
        nbytes = lib.theta_workspace_size(lib.THETA_OP_LINEAR_FORWARD, M, O, I, r, X)
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        lib.theta_linear_forward(X, W0, s, U, V, ref, ws)
        got = torch.full((M, O), float("nan"), dtype=X.dtype, device="cuda")
        lib.theta_linear_forward_noalloc(X, W0, s, U, V, got)
        lib.theta_device_status()
        g, r_ = got.float().cpu().numpy(), ref.float().cpu().numpy()
        assert_close(g, r_, dt, f"call {call + 1}")
        assert torch.equal(got, ref), f"call {call + 1}: not bitwise equal to the workspace forward"


@pytest.mark.gpu
def test_noalloc_forward_rank0(lib):
    import torch
    X, W0, s, _, _ = _inputs(8, 264, 200, 8, "bf16", 3)
    ref = torch.empty(8, 264, dtype=torch.bfloat16, device="cuda")
    lib.theta_linear_forward(X, W0, s, None, None, ref, None)
    got = torch.empty_like(ref)
    lib.theta_linear_forward_noalloc(X, W0, s, None, None, got)
    lib.theta_device_status()
    assert torch.equal(got, ref), "rank 0: not bitwise equal to the workspace forward"


def test_noalloc_rejects_requests_beyond_the_builtin_scratch(lib):
    """M * rank beyond the 4 MiB array: refused on the host, nothing enqueued
    (runs without a GPU: the check comes before any CUDA call)."""
    raw = lib.lib
    p = ctypes.c_void_p(256)
    M, r = 65536, 64  # needs 16 MiB of scratch
    st = raw.theta_linear_forward_noalloc(p, M, 64, p, 64, p, p, p, r, lib.THETA_BF16, p, None)
    assert st == -6
    msg = lib.theta_last_error()
    assert "built-in" in msg and "4194304" in msg
    st = raw.theta_linear_forward_noalloc(p, M, 64, p, 64, p, p, p, r, lib.THETA_F32, p, None)
    assert st == -6
    st = raw.theta_linear_forward_noalloc(p, 0, 64, p, 64, p, p, p, r, lib.THETA_F32, p, None)
    assert st == -1
