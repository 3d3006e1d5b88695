"""Failure detection on the GPU without a fault: a bounded wait that nothing
completes gives up, the host sees THETA_ERR_TIMEOUT through
theta_device_status, the flag clears, and the context keeps working. While
the flag is set, kernels with waits skip their work instead of each waiting
out its own limit."""
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


def test_timeout_is_reported_then_cleared(lib, torch):
    lib.theta_device_status()  # start clean
    lib.theta_selftest_wait_timeout(50)
    with pytest.raises(lib.ThetaError) as err:
        lib.theta_device_status()
    assert err.value.status == -5  # THETA_ERR_TIMEOUT
    lib.theta_device_status()  # read once, then clear


def test_selftest_rejects_bad_limits(lib):
    with pytest.raises(lib.ThetaError):
        lib.theta_selftest_wait_timeout(0)
    with pytest.raises(lib.ThetaError):
        lib.theta_selftest_wait_timeout(5000)


def test_work_after_a_timeout_is_flagged_then_recovers(lib, torch):
    M, O, I, r = 16, 1024, 1152, 32
    X = syn.host_activations(M, I, seed=1, tag="fail", dtype="bf16")
    W0 = syn.host_normal((O, I), 0.02, 1, "W0f", dtype="bf16")
    s = (1.0 + syn.host_normal((O,), 0.05, 1, "sf")).astype(np.float32)
    U = syn.host_normal((O, r), 0.01, 1, "Uf", dtype="bf16")
    V = syn.host_normal((I, r), 0.01, 1, "Vf", dtype="bf16")
    Xd, W0d, sd, Ud, Vd = dev(X, "bf16"), dev(W0, "bf16"), dev(s, "f32"), dev(U, "bf16"), dev(V, "bf16")
    Y = torch.empty(M, O, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(lib.theta_workspace_size(lib.THETA_OP_LINEAR_FORWARD, M, O, I, r, lib.THETA_BF16),
                     dtype=torch.uint8, device="cuda")
    lib.theta_device_status()
    lib.theta_selftest_wait_timeout(20)
    lib.theta_linear_forward(Xd, W0d, sd, Ud, Vd, Y, ws)  # enqueued while the flag is set
    with pytest.raises(lib.ThetaError) as err:
        lib.theta_device_status()
    assert err.value.status == -5
    lib.theta_linear_forward(Xd, W0d, sd, Ud, Vd, Y, ws)  # flag cleared: a normal call
    lib.theta_device_status()
    assert_close(host(Y), oracle.linear_forward(X, W0, s, U, V), "bf16", "Y after recovery")
