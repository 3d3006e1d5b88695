"""The row-split wrappers on one GPU: a one-rank NCCL group runs the same
host logic the multi-GPU path runs (library calls on the block, then the
collective), and the results equal the unsplit library calls. The combine
logic for two and three ranks is covered on the CPU by tests/test_sharding.py.
"""
import pytest

import oracle
import synthetic as syn
from gpu_helpers import assert_scalar_close, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def group():
    import torch.distributed as dist
    dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1)
    yield None
    dist.destroy_process_group()


def test_forward_rows_and_k_on_one_rank(lib, group):
    import torch
    from linear_theta_forward_b200 import sharding as sh
    M, O, I, r = 16, 392, 328, 32
    X = dev(syn.host_activations(M, I, seed=5, tag="shard", dtype="bf16"), "bf16")
    W0 = dev(syn.host_normal((O, I), 0.02, 5, "W0", dtype="bf16"), "bf16")
    s = dev(1.0 + syn.host_normal((O,), 0.05, 5, "s"), "f32")
    U = dev(syn.host_normal((O, r), 0.05, 5, "U", dtype="bf16"), "bf16")
    V = dev(syn.host_normal((I, r), 0.05, 5, "V", dtype="bf16"), "bf16")
    ws = torch.empty(lib.theta_workspace_size(lib.THETA_OP_LINEAR_FORWARD, M, O, I, r, X), dtype=torch.uint8,
                     device="cuda")
    ref = torch.empty(M, O, dtype=torch.bfloat16, device="cuda")
    lib.theta_linear_forward(X, W0, s, U, V, ref, ws)
    assert torch.equal(sh.forward_rows(X, W0, s, U, V, ws, O), ref)
    assert torch.equal(sh.forward_k(X, W0, s, U, V, ws), ref)


def test_sharded_frob_error_on_one_rank(lib, group):
    import torch
    from linear_theta_forward_b200 import sharding as sh
    a = syn.host_normal((300, 264), 0.02, 6, "A", dtype="bf16")
    b = syn.as_dtype_values(a + syn.host_normal((300, 264), 0.005, 6, "B"), "bf16")
    ws = torch.empty(lib.theta_workspace_size(lib.THETA_OP_FROB_ERROR, 1, 1, 1, 0, 0), dtype=torch.uint8,
                     device="cuda")
    e = sh.sharded_frob_error(dev(a, "bf16"), dev(b, "bf16"), ws)
    out = torch.empty(1, dtype=torch.float64, device="cuda")
    lib.theta_frob_error(dev(a, "bf16"), dev(b, "bf16"), out, ws)
    assert e == out.item()
    assert_scalar_close(e, oracle.frob_error(a, b), 1e-5, "frob")
