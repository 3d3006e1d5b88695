"""The row-split (and input-split) theta path across ranks, on the CPU.

Every quantity of "The theta bundle" component table is indexed by output
row, so a family's rows split across GPUs with no exchange for the prelude
and reconstruct, an all-gather of output columns for the forward, and an
all-reduce of two sums for the relative Frobenius error. Here gloo ranks
(world sizes 2 and 3, as torchrun would start them) each run the oracle on
their block and combine through linear_theta_forward_b200.sharding; the
combined results must equal the oracle on the whole problem: bit for bit
where every element is computed by the same operations in both (forward
columns, W0, s, R), and to fp64 rounding where a sum is split (the Frobenius
sums, exact on integer data; the input-split forward).
"""
import os
import socket

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_row_blocks_cover_rows_in_aligned_blocks():
    from linear_theta_forward_b200.sharding import row_blocks, block_of
    for n in (0, 1, 7, 8, 100, 1024, 5376, 21504, 21505):
        for world in (1, 2, 3, 4, 8):
            b = row_blocks(n, world)
            assert len(b) == world and b[0][0] == 0 and b[-1][1] == n
            assert all(b[k][1] == b[k + 1][0] for k in range(world - 1))  # contiguous
            assert all(a % 8 == 0 for a, _ in b)                           # aligned starts
            sizes = [e - a for a, e in b[:-1]] + [(b[-1][1] - b[-1][0]) - n % 8]
            assert all(s % 8 == 0 and s >= 0 for s in sizes)
            assert max(sizes) - min(sizes) <= 8 and sizes == sorted(sizes, reverse=True)
            assert [block_of(n, k, world) for k in range(world)] == b
    assert row_blocks(100, 2) == [(0, 48), (48, 100)]  # 12 whole units split 6 + 6; the 4-row tail goes last
    assert row_blocks(104, 2) == [(0, 56), (56, 104)]  # 13 units: the earlier block takes the extra one
    assert row_blocks(21504, 8) == [(k * 2688, (k + 1) * 2688) for k in range(8)]
    with pytest.raises(ValueError):
        row_blocks(10, 0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import sys
    import datetime
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch
    import torch.distributed as dist
    import oracle
    import synthetic as syn
    from linear_theta_forward_b200 import sharding as sh
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    res = {}
    try:
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))  # noqa: E731
        L, G, O, I, r, M = 5, 2, 100, 72, 8, 6   # O not a multiple of 8 * world: a ragged last block
        w = syn.host_family_weights(L, O, I, seed=3, family="shard", dtype="bf16")
        U = syn.host_normal((O, r), 0.05, 3, "U", dtype="bf16")
        V = syn.host_normal((I, r), 0.05, 3, "V", dtype="bf16")
        X = syn.host_activations(M, I, seed=3, tag="shard", dtype="bf16")
        o0, o1 = sh.block_of(O, rank, world)

        # prelude on the row block: W0, s, R rows equal the whole problem's
        whole = oracle.decompose_family(w, G, 0, "bf16")
        part = oracle.decompose_family(w[:, o0:o1], G, 0, "bf16")
        W0 = [sh.gather_rows(t(part["W0"][b]), O) for b in range(G)]
        s = [sh.gather_rows(t(part["s"][l]), O) for l in range(L)]
        R = [sh.gather_rows(t(part["R"][l]), O) for l in range(L)]
        res["prelude"] = (all(np.array_equal(W0[b].numpy(), whole["W0"][b]) for b in range(G))
                          and all(np.array_equal(s[l].numpy(), whole["s"][l]) for l in range(L))
                          and all(np.array_equal(R[l].numpy(), whole["R"][l]) for l in range(L)))

        # forward split by output rows: column blocks gathered
        band, _ = oracle.band_index(L, G)
        l = 3
        w0, s32 = whole["W0"][band[l]], oracle.round_to(whole["s"][l], "f32")
        y_whole = oracle.linear_forward(X, w0, s32, U, V)
        y_block = oracle.linear_forward(X, w0[o0:o1], s32[o0:o1], U[o0:o1], V)
        y = sh.gather_columns(t(y_block), O).numpy()
        res["forward_rows"] = np.array_equal(y, y_whole)

        # forward split along the input (a down projection fed by split gate/up outputs)
        i0, i1 = sh.block_of(I, rank, world)
        yk = sh.allreduce_partials(t(oracle.linear_forward(X[:, i0:i1], w0[:, i0:i1], s32, U, V[i0:i1])))
        res["forward_k_err"] = float(np.max(np.abs(yk.numpy() - y_whole)) / np.max(np.abs(y_whole)))

        # relative Frobenius error from the blocks' sums
        rec = oracle.reconstruct(s32, w0, U, V, "bf16")
        sums = sh.allreduce_partials(t(oracle.frob_partials(w[l][o0:o1], rec[o0:o1])))
        e = sh.frob_from_sums(*sums.tolist())
        res["frob_err"] = abs(e - oracle.frob_error(w[l], rec)) / oracle.frob_error(w[l], rec)
        rng = np.random.default_rng(11)
        Ai = rng.integers(-40, 40, size=(O, I)).astype(np.float64)
        Bi = rng.integers(-40, 40, size=(O, I)).astype(np.float64)
        si = sh.allreduce_partials(t(oracle.frob_partials(Ai[o0:o1], Bi[o0:o1])))
        res["frob_int_exact"] = tuple(si.tolist()) == oracle.frob_partials(Ai, Bi)
        res["frob_int_ratio"] = sh.frob_from_sums(*si.tolist()) == oracle.frob_error(Ai, Bi)
        dist.barrier()
        out.put((rank, res))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_row_split_path_with_gloo_ranks(world):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    results = dict(out.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert sorted(results) == list(range(world))
    for rank, res in results.items():
        assert res["prelude"], rank
        assert res["forward_rows"], rank
        assert res["forward_k_err"] < 1e-13, (rank, res["forward_k_err"])
        assert res["frob_err"] < 1e-13, (rank, res["frob_err"])
        assert res["frob_int_exact"] and res["frob_int_ratio"], rank
