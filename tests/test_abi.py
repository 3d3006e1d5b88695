"""The C ABI on the host: loads, exports what include/theta.h declares, and
validates arguments before touching a GPU (no GPU needed)."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import oracle_checks as oc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "theta.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(theta_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ["theta_band_index", "theta_band_mean", "theta_row_scale", "theta_residual",
                     "theta_decompose_prelude", "theta_reconstruct", "theta_frob_error",
                     "theta_linear_forward", "theta_workspace_size", "theta_device_status"]:
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    raw = ctypes.CDLL(lib.LIB_PATH)
    for name in declared_functions():
        assert hasattr(raw, name), f"{name} declared in theta.h but not exported"


def test_binding_names_match_c_names(lib):
    for name in declared_functions():
        assert callable(getattr(lib, name)), name


def test_version_and_status_strings(lib):
    assert lib.theta_version() == 1
    assert lib.theta_status_string(0) == "THETA_OK"
    assert lib.theta_status_string(-5) == "THETA_ERR_TIMEOUT"
    assert lib.theta_status_string(12345) == "THETA_ERR_UNKNOWN"


@pytest.mark.parametrize("L,G", [(4, 2), (26, 1), (26, 4), (26, 7), (26, 26), (60, 15), (60, 4), (1, 1),
                                 (256, 3), (97, 13)])
def test_band_index_matches_oracle_bit_exactly(lib, L, G):
    bol, start = lib.theta_band_index(L, G)
    obol, ostart = oracle.band_index(L, G)
    assert bol.dtype == np.int32 and np.array_equal(bol, obol)
    assert np.array_equal(start, ostart)


def test_band_index_golden_table(lib):
    for L, G, sizes in oc.read_band_golden():
        _, start = lib.theta_band_index(L, G)
        assert list(np.diff(start)) == sizes


@pytest.mark.parametrize("L,G", [(4, 0), (4, 5), (0, 1), (-1, 1), (3, -2)])
def test_band_index_rejects(lib, L, G):
    with pytest.raises(lib.ThetaError) as e:
        lib.theta_band_index(L, G)
    assert e.value.status == -1
    assert "G" in lib.theta_last_error()


def test_validation_happens_before_any_cuda_call(lib):
    raw = lib.lib
    # each call below has an argument error; none may reach the CUDA runtime
    assert raw.theta_band_mean(None, 0, 4, 4, 0, None, None) == -1
    assert raw.theta_band_mean(None, 1, 4, 4, 7, None, None) == -1           # bad dtype
    assert raw.theta_row_scale(None, None, 0, 4, 0, None, None) == -1
    assert raw.theta_residual(None, None, None, 4, 4, 0, None, None) == -1
    assert raw.theta_decompose_prelude(None, 4, 5, 8, 8, 0, None, None, None, None) == -1
    assert raw.theta_decompose_prelude(None, 300, 1, 8, 8, 0, None, None, None, None) == -1
    assert raw.theta_reconstruct(None, None, None, None, 8, 8, -1, 0, None, None) == -1
    assert raw.theta_frob_error(None, None, -1, 0, None, None, 0, None) == -1
    assert raw.theta_frob_error(None, None, 0, 0, ctypes.c_void_p(16), None, 0, None) == -6
    assert raw.theta_frob_partials(None, None, -1, 0, None, None, 0, None) == -1
    assert raw.theta_frob_partials(None, None, 0, 0, ctypes.c_void_p(12), None, 0, None) == -3   # out misaligned
    assert raw.theta_frob_partials(None, None, 0, 0, ctypes.c_void_p(16), None, 0, None) == -6
    assert raw.theta_linear_forward(None, 0, 8, None, 8, None, None, None, 0, 0, None, None, 0, None) == -1
    assert raw.theta_linear_forward(ctypes.c_void_p(16), 4, 8, ctypes.c_void_p(16), 8, ctypes.c_void_p(16),
                                    None, None, 8, 0, ctypes.c_void_p(16), None, 0, None) == -1  # rank>0, U NULL
    assert raw.theta_linear_forward(ctypes.c_void_p(16), 4, 8, ctypes.c_void_p(16), 8, ctypes.c_void_p(16),
                                    ctypes.c_void_p(16), ctypes.c_void_p(16), 8, 1, ctypes.c_void_p(16),
                                    None, 0, None) == -6                                         # no workspace
    p = ctypes.c_void_p(16)
    assert raw.theta_linear_gate_up_forward(None, 4, 8, 8, 0, 1, None, None, None, None, None, None, None, None,
                                            None, None, 0, None) == -1                           # NULL inputs
    assert raw.theta_linear_gate_up_forward(p, 4, 8, 8, 8, 0, p, p, p, p, p, p, p, p, p, p, 1 << 20,
                                            None) == -2                                          # fp32: bf16 only
    assert raw.theta_linear_gate_up_forward(p, 4, 8, 8, 8, 1, p, p, p, p, p, p, p, p, p, None, 0,
                                            None) == -6                                          # no workspace
    assert raw.theta_linear_gate_up_forward(p, 4, 12, 8, 8, 1, p, p, p, p, p, p, p, p, p, p, 1 << 20,
                                            None) == -3                                          # I % 8 != 0


def test_sizes_beyond_the_grid_limits_are_refused_on_the_host(lib):
    """Token counts whose grids would exceed the 65535-block y extent come back
    as THETA_ERR_UNSUPPORTED before any CUDA call (no launch error later)."""
    raw = lib.lib
    p = ctypes.c_void_p(256)
    M = 65535 * 128 + 1  # one token past the T = X.V grid of the tensor-core path
    assert raw.theta_linear_forward(p, M, 64, p, 64, p, p, p, 8, 1, p, p, 1 << 40, None) == -2
    assert "tokens" in lib.theta_last_error()
    assert raw.theta_linear_gate_up_forward(p, M, 64, 64, 8, 1, p, p, p, p, p, p, p, p, p, p, 1 << 40,
                                            None) == -2
    M32 = 65535 * 64 + 1  # past the fp32 tile grid
    assert raw.theta_linear_forward(p, M32, 64, p, 64, p, None, None, 0, 0, p, None, 0, None) == -2
    assert raw.theta_reconstruct(p, p, None, None, M32, 64, 0, 0, p, None) == -2


def test_reconstruct_band_validation(lib):
    raw = lib.lib
    p = ctypes.c_void_p(16)
    arr = (ctypes.c_void_p * 2)(16, 16)
    bad = (ctypes.c_void_p * 2)(16, None)
    a = ctypes.cast(arr, ctypes.c_void_p)
    assert raw.theta_reconstruct_band(a, p, a, a, 0, 8, 8, 8, 1, a, None) == -1            # n = 0
    assert raw.theta_reconstruct_band(a, p, a, a, 300, 8, 8, 8, 1, a, None) == -1          # n > max
    assert raw.theta_reconstruct_band(None, p, a, a, 2, 8, 8, 8, 1, a, None) == -1         # NULL array
    assert raw.theta_reconstruct_band(a, p, ctypes.cast(bad, ctypes.c_void_p), a, 2, 8, 8, 8, 1, a, None) == -1
    assert raw.theta_reconstruct_band(a, p, a, a, 2, 8, 12, 8, 1, a, None) == -3           # I % 8
    assert raw.theta_reconstruct_band(a, p, a, a, 2, 8, 8, 8, 7, a, None) == -1            # dtype


def test_nvfp4_validation(lib):
    raw = lib.lib
    p = ctypes.c_void_p(16)
    assert raw.theta_nvfp4_quantize(p, 8, 48, p, p, p, p, 16, None) == -1        # I not a multiple of 32
    assert raw.theta_nvfp4_quantize(p, 8, 64, p, p, p, None, 0, None) == -6      # no workspace
    assert raw.theta_nvfp4_quantize(p, 8, 64, p, ctypes.c_void_p(17), p, p, 16, None) == -3  # odd scales
    assert raw.theta_linear_forward_nvfp4(p, 4, 64, p, p, p, 8, p, p, p, 8, p, p, 1 << 20, None) == -2  # M > 2
    assert raw.theta_linear_forward_nvfp4(p, 1, 64, p, p, p, 8, p, None, None, 8, p, p, 1 << 20, None) == -1
    assert raw.theta_linear_forward_nvfp4(p, 1, 64, p, p, p, 8, p, p, p, 8, p, None, 0, None) == -6
    assert lib.theta_workspace_size(lib.THETA_OP_NVFP4_QUANTIZE, 1, 8, 64, 0, lib.THETA_BF16) == 16


def test_grouped_forward_validation(lib):
    raw = lib.lib
    P = lib.theta_forward_problem
    p = 4096  # a 16-byte aligned fake device address: validation fails before any launch

    def table(*probs):
        arr = (P * len(probs))(*probs)
        return ctypes.cast(arr, ctypes.c_void_p), arr

    good = P(p, p, p, p, p, p, 64, 128, 16)
    h, keep = table(good, P(p, p, p, None, None, p, 8, 8, 0))
    d = ctypes.c_void_p(p)
    assert ctypes.sizeof(P) == 72
    assert raw.theta_linear_forward_grouped(None, d, 2, 1, d, 1 << 20, None) == -1          # no host table
    assert raw.theta_linear_forward_grouped(h, d, 0, 1, d, 1 << 20, None) == -1             # count 0
    assert raw.theta_linear_forward_grouped(h, d, 257, 1, d, 1 << 20, None) == -1           # count > max
    assert raw.theta_linear_forward_grouped(h, d, 2, 3, d, 1 << 20, None) == -2             # M > 2
    assert raw.theta_linear_forward_grouped(h, ctypes.c_void_p(p + 4), 2, 1, d, 1 << 20, None) == -3
    assert raw.theta_linear_forward_grouped(h, d, 2, 1, None, 0, None) == -6                # no workspace
    need = lib.theta_workspace_size(lib.THETA_OP_LINEAR_FORWARD_GROUPED, 1, 2, 0, 16, lib.THETA_BF16)
    assert need == 2 * 16 * 4 * 9
    assert raw.theta_linear_forward_grouped(h, d, 2, 1, d, need - 1, None) == -6
    h2, keep2 = table(good, P(p, p, p, p, p, p, 64, 128, 12))                               # rank % 8
    assert raw.theta_linear_forward_grouped(h2, d, 2, 1, d, 1 << 20, None) == -3
    h3, keep3 = table(good, P(p, p, p, None, p, p, 64, 128, 8))                             # rank > 0, no U
    assert raw.theta_linear_forward_grouped(h3, d, 2, 1, d, 1 << 20, None) == -1
    h4, keep4 = table(P(p + 2, p, p, p, p, p, 64, 128, 16))                                 # X misaligned
    assert raw.theta_linear_forward_grouped(h4, d, 1, 1, d, 1 << 20, None) == -3
    assert lib.theta_workspace_size(lib.THETA_OP_LINEAR_FORWARD_GROUPED, 2, 1, 0, 0, lib.THETA_BF16) == 0
    with pytest.raises(lib.ThetaError):
        lib.theta_workspace_size(lib.THETA_OP_LINEAR_FORWARD_GROUPED, 3, 1, 0, 0, lib.THETA_BF16)


def test_forward_problem_layout(lib):
    """The binding's struct matches theta_forward_problem field for field:
    six pointers, then O, I, rank as int64, 72 bytes in the header's order."""
    text = open(HEADER).read()
    body = re.search(r"typedef struct theta_forward_problem \{(.*?)\} theta_forward_problem;", text, re.S).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    fields = re.findall(r"\b(\w+);", body)
    P = lib.theta_forward_problem
    assert fields == [name for name, _ in P._fields_]
    assert [getattr(P, name).offset for name in fields] == [0, 8, 16, 24, 32, 40, 48, 56, 64]
    assert ctypes.sizeof(P) == 72 and ctypes.alignment(P) == 8


def test_residual_svd_validation(lib):
    raw = lib.lib
    p = ctypes.c_void_p(16)
    assert raw.theta_residual_svd(p, 64, 64, 0, 0, 8, 1, p, p, p, p, 1 << 30, None) == -1     # rank 0
    assert raw.theta_residual_svd(p, 64, 64, 0, 9, 8, 1, p, p, p, p, 1 << 30, None) == -1     # rank > samples
    assert raw.theta_residual_svd(p, 64, 64, 0, 4, 8, 9, p, p, p, p, 1 << 30, None) == -1     # power_iters > 8
    assert raw.theta_residual_svd(p, 200, 200, 0, 4, 97, 1, p, p, p, p, 1 << 30, None) == -2  # samples > 96
    assert raw.theta_residual_svd(p, 64, 20, 0, 4, 24, 1, p, p, p, p, 1 << 30, None) == -2    # samples > I
    assert raw.theta_residual_svd(p, 64, 64, 0, 4, 8, 1, p, p, p, None, 0, None) == -6        # no workspace
    big_rows = 65535 * 64 + 1  # past the products' grid limit: refused on the host
    assert raw.theta_residual_svd(p, big_rows, 64, 0, 4, 8, 1, p, p, p, p, 1 << 62, None) == -2
    assert raw.theta_residual_svd(p, 64, big_rows, 0, 4, 8, 1, p, p, p, p, 1 << 62, None) == -2
    small = lib.theta_workspace_size(lib.THETA_OP_RESIDUAL_SVD, 8, 64, 64, 4, lib.THETA_F32)
    big = lib.theta_workspace_size(lib.THETA_OP_RESIDUAL_SVD, 74, 21504, 5376, 64, lib.THETA_BF16)
    assert small >= 4 * (2 * 64 * 8 + 3 * 8 * 64) and big > small


def test_gate_up_workspace_covers_both_projections(lib):
    for M, r in [(1, 8), (16, 32), (300, 64)]:
        one = lib.theta_workspace_size(lib.THETA_OP_LINEAR_FORWARD, M, 64, 64, r, lib.THETA_BF16)
        both = lib.theta_workspace_size(lib.THETA_OP_GATE_UP_FORWARD, M, 64, 64, r, lib.THETA_BF16)
        assert both >= 4 * M * r * 2 and both % 256 == 0 and both >= 2 * min(one, 4 * M * r * 2)
    assert lib.theta_workspace_size(lib.THETA_OP_GATE_UP_FORWARD, 16, 64, 64, 0, lib.THETA_BF16) == 0


def test_workspace_sizes(lib):
    assert lib.theta_workspace_size(lib.THETA_OP_FROB_ERROR, 1, 1, 1, 0, lib.THETA_F32) >= 16
    assert lib.theta_workspace_size(lib.THETA_OP_LINEAR_FORWARD, 16, 256, 256, 0, lib.THETA_F32) == 0
    for dt in (lib.THETA_F32, lib.THETA_BF16):
        b = lib.theta_workspace_size(lib.THETA_OP_LINEAR_FORWARD, 300, 64, 64, 24, dt)
        assert b >= 300 * 24 * 4 and b % 256 == 0
    with pytest.raises(lib.ThetaError):
        lib.theta_workspace_size(99, 1, 1, 1, 0, lib.THETA_F32)


def test_launch_policy_round_trip(lib):
    assert lib.theta_get_policy() == lib.THETA_POLICY_LATENCY
    try:
        lib.theta_set_policy(lib.THETA_POLICY_THROUGHPUT)
        assert lib.theta_get_policy() == lib.THETA_POLICY_THROUGHPUT
        with pytest.raises(lib.ThetaError):
            lib.theta_set_policy(7)
        assert lib.theta_get_policy() == lib.THETA_POLICY_THROUGHPUT  # a rejected value changes nothing
    finally:
        lib.theta_set_policy(lib.THETA_POLICY_LATENCY)
    assert lib.theta_get_policy() == lib.THETA_POLICY_LATENCY
