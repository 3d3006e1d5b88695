"""Python binding of libtheta (theta-bundle projections on B200, sm_100a).

Argument marshalling only: every function has the name of the C entry point
it calls (see include/theta.h), passes raw device pointers from torch tensors
and the current CUDA stream, and raises ThetaError on a non-zero status. All
arithmetic happens in the library's CUDA kernels; there is no fallback path,
and importing this module fails loudly if libtheta.so has not been built.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

__all__ = [
    "ThetaError", "THETA_F32", "THETA_BF16", "THETA_OP_FROB_ERROR", "THETA_OP_LINEAR_FORWARD",
    "THETA_OP_GATE_UP_FORWARD", "theta_linear_gate_up_forward", "THETA_OP_RESIDUAL_SVD", "theta_residual_svd",
    "THETA_OP_NVFP4_QUANTIZE", "THETA_OP_LINEAR_FORWARD_NVFP4", "theta_nvfp4_quantize", "theta_linear_forward_nvfp4",
    "THETA_MAX_LAYERS", "LIB_PATH", "lib", "THETA_OP_LINEAR_FORWARD_GROUPED", "THETA_MAX_GROUP",
    "theta_forward_problem", "ForwardGroup", "theta_linear_forward_grouped",
    "theta_version", "theta_status_string", "theta_last_error", "theta_band_index",
    "theta_band_mean", "theta_row_scale", "theta_residual", "theta_decompose_prelude",
    "theta_reconstruct", "theta_reconstruct_band", "theta_frob_error", "theta_frob_partials", "theta_linear_forward", "theta_workspace_size",
    "theta_device_status", "theta_linear_forward_noalloc", "theta_set_policy", "theta_get_policy",
    "theta_selftest_wait_timeout", "THETA_POLICY_LATENCY", "THETA_POLICY_THROUGHPUT",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtheta.so")

THETA_F32, THETA_BF16 = 0, 1
(THETA_OP_FROB_ERROR, THETA_OP_LINEAR_FORWARD, THETA_OP_GATE_UP_FORWARD, THETA_OP_RESIDUAL_SVD, THETA_OP_NVFP4_QUANTIZE,
 THETA_OP_LINEAR_FORWARD_NVFP4, THETA_OP_LINEAR_FORWARD_GROUPED) = 0, 1, 2, 3, 4, 5, 6
THETA_POLICY_LATENCY, THETA_POLICY_THROUGHPUT = 0, 1
THETA_MAX_LAYERS = 256
THETA_MAX_GROUP = 256

_i32p = ctypes.POINTER(ctypes.c_int32)
_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_int = ctypes.c_int
_sz = ctypes.c_size_t

_SIGNATURES = {
    "theta_version": (_int,),
    "theta_set_policy": (_int, _int),
    "theta_selftest_wait_timeout": (_int, ctypes.c_uint, _vp),
    "theta_get_policy": (_int,),
    "theta_status_string": (ctypes.c_char_p, _int),
    "theta_last_error": (ctypes.c_char_p,),
    "theta_band_index": (_int, _int, _int, _i32p, _i32p),
    "theta_band_mean": (_int, _vp, _int, _i64, _i64, _int, _vp, _vp),
    "theta_row_scale": (_int, _vp, _vp, _i64, _i64, _int, _vp, _vp),
    "theta_residual": (_int, _vp, _vp, _vp, _i64, _i64, _int, _vp, _vp),
    "theta_decompose_prelude": (_int, _vp, _int, _int, _i64, _i64, _int, _vp, _vp, _vp, _vp),
    "theta_reconstruct": (_int, _vp, _vp, _vp, _vp, _i64, _i64, _int, _int, _vp, _vp),
    "theta_frob_error": (_int, _vp, _vp, _i64, _int, _vp, _vp, _sz, _vp),
    "theta_frob_partials": (_int, _vp, _vp, _i64, _int, _vp, _vp, _sz, _vp),
    "theta_reconstruct_band": (_int, _vp, _vp, _vp, _vp, _int, _i64, _i64, _int, _int, _vp, _vp),
    "theta_linear_forward": (_int, _vp, _i64, _i64, _vp, _i64, _vp, _vp, _vp, _int, _int, _vp, _vp, _sz, _vp),
    "theta_linear_forward_noalloc": (_int, _vp, _i64, _i64, _vp, _i64, _vp, _vp, _vp, _int, _int, _vp, _vp),
    "theta_nvfp4_quantize": (_int, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _sz, _vp),
    "theta_linear_forward_nvfp4": (_int, _vp, _i64, _i64, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _int, _vp, _vp, _sz,
                                   _vp),
    "theta_residual_svd": (_int, _vp, _i64, _i64, _int, _int, _int, _int, _vp, _vp, _vp, _vp, _sz, _vp),
    "theta_linear_gate_up_forward": (_int, _vp, _i64, _i64, _i64, _int, _int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                     _vp, _vp, _sz, _vp),
    "theta_linear_forward_grouped": (_int, _vp, _vp, _int, _i64, _vp, _sz, _vp),
    "theta_workspace_size": (_int, _int, _i64, _i64, _i64, _int, _int, ctypes.POINTER(_sz)),
    "theta_device_status": (_int, _vp),
}

_LIB = None


def _load():
    """The loaded libtheta.so (loaded on first use; a missing build is an error)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m linear_theta_forward_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, *args) in _SIGNATURES.items():
            f = getattr(handle, name)
            f.restype = res
            f.argtypes = list(args)
        _LIB = handle
    return _LIB


def __getattr__(name):
    if name == "lib":
        return _load()
    raise AttributeError(name)


class ThetaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _load().theta_last_error().decode(errors="replace")
        name = _load().theta_status_string(status).decode()
        super().__init__(f"{where}: {name} ({status}): {msg}")


def _check(status: int, where: str) -> None:
    if status != 0:
        raise ThetaError(status, where)


def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float32:
        return THETA_F32
    if t.dtype == torch.bfloat16:
        return THETA_BF16
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _dtype_of(code_or_tensor) -> int:
    return code_or_tensor if isinstance(code_or_tensor, int) else _dtype_code(code_or_tensor)


def _ptr(t, name: str, *, optional: bool = False) -> int | None:
    if t is None:
        if optional:
            return None
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (row-major, no padding)")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is not None:
        return int(stream) if isinstance(stream, int) else stream.cuda_stream
    return _torch().cuda.current_stream().cuda_stream


def _ptr_array(tensors, name):
    arr = (_vp * len(tensors))()
    for i, t in enumerate(tensors):
        arr[i] = _ptr(t, f"{name}[{i}]")
    return arr


# ------------------------------------------------------------------ host-only
def theta_version() -> int:
    return _load().theta_version()


def theta_status_string(status: int) -> str:
    return _load().theta_status_string(status).decode()


def theta_last_error() -> str:
    return _load().theta_last_error().decode(errors="replace")


def theta_band_index(num_layers: int, G: int):
    """(band_of_layer int32[num_layers], band_start int32[G + 1])."""
    if num_layers < 1:
        _check(_load().theta_band_index(num_layers, G, None, None), "theta_band_index")
    bol = np.zeros(num_layers, dtype=np.int32)
    start = np.zeros(max(G, 0) + 1, dtype=np.int32)
    _check(_load().theta_band_index(num_layers, G, bol.ctypes.data_as(_i32p), start.ctypes.data_as(_i32p)),
           "theta_band_index")
    return bol, start


def theta_workspace_size(op: int, M: int, O: int, I: int, rank: int, dtype) -> int:
    out = _sz(0)
    _check(_load().theta_workspace_size(op, M, O, I, rank, _dtype_of(dtype), ctypes.byref(out)),
           "theta_workspace_size")
    return out.value


# ------------------------------------------------------------------ device
def theta_band_mean(weights, W0, stream=None) -> None:
    O, I = W0.shape
    arr = _ptr_array(weights, "weights")
    _check(_load().theta_band_mean(ctypes.cast(arr, _vp), len(weights), O, I, _dtype_code(W0),
                               _ptr(W0, "W0"), _stream(stream)), "theta_band_mean")


def theta_row_scale(weight, W0, s, stream=None) -> None:
    O, I = W0.shape
    _check(_load().theta_row_scale(_ptr(weight, "weight"), _ptr(W0, "W0"), O, I, _dtype_code(W0),
                               _ptr(s, "s"), _stream(stream)), "theta_row_scale")


def theta_residual(weight, W0, s, R, stream=None) -> None:
    O, I = W0.shape
    _check(_load().theta_residual(_ptr(weight, "weight"), _ptr(W0, "W0"), _ptr(s, "s"), O, I,
                              _dtype_code(W0), _ptr(R, "R"), _stream(stream)), "theta_residual")


def theta_decompose_prelude(weights, G: int, W0, s, residual=None, stream=None) -> None:
    """weights: L tensors [O, I]; W0: G tensors; s: L fp32 tensors [O];
    residual: L tensors or None."""
    O, I = weights[0].shape
    w = _ptr_array(weights, "weights")
    w0 = _ptr_array(W0, "W0")
    sp = _ptr_array(s, "s")
    rp = _ptr_array(residual, "residual") if residual is not None else None
    _check(_load().theta_decompose_prelude(ctypes.cast(w, _vp), len(weights), G, O, I,
                                       _dtype_code(weights[0]), ctypes.cast(w0, _vp),
                                       ctypes.cast(sp, _vp),
                                       ctypes.cast(rp, _vp) if rp is not None else None,
                                       _stream(stream)), "theta_decompose_prelude")


def theta_reconstruct(s, W0, U, V, W_out, stream=None) -> None:
    O, I = W0.shape
    rank = 0 if U is None else U.shape[1]
    _check(_load().theta_reconstruct(_ptr(s, "s"), _ptr(W0, "W0"), _ptr(U, "U", optional=True),
                                 _ptr(V, "V", optional=True), O, I, rank, _dtype_code(W0),
                                 _ptr(W_out, "W_out"), _stream(stream)), "theta_reconstruct")


def theta_reconstruct_band(s, W0, U, V, W_out, stream=None) -> None:
    """The reconstructions of the layers of one band: s, U, V, W_out are
    lists with one tensor per layer (U and V None for rank 0); W0 is shared."""
    O, I = W0.shape
    rank = 0 if U is None else U[0].shape[1]
    sp = _ptr_array(s, "s")
    op = _ptr_array(W_out, "W_out")
    up = _ptr_array(U, "U") if rank > 0 else None
    vp = _ptr_array(V, "V") if rank > 0 else None
    _check(_load().theta_reconstruct_band(ctypes.cast(sp, _vp), _ptr(W0, "W0"),
                                      ctypes.cast(up, _vp) if up is not None else None,
                                      ctypes.cast(vp, _vp) if vp is not None else None, len(s), O, I, rank,
                                      _dtype_code(W0), ctypes.cast(op, _vp), _stream(stream)),
           "theta_reconstruct_band")


def theta_frob_error(original, reconstructed, out, workspace, stream=None) -> None:
    """out: float64 CUDA tensor of one element; workspace: CUDA tensor of at
    least theta_workspace_size(THETA_OP_FROB_ERROR, ...) bytes."""
    _check(_load().theta_frob_error(_ptr(original, "original"), _ptr(reconstructed, "reconstructed"),
                                original.numel(), _dtype_code(original), _ptr(out, "out"),
                                _ptr(workspace, "workspace"),
                                workspace.numel() * workspace.element_size(), _stream(stream)),
           "theta_frob_error")


def theta_frob_partials(original, reconstructed, out, workspace, stream=None) -> None:
    """out: float64 CUDA tensor of two elements, receives (sum (A-B)^2,
    sum A^2); workspace as for theta_frob_error."""
    _check(_load().theta_frob_partials(_ptr(original, "original"), _ptr(reconstructed, "reconstructed"),
                                   original.numel(), _dtype_code(original), _ptr(out, "out"),
                                   _ptr(workspace, "workspace"),
                                   workspace.numel() * workspace.element_size(), _stream(stream)),
           "theta_frob_partials")


def theta_linear_forward(X, W0, s, U, V, Y, workspace=None, stream=None) -> None:
    """Y [M, O] = s * (X W0^T) + (X V) U^T. workspace: CUDA tensor of at least
    theta_workspace_size(THETA_OP_LINEAR_FORWARD, ...) bytes (None if 0)."""
    M, I = X.shape
    O = W0.shape[0]
    rank = 0 if U is None else U.shape[1]
    ws_ptr = _ptr(workspace, "workspace", optional=True)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_load().theta_linear_forward(_ptr(X, "X"), M, I, _ptr(W0, "W0"), O, _ptr(s, "s"),
                                    _ptr(U, "U", optional=True), _ptr(V, "V", optional=True), rank,
                                    _dtype_code(X), _ptr(Y, "Y"), ws_ptr, ws_bytes, _stream(stream)),
           "theta_linear_forward")


class theta_forward_problem(ctypes.Structure):
    """One problem of theta_linear_forward_grouped (the C struct, 72 bytes)."""
    _fields_ = [("X", _vp), ("W0", _vp), ("s", _vp), ("U", _vp), ("V", _vp), ("Y", _vp), ("O", _i64), ("I", _i64),
                ("rank", _i64)]


class ForwardGroup:
    """The problem table of a grouped forward: `problems` is a list of
    (X, W0, s, U, V, Y) tuples (U = V = None at rank 0) with one token count
    M. Holds the host array, its device copy and references to the tensors,
    so build it once and reuse it while the tensors stay where they are."""

    def __init__(self, problems):
        if not problems:
            raise ValueError("ForwardGroup: no problems")
        n = len(problems)
        self.count = n
        self.M = int(problems[0][0].shape[0])
        self.rmax = 0
        self.host = (theta_forward_problem * n)()
        for i, (X, W0, s, U, V, Y) in enumerate(problems):
            O, I = W0.shape
            rank = 0 if U is None else int(U.shape[1])
            self.rmax = max(self.rmax, rank)
            self.host[i] = theta_forward_problem(_ptr(X, "X"), _ptr(W0, "W0"), _ptr(s, "s"),
                                                 _ptr(U, "U", optional=True), _ptr(V, "V", optional=True),
                                                 _ptr(Y, "Y"), O, I, rank)
        raw = ctypes.string_at(ctypes.addressof(self.host), ctypes.sizeof(self.host))
        import torch
        self.device = torch.frombuffer(bytearray(raw), dtype=torch.uint8).to(problems[0][0].device)
        self._tensors = problems

    def workspace_size(self) -> int:
        return theta_workspace_size(THETA_OP_LINEAR_FORWARD_GROUPED, self.M, self.count, 0, self.rmax, THETA_BF16)


def theta_linear_forward_grouped(group: ForwardGroup, workspace=None, stream=None) -> None:
    """Every problem's Y [M, O] = s * (X W0^T) + (X V) U^T in one call.
    workspace: CUDA tensor of at least group.workspace_size() bytes (None if 0)."""
    ws_ptr = _ptr(workspace, "workspace", optional=True)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_load().theta_linear_forward_grouped(ctypes.cast(group.host, _vp), _ptr(group.device, "problems_device"),
                                                group.count, group.M, ws_ptr, ws_bytes, _stream(stream)),
           "theta_linear_forward_grouped")


def theta_linear_gate_up_forward(X, gate, up, Y, workspace=None, stream=None) -> None:
    """Y [M, O] = gelu_tanh(gate projection) * (up projection), each a theta
    forward on X; gate and up are (W0, s, U, V) tuples (U = V = None at rank
    0). workspace: CUDA tensor of at least theta_workspace_size(
    THETA_OP_GATE_UP_FORWARD, ...) bytes (None if 0)."""
    M, I = X.shape
    (W0g, sg, Ug, Vg), (W0u, su, Uu, Vu) = gate, up
    O = W0g.shape[0]
    rank = 0 if Ug is None else Ug.shape[1]
    ws_ptr = _ptr(workspace, "workspace", optional=True)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_load().theta_linear_gate_up_forward(
        _ptr(X, "X"), M, I, O, rank, _dtype_code(X), _ptr(W0g, "W0_gate"), _ptr(sg, "s_gate"),
        _ptr(Ug, "U_gate", optional=True), _ptr(Vg, "V_gate", optional=True), _ptr(W0u, "W0_up"), _ptr(su, "s_up"),
        _ptr(Uu, "U_up", optional=True), _ptr(Vu, "V_up", optional=True), _ptr(Y, "Y"), ws_ptr, ws_bytes,
        _stream(stream)), "theta_linear_gate_up_forward")


def theta_nvfp4_quantize(W0, codes, scales, g, workspace, stream=None) -> None:
    """Encode W0 [O, I] bf16 in NVFP4: codes uint8 [O, I/2], scales uint8
    [O, I/16] (E4M3), g fp32 device scalar [1]; workspace >= 16 bytes."""
    O, I = W0.shape
    _check(_load().theta_nvfp4_quantize(_ptr(W0, "W0"), O, I, _ptr(codes, "codes"), _ptr(scales, "scales"),
                                        _ptr(g, "g"), _ptr(workspace, "workspace"),
                                        workspace.numel() * workspace.element_size(), _stream(stream)),
           "theta_nvfp4_quantize")


def theta_linear_forward_nvfp4(X, codes, scales, g, s, U, V, Y, workspace=None, stream=None) -> None:
    """Y [M, O] = s * (X W0q^T) + (X V) U^T with W0q the NVFP4 block (M <= 2)."""
    M, I = X.shape
    O = codes.shape[0]
    rank = 0 if U is None else U.shape[1]
    ws_ptr = _ptr(workspace, "workspace", optional=True)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_load().theta_linear_forward_nvfp4(_ptr(X, "X"), M, I, _ptr(codes, "codes"), _ptr(scales, "scales"),
                                              _ptr(g, "g"), O, _ptr(s, "s"), _ptr(U, "U", optional=True),
                                              _ptr(V, "V", optional=True), rank, _ptr(Y, "Y"), ws_ptr, ws_bytes,
                                              _stream(stream)),
           "theta_linear_forward_nvfp4")


def theta_residual_svd(R, rank, omega, U, V, workspace, power_iters=2, stream=None) -> None:
    """U [O, rank], V [I, rank] with U·Vᵀ ≈ R by the randomized SVD; omega is
    the fp32 Gaussian test matrix [samples, I]; workspace: CUDA tensor of at
    least theta_workspace_size(THETA_OP_RESIDUAL_SVD, samples, O, I, rank) bytes."""
    O, I = R.shape
    samples = omega.shape[0]
    _check(_load().theta_residual_svd(_ptr(R, "R"), O, I, _dtype_code(R), int(rank), int(samples), int(power_iters),
                                      _ptr(omega, "omega"), _ptr(U, "U"), _ptr(V, "V"), _ptr(workspace, "workspace"),
                                      workspace.numel() * workspace.element_size(), _stream(stream)),
           "theta_residual_svd")


def theta_linear_forward_noalloc(X, W0, s, U, V, Y, stream=None) -> None:
    """theta_linear_forward without a workspace argument: the scratch is the
    library's built-in array (for callers that cannot allocate device memory;
    see include/theta.h for its capacity and sharing rules)."""
    M, I = X.shape
    O = W0.shape[0]
    rank = 0 if U is None else U.shape[1]
    _check(_load().theta_linear_forward_noalloc(_ptr(X, "X"), M, I, _ptr(W0, "W0"), O, _ptr(s, "s"),
                                            _ptr(U, "U", optional=True), _ptr(V, "V", optional=True), rank,
                                            _dtype_code(X), _ptr(Y, "Y"), _stream(stream)),
           "theta_linear_forward_noalloc")


def theta_set_policy(policy: int) -> None:
    """Grid sizing of the tensor-core forward kernels for the calls that
    follow: THETA_POLICY_LATENCY (split-K, default) or THETA_POLICY_THROUGHPUT
    (one CTA per output tile, for many concurrent calls)."""
    _check(_load().theta_set_policy(int(policy)), "theta_set_policy")


def theta_get_policy() -> int:
    return _load().theta_get_policy()


def theta_selftest_wait_timeout(limit_ms: int, stream=None) -> None:
    """Enqueues one bounded wait that nothing completes; the next
    theta_device_status() raises THETA_ERR_TIMEOUT."""
    _check(_load().theta_selftest_wait_timeout(int(limit_ms), _stream(stream)), "theta_selftest_wait_timeout")


def theta_device_status(stream=None) -> None:
    _check(_load().theta_device_status(_stream(stream)), "theta_device_status")
