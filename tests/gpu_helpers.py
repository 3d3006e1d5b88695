"""Helpers for the GPU parity tests: moving seeded inputs to the device and the
tolerance rules the parity bar is stated in.

Tolerances
  fp32 results:  max_i |g_i - o_i| / max(|o_i|, rms(o))  <= 1e-5
  bf16 results:  max_i |g_i - o_i| / rms(o)              <= 2e-2
  scalars:       |g - o| / |o|                           <= 1e-5
where o is the fp64 oracle on the same (rounded) inputs. The row scale s is
an fp32 output of fp32 arithmetic and is held to the fp32 rule whatever the
storage dtype of the weights.
"""
import numpy as np

TOL = {"f32": 1e-5, "bf16": 2e-2}


def torch_dtype(dt):
    import torch
    return {"f32": torch.float32, "bf16": torch.bfloat16}[dt]


def code(dt):
    return {"f32": 0, "bf16": 1}[dt]


def dev(a, dt="f32"):
    """float32 numpy array (values exact in dt) -> CUDA tensor of dt."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch_dtype(dt)).cuda()


def host(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def rms(a):
    a = np.asarray(a, dtype=np.float64)
    return float(np.sqrt(np.mean(a * a))) if a.size else 0.0


def err_f32(got, ref):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    if ref.size == 0:
        return 0.0
    den = np.maximum(np.abs(ref), rms(ref))
    den = np.where(den == 0, 1.0, den)
    return float(np.max(np.abs(got - ref) / den))


def err_bf16(got, ref):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    if ref.size == 0:
        return 0.0
    r = rms(ref)
    d = float(np.max(np.abs(got - ref)))
    return d / r if r > 0 else d


def assert_close(got, ref, dt, what=""):
    e = err_f32(got, ref) if dt == "f32" else err_bf16(got, ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    assert e <= TOL[dt], f"{what}: error {e:.3e} > {TOL[dt]:.0e} ({dt})"
    return e


def err_bf16_product(got, ref):
    """The bf16 bound for an output that is a product of two projections
    (the fused gate/up): the forward's 2e-2 of the RMS, plus half a bf16 unit
    in the last place of each element's own magnitude (2^-8 |ref|) for the
    one rounding of the result. A product is heavy-tailed -- its largest
    elements sit many RMS above zero -- so the rounding of those elements
    alone can reach 2e-2 of the RMS; this keeps that part relative to the
    element."""
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    if ref.size == 0:
        return 0.0
    r = rms(ref)
    d = float(np.max(np.maximum(np.abs(got - ref) - 2.0 ** -8 * np.abs(ref), 0.0)))
    return d / r if r > 0 else d


def assert_close_product(got, ref, what=""):
    e = err_bf16_product(got, ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    assert e <= TOL["bf16"], f"{what}: error {e:.3e} > {TOL['bf16']:.0e} (bf16 product)"
    return e


def assert_scalar_close(got, ref, tol=1e-5, what=""):
    if ref == 0.0 or np.isinf(ref):
        assert got == ref, f"{what}: {got} != {ref}"
        return 0.0
    e = abs(got - ref) / abs(ref)
    assert e <= tol, f"{what}: relative error {e:.3e} > {tol:.0e}"
    return e
