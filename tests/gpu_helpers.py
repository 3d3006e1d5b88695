"""Helpers for the GPU parity tests: moving seeded inputs to the device and the
tolerance rules the parity bar is stated in.

Tolerances
  fp32 results:  max_i |g_i - o_i| / max(|o_i|, rms(o))  <= 1e-5
  bf16 results:  max_i |g_i - o_i| / rms(o)              <= 2e-2
  scalars:       |g - o| / |o|                           <= 1e-5
where o is the fp64 oracle on the same (rounded) inputs. The row scale s is
an fp32 output of fp32 arithmetic and is held to the fp32 rule whatever the
storage dtype of the weights.

One derived bound: a bf16 output that the GPU forms from an fp32
intermediate of its own (the residual w - s W0 from the fp32 row scale s)
can land one bf16 ulp away from the fp64 chain's, whenever the chain's exact
value lies between the rounding boundary and the GPU's (s agrees to ~1e-7
relative, which moves s W0 by far less than an ulp of R, but across a
boundary all the same). R's largest elements sit near 5 of its RMS, where one
ulp is 2.5% of the RMS, so against the whole chain the bound is
  max_i max(0, |g_i - o_i| - ulp(o_i)) / rms(o)  <= 2e-2      (assert_close_chain)
while the step itself, given the GPU's own W0 and s, is compared exactly.
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


def ulp_bf16(x):
    """Spacing of bf16 values at |x| (8 significant bits)."""
    a = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.exp2(e - 7), np.exp2(-133.0))


def err_bf16_chain(got, ref):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    if ref.size == 0:
        return 0.0
    r = rms(ref)
    d = float(np.max(np.maximum(np.abs(got - ref) - ulp_bf16(ref), 0.0)))
    return d / r if r > 0 else d


def assert_close_chain(got, ref, dt, what=""):
    """assert_close for a bf16 output formed from the GPU's own fp32
    intermediates, against the fp64 chain: one ulp of slack per element."""
    if dt == "f32":
        return assert_close(got, ref, dt, what)
    e = err_bf16_chain(got, ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    assert e <= TOL[dt], f"{what}: error {e:.3e} beyond one ulp > {TOL[dt]:.0e} (bf16 chain)"


def assert_residual_step(got, w, W0_gpu, s_gpu, dt, what=""):
    """The residual step against the oracle fed the GPU's own stored W0 and
    fp32 s. bf16: the GPU rounds w - s W0 to fp32 (one fused multiply-add)
    and then to bf16, the oracle rounds the exact value once; the two agree
    except where the fp32 value is exactly halfway between two bf16 values,
    so every element is within one ulp and nearly all are equal. fp32: the
    fp32 rule."""
    import oracle
    ref = oracle.residual(w, W0_gpu, s_gpu, dt)
    if dt == "bf16":
        g = np.asarray(got, np.float64)
        far = int(np.count_nonzero(np.abs(g - ref) > ulp_bf16(ref)))
        assert far == 0, f"{what}: {far} elements more than one ulp from the oracle's residual of the same W0 and s"
        diff = int(np.count_nonzero(g != ref))
        assert diff <= max(2, g.size // 1000), f"{what}: {diff} of {g.size} elements differ by an ulp"
    else:
        assert_close(got, ref, dt, what)


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
