"""CPU oracle for the theta-bundle path (test infrastructure, not the product).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU baseline leg
may import this package.
"""
from .theta_oracle import (  # noqa: F401
    round_to, band_sizes, band_index, band_mean, row_scale, residual,
    truncated_svd, reconstruct, frob_error, frob_partials, frob_from_partials, linear_forward, decompose_family, gelu_tanh, gate_up_forward,
    randomized_svd, _grid_round, e2m1_values, e4m3_values, nvfp4_quantize, nvfp4_dequantize, linear_forward_nvfp4,
)
