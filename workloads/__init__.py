"""Seeded synthetic workloads for the tensor-parallel reconciliation point.

This package holds the workload shapes and the seeded input generator. It
holds none of the reconciliation arithmetic: it only draws the bf16 inputs
(activations x, weights W in the ``torch.nn.Linear`` layout [H, K], and the
residual stream) that both the CPU oracle and the CUDA path consume.

The generator is counter based (Philox4x32-10, Salmon et al., "Parallel
random numbers: as easy as 1, 2, 3", SC'11), so any element range of any
tensor can be drawn on its own, on the CPU or on a CUDA device, with the same
bits on both.
"""

from .configs import CONFIGS, Config, Point, get_config
from .generator import (
    KIND_RESIDUAL,
    KIND_W,
    KIND_X,
    gaussian_bf16,
    gaussian_table,
    philox4x32_10,
    point_tensor,
    point_tensor_rows,
    tensor_id,
)

__all__ = [
    "CONFIGS",
    "Config",
    "Point",
    "get_config",
    "KIND_X",
    "KIND_W",
    "KIND_RESIDUAL",
    "gaussian_bf16",
    "gaussian_table",
    "philox4x32_10",
    "point_tensor",
    "point_tensor_rows",
    "tensor_id",
]
