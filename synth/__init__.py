"""Seeded synthetic inputs shared by the fp64 oracle, the tests and the bench.

This package holds workload shapes (``presets``) and seeded random tensors
(``rng``) only.  It contains none of the layer's arithmetic: no norms, no
positions, no masks, no attention.  Both the CPU oracle and the CUDA path take
their inputs from here, so that a parity test compares the two on identical
bits.
"""

from .presets import (  # noqa: F401
    ModelDims,
    VideoSpec,
    StreamSpec,
    LayoutSpec,
    Workload,
    PRESETS,
    preset,
)
from .rng import (  # noqa: F401
    bf16_round,
    bf16_to_f32,
    bf16_to_f64,
    normal_bf16,
    make_weights,
    make_stack_weights,
    stack_layer_seed,
    make_activations,
    make_action_weights,
    make_actions,
    WEIGHT_NAMES,
)
