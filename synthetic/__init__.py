"""Seeded synthetic inputs for the routed-MoE FFN layer.

This package is the one piece of code that the CUDA path and the CPU oracle
share: it draws the random tensors (activations, router weight, expert weights,
the optional per-expert logit bias and the FP8 encoding of the expert weights)
and nothing else. It holds none of the layer's arithmetic.
"""

from .moe_inputs import CONFIGS, LayerShape, make_layer, shape_of, tensor_shapes, zipf_logit_bias  # noqa: F401
