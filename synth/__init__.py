"""Seeded synthetic inputs for the W4A4 + low-rank linear layer.

This package only draws random numbers and assembles input tensors. It holds
none of the layer's arithmetic (no rotation, no quantization, no GEMM), so both
the CPU oracle and the CUDA path can consume its output without sharing code.
"""
from .gen import LayerShape, CONFIGS, make_activations, make_weights, make_layer

__all__ = ["LayerShape", "CONFIGS", "make_activations", "make_weights", "make_layer"]
