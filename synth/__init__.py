"""Seeded synthetic inputs shaped like GLM-5.2's routed-MoE layer.

Test and benchmark infrastructure shared by the CPU oracle and the GPU path.
It holds none of the layer's arithmetic: only counter-hash words mapped onto
bytes, integer codes, uniform scales and Box-Muller normals.
"""
from .synth import *  # noqa: F401,F403
