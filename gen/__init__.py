"""Seeded synthetic inputs for the MoE routing / dispatch / combine path.

This module is shared by the oracle tests, the GPU parity tests and the
benchmark.  It holds no step of the method itself: only the random streams,
the workload shapes and the host-side redundant-expert placement that feeds
the skewed workload as an input.
"""

from .inputs import (  # noqa: F401
    CONFIGS,
    Workload,
    WorkloadConfig,
    device_normal_bf16,
    expert_permutation,
    normals,
    redundant_expert_map,
    splitmix64_stream,
    stream_key,
    uniforms,
)
