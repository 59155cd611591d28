"""Fine-grained sparse MoE feed-forward layer (Kolibri-1 shape) for NVIDIA B200.

The compute path is the CUDA library libkmoe.so (C ABI in include/kmoe.h);
`kmoe` is its thin ctypes binding and `inputs` the seeded input generator.
"""
from . import inputs  # noqa: F401
from .kmoe import (  # noqa: F401
    Experts, KmoeError, Layer, load, moe_combine, moe_forward, moe_grouped_ffn, moe_permute,
    moe_router_topk, moe_workspace_size, workspace,
)
