"""B200 (sm_100a) forward pass of one Flint mixture-of-experts layer.

The layer runs in the CUDA library libflint_moe.so behind the C ABI in include/flint_moe.h;
`binding` marshals arguments to it, `layer` keeps a layer's weights and workspace in PyTorch device
memory, `synthetic` draws the seeded workloads.
"""

__all__ = ["binding", "layer", "synthetic", "build"]
