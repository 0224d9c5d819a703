"""B200-native E(3)-equivariant message-passing convolution (libeqconv).

The compute lives in ``libeqconv.so`` (hand-written sm_100a CUDA behind the C
ABI of ``include/eqconv.h``); ``binding`` marshals arguments to it and
``conv`` wraps it for PyTorch users.  ``workloads`` draws seeded synthetic
inputs.  Importing this package does not load the library; the first call does,
and fails loudly when it is missing.
"""

__all__ = ["binding", "conv", "workloads"]
