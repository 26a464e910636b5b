"""Streaming edge-conditioned O(3) tensor-product convolution for B200 (sm_100a).

The compute path is the C-ABI library ``libtpconv.so`` built from ``csrc/``
(declared in ``include/tpconv.h``); ``binding`` marshals arguments to it with
ctypes.  ``workloads`` draws seeded synthetic graphs and features.
"""

__all__ = ["binding", "workloads"]
