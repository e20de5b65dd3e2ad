"""HCA (Heavily Compressed Attention) for B200 / sm_100a.

The product is ``libhca.so`` (C ABI in include/hca.h) built from ``csrc/``;
``binding`` marshals arguments to it, ``ops`` wraps the common calls around torch
tensors, and ``inputs`` draws the seeded synthetic workloads.
"""

__all__ = ["binding", "inputs", "ops"]
