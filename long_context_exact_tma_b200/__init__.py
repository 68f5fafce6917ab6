"""B200-native (sm_100a) per-rank hot path of USP (Ulysses + Ring) context-parallel attention.

The compute lives in libusp.so (CUDA kernels behind the C ABI of include/usp.h);
`binding` mirrors that ABI one function per entry point and `api` allocates
outputs and workspaces with torch.
"""
from . import binding  # noqa: F401

__all__ = ["binding", "api"]
