"""libgdattn: split-KV single-token decode attention for Gemma-4-style stacks on B200.

The compute lives in ``libgdattn.so`` (hand-written CUDA for sm_100a behind a C
ABI declared in ``include/gdattn.h``).  ``binding`` marshals arguments to it;
nothing here computes attention.  Importing the package does not load the
library; the first call does, and raises if it has not been built.
"""
from . import accounting, binding  # noqa: F401

__all__ = ["accounting", "binding"]
