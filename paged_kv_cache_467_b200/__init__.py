"""Paged KV-cache decode attention for B200 (sm_100a).

The compute path is the C-ABI library ``libpkv.so`` built from ``csrc/``;
``ops`` marshals torch tensors into its calls.  Importing ``ops`` raises if the
library has not been built: there is no fallback path.
"""
from . import accounting, workloads  # noqa: F401

__all__ = ["accounting", "workloads"]
